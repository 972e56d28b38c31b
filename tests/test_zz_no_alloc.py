"""gdr_fwd_noalloc: the prefill for callers that cannot allocate device memory.

Some callers run under a memory manager that owns the whole device heap (no
further cudaMalloc allowed) or cannot afford the device synchronisation an
allocation may cause, and cannot hand over a workspace either.  For them the
library offers gdr_fwd_noalloc, which takes its scratch from a fixed array
built into the library.  These tests call it through the C-ABI, twice in a
row, and check its results against the regular gdr_fwd entry point on the
tensor-core path (which gets a torch-allocated workspace).  Both run the same
deterministic kernels on the same inputs, so the results must be equal bit
for bit -- a looser tolerance would hide a scratch-offset mistake -- and
they also meet the bf16 parity tolerance against each other trivially.  Cases:
a regular batch for either gate, a packed batch with empty and one-token
sequences, and a batch of zero tokens (S_final = S0).  The file is collected
last and passes alone or after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

from gated_delta_rule_90_b200 import binding, inputs
from helpers import prefill_out_rel, state_rel, to_dev, to_np

pytestmark = pytest.mark.gpu
TOL = 1e-2


def _noalloc_fn():
    L = binding.lib()
    fn = L.gdr_fwd_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.restype = i
    fn.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, i, i, i, vp]
    L.gdr_fwd_noalloc_scratch_bytes.restype = ctypes.c_size_t
    return fn, int(L.gdr_fwd_noalloc_scratch_bytes())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call(fn, q, k, v, g, b, S0, out, SF, B, T, H, cu, n_seq, gate):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(S0), _ptr(out), _ptr(SF), B, T, H,
              128, 128, 64, _ptr(cu), n_seq, binding.GDR_BF16, 1 if gate == "channel" else 0,
              stream)


def _upload(inp, dev):
    q, k, v = (to_dev(x, "bf16", dev) for x in (inp.q, inp.k, inp.v))
    g, b, S0 = (to_dev(x, "f32", dev) for x in (inp.g, inp.beta, inp.S0))
    return q, k, v, g, b, S0


def _twice_equal(fn, scratch, args, ref_o, ref_s, B, T, H, cu, n_seq, gate):
    q, k, v, g, b, S0 = args
    need = binding.fwd_workspace_size(B, T, H, 128, 128, 64, n_seq, cu is not None,
                                      binding.GDR_BF16, 1 if gate == "channel" else 0, "tc")
    assert 0 < need <= scratch
    for _ in range(2):
        out = torch.full_like(ref_o, float("nan"))
        SF = torch.full_like(ref_s, float("nan"))
        st = _call(fn, q, k, v, g, b, S0, out, SF, B, T, H, cu, n_seq, gate)
        assert st == binding.GDR_OK, binding.status_string(st)
        torch.cuda.synchronize()
        assert binding.device_status() == binding.GDR_OK
        assert torch.equal(out, ref_o) and torch.equal(SF, ref_s)
        assert prefill_out_rel(to_np(out), to_np(ref_o)) <= TOL
        assert state_rel(to_np(SF), to_np(ref_s)) <= TOL


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_noalloc_matches_gdr_fwd_twice(cuda_device, gate):
    fn, scratch = _noalloc_fn()
    cfg = inputs.PREFILL["gdn_prefill"].replace(B=2, T=1000, H=4, gate=gate,
                                                gate_scale=0.1 if gate == "scalar" else 0.05)
    inp = inputs.prefill_inputs(cfg, seed=901)
    args = _upload(inp, cuda_device)
    ref_o, ref_s = binding.gdr_fwd(*args, path="tc")
    torch.cuda.synchronize()
    _twice_equal(fn, scratch, args, ref_o, ref_s, 2, 1000, 4, None, 0, gate)


def test_noalloc_packed_sequences_match_gdr_fwd(cuda_device):
    """Packed batch with an empty, a one-token and a chunk-straddling sequence."""
    fn, scratch = _noalloc_fn()
    cfg = inputs.PREFILL["varlen_prefill"].replace(T=700, H=3, n_seq=0)
    inp = inputs.prefill_inputs(cfg, seed=902)
    cu_np = np.array([0, 0, 1, 65, 300, 700], dtype=np.int32)
    inp.S0 = np.random.default_rng(9).standard_normal((5, 3, 128, 128)).astype(np.float32) * 0.1
    args = _upload(inp, cuda_device)
    cu = torch.from_numpy(cu_np).to(cuda_device)
    ref_o, ref_s = binding.gdr_fwd(*args, cu_seqlens=cu, path="tc")
    torch.cuda.synchronize()
    _twice_equal(fn, scratch, args, ref_o, ref_s, 1, 700, 3, cu, 5, "scalar")


def test_noalloc_zero_tokens_copies_the_state(cuda_device):
    fn, _ = _noalloc_fn()
    S0 = torch.randn((2, 3, 128, 128), dtype=torch.float32, device=cuda_device)
    for _ in range(2):
        SF = torch.full_like(S0, float("nan"))
        st = fn(None, None, None, None, None, _ptr(S0), None, _ptr(SF), 2, 0, 3, 128, 128, 64,
                None, 0, binding.GDR_BF16, 0,
                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == binding.GDR_OK, binding.status_string(st)
        torch.cuda.synchronize()
        assert binding.device_status() == binding.GDR_OK
        assert torch.equal(SF, S0)


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_device):
    fn, scratch = _noalloc_fn()
    # the full Gated DeltaNet prefill needs far more scratch than the fixed array
    assert binding.fwd_workspace_size(4, 4096, 16, 128, 128, 64, 4, False, binding.GDR_BF16, 0,
                                      "tc") > scratch
    q = torch.zeros((4, 4096, 16, 128), dtype=torch.bfloat16, device=cuda_device)
    g = torch.zeros((4, 4096, 16), dtype=torch.float32, device=cuda_device)
    st = fn(_ptr(q), _ptr(q), _ptr(q), _ptr(g), _ptr(g), None, _ptr(q), None, 4, 4096, 16, 128,
            128, 64, None, 0, binding.GDR_BF16, 0, None)
    assert st == binding.GDR_ERR_UNSUPPORTED
