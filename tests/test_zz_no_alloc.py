"""gdr_fwd_noalloc: the prefill for callers that cannot allocate device memory.

Some callers run under a memory manager that owns the whole device heap (no
further cudaMalloc allowed) or cannot afford the device synchronisation an
allocation may cause, and cannot hand over a workspace either.  For them the
library offers gdr_fwd_noalloc, which takes its scratch from a fixed array
built into the library.  This test calls it through the C-ABI, twice in a
row, and checks both results against the regular gdr_fwd entry point (which
gets a torch-allocated workspace) within the bf16 parity tolerance.  It lives
in its own file, collected last, and passes alone or after the other tests.
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


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_noalloc_matches_gdr_fwd_twice(cuda_device, gate):
    fn, scratch = _noalloc_fn()
    cfg = inputs.PREFILL["gdn_prefill"].replace(B=2, T=1000, H=4, gate=gate,
                                                gate_scale=0.1 if gate == "scalar" else 0.05)
    inp = inputs.prefill_inputs(cfg, seed=901)
    dev = cuda_device
    q, k, v = (to_dev(x, "bf16", dev) for x in (inp.q, inp.k, inp.v))
    g, b, S0 = (to_dev(x, "f32", dev) for x in (inp.g, inp.beta, inp.S0))
    need = binding.fwd_workspace_size(2, 1000, 4, 128, 128, 64, 2, False, binding.GDR_BF16,
                                      1 if gate == "channel" else 0, "tc")
    assert 0 < need <= scratch
    ref_o, ref_s = binding.gdr_fwd(q, k, v, g, b, S0, path="tc")
    torch.cuda.synchronize()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        out = torch.full_like(ref_o, float("nan"))
        SF = torch.full_like(ref_s, float("nan"))
        st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(S0), _ptr(out), _ptr(SF),
                2, 1000, 4, 128, 128, 64, None, 0, binding.GDR_BF16,
                1 if gate == "channel" else 0, stream)
        assert st == binding.GDR_OK, binding.status_string(st)
        assert binding.device_status() == binding.GDR_OK
        assert prefill_out_rel(to_np(out), to_np(ref_o)) <= TOL
        assert state_rel(to_np(SF), to_np(ref_s)) <= TOL


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
