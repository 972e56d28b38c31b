"""GPU parity of Gated DeltaNet-2 ("Gated DeltaNet-2, and the gate that was
doing two jobs", section "What decoupling actually means here") through
gdr_fwd_gdn2 / gdr_decode_step_gdn2 against the fp64 oracle on the same seeded,
dtype-rounded inputs.  Tolerance as for the gated delta rule: max relative
Frobenius error per (sequence, head) of O and S_final, <= 1e-4 with fp32
inputs and <= 1e-2 with bf16 inputs."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_90_b200 import binding, inputs
from helpers import max_rel_fro, prefill_out_rel, state_rel, to_dev, to_np

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 1e-2}


def cfg_of(**kw):
    return inputs.PREFILL["gdn2_prefill"].replace(**kw)


def run_gpu(inp, dev, chunk=None, path="auto"):
    c = inp.cfg
    q, k, v = (to_dev(x, c.dtype, dev) for x in (inp.q, inp.k, inp.v))
    g, b, w = (to_dev(x, "f32", dev) for x in (inp.g, inp.b, inp.w))
    S0 = to_dev(inp.S0, "f32", dev)
    cu = None if inp.cu_seqlens is None else torch.from_numpy(inp.cu_seqlens).to(dev)
    out, SF = binding.gdr_fwd_gdn2(q, k, v, g, b, w, S0, chunk=chunk or c.chunk, cu_seqlens=cu,
                                   path=path)
    torch.cuda.synchronize()
    assert binding.device_status() == binding.GDR_OK
    return to_np(out), to_np(SF)


def check(inp, dev, chunk=None, path="auto"):
    O, SF = run_gpu(inp, dev, chunk, path)
    Or, SFr = oracle.gdn2_fwd(inp.q, inp.k, inp.v, inp.g, inp.b, inp.w, inp.S0, inp.cu_seqlens)
    eo, es = prefill_out_rel(O, Or, inp.cu_seqlens), state_rel(SF, SFr)
    tol = TOL[inp.cfg.dtype]
    assert eo <= tol and es <= tol, (eo, es)


@pytest.mark.parametrize("chunk", [16, 32, 64, 128])
@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_gdn2_fp32_every_chunk_size(cuda_device, chunk, gate):
    cfg = cfg_of(B=2, T=203, H=2, d_k=64, d_v=48, dtype="f32", gate=gate,
                 gate_scale=0.1 if gate == "scalar" else 0.05, s0_var=0.01)
    check(inputs.gdn2_inputs(cfg, seed=601), cuda_device, chunk)


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("chunk", [64, 128])
def test_gdn2_bf16_d128(cuda_device, gate, chunk):
    cfg = cfg_of(B=2, T=300, H=3, gate=gate, gate_scale=0.1 if gate == "scalar" else 0.05,
                 s0_var=0.01)
    check(inputs.gdn2_inputs(cfg, seed=602), cuda_device, chunk)


@pytest.mark.parametrize("gate", ["channel", "scalar"])
@pytest.mark.parametrize("T", [64, 300, 1])
def test_gdn2_tc_against_oracle(cuda_device, T, gate):
    """The tensor-core path (bf16, d = 128, C = 64), per-channel decay or a
    scalar one broadcast inside the WY kernel."""
    cfg = cfg_of(B=2, T=T, H=3, s0_var=0.01, gate=gate,
                 gate_scale=0.05 if gate == "channel" else 0.1)
    check(inputs.gdn2_inputs(cfg, seed=611), cuda_device, path="tc")


def test_gdn2_tc_scalar_decay_matches_broadcast_channel_decay(cuda_device):
    """A scalar decay on the tensor-core path equals the same decay given per
    channel (broadcast on the host): the kernel's in-tile broadcast is exact."""
    cfg = cfg_of(B=1, T=333, H=2, s0_var=0.01, gate="scalar", gate_scale=0.1)
    inp = inputs.gdn2_inputs(cfg, seed=615)
    O1, S1 = run_gpu(inp, cuda_device, path="tc")
    inp.g = np.ascontiguousarray(np.broadcast_to(inp.g[..., None], inp.g.shape + (128,)))
    O2, S2 = run_gpu(inp, cuda_device, path="tc")
    assert np.array_equal(O1, O2) and np.array_equal(S1, S2)


def test_gdn2_tc_varlen_with_empty_and_unit_sequences(cuda_device):
    cfg = cfg_of(B=1, T=600, H=2)
    inp = inputs.gdn2_inputs(cfg, seed=612)
    inp.cu_seqlens = np.array([0, 0, 1, 65, 129, 200, 200, 600], dtype=np.int32)
    inp.S0 = np.random.default_rng(9).standard_normal((7, 2, 128, 128)).astype(np.float32) * 0.1
    check(inp, cuda_device, path="tc")


def test_gdn2_tc_matches_simt(cuda_device):
    inp = inputs.gdn2_inputs(cfg_of(B=1, T=515, H=4, s0_var=0.01), seed=613)
    O1, S1 = run_gpu(inp, cuda_device, path="tc")
    O2, S2 = run_gpu(inp, cuda_device, path="simt")
    assert prefill_out_rel(O1, O2) < 1e-2 and state_rel(S1, S2) < 1e-2


def test_gdn2_tc_with_equal_gates_is_kda(cuda_device):
    """b = w = beta on the tensor-core path against gdr_fwd's per-channel
    (KDA) tensor-core path: the same maths through different roundings."""
    cfg = inputs.PREFILL["kda_prefill"].replace(B=1, T=400, H=2, s0_var=0.01)
    inp = inputs.prefill_inputs(cfg, seed=614)
    dev = cuda_device
    q, k, v = (to_dev(x, "bf16", dev) for x in (inp.q, inp.k, inp.v))
    g, beta, S0 = (to_dev(x, "f32", dev) for x in (inp.g, inp.beta, inp.S0))
    b = beta[..., None].expand(*beta.shape, 128).contiguous()
    O1, S1 = binding.gdr_fwd_gdn2(q, k, v, g, b, b, S0, path="tc")
    O2, S2 = binding.gdr_fwd(q, k, v, g, beta, S0, path="tc")
    assert prefill_out_rel(to_np(O1), to_np(O2)) < 1e-2 and state_rel(to_np(S1), to_np(S2)) < 1e-2


def test_gdn2_varlen_with_empty_and_unit_sequences(cuda_device):
    cfg = cfg_of(B=1, T=400, H=2, d_k=64, d_v=64, dtype="f32")
    inp = inputs.gdn2_inputs(cfg, seed=603)
    inp.cu_seqlens = np.array([0, 0, 1, 65, 129, 200, 200, 400], dtype=np.int32)
    inp.S0 = np.random.default_rng(8).standard_normal((7, 2, 64, 64)).astype(np.float32) * 0.1
    check(inp, cuda_device, chunk=32)


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_gdn2_with_equal_gates_is_the_gated_delta_rule(cuda_device, gate):
    """b = w = beta (broadcast) on the GPU equals gdr_fwd on the same path."""
    cfg = inputs.PREFILL["gdn_prefill"].replace(B=2, T=150, H=2, d_k=64, d_v=64, dtype="f32",
                                                gate=gate, s0_var=0.01)
    inp = inputs.prefill_inputs(cfg, seed=604)
    dev = cuda_device
    q, k, v, g, beta, S0 = (to_dev(x, "f32", dev) for x in (inp.q, inp.k, inp.v, inp.g,
                                                            inp.beta, inp.S0))
    b = beta[..., None].expand(*beta.shape, 64).contiguous()
    w = beta[..., None].expand(*beta.shape, 64).contiguous()
    O1, S1 = binding.gdr_fwd_gdn2(q, k, v, g, b, w, S0, chunk=32)
    O2, S2 = binding.gdr_fwd(q, k, v, g, beta, S0, chunk=32, path="simt")
    assert prefill_out_rel(to_np(O1), to_np(O2)) < 1e-5 and state_rel(to_np(S1), to_np(S2)) < 1e-5


def test_gdn2_zero_tokens_copies_state(cuda_device):
    inp = inputs.gdn2_inputs(cfg_of(B=2, T=0, H=2, d_k=64, d_v=64, dtype="f32", s0_var=0.01),
                             seed=605)
    O, SF = run_gpu(inp, cuda_device)
    assert O.size == 0 and np.array_equal(SF, inp.S0.astype(np.float64))


@pytest.mark.parametrize("dtype,dk,gate", [("bf16", 128, "channel"), ("f32", 64, "scalar"),
                                           ("bf16", 64, "channel")])
def test_gdn2_decode_steps(cuda_device, dtype, dk, gate):
    """20 decode steps in place against the oracle run one token at a time."""
    rng = np.random.default_rng(606)
    N, H, dv = 6, 4, dk
    S = (rng.standard_normal((N, H, dv, dk)) * 0.3).astype(np.float32)
    Sd = torch.from_numpy(S.copy()).to(cuda_device)
    Sr = S.astype(np.float64)
    for step in range(20):
        cfg = cfg_of(B=N, T=1, H=H, d_k=dk, d_v=dv, dtype=dtype, gate=gate)
        tok = inputs.gdn2_inputs(cfg, seed=1000 + step)
        sq = lambda x: np.ascontiguousarray(x[:, 0])
        q, k, v, g, b, w = (sq(x) for x in (tok.q, tok.k, tok.v, tok.g, tok.b, tok.w))
        out = binding.gdr_decode_step_gdn2(to_dev(q, dtype, cuda_device), to_dev(k, dtype, cuda_device),
                                           to_dev(v, dtype, cuda_device), to_dev(g, "f32", cuda_device),
                                           to_dev(b, "f32", cuda_device), to_dev(w, "f32", cuda_device), Sd)
        Or, SFr = oracle.gdn2_fwd(tok.q, tok.k, tok.v, tok.g, tok.b, tok.w, Sr)
        Sr = SFr
        assert max_rel_fro(to_np(out), Or[:, 0], lead=(0, 1)) <= TOL[dtype]
    assert state_rel(to_np(Sd), Sr) <= 1e-4


def test_gdn2_prefill_full_size_sampled(cuda_device):
    """The Gated DeltaNet-2 workload (B=2, H=16, T=4096, per-channel decay) in
    full on the GPU; the oracle checks 2 heads of both sequences."""
    inp = inputs.gdn2_inputs(inputs.PREFILL["gdn2_prefill"])
    O, SF = run_gpu(inp, cuda_device)
    hs = [0, 9]
    sl = lambda x: np.ascontiguousarray(x[:, :, hs])
    Or, SFr = oracle.gdn2_fwd(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.g), sl(inp.b), sl(inp.w))
    assert np.isfinite(O).all() and np.isfinite(SF).all()
    eo, es = prefill_out_rel(O[:, :, hs], Or), state_rel(SF[:, hs], SFr)
    assert eo <= 1e-2 and es <= 1e-2, (eo, es)


@pytest.mark.parametrize("gate", ["channel", "scalar"])
@pytest.mark.parametrize("T", [64, 300])
def test_gdn2_tc_chunk16_against_oracle(cuda_device, T, gate):
    """Gated DeltaNet-2 with 16-token chunks on the tensor cores."""
    cfg = cfg_of(B=2, T=T, H=3, s0_var=0.01, gate=gate, chunk=16,
                 gate_scale=0.05 if gate == "channel" else 0.1)
    check(inputs.gdn2_inputs(cfg, seed=612), cuda_device, chunk=16, path="tc")
