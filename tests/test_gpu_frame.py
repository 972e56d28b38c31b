"""GPU parity of the implicit frame-level update ("video-delta-rule", section
"A Different Route") through gdr_fwd_frame against the fp64 oracle on the
same seeded, dtype-rounded inputs.  Tolerance: max relative Frobenius error per
(sequence, head) of O and S_final, <= 1e-4 with fp32 inputs and <= 1e-2 with
bf16 inputs."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_90_b200 import binding, inputs
from helpers import prefill_out_rel, state_rel, to_dev, to_np

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 1e-2}


def cfg_of(**kw):
    return inputs.FRAME["frame_prefill"].replace(**kw)


def run_gpu(inp, dev):
    c = inp.cfg
    q, k, v = (to_dev(x, c.dtype, dev) for x in (inp.q, inp.k, inp.v))
    g, gam = to_dev(inp.g, "f32", dev), to_dev(inp.gamma, "f32", dev)
    S0 = to_dev(inp.S0, "f32", dev)
    out, SF = binding.gdr_fwd_frame(q, k, v, g, gam, c.n, S0)
    torch.cuda.synchronize()
    assert binding.device_status() == binding.GDR_OK
    return to_np(out), to_np(SF)


def check(inp, dev):
    O, SF = run_gpu(inp, dev)
    Or, SFr = oracle.frame_fwd(inp.q, inp.k, inp.v, inp.g, inp.gamma, inp.cfg.n, inp.S0)
    eo, es = prefill_out_rel(O, Or), state_rel(SF, SFr)
    tol = TOL[inp.cfg.dtype]
    assert eo <= tol and es <= tol, (eo, es)


@pytest.mark.parametrize("n", [1, 16, 50])
@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_frame_fp32(cuda_device, n, gate):
    cfg = cfg_of(B=2, T=130, H=2, d_k=32, d_v=48, n=n, dtype="f32", gate=gate, s0_var=0.01)
    check(inputs.frame_inputs(cfg, seed=701), cuda_device)


@pytest.mark.parametrize("dk,dv", [(16, 8), (48, 40), (112, 128), (128, 128)])
def test_frame_fp32_key_widths(cuda_device, dk, dv):
    """Every register layout of the inverse pass (d_k / 4 columns per thread)
    that the shapes reach, on the fp32 path."""
    cfg = cfg_of(B=1, T=150, H=2, d_k=dk, d_v=dv, n=40, dtype="f32", gate="channel",
                 s0_var=0.01)
    check(inputs.frame_inputs(cfg, seed=704), cuda_device)


@pytest.mark.parametrize("scale", [20.0, 200.0])
def test_frame_fp32_strong_writes(cuda_device, scale):
    """Writing strengths scaled up so that I + G_t is far from the identity
    (eigenvalues in the hundreds to thousands): the inverse still meets the fp32
    tolerance."""
    cfg = cfg_of(B=1, T=256, H=2, d_k=64, d_v=64, n=64, dtype="f32", gate="scalar", s0_var=0.01)
    inp = inputs.frame_inputs(cfg, seed=705)
    inp.gamma = (inp.gamma * np.float32(scale)).astype(np.float32)
    check(inp, cuda_device)


@pytest.mark.parametrize("n", [64, 256])
def test_frame_bf16_d128(cuda_device, n):
    cfg = cfg_of(B=1, T=1000, H=3, n=n, s0_var=0.01)
    check(inputs.frame_inputs(cfg, seed=702), cuda_device)


@pytest.mark.parametrize("gate,s0_var", [("scalar", 0.01), ("channel", 0.0), ("scalar", 0.0)])
def test_frame_bf16_d128_gates_and_zero_state(cuda_device, gate, s0_var):
    """The tensor-core passes with one scalar decay per frame (broadcast over
    the key channels inside the chain) and with no initial state (S0 = 0);
    two sequences, a partial last frame."""
    cfg = cfg_of(B=2, T=700, H=2, n=128, gate=gate, s0_var=s0_var)
    inp = inputs.frame_inputs(cfg, seed=707)
    assert (inp.S0 is None) == (s0_var == 0.0)
    check(inp, cuda_device)


@pytest.mark.parametrize("T,n", [(100, 128), (256, 128), (129, 128)])
def test_frame_bf16_d128_few_frames(cuda_device, T, n):
    """The tensor-core chain's pipeline ends: one frame (the loop runs only its
    first step), exactly as many frames as it has stages, and a one-token last
    frame."""
    cfg = cfg_of(B=2, T=T, H=2, n=n, s0_var=0.01)
    check(inputs.frame_inputs(cfg, seed=708), cuda_device)


def test_frame_one_token_is_the_delta_rule_on_gpu(cuda_device):
    """n = 1 against gdr_fwd with beta = gamma / (1 + gamma) (Sherman-Morrison)."""
    cfg = cfg_of(B=1, T=96, H=2, d_k=64, d_v=64, n=1, dtype="f32", gate="channel", s0_var=0.01)
    inp = inputs.frame_inputs(cfg, seed=703)
    O, SF = run_gpu(inp, cuda_device)
    dev = cuda_device
    f = lambda x: to_dev(x, "f32", dev)
    beta = inp.gamma / (1 + inp.gamma)
    O2, S2 = binding.gdr_fwd(f(inp.q), f(inp.k), f(inp.v), f(inp.g), f(beta), f(inp.S0), chunk=32,
                             path="simt")
    assert prefill_out_rel(O, to_np(O2)) < 1e-4 and state_rel(SF, to_np(S2)) < 1e-4


def test_frame_permutation_invariance_on_gpu(cuda_device):
    cfg = cfg_of(B=1, T=128, H=2, d_k=64, d_v=64, n=32, dtype="f32", s0_var=0.01)
    inp = inputs.frame_inputs(cfg, seed=704)
    O, SF = run_gpu(inp, cuda_device)
    perm = np.concatenate([f * 32 + np.random.default_rng(f).permutation(32) for f in range(4)])
    for name in ("q", "k", "v", "gamma"):
        setattr(inp, name, np.ascontiguousarray(getattr(inp, name)[:, perm]))
    Op, SFp = run_gpu(inp, cuda_device)
    assert state_rel(SFp, SF) < 1e-5 and prefill_out_rel(Op, O[:, perm]) < 1e-5


def test_frame_zero_tokens_copies_state(cuda_device):
    inp = inputs.frame_inputs(cfg_of(B=2, T=0, H=2, d_k=32, d_v=32, n=8, dtype="f32", s0_var=0.01),
                              seed=705)
    O, SF = run_gpu(inp, cuda_device)
    assert O.size == 0 and np.array_equal(SF, inp.S0.astype(np.float64))


def test_frame_prefill_full_size_sampled(cuda_device):
    """The frame workload (B=1, H=16, 16 frames of 1024 tokens, d=128) in full;
    the oracle checks 2 heads."""
    inp = inputs.frame_inputs(inputs.FRAME["frame_prefill"])
    O, SF = run_gpu(inp, cuda_device)
    hs = [0, 13]
    sl = lambda x: np.ascontiguousarray(x[:, :, hs])
    Or, SFr = oracle.frame_fwd(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.g), sl(inp.gamma),
                               inp.cfg.n)
    assert np.isfinite(O).all() and np.isfinite(SF).all()
    eo, es = prefill_out_rel(O[:, :, hs], Or), state_rel(SF[:, hs], SFr)
    assert eo <= 1e-2 and es <= 1e-2, (eo, es)


def test_frame_tc_chain_keeps_fp32_accuracy(cuda_device):
    """The tensor-core chain multiplies in a three-term bf16 split.  With every
    writing strength a power of two, gamma * k is exact in bf16, so the
    tensor-core Gram pass matches the fp32 one up to summation order, and the
    gap between the two paths' S_final on the same (bf16-valued) inputs is the
    chain's own rounding: about 1e-5 for the split, about 1e-3 had the chain
    multiplied plain bf16 values."""
    dev = cuda_device
    cfg = cfg_of(B=1, T=4096, H=3, n=256, s0_var=0.01)
    inp = inputs.frame_inputs(cfg, seed=706)
    inp.gamma = np.exp2(np.round(np.log2(inp.gamma))).astype(np.float32)
    _, SF_tc = run_gpu(inp, dev)
    f = lambda x: to_dev(x, "f32", dev)
    _, SF32 = binding.gdr_fwd_frame(f(inp.q), f(inp.k), f(inp.v), f(inp.g), f(inp.gamma), cfg.n,
                                    f(inp.S0))  # fp32 inputs: the CUDA-core passes
    torch.cuda.synchronize()
    assert binding.device_status() == binding.GDR_OK
    gap = state_rel(SF_tc, to_np(SF32))
    assert gap <= 1e-4, gap
