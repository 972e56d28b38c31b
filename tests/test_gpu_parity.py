"""GPU parity: libgdr (through its C-ABI) against the fp64 CPU oracle on the
same seeded, dtype-rounded inputs.

Tolerance (the problem statement's): max relative Frobenius error over
(sequence, head) slices of O and of S_final, <= 1e-4 with fp32 inputs and
<= 1e-2 with bf16 inputs (fp32 state).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_90_b200 import binding, inputs
from helpers import max_rel_fro, prefill_out_rel, state_rel, to_dev, to_np

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 1e-2}


def small_cfg(**kw):
    base = inputs.PREFILL["gdn_prefill"]
    return base.replace(**kw)


def run_fwd(inp, dev, path="auto", chunk=None, S0=True):
    cfg = inp.cfg
    q, k, v = (to_dev(x, cfg.dtype, dev) for x in (inp.q, inp.k, inp.v))
    g, b = to_dev(inp.g, "f32", dev), to_dev(inp.beta, "f32", dev)
    S0d = to_dev(inp.S0, "f32", dev) if (S0 and inp.S0 is not None) else None
    cu = None if inp.cu_seqlens is None else torch.from_numpy(inp.cu_seqlens).to(dev)
    out, SF = binding.gdr_fwd(q, k, v, g, b, S0d, chunk=chunk or cfg.chunk, cu_seqlens=cu,
                              path=path)
    assert binding.device_status() == binding.GDR_OK
    return to_np(out), to_np(SF)


def run_oracle(inp, S0=True):
    return oracle.recurrence_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta,
                                 S0=inp.S0 if S0 else None, cu_seqlens=inp.cu_seqlens)


def check(inp, dev, path="auto", chunk=None, tol=None):
    tol = tol or TOL[inp.cfg.dtype]
    O, SF = run_fwd(inp, dev, path, chunk)
    Or, SFr = run_oracle(inp)
    eo, es = prefill_out_rel(O, Or, inp.cu_seqlens), state_rel(SF, SFr)
    assert eo <= tol and es <= tol, (eo, es)
    return eo, es


# ------------------------------------------------------------------ SIMT prefill
def test_tiny_fp32_workload(cuda_device):
    """The tiny fp32 workload, in full, at 1e-4."""
    check(inputs.prefill_inputs(inputs.PREFILL["tiny_fp32"]), cuda_device)


@pytest.mark.parametrize("chunk", [16, 32, 64, 128])
@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_simt_fp32_every_chunk_size(cuda_device, chunk, gate):
    cfg = small_cfg(B=2, T=203, H=2, d_k=64, d_v=48, dtype="f32", gate=gate, chunk=chunk,
                    gate_scale=0.1 if gate == "scalar" else 0.05, s0_var=0.01)
    check(inputs.prefill_inputs(cfg, seed=101), cuda_device, path="simt")


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_simt_bf16_d128(cuda_device, gate):
    cfg = small_cfg(B=2, T=300, H=3, gate=gate, gate_scale=0.1 if gate == "scalar" else 0.05)
    check(inputs.prefill_inputs(cfg, seed=102), cuda_device, path="simt")


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_simt_bf16_d128_chunk128(cuda_device, gate):
    """Chunk 128 at d = 128: the channel-blocked kernel (two full chunks and a
    44-token tail per sequence)."""
    cfg = small_cfg(B=2, T=300, H=3, gate=gate, gate_scale=0.1 if gate == "scalar" else 0.05,
                    chunk=128)
    check(inputs.prefill_inputs(cfg, seed=105), cuda_device)


def test_simt_chunk128_fp32_d128_strong_gates(cuda_device):
    """fp32 at d = 128, chunk 128, with decays strong enough that a whole chunk
    spans several orders of magnitude: the per-channel ratios stay formed from
    differences of cumulative sums."""
    cfg = small_cfg(B=1, T=257, H=2, dtype="f32", gate="channel", gate_scale=0.3, chunk=128)
    check(inputs.prefill_inputs(cfg, seed=106), cuda_device)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("chunk", [32, 128])
def test_simt_varlen_with_empty_and_unit_sequences(cuda_device, dtype, chunk):
    cfg = inputs.PREFILL["varlen_prefill"].replace(T=400, H=2, d_k=64, d_v=64, dtype=dtype,
                                                   n_seq=0, s0_var=0.01)
    inp = inputs.prefill_inputs(cfg, seed=103)
    inp.cu_seqlens = np.array([0, 0, 1, 65, 129, 200, 200, 400], dtype=np.int32)
    inp.S0 = np.random.default_rng(5).standard_normal((7, 2, 64, 64)).astype(np.float32) * 0.1
    check(inp, cuda_device, path="simt", chunk=chunk)


def test_simt_zero_length_batch_copies_state(cuda_device):
    cfg = small_cfg(B=2, T=0, H=2, d_k=64, d_v=64, dtype="f32", s0_var=0.01)
    inp = inputs.prefill_inputs(cfg, seed=104)
    O, SF = run_fwd(inp, cuda_device, path="simt")
    assert O.size == 0 and np.array_equal(SF, inp.S0.astype(np.float64))


def test_swap_reflection_on_gpu(cuda_device):
    """k = (e_i - e_j)/sqrt(2), beta = 2, alpha = 1, v = 0 permutes key columns
    ("A Swap Is a Reflection...", Technical Details); fp32, exact to a few ulp."""
    rng = np.random.default_rng(6)
    dk, dv, T = 64, 32, 40
    perm = np.arange(dk)
    k = np.zeros((1, T, 1, dk), np.float32)
    for t in range(T):
        i, j = rng.choice(dk, 2, replace=False)
        k[0, t, 0, i], k[0, t, 0, j] = 1 / math.sqrt(2), -1 / math.sqrt(2)
        perm[[i, j]] = perm[[j, i]]
    S0 = rng.standard_normal((1, 1, dv, dk)).astype(np.float32)
    dev = cuda_device
    T_ = lambda x: torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(dev)
    out, SF = binding.gdr_fwd(T_(np.zeros_like(k)), T_(k), T_(np.zeros((1, T, 1, dv))),
                              T_(np.zeros((1, T, 1))), T_(np.full((1, T, 1), 2.0)), T_(S0),
                              chunk=16, path="simt")
    assert np.max(np.abs(to_np(SF)[0, 0] - S0[0, 0][:, perm])) < 1e-5


def test_split_and_continue_on_gpu(cuda_device):
    """Affine lemma: [0, tau) then [tau, T) from S_tau equals [0, T)."""
    cfg = small_cfg(B=2, T=256, H=2, d_k=64, d_v=64, dtype="f32", gate="channel",
                    gate_scale=0.05, s0_var=0.01)
    inp = inputs.prefill_inputs(cfg, seed=107)
    dev = cuda_device
    q, k, v, g, b, S0 = (to_dev(x, "f32", dev) for x in (inp.q, inp.k, inp.v, inp.g, inp.beta,
                                                        inp.S0))
    O, SF = binding.gdr_fwd(q, k, v, g, b, S0, path="simt")
    tau = 100
    sl = lambda x, a, e: x[:, a:e].contiguous()
    O1, S1 = binding.gdr_fwd(sl(q, 0, tau), sl(k, 0, tau), sl(v, 0, tau), sl(g, 0, tau),
                             sl(b, 0, tau), S0, path="simt")
    O2, S2 = binding.gdr_fwd(sl(q, tau, 256), sl(k, tau, 256), sl(v, tau, 256), sl(g, tau, 256),
                             sl(b, tau, 256), S1, path="simt")
    assert max_rel_fro(to_np(torch.cat([O1, O2], 1)), to_np(O), (0, 2)) < 1e-5
    assert state_rel(to_np(S2), to_np(SF)) < 1e-5


def test_kda_broadcast_gate_equals_gdn_on_gpu(cuda_device):
    cfg = small_cfg(B=1, T=130, H=2, d_k=64, d_v=64, dtype="f32", s0_var=0.01)
    inp = inputs.prefill_inputs(cfg, seed=108)
    O1, S1 = run_fwd(inp, cuda_device, path="simt")
    inp.g = np.repeat(inp.g[..., None], 64, axis=-1).copy()
    O2, S2 = run_fwd(inp, cuda_device, path="simt")
    assert max_rel_fro(O2, O1, (0, 2)) < 1e-5 and state_rel(S2, S1) < 1e-5


def test_output_canary_untouched(cuda_device):
    """The kernels write exactly out[:B*T*H*d_v] and S_final[:N*H*d_v*d_k]."""
    cfg = small_cfg(B=1, T=77, H=2, d_k=64, d_v=64, dtype="bf16", s0_var=0.01)
    inp = inputs.prefill_inputs(cfg, seed=109)
    dev = cuda_device
    q, k, v = (to_dev(x, "bf16", dev) for x in (inp.q, inp.k, inp.v))
    g, b, S0 = (to_dev(x, "f32", dev) for x in (inp.g, inp.beta, inp.S0))
    n_out = 77 * 2 * 64
    obuf = torch.full((n_out + 4096,), 7.0, dtype=torch.bfloat16, device=dev)
    sbuf = torch.full((2 * 64 * 64 + 4096,), 7.0, dtype=torch.float32, device=dev)
    binding.gdr_fwd(q, k, v, g, b, S0, out=obuf[:n_out].view(1, 77, 2, 64),
                    S_final=sbuf[:2 * 64 * 64].view(1, 2, 64, 64), path="simt")
    torch.cuda.synchronize()
    assert bool((obuf[n_out:] == 7.0).all()) and bool((sbuf[2 * 64 * 64:] == 7.0).all())


# ------------------------------------------------------------------ decode
def decode_case(cfg, steps, seed, dev):
    S = inputs.decode_state(cfg, seed=seed)
    Sd = torch.from_numpy(S).to(dev)
    Sr = S.astype(np.float64)
    worst_o = 0.0
    for step in range(steps):
        tok = inputs.decode_token(cfg, step, seed=seed)
        out = binding.gdr_decode_step(*(to_dev(x, cfg.dtype, dev) for x in (tok.q, tok.k, tok.v)),
                                      to_dev(tok.g, "f32", dev), to_dev(tok.beta, "f32", dev), Sd)
        o_ref, Sr = oracle.recurrence_decode_step(tok.q, tok.k, tok.v, tok.g, tok.beta, Sr)
        worst_o = max(worst_o, max_rel_fro(to_np(out), o_ref, (0, 1)))
    assert binding.device_status() == binding.GDR_OK
    return worst_o, state_rel(to_np(Sd), Sr)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 32), (128, 256)])
def test_decode_small(cuda_device, dtype, gate, dk, dv):
    cfg = inputs.DECODE["decode"].replace(N=3, H=5, d_k=dk, d_v=dv, dtype=dtype, gate=gate)
    eo, es = decode_case(cfg, 6, 201, cuda_device)
    assert eo <= TOL[dtype] and es <= TOL[dtype], (eo, es)


@pytest.mark.parametrize("name", ["decode", "kda_decode"])
def test_decode_full_size_sampled(cuda_device, name):
    """The decode workloads at full size (256 x 32 heads, d = 128; scalar and
    per-key-channel decay) for 1000 steps; the oracle follows a fixed sample of
    8 sequences x 8 heads."""
    cfg = inputs.DECODE[name]
    dev = cuda_device
    S = inputs.decode_state(cfg)
    Sd = torch.from_numpy(S).to(dev)
    sn, sh = np.arange(0, 256, 32), np.arange(0, 32, 4)
    Sr = S[np.ix_(sn, sh)].astype(np.float64)
    worst = 0.0
    for step in range(cfg.steps):
        tok = inputs.decode_token(cfg, step)
        out = binding.gdr_decode_step(*(to_dev(x, "bf16", dev) for x in (tok.q, tok.k, tok.v)),
                                      to_dev(tok.g, "f32", dev), to_dev(tok.beta, "f32", dev), Sd)
        pick = lambda x: x[np.ix_(sn, sh)]
        o_ref, Sr = oracle.recurrence_decode_step(pick(tok.q), pick(tok.k), pick(tok.v),
                                                  pick(tok.g), pick(tok.beta), Sr)
        if step % 50 == 0 or step == cfg.steps - 1:
            worst = max(worst, max_rel_fro(to_np(out)[np.ix_(sn, sh)], o_ref, (0, 1)))
    assert binding.device_status() == binding.GDR_OK
    es = state_rel(to_np(Sd)[np.ix_(sn, sh)], Sr)
    assert worst <= 1e-2 and es <= 1e-2, (worst, es)


@pytest.mark.parametrize("name", ["decode", "kda_decode"])
def test_decode_full_size_every_head_first_steps(cuda_device, name):
    """The decode workloads at full size for their first 10 steps with the
    oracle following all 256 x 32 heads: every output of every step and the
    whole final state."""
    cfg = inputs.DECODE[name]
    dev = cuda_device
    S = inputs.decode_state(cfg)
    Sd = torch.from_numpy(S).to(dev)
    Sr = S.astype(np.float64)
    worst = 0.0
    for step in range(10):
        tok = inputs.decode_token(cfg, step)
        out = binding.gdr_decode_step(*(to_dev(x, "bf16", dev) for x in (tok.q, tok.k, tok.v)),
                                      to_dev(tok.g, "f32", dev), to_dev(tok.beta, "f32", dev), Sd)
        o_ref, Sr = oracle.recurrence_decode_step(tok.q, tok.k, tok.v, tok.g, tok.beta, Sr)
        worst = max(worst, max_rel_fro(to_np(out), o_ref, (0, 1)))
    assert binding.device_status() == binding.GDR_OK
    es = state_rel(to_np(Sd), Sr)
    assert worst <= 1e-2 and es <= 1e-2, (worst, es)


# ------------------------------------------------------------------ error path
def test_bounded_wait_reports_timeout_and_context_survives(cuda_device):
    assert binding.selftest_wait_timeout(4096) == binding.GDR_OK
    assert binding.device_status() == binding.GDR_ERR_TIMEOUT
    assert binding.device_status() == binding.GDR_OK  # cleared
    check(inputs.prefill_inputs(inputs.PREFILL["tiny_fp32"]), cuda_device)


# ------------------------------------------------------------------ tensor-core prefill
def sample_oracle(inp, heads, seqs=None):
    """Oracle on a sample of (sequence, head) units: all tokens of the chosen
    heads (and, for a regular batch, the chosen batch rows)."""
    cfg = inp.cfg
    hs = np.asarray(heads)
    if inp.cu_seqlens is None:
        bs = np.arange(cfg.B) if seqs is None else np.asarray(seqs)
        sl = lambda x: np.ascontiguousarray(x[bs][:, :, hs])
        S0 = None if inp.S0 is None else np.ascontiguousarray(inp.S0[bs][:, hs])
        O, SF = oracle.recurrence_fwd(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.g), sl(inp.beta),
                                      S0=S0)
        return O, SF, (bs, hs)
    sl = lambda x: np.ascontiguousarray(x[:, :, hs])
    S0 = None if inp.S0 is None else np.ascontiguousarray(inp.S0[:, hs])
    O, SF = oracle.recurrence_fwd(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.g), sl(inp.beta), S0=S0,
                                  cu_seqlens=inp.cu_seqlens)
    return O, SF, (None, hs)


def check_sampled(inp, dev, heads, seqs=None, path="tc", tol=1e-2):
    O, SF = run_fwd(inp, dev, path)
    Or, SFr, (bs, hs) = sample_oracle(inp, heads, seqs)
    if bs is None:
        Og, SFg = O[:, :, hs], SF[:, hs]
    else:
        Og, SFg = O[bs][:, :, hs], SF[bs][:, hs]
    eo, es = prefill_out_rel(Og, Or, inp.cu_seqlens), state_rel(SFg, SFr)
    assert np.isfinite(O).all() and np.isfinite(SF).all()
    assert eo <= tol and es <= tol, (eo, es)
    return eo, es


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("T", [64, 300, 1])
def test_tc_small_against_oracle(cuda_device, gate, T):
    cfg = small_cfg(B=2, T=T, H=3, gate=gate, gate_scale=0.1 if gate == "scalar" else 0.05)
    check(inputs.prefill_inputs(cfg, seed=301), cuda_device, path="tc")


@pytest.mark.parametrize("gate_scale", [1.5, 4.0])
def test_tc_strong_scalar_gates(cuda_device, gate_scale):
    """Scalar log-decays far larger than the workloads': with scale 1.5 the
    Gram weights come from the factorised exponentials with wide exponent
    ranges; with scale 4 the spread inside a chunk passes the factorisation's
    limit and the kernel takes the exp of every difference."""
    cfg = small_cfg(B=2, T=300, H=2, gate_scale=gate_scale)
    check(inputs.prefill_inputs(cfg, seed=305), cuda_device, path="tc")


def test_tc_varlen_with_empty_and_unit_sequences(cuda_device):
    cfg = inputs.PREFILL["varlen_prefill"].replace(T=600, H=2, n_seq=0, s0_var=0.01)
    inp = inputs.prefill_inputs(cfg, seed=302)
    inp.cu_seqlens = np.array([0, 0, 1, 65, 129, 200, 200, 600], dtype=np.int32)
    inp.S0 = np.random.default_rng(6).standard_normal((7, 2, 128, 128)).astype(np.float32) * 0.1
    check(inp, cuda_device, path="tc")


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_tc_matches_simt(cuda_device, gate):
    cfg = small_cfg(B=1, T=515, H=4, gate=gate, gate_scale=0.1 if gate == "scalar" else 0.05)
    inp = inputs.prefill_inputs(cfg, seed=303)
    O1, S1 = run_fwd(inp, cuda_device, path="tc")
    O2, S2 = run_fwd(inp, cuda_device, path="simt")
    assert prefill_out_rel(O1, O2) < 1e-2 and state_rel(S1, S2) < 1e-2


def test_tc_gdn_prefill_full_size_sampled(cuda_device):
    """Gated DeltaNet prefill workload at full size (B=4, H=16, T=4096) in the
    launch configuration the benchmark times; oracle on 3 heads x 4 sequences."""
    inp = inputs.prefill_inputs(inputs.PREFILL["gdn_prefill"])
    check_sampled(inp, cuda_device, heads=[0, 7, 15])


def test_tc_kda_prefill_full_size_sampled(cuda_device):
    """Per-channel-gate workload at full size (B=2, H=32, T=8192)."""
    inp = inputs.prefill_inputs(inputs.PREFILL["kda_prefill"])
    check_sampled(inp, cuda_device, heads=[0, 31])


def test_tc_kda_prefill_nonzero_state_sampled(cuda_device):
    cfg = inputs.PREFILL["kda_prefill"].replace(T=2048)
    inp = inputs.prefill_inputs(cfg, s0_var=0.01)
    check_sampled(inp, cuda_device, heads=[3, 17])


def test_tc_varlen_prefill_full_size_sampled(cuda_device):
    """Packed variable-length workload at full size (16 sequences, 65536 tokens)."""
    inp = inputs.prefill_inputs(inputs.PREFILL["varlen_prefill"])
    check_sampled(inp, cuda_device, heads=[5, 12])


def test_tc_varlen_nonzero_state_sampled(cuda_device):
    inp = inputs.prefill_inputs(inputs.PREFILL["varlen_prefill"], s0_var=0.01)
    check_sampled(inp, cuda_device, heads=[1])


# ------------------------------------------------------------------ tensor cores, 16-token chunks
@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("T", [16, 64, 300, 1])
def test_tc_chunk16_against_oracle(cuda_device, T, gate):
    """16-token chunks on the tensor cores: each 64-token tile is four chunks
    of the method, so sequences of 1, 16, 64 and 300 tokens cover a partial
    chunk, whole tiles and a partial tile."""
    cfg = small_cfg(B=2, T=T, H=3, chunk=16, gate=gate,
                    gate_scale=0.1 if gate == "scalar" else 0.05, s0_var=0.01)
    check(inputs.prefill_inputs(cfg, seed=311), cuda_device, path="tc", chunk=16)


@pytest.mark.parametrize("gate,gate_scale", [("scalar", 0.1), ("scalar", 4.0),
                                             ("channel", 0.05), ("channel", 12.0)])
def test_tc_chunk16_matches_simt(cuda_device, gate, gate_scale):
    """The same 16-token chunk algorithm on the tensor cores and on the CUDA
    cores; with the large scales the per-chunk spread passes the
    factorisation's limit and the chunks take the exact route."""
    cfg = small_cfg(B=1, T=515, H=4, chunk=16, gate=gate, gate_scale=gate_scale)
    inp = inputs.prefill_inputs(cfg, seed=312)
    O1, S1 = run_fwd(inp, cuda_device, path="tc", chunk=16)
    O2, S2 = run_fwd(inp, cuda_device, path="simt", chunk=16)
    assert prefill_out_rel(O1, O2) < 1e-2 and state_rel(S1, S2) < 1e-2
    check(inp, cuda_device, path="tc", chunk=16)


def test_tc_chunk16_varlen_with_empty_and_unit_sequences(cuda_device):
    cfg = inputs.PREFILL["varlen_prefill"].replace(T=600, H=2, n_seq=0, s0_var=0.01, chunk=16)
    inp = inputs.prefill_inputs(cfg, seed=313)
    inp.cu_seqlens = np.array([0, 0, 1, 17, 65, 200, 200, 600], dtype=np.int32)
    inp.S0 = np.random.default_rng(7).standard_normal((7, 2, 128, 128)).astype(np.float32) * 0.1
    check(inp, cuda_device, path="tc", chunk=16)


def test_tc_gdn_prefill_chunk16_full_size_sampled(cuda_device):
    """The Gated DeltaNet prefill workload at 16-token chunks, full size, as
    the benchmark's chunk-16 line runs it; oracle on 2 heads x 4 sequences."""
    inp = inputs.prefill_inputs(inputs.PREFILL["gdn_prefill_c16"])
    check_sampled(inp, cuda_device, heads=[2, 13])


def test_tc_kda_prefill_chunk16_full_size_sampled(cuda_device):
    """The per-channel-gate workload (B=2, H=32, T=8192) at 16-token chunks."""
    inp = inputs.prefill_inputs(inputs.PREFILL["kda_prefill"].replace(chunk=16))
    check_sampled(inp, cuda_device, heads=[4, 27])
