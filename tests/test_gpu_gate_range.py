"""GPU parity of the tensor-core prefill under strong decays: chunks whose
cumulative log-decay spans more than the factorised Gram weights allow.

Inside a chunk the kernels take e^(G_l - G_m) as e^(G_l - G_r) e^(G_r - G_m)
around row r = 31; once max_l |G_l - G_r| reaches the range limit (60 by
default) a chunk exponentiates every difference instead ("Linear Attention,
Visualized", sections "Kimi Delta Attention (KDA) / Complete per-chunk
algorithm" and "Gated DeltaNet (GDN) / Complete per-chunk algorithm": the
decay products there are defined for any decay in (0, 1]).  These tests drive
per-key-channel decays far past that limit (gate scale 3 and 6: a typical
token decays by e^-2.4 and e^-4.8 per channel, so a 64-token chunk spans
about 150 and 300), mix fast and slow channels in one head, and run the
Kimi Delta Attention, Gated DeltaNet-2 and Gated DeltaProduct entry points
against their fp64 oracles at the bf16 tolerance (1e-2, max relative
Frobenius error per (sequence, head) of O and S_final).  A last pair of tests
forces every chunk onto the exact route on ordinary decays and checks it
against the factorised route and the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_90_b200 import binding, inputs
from helpers import prefill_out_rel, state_rel, to_dev, to_np

pytestmark = pytest.mark.gpu
TOL = 1e-2
DEFAULT_LIMIT = 60.0


@pytest.fixture
def spread_limit():
    """Set the Gram range limit for one test; the default is restored after."""
    prev = binding.set_gram_spread_limit(DEFAULT_LIMIT)
    assert prev == DEFAULT_LIMIT
    yield binding.set_gram_spread_limit
    binding.set_gram_spread_limit(DEFAULT_LIMIT)


def max_chunk_spread(g, chunk=64, cu=None):
    """Largest |G_l - G_31| over chunks and channels (G = in-chunk cumsum of g),
    with the chunks starting at every sequence start as the kernels cut them."""
    g = np.asarray(g, np.float64)
    if g.ndim == 3:
        g = g[..., None]
    starts = [(b, 0, g.shape[1]) for b in range(g.shape[0])] if cu is None else \
        [(0, int(cu[s]), int(cu[s + 1])) for s in range(len(cu) - 1)]
    worst = 0.0
    for b, t0, t1 in starts:
        for c0 in range(t0, t1, chunk):
            G = np.cumsum(g[b, c0:min(c0 + chunk, t1)], axis=0)
            if G.shape[0] > 31:
                worst = max(worst, float(np.max(np.abs(G - G[31]))))
    return worst


def strong_channel_gate(inp, scale, mixed):
    """Per-channel log-decays -softplus(N(0,1)) * scale drawn from the input
    recipe's own gate noise (its gate_scale divided out); with ``mixed`` only
    the upper half of the key channels is strong, the lower half keeps the
    recipe's scale."""
    base = inp.g / np.float32(inp.cfg.gate_scale)
    g = (base * np.float32(scale)).astype(np.float32)
    if mixed:
        g[..., : g.shape[-1] // 2] = inp.g[..., : g.shape[-1] // 2]
    return np.ascontiguousarray(g)


def run_kda(inp, dev):
    q, k, v = (to_dev(x, "bf16", dev) for x in (inp.q, inp.k, inp.v))
    g, b = to_dev(inp.g, "f32", dev), to_dev(inp.beta, "f32", dev)
    S0 = to_dev(inp.S0, "f32", dev)
    cu = None if inp.cu_seqlens is None else torch.from_numpy(inp.cu_seqlens).to(dev)
    out, SF = binding.gdr_fwd(q, k, v, g, b, S0, cu_seqlens=cu, path="tc")
    torch.cuda.synchronize()
    assert binding.device_status() == binding.GDR_OK
    return to_np(out), to_np(SF)


def check_kda(inp, dev):
    O, SF = run_kda(inp, dev)
    Or, SFr = oracle.recurrence_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, S0=inp.S0,
                                    cu_seqlens=inp.cu_seqlens)
    assert np.isfinite(O).all() and np.isfinite(SF).all()
    eo, es = prefill_out_rel(O, Or, inp.cu_seqlens), state_rel(SF, SFr)
    assert eo <= TOL and es <= TOL, (eo, es)
    return O, SF


@pytest.mark.parametrize("scale", [3.0, 6.0])
@pytest.mark.parametrize("mixed", [False, True])
def test_kda_tc_strong_channel_decay(cuda_device, spread_limit, scale, mixed):
    cfg = inputs.PREFILL["kda_prefill"].replace(B=2, T=300, H=3)
    inp = inputs.prefill_inputs(cfg, seed=701, s0_var=0.01)
    inp.g = strong_channel_gate(inp, scale, mixed)
    assert max_chunk_spread(inp.g) > 88.0  # past where e^x leaves the fp32 range
    check_kda(inp, cuda_device)


def test_kda_tc_strong_decay_varlen(cuda_device, spread_limit):
    """Packed sequences with a partial first chunk after each boundary."""
    cfg = inputs.PREFILL["kda_prefill"].replace(B=1, T=500, H=2)
    inp = inputs.prefill_inputs(cfg, seed=702, s0_var=0.01)
    inp.cu_seqlens = np.array([0, 37, 37, 200, 500], dtype=np.int32)
    inp.S0 = np.random.default_rng(8).standard_normal((4, 2, 128, 128)).astype(np.float32) * 0.1
    inp.g = strong_channel_gate(inp, 6.0, True)
    assert max_chunk_spread(inp.g, cu=inp.cu_seqlens) > 88.0
    check_kda(inp, cuda_device)


@pytest.mark.parametrize("gate", ["channel", "scalar"])
def test_gdn2_tc_strong_decay(cuda_device, spread_limit, gate):
    """Gated DeltaNet-2 with strong decays (per channel, or one scalar per
    token broadcast over the key channels inside the WY kernel)."""
    cfg = inputs.PREFILL["gdn2_prefill"].replace(B=2, T=300, H=3, gate=gate, s0_var=0.01,
                                                 gate_scale=0.05 if gate == "channel" else 0.1)
    inp = inputs.gdn2_inputs(cfg, seed=703)
    inp.g = strong_channel_gate(inp, 5.0, gate == "channel")
    assert max_chunk_spread(inp.g) > 88.0
    dev = cuda_device
    q, k, v = (to_dev(x, "bf16", dev) for x in (inp.q, inp.k, inp.v))
    g, b, w = (to_dev(x, "f32", dev) for x in (inp.g, inp.b, inp.w))
    out, SF = binding.gdr_fwd_gdn2(q, k, v, g, b, w, to_dev(inp.S0, "f32", dev), path="tc")
    torch.cuda.synchronize()
    assert binding.device_status() == binding.GDR_OK
    O, SF = to_np(out), to_np(SF)
    Or, SFr = oracle.gdn2_fwd(inp.q, inp.k, inp.v, inp.g, inp.b, inp.w, inp.S0, None)
    assert np.isfinite(O).all() and np.isfinite(SF).all()
    eo, es = prefill_out_rel(O, Or), state_rel(SF, SFr)
    assert eo <= TOL and es <= TOL, (eo, es)


@pytest.mark.parametrize("n_h", [2, 3])
def test_gdp_tc_strong_channel_decay(cuda_device, spread_limit, n_h):
    """Gated DeltaProduct: the token's decay sits on its first substep, so a
    chunk of the virtual sequence covers 64 / n_h tokens' decays."""
    cfg = inputs.PREFILL["gdp_prefill"].replace(B=2, T=150, H=2, gate="channel", n_h=n_h,
                                                gate_scale=0.05)
    inp = inputs.product_inputs(cfg, seed=704)
    inp.g = strong_channel_gate(inp, 12.0, True)
    dev = cuda_device
    q, k, v = (to_dev(x, "bf16", dev) for x in (inp.q, inp.k, inp.v))
    g, b = to_dev(inp.g, "f32", dev), to_dev(inp.beta, "f32", dev)
    out, SF = binding.gdr_fwd_product(q, k, v, g, b, to_dev(inp.S0, "f32", dev), path="tc")
    torch.cuda.synchronize()
    assert binding.device_status() == binding.GDR_OK
    O, SF = to_np(out), to_np(SF)
    Or, SFr = oracle.product_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.S0, None)
    assert np.isfinite(O).all() and np.isfinite(SF).all()
    eo, es = prefill_out_rel(O, Or), state_rel(SF, SFr)
    assert eo <= TOL and es <= TOL, (eo, es)


@pytest.mark.parametrize("gate", ["channel", "scalar"])
def test_exact_route_agrees_with_factorised_route(cuda_device, spread_limit, gate):
    """On the workloads' ordinary decays both routes apply: limit 0 sends every
    chunk the exact way, the default sends none.  Both meet the oracle, and
    they agree with each other to within the same tolerance."""
    cfg = inputs.PREFILL["kda_prefill"].replace(B=2, T=300, H=3, gate=gate,
                                                gate_scale=0.05 if gate == "channel" else 0.1)
    inp = inputs.prefill_inputs(cfg, seed=705, s0_var=0.01)
    assert max_chunk_spread(inp.g) < DEFAULT_LIMIT
    O1, S1 = check_kda(inp, cuda_device)
    spread_limit(0.0)
    O2, S2 = check_kda(inp, cuda_device)
    assert not np.array_equal(O1, O2)  # the two routes round differently
    assert prefill_out_rel(O2, O1) <= TOL and state_rel(S2, S1) <= TOL

