"""Pins for the CPU oracle: what the pages and the mathematics fix.

Every pin is a function of an implementation ``impl(q, k, v, g, beta, S0,
cu_seqlens) -> (O, S_final)`` (column convention, S is d_v x d_k).  The oracle
must pass all of them; every planted mistake (``MUTANTS`` below: a dropped
term, a wrong sign, a wrong order, a swapped operand) must fail at least one.
Shapes use d_k != d_v so that a transposed state cannot pass silently.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg

import oracle
from oracle.chunked import chunked_fwd

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
TOL = 1e-12


def rel(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-300))


def unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def rand_case(seed, B=2, T=11, H=2, dk=5, dv=3, gate="scalar", beta=None, g_scale=0.3,
              s0=True):
    rng = np.random.default_rng(seed)
    q = unit_rows(rng.standard_normal((B, T, H, dk)))
    k = unit_rows(rng.standard_normal((B, T, H, dk)))
    v = rng.standard_normal((B, T, H, dv))
    b = rng.uniform(0.05, 1.0, (B, T, H)) if beta is None else np.full((B, T, H), float(beta))
    gshape = (B, T, H, dk) if gate == "channel" else (B, T, H)
    g = -rng.uniform(0.0, g_scale, gshape)
    S0 = rng.standard_normal((B, H, dv, dk)) if s0 else None
    return q, k, v, g, b, S0


def oracle_impl(q, k, v, g, beta, S0=None, cu_seqlens=None):
    return oracle.recurrence_fwd(q, k, v, g, beta, S0=S0, cu_seqlens=cu_seqlens, threads=2)


# --------------------------------------------------------------------------
# planted mistakes (each is a plausible slip in writing the recurrence)
# --------------------------------------------------------------------------
def _mutant(kind):
    def impl(q, k, v, g, beta, S0=None, cu_seqlens=None):
        q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        segs = ([(b, 0, T) for b in range(B)] if cu_seqlens is None else
                [(0, int(cu_seqlens[i]), int(cu_seqlens[i + 1])) for i in range(len(cu_seqlens) - 1)])
        O = np.zeros((B, T, H, dv))
        SF = np.zeros((len(segs), H, dv, dk))
        for s, (b, t0, t1) in enumerate(segs):
            for h in range(H):
                S = np.zeros((dv, dk)) if S0 is None else np.array(S0[s, h], dtype=np.float64)
                for t in range(t0, t1):
                    kt, qt, vt, bt = k[b, t, h], q[b, t, h], v[b, t, h], beta[b, t, h]
                    gt = g[b, t, h]
                    a = np.exp(-gt if kind == "gate_sign" else gt)
                    dec = (lambda M: M * a[None, :]) if np.ndim(a) else (lambda M: M * a)
                    if kind == "erase_then_decay":
                        S = dec(S @ (np.eye(dk) - bt * np.outer(kt, kt)) + bt * np.outer(vt, kt))
                        O[b, t, h] = S @ qt
                        continue
                    Sd = dec(S)
                    p = (S if kind == "no_decay_in_prediction" else Sd) @ kt
                    u = bt * (vt + p) if kind == "wrong_sign" else bt * (vt - p)
                    if kind == "beta_twice":
                        u = bt * u
                    Snew = Sd + np.outer(u, kt)
                    if kind == "read_before_write":
                        O[b, t, h] = Sd @ qt
                    elif kind == "read_with_key":
                        O[b, t, h] = Snew @ kt
                    else:
                        O[b, t, h] = Snew @ qt
                    S = Snew
                SF[s, h] = S
        return O, SF
    return impl


MUTANTS = ["no_decay_in_prediction", "erase_then_decay", "wrong_sign", "beta_twice",
           "read_before_write", "read_with_key", "gate_sign"]


# --------------------------------------------------------------------------
# pins
# --------------------------------------------------------------------------
def pin_beta_zero_pure_decay(impl):
    """beta = 0 leaves only the decay (the Mamba-2 limit): S_t = S0 D_1...D_t.
    Sources: "Gated DeltaNet: Householder Transitions...", The gated delta rule
    (beta -> 0 gives Mamba2's decay); "Linear Attention, Visualized", Mamba-2."""
    for gate in ("scalar", "channel"):
        q, k, v, g, b, S0 = rand_case(1, gate=gate, beta=0.0)
        O, SF = impl(q, k, v, g, b, S0)
        cum = np.cumsum(g, axis=1)
        B, T, H = b.shape
        for bb in range(B):
            for h in range(H):
                for t in range(T):
                    dec = np.exp(cum[bb, t, h])
                    St = S0[bb, h] * (dec[None, :] if gate == "channel" else dec)
                    assert rel(O[bb, t, h], St @ q[bb, t, h]) < TOL
                assert rel(SF[bb, h], St) < TOL


def pin_alpha_one_deltanet_parallel(impl):
    """alpha = 1 is DeltaNet; with S0 = 0 its full-sequence parallel form is
    U = (I + B (K K^T . M^-))^{-1} B V, O = (Q K^T . M) U, S = sum_t u_t k_t^T.
    Source: "Linear Attention, Visualized", DeltaNet / The triangular
    correction system and Parallel output."""
    q, k, v, g, b, _ = rand_case(2, T=13, g_scale=0.0, s0=False)
    g = np.zeros_like(g)
    O, SF = impl(q, k, v, g, b, None)
    B, T, H = b.shape
    for bb in range(B):
        for h in range(H):
            K, Q, V, beta = k[bb, :, h], q[bb, :, h], v[bb, :, h], b[bb, :, h]
            L = np.tril(K @ K.T, -1)
            U = scipy.linalg.solve_triangular(np.eye(T) + beta[:, None] * L, beta[:, None] * V,
                                              lower=True, unit_diagonal=True)
            assert rel(O[bb, :, h], np.tril(Q @ K.T) @ U) < TOL
            assert rel(SF[bb, h], U.T @ K) < TOL


def pin_beta_one_exact_overwrite(impl):
    """beta = 1 with a unit key stores v exactly: S_t k_t = v_t, whatever the
    decay.  Source: "Linear Attention, Visualized", An intuitive example
    (k_t S_t = (1 - beta) v_hat + beta v for a unit key)."""
    for gate in ("scalar", "channel"):
        q, k, v, g, b, S0 = rand_case(3, B=1, T=7, gate=gate, beta=1.0)
        for t in range(1, 8):
            _, SF = impl(q[:, :t], k[:, :t], v[:, :t], g[:, :t], b[:, :t], S0)
            for h in range(q.shape[2]):
                assert rel(SF[0, h] @ k[0, t - 1, h], v[0, t - 1, h]) < 1e-12


def pin_swap_is_reflection(impl):
    """k = (e_i - e_j)/sqrt(2), beta = 2, alpha = 1, v = 0 exchanges key
    columns i and j; a run of such tokens composes into a permutation (golden
    fixture tests/golden/swap_permutation.json)."""
    gold = json.load(open(os.path.join(GOLD, "swap_permutation.json")))
    dk, dv = gold["d_k"], gold["d_v"]
    n = len(gold["swaps"])
    k = np.zeros((1, n, 1, dk))
    q = np.zeros((1, n, 1, dk))
    for t, (i, j) in enumerate(gold["swaps"]):
        k[0, t, 0, i] = 1 / math.sqrt(2)
        k[0, t, 0, j] = -1 / math.sqrt(2)
        q[0, t, 0, gold["q_index"][t]] = 1.0
    v = np.zeros((1, n, 1, dv))
    beta = np.full((1, n, 1), 2.0)
    g = np.zeros((1, n, 1))
    S0 = np.array(gold["S0"], dtype=np.float64)[None, None]
    O, SF = impl(q, k, v, g, beta, S0)
    assert np.max(np.abs(O[0, :, 0] - np.array(gold["expected_out"]))) < 1e-13
    assert np.max(np.abs(SF[0, 0] - np.array(gold["expected_S_final"]))) < 1e-13
    # a random run of swaps tracks the composed permutation
    rng = np.random.default_rng(4)
    dk = 6
    S0 = rng.standard_normal((1, 1, 4, dk))
    perm = np.arange(dk)
    T = 20
    k = np.zeros((1, T, 1, dk))
    for t in range(T):
        i, j = rng.choice(dk, 2, replace=False)
        k[0, t, 0, i], k[0, t, 0, j] = 1 / math.sqrt(2), -1 / math.sqrt(2)
        perm[[i, j]] = perm[[j, i]]
    _, SF = impl(np.zeros((1, T, 1, dk)), k, np.zeros((1, T, 1, 4)), np.zeros((1, T, 1)),
                 np.full((1, T, 1), 2.0), S0)
    assert np.max(np.abs(SF[0, 0] - S0[0, 0][:, perm])) < 1e-12


def pin_chunkwise_equals_recurrence(impl):
    """Every chunk size gives the exact result ("Linear Attention, Visualized",
    Chunkwise algorithm / Cost): the independent chunkwise WY/UT form
    (oracle.chunked) agrees at C in {1, 16, 37, 64, 128}, with a partial last chunk,
    scalar and per-channel gates, nonzero S0 and a packed variable-length
    batch."""
    for gate in ("scalar", "channel"):
        q, k, v, g, b, S0 = rand_case(5, B=1, T=150, H=1, dk=6, dv=4, gate=gate, g_scale=0.1)
        O, SF = impl(q, k, v, g, b, S0)
        for C in (1, 16, 37, 64, 128):
            Oc, SFc = chunked_fwd(q, k, v, g, b, C, S0=S0)
            assert rel(Oc, O) < 1e-11 and rel(SFc, SF) < 1e-11, (gate, C)
    q, k, v, g, b, _ = rand_case(6, B=1, T=90, H=2, dk=5, dv=3, g_scale=0.2)
    cu = np.array([0, 17, 17, 60, 90])
    S0 = np.random.default_rng(7).standard_normal((4, 2, 3, 5))
    O, SF = impl(q, k, v, g, b, S0, cu)
    Oc, SFc = chunked_fwd(q, k, v, g, b, 16, S0=S0, cu_seqlens=cu)
    assert rel(Oc, O) < 1e-11 and rel(SFc, SF) < 1e-11


def pin_kda_broadcast_gate_is_gdn(impl):
    """A per-channel gate equal in every channel is the scalar gate ("Linear
    Attention, Visualized", KDA: if a_t = a_t 1 it reduces exactly to GDN)."""
    q, k, v, g, b, S0 = rand_case(8)
    O1, S1 = impl(q, k, v, g, b, S0)
    O2, S2 = impl(q, k, v, np.repeat(g[..., None], q.shape[-1], axis=-1), b, S0)
    assert rel(O2, O1) < 1e-14 and rel(S2, S1) < 1e-14


def pin_orthonormal_keys(impl):
    """With orthonormal keys the correction terms vanish and the gated delta
    rule is decayed linear attention ("video-delta-rule", permutation analysis:
    with orthogonal keys the delta rule loses its corrections; "Linear
    Attention, Visualized", Mamba-2 parallel form O = (Q K^T . Gamma) V) with
    values beta_t v_t.  For a per-channel gate the decay of entry (t, i) is
    that of key channel c_i."""
    rng = np.random.default_rng(9)
    T, dk, dv = 6, 8, 3
    order = rng.permutation(dk)[:T]
    k = np.zeros((1, T, 1, dk))
    for t in range(T):
        k[0, t, 0, order[t]] = 1.0
    q = rng.standard_normal((1, T, 1, dk))
    v = rng.standard_normal((1, T, 1, dv))
    b = rng.uniform(0.1, 1.0, (1, T, 1))
    for gate in ("scalar", "channel"):
        g = -rng.uniform(0, 0.5, (1, T, 1, dk) if gate == "channel" else (1, T, 1))
        O, _ = impl(q, k, v, g, b, None)
        ref = np.zeros((T, dv))
        for t in range(T):
            for i in range(t + 1):
                c = order[i]
                if gate == "channel":
                    lam = np.exp(np.sum(g[0, i + 1:t + 1, 0, c]))
                else:
                    lam = np.exp(np.sum(g[0, i + 1:t + 1, 0]))
                ref[t] += q[0, t, 0, c] * lam * b[0, i, 0] * v[0, i, 0]
        assert rel(O[0, :, 0], ref) < TOL


def _dyadic(rng, shape, denom=8):
    return rng.integers(-denom, denom + 1, shape) / denom


def pin_worked_correction_rows(impl):
    """Exact rationals: u_1 = beta_1 v_1, u_l = beta_l (v_l - sum_{i<l} (k_l . k_i) u_i)
    and S_t = sum_{i<=t} u_i k_i^T ("Linear Attention, Visualized", DeltaNet /
    The triangular correction system, first three rows and general row)."""
    rng = np.random.default_rng(10)
    T, dk, dv = 4, 3, 2
    k = _dyadic(rng, (1, T, 1, dk), 4)
    q = _dyadic(rng, (1, T, 1, dk), 4)
    v = _dyadic(rng, (1, T, 1, dv), 4)
    b = np.array([0.5, 0.25, 1.0, 0.75]).reshape(1, T, 1)
    O, SF = impl(q, k, v, np.zeros((1, T, 1)), b, None)
    F = lambda x: Fraction(float(x))
    K = [[F(x) for x in k[0, t, 0]] for t in range(T)]
    Q = [[F(x) for x in q[0, t, 0]] for t in range(T)]
    V = [[F(x) for x in v[0, t, 0]] for t in range(T)]
    Bt = [F(x) for x in b[0, :, 0]]
    dot = lambda a, c: sum(x * y for x, y in zip(a, c))
    U = []
    for l in range(T):
        row = [V[l][j] - sum(dot(K[l], K[i]) * U[i][j] for i in range(l)) for j in range(dv)]
        U.append([Bt[l] * x for x in row])
    for t in range(T):
        o = [sum(U[i][j] * dot(K[i], Q[t]) for i in range(t + 1)) for j in range(dv)]
        assert np.max(np.abs(O[0, t, 0] - np.array([float(x) for x in o]))) < 1e-14
    S = [[float(sum(U[i][r] * K[i][c] for i in range(T))) for c in range(dk)] for r in range(dv)]
    assert np.max(np.abs(SF[0, 0] - np.array(S))) < 1e-14


def pin_product_form_exact(impl):
    """Brute force in exact rationals of the product form of the problem
    statement, S_t = (S_{t-1} D_t)(I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
    o_t = S_t q_t, for decays in {1, 1/2}, scalar and per-channel
    ("Gated DeltaNet: Householder Transitions...", The gated delta rule;
    "Linear Attention, Visualized", KDA: decay first, then the correction)."""
    rng = np.random.default_rng(11)
    T, dk, dv = 4, 3, 2
    for gate in ("scalar", "channel"):
        k = _dyadic(rng, (1, T, 1, dk), 4)
        q = _dyadic(rng, (1, T, 1, dk), 4)
        v = _dyadic(rng, (1, T, 1, dv), 4)
        b = rng.integers(1, 5, (1, T, 1)) / 4
        halves = rng.integers(0, 2, (1, T, 1, dk) if gate == "channel" else (1, T, 1))
        g = np.where(halves == 1, math.log(0.5), 0.0)
        S0 = _dyadic(rng, (1, 1, dv, dk), 2)
        O, SF = impl(q, k, v, g, b, S0)
        F = lambda x: Fraction(float(x))
        S = [[F(S0[0, 0, r, c]) for c in range(dk)] for r in range(dv)]
        for t in range(T):
            kt = [F(x) for x in k[0, t, 0]]
            if gate == "channel":
                a = [Fraction(1, 2) if halves[0, t, 0, c] else Fraction(1) for c in range(dk)]
            else:
                a = [Fraction(1, 2) if halves[0, t, 0] else Fraction(1)] * dk
            bt = F(b[0, t, 0])
            P = [[(1 if r == c else 0) - bt * kt[r] * kt[c] for c in range(dk)] for r in range(dk)]
            Sd = [[S[r][c] * a[c] for c in range(dk)] for r in range(dv)]
            S = [[sum(Sd[r][m] * P[m][c] for m in range(dk)) + bt * F(v[0, t, 0, r]) * kt[c]
                  for c in range(dk)] for r in range(dv)]
            o = [sum(S[r][c] * F(q[0, t, 0, c]) for c in range(dk)) for r in range(dv)]
            assert np.max(np.abs(O[0, t, 0] - np.array([float(x) for x in o]))) < 1e-13, gate
        assert np.max(np.abs(SF[0, 0] - np.array([[float(x) for x in r] for r in S]))) < 1e-13


def pin_alice_bob(impl):
    """Golden fixture tests/golden/alice_bob.json ("Linear Attention,
    Visualized", DeltaNet / An intuitive example)."""
    gold = json.load(open(os.path.join(GOLD, "alice_bob.json")))
    k = np.array(gold["k"], dtype=np.float64)[None, :, None]
    q = np.array(gold["q"], dtype=np.float64)[None, :, None]
    v = np.array(gold["v"], dtype=np.float64)[None, :, None]
    b = np.array(gold["beta"])[None, :, None]
    g = np.array(gold["g"])[None, :, None]
    S0 = np.array(gold["S0"], dtype=np.float64)[None, None]
    O, _ = impl(q, k, v, g, b, S0)
    assert np.max(np.abs(O[0, :, 0] - np.array(gold["expected_out"]))) < 1e-15


PINS = [pin_beta_zero_pure_decay, pin_alpha_one_deltanet_parallel, pin_beta_one_exact_overwrite,
        pin_swap_is_reflection, pin_chunkwise_equals_recurrence, pin_kda_broadcast_gate_is_gdn,
        pin_orthonormal_keys, pin_worked_correction_rows, pin_product_form_exact, pin_alice_bob]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_passes_pin(pin):
    pin(oracle_impl)


@pytest.mark.parametrize("kind", MUTANTS)
def test_planted_mistake_fails_some_pin(kind):
    impl = _mutant(kind)
    failed = []
    for pin in PINS:
        try:
            pin(impl)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"planted mistake {kind!r} passed every pin"


def test_mutant_harness_is_faithful_without_mistake():
    """The planted-mistake harness with no mistake passes every pin, so a
    failure above is due to the planted mistake alone."""
    impl = _mutant("none")
    for pin in PINS:
        pin(impl)


# --------------------------------------------------------------------------
# structural properties of the oracle's entry points
# --------------------------------------------------------------------------
def test_decode_step_equals_prefill():
    """T decode steps equal one prefill over the same T tokens (the chunk size
    1 case of "Every valid C provides exact results")."""
    for gate in ("scalar", "channel"):
        q, k, v, g, b, S0 = rand_case(12, B=3, T=5, H=2, gate=gate)
        O, SF = oracle_impl(q, k, v, g, b, S0)
        S = S0.copy()
        for t in range(q.shape[1]):
            o, S = oracle.recurrence_decode_step(q[:, t], k[:, t], v[:, t], g[:, t], b[:, t], S)
            assert rel(o, O[:, t]) < 1e-14
        assert rel(S, SF) < 1e-14


def test_varlen_equals_separate_sequences():
    """A packed batch resets the state at every boundary: it equals separate
    runs of its sequences."""
    q, k, v, g, b, _ = rand_case(13, B=1, T=40, H=2)
    cu = np.array([0, 7, 7, 31, 40])
    S0 = np.random.default_rng(14).standard_normal((4, 2, 3, 5))
    O, SF = oracle_impl(q, k, v, g, b, S0, cu)
    for s in range(4):
        a, e = cu[s], cu[s + 1]
        Os, Ss = oracle_impl(q[:, a:e], k[:, a:e], v[:, a:e], g[:, a:e], b[:, a:e], S0[s:s + 1])
        assert rel(O[:, a:e], Os) < 1e-15 if e > a else True
        assert rel(SF[s], Ss[0]) < 1e-15


def test_split_and_continue():
    """Affine lemma ("Linear Attention, Visualized", One chunk as an affine
    recurrence): running [0, tau) and then [tau, T) from S_tau equals [0, T)."""
    q, k, v, g, b, S0 = rand_case(15, T=20, gate="channel")
    O, SF = oracle_impl(q, k, v, g, b, S0)
    O1, S1 = oracle_impl(q[:, :8], k[:, :8], v[:, :8], g[:, :8], b[:, :8], S0)
    O2, S2 = oracle_impl(q[:, 8:], k[:, 8:], v[:, 8:], g[:, 8:], b[:, 8:], S1)
    assert rel(np.concatenate([O1, O2], axis=1), O) < 1e-15 and rel(S2, SF) < 1e-15


def test_state_size_of_the_published_shape():
    """16 heads x 128 x 128 is 262,144 state floats per layer ("Gated
    DeltaNet-2, and the gate that was doing two jobs", section 3)."""
    rng = np.random.default_rng(16)
    S0 = np.zeros((1, 16, 128, 128))
    q = unit_rows(rng.standard_normal((1, 1, 16, 128)))
    _, SF = oracle_impl(q, q, rng.standard_normal((1, 1, 16, 128)), np.zeros((1, 1, 16)),
                        np.ones((1, 1, 16)), S0)
    assert SF.size == 262144


def test_oracle_rejects_bad_varlen():
    q, k, v, g, b, _ = rand_case(17, B=1, T=10)
    with pytest.raises(ValueError):
        oracle_impl(q, k, v, g, b, None, np.array([0, 6, 4, 10]))
    with pytest.raises(ValueError):
        oracle_impl(q, k, v, g, b, None, np.array([0, 4, 9]))


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_chunked_oracle_passes_pin(pin):
    """The chunkwise oracle (chunk 4) meets the same pins on its own."""
    pin(lambda q, k, v, g, b, S0=None, cu=None: chunked_fwd(q, k, v, g, b, 4, S0=S0,
                                                            cu_seqlens=cu))
