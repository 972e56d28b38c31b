"""Pins for the Gated DeltaNet-2 oracle ("Gated DeltaNet-2, and the gate that
was doing two jobs", section "What decoupling actually means here")."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle.chunked import gdn2_chunked_fwd


def unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def case(seed, B=2, T=23, H=2, dk=6, dv=5, gate="channel", scale=0.2):
    rng = np.random.default_rng(seed)
    q = unit_rows(rng.standard_normal((B, T, H, dk)))
    k = unit_rows(rng.standard_normal((B, T, H, dk)))
    v = rng.standard_normal((B, T, H, dv))
    b = rng.uniform(0, 1, (B, T, H, dk))
    w = rng.uniform(0, 1, (B, T, H, dv))
    g = -rng.uniform(0, scale, (B, T, H, dk) if gate == "channel" else (B, T, H))
    S0 = rng.standard_normal((B, H, dv, dk))
    return q, k, v, g, b, w, S0


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_equal_scalar_gates_collapse_to_the_gated_delta_rule(gate):
    """b = beta 1 and w = beta 1 give KDA (per-channel decay) or Gated DeltaNet
    (scalar decay): checked against the gated delta rule oracle."""
    q, k, v, g, _, _, S0 = case(1, gate=gate)
    beta = np.random.default_rng(2).uniform(0.05, 1.0, q.shape[:3])
    b = np.repeat(beta[..., None], q.shape[-1], axis=-1)
    w = np.repeat(beta[..., None], v.shape[-1], axis=-1)
    O, SF = oracle.gdn2_fwd(q, k, v, g, b, w, S0)
    O2, SF2 = oracle.recurrence_fwd(q, k, v, g, beta, S0=S0, threads=2)
    assert np.max(np.abs(O - O2)) < 1e-12 and np.max(np.abs(SF - SF2)) < 1e-12


@pytest.mark.parametrize("C", [1, 5, 16, 64, 128])
@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_chunkwise_form_matches(C, gate):
    """The page's chunkwise form (decay normalised out, one triangular solve
    with two right-hand sides) equals the token recurrence for every C."""
    q, k, v, g, b, w, S0 = case(3, T=37 if C < 64 else 150, gate=gate)
    O, SF = oracle.gdn2_fwd(q, k, v, g, b, w, S0)
    Oc, SFc = gdn2_chunked_fwd(q, k, v, g, b, w, S0, C=C)
    assert np.max(np.abs(O - Oc)) < 1e-11 and np.max(np.abs(SF - SFc)) < 1e-11


def test_exact_rationals_row_convention():
    """Exact brute force of the page's formula as printed, in its row
    convention S_t = (I - k e^T) D S + k z^T, o = S^T q, against the oracle's
    column-convention state (its transpose)."""
    rng = np.random.default_rng(4)
    T, dk, dv = 4, 3, 2
    d = lambda shape, den: rng.integers(-den, den + 1, shape) / den
    q, k, v = d((1, T, 1, dk), 4), d((1, T, 1, dk), 4), d((1, T, 1, dv), 4)
    b = rng.integers(0, 5, (1, T, 1, dk)) / 4
    w = rng.integers(0, 5, (1, T, 1, dv)) / 4
    halves = rng.integers(0, 2, (1, T, 1, dk))
    g = np.where(halves == 1, np.log(0.5), 0.0)
    S0 = d((1, 1, dv, dk), 2)
    O, SF = oracle.gdn2_fwd(q, k, v, g, b, w, S0)
    F = lambda x: Fraction(float(x))
    S = [[F(S0[0, 0, j, i]) for j in range(dv)] for i in range(dk)]   # row convention
    for t in range(T):
        D = [Fraction(1, 2) if halves[0, t, 0, i] else Fraction(1) for i in range(dk)]
        kt = [F(x) for x in k[0, t, 0]]
        e = [F(b[0, t, 0, i]) * kt[i] for i in range(dk)]
        z = [F(w[0, t, 0, j]) * F(v[0, t, 0, j]) for j in range(dv)]
        DS = [[D[i] * S[i][j] for j in range(dv)] for i in range(dk)]
        eDS = [sum(e[i] * DS[i][j] for i in range(dk)) for j in range(dv)]
        S = [[DS[i][j] - kt[i] * eDS[j] + kt[i] * z[j] for j in range(dv)] for i in range(dk)]
        o = [sum(S[i][j] * F(q[0, t, 0, i]) for i in range(dk)) for j in range(dv)]
        assert np.max(np.abs(O[0, t, 0] - np.array([float(x) for x in o]))) < 1e-13
    ST = np.array([[float(S[i][j]) for i in range(dk)] for j in range(dv)])
    assert np.max(np.abs(SF[0, 0] - ST)) < 1e-13


def test_no_erase_is_decayed_accumulation():
    """b = 0: nothing is erased, S_T = S0 Gamma_T + sum_t z_t k_t^T (Gamma_T / Gamma_t)."""
    q, k, v, g, _, w, S0 = case(5, B=1, H=1)
    b = np.zeros_like(k)
    _, SF = oracle.gdn2_fwd(q, k, v, g, b, w, S0)
    G = np.cumsum(g[0, :, 0], axis=0)
    S = S0[0, 0] * np.exp(G[-1])
    for t in range(q.shape[1]):
        S = S + np.outer(w[0, t, 0] * v[0, t, 0], k[0, t, 0] * np.exp(G[-1] - G[t]))
    assert np.max(np.abs(SF[0, 0] - S)) < 1e-12


def test_full_erase_reads_back_the_write():
    """b = 1, w = 1, unit keys: e = k, so S_t k_t = z_t = v_t after every token."""
    q, k, v, g, _, _, S0 = case(6, B=1, H=1, T=9)
    b, w = np.ones_like(k), np.ones_like(v)
    for t in range(1, 10):
        _, SF = oracle.gdn2_fwd(q[:, :t], k[:, :t], v[:, :t], g[:, :t], b[:, :t], w[:, :t], S0)
        assert np.max(np.abs(SF[0, 0] @ k[0, t - 1, 0] - v[0, t - 1, 0])) < 1e-12
