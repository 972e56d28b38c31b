"""Pins for the Gated DeltaProduct oracle ("Linear Attention, Visualized",
section "Gated Delta Product (GDP)")."""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle


def unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def gdp_case(seed, B=2, T=9, H=2, nh=3, dk=5, dv=3, gate="scalar"):
    rng = np.random.default_rng(seed)
    q = unit_rows(rng.standard_normal((B, T, H, dk)))
    k = unit_rows(rng.standard_normal((B, T, nh, H, dk)))
    v = rng.standard_normal((B, T, nh, H, dv))
    b = rng.uniform(0.05, 1.0, (B, T, nh, H))
    g = -rng.uniform(0.0, 0.3, (B, T, H, dk) if gate == "channel" else (B, T, H))
    S0 = rng.standard_normal((B, H, dv, dk))
    return q, k, v, g, b, S0


def virtual_sequence(q, k, v, g, b):
    """The page's mapping: substeps as consecutive virtual steps, the decay on
    the first substep, the query on the last."""
    B, T, nh, H, dk = k.shape
    kv = k.reshape(B, T * nh, H, dk)
    vv = v.reshape(B, T * nh, H, v.shape[-1])
    bv = b.reshape(B, T * nh, H)
    qv = np.zeros((B, T, nh) + q.shape[2:])
    qv[:, :, nh - 1] = q
    gv = np.zeros((B, T, nh) + g.shape[2:])
    gv[:, :, 0] = g
    return (qv.reshape((B, T * nh) + q.shape[2:]), kv, vv,
            gv.reshape((B, T * nh) + g.shape[2:]), bv)


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("nh", [1, 2, 3])
def test_gdp_equals_gdn_over_virtual_sequence(gate, nh):
    """"GDP as GDN over a virtual sequence": every n_h-th output and the final
    state of the gated delta rule on the flattened substeps."""
    q, k, v, g, b, S0 = gdp_case(1, nh=nh, gate=gate)
    O, SF = oracle.product_fwd(q, k, v, g, b, S0)
    qv, kv, vv, gv, bv = virtual_sequence(q, k, v, g, b)
    Ov, SFv = oracle.recurrence_fwd(qv, kv, vv, gv, bv, S0=S0, threads=2)
    assert np.max(np.abs(O - Ov[:, nh - 1::nh])) < 1e-12
    assert np.max(np.abs(SF - SFv)) < 1e-12


def test_gdp_one_substep_is_gdn():
    q, k, v, g, b, S0 = gdp_case(2, nh=1)
    O, SF = oracle.product_fwd(q, k, v, g, b, S0)
    O2, SF2 = oracle.recurrence_fwd(q, k[:, :, 0], v[:, :, 0], g, b[:, :, 0], S0=S0, threads=2)
    assert np.max(np.abs(O - O2)) < 1e-13 and np.max(np.abs(SF - SF2)) < 1e-13


def test_gdp_swaps_compose_within_a_token():
    """Two swap substeps per token (beta = 2, v = 0) apply their composed
    permutation to the key columns in one token ("A Swap Is a Reflection...":
    composing swaps tracks a permutation)."""
    rng = np.random.default_rng(3)
    dk, dv, T, nh = 6, 4, 5, 2
    k = np.zeros((1, T, nh, 1, dk))
    perm = np.arange(dk)
    for t in range(T):
        for j in range(nh):
            a, c = rng.choice(dk, 2, replace=False)
            k[0, t, j, 0, a], k[0, t, j, 0, c] = 1 / math.sqrt(2), -1 / math.sqrt(2)
            perm[[a, c]] = perm[[c, a]]
    S0 = rng.standard_normal((1, 1, dv, dk))
    _, SF = oracle.product_fwd(np.zeros((1, T, 1, dk)), k, np.zeros((1, T, nh, 1, dv)),
                               np.zeros((1, T, 1)), np.full((1, T, nh, 1), 2.0), S0)
    assert np.max(np.abs(SF[0, 0] - S0[0, 0][:, perm])) < 1e-12


def test_gdp_exact_rationals():
    """Brute force in exact rationals of the page's update: decay once, then
    S_tj = S_t(j-1) (I - beta k k^T) + beta v k^T for each substep."""
    rng = np.random.default_rng(4)
    T, nh, dk, dv = 3, 2, 3, 2
    d = lambda shape, den: rng.integers(-den, den + 1, shape) / den
    q, k, v = d((1, T, 1, dk), 4), d((1, T, nh, 1, dk), 4), d((1, T, nh, 1, dv), 4)
    b = rng.integers(1, 5, (1, T, nh, 1)) / 4
    halves = rng.integers(0, 2, (1, T, 1))
    g = np.where(halves == 1, math.log(0.5), 0.0)
    S0 = d((1, 1, dv, dk), 2)
    O, SF = oracle.product_fwd(q, k, v, g, b, S0)
    F = lambda x: Fraction(float(x))
    S = [[F(S0[0, 0, r, c]) for c in range(dk)] for r in range(dv)]
    for t in range(T):
        a = Fraction(1, 2) if halves[0, t, 0] else Fraction(1)
        S = [[x * a for x in row] for row in S]
        for j in range(nh):
            kt = [F(x) for x in k[0, t, j, 0]]
            bt = F(b[0, t, j, 0])
            P = [[(1 if r == c else 0) - bt * kt[r] * kt[c] for c in range(dk)] for r in range(dk)]
            S = [[sum(S[r][m] * P[m][c] for m in range(dk)) + bt * F(v[0, t, j, 0, r]) * kt[c]
                  for c in range(dk)] for r in range(dv)]
        o = [sum(S[r][c] * F(q[0, t, 0, c]) for c in range(dk)) for r in range(dv)]
        assert np.max(np.abs(O[0, t, 0] - np.array([float(x) for x in o]))) < 1e-13
    assert np.max(np.abs(SF[0, 0] - np.array([[float(x) for x in r] for r in S]))) < 1e-13


def test_gdp_varlen_resets_state():
    q, k, v, g, b, _ = gdp_case(5, B=1, T=12, nh=2)
    cu = np.array([0, 5, 5, 12])
    S0 = np.random.default_rng(6).standard_normal((3, 2, 3, 5))
    O, SF = oracle.product_fwd(q, k, v, g, b, S0, cu)
    for s in range(3):
        a, e = cu[s], cu[s + 1]
        Os, Ss = oracle.product_fwd(q[:, a:e], k[:, a:e], v[:, a:e], g[:, a:e], b[:, a:e],
                                    S0[s:s + 1])
        assert np.max(np.abs(O[:, a:e] - Os)) < 1e-15 if e > a else True
        assert np.max(np.abs(SF[s] - Ss[0])) < 1e-15
