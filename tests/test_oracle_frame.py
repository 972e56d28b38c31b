"""Pins for the implicit frame-level update oracle ("video-delta-rule",
sections "A First Attempt at Frame-Level Updates" and "A Different Route")."""
from fractions import Fraction

import numpy as np
import pytest

import oracle


def unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def case(seed, B=2, T=20, H=2, dk=6, dv=5, n=4, gate="channel"):
    rng = np.random.default_rng(seed)
    F = -(-T // n)
    q = unit_rows(rng.standard_normal((B, T, H, dk)))
    k = unit_rows(rng.standard_normal((B, T, H, dk)))
    v = rng.standard_normal((B, T, H, dv))
    gam = rng.uniform(0, 2.0, (B, T, H))
    g = -rng.uniform(0, 0.3, (B, F, H, dk) if gate == "channel" else (B, F, H))
    S0 = rng.standard_normal((B, H, dv, dk))
    return q, k, v, g, gam, S0


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_one_token_frames_are_the_delta_rule(gate):
    """n = 1: by Sherman-Morrison the step is the gated delta rule with
    learning rate gamma / (1 + gamma) (section "A Different Route")."""
    q, k, v, g, gam, S0 = case(1, n=1, gate=gate)
    O, SF = oracle.frame_fwd(q, k, v, g, gam, 1, S0)
    O2, SF2 = oracle.recurrence_fwd(q, k, v, g, gam / (1 + gam), S0=S0, threads=2)
    assert np.max(np.abs(O - O2)) < 1e-12 and np.max(np.abs(SF - SF2)) < 1e-12


def test_permutation_invariance_within_frames():
    """Permuting the tokens inside every frame leaves the state unchanged and
    permutes the outputs with the tokens."""
    q, k, v, g, gam, S0 = case(2, T=24, n=6)
    O, SF = oracle.frame_fwd(q, k, v, g, gam, 6, S0)
    perm = np.concatenate([f * 6 + np.random.default_rng(3 + f).permutation(6) for f in range(4)])
    P = lambda x: x[:, perm]
    Op, SFp = oracle.frame_fwd(P(q), P(k), P(v), g, P(gam), 6, S0)
    assert np.max(np.abs(SFp - SF)) < 1e-12
    assert np.max(np.abs(Op - O[:, perm])) < 1e-12


def test_orthonormal_keys_closed_form():
    """With orthonormal keys in a frame, (I + G)^-1 = I - sum_i b_i k_i k_i^T,
    b_i = gamma_i / (1 + gamma_i): S_t = (S D + C)(I - sum_i b_i k_i k_i^T)."""
    rng = np.random.default_rng(4)
    dk, dv, n, F = 8, 3, 5, 3
    T = n * F
    k = np.zeros((1, T, 1, dk))
    for f in range(F):
        Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
        k[0, f * n:(f + 1) * n, 0] = Qm[:, :n].T
    q = rng.standard_normal((1, T, 1, dk))
    v = rng.standard_normal((1, T, 1, dv))
    gam = rng.uniform(0, 3, (1, T, 1))
    g = -rng.uniform(0, 0.4, (1, F, 1, dk))
    S0 = rng.standard_normal((1, 1, dv, dk))
    O, SF = oracle.frame_fwd(q, k, v, g, gam, n, S0)
    S = S0[0, 0].copy()
    for f in range(F):
        sl = slice(f * n, (f + 1) * n)
        Kf, Vf, gf = k[0, sl, 0], v[0, sl, 0], gam[0, sl, 0]
        Bm = S * np.exp(g[0, f, 0])[None, :] + (Vf.T * gf) @ Kf
        P = np.eye(dk) - (Kf.T * (gf / (1 + gf))) @ Kf
        S = Bm @ P
        assert np.max(np.abs(O[0, sl, 0] - q[0, sl, 0] @ S.T)) < 1e-12
    assert np.max(np.abs(SF[0, 0] - S)) < 1e-12


def test_no_writing_strength_is_pure_decay():
    q, k, v, g, _, S0 = case(5, gate="scalar")
    gam = np.zeros(q.shape[:3])
    _, SF = oracle.frame_fwd(q, k, v, g, gam, 4, S0)
    assert np.max(np.abs(SF - S0 * np.exp(g.sum(axis=1))[:, :, None, None])) < 1e-12


def test_exact_rationals_gaussian_elimination():
    """Exact brute force: S_t solves S_t (I + G_t) = S_{t-1} D_t + C_t, found by
    Gaussian elimination in rationals (no Cholesky), then o_i = S_t q_i."""
    rng = np.random.default_rng(6)
    T, n, dk, dv = 5, 2, 3, 2
    d = lambda shape, den: rng.integers(-den, den + 1, shape) / den
    q, k, v = d((1, T, 1, dk), 4), d((1, T, 1, dk), 4), d((1, T, 1, dv), 4)
    gam = rng.integers(0, 5, (1, T, 1)) / 2
    halves = rng.integers(0, 2, (1, 3, 1, dk))
    g = np.where(halves == 1, np.log(0.5), 0.0)
    S0 = d((1, 1, dv, dk), 2)
    O, SF = oracle.frame_fwd(q, k, v, g, gam, n, S0)
    F = lambda x: Fraction(float(x))
    S = [[F(S0[0, 0, i, j]) for j in range(dk)] for i in range(dv)]
    for f in range(3):
        toks = range(f * n, min(T, f * n + n))
        A = [[Fraction(int(i == j)) for j in range(dk)] for i in range(dk)]
        Bm = [[S[i][j] * (Fraction(1, 2) if halves[0, f, 0, j] else 1) for j in range(dk)]
              for i in range(dv)]
        for t in toks:
            kt, vt, gt = [F(x) for x in k[0, t, 0]], [F(x) for x in v[0, t, 0]], F(gam[0, t, 0])
            for i in range(dk):
                for j in range(dk):
                    A[i][j] += gt * kt[i] * kt[j]
            for i in range(dv):
                for j in range(dk):
                    Bm[i][j] += gt * vt[i] * kt[j]
        # S A = Bm  <=>  A^T S^T = Bm^T; Gauss-Jordan on [A^T | Bm^T]
        M = [[A[j][i] for j in range(dk)] + [Bm[r][i] for r in range(dv)] for i in range(dk)]
        for c in range(dk):
            piv = next(r for r in range(c, dk) if M[r][c] != 0)
            M[c], M[piv] = M[piv], M[c]
            pv = M[c][c]
            M[c] = [x / pv for x in M[c]]
            for r in range(dk):
                if r != c and M[r][c] != 0:
                    fac = M[r][c]
                    M[r] = [a - fac * b for a, b in zip(M[r], M[c])]
        S = [[M[j][dk + i] for j in range(dk)] for i in range(dv)]
        for t in toks:
            o = [sum(S[i][j] * F(q[0, t, 0, j]) for j in range(dk)) for i in range(dv)]
            assert np.max(np.abs(O[0, t, 0] - np.array([float(x) for x in o]))) < 1e-13
    assert np.max(np.abs(SF[0, 0] - np.array([[float(x) for x in r] for r in S]))) < 1e-13


def test_partial_last_frame_and_split():
    """A shorter last frame is one more step; running the frames in two calls
    (S_final -> S0) gives the same state."""
    q, k, v, g, gam, S0 = case(7, T=22, n=4)
    O, SF = oracle.frame_fwd(q, k, v, g, gam, 4, S0)
    O1, S1 = oracle.frame_fwd(q[:, :12], k[:, :12], v[:, :12], g[:, :3], gam[:, :12], 4, S0)
    O2, S2 = oracle.frame_fwd(q[:, 12:], k[:, 12:], v[:, 12:], g[:, 3:], gam[:, 12:], 4, S1)
    assert np.max(np.abs(SF - S2)) < 1e-12
    assert np.max(np.abs(O - np.concatenate([O1, O2], axis=1))) < 1e-12
