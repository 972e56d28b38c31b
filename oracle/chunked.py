"""Chunkwise fp64 form of the gated delta rule -- TEST INFRASTRUCTURE ONLY.

A second, independent CPU implementation used to pin the token recurrence: the
pages state that the chunkwise regrouping is exact for every chunk size
("Linear Attention, Visualized", section "Chunkwise algorithm / Cost").

Written in the row convention of "Linear Attention, Visualized" (state
S in R^{d_k x d_v}, o = q S, tokens are row vectors) and transposed to the
column convention (S in R^{d_v x d_k}) only at the boundary.  Per chunk r it
takes the steps of that page in order:

* "Gated DeltaNet (GDN) / Complete per-chunk algorithm" (scalar gate):
  lambda_r[i:j] = prod_{s=i..j} a_s, Gamma_{C,r}[l,i] = lambda_r[i+1:l] (i <= l),
  left/right-decayed q, k; L_r = (K K^T . Gamma) . M^-; (I + B L) T = B;
  U = T V; W<- = T K<-; Z = U - W<- S; O = Q<- S + (Q K^T . Gamma) Z;
  S_{r+1} = lambda_r[1:C] S + K->^T Z.
* "Kimi Delta Attention (KDA) / Complete per-chunk algorithm" (per-channel
  gate): the same with channelwise products, A_r[l,m] = q_l (lambda[m+1:l] . k_m)^T
  (m <= l), L_r[l,m] = k_l (lambda[m+1:l] . k_m)^T (m < l), and
  S_{r+1} = Diag(lambda_r[1:C]) S + K->^T Z.

The pages assume C divides n; a shorter last chunk uses the same formulas
with C replaced by its length (the regrouping argument does not depend on C).
Decay products are taken literally as products of a = exp(g).
"""
from __future__ import annotations

import numpy as np


def _prod_range(a, i, j):
    """lambda[i:j] = a_i * ... * a_j over 1-based local positions; 1 if i > j."""
    if i > j:
        return np.ones(a.shape[1:], dtype=np.float64) if a.ndim == 2 else 1.0
    return np.prod(a[i - 1:j], axis=0)


def _chunk_step(Qc, Kc, Vc, ac, bc, S):
    """One chunk in row convention. S is d_k x d_v; returns (O_c, S_next)."""
    C = Qc.shape[0]
    per_channel = ac.ndim == 2
    Bm = np.diag(bc)
    # decay products lambda_r[1:l], lambda_r[l+1:C], lambda_r[m+1:l]
    lam_left = [_prod_range(ac, 1, l) for l in range(1, C + 1)]
    lam_right = [_prod_range(ac, l + 1, C) for l in range(1, C + 1)]
    lam_all = _prod_range(ac, 1, C)
    Ql = np.stack([lam_left[l] * Qc[l] for l in range(C)])
    Kl = np.stack([lam_left[l] * Kc[l] for l in range(C)])
    Kr = np.stack([lam_right[l] * Kc[l] for l in range(C)])
    L = np.zeros((C, C))
    A = np.zeros((C, C))
    for l in range(1, C + 1):
        for m in range(1, l + 1):
            lam = _prod_range(ac, m + 1, l)
            if per_channel:
                a_lm = Qc[l - 1] @ (lam * Kc[m - 1])
                l_lm = Kc[l - 1] @ (lam * Kc[m - 1])
            else:
                a_lm = lam * (Qc[l - 1] @ Kc[m - 1])
                l_lm = lam * (Kc[l - 1] @ Kc[m - 1])
            A[l - 1, m - 1] = a_lm
            if m < l:
                L[l - 1, m - 1] = l_lm
    T = np.linalg.solve(np.eye(C) + Bm @ L, Bm)
    U = T @ Vc
    Wl = T @ Kl
    Z = U - Wl @ S
    O = Ql @ S + A @ Z
    if per_channel:
        S_next = lam_all[:, None] * S + Kr.T @ Z
    else:
        S_next = lam_all * S + Kr.T @ Z
    return O, S_next


def chunked_fwd(q, k, v, g, beta, chunk, S0=None, cu_seqlens=None):
    """Chunkwise forward with chunk size ``chunk``; same shapes and return
    values as :func:`oracle.recurrence_fwd` (column-convention states)."""
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        segs = [(b, 0, T) for b in range(B)]
    else:
        cu = [int(x) for x in cu_seqlens]
        segs = [(0, cu[i], cu[i + 1]) for i in range(len(cu) - 1)]
    out = np.zeros((B, T, H, dv))
    S_final = np.zeros((len(segs), H, dv, dk))
    for s, (b, t0, t1) in enumerate(segs):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.asarray(S0[s, h], dtype=np.float64).T.copy()
            for c0 in range(t0, t1, chunk):
                c1 = min(c0 + chunk, t1)
                a = np.exp(g[b, c0:c1, h])
                O, S = _chunk_step(q[b, c0:c1, h], k[b, c0:c1, h], v[b, c0:c1, h], a,
                                   beta[b, c0:c1, h], S)
                out[b, c0:c1, h] = O
            S_final[s, h] = S.T
    return out, S_final


def gdn2_chunked_fwd(q, k, v, g, b, w, S0=None, C=64):
    """Chunkwise Gated DeltaNet-2 in fp64 -- pins :func:`oracle.gdn2_fwd`.

    "Gated DeltaNet-2, and the gate that was doing two jobs", section "What
    decoupling actually means here", in its row convention (S is d_k x d_v,
    o = S^T q).  Inside a chunk the decay is normalised out: with Gamma_t the
    product of the chunk's decays up to t, the keys are scaled by the inverse
    decay (k~ = Gamma_t^-1 k) and the erase vectors by the decay
    (e~ = Gamma_t e), which leaves an undecayed recurrence
    S~_t = (I - k~_t e~_t^T) S~_{t-1} + k~_t z_t^T.  Then T = tril(E~ K~^T, -1),
    A = (I + T)^-1, and the one solve serves both right-hand sides, Y = A E~
    and U = A Z, with the chunk's correction rows U - Y S0.
    Shapes as :func:`oracle.gdn2_fwd` for one batch row set (B sequences of
    length T); returns the column-convention state.
    """
    q, k, v, g, b, w = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, b, w))
    Bn, T, H, dk = q.shape
    dv = v.shape[-1]
    out = np.zeros((Bn, T, H, dv))
    Sf = np.zeros((Bn, H, dv, dk))
    for s in range(Bn):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.array(S0[s, h], dtype=np.float64).T.copy()
            for c0 in range(0, T, C):
                c1 = min(T, c0 + C)
                Kc, Qc, Vc = k[s, c0:c1, h], q[s, c0:c1, h], v[s, c0:c1, h]
                E = b[s, c0:c1, h] * Kc
                Z = w[s, c0:c1, h] * Vc
                a = np.exp(g[s, c0:c1, h])
                if a.ndim == 1:
                    a = np.repeat(a[:, None], dk, axis=1)
                Gam = np.cumprod(a, axis=0)            # Gamma_t, one row per token
                Kt, Et, Qt = Kc / Gam, E * Gam, Qc * Gam
                n = c1 - c0
                Tm = np.tril(Et @ Kt.T, -1)
                A = np.linalg.solve(np.eye(n) + Tm, np.eye(n))
                Y, U = A @ Et, A @ Z
                Ucorr = U - Y @ S                      # rows u_t^T
                out[s, c0:c1, h] = Qt @ S + np.tril(Qt @ Kt.T) @ Ucorr
                S = Gam[-1][:, None] * (S + Kt.T @ Ucorr)
            Sf[s, h] = S.T
    return out, Sf
