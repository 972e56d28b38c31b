"""Shared test helpers: uploads and the parity metric."""
import numpy as np
import torch


def max_rel_fro(x, ref, lead):
    """Max over slices of ||x - ref||_F / ||ref||_F.

    ``lead`` is the tuple of axes that index the (sequence, head) slices; the
    norm runs over every other axis.  A slice whose reference is zero counts
    with its absolute error."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    axes = tuple(a for a in range(x.ndim) if a not in lead)
    num = np.sqrt(np.sum((x - ref) ** 2, axis=axes))
    den = np.sqrt(np.sum(ref ** 2, axis=axes))
    mask = den > 0
    worst = float(np.max(num[mask] / den[mask])) if mask.any() else 0.0
    if (~mask).any():
        worst = max(worst, float(np.max(num[~mask])))
    return worst


def prefill_out_rel(out, ref, cu=None):
    """Per (sequence, head) relative Frobenius error of out [B,T,H,d_v]."""
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if cu is None:
        return max_rel_fro(out, ref, lead=(0, 2))
    worst = 0.0
    for s in range(len(cu) - 1):
        a, e = int(cu[s]), int(cu[s + 1])
        if e > a:
            worst = max(worst, max_rel_fro(out[:, a:e], ref[:, a:e], lead=(2,)))
    return worst


def state_rel(S, ref):
    return max_rel_fro(S, ref, lead=(0, 1))


def to_dev(x, dtype, device):
    """Upload an fp32 numpy array holding dtype-representable values."""
    if x is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t.to(device)


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)
