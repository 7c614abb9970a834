"""Shared helpers of the parity tests (no arithmetic of the layer here)."""
import numpy as np
import torch

# Tolerances: bf16 outputs, fp32 accumulate -> normwise max relative error
# max|gpu - oracle| / max|oracle| <= 2e-2; MXFP8 operands -> 6e-2.
TOL_BF16 = 2e-2
TOL_MXFP8 = 6e-2
# Selection-parity margin: tokens whose k-th vs (k+1)-th oracle logit gap is
# above this must get identical expert ids from fp32 logits.
TAU = 1e-3
# Elements whose oracle magnitude is at least this fraction of the tensor's
# largest one enter the elementwise relative error (reported beside the
# normwise one; an elementwise ratio means nothing for values near zero).
ELEM_FLOOR = 1e-2

# (name, normwise, elementwise) of every comparison made by assert_close in
# this process, so that a test can print what it checked.
LOG = []


def np64(t):
    return t.detach().to("cpu").to(torch.float64).numpy() if t.dtype != torch.int32 \
        else t.detach().to("cpu").numpy().astype(np.int64)


def rel_err(g, o):
    """Normwise: max_i |g_i - o_i| / max_i |o_i| (the asserted metric)."""
    g = np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    den = np.max(np.abs(o)) if o.size else 0.0
    if den == 0:
        return float(np.max(np.abs(g))) if g.size else 0.0
    return float(np.max(np.abs(g - o)) / den)


def rel_err_elementwise(g, o, floor=ELEM_FLOOR):
    """Elementwise: max_i |g_i - o_i| / |o_i| over the elements with
    |o_i| > floor * max|o| (0 when there are none)."""
    g = np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    if o.size == 0:
        return 0.0
    a = np.abs(o)
    keep = a > floor * a.max()
    if not keep.any():
        return 0.0
    return float(np.max(np.abs(g[keep] - o[keep]) / a[keep]))


def assert_close(name, g, o, tol=TOL_BF16):
    e = rel_err(g, o)
    el = rel_err_elementwise(g, o)
    LOG.append((name, e, el))
    assert e <= tol, (f"{name}: normwise max relative error {e:.3e} > {tol:.1e} "
                      f"(elementwise over |o| > {ELEM_FLOOR:g} max|o|: {el:.3e})")
    return e


def report(title, start=0):
    """Prints the comparisons logged since index `start` (shown with -s or -rA)."""
    print(f"\n{title}: normwise / elementwise max relative error")
    for name, e, el in LOG[start:]:
        print(f"  {name:<28s} {e:.3e}  {el:.3e}")


def topk_margin(logits, k):
    L = -np.sort(-np.asarray(logits, np.float64), axis=1)
    if k >= L.shape[1]:
        return np.full(L.shape[0], np.inf)
    return L[:, k - 1] - L[:, k]
