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


def np64(t):
    return t.detach().to("cpu").to(torch.float64).numpy() if t.dtype != torch.int32 \
        else t.detach().to("cpu").numpy().astype(np.int64)


def rel_err(g, o):
    g = np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    den = np.max(np.abs(o))
    if den == 0:
        return float(np.max(np.abs(g)))
    return float(np.max(np.abs(g - o)) / den)


def assert_close(name, g, o, tol=TOL_BF16):
    e = rel_err(g, o)
    assert e <= tol, f"{name}: normwise max relative error {e:.3e} > {tol:.1e}"
    return e


def topk_margin(logits, k):
    L = -np.sort(-np.asarray(logits, np.float64), axis=1)
    if k >= L.shape[1]:
        return np.full(L.shape[0], np.inf)
    return L[:, k - 1] - L[:, k]
