"""CPU oracle for the MXFP8 path: the E4M3 / E8M0 codec, blockwise
quantisation, and the MXFP8 emulation of the expert GEMMs.

TEST INFRASTRUCTURE ONLY (same rule as moe_ref: only tests/, smoke() and
bench.py's CPU legs use it; the CUDA path shares nothing with it).

The pages name the format only ("MXFP8 low-precision format for selected
operations; the gains come from the feed-forward network and expert data
movement" -- Olmo-core 3 introduction page, section 3 "MXFP8").  The
definition used here is the public OCP Microscaling (MX) v1.0 one:
  * element E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits; exponent 0
    is subnormal (m/8 * 2^-6); S.1111.111 is NaN; no infinities; largest
    finite 1.75 * 2^8 = 448;
  * scale E8M0: 2^(code - 127), code 255 = NaN;
  * one scale per block of 32 consecutive elements along the GEMM's
    contraction axis;
  * scale exponent = floor(log2(amax)) - 8 (8 = largest E4M3 exponent),
    clamped to [-127, 127]; an all-zero block takes code 0;
  * element = round-to-nearest-even(v / scale), saturated to +-448.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64
E4M3_MAX = 448.0
BLOCK = 32


def e4m3_decode(codes):
    """Value of each E4M3 code (NaN for S.1111.111)."""
    c = np.asarray(codes, np.int64) & 0xFF
    s = np.where(c >> 7, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 7).astype(F64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7.0))
    val = s * mag
    return np.where((e == 15) & ((c & 7) == 7), np.nan, val)


# non-negative finite codes 0x00..0x7E are increasing in value
_POS_CODES = np.arange(0x7F, dtype=np.int64)
_POS_VALS = e4m3_decode(_POS_CODES)


def e4m3_encode(v):
    """Nearest E4M3 code, ties to the even code (even mantissa), values
    beyond the largest finite magnitude saturate to +-448."""
    v = np.asarray(v, F64)
    a = np.minimum(np.abs(v), E4M3_MAX)
    hi = np.searchsorted(_POS_VALS, a, side="left")      # first value >= a
    hi = np.minimum(hi, len(_POS_VALS) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _POS_VALS[lo]
    d_hi = _POS_VALS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (_POS_CODES[hi] % 2 == 0))
    code = np.where(pick_hi, _POS_CODES[hi], _POS_CODES[lo])
    code = np.where(_POS_VALS[hi] == a, _POS_CODES[hi], code)
    sign = (v < 0) | ((v == 0) & np.signbit(v))
    return (code | np.where(sign, 0x80, 0)).astype(np.uint8)


def e8m0_decode(codes):
    c = np.asarray(codes, np.int64)
    return np.where(c == 255, np.nan, 2.0 ** (c - 127.0))


def scale_exponent(amax):
    """floor(log2(amax)) - 8, clamped to [-127, 127]; -127 for amax == 0."""
    amax = np.asarray(amax, F64)
    _, ex = np.frexp(amax)          # amax = m * 2^ex, m in [0.5, 1)
    e = (ex - 1) - 8
    e = np.clip(e, -127, 127)
    return np.where(amax == 0, -127, e).astype(np.int64)


def quantize_blocks(a, axis):
    """Quantise a 2-D array with one scale per 32 consecutive elements
    along `axis` (axis=1: along each row; axis=0: down each column).
    Returns (codes uint8 same shape, scale codes uint8 with that axis
    divided by 32)."""
    a = np.asarray(a, F64)
    if axis == 0:
        q, s = quantize_blocks(a.T, 1)
        return q.T.copy(), s.T.copy()
    R, C = a.shape
    assert C % BLOCK == 0
    blk = a.reshape(R, C // BLOCK, BLOCK)
    amax = np.abs(blk).max(axis=2)
    e = scale_exponent(amax)
    scale = 2.0 ** e.astype(F64)
    q = e4m3_encode(blk / scale[:, :, None]).reshape(R, C)
    return q, (e + 127).astype(np.uint8)


def dequantize_blocks(q, s, axis):
    q = np.asarray(q)
    s = np.asarray(s)
    if axis == 0:
        return dequantize_blocks(q.T, s.T, 1).T.copy()
    R, C = q.shape
    v = e4m3_decode(q).reshape(R, C // BLOCK, BLOCK)
    return (v * e8m0_decode(s)[:, :, None]).reshape(R, C)


def fake_quant(a, axis):
    """Quantise then dequantise (the value an MXFP8 GEMM consumes)."""
    q, s = quantize_blocks(a, axis)
    return dequantize_blocks(q, s, axis)


# --------------------------------------------------------------------------
# MXFP8 emulation of the expert GEMMs.  Every GEMM operand is quantised
# along its own contraction axis; accumulation is in full precision and
# outputs are rounded to bf16 exactly where the bf16 path stores them.
#   forward : x_perm rowwise (K=d), W_gu along d; H rowwise (K=f), W_d along f
#   dgrad   : dO rowwise (K=d), W_d along d; dAU rowwise (K=2f), W_gu along 2f
#   wgrad   : dO, H, dAU, x_perm along tokens in 32-row blocks; expert
#             segments start at multiples of 32 rows, so no block straddles
#             two experts.
# --------------------------------------------------------------------------
def expert_ffn_fwd_mx(x_perm, offsets, counts, w_gu, w_d, rnd):
    from .moe_ref import silu
    x_perm = np.asarray(x_perm, F64)
    M_pad, d = x_perm.shape
    E = len(counts)
    f = w_gu.shape[1] // 2
    xq = fake_quant(x_perm, 1)
    AU = np.zeros((M_pad, 2 * f), F64)
    H = np.zeros((M_pad, f), F64)
    O = np.zeros((M_pad, d), F64)
    for e in range(E):
        r0, r1 = offsets[e], offsets[e] + counts[e]
        if r1 == r0:
            continue
        Wgu = fake_quant(np.asarray(w_gu[e], F64), 1)
        A = xq[r0:r1] @ Wgu[:f].T
        U = xq[r0:r1] @ Wgu[f:].T
        AU[r0:r1, :f] = rnd(A)
        AU[r0:r1, f:] = rnd(U)
        H[r0:r1] = rnd(silu(A) * U)
    Hq = fake_quant(H, 1)
    for e in range(E):
        r0, r1 = offsets[e], offsets[e] + counts[e]
        if r1 == r0:
            continue
        Wd = fake_quant(np.asarray(w_d[e], F64), 1)
        O[r0:r1] = rnd(Hq[r0:r1] @ Wd.T)
    return {"AU": AU, "H": H, "O": O}


def expert_ffn_bwd_mx(dO, x_perm, AU, H, offsets, counts, w_gu, w_d, rnd):
    from .moe_ref import sigmoid
    dO = np.asarray(dO, F64)
    x_perm = np.asarray(x_perm, F64)
    AU = np.asarray(AU, F64)
    H = np.asarray(H, F64)
    E, two_f, d = w_gu.shape
    f = two_f // 2
    M_pad = x_perm.shape[0]
    dO_row = fake_quant(dO, 1)
    dO_col = fake_quant(dO, 0)
    H_col = fake_quant(H, 0)
    X_col = fake_quant(x_perm, 0)
    dAU = np.zeros((M_pad, 2 * f), F64)
    for e in range(E):
        r0, r1 = offsets[e], offsets[e] + counts[e]
        if r1 == r0:
            continue
        Wd_k = fake_quant(np.asarray(w_d[e], F64), 0)     # blocks along d
        dH = dO_row[r0:r1] @ Wd_k
        A = AU[r0:r1, :f]
        U = AU[r0:r1, f:]
        s = sigmoid(A)
        dAU[r0:r1, :f] = rnd(dH * U * s * (1.0 + A * (1.0 - s)))
        dAU[r0:r1, f:] = rnd(dH * A * s)
    dAU_row = fake_quant(dAU, 1)
    dAU_col = fake_quant(dAU, 0)
    dX = np.zeros((M_pad, d), F64)
    dW_gu = np.zeros((E, 2 * f, d), F64)
    dW_d = np.zeros((E, d, f), F64)
    for e in range(E):
        r0, r1 = offsets[e], offsets[e] + counts[e]
        if r1 == r0:
            continue
        Wgu_k = fake_quant(np.asarray(w_gu[e], F64), 0)   # blocks along 2f
        dX[r0:r1] = rnd(dAU_row[r0:r1] @ Wgu_k)
        dW_d[e] = rnd(dO_col[r0:r1].T @ H_col[r0:r1])
        dW_gu[e] = rnd(dAU_col[r0:r1].T @ X_col[r0:r1])
    return {"dAU": dAU, "dX_perm": dX, "dW_gu": dW_gu, "dW_d": dW_d}
