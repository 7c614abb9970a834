"""Pins for the oracle's MXFP8 emulation of the expert GEMMs (CPU only).

Each GEMM operand is quantised along its own contraction axis. Build an
operand as small integers (|n| <= 14) times a power of two, where the power
is constant along one axis. Such an operand is exactly representable in
MXFP8 along that axis:
- every 32-block shares one power of two;
- the block's integers fit E4M3 under the block's scale (at most four
  significant bits, and a leading part of at most 1.75, so nothing
  saturates).
Along the other axis the powers spread over 2^-10..2^10, so the small
entries of a block lose bits. Each test asserts this for its operands.

An MXFP8 GEMM whose operands are exact along their contraction axes equals
the unquantised GEMM. So where every operand the emulation quantises is
exact along the right axis, the emulation must equal the plain bf16 oracle
bit for bit. That oracle is pinned against torch and finite differences.
Where an operand is produced inside the layer (H, dAU), the expected value
is that operand from the plain oracle, quantised by the pinned codec along
the axis the GEMM contracts. A wrong axis, a transposed operand (d != f
here) or a wrong segment breaks the equality.
"""
import numpy as np

from oracle import moe_ref as R
from oracle import mxfp8_ref as M

E, D, F = 3, 96, 64
COUNTS = np.array([40, 0, 70])
OFFSETS = np.array([0, 64, 64])  # segments start at multiples of 32 rows
M_PAD = 160


def _live():
    m = np.zeros(M_PAD, bool)
    for o, c in zip(OFFSETS, COUNTS):
        m[o:o + c] = True
    return m


def _exact_along(rng, rows, cols, axis):
    """Integers in [-14, 14] times 2^s, s constant along `axis` (per column
    for axis 0, per row for axis 1)."""
    n = rng.integers(-14, 15, size=(rows, cols)).astype(np.float64)
    if axis == 0:
        return n * 2.0 ** rng.integers(-10, 11, size=(1, cols))
    return n * 2.0 ** rng.integers(-10, 11, size=(rows, 1))


def _stack(rng, rows, cols, axis):
    return np.stack([_exact_along(rng, rows, cols, axis) for _ in range(E)])


def _lossy_along(a, axis):
    return not np.array_equal(M.fake_quant(a, axis), a)


def _segments():
    for e in range(E):
        yield e, OFFSETS[e], OFFSETS[e] + COUNTS[e]


def test_forward_exact_operands():
    rng = np.random.default_rng(11)
    x = _exact_along(rng, M_PAD, D, 1) * _live()[:, None]   # along d: per-row powers
    w_gu = _stack(rng, 2 * F, D, 1)                         # [2f, d] along d
    w_d = _stack(rng, D, F, 1)                              # [d, f] along f
    assert _lossy_along(x, 0) and _lossy_along(w_gu[0], 0) and _lossy_along(w_d[0], 0)
    with np.errstate(over="ignore"):  # silu of a large negative logit: exp overflows to 0
        mx = M.expert_ffn_fwd_mx(x, OFFSETS, COUNTS, w_gu, w_d, R.bf16_round)
        ref = R.expert_ffn_fwd(x, OFFSETS, COUNTS, w_gu, w_d, rnd=R.bf16_round)
    np.testing.assert_array_equal(mx["AU"], ref["AU"])
    np.testing.assert_array_equal(mx["H"], ref["H"])
    Hq = M.fake_quant(ref["H"], 1)                          # H along f
    want = np.zeros_like(ref["O"])
    for e, r0, r1 in _segments():
        want[r0:r1] = R.bf16_round(Hq[r0:r1] @ w_d[e].T)
    np.testing.assert_array_equal(mx["O"], want)
    assert not np.array_equal(mx["O"], ref["O"])            # H's quantisation is seen


def _bwd_inputs(rng, dO_axis, wd_axis, wgu_axis):
    live = _live()[:, None]
    dO = _exact_along(rng, M_PAD, D, dO_axis) * live
    x = _exact_along(rng, M_PAD, D, 0) * live               # along tokens: per-column powers
    H = _exact_along(rng, M_PAD, F, 0) * live
    AU = R.bf16_round(rng.standard_normal((M_PAD, 2 * F))) * live
    w_d = _stack(rng, D, F, wd_axis)
    w_gu = _stack(rng, 2 * F, D, wgu_axis)
    return dO, x, AU, H, w_gu, w_d


def test_dgrad_exact_operands():
    """dO along d, W_d along d, W_gu along 2f: dAU equals the plain oracle's,
    and dX, dW_gu, dW_d consume dAU / dO quantised along their own axes."""
    rng = np.random.default_rng(12)
    dO, x, AU, H, w_gu, w_d = _bwd_inputs(rng, dO_axis=1, wd_axis=0, wgu_axis=0)
    assert _lossy_along(dO, 0) and _lossy_along(w_d[0], 1) and _lossy_along(w_gu[0], 1)
    assert _lossy_along(x, 1) and _lossy_along(H, 1)
    mx = M.expert_ffn_bwd_mx(dO, x, AU, H, OFFSETS, COUNTS, w_gu, w_d, R.bf16_round)
    ref = R.expert_ffn_bwd(dO, x, AU, H, OFFSETS, COUNTS, w_gu, w_d, rnd=R.bf16_round)
    np.testing.assert_array_equal(mx["dAU"], ref["dAU"])
    dau_row = M.fake_quant(ref["dAU"], 1)                   # dgrad gate/up: along 2f
    dau_col = M.fake_quant(ref["dAU"], 0)                   # wgrad gate/up: along tokens
    dO_col = M.fake_quant(dO, 0)                            # wgrad down: along tokens
    dX = np.zeros((M_PAD, D))
    dW_gu = np.zeros((E, 2 * F, D))
    dW_d = np.zeros((E, D, F))
    for e, r0, r1 in _segments():
        if r1 == r0:
            continue
        dX[r0:r1] = R.bf16_round(dau_row[r0:r1] @ w_gu[e])
        dW_gu[e] = R.bf16_round(dau_col[r0:r1].T @ x[r0:r1])
        dW_d[e] = R.bf16_round(dO_col[r0:r1].T @ H[r0:r1])
    np.testing.assert_array_equal(mx["dX_perm"], dX)
    np.testing.assert_array_equal(mx["dW_gu"], dW_gu)
    np.testing.assert_array_equal(mx["dW_d"], dW_d)
    assert not np.any(mx["dW_gu"][1]) and not np.any(mx["dW_d"][1])   # the empty expert


def test_wgrad_exact_operands():
    """dO, H and x along tokens: dW_d equals the plain oracle's bit for bit,
    and dW_gu takes x unquantised."""
    rng = np.random.default_rng(13)
    dO, x, AU, H, w_gu, w_d = _bwd_inputs(rng, dO_axis=0, wd_axis=0, wgu_axis=0)
    assert _lossy_along(dO, 1) and _lossy_along(H, 1) and _lossy_along(x, 1)
    mx = M.expert_ffn_bwd_mx(dO, x, AU, H, OFFSETS, COUNTS, w_gu, w_d, R.bf16_round)
    ref = R.expert_ffn_bwd(dO, x, AU, H, OFFSETS, COUNTS, w_gu, w_d, rnd=R.bf16_round)
    np.testing.assert_array_equal(mx["dW_d"], ref["dW_d"])
    dau_col = M.fake_quant(mx["dAU"], 0)
    for e, r0, r1 in _segments():
        np.testing.assert_array_equal(mx["dW_gu"][e],
                                      R.bf16_round(dau_col[r0:r1].T @ x[r0:r1]))
    # dO is not exact along d here, so dAU must differ from the plain oracle's
    assert not np.array_equal(mx["dAU"], ref["dAU"])
