"""Device-side error paths, exercised without faulting the GPU.

1. An expert id outside [0, E) in a caller-written topk_idx: the kernels
   check every id, skip the bad entries (row_map -1, not counted, no row
   written) and record MOE_ERR_DEVICE_CHECK; the call itself succeeds and
   the metadata of the valid entries is exactly the oracle's.
2. A bounded wait that runs out: with the handle's wait limit set to 0 the
   grouped GEMM's main-loop waits give up at once; the kernel drains its own
   copies and MMAs, records MOE_ERR_TIMEOUT and returns.  The context stays
   usable: the same call with the default limit then gives the bits a fresh
   handle gives.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_39_b200 import ops
from mixture_experts_layer_39_b200._lib import MOE_DTYPE_BF16
from oracle import moe_ref as R

pytestmark = pytest.mark.gpu

MOE_ERR_DEVICE_CHECK = 5
MOE_ERR_TIMEOUT = 6


def _ids_with_bad_entries(T, E, k, seed):
    """Distinct ids per token, then one entry in some tokens replaced by an
    id outside [0, E) (E, E + 5, -1, -7).  Returns (ids, mask of bad)."""
    g = torch.Generator().manual_seed(seed)
    idx = torch.rand(T, E, generator=g).argsort(dim=1)[:, :k].to(torch.int32)
    bad = np.zeros((T, k), bool)
    for t, j, v in [(0, 0, E), (3, k - 1, -1), (T // 2, 1 % k, E + 5), (T - 1, k - 1, -7)]:
        idx[t, j] = v
        bad[t, j] = True
    return idx, bad


def _expected(idx, bad, E):
    """The oracle's metadata for the valid entries: the bad entries are given
    to an extra expert E, whose segment comes after all real ones, so the
    real experts' counts, offsets and rows are unchanged by them."""
    io = idx.numpy().astype(np.int64).copy()
    io[bad] = E
    m = R.routing_metadata(io, E + 1)
    rm = m["row_map"].copy()
    rm[bad] = -1
    return m["counts"][:E], m["offsets"][:E + 1], rm, m


@pytest.mark.parametrize("T,d,E,k", [(300, 256, 8, 3), (1000, 384, 128, 4)])
def test_out_of_range_ids_skipped_and_reported(cuda_ok, T, d, E, k):
    h = ops.Handle(0)
    shape = ops.make_shape(T, d, 256, E, k, MOE_DTYPE_BF16)
    M = ops.max_rows(shape)
    ws = torch.empty(h.workspace_size(shape), dtype=torch.uint8, device="cuda")
    g = torch.Generator().manual_seed(T)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16)
    idx, bad = _ids_with_bad_entries(T, E, k, seed=T + E)
    counts = torch.full((E,), -9, dtype=torch.int32, device="cuda")
    offsets = torch.full((E + 1,), -9, dtype=torch.int32, device="cuda")
    row_map = torch.full((T, k), -9, dtype=torch.int32, device="cuda")
    x_perm = torch.full((M, d), 7.0, dtype=torch.bfloat16, device="cuda")
    assert h.get_status() == 0
    ops.moe_permute(h, shape, x.cuda(), idx.cuda(), counts, offsets, row_map, x_perm, ws)
    torch.cuda.synchronize()
    assert h.get_status() == MOE_ERR_DEVICE_CHECK
    assert h.get_status() == 0  # reading the status clears it

    c_ref, o_ref, rm_ref, m = _expected(idx, bad, E)
    np.testing.assert_array_equal(counts.cpu().numpy(), c_ref)
    np.testing.assert_array_equal(offsets.cpu().numpy(), o_ref)
    np.testing.assert_array_equal(row_map.cpu().numpy(), rm_ref)
    assert int(counts.sum()) == T * k - int(bad.sum())
    Mp = int(o_ref[E])
    xp_ref = R.permute(x.double().numpy(), m["row_map"], m["M_pad"])[:Mp]
    np.testing.assert_array_equal(x_perm[:Mp].double().cpu().numpy(), xp_ref)
    # rows past the last real segment were not written
    assert bool((x_perm[Mp:] == 7.0).all())

    # the gather form's row table: the bad entries own no row
    row_src = torch.full((M,), -9, dtype=torch.int32, device="cuda")
    ops.moe_route(h, shape, idx.cuda(), counts, offsets, row_map, row_src, ws)
    torch.cuda.synchronize()
    assert h.get_status() == MOE_ERR_DEVICE_CHECK
    src_ref = np.full(M, T, np.int64)
    for t in range(T):
        for j in range(k):
            if not bad[t, j]:
                src_ref[rm_ref[t, j]] = t
    np.testing.assert_array_equal(row_src.cpu().numpy(), src_ref)
    np.testing.assert_array_equal(row_map.cpu().numpy(), rm_ref)


def _gemm_inputs(T, d, f, E, k, seed):
    """x_perm with segments of the given counts at 32-row offsets (pad rows
    zero), and the expert weights."""
    shape = ops.make_shape(T, d, f, E, k, MOE_DTYPE_BF16)
    M = ops.max_rows(shape)
    counts = np.array([128, 100, 160, 124])[:E]
    assert counts.sum() == T * k
    padded = (counts + 31) // 32 * 32
    offsets = np.concatenate([[0], np.cumsum(padded)]).astype(np.int32)
    g = torch.Generator().manual_seed(seed)
    x_perm = torch.zeros(M, d, dtype=torch.bfloat16)
    for e in range(E):
        x_perm[offsets[e]:offsets[e] + counts[e]] = torch.randn(int(counts[e]), d, generator=g)
    w_gu = (torch.randn(E, 2 * f, d, generator=g) / d ** 0.5).to(torch.bfloat16)
    w_d = (torch.randn(E, d, f, generator=g) / d ** 0.5).to(torch.bfloat16)
    return shape, M, x_perm.cuda(), torch.from_numpy(offsets).cuda(), w_gu.cuda(), w_d.cuda()


def _fwd(h, shape, M, d, f, x_perm, offsets, w_gu, w_d):
    ws = torch.empty(h.workspace_size(shape), dtype=torch.uint8, device="cuda")
    au = torch.zeros(M, 2 * f, dtype=torch.bfloat16, device="cuda")
    hb = torch.zeros(M, f, dtype=torch.bfloat16, device="cuda")
    o = torch.zeros(M, d, dtype=torch.bfloat16, device="cuda")
    ops.moe_grouped_swiglu_fwd(h, shape, x_perm, offsets, w_gu, w_d, au, hb, o, ws)
    return au, hb, o


def test_gemm_wait_limit_runs_out_and_context_survives(cuda_ok):
    # T*k = 512 rows over 4 experts: single-CTA 128-row tiles (no CTA pairs);
    # d = 8192 gives every tile a 128-block main loop, so the epilogue's first
    # test of its accumulator barrier cannot find the tile finished
    T, d, f, E, k = 256, 8192, 256, 4, 2
    shape, M, x_perm, offsets, w_gu, w_d = _gemm_inputs(T, d, f, E, k, seed=3)
    h = ops.Handle(0)
    assert h.get_status() == 0
    h.set_wait_limit(0)
    _fwd(h, shape, M, d, f, x_perm, offsets, w_gu, w_d)
    torch.cuda.synchronize()
    assert h.get_status() == MOE_ERR_TIMEOUT

    # same handle, default limit: a clean run, equal to a fresh handle's bits
    h.set_wait_limit(2_000_000_000)
    got = _fwd(h, shape, M, d, f, x_perm, offsets, w_gu, w_d)
    torch.cuda.synchronize()
    assert h.get_status() == 0
    h2 = ops.Handle(0)
    ref = _fwd(h2, shape, M, d, f, x_perm, offsets, w_gu, w_d)
    torch.cuda.synchronize()
    assert h2.get_status() == 0
    Mp = int(offsets[-1])
    for a, b in zip(got, ref):
        assert torch.equal(a[:Mp], b[:Mp])
    # and the result is the oracle's on one expert (a sanity check that the
    # clean run computed the layer, not only the same bits twice)
    e, r0, n = 1, int(offsets[1]), 100
    ffn = R.expert_ffn_fwd(x_perm[r0:r0 + n].double().cpu().numpy(), np.array([0, n]),
                           np.array([n]), w_gu[e:e + 1].double().cpu().numpy(),
                           w_d[e:e + 1].double().cpu().numpy())
    err = np.abs(got[1][r0:r0 + n].double().cpu().numpy() - ffn["H"]).max() / np.abs(ffn["H"]).max()
    assert err < 2e-2
