"""MXFP8 expert GEMMs (E4M3 operands, one E8M0 scale per 32 contraction
elements) against the oracle's MXFP8 emulation, stage by stage on the GPU's
own stage inputs; normwise max relative error within 6e-2.  In this mode
expert segments start at multiples of 128 rows, on both sides."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_39_b200.inputs import CONFIGS, custom_config, make_inputs
from mixture_experts_layer_39_b200.layer import MoELayer
from oracle import moe_ref as R
from oracle import mxfp8_ref as MX
from tests import _helpers as H
from tests._helpers import TOL_MXFP8, assert_close, np64

pytestmark = pytest.mark.gpu


def _run(cfg, g):
    L = MoELayer(cfg.T, cfg.d, cfg.f, cfg.E, cfg.k, device="cuda", dtype="mxfp8")
    L.step(g["x"], g["w_r"], g["w_gu"], g["w_d"], g["dy"], g["bias"], g["route"])
    torch.cuda.synchronize()
    assert L.handle.get_status() == 0
    return L


def _segments(L, E):
    idx = np64(L.idx)
    m = R.routing_metadata(idx, E, align=128)
    np.testing.assert_array_equal(np64(L.counts), m["counts"])
    np.testing.assert_array_equal(np64(L.offsets), m["offsets"])
    np.testing.assert_array_equal(np64(L.row_map), m["row_map"])
    return m


def _edge_inputs(cfg, mode, seed):
    """Inputs of one small case.  Modes:
      random     uniform random expert ids (the workload's routing)
      empty      random ids that never pick expert 1: a zero-count segment,
                 whose weight gradients must come out zero
      skewed     router logits plus a bias that sends most tokens to expert
                 0 and none to experts 1, 3, 5 (dropless: no capacity cap)
      subnormal  random ids; x holds one 32-element row block of bf16
                 subnormals (the row-wise scale takes the exponent clamp at
                 -127) and one column of subnormals (every token-axis block
                 of that column takes it in the weight gradient)"""
    inp = make_inputs(cfg, seed=seed, device="cpu")
    if mode == "empty":
        g = torch.Generator().manual_seed(seed + 1)
        noise = torch.rand(cfg.T, cfg.E, generator=g)
        noise[:, 1] = 2.0  # sorts last, never among the k chosen (k < E)
        inp["route"] = noise.argsort(dim=1)[:, :cfg.k].to(torch.int32).contiguous()
    elif mode == "skewed":
        inp["route"] = None
        inp["bias"] = torch.tensor([4.0, -30.0, 2.0, -30.0, 0.0, -30.0][:cfg.E], dtype=torch.float32)
    elif mode == "subnormal":
        g = torch.Generator().manual_seed(seed + 2)
        x = inp["x"].float()
        t0 = cfg.T // 3
        x[t0, 32:64] = torch.randn(32, generator=g) * 2e-39   # bf16 min normal is 2^-126
        x[:, 7] = torch.randn(cfg.T, generator=g) * 3e-39
        xb = x.to(torch.bfloat16)
        sub = xb[t0, 32:64].float().abs()
        assert (sub < 2.0 ** -126).all() and int((sub > 0).sum()) >= 16
        inp["x"] = xb
    return inp


MX_CASES = [
    # T, d, f, E, k, mode
    (384, 256, 256, 4, 2, "random"),
    (700, 512, 256, 6, 3, "random"),
    (256, 256, 512, 8, 1, "random"),
    (384, 384, 384, 4, 2, "random"),
    (500, 256, 256, 6, 2, "empty"),
    (700, 384, 256, 6, 2, "skewed"),
    (600, 256, 384, 4, 2, "subnormal"),
]


@pytest.mark.parametrize("case", MX_CASES, ids=lambda c: "T%d_d%d_f%d_E%d_k%d_%s" % c)
def test_mxfp8_small_every_stage(cuda_ok, case):
    T, d, f, E, k, mode = case
    cfg = custom_config(T, d, f, E, k, random_routing=(mode != "skewed"), mxfp8=True)
    inp = _edge_inputs(cfg, mode, seed=T + d)
    L = _run(cfg, {n: (v.cuda() if v is not None else None) for n, v in inp.items()})
    m = _segments(L, E)
    if mode in ("empty", "skewed"):
        assert (m["counts"] == 0).any()
        for e in np.flatnonzero(m["counts"] == 0):
            assert torch.count_nonzero(L.dw_gu[e]) == 0 and torch.count_nonzero(L.dw_d[e]) == 0
    if mode == "skewed":
        assert m["counts"].max() > 2 * m["counts"].mean()
    Mp, off, cnt, rm = m["M_pad"], m["offsets"], m["counts"], m["row_map"]
    w_gu, w_d = np64(inp["w_gu"]), np64(inp["w_d"])
    xp = np64(L.x_perm[:Mp])
    np.testing.assert_array_equal(xp, R.permute(np64(inp["x"]), rm, Mp))
    fwd = MX.expert_ffn_fwd_mx(xp, off, cnt, w_gu, w_d, R.bf16_round)
    au, hh = np64(L.au[:Mp]), np64(L.h[:Mp])
    assert_close("AU", au, fwd["AU"], TOL_MXFP8)
    assert_close("H", hh, fwd["H"], TOL_MXFP8)
    # down projection from the GPU's own H
    o_ref = MX.expert_ffn_fwd_mx(xp, off, cnt, w_gu, w_d, R.bf16_round)["O"]
    assert_close("O_perm", np64(L.o_perm[:Mp]), o_ref, TOL_MXFP8)
    Hq = MX.fake_quant(hh, 1)
    o_own = np.zeros_like(o_ref)
    for e in range(E):
        r0, r1 = off[e], off[e] + cnt[e]
        o_own[r0:r1] = R.bf16_round(Hq[r0:r1] @ MX.fake_quant(w_d[e], 1).T)
    assert_close("O_perm (from GPU H)", np64(L.o_perm[:Mp]), o_own, TOL_MXFP8)
    # backward on the GPU's dO, x_perm, AU, H
    dO = np64(L.do_perm[:Mp])
    bwd = MX.expert_ffn_bwd_mx(dO, xp, au, hh, off, cnt, w_gu, w_d, R.bf16_round)
    assert_close("dAU", np64(L.dau[:Mp]), bwd["dAU"], TOL_MXFP8)
    assert_close("dX_perm", np64(L.dx_perm[:Mp]), bwd["dX_perm"], TOL_MXFP8)
    assert_close("dW_d", np64(L.dw_d), bwd["dW_d"], TOL_MXFP8)
    assert_close("dW_gu", np64(L.dw_gu), bwd["dW_gu"], TOL_MXFP8)
    # the rest of the layer is the bf16 path: combine and dx from the GPU's stages
    assert_close("y", np64(L.y), R.combine(np64(L.o_perm[:Mp]), rm, np64(L.w)))


def test_mxfp8_workload_sampled_experts(cuda_ok):
    """The MXFP8 workload (T=32768, d=4096, f=1536, E=128, k=4, uniform random
    expert ids) in the launch configuration the benchmark uses; the MXFP8
    emulation runs on a few experts' segments."""
    cfg = CONFIGS["mxfp8"]
    g = make_inputs(cfg, seed=0, device="cuda")
    L = _run(cfg, g)
    m = _segments(L, cfg.E)
    off, cnt = m["offsets"], m["counts"]
    log0 = len(H.LOG)
    order = np.argsort(cnt, kind="stable")
    pick = sorted({0, cfg.E - 1, int(order[-1]), int(order[0]), int(order[len(order) // 2])})
    for e in pick:
        # the whole padded segment: its pad rows are zero on both sides, and
        # token-axis scale blocks of 32 rows start at the segment start
        r0, r1 = int(off[e]), int(off[e + 1])
        n = r1 - r0
        o1, c1 = np.array([0, n]), np.array([n])
        w_gu, w_d = np64(g["w_gu"][e:e + 1]), np64(g["w_d"][e:e + 1])
        xp = np64(L.x_perm[r0:r1])
        fwd = MX.expert_ffn_fwd_mx(xp, o1, c1, w_gu, w_d, R.bf16_round)
        assert_close(f"AU[{e}]", np64(L.au[r0:r1]), fwd["AU"], TOL_MXFP8)
        assert_close(f"H[{e}]", np64(L.h[r0:r1]), fwd["H"], TOL_MXFP8)
        bwd = MX.expert_ffn_bwd_mx(np64(L.do_perm[r0:r1]), xp, np64(L.au[r0:r1]),
                                   np64(L.h[r0:r1]), o1, c1, w_gu, w_d, R.bf16_round)
        assert_close(f"dAU[{e}]", np64(L.dau[r0:r1]), bwd["dAU"], TOL_MXFP8)
        assert_close(f"dW_d[{e}]", np64(L.dw_d[e]), bwd["dW_d"][0], TOL_MXFP8)
        assert_close(f"dW_gu[{e}]", np64(L.dw_gu[e]), bwd["dW_gu"][0], TOL_MXFP8)
    H.report("full-size mxfp8 (sampled experts)", log0)


def _from_atoms(s, n_mn, n_b):
    """[n_mn, n_b] scale codes read back from the tensor cores' 512-byte atom
    order: 128 MN indices x 4 contraction blocks per atom, atoms consecutive
    along the contraction, and inside an atom byte (r % 32) * 16 +
    ((r / 32) % 4) * 4 + b % 4 (the block-scaled MMA's scale-factor layout
    for 128 rows and K = 128 per atom)."""
    r = np.arange(n_mn)[:, None]
    b = np.arange(n_b)[None, :]
    idx = ((r // 128) * (n_b // 4) + b // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + b % 4
    return s[idx]


@pytest.mark.parametrize("rows,cols,rpg", [(256, 384, 128), (384, 128, 384), (1024, 256, 256),
                                           (8192, 1024, 1024)])
def test_gemm_layout_quantiser_matches_oracle(cuda_ok, rows, cols, rpg):
    """The quantiser the MXFP8 expert calls run (both orientations from one
    read, scales in atom order), code for code against the oracle's codec:
    row-wise blocks along each row, column-wise blocks of 32 rows inside each
    group of rpg rows.  The largest case has more 32 x 128 tiles than the
    grid has blocks, so blocks walk several tiles with the next one in flight."""
    from mixture_experts_layer_39_b200 import ops
    h = ops.Handle(0)
    g = torch.Generator().manual_seed(rows + cols)
    a = torch.randn(rows, cols, generator=g) * torch.exp(torch.randn(rows, 1, generator=g) * 3)
    a = a * torch.exp(torch.randn(1, cols, generator=g) * 2)
    a[3] = 0.0                                               # all-zero blocks both ways
    a[5, :32] = -1e-30
    a[7, 64:96] = 3e4                                        # saturates nothing: scale follows amax
    a[9, 96:128] = torch.randn(32, generator=g) * 2e-39      # bf16 subnormals: scale clamp at -127
    a[:, 1] = torch.randn(rows, generator=g) * 3e-39         # every column block of a column
    a = a.to(torch.bfloat16)
    ad = a.cuda()
    q_row = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    q_col = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    s_row = torch.empty(rows * cols // 32, dtype=torch.uint8, device="cuda")
    s_col = torch.empty(rows * cols // 32, dtype=torch.uint8, device="cuda")
    ops.moe_mxfp8_quantize_gemm(h, ad, rpg, q_row, s_row, q_col, s_col)
    torch.cuda.synchronize()
    assert h.get_status() == 0
    a64 = a.double().numpy()
    qo, so = MX.quantize_blocks(a64, 1)
    np.testing.assert_array_equal(q_row.cpu().numpy(), qo)
    np.testing.assert_array_equal(_from_atoms(s_row.cpu().numpy(), rows, cols // 32), so)
    qc, sc = q_col.cpu().numpy(), s_col.cpu().numpy()
    per = cols * rpg // 32
    for gi in range(rows // rpg):
        qo, so = MX.quantize_blocks(a64[gi * rpg:(gi + 1) * rpg], 0)
        np.testing.assert_array_equal(qc[gi * rpg:(gi + 1) * rpg], qo)
        got = _from_atoms(sc[gi * per:(gi + 1) * per], cols, rpg // 32).T
        np.testing.assert_array_equal(got, so)
