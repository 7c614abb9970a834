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


@pytest.mark.parametrize("T,d,f,E,k", [(384, 256, 256, 4, 2), (700, 512, 256, 6, 3),
                                       (256, 256, 512, 8, 1), (384, 384, 384, 4, 2)])
def test_mxfp8_small_every_stage(cuda_ok, T, d, f, E, k):
    cfg = custom_config(T, d, f, E, k, random_routing=True, mxfp8=True)
    inp = make_inputs(cfg, seed=T + d, device="cpu")
    L = _run(cfg, {n: (v.cuda() if v is not None else None) for n, v in inp.items()})
    m = _segments(L, E)
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
    for e in (0, int(np.argmax(cnt)), int(np.argmin(cnt))):
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
