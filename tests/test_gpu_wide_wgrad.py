"""Weight gradients on 256 x 512 CTA-pair tiles (two N = 256 MMAs per K
step into one TMEM accumulator), at shapes where those wide tiles are
chosen: long expert segments and enough tiles to fill the SMs.  Checked
against the oracle's plain per-expert products (float64 on the GPU's own
dO_perm, H, dAU and x_perm), with an expert without rows (its tiles write
zeros), and for determinism (two runs give the same bits).

When the last wave of wide tiles would fill at most half of the 74 CTA
pairs, those tiles run as a second launch of 256 x 256 tiles (two per wide
tile).  The cases below cover that for both weight gradients, including N
ending in the first half of the last wide tile (its second half then
writes nothing)."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_39_b200.inputs import custom_config, make_inputs
from mixture_experts_layer_39_b200.layer import MoELayer
from oracle import moe_ref as R
from tests._helpers import assert_close, np64

pytestmark = pytest.mark.gpu

# T, d, f, E, k: at least 4096 routed rows per expert and enough tiles that
# 256 x 512 tiles beat 256 x 256 ones on 74 CTA pairs
CASES = [
    (8192, 2048, 1024, 4, 2),   # wgrad gate/up 128 wide tiles, wgrad down 64: one launch each
    (6144, 2048, 1024, 3, 2),   # wgrad gate/up 96 wide tiles: the last 22 as a narrow launch
    (6144, 1792, 1024, 3, 2),   # as above with N = d = 1792: a half-used last wide tile
    (8192, 3328, 768, 4, 2),    # both weight gradients with a narrow tail, both N ragged
]


def _route(T, E, k, empty, seed):
    """Caller-given expert ids: k distinct experts per token, never `empty`."""
    g = torch.Generator().manual_seed(seed)
    pool = torch.tensor([e for e in range(E) if e != empty], dtype=torch.int32)
    keys = torch.rand((T, len(pool)), generator=g)
    return pool[keys.argsort(dim=1)[:, :k]].contiguous()


def _run(cfg, inp):
    L = MoELayer(cfg.T, cfg.d, cfg.f, cfg.E, cfg.k, device="cuda")
    L.step(inp["x"], inp["w_r"], inp["w_gu"], inp["w_d"], inp["dy"], inp["bias"], inp["route"])
    torch.cuda.synchronize()
    assert L.handle.get_status() == 0
    return L


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T%d_d%d_f%d_E%d_k%d" % c)
@pytest.mark.parametrize("empty", [None, 1])
def test_wide_tile_weight_gradients(cuda_ok, case, empty):
    T, d, f, E, k = case
    cfg = custom_config(T, d, f, E, k, random_routing=True)
    inp = make_inputs(cfg, seed=T + E, device="cuda")
    inp["route"] = _route(T, E, k, empty, seed=E).cuda()
    L = _run(cfg, inp)
    off, cnt = np64(L.offsets).astype(np.int64), np64(L.counts).astype(np.int64)
    if empty is not None:
        assert cnt[empty] == 0
    for e in range(E):
        r0, r1 = off[e], off[e] + cnt[e]
        if r1 == r0:
            assert torch.count_nonzero(L.dw_d[e]) == 0 and torch.count_nonzero(L.dw_gu[e]) == 0
            continue
        dO, hh = np64(L.do_perm[r0:r1]), np64(L.h[r0:r1])
        dau, xp = np64(L.dau[r0:r1]), np64(L.x_perm[r0:r1])
        assert_close(f"dW_d[{e}]", np64(L.dw_d[e]), R.bf16_round(dO.T @ hh))
        assert_close(f"dW_gu[{e}]", np64(L.dw_gu[e]), R.bf16_round(dau.T @ xp))
    # a second run of the same step gives the same bits
    again = _run(cfg, inp)
    assert torch.equal(again.dw_d, L.dw_d) and torch.equal(again.dw_gu, L.dw_gu)
