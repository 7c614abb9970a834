"""Gather forms on the GPU (moe_route, moe_grouped_swiglu_*_gather): the
routed copies of x are gathered inside the expert GEMMs with TMA
tile::gather4 loads instead of being written by the permute.  The row index
must equal the oracle's inverse of the row map exactly, and every output
must equal the x_perm forms bit for bit (same rows, same GEMMs); the x_perm
forms are themselves checked against the oracle elsewhere."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_39_b200.inputs import CONFIGS, custom_config, make_inputs
from mixture_experts_layer_39_b200.layer import MoELayer
from oracle import moe_ref as R
from tests._helpers import np64

pytestmark = pytest.mark.gpu

OUTPUTS = ("y", "dx", "dw_gu", "dw_d", "dw_r", "dw")


def _run(cfg, inp, **kw):
    L = MoELayer(cfg.T, cfg.d, cfg.f, cfg.E, cfg.k, device="cuda", **kw)
    L.step(inp["x"], inp["w_r"], inp["w_gu"], inp["w_d"], inp["dy"], inp["bias"], inp["route"])
    torch.cuda.synchronize()
    assert L.handle.get_status() == 0
    return L


CASES = [
    # T, d, f, E, k: single CTAs with 64-row tail tiles (E = 128), CTA pairs,
    # ragged segments, k > 4, one expert
    (512, 256, 512, 8, 4),
    (300, 256, 256, 13, 5),
    (520, 256, 256, 128, 4),
    (3072, 256, 256, 8, 4),
    (2080, 512, 256, 1, 1),
    (1600, 384, 640, 2, 2),          # half-used last N tiles and wgrad M tiles
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T%d_d%d_f%d_E%d_k%d" % c)
@pytest.mark.parametrize("recompute", [False, True])
def test_gather_matches_x_perm_forms(cuda_ok, case, recompute):
    T, d, f, E, k = case
    cfg = custom_config(T, d, f, E, k)
    inp = make_inputs(cfg, seed=T + E + k, device="cuda")
    a = _run(cfg, inp)
    b = _run(cfg, inp, gather=True, recompute=recompute)
    assert b.x_perm is None
    # row_src: the inverse of the row map, T on every other row
    m = R.routing_metadata(np64(b.idx), E)
    ref = np.full(b.M_cap, T, np.int64)
    ref[m["row_map"].reshape(-1)] = np.repeat(np.arange(T), k)
    np.testing.assert_array_equal(np64(b.row_src), ref)
    Mp = int(a.offsets[-1])
    for name in ("au", "h", "o_perm", "dau", "dx_perm"):
        assert torch.equal(getattr(a, name)[:Mp], getattr(b, name)[:Mp]), name
    for name in OUTPUTS:
        assert torch.equal(getattr(a, name), getattr(b, name)), name


@pytest.mark.parametrize("name", ["e8", "e128"])
def test_gather_full_size(cuda_ok, name):
    cfg = CONFIGS[name]
    inp = make_inputs(cfg, seed=0, device="cuda")
    a = _run(cfg, inp)
    b = _run(cfg, inp, gather=True)
    for out in OUTPUTS:
        assert torch.equal(getattr(a, out), getattr(b, out)), out
