"""Activation recompute on the GPU: the forward keeps no [A | U], and the
backward's recomputation (moe_grouped_swiglu_recompute) must reproduce the
saved-activation path bit for bit, since it runs the same GEMM on the same
inputs.  That path is itself checked against the oracle elsewhere."""
import pytest
import torch

from mixture_experts_layer_39_b200.inputs import CONFIGS, custom_config, make_inputs
from mixture_experts_layer_39_b200.layer import MoELayer

pytestmark = pytest.mark.gpu

SENTINEL = 0x7FA5  # a bf16 NaN pattern no kernel writes


def _layer(cfg, inp, recompute, dtype="bf16"):
    L = MoELayer(cfg.T, cfg.d, cfg.f, cfg.E, cfg.k, device="cuda", recompute=recompute,
                 dtype=dtype)
    if recompute:
        L.au.view(torch.int16).fill_(SENTINEL)
    L.forward(inp["x"], inp["w_r"], inp["w_gu"], inp["w_d"], inp["bias"], inp["route"])
    torch.cuda.synchronize()
    if recompute:  # the forward did not store [A | U]
        assert bool((L.au.view(torch.int16) == SENTINEL).all())
    L.backward(inp["dy"], inp["x"], inp["w_r"], inp["w_gu"], inp["w_d"])
    torch.cuda.synchronize()
    assert L.handle.get_status() == 0
    return L


CASES = [
    # T, d, f, E, k, dtype
    (512, 256, 512, 8, 4, "bf16"),
    (300, 256, 256, 13, 5, "bf16"),
    (520, 256, 256, 128, 4, "bf16"),
    (1024, 256, 256, 8, 4, "mxfp8"),
    (600, 384, 384, 8, 2, "bf16"),     # half-used last N tiles
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T%d_d%d_f%d_E%d_k%d_%s" % c)
def test_recompute_matches_saved_activations(cuda_ok, case):
    T, d, f, E, k, dtype = case
    cfg = custom_config(T, d, f, E, k)
    inp = make_inputs(cfg, seed=T + E, device="cuda")
    a = _layer(cfg, inp, False, dtype)
    b = _layer(cfg, inp, True, dtype)
    Mp = int(a.offsets[-1])
    assert torch.equal(a.au[:Mp], b.au[:Mp]) and torch.equal(a.h[:Mp], b.h[:Mp])
    for name in ("y", "dx", "dw_gu", "dw_d", "dw_r", "db", "dw"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name


def test_recompute_full_size_e8(cuda_ok):
    cfg = CONFIGS["e8"]
    inp = make_inputs(cfg, seed=0, device="cuda")
    a = _layer(cfg, inp, False)
    b = _layer(cfg, inp, True)
    for name in ("y", "dx", "dw_gu", "dw_d", "dw_r"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
