"""The unpermute-combine fused into the down projection's epilogue
(moe_permute_src + moe_grouped_swiglu_fwd_combine) against the separate
combine kernel: y must be the same bits, the rest of the step unchanged,
and the arrival counts zero again after every call.  row_src from
moe_permute_src is checked against the oracle's row map."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_39_b200.inputs import CONFIGS, custom_config, make_inputs
from mixture_experts_layer_39_b200.layer import MoELayer
from oracle import moe_ref as R

pytestmark = pytest.mark.gpu

CASES = [
    # T, d, f, E, k, shared_ff
    (3072, 256, 256, 8, 4, 0),     # long segments: CTA-pair tiles
    (300, 256, 256, 4, 2, 0),      # single-CTA tiles, ragged segments
    (500, 384, 256, 7, 2, 0),      # d an odd multiple of 128: a half-used last column tile
    (257, 256, 256, 13, 5, 0),     # k = 5
    (130, 256, 256, 1, 1, 0),      # one expert, k = 1
    (700, 256, 256, 200, 6, 0),    # E = 200
    (1600, 256, 256, 6, 2, 256),   # a shared expert's output joins in the epilogue
    (2048, 512, 256, 8, 8, 0),     # k = 8 = E: every token on every expert
]


def _pair(cfg, shared_ff, seed):
    inp = make_inputs(custom_config(cfg[0], cfg[1], cfg[2], cfg[3], cfg[4], shared_ff=shared_ff),
                      seed=seed, device="cuda")
    T, d, f, E, k = cfg
    a = MoELayer(T, d, f, E, k, device="cuda", shared_ff=shared_ff)
    b = MoELayer(T, d, f, E, k, device="cuda", shared_ff=shared_ff, fuse_combine=True)
    return inp, a, b


def _fwd(L, g):
    return L.forward(g["x"], g["w_r"], g["w_gu"], g["w_d"], g["bias"], g["route"],
                     w_gu_s=g.get("w_gu_s"), w_d_s=g.get("w_d_s"))


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T%d_d%d_f%d_E%d_k%d_s%d" % c)
def test_fused_combine_same_bits(cuda_ok, case):
    T, d, f, E, k, shared_ff = case
    inp, a, b = _pair((T, d, f, E, k), shared_ff, seed=T + E)
    _fwd(a, inp)
    for call in range(2):  # the counts must come back to zero for the next call
        _fwd(b, inp)
        torch.cuda.synchronize()
        assert a.handle.get_status() == 0 and b.handle.get_status() == 0
        assert torch.equal(a.y, b.y), f"call {call}: y differs"
        Mp = int(a.offsets[-1])
        assert torch.equal(a.o_perm[:Mp], b.o_perm[:Mp])
        assert int(torch.count_nonzero(b.arrivals)) == 0, f"call {call}: arrival counts left"
    # row_src: the token of every routed row, T on pad rows
    m = R.routing_metadata(b.idx.cpu().numpy(), E)
    want = np.full(m["M_pad"], T, np.int64)
    rm = m["row_map"]
    for t in range(T):
        want[rm[t]] = t
    np.testing.assert_array_equal(b.row_src[:m["M_pad"]].cpu().numpy(), want)


def test_fused_combine_full_size_e8(cuda_ok):
    """The benchmark's e8 workload: one step each way, y bit for bit, and the
    backward unchanged (dx, dW) since it reads the same O and gate weights."""
    cfg = CONFIGS["e8"]
    g = make_inputs(cfg, seed=0, device="cuda")
    L = [MoELayer(cfg.T, cfg.d, cfg.f, cfg.E, cfg.k, device="cuda", fuse_combine=fc)
         for fc in (False, True)]
    for layer in L:
        layer.step(g["x"], g["w_r"], g["w_gu"], g["w_d"], g["dy"], g["bias"], g["route"])
    torch.cuda.synchronize()
    assert all(layer.handle.get_status() == 0 for layer in L)
    assert torch.equal(L[0].y, L[1].y)
    for name in ("dx", "dw_gu", "dw_d", "dw_r"):
        assert torch.equal(getattr(L[0], name), getattr(L[1], name)), name
    assert int(torch.count_nonzero(L[1].arrivals)) == 0
