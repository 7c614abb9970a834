"""A training step captured as a CUDA graph and replayed gives the same bits
as the same step run eagerly: every entry point launches on the caller's
stream, allocates nothing and never synchronises, so it can be captured."""
import pytest
import torch

from mixture_experts_layer_39_b200.inputs import custom_config, make_inputs
from mixture_experts_layer_39_b200.layer import MoELayer

pytestmark = pytest.mark.gpu

OUTS = ["idx", "w", "probs", "counts", "offsets", "row_map", "y", "dw", "dw_r", "dw_gu", "dw_d",
        "dx"]

CASES = [
    # T, d, f, E, k, extra layer options
    (512, 256, 512, 8, 4, {}),
    (3072, 256, 256, 8, 4, {"shared_ff": 256, "aux_alpha": 0.01}),   # CTA pairs, f2, f3
    (520, 256, 256, 128, 4, {"recompute": True}),                    # tensor-core router, f4
    (1024, 256, 256, 8, 4, {"dtype": "mxfp8"}),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T%d_d%d_f%d_E%d_k%d" % c[:5] + "_" +
                         "_".join(sorted(c[5])))
def test_graph_replay_matches_eager(cuda_ok, case):
    T, d, f, E, k, kw = case
    mx = kw.get("dtype") == "mxfp8"
    cfg = custom_config(T, d, f, E, k, random_routing=mx, mxfp8=mx,
                        shared_ff=kw.get("shared_ff", 0))
    g = make_inputs(cfg, seed=T + E, device="cuda")
    L = MoELayer(T, d, f, E, k, device="cuda", **kw)

    def step():
        L.step(g["x"], g["w_r"], g["w_gu"], g["w_d"], g["dy"], g["bias"], g["route"],
               w_gu_s=g.get("w_gu_s"), w_d_s=g.get("w_d_s"))

    step()
    torch.cuda.synchronize()
    ref = {n: getattr(L, n).clone() for n in OUTS}
    for n in OUTS:
        getattr(L, n).fill_(0) if getattr(L, n).dtype.is_floating_point else getattr(L, n).fill_(-1)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    assert L.handle.get_status() == 0
    for n in OUTS:
        assert torch.equal(getattr(L, n), ref[n]), n
