"""Regression check of the oracle against its stored tiny-workload routing
(written by tests/golden/make_golden.py from the oracle alone)."""
import os

import numpy as np

from mixture_experts_layer_39_b200.inputs import CONFIGS, make_inputs
from oracle import moe_ref as R

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_tiny_routing_fixture():
    rows = {}
    for line in open(os.path.join(HERE, "tiny_routing.txt")):
        if line.startswith("#"):
            continue
        key, *vals = line.split()
        rows[key] = vals
    cfg = CONFIGS["tiny"]
    inp = make_inputs(cfg, seed=0, device="cpu")
    r = R.router_topk(inp["x"].float().numpy(), inp["w_r"].float().numpy(), cfg.k)
    m = R.routing_metadata(r["idx"], cfg.E)
    assert [int(v) for v in rows["counts"]] == m["counts"].tolist()
    assert [int(v) for v in rows["offsets"]] == m["offsets"].tolist()
    first = [[int(v) for v in s.split(",")] for s in rows["idx_first8"]]
    assert first == r["idx"][:8].tolist()
    # top-k margins at the tiny size stay far above fp32 logit error
    assert float(rows["min_topk_margin"][0]) > 1e-4
