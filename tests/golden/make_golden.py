"""Writes tiny_routing.txt from the oracle alone (seeded CPU inputs of the
tiny workload).  Run from the repository root:
    python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from mixture_experts_layer_39_b200.inputs import CONFIGS, make_inputs  # noqa: E402
from oracle import moe_ref as R  # noqa: E402


def main():
    cfg = CONFIGS["tiny"]
    inp = make_inputs(cfg, seed=0, device="cpu")
    x = inp["x"].float().numpy()
    w_r = inp["w_r"].float().numpy()
    r = R.router_topk(x, w_r, cfg.k)
    m = R.routing_metadata(r["idx"], cfg.E)
    L = np.sort(r["logits"], axis=1)[:, ::-1]
    margin = float(np.min(L[:, cfg.k - 1] - L[:, cfg.k]))
    with open(os.path.join(HERE, "tiny_routing.txt"), "w") as fh:
        fh.write("# tiny workload, seed 0: oracle routing (fp64 logits)\n")
        fh.write("counts " + " ".join(str(int(c)) for c in m["counts"]) + "\n")
        fh.write("offsets " + " ".join(str(int(o)) for o in m["offsets"]) + "\n")
        fh.write("min_topk_margin %.6e\n" % margin)
        fh.write("idx_first8 " + " ".join(",".join(str(int(v)) for v in row)
                                          for row in r["idx"][:8]) + "\n")


if __name__ == "__main__":
    main()
