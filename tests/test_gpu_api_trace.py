"""A layer step issues kernel launches only: no device-to-host (or any) copy,
no memset, no allocation and no host synchronisation between its first and
last call.  Checked with the CUDA profiler's activity records (CUPTI through
torch.profiler), which see the library's own runtime calls too."""
import json
import os
import tempfile

import pytest
import torch

from mixture_experts_layer_39_b200.inputs import custom_config, make_inputs
from mixture_experts_layer_39_b200.layer import MoELayer

pytestmark = pytest.mark.gpu

FORBIDDEN = ("Synchronize", "cudaMemcpy", "cuMemcpy", "cudaMemset", "cuMemset", "cudaMalloc",
             "cuMemAlloc", "cudaFree", "cuMemFree", "cudaStreamQuery", "cudaEventQuery")


# (T, d, f, E, k): small steps; the last shape's weight gradients run on wide
# tiles with the last wave as an extra launch, which the count must include
SHAPES = {8: (1024, 256, 256, 8, 4), 128: (1024, 256, 256, 128, 4), 3: (6144, 2048, 1024, 3, 2)}


@pytest.mark.parametrize("E,fuse_combine", [(8, False), (128, False), (8, True), (3, False)])
def test_step_has_no_copy_or_sync(cuda_ok, E, fuse_combine):
    from torch.profiler import ProfilerActivity, profile, record_function
    cfg = custom_config(*SHAPES[E])
    g = make_inputs(cfg, seed=5, device="cuda")
    L = MoELayer(cfg.T, cfg.d, cfg.f, cfg.E, cfg.k, device="cuda", fuse_combine=fuse_combine)
    step = lambda: L.step(g["x"], g["w_r"], g["w_gu"], g["w_d"], g["dy"], g["bias"], g["route"])
    step()  # first calls set kernel attributes and load modules
    torch.cuda.synchronize()
    n0 = L.handle.launch_count()
    with profile(activities=[ProfilerActivity.CPU, ProfilerActivity.CUDA]) as prof:
        for i in range(2):
            with record_function(f"moe_step_{i}"):
                step()
        torch.cuda.synchronize()
    launches = (L.handle.launch_count() - n0) // 2
    fd, path = tempfile.mkstemp(suffix=".json")
    os.close(fd)
    try:
        prof.export_chrome_trace(path)
        with open(path) as fh:
            ev = [e for e in json.load(fh).get("traceEvents", []) if e.get("ph") == "X"]
    finally:
        os.unlink(path)
    steps = [e for e in ev if e.get("cat") == "user_annotation"
             and e.get("name", "").startswith("moe_step_")]
    assert len(steps) == 2
    api = [e for e in ev if e.get("cat") in ("cuda_runtime", "cuda_driver")]
    dev = [e for e in ev if e.get("cat") in ("kernel", "gpu_memcpy", "gpu_memset")]
    for s in steps:
        t0, t1 = s["ts"], s["ts"] + s["dur"]
        calls = [e for e in api if t0 <= e["ts"] <= t1]
        bad = [e["name"] for e in calls
               if any(f in e["name"] for f in FORBIDDEN) and "Async" not in e["name"]]
        assert not bad, f"synchronising or copying calls inside a step: {bad}"
        corr = {e.get("args", {}).get("correlation") for e in calls}
        caused = [e for e in dev if e.get("args", {}).get("correlation") in corr]
        assert not [e for e in caused if e["cat"] != "kernel"], "a step copied or set memory"
        n_kernels = sum(1 for e in caused if e["cat"] == "kernel")
        assert n_kernels == launches, (n_kernels, launches)
