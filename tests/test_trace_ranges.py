"""NVTX ranges per C-ABI call.

Every entry point that touches the device (each call that takes a stream,
plus moe_create, moe_destroy and moe_get_status) opens one NVTX range named
for itself and closes it on every return path; the host-only queries open
none.  The ranges are observed through NVTX's own injection interface: a
small recorder library (tests/nvtx_recorder.c) is named in
NVTX_INJECTION64_PATH of a child process, which then calls the library.

The CPU test calls each entry point with a null handle (an argument error
that returns before any CUDA call), so it checks the early-return path; the
GPU test runs a whole forward and backward step and checks that the ranges
seen are exactly the entry points the binding called, in order.
"""
import json
import os
import re
import subprocess
import sys
import textwrap

import pytest

from mixture_experts_layer_39_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_INC = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")

HOST_ONLY = {"moe_workspace_size", "moe_max_rows", "moe_get_launch_count", "moe_set_wait_limit",
             "moe_status_string"}


def _declarations():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(([^;]*?)\);", text, re.S)


def _traced():
    return sorted({n for n, args in _declarations() if "moe_stream_t" in args}
                  | {"moe_create", "moe_destroy", "moe_get_status"})


@pytest.fixture(scope="module")
def recorder(tmp_path_factory):
    if not os.path.exists(os.path.join(CUDA_INC, "nvtx3", "nvToolsExt.h")):
        pytest.skip("NVTX 3 headers not found")
    if not os.path.exists(_lib.LIB_PATH):
        from mixture_experts_layer_39_b200 import build
        build.build()
    out = str(tmp_path_factory.mktemp("nvtx") / "libnvtx_recorder.so")
    subprocess.run(["gcc", "-O1", "-shared", "-fPIC", "-I", CUDA_INC,
                    os.path.join(ROOT, "tests", "nvtx_recorder.c"), "-o", out, "-ldl"],
                   check=True, capture_output=True, text=True)
    return out


def _run_child(recorder, body):
    """Runs `body` in a child process with the recorder injected; `body`
    fills the dict `result`, which comes back as JSON."""
    prelude = textwrap.dedent("""
        import ctypes, json, os, sys
        sys.path.insert(0, {root!r})
        rec = ctypes.CDLL(os.environ["NVTX_INJECTION64_PATH"])
        rec.nvtx_recorder_entry.restype = ctypes.c_char_p
        def ranges():
            return [rec.nvtx_recorder_entry(i).decode()
                    for i in range(rec.nvtx_recorder_count())]
        result = {{}}
    """).format(root=ROOT)
    epilogue = "\nresult['overflow'] = rec.nvtx_recorder_overflow()\nprint(json.dumps(result))\n"
    env = dict(os.environ, NVTX_INJECTION64_PATH=recorder)
    r = subprocess.run([sys.executable, "-c", prelude + textwrap.dedent(body) + epilogue],
                       env=env, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


def test_header_split_covers_every_entry_point():
    names = {n for n, _ in _declarations()}
    assert set(_traced()) | HOST_ONLY == names
    assert not set(_traced()) & HOST_ONLY


def test_each_entry_point_opens_and_closes_its_range(recorder):
    res = _run_child(recorder, """
        from mixture_experts_layer_39_b200 import _lib
        lib = _lib.load()
        def zero(t):
            return 0 if t in (ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_uint64,
                              ctypes.c_float) else None
        for name, types in _lib.SIGNATURES.items():
            if name == "moe_status_string":
                continue
            rec.nvtx_recorder_clear()
            st = getattr(lib, name)(*[zero(t) for t in types])
            result[name] = {"status": st, "ranges": ranges(), "depth": rec.nvtx_recorder_depth()}
    """)
    assert res.pop("overflow") == 0
    traced = set(_traced())
    for name, r in res.items():
        assert r["status"] == 1, (name, r)            # MOE_ERR_INVALID_ARG, before any CUDA call
        expect = ["+" + name, "-"] if name in traced else []
        assert r["ranges"] == expect, (name, r)
        assert r["depth"] == 0, (name, r)
    assert traced <= set(res) | {"moe_status_string"}


@pytest.mark.gpu
def test_ranges_match_the_calls_of_a_layer_step(recorder, cuda_ok):
    res = _run_child(recorder, """
        import torch
        from mixture_experts_layer_39_b200 import ops
        from mixture_experts_layer_39_b200.inputs import CONFIGS, make_inputs
        from mixture_experts_layer_39_b200.layer import MoELayer
        calls = []
        _orig = ops._call
        def _logged(name, *args):
            calls.append(name)
            return _orig(name, *args)
        ops._call = _logged
        cfg = CONFIGS["tiny"]
        g = {k: (v.to("cuda:0") if v is not None else None)
             for k, v in make_inputs(cfg, seed=0, device="cpu").items()}
        L = MoELayer(cfg.T, cfg.d, cfg.f, cfg.E, cfg.k, device="cuda:0")
        torch.cuda.synchronize()
        rec.nvtx_recorder_clear()
        calls.clear()
        for _ in range(2):
            L.step(g["x"], g["w_r"], g["w_gu"], g["w_d"], g["dy"])
        torch.cuda.synchronize()
        result["status"] = L.handle.get_status()
        result["ranges"] = ranges()
        result["calls"] = list(calls)
        result["depth"] = rec.nvtx_recorder_depth()
    """)
    assert res["overflow"] == 0 and res["depth"] == 0
    assert res["status"] == 0
    traced = set(_traced())
    calls = [c for c in res["calls"] if c in traced]
    assert len(calls) >= 8, calls                      # router, permute, GEMMs, combine, backward
    # one range per traced call, in call order, never nested
    assert res["ranges"] == [e for c in calls for e in ("+" + c, "-")]
