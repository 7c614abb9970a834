"""The C-ABI library loads and exports every entry point include/moe.h
declares; host-only logic runs without a GPU (no compute calls here)."""
import ctypes
import os
import re

import pytest

from mixture_experts_layer_39_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        from mixture_experts_layer_39_b200 import build
        build.build()
    return _lib.load()


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("moe_router_topk", "moe_permute", "moe_grouped_swiglu_fwd", "moe_grouped_swiglu_bwd",
              "moe_unpermute_combine", "moe_mxfp8_quantize"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
        assert n in _lib.SIGNATURES, n


def test_status_strings(lib):
    for code in range(7):
        assert lib.moe_status_string(code)
    assert b"unknown" in lib.moe_status_string(99)


def test_max_rows_and_shape_checks(lib):
    s = _lib.MoeShape(16384, 2048, 1024, 128, 4, 0, 0)
    n = ctypes.c_int64()
    assert lib.moe_max_rows(ctypes.byref(s), ctypes.byref(n)) == 0
    assert n.value == 16384 * 4 + 31 * 128
    bad = [
        _lib.MoeShape(16, 200, 256, 8, 2, 0, 0),     # d not a multiple of 128 -> unsupported
        _lib.MoeShape(16, 256, 320, 8, 2, 0, 0),     # d_ff not a multiple of 128 -> unsupported
        _lib.MoeShape(16, 256, 256, 8, 9, 0, 0),     # k > E -> invalid
        _lib.MoeShape(16, 256, 256, 2048, 2, 0, 0),  # E > 1024 -> unsupported
        _lib.MoeShape(0, 256, 256, 8, 2, 0, 0),      # T = 0 -> invalid
        _lib.MoeShape(16, 256, 256, 8, 2, 7, 0),     # unknown dtype -> invalid
    ]
    want = [2, 2, 1, 2, 1, 1]
    for s_, w in zip(bad, want):
        assert lib.moe_max_rows(ctypes.byref(s_), ctypes.byref(n)) == w
    # multiples of 128 that are not multiples of 256, and any E up to 1024
    for good in [(16, 384, 640, 8, 2), (16, 128, 128, 200, 8), (3, 256, 384, 1024, 8)]:
        s_ = _lib.MoeShape(*good, 0, 0)
        assert lib.moe_max_rows(ctypes.byref(s_), ctypes.byref(n)) == 0


def test_null_handle_rejected_before_any_launch(lib):
    s = _lib.MoeShape(16, 256, 256, 8, 2, 0, 0)
    assert lib.moe_router_topk(None, ctypes.byref(s), *([None] * 9), 0, None) == 1
    assert lib.moe_permute(None, ctypes.byref(s), *([None] * 7), 0, None) == 1
    assert lib.moe_destroy(None) == 1
    h = ctypes.c_void_p()
    assert lib.moe_create(None, 0) == 1


def test_create_without_device_fails_cleanly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    h = ctypes.c_void_p()
    assert lib.moe_create(ctypes.byref(h), 0) != 0
    assert not h.value


def test_max_rows_mxfp8_and_row_limit(lib):
    """MXFP8 segments start at multiples of 128 rows, so the cap is the
    routed rows plus 127 per expert, rounded up to 128; shapes whose cap
    reaches 2^31 rows are refused (row indices are int32)."""
    n = ctypes.c_int64()
    s = _lib.MoeShape(32768, 4096, 1536, 128, 4, 1, 0)
    assert lib.moe_max_rows(ctypes.byref(s), ctypes.byref(n)) == 0
    r = 32768 * 4 + 127 * 128
    assert n.value == (r + 127) // 128 * 128
    s = _lib.MoeShape(3, 128, 128, 5, 2, 1, 0)
    assert lib.moe_max_rows(ctypes.byref(s), ctypes.byref(n)) == 0
    assert n.value == (6 + 127 * 5 + 127) // 128 * 128
    assert n.value % 128 == 0
    s = _lib.MoeShape(1 << 28, 128, 128, 8, 8, 0, 0)   # 2^31 routed rows
    assert lib.moe_max_rows(ctypes.byref(s), ctypes.byref(n)) == 2
    s = _lib.MoeShape((1 << 28) - 64, 128, 128, 8, 8, 0, 0)  # just under the limit
    assert lib.moe_max_rows(ctypes.byref(s), ctypes.byref(n)) == 0
    assert n.value == ((1 << 28) - 64) * 8 + 31 * 8


def test_every_entry_point_is_documented():
    """Each declaration in include/moe.h follows its own comment block
    (macros it defines may sit between the two)."""
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    for m in re.finditer(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text):
        before = text[:m.start()].rstrip().splitlines()
        while before and before[-1].startswith("#define"):
            before.pop()
        assert before and before[-1].rstrip().endswith("*/"), m.group(1)


PAGES = re.compile(r"Olmo-core 3 introduction page|discosf\.com article|vibecoding\.ru news item"
                   r"|bigchange\.ai article")
NO_COUNTERPART = re.compile(r"the pages have no counterpart|The pages describe no such call")


def _blocks():
    """(name, comment block) of every declaration in include/moe.h."""
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    out = []
    for m in re.finditer(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text):
        head = text[:m.start()]
        end = head.rstrip().rfind("*/")
        start = head.rfind("/*", 0, end)
        lines = [ln.strip().lstrip("/*").strip() for ln in head[start:end].splitlines()]
        out.append((m.group(1), " ".join(" ".join(lines).split())))
    return out


def test_every_step_call_cites_its_passage():
    """Each call that runs a step of the layer names the page and section it
    follows; each call with no counterpart on the pages (handle plumbing, the
    no-workspace permute, the wait limit) says so."""
    for name, block in _blocks():
        if NO_COUNTERPART.search(block):
            continue
        assert PAGES.search(block), f"{name}: no page/section cited in its comment block"


def test_binding_checks_dtypes():
    """The binding refuses a tensor whose element type differs from the one
    the header states, before any pointer reaches the library."""
    import torch
    from mixture_experts_layer_39_b200 import ops

    class _H:
        device = 0
    with pytest.raises(TypeError, match="bfloat16"):
        ops._arg(_H(), torch.zeros(4, dtype=torch.float32), ops.BF16, "x")
    with pytest.raises(TypeError, match="int32"):
        ops._arg(_H(), torch.zeros(4, dtype=torch.int64), ops.I32, "topk_idx")
    assert ops._arg(_H(), None, ops.F32, "bias") is None


def test_binding_refuses_strided_and_host_tensors():
    """The binding passes raw pointers; a layout it cannot express is an
    error before any call into the library."""
    import torch
    from mixture_experts_layer_39_b200 import ops
    assert ops._ptr(None) is None
    with pytest.raises(ValueError, match="contiguous"):
        ops._ptr(torch.zeros(4, 6).t())
    with pytest.raises(ValueError, match="contiguous"):
        ops._ptr(torch.zeros(8)[::2])
    with pytest.raises(ValueError, match="CUDA"):
        ops._ptr(torch.zeros(4, 6))
