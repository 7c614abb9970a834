"""Source-level rules, checked on the CPU.

- No bulk or tensor load with cluster multicast. The only multicast is the
  CTA pair's `tcgen05.commit`, which signals mbarriers and moves no data.
- No device-side trap or assert. Bounded waits set a status word instead.
- The oracle and the product path share no code.
- Every ncu command in the profile summaries leaves the GPU clocks alone."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "mixture_experts_layer_39_b200")


def _files(top, exts):
    out = []
    for d, _, names in os.walk(top):
        if "__pycache__" in d:
            continue
        out += [os.path.join(d, n) for n in names if n.endswith(exts)]
    return sorted(out)


def _native_sources():
    return _files(os.path.join(PKG, "csrc"), (".cu", ".cuh", ".h")) + \
        _files(os.path.join(ROOT, "include"), (".h",))


def test_native_sources_exist():
    names = {os.path.basename(p) for p in _native_sources()}
    assert {"tc_gemm.cuh", "gemm.cu", "mxfp8.cu", "permute.cu", "moe.h"} <= names


def test_multicast_only_on_tcgen05_commit():
    for path in _native_sources():
        text = open(path).read()
        for m in re.finditer(r"multicast", text):
            # the PTX instruction string this occurrence belongs to
            start = text.rfind('"', 0, m.start())
            stmt = text[start:m.end()]
            assert "tcgen05.commit" in stmt, f"{path}: multicast outside tcgen05.commit"
            assert "cp.async" not in stmt, path


def test_no_batched_async_copies():
    pat = re.compile(r"Memcpy(3D)?Batch")
    for path in _native_sources() + _files(PKG, (".py",)) + [os.path.join(ROOT, "bench.py")]:
        assert not pat.search(open(path).read()), path


def test_no_device_traps_or_asserts():
    for path in _native_sources():
        text = open(path).read()
        assert "__trap" not in text, path
        assert "asm(\"trap" not in text and "asm volatile(\"trap" not in text, path
        assert not re.search(r"(?<![\w_])assert\s*\(", text), path  # static_assert is fine


def test_product_path_never_imports_the_oracle():
    pat = re.compile(r"^\s*(from|import)\s+oracle\b", re.M)
    for path in _files(PKG, (".py",)):
        assert not pat.search(open(path).read()), path


def test_oracle_imports_nothing_of_the_product():
    pat = re.compile(r"mixture_experts_layer_39_b200|ctypes|libmoe")
    for path in _files(os.path.join(ROOT, "oracle"), (".py",)):
        assert not pat.search(open(path).read()), path


def test_profile_ncu_commands_keep_clock_control_off():
    for path in _files(os.path.join(ROOT, "profiles"), (".md", ".txt")):
        text = open(path).read().replace("\\\n", " ")
        for block in re.findall(r"```(.*?)```", text, re.S):
            for line in block.splitlines():
                if re.match(r"\s*ncu\s", line):
                    assert "--clock-control none" in line, f"{path}: {line.strip()}"
                    assert "\\\\" not in line, f"{path}: doubled line continuation"
