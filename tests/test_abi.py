"""The C-ABI library loads and exports every entry point that include/*.h declares (no GPU).

Only calls that need no device are made here: ss1_strerror, and the argument / handle
checks that return before touching CUDA.
"""

import ctypes
import glob
import os
import re

import pytest

from tests.conftest import ROOT


def _declared():
    names = []
    for hdr in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(hdr).read()
        names += re.findall(r"SS1_API\s+[\w\s\*]+?\b(ss1_\w+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from structured_compressed_linear_b200 import build
    build.build()
    from structured_compressed_linear_b200 import ss1
    return ss1.load_library()


def test_header_declares_entry_points():
    names = _declared()
    for need in ("ss1_create", "ss1_forward", "ss1_destroy", "ss1_get_tables", "ss1_strerror"):
        assert need in names


def test_every_declared_symbol_is_exported(lib):
    from structured_compressed_linear_b200 import ss1
    for name in _declared():
        assert hasattr(lib, name), name
        assert name in ss1.SYMBOLS, f"binding does not declare {name}"


def test_strerror(lib):
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -8):
        s = lib.ss1_strerror(code)
        assert isinstance(s, bytes) and len(s) > 0
    assert lib.ss1_strerror(12345) == b"unknown status"


def test_argument_checks_before_device(lib):
    h = ctypes.c_void_p()
    # invalid shapes are rejected before any CUDA call
    assert lib.ss1_create(768, 768, 3, 64, 64, 0, ctypes.byref(h)) == -1      # c not in {1,2,4,8}
    assert lib.ss1_create(768, 768, 2, 512, 64, 0, ctypes.byref(h)) == -1     # BK > 256
    assert lib.ss1_create(770, 768, 2, 64, 64, 0, ctypes.byref(h)) == -1      # K % BK
    assert lib.ss1_create(768, 760, 2, 64, 40, 0, ctypes.byref(h)) == -1      # BN % 16
    assert lib.ss1_create(768, 768, 2, 64, 64, 0, None) == -1
    assert lib.ss1_create(1 << 30, 1 << 20, 1, 256, 16, 0, ctypes.byref(h)) == -1   # > 2^31 table entries
    assert h.value is None
    # null / unknown handles
    assert lib.ss1_forward(None, None, None, None, 1, 0, None) == -7
    assert lib.ss1_destroy(None) == 0
    bogus = ctypes.c_void_p(0x1000)
    assert lib.ss1_get_info(bogus, None, None, None, None, None) == -7
    assert lib.ss1_destroy(bogus) == -7
    assert lib.ss1_test_device_timeout(None, 1000000, None) == -7
    assert lib.ss1_test_device_timeout(bogus, 1000000, None) == -7
    assert lib.ss1_project(None, None, None, 0, None) == -7
    assert lib.ss1_project(bogus, None, None, 0, None) == -7
    assert lib.ss1_backward_workspace(bogus, 1, 0, None, None) == -7
    assert lib.ss1_backward_input(bogus, None, None, None, 1, 0, None, 0, None) == -7
    assert lib.ss1_backward_weight(bogus, None, None, None, 1, 0, None, 0, None) == -7
    assert lib.ss1_forward_fp8(bogus, None, None, None, None, 1, None) == -7
    assert lib.ss1_forward_ex(bogus, None, None, None, 0, None, 1, 0, 0, None) == -7
    hs = (ctypes.c_void_p * 1)(bogus.value)
    f = ctypes.c_int()
    assert lib.ss1_chain_fused(hs, 1, ctypes.byref(f)) == -7
    assert lib.ss1_chain_fused(hs, 5, ctypes.byref(f)) == -1                 # more than SS1_CHAIN_MAX_LAYERS
    assert lib.ss1_chain_forward(None, 1, None, None, None, None, None, 1, None) == -1
    assert lib.ss1_test_forward_timeout(bogus, None, None, None, 1, 1000, None) == -7
    assert lib.ss1_quantize_fp8(None, 0, 4, 8, None, None, None) == -1       # NULL pointers
    assert lib.ss1_quantize_fp8(None, 5, 4, 8, None, None, None) == -1       # dtype
    assert lib.ss1_quantize_fp8(None, 0, 0, 8, None, None, None) == 0        # no rows: nothing to do
    assert lib.ss1_quantize_fp8(0x1001, 0, 4, 8, 0x2000, 0x3000, None) == -5  # Wc not 2-byte aligned
    # the allocation-free forward checks its arguments and its table limit first
    fwd = lib.ss1_forward_noalloc
    assert fwd(768, 768, 3, 64, 64, 0, None, None, None, 1, 0, None, None) == -1         # c
    assert fwd(768, 768, 2, 64, 64, 0, None, None, None, -1, 0, None, None) == -1        # M < 0
    assert fwd(8192, 16384, 2, 128, 128, 0, None, None, None, 1, 0, None, None) == -8    # > table limit
    assert fwd(768, 768, 2, 64, 64, 0, None, None, None, 0, 0, None, None) == 0          # M == 0: no-op
    assert fwd(768, 768, 2, 64, 64, 0, None, None, None, 1, 0, None, None) == -1         # null pointers
    # misaligned pointers are rejected before any device call (the addresses are never touched)
    assert fwd(768, 768, 2, 64, 64, 0, 0x1008, 0x2000, 0x3000, 1, 0, None, None) == -5   # X
    assert fwd(768, 768, 2, 64, 64, 0, 0x1000, 0x2000, 0x3000, 1, 0, 0x4002, None) == -5  # status word


def test_binding_constants_match_header():
    """The binding's enums and limits are the header's (a drift would mis-marshal arguments)."""
    from structured_compressed_linear_b200 import ss1
    text = open(os.path.join(ROOT, "include", "ss1.h")).read()
    consts = {k: int(v) for k, v in re.findall(r"\b(SS1_\w+)\s*=\s*(-?\d+)", text)}
    for k in ss1.Kernel:
        assert consts[f"SS1_KERNEL_{k.name}"] == int(k)
    for d in ss1.DType:
        assert consts[f"SS1_DTYPE_{d.name}"] == int(d)
    m = re.search(r"#define\s+SS1_NOALLOC_MAX_ENTRIES\s+(\d+)", text)
    assert m and int(m.group(1)) == ss1.NOALLOC_MAX_ENTRIES
    for a in ss1.Act:
        assert consts[f"SS1_ACT_{a.name}"] == int(a)
    m = re.search(r"#define\s+SS1_CHAIN_MAX_LAYERS\s+(\d+)", text)
    assert m and int(m.group(1)) == ss1.CHAIN_MAX_LAYERS


def test_plain_c_program_uses_the_abi(lib, tmp_path):
    """The header is plain C99 and a C program links against the library and calls it (no
    torch, no C++): status strings and argument checks, neither of which touches a device."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    src = tmp_path / "use_ss1.c"
    src.write_text(
        '#include <stdio.h>\n#include <string.h>\n#include "ss1.h"\n'
        "int main(void) {\n"
        "  ss1_handle h = 0;\n"
        '  if (strcmp(ss1_strerror(SS1_OK), "ok") != 0) return 1;\n'
        "  if (ss1_create(770, 768, 2, 64, 64, 0, &h) != SS1_ERR_INVALID_ARG || h != 0) return 2;\n"
        "  if (ss1_forward(0, 0, 0, 0, 1, SS1_DTYPE_BF16, 0) != SS1_ERR_BAD_HANDLE) return 3;\n"
        "  ss1_launch_info li;\n"
        "  if (ss1_last_launch(&li) != SS1_OK || li.kernel == 0 || li.kernel[0] != 0) return 4;\n"
        "  if (ss1_last_launch(0) != SS1_ERR_INVALID_ARG) return 5;\n"
        '  printf("c-abi ok %u\\n", (unsigned)sizeof(ss1_launch_info));\n  return 0;\n}\n')
    exe = tmp_path / "use_ss1"
    libdir = os.path.join(ROOT, "structured_compressed_linear_b200")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"), str(src),
                    "-L", libdir, "-lss1", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    from structured_compressed_linear_b200 import ss1
    expect = f"c-abi ok {ctypes.sizeof(ss1._LaunchInfo)}"
    assert out.returncode == 0 and out.stdout.strip() == expect, (out.returncode, out.stdout, out.stderr)


def test_last_launch_before_any_launch(lib):
    """ss1_last_launch is per host thread: a thread that launched nothing reads an empty record."""
    import threading
    from structured_compressed_linear_b200 import ss1
    got = {}

    def probe():
        got["info"] = ss1.last_launch()
    t = threading.Thread(target=probe)
    t.start()
    t.join()
    info = got["info"]
    assert info["kernel"] == "" and info["grid"] == (0, 0) and info["resident_clusters"] == [0] * 17
    assert lib.ss1_last_launch(None) == -1


def test_normal_build_makes_no_index_tests(lib):
    """The normal library reports itself unchecked, with an empty record, and launches no self-test."""
    checked, record = ctypes.c_int(7), ctypes.c_uint64(7)
    assert lib.ss1_bounds_check(ctypes.byref(checked), ctypes.byref(record)) == 0
    assert (checked.value, record.value) == (0, 0)
    assert lib.ss1_bounds_check(None, ctypes.byref(record)) == -1
    assert lib.ss1_test_bounds_check(5, 4) == -8   # SS1_ERR_UNSUPPORTED_SHAPE: nothing launched


def test_checked_build_exports_the_same_entry_points():
    """libss1_checked.so, the bounds-checked debug build of the same sources, has the full ABI."""
    from structured_compressed_linear_b200 import build
    from structured_compressed_linear_b200 import ss1
    path = build.build(checked=True)
    assert path == ss1.CHECKED_LIB_PATH
    clib = ss1.load_library(path)
    for name in _declared():
        assert hasattr(clib, name), name
    record = ctypes.c_uint64(0)
    assert clib.ss1_bounds_check(None, ctypes.byref(record)) == -1


def test_binding_switches_library_and_back():
    """ss1.use_library routes the module's calls through another build; LIB_PATH switches back."""
    from structured_compressed_linear_b200 import build
    from structured_compressed_linear_b200 import ss1
    build.build()
    build.build(checked=True)
    try:
        normal = ss1.use_library(ss1.LIB_PATH)
        assert ss1.bounds_check() == (False, 0)
        checked = ss1.use_library(ss1.CHECKED_LIB_PATH)
        assert checked._name == ss1.CHECKED_LIB_PATH and ss1.lib() is checked
        assert ss1.lib()._name != normal._name
    finally:
        ss1.use_library(ss1.LIB_PATH)
    assert ss1.lib()._name == ss1.LIB_PATH
