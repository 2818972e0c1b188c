"""The C-ABI library builds, loads without a GPU and exports every declared entry point.

No compute call is made here: only host-side queries and argument checks that return
before any device work (the pointers passed are never dereferenced).
"""
import ctypes
import math
import os
import re

import pytest

import int8_mixed_precision_absmax_b200 as i8
from int8_mixed_precision_absmax_b200 import build as lib_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "int8mm.h")
FAKE = ctypes.c_void_p(0x10000)  # aligned, never dereferenced: validation fails first


def declared_functions():
    text = open(HEADER, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(int8_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    lib_build.build()
    return i8.load_library()


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("int8_quant_weight", "int8_linear_forward", "int8_linear_workspace_size",
                     "int8_quantize_rows", "int8_gemm_i32", "int8_outlier_weights",
                     "int8_read_device_status", "int8_status_string"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(-11, 1):
        assert i8.int8_status_string(code) not in ("", "unknown status")
    assert i8.int8_status_string(-1234) == "unknown status"


def test_workspace_size_is_worst_case_and_rejects_bad_shapes(lib):
    M, N, K = 2048, 11008, 4096
    ws = i8.int8_linear_workspace_size(M, N, K)
    # at least: Xq (M*K) + fp16 outlier activations (M*K*2) + fp16 outlier weights (N*K*2)
    assert ws >= M * K + 2 * M * K + 2 * N * K
    assert i8.int8_linear_workspace_size(16, 16, 40) == 0      # K % 16 != 0
    assert i8.int8_linear_workspace_size(0, 16, 32) == 0
    assert i8.int8_linear_workspace_size(16, 16, 65536 + 16) == 0


def test_argument_checks_need_no_device(lib):
    L = lib
    null = None
    # NULL pointers
    assert L.int8_linear_forward(null, 4, 32, FAKE, FAKE, null, 8, 6.0, FAKE, FAKE, 1 << 20,
                                 null) == -1
    # shapes
    assert L.int8_linear_forward(FAKE, 0, 32, FAKE, FAKE, null, 8, 6.0, FAKE, FAKE, 1 << 20,
                                 null) == -2
    assert L.int8_linear_forward(FAKE, 4, 40, FAKE, FAKE, null, 8, 6.0, FAKE, FAKE, 1 << 20,
                                 null) == -3
    # misaligned pointer
    assert L.int8_linear_forward(ctypes.c_void_p(0x10002), 4, 32, FAKE, FAKE, null, 8, 6.0, FAKE,
                                 FAKE, 1 << 20, null) == -3
    # NaN threshold
    assert L.int8_linear_forward(FAKE, 4, 32, FAKE, FAKE, null, 8, math.nan, FAKE, FAKE,
                                 1 << 20, null) == -4
    # workspace too small / misaligned
    assert L.int8_linear_forward(FAKE, 4, 32, FAKE, FAKE, null, 8, 6.0, FAKE, FAKE, 16,
                                 null) == -5
    assert L.int8_linear_forward(FAKE, 4, 32, FAKE, FAKE, null, 8, 6.0, FAKE,
                                 ctypes.c_void_p(0x10010), 1 << 20, null) == -5
    assert L.int8_gemm_i32(FAKE, FAKE, 4, 8, 40, FAKE, FAKE, null) == -3
    assert L.int8_gemm_i32(FAKE, FAKE, 4, 8, 32, FAKE, null, null) == -1
    assert L.int8_quant_weight(FAKE, 8, 0, FAKE, FAKE, null) == -2
    assert L.int8_quantize_rows(FAKE, 4, 32, math.nan, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20,
                                null) == -4
    assert L.int8_read_device_status(null, null) == -1


def test_fp16_weight_entry_point_checks_its_weights(lib):
    L = lib
    # the kept fp16 weights are required and must be 16-byte aligned
    assert L.int8_linear_forward_fp16w(FAKE, 4, 32, FAKE, FAKE, None, None, 8, 6.0, FAKE, FAKE,
                                       1 << 20, None) == -1
    assert L.int8_linear_forward_fp16w(FAKE, 4, 32, FAKE, FAKE, ctypes.c_void_p(0x10002), None,
                                       8, 6.0, FAKE, FAKE, 1 << 20, None) == -3
    assert L.int8_linear_forward_fp16w(FAKE, 4, 32, FAKE, FAKE, FAKE, None, 8, math.nan, FAKE,
                                       FAKE, 1 << 20, None) == -4


def test_extended_entry_points_check_their_arguments(lib):
    L = lib
    # unknown flag bits are rejected before anything else
    assert L.int8_linear_forward_ex(FAKE, 4, 32, FAKE, FAKE, None, None, 8, 6.0, 4, FAKE, None,
                                    FAKE, 1 << 20, None) == -11
    assert L.int8_linear_forward_ex(None, 4, 32, FAKE, FAKE, None, None, 8, 6.0, 1, FAKE, None,
                                    FAKE, 1 << 20, None) == -1
    assert L.int8_activation_stats(None, 4, 32, None, FAKE, FAKE, 1 << 20, None) == -1
    assert L.int8_activation_stats(FAKE, 4, 40, None, FAKE, FAKE, 1 << 20, None) == -3
    assert L.int8_activation_stats(FAKE, 4, 32, None, FAKE, FAKE, 16, None) == -5
    assert L.int8_activation_stats_workspace_size() == 32768 * 4
    # the token split's outlier row
    assert L.int8_outlier_row(None, 32, 6.0, FAKE, None) == -1
    assert L.int8_outlier_row(FAKE, 40, 6.0, FAKE, None) == -3
    assert L.int8_outlier_row(FAKE, 32, math.nan, FAKE, None) == -4


def test_remaining_entry_points_check_their_arguments(lib):
    L = lib
    big_k = 65536 + 16  # one 16-column step past the longest supported rows
    assert L.int8_linear_forward(FAKE, 4, big_k, FAKE, FAKE, None, 8, 6.0, FAKE, FAKE, 1 << 30,
                                 None) == -2
    assert L.int8_linear_forward(FAKE, 4, 32, FAKE, FAKE, None, -8, 6.0, FAKE, FAKE, 1 << 20,
                                 None) == -2
    # the two halves of the forward
    assert L.int8_linear_quantize(None, 4, 32, FAKE, FAKE, 8, 6.0, FAKE, 1 << 20, None) == -1
    assert L.int8_linear_quantize(FAKE, 4, 32, FAKE, FAKE, 8, math.nan, FAKE, 1 << 20, None) == -4
    assert L.int8_linear_quantize(FAKE, 0, 32, FAKE, FAKE, 8, 6.0, FAKE, 1 << 20, None) == -2
    assert L.int8_linear_matmul(FAKE, 4, 32, FAKE, FAKE, None, 8, 6.0, None, FAKE, 1 << 20,
                                None) == -1
    assert L.int8_linear_matmul(FAKE, 4, 32, FAKE, FAKE, ctypes.c_void_p(0x10008), 8, 6.0, FAKE,
                                FAKE, 1 << 20, None) == -3
    # the accumulator output is required by the accumulating forward
    assert L.int8_linear_forward_acc(FAKE, 4, 32, FAKE, FAKE, None, 8, 6.0, FAKE, None, FAKE,
                                     1 << 20, None) == -1
    # the outlier-weight diagnostic
    assert L.int8_outlier_weights(FAKE, FAKE, 8, 32, None, FAKE, FAKE, None) == -1
    assert L.int8_outlier_weights(FAKE, FAKE, 8, 40, FAKE, FAKE, FAKE, None) == -3


def test_trace_entry_point_checks_its_arguments(lib):
    L = lib
    # the diagnostic forward: unknown flags, a misaligned output, a short workspace
    assert L.int8_linear_forward_trace(FAKE, 4, 32, FAKE, FAKE, None, None, 8, 6.0, 4, FAKE,
                                       None, None, None, None, None, None, FAKE, 1 << 20,
                                       None) == -11
    assert L.int8_linear_forward_trace(FAKE, 4, 32, FAKE, FAKE, None, None, 8, 6.0, 0, FAKE,
                                       None, ctypes.c_void_p(0x10004), None, None, None, None,
                                       FAKE, 1 << 20, None) == -3
    assert L.int8_linear_forward_trace(FAKE, 4, 32, FAKE, FAKE, None, None, 8, 6.0, 0, FAKE,
                                       None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 64, None) == -5
    assert L.int8_linear_forward_trace(FAKE, 4, 40, FAKE, FAKE, None, None, 8, 6.0, 0, FAKE,
                                       None, None, None, None, None, None, FAKE, 1 << 20,
                                       None) == -3


def test_noalloc_entry_point_checks_before_touching_its_scratch(lib):
    L = lib
    # beyond the few-token kernels the static scratch serves: a clear error, no device work
    assert L.int8_linear_forward_noalloc(FAKE, 17, 256, FAKE, FAKE, None, 128, 6.0, FAKE, None,
                                         None) == -10
    assert L.int8_linear_forward_noalloc(FAKE, 17, 12288, FAKE, FAKE, None, 128, 6.0, FAKE,
                                         None, None) == -10
    assert L.int8_linear_forward_noalloc(None, 8, 256, FAKE, FAKE, None, 128, 6.0, FAKE, None,
                                         None) == -1
    # the optional status word must be 4-byte aligned
    assert L.int8_linear_forward_noalloc(FAKE, 8, 256, FAKE, FAKE, None, 128, 6.0, FAKE,
                                         ctypes.c_void_p(0x10002), None) == -3
    assert L.int8_linear_forward_noalloc(FAKE, 8, 256, FAKE, FAKE, None, 128, math.nan, FAKE,
                                         None, None) == -4


def test_header_is_plain_c_and_links_from_c(lib, tmp_path):
    """The boundary is a C ABI: the header compiles as C99 with -pedantic, and a C program that
    takes the address of every declared entry point links against the library (no C++ names
    or types leak through)."""
    import shutil
    import subprocess

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    names = declared_functions()
    src = tmp_path / "abi.c"
    src.write_text("#include \"int8mm.h\"\n#include <stdio.h>\n"
                   "typedef void (*fn_t)(void);\n"
                   "int main(void) {\n  fn_t fns[] = {\n"
                   + "".join(f"    (fn_t)&{n},\n" for n in names)
                   + "  };\n  printf(\"%d %s\\n\", (int)(sizeof fns / sizeof fns[0]),"
                   " int8_status_string(INT8MM_ERR_SCRATCH));\n  return 0;\n}\n")
    exe = tmp_path / "abi"
    lib_dir = os.path.dirname(i8.library_path())
    subprocess.check_call([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                           "-I", os.path.dirname(HEADER), str(src), "-o", str(exe),
                           "-L", lib_dir, "-l:" + os.path.basename(i8.library_path()),
                           "-Wl,-rpath," + lib_dir])
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    assert int(out[0]) == len(names)
