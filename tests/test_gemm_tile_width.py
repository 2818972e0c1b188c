"""The product's tile width, chosen per shape on the host (gemm_tile_width in csrc/gemm.cu).

Compiled from the kernel source with a small host program (nvcc, no GPU needed, 148 SMs as on a
B200).  Checks that every width is a multiple of 16 in [128, 256] (the MMA's N step and the
tile's TMEM columns), and the widths the measurements were taken with: 256 for the 175B-shaped
FFN layer (20.8 waves), 240 for prefill up_proj and 224 for 13B down_proj (the widths that fill
the last wave of the persistent grid).
"""
import subprocess

import pytest

from int8_mixed_precision_absmax_b200 import build as B

PROGRAM = r'''
#include "gemm.cu"
#include <cstdio>
int i8mm::device_sm_count() { return 148; }
int main() {
  const int Ms[] = {17, 128, 129, 1000, 2048, 4096, 8192};
  for (int M : Ms)
    for (int N = 16; N <= 65536; N = N < 1024 ? N + 16 : N + 1000)
      std::printf("%d %d %d\n", M, N, i8mm::gemm_tile_width(M, N));
  std::printf("%d %d %d\n", 2048, 49152, i8mm::gemm_tile_width(2048, 49152));
  std::printf("%d %d %d\n", 2048, 11008, i8mm::gemm_tile_width(2048, 11008));
  std::printf("%d %d %d\n", 4096, 5120, i8mm::gemm_tile_width(4096, 5120));
  return 0;
}
'''


@pytest.fixture(scope="module")
def widths(tmp_path_factory):
    d = tmp_path_factory.mktemp("tilewidth")
    src = d / "tw.cu"
    src.write_text(PROGRAM)
    exe = d / "tw"
    subprocess.check_call([B.nvcc(), *B.ARCH, "-O1", "-std=c++17", "--expt-relaxed-constexpr",
                           "-I", B.INCLUDE, "-I", B.CSRC, str(src), "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout
    return [tuple(int(v) for v in line.split()) for line in out.splitlines()]


def test_widths_are_mma_steps_within_the_tile(widths):
    for M, N, bn in widths:
        assert 128 <= bn <= 256 and bn % 16 == 0, (M, N, bn)


def test_widths_of_the_measured_layers(widths):
    named = {(M, N): bn for M, N, bn in widths[-3:]}
    assert named == {(2048, 49152): 256, (2048, 11008): 240, (4096, 5120): 224}
