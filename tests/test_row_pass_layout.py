"""The row pass's launch geometry and shared-memory layout, for every legal row length.

row_pass_smem (csrc/quant.cu) is a host-and-device function: this test compiles quant.cu with a
small host program (nvcc, no GPU needed) and checks, for every K that the library accepts (a
multiple of 16 up to INT8MM_MAX_K): the threads per row are 256, 128, 64 or 32 and divide the
block; no thread owns more than 32 chunks (the width of its register bitmask of outlier chunks);
the regions (mask, prefix, counters, per-warp maxima, column window, row stage) are in order,
disjoint and large enough, the stage 128-byte aligned; the total fits the per-block opt-in of
shared memory and at least one block per SM; and the named-barrier ids stay below 16.
"""
import os
import subprocess

import pytest

from int8_mixed_precision_absmax_b200 import build as B

PROGRAM = r'''
#include "quant.cu"
#include <cstdio>
int i8mm::device_sm_count() { return 148; }
int main() {
  using namespace i8mm;
  for (int K = 16; K <= INT8MM_MAX_K; K += 16) {
    const RowPassSmem L = row_pass_smem(K);
    const int chunks = K / 8, words = (K + 31) / 32;
    std::printf("%d %d %d %d %d %d %d %d %d %d %d %d %d\n", K, chunks, words, L.words, L.tpr,
                L.rpb, L.mask, L.prefix, L.misc, L.red, L.cols, L.stage, L.total);
  }
  std::printf("consts %d %d %d %d\n", kRQThreads, kRQWarps, kGatherCols, kRQBlocksPerSM);
  return 0;
}
'''

SMEM_OPTIN = 227 * 1024          # per block, B200
SMEM_PER_SM = 228 * 1024         # per SM, of which 1 KB is reserved per block
RESERVED = 1024


@pytest.fixture(scope="module")
def layouts(tmp_path_factory):
    d = tmp_path_factory.mktemp("rowpass")
    src = d / "layout.cu"
    src.write_text(PROGRAM)
    exe = d / "layout"
    subprocess.check_call([B.nvcc(), *B.ARCH, "-O1", "-std=c++17", "--expt-relaxed-constexpr",
                           "-I", B.INCLUDE, "-I", B.CSRC, str(src), "-o", str(exe)])
    lines = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.splitlines()
    consts = [int(v) for v in lines[-1].split()[1:]]
    rows = [[int(v) for v in line.split()] for line in lines[:-1]]
    return rows, consts


def test_every_row_length(layouts):
    rows, (threads, warps, gather_cols, blocks_per_sm) = layouts
    assert threads == 256 and warps == 8
    assert len(rows) == 65536 // 16
    for K, chunks, words, lw, tpr, rpb, mask, prefix, misc, red, cols, stage, total in rows:
        assert lw == words
        assert tpr in (256, 128, 64, 32) and tpr * rpb == threads, K
        assert -(-chunks // tpr) <= 32, K                    # the outlier-chunk bitmask
        assert 0 == mask < prefix < misc < red < cols < stage < total, K
        assert prefix - mask >= 4 * words and misc - prefix >= 4 * words, K
        assert red - misc >= 4 * 16, K                       # count + per-warp sums
        assert cols - red >= 4 * 2 * warps, K                # two rows of per-warp maxima
        assert stage - cols >= 4 * gather_cols, K
        assert stage % 128 == 0, K
        assert total - stage == rpb * K * 2, K               # one binary16 row per row slot
        assert total <= SMEM_OPTIN, K
        assert min(blocks_per_sm, SMEM_PER_SM // (total + RESERVED)) >= 1, K
        if tpr >= 64:
            assert rpb <= 15, K                              # named barriers 1 .. rpb


def test_rows_share_a_block_only_while_threads_keep_eight_chunks(layouts):
    rows, _ = layouts
    for K, chunks, *_rest in rows:
        tpr, rpb = _rest[2], _rest[3]
        if rpb > 1:
            assert chunks * rpb <= 256 * 8, K
        if rpb < 8:
            assert chunks * rpb * 2 > 256 * 8, K
