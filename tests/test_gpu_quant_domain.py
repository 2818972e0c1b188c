"""The row pass's codes over the whole binary16 range of each row scale, against the oracle.

The row pass computes x / s with a division of its own (a correction of x * RN(1/s)); this test
feeds it rows whose absolute maximum is a chosen binary16 value a and whose other entries are
every binary16 value of magnitude <= a, both signs (values above a are replaced by 0).  The row
scale is then RN(a / 127) and every code of that scale's domain is produced once.  The rows take
every 64th positive binary16 pattern as a, plus the eight patterns at each end of every binade,
the smallest subnormal and the largest finite value.  Codes and scales must equal the oracle's
bit for bit ([P5] "PyTorch 2.9 支持 LLM.int8()", item 2: the activation scale and codes).
"""
import numpy as np
import pytest
import torch

import int8_mixed_precision_absmax_b200 as i8
import oracle
from tests.gpu_helpers import to_dev, to_np

pytestmark = pytest.mark.gpu

POS = np.arange(0, 0x7C00, dtype=np.uint16)  # +0 and every positive finite binary16


def sampled_absmax():
    bits = set(range(64, 0x7C00, 64))
    for e in range(31):
        base = e << 10
        bits.update(b for b in range(base, base + 8) if 0 < b < 0x7C00)
        bits.update(b for b in range(base + 0x3F8, base + 0x400) if 0 < b < 0x7C00)
    bits.update([1, 0x7BFF])
    return np.array(sorted(bits), dtype=np.uint16)


def test_row_pass_codes_every_binade():
    amax_bits = sampled_absmax()
    M, half = len(amax_bits), len(POS)
    K = 2 * half  # 63488, a multiple of 16
    pos = POS.view(np.float16).astype(np.float32)
    X = np.zeros((M, K), np.float16)
    for i, ab in enumerate(amax_bits):
        a = np.float32(np.uint16(ab).view(np.float16))
        row = np.where(pos <= a, pos, 0.0).astype(np.float16)
        X[i, :half] = row
        X[i, half:] = -row
    Xd = to_dev(X)
    ws = i8.new_workspace(M, 1, K, Xd.device)
    Xq, sx, _, n = i8.int8_quantize_rows(Xd, float("inf"), workspace=ws)
    assert int(to_np(n)[0]) == 0
    Xq_ref, sx_ref = oracle.quantize_rows(X, np.zeros((K + 31) // 32, np.uint32))
    np.testing.assert_array_equal(to_np(sx).view(np.uint32), sx_ref.view(np.uint32))
    got = to_np(Xq)
    bad = np.argwhere(got != Xq_ref)
    assert len(bad) == 0, (
        f"{len(bad)} codes differ; first at row {bad[0][0]} (absmax bits "
        f"{int(amax_bits[bad[0][0]]):#06x}), column {bad[0][1]}")
    # the sampled domain reaches every code
    assert set(np.unique(Xq_ref).tolist()) == set(range(-127, 128))
