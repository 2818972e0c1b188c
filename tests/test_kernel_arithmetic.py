"""The arithmetic shortcuts of the CUDA kernels, checked on the CPU against the plain definitions.

The kernels replace a few operations of the layer by cheaper ones that give the same bits.
Each test below restates one shortcut in numpy and compares it, exhaustively or over dense
samples of binary16 inputs, with the definition it stands in for ([P5] "PyTorch 2.9 支持
LLM.int8()" section "LLM.int8() 是怎么做到几乎无损的", item 2: q = round(x / scale) with
scale = absmax / 127; [P2] "8位量化实战：离群值处理与显存优化避坑指南" section 2.3: a column
is an outlier when |x| exceeds the threshold):

* the quantizer (codes.cuh codes8, used by every kernel): the IEEE quotient x / s from one
  correction of x * r, r = 1 / s rounded to nearest (P. Markstein's method: q0 = RN(x r),
  rho = x - q0 s exactly, q1 = RN(q0 + rho r)), the code read off the low byte of
  fl(q1 + 1.5 * 2^23);
* the threshold test on binary16 values against the threshold rounded down to binary16
  (decode.cu);
* int8 codes to float through the bit pattern 0x4B0000vv (decode.cu code_to_float);
* the byte masks that zero the codes of outlier columns (codes.cuh keep_bytes).

None of this imports the CUDA library or the oracle.
"""
import numpy as np
import pytest

F16_POS = np.arange(0x0000, 0x7C00, dtype=np.uint16).view(np.float16)  # 0 and every finite > 0
MAGIC = np.float32(12582912.0)  # 1.5 * 2^23


def _absmax_sample(n_random: int, seed: int) -> np.ndarray:
    """Row maxima: the extremes, powers of two, their neighbours and random binary16 values."""
    rng = np.random.default_rng(seed)
    bits = {0x0001, 0x0002, 0x03FF, 0x0400, 0x0401, 0x3BFF, 0x3C00, 0x3C01, 0x4000, 0x57F0,
            0x5800, 0x7BFE, 0x7BFF}
    bits |= {0x0400 * e for e in range(1, 31)}
    bits |= {0x0400 * e - 1 for e in range(1, 31)}
    bits |= set(rng.integers(1, 0x7C00, size=n_random).tolist())
    return np.array(sorted(bits), dtype=np.uint16).view(np.float16)


def _round_to_f32(hi: np.ndarray, lo: np.ndarray) -> np.ndarray:
    """RN to float32 of the exact sum hi + lo (float64, |lo| <= ulp(hi) / 2, from a two-sum)."""
    f = hi.astype(np.float32)
    f64 = f.astype(np.float64)
    up = np.nextafter(f, np.float32(np.inf)).astype(np.float64)
    down = np.nextafter(f, np.float32(-np.inf)).astype(np.float64)
    # hi exactly halfway between f and a neighbour: the sign of lo decides (lo = 0: ties to even)
    at_mid_up = (hi > f64) & (hi == (f64 + up) / 2)
    at_mid_down = (hi < f64) & (hi == (f64 + down) / 2)
    out = f.copy()
    out = np.where(at_mid_up & (lo > 0), up.astype(np.float32), out)
    out = np.where(at_mid_down & (lo < 0), down.astype(np.float32), out)
    return out


def _corrected_quotient(x: np.ndarray, s: np.float32, r: np.float32) -> np.ndarray:
    """q0 = RN(x r); rho = RN(x - q0 s) (exact when done by one FMA); q1 = RN(q0 + rho r),
    each fused operation emulated exactly in float64 (products of two float32 values have at
    most 48 significant bits; the last sum goes through a two-sum)."""
    x64 = x.astype(np.float64)
    q0 = (x64 * np.float64(r)).astype(np.float32)
    rho = (x64 - q0.astype(np.float64) * np.float64(s)).astype(np.float32)
    p = rho.astype(np.float64) * np.float64(r)
    a = q0.astype(np.float64)
    hi = a + p
    bb = hi - a
    lo = (a - (hi - bb)) + (p - bb)
    return _round_to_f32(hi, lo)


@pytest.mark.parametrize("seed", [0, 1])
def test_corrected_quotient_equals_the_ieee_quotient(seed):
    """For every binary16 x with |x| <= a, over ~300 sampled binary16 row maxima a: Markstein's
    corrected quotient q1 equals fl(x / s) (bit for bit, but for the sign of a zero quotient,
    which no code sees), its codes fit in [-127, 127], and the
    low byte of fl(q1 + 1.5 * 2^23) is the code in two's complement.  rne(x * r) alone, the
    uncorrected product, differs from the code somewhere in the sample."""
    total = wrong_uncorrected = 0
    for a in _absmax_sample(150, seed):
        s = np.float32(a) / np.float32(127.0)          # IEEE float32 division
        r = np.float32(1.0) / s                         # reciprocal rounded to nearest
        x = F16_POS[F16_POS <= a].astype(np.float32)
        x = np.concatenate([x, -x])
        ref = x / s                                     # fl(x / s)
        q1 = _corrected_quotient(x, s, r)
        # equal as values: for x = -0 the correction gives +0 where the quotient is -0
        np.testing.assert_array_equal(q1, ref, err_msg=f"row maximum {float(a)!r}")
        nz = ref != 0
        np.testing.assert_array_equal(q1[nz].view(np.uint32), ref[nz].view(np.uint32))
        code = np.rint(ref.astype(np.float64))
        assert np.abs(code).max() <= 127
        tb = (q1.astype(np.float64) + np.float64(MAGIC)).astype(np.float32)
        low = (tb.view(np.uint32) & 0xFF).astype(np.uint8)
        np.testing.assert_array_equal(low, code.astype(np.int64).astype(np.int8).view(np.uint8))
        total += x.size
        wrong_uncorrected += int((np.rint(x.astype(np.float64) * np.float64(r)) != code).sum())
    assert total > 1_000_000 and wrong_uncorrected > 0


def test_magic_constant_low_byte_for_every_int8_code_and_beyond():
    q = np.arange(-70000, 70001, dtype=np.int64)
    tb = (q.astype(np.float64) + np.float64(MAGIC)).astype(np.float32)
    assert np.array_equal(tb.astype(np.float64) - np.float64(MAGIC), q.astype(np.float64))
    np.testing.assert_array_equal(tb.view(np.uint32) & 0xFF, q & 0xFF)


def _half_round_down(t: float) -> np.float16:
    with np.errstate(over="ignore"):
        h = np.float16(t)
    if np.isnan(h) or (np.isfinite(t) and float(h) > t):
        h = np.nextafter(np.float16(np.inf) if np.isnan(h) else h, np.float16(-np.inf))
    return np.float16(h)


@pytest.mark.parametrize("seed", [0, 1])
def test_threshold_against_its_binary16_round_down(seed):
    """For every binary16 |x|: |x| > t (in float32) exactly when |x| > t rounded down to
    binary16, so the kernels compare binary16 values directly."""
    rng = np.random.default_rng(seed)
    ts = [0.0, 1e-8, 6e-8, 1e-3, 0.5, 1.0, 5.999999523162842, 6.0, 6.000000476837158, 6.001953125,
          6.0009765625, 65504.0, 65519.99609375, 65520.0, 1e6, np.inf]
    ts += rng.uniform(0, 70000, size=300).astype(np.float32).tolist()
    ts += F16_POS[rng.integers(0, F16_POS.size, size=200)].astype(np.float32).tolist()
    ax = F16_POS.astype(np.float64)
    for t in ts:
        t32 = float(np.float32(t))
        h = float(_half_round_down(t32))
        assert h <= t32
        np.testing.assert_array_equal(ax > t32, ax > h, err_msg=f"threshold {t32}")


def test_int8_code_to_float_through_the_0x4b0000vv_pattern():
    """float(code) = float32 bits (0x4B000000 | byte) ^ 0x80, minus 2^23 + 128, for every code."""
    codes = np.arange(-128, 128, dtype=np.int64)
    byte = codes.astype(np.int8).view(np.uint8).astype(np.uint32)
    bits = (np.uint32(0x4B000000) | byte) ^ np.uint32(0x80)
    val = bits.view(np.float32).astype(np.float64) - 8388736.0
    np.testing.assert_array_equal(val, codes.astype(np.float64))


def _keep_mask(bits4: int) -> int:
    return (~((((bits4 * 0x204081) & 0xFFFFFFFF) & 0x01010101) * 0xFF)) & 0xFFFFFFFF


def test_keep_mask_zeroes_exactly_the_outlier_bytes():
    for bits in range(256):
        lo, hi = _keep_mask(bits & 0xF), _keep_mask(bits >> 4)
        word = lo | (hi << 32)
        for e in range(8):
            byte = (word >> (8 * e)) & 0xFF
            assert byte == (0x00 if (bits >> e) & 1 else 0xFF), (bits, e, hex(word))


def test_decode_fragment_columns_are_one_permutation_for_both_operands():
    """decode.cu: in k-step j of a 128-column k-block, lane (g, tig) of a warp feeds the int8 MMA
    m16n8k32 the 8 consecutive columns L = 16 (4 (tig / 2) + j) + 8 (tig % 2) .. L + 7 of weight
    rows g and g + 8 (read through the 128-byte swizzle: 16-byte chunk c of row r sits at
    c ^ (r % 8)) and of token g's codes.  The MMA's k positions tig * 4 .. + 3 and 16 + tig * 4
    .. + 3 then hold the same columns in both operands, so the dot product is unchanged; every
    column of the k-block is used exactly once over the four k-steps; and the 16 lanes of each
    half-warp read 16 different 8-byte bank pairs of the weight tile and of the codes (whose rows
    start 16 bytes apart in bank space: row pitch K + 16 with K a multiple of 128)."""
    used = []
    for j in range(4):
        k_to_col_a, k_to_col_b = {}, {}
        for lane in range(32):
            g, tig = lane >> 2, lane & 3
            L = 16 * (4 * (tig >> 1) + j) + 8 * (tig & 1)
            for r in (g, g + 8):
                for half in range(2):                      # bytes 0-3, then 4-7
                    for e in range(4):
                        k = 16 * half + 4 * tig + e        # the MMA's k position
                        # the weight byte the lane loads: swizzled address back to a column
                        addr = r * 128 + (((4 * (tig >> 1) + j) ^ (r % 8)) << 4) + (tig & 1) * 8 \
                            + 4 * half + e
                        col = (((addr % 128) >> 4) ^ (r % 8)) * 16 + (addr % 16)
                        assert col == L + 4 * half + e
                        assert k_to_col_a.setdefault((r, k), col) == col
                        k_to_col_a[("any", k)] = col
            for half in range(2):
                for e in range(4):
                    k_to_col_b[16 * half + 4 * tig + e] = L + 4 * half + e
        for k, col in k_to_col_b.items():
            assert k_to_col_a[("any", k)] == col      # the same column in both operands
        assert sorted(k_to_col_b.values()) == sorted(set(k_to_col_b.values()))
        used += list(k_to_col_b.values())
    assert sorted(used) == list(range(128))
    for K in (128, 1024, 4096, 8192):
        for j in range(4):
            for half_warp in (range(16), range(16, 32)):
                w_pairs, x_pairs = set(), set()
                for lane in half_warp:
                    g, tig = lane >> 2, lane & 3
                    w_addr = g * 128 + (((4 * (tig >> 1) + j) ^ g) << 4) + (tig & 1) * 8
                    x_addr = g * (K + 16) + 64 * (tig >> 1) + 8 * (tig & 1) + 16 * j
                    w_pairs.add((w_addr // 8) % 16)
                    x_pairs.add((x_addr // 8) % 16)
                assert len(w_pairs) == 16 and len(x_pairs) == 16
