"""Format facts the GPU kernels rely on, checked on the host against an
independent decoder (ml_dtypes) -- not against the kernels' own code.

* The packed expert banks place element 2j's E2M1 sign|e1 e0 m at bits
  7|3 2 1 of the byte and element 2j+1's at bits 0|6 5 4.  A mask (even
  element) or two shifts (odd element) then give a byte that, read as E5M2,
  is the E2M1 value times 2^-14 -- for all 16 codes, subnormal and zeros
  included.
* E8M0 code c placed in the fp32 exponent field (c << 23) is 2^(c-127) for
  c = 1..254; code 0 gives +0 and code 255 gives +inf (the kernels' documented
  departure from the spec's 2^-127 and NaN).
* An E4M3 hi/lo split carries a bf16 value (the token scaled so that its
  largest magnitude is in [2^7, 2^8)) exactly when the scaled magnitude is
  at least 2^-2, and within 2^-10 below that.
* The MoE gate/up's activation digits: for a block whose largest magnitude
  lies in [2^E, 2^(E+1)), N = round(|v| 2^(15-E)) stays below 2^16, and its
  eight base-4 digits d_p, each an E2M1 code 0..3 (value d/2) with the
  value's sign at scale 2^(E-2p), sum to v exactly when v is within 2^-8 of
  the block's largest and to within 2^(E-16) of it below.
* The MoE down step's h: an fp32 slice scaled by a power of two so that its
  largest magnitude lies in [2^14, 2^15), then hi = f16(v) and
  lo = f16(v - hi) (round to nearest even; v - hi is exact in fp32), gives
  |v - (hi + lo)| <= 2^-8, i.e. 2^-22 of the slice's largest, with no f16
  overflow; and an E2M1 value (as f16) times hi or lo is exact in fp32.
"""
import itertools

import ml_dtypes
import numpy as np
import pytest


def e2m1(code):
    return float(np.array([code], np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)[0])


def e5m2(byte):
    return float(np.array([byte], np.uint8).view(ml_dtypes.float8_e5m2).astype(np.float64)[0])


def relayout(lo, hi):
    """The packer's bit placement of one byte (lo = element 2j, hi = 2j+1)."""
    return ((lo >> 3) << 7) | ((lo & 7) << 1) | (hi >> 3) | ((hi & 7) << 4)


def even_e5m2(byte):
    return byte & 0x8E


def odd_e5m2(byte):
    return ((byte >> 3) & 0x0E) | ((byte << 7) & 0x80)


@pytest.mark.parametrize("lo,hi", list(itertools.product(range(16), range(16))))
def test_packed_nibbles_unpack_to_e5m2(lo, hi):
    b = relayout(lo, hi)
    assert 0 <= b < 256
    # the placement is a bijection on bytes: both codes are recoverable
    assert e5m2(even_e5m2(b)) == e2m1(lo) * 2.0 ** -14
    assert e5m2(odd_e5m2(b)) == e2m1(hi) * 2.0 ** -14


def test_word_level_unpack_keeps_bytes_apart():
    """The 32-bit forms act byte by byte: no bit crosses into a neighbour."""
    rng = np.random.default_rng(0)
    for _ in range(2000):
        codes = rng.integers(0, 16, size=8)
        w = 0
        for j in range(4):
            w |= relayout(int(codes[2 * j]), int(codes[2 * j + 1])) << (8 * j)
        even = w & 0x8E8E8E8E
        odd = ((w >> 3) & 0x0E0E0E0E) | ((w << 7) & 0x80808080)
        for j in range(4):
            assert e5m2((even >> (8 * j)) & 0xFF) == e2m1(int(codes[2 * j])) * 2.0 ** -14
            assert e5m2((odd >> (8 * j)) & 0xFF) == e2m1(int(codes[2 * j + 1])) * 2.0 ** -14


def test_e8m0_by_exponent_placement():
    bits = (np.arange(256, dtype=np.uint64) << 23).astype(np.uint32)
    f = bits.view(np.float32).astype(np.float64)
    for c in range(1, 255):
        assert f[c] == 2.0 ** (c - 127)
    assert f[0] == 0.0 and np.isposinf(f[255])
    # the spec values the kernels depart from: 2^-127 and NaN
    spec = np.array([0, 255], np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    assert spec[0] == 2.0 ** -127 and np.isnan(spec[1])


def test_bf16_is_carried_by_two_e4m3_parts():
    """A bf16 value v, scaled so that the token's largest magnitude is in
    [2^7, 2^8), equals hi + lo (hi = rne_e4m3(v), lo = rne_e4m3(v - hi)) when
    |v| >= 2^-2: 8 significant bits = 4 + 4 with lo's last bit at or above
    E4M3's subnormal step 2^-9.  Below 2^-2 the error is at most half that
    step, 2^-10, under 2^-17 of the token's largest."""
    e4m3 = ml_dtypes.float8_e4m3fn
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]  # drop Inf and NaN codes
    vals = bits.view(ml_dtypes.bfloat16).astype(np.float64)
    vals = vals[np.abs(vals) < 2.0 ** 8]
    hi = vals.astype(np.float32).astype(e4m3).astype(np.float64)
    lo = (vals - hi).astype(np.float32).astype(e4m3).astype(np.float64)
    big = np.abs(vals) >= 2.0 ** -2
    assert np.array_equal((hi + lo)[big], vals[big])
    assert np.abs((hi + lo) - vals)[~big].max() <= 2.0 ** -10
    # the bound is tight: some value just below 2^-2 is not carried exactly
    assert (np.abs((hi + lo) - vals)[~big] > 0).any()


def bf16_values():
    """Every finite bf16 value, as float64."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    v = bits.view(ml_dtypes.bfloat16).astype(np.float64)
    return v[np.isfinite(v)]


@pytest.mark.parametrize("E", [-133, -127, -40, -1, 0, 7, 60, 127])
def test_bf16_is_carried_by_eight_e2m1_digits(E):
    v = bf16_values()
    v = v[np.abs(v) < 2.0 ** (E + 1)]  # every value a block with largest magnitude in [2^E, 2^(E+1)) can hold
    n = np.rint(np.abs(v) * 2.0 ** (15 - E))  # numpy rounds half to even, as the kernel's conversion does
    assert n.max() < 2 ** 16
    n = n.astype(np.int64)
    digits = [(n >> (14 - 2 * p)) & 3 for p in range(8)]
    # each digit is an E2M1 code (0, 0.5, 1, 1.5 for codes 0..3); decode it independently
    total = np.zeros_like(v)
    for p, d in enumerate(digits):
        codes = d.astype(np.uint8) | np.where(v < 0, 8, 0).astype(np.uint8)
        vals = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
        assert np.array_equal(np.abs(vals), d / 2.0)
        total += vals * 2.0 ** (E - 2 * p)
    big = np.abs(v) >= 2.0 ** (E - 8)
    assert np.array_equal(total[big], v[big])
    assert np.all(np.abs(total - v) <= 2.0 ** (E - 16))


def test_h_is_carried_by_two_f16_parts():
    rng = np.random.default_rng(5)
    # scaled slices: the largest magnitude in [2^14, 2^15), the rest spread
    # over 40 binades below it (f16 subnormals included), signs mixed
    top = rng.uniform(2.0 ** 14, 2.0 ** 15, 20000).astype(np.float32)
    rest = (np.float32(2.0) ** rng.uniform(-26, 15, 200000).astype(np.float32)).astype(np.float32)
    edge = np.array([2.0 ** 14, np.nextafter(np.float32(2.0 ** 15), np.float32(0)), 2.0 ** -24, 2.0 ** -25,
                     3 * 2.0 ** -26, 2.0 ** -14, np.nextafter(np.float32(2.0 ** -14), np.float32(0)), 0.0],
                    dtype=np.float32)
    v = np.concatenate([top, rest, edge])
    v = np.where(rng.random(v.size) < 0.5, -v, v).astype(np.float32)
    hi = v.astype(np.float16)
    r = (v - hi.astype(np.float32)).astype(np.float32)
    # the residual is exact: it equals the fp64 difference
    assert np.array_equal(r.astype(np.float64), v.astype(np.float64) - hi.astype(np.float64))
    lo = r.astype(np.float16)
    assert np.isfinite(hi).all() and np.isfinite(lo).all()
    err = np.abs(v.astype(np.float64) - hi.astype(np.float64) - lo.astype(np.float64))
    assert err.max() <= 2.0 ** -8
    # the down MMA's products: E2M1 magnitudes {0.5 .. 6} times any f16 part
    # need at most 11 + 2 significant bits, which fp32 holds exactly
    e2m1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    parts = np.concatenate([hi, lo]).astype(np.float64)
    prod = e2m1[:, None] * parts[None, :]
    assert np.array_equal(prod.astype(np.float32).astype(np.float64), prod)
