"""Pins for the number-format claims the GPU path relies on (no GPU needed):
e4m3 codes are exact in fp16 and in bf16, bf16 activations inside the fp16
normal range are exact in fp16, INT4 codes and INT8 codes are exact in bf16,
so the only rounding the dequantisation adds is the one stated.  INT4 with
token blocks of up to 32 rows: none, because the codes q are the MMA input
and the bf16 group scale, exact in fp32, multiplies each 128-K stage's fp32
partial sum.  INT4 with wider blocks: bf16(q * s)."""
import numpy as np

import oracle.qmoe_oracle as O


def _bf16_bits_to_f32(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


def _is_bf16_exact(v):
    f = np.asarray(v, dtype=np.float32)
    return np.array_equal((f.view(np.uint32) & 0xFFFF), np.zeros(f.shape, dtype=np.uint32))


def test_every_finite_e4m3_code_is_exact_in_fp16_and_bf16():
    codes = np.arange(256, dtype=np.uint8)
    v = O.decode_e4m3(codes)
    finite = np.isfinite(v)
    assert finite.sum() == 254                       # S.1111.111 are the two NaNs
    vf = v[finite]
    assert np.array_equal(vf.astype(np.float16).astype(np.float64), vf)
    assert _is_bf16_exact(vf.astype(np.float32))
    assert np.array_equal(vf.astype(np.float32).astype(np.float64), vf)


def test_bf16_inside_the_fp16_normal_range_is_exact_in_fp16():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 1 << 16, size=200000, dtype=np.uint32)
    bits = bits[(bits & 0x7F80) != 0x7F80]                   # drop inf / NaN patterns
    f = _bf16_bits_to_f32(bits).astype(np.float64)
    inside = np.isfinite(f) & (np.abs(f) >= 2.0 ** -14) & (np.abs(f) <= 65504.0)
    assert inside.sum() > 10000
    g = f[inside]
    assert np.array_equal(g.astype(np.float16).astype(np.float64), g)
    # and the workload's N(0,1) activations lie inside that range (or are exactly 0)
    x = rng.standard_normal(100000).astype(np.float32)
    assert np.all((np.abs(x) < 65504.0))


def test_int4_and_int8_codes_are_exact_in_bf16():
    q4 = np.arange(-8, 8, dtype=np.float32)
    q8 = np.arange(-128, 128, dtype=np.float32)
    assert _is_bf16_exact(q4) and _is_bf16_exact(q8)


def test_bf16_group_scales_are_exact_in_fp32():
    # the per-stage scaling converts the stored bf16 scale to fp32 by a shift
    # of its bits; every bf16 value, subnormals included, is an fp32 value
    bits = np.arange(0, 0x10000, dtype=np.uint32)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]                     # finite values only
    f32 = _bf16_bits_to_f32(bits)
    back = (f32.view(np.uint32) >> 16).astype(np.uint32)
    assert np.array_equal(back, bits)
    assert np.all(f32.astype(np.float64) == f32)


def test_int4_product_rounding_is_within_half_a_bf16_ulp():
    # bf16(q * s) for bf16 scales s (token blocks wider than 32 rows): one RNE
    # rounding to 8 significant bits,
    # relative error <= 2^-8 (the unit roundoff of bf16).  q * s of two bf16
    # values has at most 16 significant bits, so the fp32 step below is exact.
    rng = np.random.default_rng(1)
    s = _bf16_bits_to_f32(rng.integers(0x3800, 0x4000, size=5000, dtype=np.uint32)).astype(np.float64)
    q = rng.integers(-7, 8, size=5000).astype(np.float64)
    exact = q * s
    f32 = exact.astype(np.float32)
    # round to bf16 (RNE) by bit manipulation of the fp32 value
    b = f32.view(np.uint32).astype(np.uint64)
    rounded = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16
    r = rounded.astype(np.uint32).view(np.float32).astype(np.float64)
    nz = exact != 0
    assert np.array_equal(f32.astype(np.float64), exact)          # fp32 holds q * s exactly
    assert np.all(np.abs(r[nz] - exact[nz]) <= np.abs(exact[nz]) * 2.0 ** -8)
