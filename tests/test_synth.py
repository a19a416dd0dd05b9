"""Seeded input generator and host quantisers (CPU only)."""
import numpy as np
import pytest

from quantized_top_routed_b200 import synth
import oracle.qmoe_oracle as O


def test_determinism_and_prefix_stability():
    a = synth.make_layer("tiny", T=16)
    b = synth.make_layer("tiny", T=16)
    np.testing.assert_array_equal(a.x, b.x)
    np.testing.assert_array_equal(a.experts[3].w13, b.experts[3].w13)
    c = synth.make_layer("tiny", T=8)
    np.testing.assert_array_equal(a.x[:8], c.x)          # decode sweep shares token rows
    d = synth.make_layer("tiny", T=16, seed=1)
    assert not np.array_equal(a.x, d.x)


@pytest.mark.parametrize("fmt", [synth.FMT_INT8, synth.FMT_INT4, synth.FMT_FP8])
def test_quantizer_error_bounds(fmt):
    rng = np.random.default_rng(fmt)
    w = (rng.standard_normal((32, 256)) / 16).astype(np.float32)
    w[3] = 0.0                                            # an all-zero row
    q, s = synth.quantize(fmt, w)
    deq = O.dequantize(fmt, q, s, 32, 256)
    assert np.all(deq[3] == 0.0)
    if fmt == synth.FMT_FP8:
        # e4m3 has 3 mantissa bits: relative error <= 2^-4 for normal codes
        big = np.abs(w) > (np.abs(w).max(axis=1, keepdims=True) / 448) * 2.0 ** -6
        rel = np.abs(deq - w)[big] / np.abs(w)[big]
        assert rel.max() <= 2.0 ** -4 + 1e-7
        assert np.abs(deq).max(axis=1)[0] == pytest.approx(np.abs(w).max(axis=1)[0], rel=1e-6)
    else:
        step = np.repeat(O.bf16_to_f64(s), 128, axis=1) if fmt == synth.FMT_INT4 else s[:, None].astype(np.float64)
        qmax = 7 if fmt == synth.FMT_INT4 else 127
        assert np.all(np.abs(deq - w) <= step / 2 * (1 + 1e-6) + np.abs(w) * 2.0 ** -8 * (fmt == synth.FMT_INT4))
        if fmt == synth.FMT_INT8:
            assert np.abs(q).max() == qmax


def test_int4_scale_is_bf16_and_codes_in_range():
    w = np.random.default_rng(0).standard_normal((4, 384)).astype(np.float32)
    q, s = synth.quantize_int4_g128(w)
    assert s.dtype == np.uint16 and s.shape == (4, 3)
    vals = O.unpack_int4(q, 384)
    assert vals.min() >= -7 and vals.max() <= 7


def test_zipf_bias_ranks_experts():
    b = synth.zipf_bias(64, 1.2)
    assert abs(float(b.mean())) < 1e-5
    assert len(set(np.round(b, 6).tolist())) == 64
    assert b.max() - b.min() == pytest.approx(1.2 * np.log(64), rel=1e-5)


def test_mixed_formats():
    L = synth.make_layer("mixed", T=4, d=256, I=128, E=4)
    assert [ex.fmt for ex in L.experts] == [synth.FMT_INT8, synth.FMT_INT8, synth.FMT_INT4, synth.FMT_INT4]
