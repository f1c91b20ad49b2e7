"""Pins of the oracle's INT8 KV cache mode (CPU only).

The pages name an INT8 KV cache mode (TinyLoop README, "Python API
reference", KV cache modes) but not its format; the oracle's reading is one
fp32 scale per stored vector (a position's key or value of one kv head),
scale = max|x| / 127, codes = round-half-even(x / scale).  Pinned by:
* worked examples whose scale is a power of two, so every quotient is exact
  and the codes follow from the rounding rule by hand (ties to even);
* the all-zero vector (scale 0, codes 0);
* the error bound |code * scale - x| <= scale / 2 and |code| <= 127, with
  +-127 at the largest magnitude;
* odd symmetry and exact power-of-two scaling;
* the model: cached decode equals the uncached recompute in INT8 mode too,
  and INT8 logits stay within the quantisation's reach of FP16 logits.
Planted mistakes (truncation instead of rounding, a 128 divisor, a scale per
head instead of per position) are each caught by one of these pins.
"""

import numpy as np
import pytest

import tl_synth
from oracle import ref


def test_worked_example_scale_one():
    # max |x| = 127 -> scale 1: codes are the rounded values, ties to even
    x = np.array([[127.0, -63.5, 0.5, 1.5, 2.5, -2.5, 3.49, -127.0]])
    codes, scale = ref.quantize_kv_int8(x)
    assert scale.dtype == np.float32 and scale.tolist() == [1.0]
    assert codes.dtype == np.int8
    assert codes.tolist() == [[127, -64, 0, 2, 2, -2, 3, -127]]


def test_worked_example_power_of_two_scale():
    # max |x| = 127 / 32 -> scale 2^-5; x = (k + 1/2) / 32 are exact ties
    s = 2.0 ** -5
    x = np.array([[127 * s, 0.5 * s, 1.5 * s, -0.5 * s, 10.5 * s, 11.5 * s, -11.5 * s, 0.25 * s]])
    codes, scale = ref.quantize_kv_int8(x)
    assert scale.tolist() == [s]
    assert codes.tolist() == [[127, 0, 2, 0, 10, 12, -12, 0]]
    np.testing.assert_array_equal(ref.dequantize_kv_int8(codes, scale), codes.astype(np.float64) * s)


def test_zero_vector():
    codes, scale = ref.quantize_kv_int8(np.zeros((3, 64)))
    assert scale.tolist() == [0.0, 0.0, 0.0]
    assert not codes.any()
    assert not ref.to_int8_storage(np.zeros((2, 8))).any()


def test_error_bound_and_range():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((500, 128)) * rng.uniform(0.01, 50.0, size=(500, 1))
    codes, scale = ref.quantize_kv_int8(x)
    assert codes.shape == x.shape and scale.shape == (500,)
    assert np.abs(codes.astype(np.int32)).max() <= 127
    err = np.abs(ref.dequantize_kv_int8(codes, scale) - x)
    # half a step plus the float32 rounding of x and of the quotient
    bound = scale[:, None] * (0.5 + 1e-5) + np.abs(x) * 2.0 ** -23
    assert (err <= bound).all()
    # the largest magnitude of every vector maps to +-127
    i = np.argmax(np.abs(x), axis=1)
    assert (np.abs(codes[np.arange(500), i].astype(np.int32)) == 127).all()
    # one scale per vector: every vector uses its own range
    assert np.allclose(scale, np.abs(x).max(axis=1).astype(np.float32) / 127, rtol=1e-6)


def test_symmetry_and_power_of_two_scaling():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((40, 64)).astype(np.float32)
    c, s = ref.quantize_kv_int8(x)
    cn, sn = ref.quantize_kv_int8(-x)
    np.testing.assert_array_equal(cn, -c)
    np.testing.assert_array_equal(sn, s)
    c4, s4 = ref.quantize_kv_int8(x * np.float32(4.0))
    np.testing.assert_array_equal(c4, c)
    np.testing.assert_array_equal(s4, s * np.float32(4.0))


@pytest.fixture(scope="module")
def tiny():
    w = tl_synth.make_model_weights(tl_synth.TINY_LM, tl_synth.SEED_TINY)
    return w, ref.LoopedModel(w, kv_mode="int8"), ref.LoopedModel(w)


def test_int8_cached_decode_equals_recompute(tiny):
    w, om8, _ = tiny
    toks = tl_synth.make_tokens(41, w.shape.vocab, 20)
    cache, logits = om8.prefill(toks[:16], 3)
    np.testing.assert_allclose(logits, om8.score_last(toks[:16], 3), rtol=0, atol=1e-9)
    for i in range(16, 20):
        step = om8.decode(cache, int(toks[i]), 3)
        np.testing.assert_allclose(step, om8.score_last(toks[: i + 1], 3), rtol=0, atol=1e-9)


def test_int8_close_to_fp16(tiny):
    w, om8, om16 = tiny
    toks = tl_synth.make_tokens(43, w.shape.vocab, 24)
    l8, l16 = om8.score_last(toks, 4), om16.score_last(toks, 4)
    d = np.abs(l8 - l16).max()
    # int8 steps are ~max|x| / 254 against fp16's ~|x| / 2048: visibly
    # different, yet small against the logits' own spread
    assert 1e-6 < d < 0.05 * np.abs(l16).max()


def _pins_pass(quant):
    """Run the worked-example and bound pins against a quantiser variant."""
    try:
        x = np.array([[127.0, -63.5, 0.5, 1.5, 2.5, -2.5, 3.49, -127.0]])
        codes, scale = quant(x)
        if codes.tolist() != [[127, -64, 0, 2, 2, -2, 3, -127]] or scale.tolist() != [1.0]:
            return False
        rng = np.random.default_rng(5)
        xr = rng.standard_normal((50, 128)) * rng.uniform(0.01, 50.0, size=(50, 1))
        c, s = quant(xr)
        if s.shape != (50,):
            return False
        i = np.argmax(np.abs(xr), axis=1)
        if not (np.abs(c[np.arange(50), i].astype(np.int32)) == 127).all():
            return False
        err = np.abs(c.astype(np.float64) * s.astype(np.float64)[:, None] - xr)
        return bool((err <= s[:, None] * (0.5 + 1e-5) + np.abs(xr) * 2.0 ** -23).all())
    except Exception:
        return False


def test_planted_mistakes_are_caught():
    assert _pins_pass(ref.quantize_kv_int8)

    def truncating(x):
        x32 = np.asarray(x, np.float32)
        s = (np.abs(x32).max(-1) / np.float32(127)).astype(np.float32)
        return np.trunc(x32 / s[..., None]).astype(np.int8), s

    def divisor_128(x):
        x32 = np.asarray(x, np.float32)
        s = (np.abs(x32).max(-1) / np.float32(128)).astype(np.float32)
        return np.clip(np.rint(x32 / s[..., None]), -127, 127).astype(np.int8), s

    def one_scale_for_all(x):
        x32 = np.asarray(x, np.float32)
        s = np.full(x32.shape[:-1], np.abs(x32).max() / np.float32(127), np.float32)
        return np.rint(x32 / s[..., None]).astype(np.int8), s

    for bad in (truncating, divisor_128, one_scale_for_all):
        assert not _pins_pass(bad), bad.__name__
