"""Pins of the oracle's INT2 body (CPU only).

The pages name an INT2 body (TinyLoop README, "Current Runtime Snapshot": INT2
is the default body) but give no format; the reading is the INT4 storage
with 2-bit fields (element k in bits 2*(k%16) of word k//16, 16 zero points
per word, w = (q - z) * s with q, z in {0..3}).  Pinned by:
* hand-decoded golden words (tests/golden/int2_crumb_order.txt) for the
  decoder and the encoder;
* an encode/decode round trip;
* every (q, z) pair times a set of fp16 scales against exact rationals;
* group indexing where the zero points span several words (K = 5632:
  44 groups, 3 words per row), with one-hot groups;
* the model built on it: looped equals flattened and cached equals
  uncached, as for INT4.
A planted mistake (decoding INT2 words as nibbles, or 2-bit fields highest
first) fails the golden pin.
"""

import os
from fractions import Fraction

import numpy as np

import tl_synth
from oracle import ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "int2_crumb_order.txt")


def _golden():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            rows.append((int(parts[0], 16), [int(v) for v in parts[1:]]))
    assert len(rows) >= 6
    return rows


def test_golden_decode():
    for w, expect in _golden():
        got = ref.unpack_crumbs(np.array([[w]], np.uint32), 16)[0].tolist()
        assert got == expect, hex(w)


def test_golden_encode():
    for w, expect in _golden():
        assert int(tl_synth.pack_crumbs(np.array([expect], np.uint8))[0, 0]) == w, hex(w)


def test_round_trip():
    rng = np.random.default_rng(3)
    v = rng.integers(0, 4, size=(7, 300), dtype=np.uint8)
    np.testing.assert_array_equal(ref.unpack_crumbs(tl_synth.pack_crumbs(v), 300), v)


def test_exhaustive_pairs_exact():
    # row r holds the pair (q, z) = (r // 4, r % 4) in every element of one
    # group; scales are exact fp16 values of several binades
    scales = np.array([0.02, 0.0498, 0.0625, 0.07998, 1.0, 3.0e-5], dtype=np.float16)
    K = 128
    q = np.array([[r // 4] * K for r in range(16)], np.uint8)
    z = np.array([[r % 4] for r in range(16)], np.uint8)
    for s in scales:
        S = np.full((16, 1), s, np.float16)
        W = ref.dequantize_int2(tl_synth.pack_crumbs(q), S, tl_synth.pack_crumbs(z), K)
        for r in range(16):
            exact = (Fraction(r // 4) - Fraction(r % 4)) * Fraction(float(s))
            assert all(Fraction(float(v)) == exact for v in W[r]), (r, float(s))


def test_group_indexing_many_words():
    K, N = 5632, 3
    G = K // 128
    rng = np.random.default_rng(11)
    z = rng.integers(0, 4, size=(N, G), dtype=np.uint8)
    q = np.repeat(z, 128, axis=1).copy()          # q == z: every weight is 0
    hot = [0, 17, 43]                             # one group per row differs
    for r, g in enumerate(hot):
        q[r, g * 128:(g + 1) * 128] = (z[r, g] + 1) % 4
    s = rng.uniform(0.02, 0.08, size=(N, G)).astype(np.float16)
    W = ref.dequantize_int2(tl_synth.pack_crumbs(q), s, tl_synth.pack_crumbs(z), K)
    assert tl_synth.pack_crumbs(z).shape == (N, 3)
    for r, g in enumerate(hot):
        nz = np.nonzero(W[r])[0]
        assert nz.min() == g * 128 and nz.max() == g * 128 + 127, r
        d = ((int(z[r, g]) + 1) % 4) - int(z[r, g])
        np.testing.assert_array_equal(W[r, nz], d * s[r, g].astype(np.float64))


def test_int2_model_structure():
    w = tl_synth.make_model_weights(tl_synth.TINY_LM, tl_synth.SEED_TINY, bits=2)
    assert w.loop.qkv.bits == 2 and w.loop.qkv.qweight.shape[1] == w.shape.d_model // 16
    om = ref.LoopedModel(w)
    toks = tl_synth.make_tokens(51, w.shape.vocab, 14)
    # looped with L = 3 equals the flattened stack of the same blocks
    flat = om.blocks(3)
    h1 = om.forward(toks, 3)
    h2 = om.forward_stack(toks, flat)
    np.testing.assert_array_equal(h1, h2)
    # cached decode equals the uncached recompute
    cache, _ = om.prefill(toks[:10], 3)
    for i in range(10, 14):
        np.testing.assert_allclose(om.decode(cache, int(toks[i]), 3), om.score_last(toks[: i + 1], 3),
                                   rtol=0, atol=1e-9)
    lg = om.score_last(toks, 3)
    assert np.isfinite(lg).all() and lg.std() > 1e-3


def test_planted_mistakes_fail_golden():
    def as_nibbles(words, n):
        return ref.unpack_nibbles(words, n)

    def highest_first(words, n):
        w = np.asarray(words, np.uint32)
        out = np.empty(w.shape[:-1] + (w.shape[-1] * 16,), np.uint8)
        for j in range(16):
            out[..., j::16] = (w >> np.uint32(30 - 2 * j)) & np.uint32(3)
        return out[..., :n]

    for bad in (as_nibbles, highest_first):
        ok = all(bad(np.array([[w]], np.uint32), 16)[0].tolist() == e for w, e in _golden())
        assert not ok, bad.__name__
