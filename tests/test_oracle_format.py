"""Pins of the oracle's INT4 decoding and dequantisation (CPU only).

The decoder under test is ``oracle.ref``; the encoder is the independent
``tl_synth.pack_nibbles``.  Expected values come from the hand-decoded golden
words, from exact rational arithmetic, and from brute force.
"""

import os
from fractions import Fraction

import numpy as np
import pytest

import tl_synth
from oracle import ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_words():
    rows = []
    with open(os.path.join(GOLDEN, "int4_nibble_order.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            rows.append((int(parts[0], 16), [int(p) for p in parts[1:]]))
    return rows


def test_golden_nibble_order():
    rows = _golden_words()
    assert len(rows) >= 6
    words = np.array([[w] for w, _ in rows], dtype=np.uint32)
    got = ref.unpack_nibbles(words, 8)
    for (w, expect), g in zip(rows, got):
        assert list(g) == expect, hex(w)


def test_golden_nibble_order_encoder_agrees():
    # The generator's encoder must produce the same hand-decoded words.
    for w, expect in _golden_words():
        assert int(tl_synth.pack_nibbles(np.array([expect]))[0, 0]) == w


@pytest.mark.parametrize("n", [1, 7, 8, 9, 16, 44, 128, 2048])
def test_pack_unpack_roundtrip(n):
    rng = np.random.default_rng(n)
    vals = rng.integers(0, 16, size=(5, n), dtype=np.uint8)
    words = tl_synth.pack_nibbles(vals)
    assert words.shape == (5, (n + 7) // 8)
    assert np.array_equal(ref.unpack_nibbles(words, n), vals)


def test_dequant_exhaustive_codes_exact():
    # Every (q, z) pair with a spread of fp16 scales; compared with exact
    # rational arithmetic, element by element.
    rng = np.random.default_rng(7)
    scales = np.concatenate([
        np.array([0.005, 0.02, 1.0, 2.0 ** -14, 65504.0], np.float16),
        rng.uniform(0.005, 0.02, 27).astype(np.float16)])
    N = 256 * len(scales)
    K = 128
    q = np.zeros((N, K), np.uint8)
    z = np.zeros((N, 1), np.uint8)
    s = np.zeros((N, 1), np.float16)
    r = 0
    for sc in scales:
        for qq in range(16):
            for zz in range(16):
                q[r, :] = qq
                q[r, r % K] = (qq + 5) % 16   # one odd element per row
                z[r, 0] = zz
                s[r, 0] = sc
                r += 1
    W = ref.dequantize(tl_synth.pack_nibbles(q), s, tl_synth.pack_nibbles(z), K)
    for r in range(0, N, 37):
        for k in (0, r % K, K - 1):
            expect = (int(q[r, k]) - int(z[r, 0])) * Fraction(float(s[r, 0]))
            assert Fraction(float(W[r, k])) == expect


def test_dequant_group_indexing():
    # Distinct zero and scale per group: every element must pick its own group.
    rng = np.random.default_rng(3)
    N, K = 3, 5632   # 44 groups, 6 zero words per row
    lin = tl_synth.make_int4_linear(rng, N, K)
    W = ref.dequantize(lin.qweight, lin.scales, lin.qzeros, K)
    for n in range(N):
        for k in range(0, K, 97):
            g = k // 128
            expect = (int(lin.q[n, k]) - int(lin.z[n, g])) * float(lin.scales[n, g])
            assert W[n, k] == expect


def test_one_hot_activation_returns_column():
    rng = np.random.default_rng(11)
    lin = tl_synth.make_int4_linear(rng, 40, 256)
    W = ref.dequantize(lin.qweight, lin.scales, lin.qzeros, lin.K)
    for k in (0, 1, 127, 128, 255):
        x = np.zeros((1, lin.K))
        x[0, k] = 1.0
        assert np.array_equal(ref.int4_linear(x, W)[0], W[:, k])


def test_linear_brute_force():
    rng = np.random.default_rng(5)
    M, N, K = 3, 6, 256
    lin = tl_synth.make_int4_linear(rng, N, K)
    x = tl_synth.make_activations(9, M, K)
    W = ref.dequantize(lin.qweight, lin.scales, lin.qzeros, K)
    y = ref.int4_linear(x, W)
    for m in range(M):
        for n in range(N):
            acc = Fraction(0)
            for k in range(K):
                g = k // 128
                w = (int(lin.q[n, k]) - int(lin.z[n, g])) * Fraction(float(lin.scales[n, g]))
                acc += Fraction(float(x[m, k])) * w
            assert abs(float(acc) - y[m, n]) <= 1e-12 * max(1.0, abs(float(acc)))
