"""Pins of the oracle's per-op definitions (CPU only).

Each op is checked against closed forms, invariants, brute force, or a library
routine (torch, float64) that computes the same textbook operation.
"""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as tF

from oracle import ref


# ---------------------------------------------------------------- RMSNorm ---

def test_rmsnorm_closed_form_unit_gain():
    rng = np.random.default_rng(0)
    x = rng.normal(0, 3.0, size=(4, 64))
    eps = 1e-5
    y = ref.rms_norm(x, np.ones(64), eps)
    m = np.mean(x * x, axis=-1)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), np.sqrt(m / (m + eps)), rtol=1e-13)


def test_rmsnorm_constant_vector():
    for c in (0.5, -2.0, 100.0):
        x = np.full((1, 8), c)
        g = np.arange(1, 9, dtype=np.float64)
        y = ref.rms_norm(x, g, 1e-5)
        assert np.allclose(y[0], c / math.sqrt(c * c + 1e-5) * g, rtol=1e-14)


def test_rmsnorm_scale_invariant_without_eps():
    rng = np.random.default_rng(1)
    x = rng.normal(size=(3, 32))
    g = rng.uniform(0.8, 1.2, 32)
    assert np.allclose(ref.rms_norm(x, g, 0.0), ref.rms_norm(7.5 * x, g, 0.0), rtol=1e-13)


def test_rmsnorm_matches_torch():
    rng = np.random.default_rng(2)
    x = rng.normal(size=(5, 256))
    g = rng.uniform(0.8, 1.2, 256)
    t = tF.rms_norm(torch.tensor(x), (256,), torch.tensor(g), eps=1e-5).numpy()
    assert np.allclose(ref.rms_norm(x, g, 1e-5), t, rtol=1e-13, atol=1e-15)


# ------------------------------------------------------------------- RoPE ---

def test_rope_two_dims_is_plane_rotation():
    # hd = 2: one pair at frequency theta^0 = 1, i.e. rotation by p radians.
    for p in (0, 1, 5, 2047):
        x = np.array([[[0.3, -1.7]]])
        y = ref.rope(x, [p], 1e4)[0, 0]
        c, s = math.cos(p), math.sin(p)
        assert np.allclose(y, [0.3 * c + 1.7 * s, 0.3 * s - 1.7 * c], rtol=1e-14, atol=1e-15)


def test_rope_complex_form():
    # Textbook complex form: (x_j + i x_{j+hd/2}) * exp(i p theta^(-2j/hd)).
    # (1e-10: the angle at p = 8191 carries the rounding of theta^(-2j/hd).)
    rng = np.random.default_rng(3)
    hd, theta = 64, 1e4
    x = rng.normal(size=(6, 3, hd))
    pos = [0, 1, 17, 128, 1000, 8191]
    y = ref.rope(x, pos, theta)
    for t, p in enumerate(pos):
        for j in range(hd // 2):
            w = complex(x[t, 0, j], x[t, 0, j + hd // 2]) * complex(
                math.cos(p * theta ** (-2 * j / hd)), math.sin(p * theta ** (-2 * j / hd)))
            assert abs(y[t, 0, j] - w.real) < 1e-10 and abs(y[t, 0, j + hd // 2] - w.imag) < 1e-10


def test_rope_preserves_norm_and_identity_at_zero():
    rng = np.random.default_rng(4)
    x = rng.normal(size=(9, 4, 128))
    pos = np.arange(9) * 911
    y = ref.rope(x, pos, 1e4)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    assert np.array_equal(ref.rope(x[:1], [0], 1e4), x[:1])


def test_rope_relative_position():
    rng = np.random.default_rng(5)
    q = rng.normal(size=(1, 1, 128))
    k = rng.normal(size=(1, 1, 128))
    dots = []
    for m, n in ((10, 3), (107, 100), (2007, 2000)):
        dots.append(float(np.sum(ref.rope(q, [m], 1e4) * ref.rope(k, [n], 1e4))))
    assert np.allclose(dots, dots[0], rtol=1e-9)


# -------------------------------------------------------------- Attention ---

def _brute_attention(q, k, v, pos):
    T, Hq, hd = q.shape
    Hkv = k.shape[1]
    out = np.zeros_like(q)
    for t in range(T):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            s = [sum(q[t, h, d] * k[j, g, d] for d in range(hd)) / math.sqrt(hd)
                 for j in range(pos[t] + 1)]
            m = max(s)
            e = [math.exp(si - m) for si in s]
            z = sum(e)
            for d in range(hd):
                out[t, h, d] = sum(e[j] / z * v[j, g, d] for j in range(pos[t] + 1))
    return out


def test_attention_brute_force():
    rng = np.random.default_rng(6)
    q = rng.normal(size=(3, 4, 8))
    k = rng.normal(size=(5, 2, 8))
    v = rng.normal(size=(5, 2, 8))
    pos = [2, 3, 4]
    assert np.allclose(ref.gqa_attention(q, k, v, pos), _brute_attention(q, k, v, pos),
                       rtol=1e-12, atol=1e-14)


def test_attention_single_key_returns_value():
    rng = np.random.default_rng(7)
    q = rng.normal(size=(1, 4, 16)) * 50
    k = rng.normal(size=(1, 2, 16))
    v = rng.normal(size=(1, 2, 16))
    out = ref.gqa_attention(q, k, v, [0])
    assert np.allclose(out[0], np.repeat(v[0], 2, axis=0), rtol=1e-14)


def test_attention_equal_keys_average_values():
    rng = np.random.default_rng(8)
    q = rng.normal(size=(1, 2, 16))
    k = np.repeat(rng.normal(size=(1, 1, 16)), 6, axis=0)
    v = rng.normal(size=(6, 1, 16))
    out = ref.gqa_attention(q, k, v, [5])
    assert np.allclose(out[0, 0], v[:, 0].mean(axis=0), rtol=1e-13)
    assert np.allclose(out[0, 1], v[:, 0].mean(axis=0), rtol=1e-13)


def _torch_sdpa(q, k, v, gqa):
    # q [T][Hq][hd] -> [1][Hq][T][hd]; causal with queries at positions 0..T-1.
    tq = torch.tensor(q).permute(1, 0, 2)[None]
    tk = torch.tensor(k).permute(1, 0, 2)[None]
    tv = torch.tensor(v).permute(1, 0, 2)[None]
    o = tF.scaled_dot_product_attention(tq, tk, tv, is_causal=True, enable_gqa=gqa)
    return o[0].permute(1, 0, 2).numpy()


def test_attention_mha_matches_torch():
    rng = np.random.default_rng(9)
    q, k, v = (rng.normal(size=(12, 4, 32)) for _ in range(3))
    out = ref.gqa_attention(q, k, v, np.arange(12))
    assert np.allclose(out, _torch_sdpa(q, k, v, False), rtol=1e-12, atol=1e-13)


def test_attention_gqa_matches_torch():
    rng = np.random.default_rng(10)
    q = rng.normal(size=(10, 16, 32))
    k = rng.normal(size=(10, 4, 32))
    v = rng.normal(size=(10, 4, 32))
    out = ref.gqa_attention(q, k, v, np.arange(10))
    assert np.allclose(out, _torch_sdpa(q, k, v, True), rtol=1e-12, atol=1e-13)


def test_attention_gqa_equals_mha_on_repeated_heads():
    rng = np.random.default_rng(11)
    q = rng.normal(size=(7, 8, 16))
    k = rng.normal(size=(9, 2, 16))
    v = rng.normal(size=(9, 2, 16))
    pos = [2, 3, 4, 5, 6, 7, 8]
    gqa = ref.gqa_attention(q, k, v, pos)
    mha = ref.gqa_attention(q, np.repeat(k, 4, axis=1), np.repeat(v, 4, axis=1), pos)
    assert np.allclose(gqa, mha, rtol=1e-14)


def test_attention_offset_queries_equal_suffix_of_full():
    # Queries at positions p0..p0+T-1 over keys 0..p0+T-1 give the suffix rows
    # of the full causal attention (the cached-decode case).
    rng = np.random.default_rng(12)
    q = rng.normal(size=(20, 4, 16))
    k = rng.normal(size=(20, 2, 16))
    v = rng.normal(size=(20, 2, 16))
    full = ref.gqa_attention(q, k, v, np.arange(20))
    tail = ref.gqa_attention(q[15:], k, v, np.arange(15, 20))
    assert np.allclose(full[15:], tail, rtol=1e-14)


# ----------------------------------------------------- SwiGLU and argmax ---

def test_silu_matches_torch():
    u = np.linspace(-30, 30, 241)
    assert np.allclose(ref.silu(u), tF.silu(torch.tensor(u)).numpy(), rtol=1e-14, atol=1e-300)


def test_swiglu_halves():
    rng = np.random.default_rng(13)
    gu = rng.normal(size=(3, 10))
    out = ref.swiglu(gu, 5)
    expect = tF.silu(torch.tensor(gu[:, :5])).numpy() * gu[:, 5:]
    assert np.allclose(out, expect, rtol=1e-14)


def test_greedy_ties_lowest_index():
    assert ref.greedy(np.array([1.0, 3.0, 3.0, 2.0])) == 1
    assert ref.greedy(np.array([5.0, 5.0])) == 0
    rng = np.random.default_rng(14)
    for _ in range(20):
        x = rng.integers(0, 4, size=50).astype(np.float64)
        assert ref.greedy(x) == int(np.argmax(x)) == min(np.flatnonzero(x == x.max()))


def test_top2_margin():
    assert ref.top2_margin(np.array([0.0, 2.0, 1.5])) == pytest.approx(0.5)
