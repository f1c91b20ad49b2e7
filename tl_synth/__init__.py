"""Seeded synthetic inputs for the looped INT4 transformer.

This module is shared by the CPU oracle tests, the CUDA-path tests and the
benchmark.  It only *draws* numbers and lays them out in the storage format
that the C ABI accepts; it contains none of the model's arithmetic (no
dequantisation, normalisation, rotation, attention or matmul).

Storage format of one group-wise INT4 linear layer with K inputs, N outputs and
group size 128 along K (TinyLoop README, "Status": INT4 loop / pre linears with
zero points; the group size, fp16 scale and 4-bit zero are the workload's
definition w = (q - z) * s):

* ``qweight``  uint32 [N][K/8]       element k of row n sits in bits 4*(k%8)..4*(k%8)+3
                                      of word k//8 (low nibble first)
* ``scales``   float16 [N][K/128]    one scale per (row, group)
* ``qzeros``   uint32 [N][ceil(G/8)] the G = K/128 zero points of row n, packed
                                      eight per word with the same nibble order;
                                      unused nibbles are 0
* no "+1" offset is applied to the stored zero point.

The INT2 body (TinyLoop README, "Current Runtime Snapshot": INT2 is the
default body; the pages give no format) uses the same layout with 2-bit
fields, this library's reading: ``qweight`` uint32 [N][K/16] with element k in
bits 2*(k%16)..2*(k%16)+1 of word k//16 (lowest field first), ``scales``
float16 [N][K/128], ``qzeros`` uint32 [N][ceil(G/16)] (16 zero points per
word), w = (q - z) * s with q, z in {0..3}.  Its draws: q ~ U{0..3},
z ~ U{0..3}, s ~ U(0.02, 0.08) (a stated choice: it gives the weights about the
INT4 draws' spread, std(q - z) * mean(s) ~ 0.08).

Draw order for :func:`make_model_weights` (one ``numpy.random.default_rng(seed)``
stream, PCG64): embedding, then for each block in the order pre[0] .. pre[n_pre-1],
loop: attn_norm gain, ffn_norm gain, then the linears qkv, o, gate_up, down, each
as (q, z, s); then out_norm gain, then head.  Values are drawn in float64 and
rounded to float16 with round-to-nearest-even (numpy's cast).

Distributions (the workload definition): q ~ U{0..15}, z ~ U{0..15},
s ~ U(0.005, 0.02), embedding and head ~ N(0, 0.02), norm gains ~ U(0.8, 1.2)
(a stated choice: the pages give no distribution for the gains), token ids
~ U[0, vocab).
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import List

import numpy as np

GROUP_SIZE = 128


@dataclass(frozen=True)
class ModelShape:
    """Dimensions of a weight-shared looped transformer."""

    d_model: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn_dim: int
    vocab: int
    n_pre: int
    rms_eps: float = 1e-5
    rope_theta: float = 1e4
    group_size: int = GROUP_SIZE

    @property
    def qkv_rows(self) -> int:
        return (self.n_q_heads + 2 * self.n_kv_heads) * self.head_dim


# Tiny looped LM: d_model 256, 4 Q / 2 KV heads of 64, SwiGLU 1024, vocab 512,
# one pre block + one shared loop block.
TINY_LM = ModelShape(d_model=256, n_q_heads=4, n_kv_heads=2, head_dim=64,
                     ffn_dim=1024, vocab=512, n_pre=1)

# The ~400M-unique-parameter looped LM: d_model 2048, 16 Q / 4 KV heads of 128,
# SwiGLU 5632, vocab 32000, two pre blocks + one shared loop block.
LOOPED_LM = ModelShape(d_model=2048, n_q_heads=16, n_kv_heads=4, head_dim=128,
                       ffn_dim=5632, vocab=32000, n_pre=2)

# INT4 linear sweep shapes (K, N) and row counts M.
LINEAR_SWEEP_KN = [(2048, 3072), (2048, 2048), (2048, 11264), (5632, 2048)]
LINEAR_SWEEP_M = [1, 4, 16, 128]

# Seeds: 1000 + index of the workload in the list
# [tiny LM, linear sweep, attention, looped LM, L-sweep].
SEED_TINY, SEED_LINEAR, SEED_ATTN, SEED_LM, SEED_LSWEEP = 1000, 1001, 1002, 1003, 1004


def pack_nibbles(values: np.ndarray) -> np.ndarray:
    """Pack 4-bit values along the last axis, eight per uint32, low nibble first.

    ``values[..., k]`` lands in bits 4*(k%8) of word ``k//8``.  The last axis is
    zero-padded to a multiple of eight.
    """
    v = np.asarray(values, dtype=np.uint32)
    if v.size and (v.max() > 15):
        raise ValueError("nibble out of range")
    n = v.shape[-1]
    pad = (-n) % 8
    if pad:
        v = np.concatenate([v, np.zeros(v.shape[:-1] + (pad,), np.uint32)], axis=-1)
    v = v.reshape(v.shape[:-1] + (v.shape[-1] // 8, 8))
    out = np.zeros(v.shape[:-1], dtype=np.uint32)
    for j in range(8):
        out |= v[..., j] << np.uint32(4 * j)
    return out


def pack_crumbs(values: np.ndarray) -> np.ndarray:
    """Pack 2-bit values along the last axis, sixteen per uint32, lowest field
    first: ``values[..., k]`` lands in bits 2*(k%16) of word ``k//16``.  The
    last axis is zero-padded to a multiple of sixteen."""
    v = np.asarray(values, dtype=np.uint32)
    if v.size and (v.max() > 3):
        raise ValueError("2-bit value out of range")
    n = v.shape[-1]
    pad = (-n) % 16
    if pad:
        v = np.concatenate([v, np.zeros(v.shape[:-1] + (pad,), np.uint32)], axis=-1)
    v = v.reshape(v.shape[:-1] + (v.shape[-1] // 16, 16))
    out = np.zeros(v.shape[:-1], dtype=np.uint32)
    for j in range(16):
        out |= v[..., j] << np.uint32(2 * j)
    return out


@dataclass
class Int4Linear:
    """One INT4 (or INT2: bits = 2) linear layer in the storage format, plus
    the raw draws."""

    K: int
    N: int
    qweight: np.ndarray  # uint32 [N][K/8] (INT2: [N][K/16])
    scales: np.ndarray   # float16 [N][K/128]
    qzeros: np.ndarray   # uint32 [N][ceil(K/128/8)] (INT2: [N][ceil(K/128/16)])
    q: np.ndarray        # uint8 [N][K]   raw codes (kept for format tests)
    z: np.ndarray        # uint8 [N][K/128] raw zero points
    bits: int = 4

    @property
    def n_groups(self) -> int:
        return self.K // GROUP_SIZE


def make_int4_linear(rng: np.random.Generator, N: int, K: int,
                     scale_lo: float = 0.005, scale_hi: float = 0.02) -> Int4Linear:
    if K % GROUP_SIZE:
        raise ValueError("K must be a multiple of the group size")
    G = K // GROUP_SIZE
    q = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    z = rng.integers(0, 16, size=(N, G), dtype=np.uint8)
    s = rng.uniform(scale_lo, scale_hi, size=(N, G)).astype(np.float16)
    return Int4Linear(K=K, N=N, qweight=pack_nibbles(q), scales=s,
                      qzeros=pack_nibbles(z), q=q, z=z)


def make_int2_linear(rng: np.random.Generator, N: int, K: int,
                     scale_lo: float = 0.02, scale_hi: float = 0.08) -> Int4Linear:
    if K % GROUP_SIZE:
        raise ValueError("K must be a multiple of the group size")
    G = K // GROUP_SIZE
    q = rng.integers(0, 4, size=(N, K), dtype=np.uint8)
    z = rng.integers(0, 4, size=(N, G), dtype=np.uint8)
    s = rng.uniform(scale_lo, scale_hi, size=(N, G)).astype(np.float16)
    return Int4Linear(K=K, N=N, qweight=pack_crumbs(q), scales=s, qzeros=pack_crumbs(z), q=q, z=z, bits=2)


@dataclass
class BlockWeights:
    attn_norm: np.ndarray  # float16 [d]
    ffn_norm: np.ndarray   # float16 [d]
    qkv: Int4Linear        # N = (Hq + 2 Hkv) * hd, rows: q heads, k heads, v heads
    o: Int4Linear          # N = d, K = Hq * hd
    gate_up: Int4Linear    # N = 2F: rows [0, F) gate, [F, 2F) up
    down: Int4Linear       # N = d, K = F


@dataclass
class ModelWeights:
    shape: ModelShape
    embed: np.ndarray      # float16 [V][d]
    out_norm: np.ndarray   # float16 [d]
    head: np.ndarray       # float16 [V][d]
    pre: List[BlockWeights] = field(default_factory=list)
    loop: BlockWeights = None


def _gain(rng, d):
    return rng.uniform(0.8, 1.2, size=d).astype(np.float16)


def make_block(rng: np.random.Generator, shape: ModelShape, bits: int = 4) -> BlockWeights:
    d, F = shape.d_model, shape.ffn_dim
    lin = make_int4_linear if bits == 4 else make_int2_linear
    attn_norm = _gain(rng, d)
    ffn_norm = _gain(rng, d)
    qkv = lin(rng, shape.qkv_rows, d)
    o = lin(rng, d, shape.n_q_heads * shape.head_dim)
    gate_up = lin(rng, 2 * F, d)
    down = lin(rng, d, F)
    return BlockWeights(attn_norm, ffn_norm, qkv, o, gate_up, down)


def make_model_weights(shape: ModelShape, seed: int, bits: int = 4) -> ModelWeights:
    """Every block's linears INT4 (bits = 4) or INT2 (bits = 2)."""
    if bits not in (2, 4):
        raise ValueError("bits must be 2 or 4")
    rng = np.random.default_rng(seed)
    embed = rng.normal(0.0, 0.02, size=(shape.vocab, shape.d_model)).astype(np.float16)
    pre = [make_block(rng, shape, bits) for _ in range(shape.n_pre)]
    loop = make_block(rng, shape, bits)
    out_norm = _gain(rng, shape.d_model)
    head = rng.normal(0.0, 0.02, size=(shape.vocab, shape.d_model)).astype(np.float16)
    return ModelWeights(shape=shape, embed=embed, out_norm=out_norm, head=head,
                        pre=pre, loop=loop)


def make_tokens(seed: int, vocab: int, n: int) -> np.ndarray:
    """n token ids ~ U[0, vocab), int32."""
    return np.random.default_rng(seed).integers(0, vocab, size=n, dtype=np.int64).astype(np.int32)


def make_lane_prompts(seed: int, vocab: int, n_lanes: int, length: int) -> np.ndarray:
    """int32 [n_lanes][length] prompts, one independent stream of ids per call."""
    rng = np.random.default_rng(seed)
    return rng.integers(0, vocab, size=(n_lanes, length), dtype=np.int64).astype(np.int32)


def make_lane_loops(seed: int, n_lanes: int, choices=(4, 8, 16)) -> np.ndarray:
    """Per-lane loop counts drawn uniformly from ``choices``."""
    rng = np.random.default_rng(seed)
    return np.asarray(choices, dtype=np.int32)[rng.integers(0, len(choices), size=n_lanes)]


def make_activations(seed: int, M: int, K: int) -> np.ndarray:
    """float16 [M][K] activations ~ N(0, 1)."""
    return np.random.default_rng(seed).normal(0.0, 1.0, size=(M, K)).astype(np.float16)


def make_qkv(seed: int, batch: int, T: int, n_q_heads: int, n_kv_heads: int,
             head_dim: int, T_q: int = None):
    """float16 K and V [B][T][Hkv][hd], then Q [B][T_q][Hq][hd] (T_q defaults
    to T), all ~ N(0, 1), drawn in that order from one stream."""
    rng = np.random.default_rng(seed)
    k = rng.normal(0.0, 1.0, size=(batch, T, n_kv_heads, head_dim)).astype(np.float16)
    v = rng.normal(0.0, 1.0, size=(batch, T, n_kv_heads, head_dim)).astype(np.float16)
    tq = T if T_q is None else T_q
    q = rng.normal(0.0, 1.0, size=(batch, tq, n_q_heads, head_dim)).astype(np.float16)
    return q, k, v
