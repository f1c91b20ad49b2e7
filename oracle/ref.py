"""Plain CPU float64 oracle of the weight-shared looped INT4 transformer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` use it.  It shares no code with the CUDA library; both sides only
share the seeded input generator ``tl_synth``, which holds none of the model's
arithmetic.

What it computes, step by step, in the order the pages give it:

* the pipeline tokens -> embed -> pre blocks -> shared loop block x L ->
  output norm -> head (TinyLoop README, "Why TinyLoop Exists");
* the loop block's weights are the same object on every iteration, so memory
  follows unique blocks while L is a per-call compute knob (same section, items
  1 and 2; TinyLoop docs, "Async API", "Scoring"/"Generation": ``loops=`` on every
  call);
* group-wise INT4 weights with zero points, w = (q - z) * s, group 128 along K
  (TinyLoop README, "Status", INT4 loop / pre linears with zero points), or the
  INT2 body with the same form and 2-bit fields (TinyLoop README, "Current
  Runtime Snapshot": INT2 is the default body; format read as INT4's);
* RMSNorm (tiny-llm feature list, "Root Mean Square Normalizations");
* RoPE applied to Q and K with a configurable theta (TinyLoop README, "Status",
  Rotary Position Embeddings; tiny-llm feature list, "Rotary Positional
  Embeddings");
* grouped-query attention with a causal mask (TinyLoop README, "Status", GQA;
  tiny-llm feature list, "Grouped-Query Attention", "Causal Masking");
* a SwiGLU gated MLP (tiny-llm feature list, "Gated Linear Units");
* a per-layer KV cache, one slice per effective layer, so each loop iteration
  owns its slice (TinyLoop README, "Status", GQA item: the per-layer KV cache
  whose cost multiplies across L iterations) and cached decode agrees with the
  uncached recompute (TinyLoop README, "Current Runtime Snapshot" quality notes
  and "Quick CLI Tour", Generate);
* greedy decoding = argmax, lowest index on ties (TinyLoop docs, "Async API",
  "Generation", temperature 0);
* around that pass: the logit lens (the head after every loop iteration;
  TinyLoop docs, "Async API", "Scoring", score_logit_lens), token-stable early
  exit (TinyLoop README, "Runtime Flags", TINYLOOP_TOKEN_EXIT), greedy
  self-speculative decoding with a draft that runs fewer loops of the same
  block (TinyLoop docs, "Async API", "Speculative decode"; TinyLoop README,
  "Why TinyLoop Exists", item 3) and forking a cached prefix (TinyLoop README,
  "Python Quick Start", build_prefix_cache / generate_from_prefix_cache).

Readings taken where the pages are silent (each is listed with its reason in
the design notes): Llama-style pre-norm block with no Q/K norm; iteration i+1
consumes iteration i's residual stream unchanged; positions are the absolute
token positions on every layer and iteration; RoPE pairs element j with
j + hd/2 (rotate-half) at angle p * theta^(-2j/hd); kv head of q head h is
h // (Hq/Hkv); scale 1/sqrt(hd); RMSNorm y = x / sqrt(mean(x^2) + eps) * g;
gate rows [0, F) and up rows [F, 2F) of the fused gate_up weight;
the head is a separate matrix (not tied to the embedding).

Everything is float64; the fp16 inputs (scales, gains, embedding, head,
activations) are widened exactly.  One precision is fixed by the pages and so
kept: keys and values are stored in an FP16 KV cache (TinyLoop README, "Python
API reference": KV cache modes, "FP16 KV"; the workload's "KV cache fp16").  By
default (``kv_mode="fp16"``) the rotated keys and the values are rounded to
fp16 (round-to-nearest-even) when they are produced, on the cached and the
uncached path alike, so attention always reads the stored fp16 values.  The
pages also name an INT8 KV mode (TinyLoop README, "Python API reference", KV
cache modes) without its format; ``kv_mode="int8"`` takes the plainest reading:
each produced key and value vector (one position, one kv head, hd elements) is
stored as symmetric int8 codes with one fp32 scale, see ``quantize_kv_int8``,
and attention reads the dequantized codes.  With ``kv_mode="none"`` (or
``kv_fp16=False``) nothing at all is rounded (used to compare against a
float64 library model).  No other rounding is emulated.
"""

from __future__ import annotations

import math
from dataclasses import dataclass
from typing import List, Optional, Sequence

import numpy as np

GROUP_SIZE = 128


# ---------------------------------------------------------------------------
# INT4 storage format
# ---------------------------------------------------------------------------

def unpack_nibbles(words: np.ndarray, n: int) -> np.ndarray:
    """Decode ``n`` 4-bit values per row from uint32 words, low nibble first.

    Element k of a row is bits 4*(k % 8) .. 4*(k % 8)+3 of word k // 8.
    """
    w = np.asarray(words, dtype=np.uint32)
    out = np.empty(w.shape[:-1] + (w.shape[-1] * 8,), dtype=np.uint8)
    for j in range(8):
        out[..., j::8] = (w >> np.uint32(4 * j)) & np.uint32(0xF)
    return out[..., :n]


def dequantize(qweight: np.ndarray, scales: np.ndarray, qzeros: np.ndarray,
               K: int) -> np.ndarray:
    """W[n, k] = (q[n, k] - z[n, k // 128]) * s[n, k // 128] in float64.

    Every value is exact: q, z are integers in [0, 15] and s is an fp16 value,
    so the product has at most 15 significant bits.
    """
    if K % GROUP_SIZE:
        raise ValueError("K must be a multiple of 128")
    G = K // GROUP_SIZE
    q = unpack_nibbles(qweight, K).astype(np.float64)            # [N][K]
    z = unpack_nibbles(qzeros, G).astype(np.float64)             # [N][G]
    s = np.asarray(scales, dtype=np.float16).astype(np.float64)  # [N][G]
    group = np.arange(K) // GROUP_SIZE
    return (q - z[:, group]) * s[:, group]


def unpack_crumbs(words: np.ndarray, n: int) -> np.ndarray:
    """Decode ``n`` 2-bit values per row from uint32 words, lowest field first.

    Element k of a row is bits 2*(k % 16) .. 2*(k % 16)+1 of word k // 16 (the
    INT2 body's storage, this library's reading; the pages name the INT2 body,
    TinyLoop README "Current Runtime Snapshot", but give no format).
    """
    w = np.asarray(words, dtype=np.uint32)
    out = np.empty(w.shape[:-1] + (w.shape[-1] * 16,), dtype=np.uint8)
    for j in range(16):
        out[..., j::16] = (w >> np.uint32(2 * j)) & np.uint32(0x3)
    return out[..., :n]


def dequantize_int2(qweight: np.ndarray, scales: np.ndarray, qzeros: np.ndarray,
                    K: int) -> np.ndarray:
    """W[n, k] = (q[n, k] - z[n, k // 128]) * s[n, k // 128] for the INT2
    storage (q, z in [0, 3]), in float64; every value is exact."""
    if K % GROUP_SIZE:
        raise ValueError("K must be a multiple of 128")
    G = K // GROUP_SIZE
    q = unpack_crumbs(qweight, K).astype(np.float64)
    z = unpack_crumbs(qzeros, G).astype(np.float64)
    s = np.asarray(scales, dtype=np.float16).astype(np.float64)
    group = np.arange(K) // GROUP_SIZE
    return (q - z[:, group]) * s[:, group]


def int4_linear(x: np.ndarray, W: np.ndarray) -> np.ndarray:
    """y = x W^T with x [..., K] and the dequantized W [N][K]."""
    return np.asarray(x, dtype=np.float64) @ W.T


# ---------------------------------------------------------------------------
# Per-op definitions
# ---------------------------------------------------------------------------

def rms_norm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2 over the last axis) + eps) * g."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(g, dtype=np.float64)


def rope_angles(positions: Sequence[int], head_dim: int, theta: float) -> np.ndarray:
    """angle[t, j] = p_t * theta^(-2j/hd) for j < hd/2, float64 [T][hd/2]."""
    half = head_dim // 2
    j = np.arange(half, dtype=np.float64)
    inv_freq = theta ** (-2.0 * j / head_dim)
    return np.asarray(positions, dtype=np.float64)[:, None] * inv_freq[None, :]


def rope(x: np.ndarray, positions: Sequence[int], theta: float) -> np.ndarray:
    """Rotate x [T][H][hd]: pair (j, j + hd/2) turns by angle[t, j]."""
    x = np.asarray(x, dtype=np.float64)
    hd = x.shape[-1]
    half = hd // 2
    ang = rope_angles(positions, hd, theta)[:, None, :]   # [T][1][half]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def gqa_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                  q_positions: Sequence[int]) -> np.ndarray:
    """Causal grouped-query attention.

    q [T][Hq][hd]; k, v [S][Hkv][hd] with key j at absolute position j.  Query t
    at position p_t attends to keys 0..p_t, q head h reads kv head h // (Hq/Hkv),
    scores are scaled by 1/sqrt(hd).  Returns [T][Hq][hd].
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    T, Hq, hd = q.shape
    S, Hkv, _ = k.shape
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    rep = Hq // Hkv
    pos = np.asarray(q_positions, dtype=np.int64)
    if pos.size and pos.max() >= S:
        raise ValueError("query position beyond the keys")
    qg = q.reshape(T, Hkv, rep, hd).transpose(1, 2, 0, 3)       # [Hkv][rep][T][hd]
    kg = k.transpose(1, 0, 2)                                   # [Hkv][S][hd]
    vg = v.transpose(1, 0, 2)
    scores = np.einsum("grtd,gsd->grts", qg, kg) / math.sqrt(hd)
    mask = np.arange(S)[None, :] > pos[:, None]                 # [T][S]
    scores = np.where(mask[None, None], -np.inf, scores)
    m = scores.max(axis=-1, keepdims=True)
    p = np.exp(scores - m)
    p = p / p.sum(axis=-1, keepdims=True)
    out = np.einsum("grts,gsd->grtd", p, vg)                    # [Hkv][rep][T][hd]
    return out.transpose(2, 0, 1, 3).reshape(T, Hq, hd)


def to_fp16_storage(x: np.ndarray) -> np.ndarray:
    """Round to the nearest fp16 value (ties to even) and widen back to float64:
    the value an FP16 KV cache holds."""
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def quantize_kv_int8(x: np.ndarray):
    """INT8 KV storage of vectors along the last axis (hd elements each).

    Per vector: scale = max|x| / 127 and code = round-half-even(x / scale),
    so the codes lie in [-127, 127] and the largest magnitude maps to +-127; an
    all-zero vector has scale 0 and codes 0.  The stored value is code * scale.
    The quantisation takes its integer decisions in float32, the precision the
    kernels take them in (x rounded to float32, the scale and the quotient
    float32 operations), so both sides choose the same codes for the same
    float32 input.  Returns (codes int8 [..., hd], scales float32 [...]).
    """
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x32), axis=-1)
    scale = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    q = np.rint((x32 / safe[..., None]).astype(np.float32))
    q = np.where(scale[..., None] > 0, q, np.float32(0.0))
    codes = np.clip(q, -127, 127).astype(np.int8)
    return codes, scale


def dequantize_kv_int8(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """code * scale in float64 (the value an INT8 KV cache holds)."""
    return np.asarray(codes, np.float64) * np.asarray(scales, np.float64)[..., None]


def to_int8_storage(x: np.ndarray) -> np.ndarray:
    """Quantise to the INT8 KV format and widen back: the value the cache holds."""
    return dequantize_kv_int8(*quantize_kv_int8(x))


def silu(u: np.ndarray) -> np.ndarray:
    return u / (1.0 + np.exp(-u))


def swiglu(gate_up: np.ndarray, F: int) -> np.ndarray:
    """silu(gate) * up with gate = columns [0, F), up = columns [F, 2F)."""
    return silu(gate_up[..., :F]) * gate_up[..., F:2 * F]


def greedy(logits: np.ndarray) -> int:
    """Index of the largest logit; the lowest index wins a tie."""
    logits = np.asarray(logits)
    best = 0
    for i in range(1, logits.shape[-1]):
        if logits[i] > logits[best]:
            best = i
    return best


def top2_margin(logits: np.ndarray) -> float:
    """Largest minus second-largest logit."""
    s = np.sort(np.asarray(logits, dtype=np.float64))
    return float(s[-1] - s[-2])


# ---------------------------------------------------------------------------
# Model
# ---------------------------------------------------------------------------

@dataclass
class DenseBlock:
    """One transformer block with dequantized float64 weights."""
    attn_norm: np.ndarray
    ffn_norm: np.ndarray
    w_qkv: np.ndarray
    w_o: np.ndarray
    w_gate_up: np.ndarray
    w_down: np.ndarray


def dense_block(blk) -> DenseBlock:
    """Dequantize every linear of a ``tl_synth.BlockWeights``."""
    def deq(lin):
        if getattr(lin, "bits", 4) == 2:
            return dequantize_int2(lin.qweight, lin.scales, lin.qzeros, lin.K)
        return dequantize(lin.qweight, lin.scales, lin.qzeros, lin.K)
    return DenseBlock(
        attn_norm=np.asarray(blk.attn_norm, np.float64),
        ffn_norm=np.asarray(blk.ffn_norm, np.float64),
        w_qkv=deq(blk.qkv), w_o=deq(blk.o),
        w_gate_up=deq(blk.gate_up), w_down=deq(blk.down))


class KVCache:
    """Keys and values of one sequence: one [S][Hkv][hd] pair per effective layer."""

    def __init__(self, n_layers: int):
        self.k: List[Optional[np.ndarray]] = [None] * n_layers
        self.v: List[Optional[np.ndarray]] = [None] * n_layers

    @property
    def length(self) -> int:
        return 0 if self.k[0] is None else self.k[0].shape[0]

    def fork(self, n: int) -> "KVCache":
        """A new cache holding copies of this one's first ``n`` positions in
        every slice (the prefix cache: TinyLoop README, "Python Quick Start",
        build_prefix_cache / generate_from_prefix_cache)."""
        if not 1 <= n <= self.length:
            raise ValueError("fork length out of range")
        out = KVCache(len(self.k))
        for layer in range(len(self.k)):
            out.k[layer] = self.k[layer][:n].copy()
            out.v[layer] = self.v[layer][:n].copy()
        return out

    def append(self, layer: int, k: np.ndarray, v: np.ndarray):
        if self.k[layer] is None:
            self.k[layer], self.v[layer] = k, v
        else:
            self.k[layer] = np.concatenate([self.k[layer], k], axis=0)
            self.v[layer] = np.concatenate([self.v[layer], v], axis=0)
        return self.k[layer], self.v[layer]


class LoopedModel:
    """The looped transformer with the weights of a ``tl_synth.ModelWeights``."""

    def __init__(self, weights, kv_fp16: bool = True, kv_mode: Optional[str] = None):
        sh = weights.shape
        self.shape = sh
        if kv_mode is None:
            kv_mode = "fp16" if kv_fp16 else "none"
        if kv_mode not in ("fp16", "int8", "none"):
            raise ValueError("kv_mode must be fp16, int8 or none")
        self.kv_mode = kv_mode
        # when a list: (layer, k, v) of every block call, the rotated keys and
        # the values before the cache's storage rounding (for checking what a
        # cache stores against what it was given)
        self.kv_trace: Optional[list] = None
        self.embed = np.asarray(weights.embed, np.float64)
        self.out_norm = np.asarray(weights.out_norm, np.float64)
        self.head = np.asarray(weights.head, np.float64)
        self.pre = [dense_block(b) for b in weights.pre]
        self.loop = dense_block(weights.loop)

    # -- structure ----------------------------------------------------------
    def blocks(self, loops: int) -> List[DenseBlock]:
        """Effective layers: pre[0..n_pre-1] then the same loop block ``loops`` times."""
        if loops < 1:
            raise ValueError("loops must be >= 1")
        return list(self.pre) + [self.loop] * loops

    # -- one block ----------------------------------------------------------
    def block(self, blk: DenseBlock, x: np.ndarray, positions: np.ndarray,
              cache: Optional[KVCache], layer: int) -> np.ndarray:
        sh = self.shape
        Hq, Hkv, hd, F = sh.n_q_heads, sh.n_kv_heads, sh.head_dim, sh.ffn_dim
        T = x.shape[0]
        a = rms_norm(x, blk.attn_norm, sh.rms_eps)
        qkv = int4_linear(a, blk.w_qkv)
        q = qkv[:, :Hq * hd].reshape(T, Hq, hd)
        k = qkv[:, Hq * hd:(Hq + Hkv) * hd].reshape(T, Hkv, hd)
        v = qkv[:, (Hq + Hkv) * hd:].reshape(T, Hkv, hd)
        q = rope(q, positions, sh.rope_theta)
        k = rope(k, positions, sh.rope_theta)
        if self.kv_trace is not None:
            self.kv_trace.append((layer, k.copy(), v.copy()))
        if self.kv_mode == "fp16":
            k, v = to_fp16_storage(k), to_fp16_storage(v)
        elif self.kv_mode == "int8":
            k, v = to_int8_storage(k), to_int8_storage(v)
        if cache is not None:
            k_all, v_all = cache.append(layer, k, v)
        else:
            k_all, v_all = k, v
        o = gqa_attention(q, k_all, v_all, positions).reshape(T, Hq * hd)
        x = x + int4_linear(o, blk.w_o)
        b = rms_norm(x, blk.ffn_norm, sh.rms_eps)
        h = swiglu(int4_linear(b, blk.w_gate_up), F)
        return x + int4_linear(h, blk.w_down)

    # -- stacks -------------------------------------------------------------
    def forward_stack(self, tokens: Sequence[int], blocks: Sequence[DenseBlock],
                      cache: Optional[KVCache] = None) -> np.ndarray:
        """Final residual stream [T][d] of the given explicit block stack.

        With a cache, the tokens continue the cached sequence (positions start
        at the cache length); without one, positions start at 0 and nothing is
        kept.
        """
        tokens = np.asarray(tokens, dtype=np.int64)
        if tokens.size and (tokens.min() < 0 or tokens.max() >= self.shape.vocab):
            raise ValueError("token id out of range")
        start = cache.length if cache is not None else 0
        positions = np.arange(start, start + tokens.shape[0])
        x = self.embed[tokens]
        for layer, blk in enumerate(blocks):
            x = self.block(blk, x, positions, cache, layer)
        return x

    def forward(self, tokens, loops: int, cache: Optional[KVCache] = None) -> np.ndarray:
        return self.forward_stack(tokens, self.blocks(loops), cache)

    def logits(self, h: np.ndarray) -> np.ndarray:
        """Output norm then head: [..., d] -> [..., V]."""
        return rms_norm(h, self.out_norm, self.shape.rms_eps) @ self.head.T

    # -- the entry points ---------------------------------------------------
    def score_last(self, tokens, loops: int) -> np.ndarray:
        """Logits [V] of the last position, no cache (a stateless forward)."""
        return self.logits(self.forward(tokens, loops)[-1])

    def score_logit_lens(self, tokens, loops: int) -> np.ndarray:
        """Logit lens [loops][V] (TinyLoop docs, "Async API", "Scoring",
        score_logit_lens): output norm + head of the last position after each
        loop iteration, no cache."""
        tokens = np.asarray(tokens, dtype=np.int64)
        positions = np.arange(tokens.shape[0])
        x = self.embed[tokens]
        for layer, blk in enumerate(self.pre):
            x = self.block(blk, x, positions, None, layer)
        rows = []
        for i in range(loops):
            x = self.block(self.loop, x, positions, None, self.shape.n_pre + i)
            rows.append(self.logits(x[-1]))
        return np.asarray(rows)

    def score_early_exit(self, tokens, max_loops: int, stable_n: int):
        """Token-stable early exit (TinyLoop README, "Runtime Flags",
        TINYLOOP_TOKEN_EXIT=N): iterate the loop block on the last position's
        stream until the greedy token of the last ``stable_n`` iterations is
        the same (or ``max_loops`` iterations ran).  Returns (logits of the
        exit iteration, iterations run)."""
        if stable_n < 1:
            raise ValueError("stable_n must be >= 1")
        tokens = np.asarray(tokens, dtype=np.int64)
        positions = np.arange(tokens.shape[0])
        x = self.embed[tokens]
        for layer, blk in enumerate(self.pre):
            x = self.block(blk, x, positions, None, layer)
        history = []
        for i in range(max_loops):
            x = self.block(self.loop, x, positions, None, self.shape.n_pre + i)
            logits = self.logits(x[-1])
            history.append(greedy(logits))
            if len(history) >= stable_n and len(set(history[-stable_n:])) == 1:
                break
        return logits, len(history)

    def generate_speculative(self, prompt, draft_loops: int, verify_loops: int, draft_ahead: int,
                             max_tokens: int):
        """Greedy self-speculative decoding (TinyLoop docs, "Async API",
        "Speculative decode"; TinyLoop README, "Why TinyLoop Exists" item 3):
        the draft model is the same network run with ``draft_loops``
        iterations.  Each round drafts k = min(draft_ahead, tokens left)
        tokens greedily, then the ``verify_loops`` model scores the sequence
        extended by the drafts; drafts are kept while they equal the
        verifier's greedy tokens and the verifier's token replaces the first
        rejected one.  Written without a cache (the cache changes no value).
        Returns (tokens, {"rounds", "drafted", "accepted"})."""
        seq = [int(t) for t in prompt]
        out = []
        stats = {"rounds": 0, "drafted": 0, "accepted": 0}
        while len(out) < max_tokens:
            k = min(draft_ahead, max_tokens - len(out))
            drafts = []
            for _ in range(k):
                drafts.append(greedy(self.score_last(seq + drafts, draft_loops)))
            h = self.forward(seq + drafts[:k - 1], verify_loops)
            ver = [greedy(self.logits(h[len(seq) - 1 + i])) for i in range(k)]
            acc = 0
            while acc < k and drafts[acc] == ver[acc]:
                acc += 1
            emit = min(acc + 1, k)
            out += ver[:emit]
            seq += ver[:emit]
            stats["rounds"] += 1
            stats["drafted"] += k
            stats["accepted"] += acc
        return out, stats

    def new_cache(self, loops: int) -> KVCache:
        return KVCache(self.shape.n_pre + loops)

    def prefill(self, tokens, loops: int):
        """Run the prompt, keep its KV; returns (cache, last-position logits)."""
        cache = self.new_cache(loops)
        h = self.forward(tokens, loops, cache)
        return cache, self.logits(h[-1])

    def decode(self, cache: KVCache, token: int, loops: int) -> np.ndarray:
        """One cached decode step: logits [V] for ``token`` at position cache.length."""
        if len(cache.k) != self.shape.n_pre + loops:
            raise ValueError("loops differ from the prefill's")
        h = self.forward([token], loops, cache)
        return self.logits(h[-1])

    def generate_greedy(self, prompt, loops: int, n_steps: int, cached: bool = True,
                        teacher: Optional[Sequence[int]] = None):
        """Greedy continuation.

        Returns (tokens, logits) where logits[i] are the logits that produced
        tokens[i].  With ``teacher`` the fed-back token of step i is teacher[i]
        instead of the argmax (teacher forcing); the argmax is still reported.
        ``cached=False`` recomputes the whole sequence for every step.
        """
        seq = list(int(t) for t in prompt)
        out_tokens, out_logits = [], []
        if cached:
            cache, logits = self.prefill(seq, loops)
        else:
            logits = self.score_last(seq, loops)
        for i in range(n_steps):
            tok = greedy(logits)
            out_tokens.append(tok)
            out_logits.append(logits)
            if i == n_steps - 1:
                break
            fed = tok if teacher is None else int(teacher[i])
            seq.append(fed)
            if cached:
                logits = self.decode(cache, fed, loops)
            else:
                logits = self.score_last(seq, loops)
        return out_tokens, np.asarray(out_logits)
