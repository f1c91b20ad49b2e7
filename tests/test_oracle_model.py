"""Pins of the oracle's whole-model behaviour (CPU only).

* looped with L iterations == a flattened stack of n_pre + L explicit blocks;
* cached decode == uncached recompute, token by token;
* the model with every block materialised is a Llama-family decoder (TinyLoop
  README, "Status": RoPE "enables Llama-family model support"), so it must
  agree with the independent ``transformers`` LlamaForCausalLM given the same
  dequantized weights.  That library keeps RMSNorm, the RoPE angles and the
  softmax in float32 internally, so the agreement is to ~1e-6, not 1e-15.
* planted mistakes in the oracle (on the CPU) are caught by that comparison.
"""

import copy

import numpy as np
import pytest
import torch

import tl_synth
from oracle import ref


@pytest.fixture(scope="module")
def tiny():
    w = tl_synth.make_model_weights(tl_synth.TINY_LM, tl_synth.SEED_TINY)
    return w, ref.LoopedModel(w)


@pytest.fixture(scope="module")
def tiny_exact(tiny):
    # no rounding anywhere: the form compared with the float64 library model
    return tiny[0], ref.LoopedModel(tiny[0], kv_fp16=False)


def test_looped_equals_flattened(tiny):
    _, m = tiny
    toks = tl_synth.make_tokens(1, m.shape.vocab, 17)
    for L in (1, 2, 4):
        looped = m.forward(toks, L)
        flat_blocks = list(m.pre) + [copy.deepcopy(m.loop) for _ in range(L)]
        assert all(b is not m.loop for b in flat_blocks[m.shape.n_pre:])
        flat = m.forward_stack(toks, flat_blocks)
        assert np.array_equal(looped, flat)


def test_loops_change_the_result(tiny):
    _, m = tiny
    toks = tl_synth.make_tokens(2, m.shape.vocab, 9)
    a = m.score_last(toks, 2)
    b = m.score_last(toks, 3)
    assert np.max(np.abs(a - b)) > 1e-3


def test_prefill_logits_equal_score_last(tiny):
    _, m = tiny
    toks = tl_synth.make_tokens(3, m.shape.vocab, 12)
    cache, logits = m.prefill(toks, 4)
    assert cache.length == 12
    assert len(cache.k) == m.shape.n_pre + 4
    assert np.allclose(logits, m.score_last(toks, 4), rtol=1e-12, atol=1e-12)


def test_cached_decode_equals_uncached(tiny):
    _, m = tiny
    prompt = tl_synth.make_tokens(4, m.shape.vocab, 10)
    teacher = tl_synth.make_tokens(5, m.shape.vocab, 6)
    t1, l1 = m.generate_greedy(prompt, 4, 6, cached=True, teacher=teacher)
    t2, l2 = m.generate_greedy(prompt, 4, 6, cached=False, teacher=teacher)
    assert t1 == t2
    assert np.allclose(l1, l2, rtol=1e-12, atol=1e-12)


def test_decode_rejects_other_loop_count(tiny):
    _, m = tiny
    cache, _ = m.prefill([1, 2, 3], 4)
    with pytest.raises(ValueError):
        m.decode(cache, 5, 3)


def test_token_range_checked(tiny):
    _, m = tiny
    with pytest.raises(ValueError):
        m.score_last([0, m.shape.vocab], 1)


# ------------------------------------------------------- Llama comparison ---

def _hf_model(m: ref.LoopedModel, loops: int):
    from transformers import LlamaConfig, LlamaForCausalLM
    sh = m.shape
    cfg = LlamaConfig(
        vocab_size=sh.vocab, hidden_size=sh.d_model, intermediate_size=sh.ffn_dim,
        num_hidden_layers=sh.n_pre + loops, num_attention_heads=sh.n_q_heads,
        num_key_value_heads=sh.n_kv_heads, head_dim=sh.head_dim, rms_norm_eps=sh.rms_eps,
        rope_theta=sh.rope_theta, max_position_embeddings=4096, tie_word_embeddings=False,
        attention_bias=False, mlp_bias=False, attn_implementation="eager")
    hf = LlamaForCausalLM(cfg).double().eval()
    Hq, Hkv, hd, F = sh.n_q_heads, sh.n_kv_heads, sh.head_dim, sh.ffn_dim
    T = torch.tensor
    with torch.no_grad():
        hf.model.embed_tokens.weight.copy_(T(m.embed))
        for layer, blk in zip(hf.model.layers, m.blocks(loops)):
            layer.input_layernorm.weight.copy_(T(blk.attn_norm))
            layer.post_attention_layernorm.weight.copy_(T(blk.ffn_norm))
            layer.self_attn.q_proj.weight.copy_(T(blk.w_qkv[:Hq * hd]))
            layer.self_attn.k_proj.weight.copy_(T(blk.w_qkv[Hq * hd:(Hq + Hkv) * hd]))
            layer.self_attn.v_proj.weight.copy_(T(blk.w_qkv[(Hq + Hkv) * hd:]))
            layer.self_attn.o_proj.weight.copy_(T(blk.w_o))
            layer.mlp.gate_proj.weight.copy_(T(blk.w_gate_up[:F]))
            layer.mlp.up_proj.weight.copy_(T(blk.w_gate_up[F:]))
            layer.mlp.down_proj.weight.copy_(T(blk.w_down))
        hf.model.norm.weight.copy_(T(m.out_norm))
        hf.lm_head.weight.copy_(T(m.head))
    return hf


def _hf_logits(hf, toks):
    with torch.no_grad():
        return hf(torch.tensor(np.asarray(toks, np.int64))[None]).logits[0].numpy()


def _oracle_all_logits(m, toks, loops):
    return m.logits(m.forward(toks, loops))


HF_TOL = 2e-5   # float32 internals of the library; logits are O(1)


@pytest.mark.parametrize("loops", [1, 4])
def test_matches_llama_decoder(tiny_exact, loops):
    _, m = tiny_exact
    toks = tl_synth.make_tokens(6, m.shape.vocab, 33)
    hf = _hf_model(m, loops)
    ours = _oracle_all_logits(m, toks, loops)
    theirs = _hf_logits(hf, toks)
    assert ours.shape == theirs.shape
    err = np.max(np.abs(ours - theirs))
    assert err < HF_TOL, err
    assert np.std(ours) > 0.1   # a real signal, not all zeros


def _interleaved_rope(x, positions, theta):
    x = np.asarray(x, np.float64)
    hd = x.shape[-1]
    ang = ref.rope_angles(positions, hd, theta)[:, None, :]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = b * c + a * s
    return out


_ORIG_GQA = ref.gqa_attention
_ORIG_ROPE = ref.rope


def _modulo_gqa(q, k, v, pos):
    # wrong head mapping: q head h reads kv head h % Hkv
    Hq, Hkv = q.shape[1], k.shape[1]
    idx = np.arange(Hq) % Hkv
    return _ORIG_GQA(q, k[:, idx], v[:, idx], pos)


def _swapped_swiglu(gu, F):
    return ref.silu(gu[..., F:2 * F]) * gu[..., :F]


def _sign_flipped_rope(x, positions, theta):
    return _ORIG_ROPE(x, -np.asarray(positions), theta)


_ORIG_RMS_NORM = ref.rms_norm


def _no_eps_norm(x, g, eps):
    return _ORIG_RMS_NORM(x, g, 1e-1)   # eps far from the model's


MUTATIONS = {
    "interleaved_rope": ("rope", _interleaved_rope),
    "rope_sign": ("rope", _sign_flipped_rope),
    "gqa_modulo_mapping": ("gqa_attention", _modulo_gqa),
    "swiglu_swapped": ("swiglu", _swapped_swiglu),
    "norm_eps_inflated": ("rms_norm", _no_eps_norm),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(tiny_exact, monkeypatch, name):
    _, m = tiny_exact
    toks = tl_synth.make_tokens(6, m.shape.vocab, 33)
    hf = _hf_model(m, 2)
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(ref, attr, fn)
    err = np.max(np.abs(_oracle_all_logits(m, toks, 2) - _hf_logits(hf, toks)))
    assert err > 100 * HF_TOL, (name, err)


# ------------------------------------------------------------ FP16 KV cache ---

def test_kv_cache_holds_fp16_values(tiny, tiny_exact):
    _, m = tiny
    _, mx = tiny_exact
    toks = tl_synth.make_tokens(8, m.shape.vocab, 9)
    c16, _ = m.prefill(toks, 2)
    cx, _ = mx.prefill(toks, 2)
    for layer in range(m.shape.n_pre + 2):
        k16, kx = c16.k[layer], cx.k[layer]
        # stored values are fp16 numbers ...
        assert np.array_equal(k16, k16.astype(np.float16).astype(np.float64))
        assert np.array_equal(c16.v[layer], c16.v[layer].astype(np.float16).astype(np.float64))
    # ... and the first layer's keys are exactly the rounded exact keys
    assert np.array_equal(c16.k[0], cx.k[0].astype(np.float16).astype(np.float64))
    # rounding the cache changes the result only a little
    a = m.score_last(toks, 2)
    b = mx.score_last(toks, 2)
    assert 0 < np.max(np.abs(a - b)) < 1e-2


def test_fp16_storage_rounding():
    # ties go to even: 2049 lies halfway between fp16 neighbours 2048 and 2050
    assert ref.to_fp16_storage(np.array([2049.0]))[0] == 2048.0
    assert ref.to_fp16_storage(np.array([2051.0]))[0] == 2052.0
    assert ref.to_fp16_storage(np.array([1.0 + 2.0 ** -11]))[0] == 1.0
    assert ref.to_fp16_storage(np.array([65504.0]))[0] == 65504.0


def test_dense_block_wiring(tiny):
    # every dense weight is its own linear's dequantisation, in [out][in]
    # orientation (a swapped or transposed operand changes a shape or a value)
    w, _ = tiny
    s = w.shape
    for blk in list(w.pre) + [w.loop]:
        db = ref.dense_block(blk)
        qkv_rows = (s.n_q_heads + 2 * s.n_kv_heads) * s.head_dim
        assert db.w_qkv.shape == (qkv_rows, s.d_model)
        assert db.w_o.shape == (s.d_model, s.n_q_heads * s.head_dim)
        assert db.w_gate_up.shape == (2 * s.ffn_dim, s.d_model)
        assert db.w_down.shape == (s.d_model, s.ffn_dim)
        for name, lin in (("w_qkv", blk.qkv), ("w_o", blk.o), ("w_gate_up", blk.gate_up), ("w_down", blk.down)):
            np.testing.assert_array_equal(getattr(db, name),
                                          ref.dequantize(lin.qweight, lin.scales, lin.qzeros, lin.K))
        np.testing.assert_array_equal(db.attn_norm, np.asarray(blk.attn_norm, np.float64))
        np.testing.assert_array_equal(db.ffn_norm, np.asarray(blk.ffn_norm, np.float64))
        assert not np.array_equal(db.attn_norm, db.ffn_norm)
