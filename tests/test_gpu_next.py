"""Appending to a lane, greedy self-speculative decoding, the logit lens,
token-stable early exit and the prefix-cache fork, on the GPU against the
fp64 oracle.

Bounds as for the model tests: logits max-abs <= 2e-2, greedy tokens exact
unless the oracle's top-2 margin is below 1e-3 (after such a near-tie a
free-running sequence may legitimately part from the oracle's, so the
comparison stops there).
"""

import numpy as np
import pytest
import torch

import tl_synth
import weight_shared_looped_int4_b200 as tl
from gpu_helpers import DEV, LOGIT_MAX_ABS, ARGMAX_MARGIN, GpuModel, check_argmax, need_gpu
from oracle import ref

pytestmark = pytest.mark.gpu


def _max_abs(a, b):
    return float(np.max(np.abs(np.asarray(a) - np.asarray(b))))


@pytest.fixture(scope="module")
def tiny():
    need_gpu()
    w = tl_synth.make_model_weights(tl_synth.TINY_LM, tl_synth.SEED_TINY)
    om = ref.LoopedModel(w)
    gm = GpuModel(w, max_loops=16, max_ctx=256, max_lanes=8)
    yield w, om, gm
    gm.close()


def _extend(gm, lane, tokens, logits=True):
    V = gm.shape.vocab
    n = len(tokens)
    d_tok = torch.as_tensor(np.asarray(tokens, np.int32), device=DEV)
    lg = torch.empty((n, V), dtype=torch.float32, device=DEV) if logits else None
    am = torch.empty(n, dtype=torch.int32, device=DEV) if logits else None
    tl.tl_extend(gm.handle, lane, d_tok, n, lg, am)
    torch.cuda.synchronize()
    if not logits:
        return None, None
    return lg.cpu().numpy().astype(np.float64), am.cpu().numpy()


def _compare_free_running(got, oracle_tokens, oracle_logits, where):
    """Token lists agree up to the first position whose oracle margin is a
    near-tie; returns how many positions were compared."""
    for i, (g, o) in enumerate(zip(got, oracle_tokens)):
        if g != o:
            assert ref.top2_margin(oracle_logits[i]) < ARGMAX_MARGIN, f"{where}: token {i}: {g} != {o}"
            return i
    return len(got)


# ---------------------------------------------------------------- extend ---

def test_extend_every_position(tiny):
    # 20-token prompt, then 6 appended tokens with per-position logits
    w, om, gm = tiny
    gm.set_path(tl.DECODE_AUTO)
    toks = tl_synth.make_tokens(301, w.shape.vocab, 40)
    L = 3
    gm.prefill_lane(0, toks[:20], L, logits=False)
    lg, am = _extend(gm, 0, toks[20:26])
    cache, _ = om.prefill(toks[:20], L)
    h = om.forward(toks[20:26], L, cache)
    expect = om.logits(h)
    for i in range(6):
        assert _max_abs(lg[i], expect[i]) <= LOGIT_MAX_ABS, i
        check_argmax(int(am[i]), expect[i], f"position {20 + i}")
    assert tl.tl_lane_length(gm.handle, 0) == 26
    # and decode continues from the appended positions
    glg, gam = gm.decode([0], [int(toks[26])], [L])
    expect = om.decode(cache, int(toks[26]), L)
    assert _max_abs(glg[0], expect) <= LOGIT_MAX_ABS


def test_chunked_prefill_tensor_core_chunks(tiny):
    # a 100-token prompt as 40 + 36 + 24 (the first two chunks take the
    # tensor-core path at positions > 0), then decode steps
    w, om, gm = tiny
    gm.set_path(tl.DECODE_AUTO)
    toks = tl_synth.make_tokens(302, w.shape.vocab, 104)
    L = 4
    gm.prefill_lane(1, toks[:40], L, logits=False)
    _extend(gm, 1, toks[40:76], logits=False)
    _extend(gm, 1, toks[76:100], logits=False)
    cache, _ = om.prefill(toks[:100], L)
    for i in range(100, 104):
        glg, gam = gm.decode([1], [int(toks[i])], [L])
        expect = om.decode(cache, int(toks[i]), L)
        assert _max_abs(glg[0], expect) <= LOGIT_MAX_ABS, i
        check_argmax(int(gam[0]), expect, f"position {i}")


def test_extend_errors(tiny):
    w, om, gm = tiny
    d = torch.zeros(20, dtype=torch.int32, device=DEV)
    with pytest.raises(tl.TLError) as e:
        tl.tl_extend(gm.handle, 7, d, 4)          # never prefilled
    assert e.value.status == tl.TL_ERR_NOT_PREFILLED
    gm.prefill_lane(2, [1, 2, 3], 2, logits=False)
    lg = torch.empty((17, w.shape.vocab), dtype=torch.float32, device=DEV)
    with pytest.raises(tl.TLError) as e:
        tl.tl_extend(gm.handle, 2, d, 17, lg)     # per-position logits beyond 16 rows
    assert e.value.status == tl.TL_ERR_UNSUPPORTED
    gm.prefill_lane(2, list(range(250)), 2, logits=False)
    with pytest.raises(tl.TLError) as e:
        tl.tl_extend(gm.handle, 2, d, 7)          # past max_ctx
    assert e.value.status == tl.TL_ERR_CONTEXT_FULL


# ----------------------------------------------------------- speculation ---

@pytest.mark.parametrize("draft_loops,ahead", [(1, 4), (2, 3), (4, 5)])
def test_speculative_equals_greedy(tiny, draft_loops, ahead):
    w, om, gm = tiny
    gm.set_path(tl.DECODE_AUTO)
    L, P, n = 4, 20, 24
    prompt = tl_synth.make_tokens(310 + draft_loops, w.shape.vocab, P + 1)
    o_tokens, o_logits = om.generate_greedy(prompt, L, n)
    gm.prefill_lane(3, prompt[:P], L, logits=False)
    first = torch.as_tensor(prompt[P:P + 1], device=DEV)
    out = torch.full((n,), -1, dtype=torch.int32, device=DEV)
    stats = tl.tl_generate_speculative(gm.handle, 3, first, n, draft_loops, ahead, out)
    torch.cuda.synchronize()
    got = [int(t) for t in out.cpu().numpy()]
    compared = _compare_free_running(got, o_tokens, o_logits, "speculative")
    assert compared >= 8
    assert tl.tl_lane_length(gm.handle, 3) == P + n
    assert stats["rounds"] >= -(-n // ahead)
    assert 0 <= stats["accepted"] <= stats["drafted"]
    if draft_loops == L:
        assert stats["accepted"] == stats["drafted"]
    if compared == n:
        # the lane continues like a plain greedy decode of the same tokens
        glg, _ = gm.decode([3], [got[-1]], [L])
        cache, _ = om.prefill(list(prompt) + got[:-1], L)
        assert _max_abs(glg[0], om.decode(cache, got[-1], L)) <= LOGIT_MAX_ABS


def test_speculative_errors(tiny):
    w, om, gm = tiny
    gm.prefill_lane(4, [5, 6, 7], 2, logits=False)
    first = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = torch.zeros(8, dtype=torch.int32, device=DEV)
    for args in ((4, first, 8, 3, 2, out),      # draft loops above the lane's
                 (4, first, 8, 1, 17, out),     # look-ahead beyond 16
                 (4, first, 0, 1, 2, out)):
        with pytest.raises(tl.TLError) as e:
            tl.tl_generate_speculative(gm.handle, *args)
        assert e.value.status == tl.TL_ERR_INVALID_ARG
    with pytest.raises(tl.TLError) as e:
        tl.tl_generate_speculative(gm.handle, 6, first, 8, 1, 2, out)
    assert e.value.status == tl.TL_ERR_NOT_PREFILLED


# ------------------------------------------------- logit lens, early exit ---

def _lens(gm, toks, loops):
    V = gm.shape.vocab
    d_tok = torch.as_tensor(np.asarray(toks, np.int32), device=DEV)
    lg = torch.empty((loops, V), dtype=torch.float32, device=DEV)
    am = torch.empty(loops, dtype=torch.int32, device=DEV)
    tl.tl_score_logit_lens(gm.handle, d_tok, len(toks), loops, lg, am)
    torch.cuda.synchronize()
    return lg.cpu().numpy().astype(np.float64), am.cpu().numpy()


@pytest.mark.parametrize("n,loops", [(9, 6), (40, 5)])
def test_logit_lens(tiny, n, loops):
    w, om, gm = tiny
    toks = tl_synth.make_tokens(320 + n, w.shape.vocab, n)
    lg, am = _lens(gm, toks, loops)
    expect = om.score_logit_lens(toks, loops)
    for i in range(loops):
        assert _max_abs(lg[i], expect[i]) <= LOGIT_MAX_ABS, i
        check_argmax(int(am[i]), expect[i], f"iteration {i + 1}")
    # the last row is score_last
    sl, _ = gm.score_last(toks, loops)
    assert _max_abs(sl, lg[-1]) <= 1e-3


@pytest.mark.parametrize("seed,n,max_loops,stable_n", [(331, 9, 12, 2), (332, 36, 16, 3), (333, 5, 6, 1)])
def test_early_exit(tiny, seed, n, max_loops, stable_n):
    w, om, gm = tiny
    toks = tl_synth.make_tokens(seed, w.shape.vocab, n)
    d_tok = torch.as_tensor(np.asarray(toks, np.int32), device=DEV)
    lg = torch.empty(w.shape.vocab, dtype=torch.float32, device=DEV)
    am = torch.empty(1, dtype=torch.int32, device=DEV)
    used = tl.tl_score_early_exit(gm.handle, d_tok, n, max_loops, stable_n, lg, am)
    torch.cuda.synchronize()
    o_logits, o_used = om.score_early_exit(toks, max_loops, stable_n)
    if used != o_used:
        # only a near-tie in one of the iterations' greedy tokens may move it
        lens = om.score_logit_lens(toks, max(used, o_used))
        assert min(ref.top2_margin(r) for r in lens) < ARGMAX_MARGIN, (used, o_used)
        return
    assert _max_abs(lg.cpu().numpy(), o_logits) <= LOGIT_MAX_ABS
    check_argmax(int(am.item()), o_logits, "early exit")


# ------------------------------------------------------------ prefix fork ---

def test_fork_prefix(tiny):
    w, om, gm = tiny
    gm.set_path(tl.DECODE_AUTO)
    toks = tl_synth.make_tokens(340, w.shape.vocab, 50)
    L = 3
    gm.prefill_lane(5, toks[:40], L, logits=False)     # the prefix cache
    gm.prefill_lane(6, toks[:40], L, logits=False)     # a fresh copy of it
    tl.tl_lane_fork(gm.handle, 5, 7, 40)
    torch.cuda.synchronize()
    assert tl.tl_lane_length(gm.handle, 7) == 40
    for i in range(40, 44):      # the fork decodes bit for bit like the fresh lane
        a, _ = gm.decode([7], [int(toks[i])], [L])
        b, _ = gm.decode([6], [int(toks[i])], [L])
        assert np.array_equal(a, b), i
    # a shorter fork continues like the oracle's prefill of that prefix
    tl.tl_lane_fork(gm.handle, 5, 7, 30)
    cache, _ = om.prefill(toks[:30], L)
    for i in range(30, 34):
        glg, gam = gm.decode([7], [int(toks[i])], [L])
        expect = om.decode(cache, int(toks[i]), L)
        assert _max_abs(glg[0], expect) <= LOGIT_MAX_ABS, i
        check_argmax(int(gam[0]), expect, f"fork position {i}")
    # the source lane is untouched
    assert tl.tl_lane_length(gm.handle, 5) == 40
    with pytest.raises(tl.TLError) as e:
        tl.tl_lane_fork(gm.handle, 5, 7, 41)
    assert e.value.status == tl.TL_ERR_INVALID_ARG


# ----------------------------------------------------------- the 400M LM ---

@pytest.fixture(scope="module")
def lm():
    need_gpu()
    w = tl_synth.make_model_weights(tl_synth.LOOPED_LM, tl_synth.SEED_LM)
    om = ref.LoopedModel(w)
    gm = GpuModel(w, max_loops=8, max_ctx=256, max_lanes=2)
    yield w, om, gm
    gm.close()


def test_lm_speculative(lm):
    # draft with 2 loops, verify with 8, 4 ahead, 32 tokens after a 128-token
    # prompt
    w, om, gm = lm
    L, P, n = 8, 128, 32
    prompt = tl_synth.make_tokens(tl_synth.SEED_LM, w.shape.vocab, P + 1)
    o_tokens, o_logits = om.generate_greedy(prompt, L, n)
    gm.prefill_lane(0, prompt[:P], L, logits=False)
    first = torch.as_tensor(prompt[P:P + 1], device=DEV)
    out = torch.full((n,), -1, dtype=torch.int32, device=DEV)
    tl.tl_generate_speculative(gm.handle, 0, first, n, 2, 4, out)
    torch.cuda.synchronize()
    got = [int(t) for t in out.cpu().numpy()]
    assert _compare_free_running(got, o_tokens, o_logits, "LM speculative") >= 8


def test_lm_logit_lens(lm):
    w, om, gm = lm
    toks = tl_synth.make_tokens(17, w.shape.vocab, 40)
    lg, am = _lens(gm, toks, 8)
    expect = om.score_logit_lens(toks, 8)
    for i in range(8):
        assert _max_abs(lg[i], expect[i]) <= LOGIT_MAX_ABS, i
        check_argmax(int(am[i]), expect[i], f"iteration {i + 1}")
