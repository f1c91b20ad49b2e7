"""Pins of the oracle's logit lens, token-stable early exit, self-speculative
decoding and prefix-cache fork (CPU only).

Each is pinned to a plain definition it must reduce to:
* the logit lens row i equals score_last with i + 1 loops (the first i + 1
  iterations of a longer run are that run), bit for bit in float64;
* early exit equals a brute-force search over score_last for every loop
  count, and stable_n = 1 stops after one iteration;
* greedy speculation emits exactly the plain greedy continuation at the
  verifier's loop count, whatever the draft loop count and look-ahead, and a
  draft identical to the verifier has every draft accepted;
* a forked prefix cache continues exactly like a fresh prefill of the same
  prefix.
A planted mistake in the acceptance rule (keeping the rejected draft) is
caught by the greedy-equality pin.
"""

import numpy as np
import pytest

import tl_synth
from oracle import ref


@pytest.fixture(scope="module")
def tiny():
    w = tl_synth.make_model_weights(tl_synth.TINY_LM, tl_synth.SEED_TINY)
    return w, ref.LoopedModel(w)


def test_logit_lens_rows_are_shorter_runs(tiny):
    w, om = tiny
    toks = tl_synth.make_tokens(31, w.shape.vocab, 23)
    lens = om.score_logit_lens(toks, 6)
    assert lens.shape == (6, w.shape.vocab)
    for i in range(6):
        assert np.array_equal(lens[i], om.score_last(toks, i + 1)), i


def test_early_exit_matches_brute_force(tiny):
    w, om = tiny
    for seed, n, max_loops, stable_n in ((41, 9, 12, 2), (42, 30, 16, 3), (43, 5, 4, 5)):
        toks = tl_synth.make_tokens(seed, w.shape.vocab, n)
        picks = [ref.greedy(om.score_last(toks, L)) for L in range(1, max_loops + 1)]
        expect_used = max_loops
        for i in range(stable_n - 1, max_loops):
            if len(set(picks[i - stable_n + 1:i + 1])) == 1:
                expect_used = i + 1
                break
        logits, used = om.score_early_exit(toks, max_loops, stable_n)
        assert used == expect_used, (seed, used, expect_used, picks)
        assert np.array_equal(logits, om.score_last(toks, used))
    logits, used = om.score_early_exit(tl_synth.make_tokens(44, w.shape.vocab, 7), 8, 1)
    assert used == 1


@pytest.mark.parametrize("draft_loops,verify_loops,ahead", [(1, 4, 4), (2, 4, 3), (1, 8, 5), (3, 3, 4)])
def test_speculation_equals_plain_greedy(tiny, draft_loops, verify_loops, ahead):
    w, om = tiny
    prompt = tl_synth.make_tokens(50 + draft_loops, w.shape.vocab, 12)
    n = 11
    expect, _ = om.generate_greedy(prompt, verify_loops, n)
    got, stats = om.generate_speculative(prompt, draft_loops, verify_loops, ahead, n)
    assert got == list(expect)
    assert stats["drafted"] >= n - stats["rounds"] + 1
    assert 0 <= stats["accepted"] <= stats["drafted"]
    if draft_loops == verify_loops:
        assert stats["accepted"] == stats["drafted"]
        assert stats["rounds"] == -(-n // ahead)


def test_speculation_pin_catches_keeping_a_rejected_draft(tiny, monkeypatch):
    w, om = tiny
    prompt = tl_synth.make_tokens(60, w.shape.vocab, 12)
    expect, _ = om.generate_greedy(prompt, 8, 10)
    got, stats = om.generate_speculative(prompt, 1, 8, 4, 10)
    assert stats["accepted"] < stats["drafted"], "the pin needs at least one rejection"

    def wrong(self, prompt, draft_loops, verify_loops, draft_ahead, max_tokens):
        # emits the drafts themselves at the first mismatch
        seq, out = [int(t) for t in prompt], []
        while len(out) < max_tokens:
            k = min(draft_ahead, max_tokens - len(out))
            drafts = []
            for _ in range(k):
                drafts.append(ref.greedy(self.score_last(seq + drafts, draft_loops)))
            out += drafts
            seq += drafts
        return out[:max_tokens], {}

    monkeypatch.setattr(ref.LoopedModel, "generate_speculative", wrong)
    bad, _ = om.generate_speculative(prompt, 1, 8, 4, 10)
    assert bad != list(expect)


def test_forked_prefix_continues_like_a_fresh_prefill(tiny):
    w, om = tiny
    toks = tl_synth.make_tokens(70, w.shape.vocab, 30)
    cache, _ = om.prefill(toks[:24], 3)
    fork = cache.fork(16)
    fresh, _ = om.prefill(toks[:16], 3)
    assert fork.length == 16
    for t in toks[16:20]:
        a = om.decode(fork, int(t), 3)
        b = om.decode(fresh, int(t), 3)
        assert np.max(np.abs(a - b)) <= 1e-12
    # the source is untouched by the fork's decoding
    assert cache.length == 24
    with pytest.raises(ValueError):
        cache.fork(25)
