"""The looped model end to end on the GPU against the fp64 oracle.

Workloads:
* tiny looped LM (d 256, 4/2 heads of 64, F 1024, V 512, 1 pre block, L = 4):
  32-token prompt, then 8 greedy decode steps, batch 1;
* the ~400M-unique looped LM (d 2048, 16/4 heads of 128, F 5632, V 32000,
  2 pre blocks, L = 8): 128-token prompt prefilled with no logits, then greedy
  decode steps at batch 1;
* the same model with per-lane loops drawn from {4, 8, 16}.

Decoding is teacher-forced with the oracle's tokens, so an allowed near-tie
argmax flip cannot change later steps.  Bounds: logits max-abs <= 2e-2, argmax
exact unless the oracle's top-2 margin is < 1e-3.

Decode tests run on both decode paths: the single persistent kernel per step
("fused") and one kernel per projection / attention / head ("layered").
"""

import numpy as np
import pytest
import torch

import tl_synth
import weight_shared_looped_int4_b200 as tl
from gpu_helpers import DEV, LOGIT_MAX_ABS, GpuModel, check_argmax, need_gpu
from oracle import ref

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny():
    need_gpu()
    w = tl_synth.make_model_weights(tl_synth.TINY_LM, tl_synth.SEED_TINY)
    om = ref.LoopedModel(w)
    gm = GpuModel(w, max_loops=16, max_ctx=256, max_lanes=16)
    yield w, om, gm
    gm.close()


def _max_abs(a, b):
    return float(np.max(np.abs(np.asarray(a) - np.asarray(b))))


# Decode forms: the single-kernel step, the per-op step through the clustered
# QKV + attention kernel, and the per-op step through the QKV GEMV + split-KV
# attention (a model's default between the last two follows its max_lanes).
@pytest.fixture(params=["fused", "layered", "split"])
def path(request):
    return request.param


def _set_clustered(gm, enable):
    """Select the per-op form; False where the clustered kernel does not fit."""
    try:
        tl.tl_model_set_clustered_decode(gm.handle, enable)
        return enable
    except tl.TLError as e:
        assert enable and e.status == tl.TL_ERR_UNSUPPORTED
        tl.tl_model_set_clustered_decode(gm.handle, False)
        return False


def _use(gm, path):
    if path == "fused":
        gm.set_path(tl.DECODE_FUSED)
    else:
        gm.set_path(tl.DECODE_LAYERED)
        _set_clustered(gm, path == "layered")
    return gm


def test_tiny_prefill_decode(tiny, path):
    w, om, gm = tiny
    _use(gm, path)
    L, P, steps = 4, 32, 8
    prompt = tl_synth.make_tokens(tl_synth.SEED_TINY, w.shape.vocab, P + 1)
    # oracle: logits at positions P .. P+steps-1 (prefill of P+1 ids = first decode step)
    o_tokens, o_logits = om.generate_greedy(prompt, L, steps)
    # GPU: prefill P ids with logits of position P-1, then decode prompt[P], ...
    lg, am = gm.prefill_lane(0, prompt[:P], L)
    _, o_prefill_logits = om.prefill(prompt[:P], L)
    assert _max_abs(lg, o_prefill_logits) <= LOGIT_MAX_ABS
    check_argmax(am, o_prefill_logits, "prefill")
    fed = int(prompt[P])
    for i in range(steps):
        glg, gam = gm.decode([0], [fed], [L])
        err = _max_abs(glg[0], o_logits[i])
        assert err <= LOGIT_MAX_ABS, (i, err)
        check_argmax(int(gam[0]), o_logits[i], f"step {i}")
        fed = o_tokens[i]
    assert tl.tl_lane_length(gm.handle, 0) == P + steps


def test_tiny_score_last(tiny):
    w, om, gm = tiny
    for n, L in ((1, 1), (17, 3), (100, 16)):
        toks = tl_synth.make_tokens(n + L, w.shape.vocab, n)
        lg, am = gm.score_last(toks, L)
        expect = om.score_last(toks, L)
        assert _max_abs(lg, expect) <= LOGIT_MAX_ABS
        check_argmax(am, expect, "score_last")


def test_tiny_cached_equals_uncached_on_gpu(tiny, path):
    # Decode step i must agree with a fresh uncached forward of the prefix.
    w, om, gm = tiny
    _use(gm, path)
    prompt = tl_synth.make_tokens(55, w.shape.vocab, 20)
    gm.prefill_lane(1, prompt[:12], 4, logits=False)
    seq = list(prompt[:12])
    for i in range(12, 20):
        glg, _ = gm.decode([1], [int(prompt[i])], [4])
        seq.append(int(prompt[i]))
        ulg, _ = gm.score_last(seq, 4)
        assert _max_abs(glg[0], ulg) <= 2e-3


def test_tiny_looped_equals_flattened_on_gpu(tiny):
    # A model whose pre blocks are [pre..., loop x (L-1)] and whose loop block
    # runs once is the same computation with distinct weight copies.
    w, om, gm = tiny
    L = 4
    flat = tl_synth.ModelWeights(
        shape=tl_synth.ModelShape(**{**w.shape.__dict__, "n_pre": w.shape.n_pre + L - 1}),
        embed=w.embed, out_norm=w.out_norm, head=w.head,
        pre=list(w.pre) + [w.loop] * (L - 1), loop=w.loop)
    fm = GpuModel(flat, max_loops=1, max_ctx=64, max_lanes=1)
    try:
        toks = tl_synth.make_tokens(99, w.shape.vocab, 40)
        a, _ = gm.score_last(toks, L)
        b, _ = fm.score_last(toks, 1)
        assert np.array_equal(a, b)
    finally:
        fm.close()


def test_tiny_per_lane_loops_independent(tiny, path):
    # Lanes with loops 4, 8, 16 decoded together give bitwise the results of
    # decoding each lane alone.
    w, om, gm = tiny
    _use(gm, path)
    loops = [4, 16, 8]
    prompts = tl_synth.make_lane_prompts(7, w.shape.vocab, 3, 10)
    nxt = [5, 6, 7]
    for lane, L in enumerate(loops):
        gm.prefill_lane(2 + lane, prompts[lane], L, logits=False)
    together, _ = gm.decode([2, 3, 4], nxt, loops)
    for lane, L in enumerate(loops):
        gm.prefill_lane(2 + lane, prompts[lane], L, logits=False)
    for lane, L in enumerate(loops):
        alone, _ = gm.decode([2 + lane], [nxt[lane]], [L])
        assert np.array_equal(alone[0], together[lane])
        # and against the oracle
        cache, _ = om.prefill(prompts[lane], L)
        expect = om.decode(cache, nxt[lane], L)
        assert _max_abs(alone[0], expect) <= LOGIT_MAX_ABS


def test_tiny_paths_agree_and_auto(tiny):
    # Both decode paths on the same step: same argmax, logits within rounding
    # of each other; asking FUSED for more than 4 lanes is refused and AUTO
    # takes any lane count.
    w, om, gm = tiny
    prompts = tl_synth.make_lane_prompts(21, w.shape.vocab, 6, 9)
    res = {}
    for p in (tl.DECODE_FUSED, tl.DECODE_LAYERED):
        gm.set_path(p)
        for lane in range(6):
            gm.prefill_lane(lane, prompts[lane, :8], 4, logits=False)
        res[p] = gm.decode([0, 1], [int(prompts[0, 8]), int(prompts[1, 8])], [4, 4])
    assert np.array_equal(res[tl.DECODE_FUSED][1], res[tl.DECODE_LAYERED][1])
    assert _max_abs(res[tl.DECODE_FUSED][0], res[tl.DECODE_LAYERED][0]) <= 1e-3
    gm.set_path(tl.DECODE_FUSED)
    with pytest.raises(tl.TLError) as e:
        gm.decode(list(range(5)), [1] * 5, [4] * 5)
    assert e.value.status == tl.TL_ERR_UNSUPPORTED
    gm.set_path(tl.DECODE_AUTO)
    lg, _ = gm.decode(list(range(5)), [int(p[8]) for p in prompts[:5]], [4] * 5)
    for lane in range(2, 5):   # lanes 0, 1 already took one step above
        cache, _ = om.prefill(prompts[lane, :8], 4)
        assert _max_abs(lg[lane], om.decode(cache, int(prompts[lane, 8]), 4)) <= LOGIT_MAX_ABS


def test_tiny_long_context(path):
    # A 1100-token context: the clustered decode kernel's key split exceeds
    # one 64-key chunk (later chunks are loaded inside the kernel), and the
    # single-kernel step uses its long-context splits with a ticketed merge.
    need_gpu()
    w = tl_synth.make_model_weights(tl_synth.TINY_LM, tl_synth.SEED_TINY)
    om = ref.LoopedModel(w)
    gm = GpuModel(w, max_loops=2, max_ctx=1104, max_lanes=1)
    try:
        _use(gm, path)
        L, P, steps = 2, 1100, 2
        prompt = tl_synth.make_tokens(1100, w.shape.vocab, P + 1)
        o_tokens, o_logits = om.generate_greedy(prompt, L, steps)
        gm.prefill_lane(0, prompt[:P], L, logits=False)
        fed = int(prompt[P])
        for i in range(steps):
            glg, gam = gm.decode([0], [fed], [L])
            err = _max_abs(glg[0], o_logits[i])
            assert err <= LOGIT_MAX_ABS, (i, err)
            check_argmax(int(gam[0]), o_logits[i], f"step {i}")
            fed = o_tokens[i]
    finally:
        gm.close()


def test_width_not_multiple_of_512(path):
    # d_model 640: the head's k items (512 wide at d_model 2048) must divide
    # d_model, so the head streams 128-wide items here; prefill on the tensor
    # cores (40 tokens), then greedy decode teacher-forced with the oracle.
    need_gpu()
    shape = tl_synth.ModelShape(d_model=640, n_q_heads=10, n_kv_heads=5, head_dim=64,
                                ffn_dim=1280, vocab=1024, n_pre=1)
    w = tl_synth.make_model_weights(shape, 640)
    om = ref.LoopedModel(w)
    gm = GpuModel(w, max_loops=4, max_ctx=64, max_lanes=1)
    try:
        _use(gm, path)
        L, P, steps = 3, 40, 3
        prompt = tl_synth.make_tokens(641, shape.vocab, P + 1)
        o_tokens, o_logits = om.generate_greedy(prompt, L, steps)
        gm.prefill_lane(0, prompt[:P], L, logits=False)
        fed = int(prompt[P])
        for i in range(steps):
            glg, gam = gm.decode([0], [fed], [L])
            err = _max_abs(glg[0], o_logits[i])
            assert err <= LOGIT_MAX_ABS, (i, err)
            check_argmax(int(gam[0]), o_logits[i], f"step {i}")
            fed = o_tokens[i]
    finally:
        gm.close()


def test_width_not_multiple_of_512_five_lanes():
    # The same width with five lanes in one step: beyond the single-kernel
    # head's four rows, the standalone head kernel takes the step; its stages
    # must divide the 640-wide rows too.
    need_gpu()
    shape = tl_synth.ModelShape(d_model=640, n_q_heads=10, n_kv_heads=5, head_dim=64,
                                ffn_dim=1280, vocab=1024, n_pre=1)
    w = tl_synth.make_model_weights(shape, 640)
    om = ref.LoopedModel(w)
    gm = GpuModel(w, max_loops=4, max_ctx=64, max_lanes=5)
    try:
        gm.set_path(tl.DECODE_AUTO)
        prompts = tl_synth.make_lane_prompts(642, shape.vocab, 5, 9)
        for lane in range(5):
            gm.prefill_lane(lane, prompts[lane, :8], 2, logits=False)
        lg, am = gm.decode(list(range(5)), [int(p[8]) for p in prompts], [2] * 5)
        for lane in range(5):
            cache, _ = om.prefill(prompts[lane, :8], 2)
            o = om.decode(cache, int(prompts[lane, 8]), 2)
            assert _max_abs(lg[lane], o) <= LOGIT_MAX_ABS, lane
            check_argmax(int(am[lane]), o, f"lane {lane}")
    finally:
        gm.close()


def test_tiny_errors(tiny):
    w, om, gm = tiny
    gm.set_path(tl.DECODE_AUTO)
    gm.prefill_lane(5, [1, 2, 3], 4, logits=False)
    with pytest.raises(tl.TLError) as e:
        gm.decode([5], [1], [8])
    assert e.value.status == tl.TL_ERR_LOOPS_MISMATCH
    with pytest.raises(tl.TLError) as e:
        gm.decode([15], [1], [4])
    assert e.value.status == tl.TL_ERR_NOT_PREFILLED
    with pytest.raises(tl.TLError) as e:
        gm.decode([5, 5], [1, 1], [4, 4])
    assert e.value.status == tl.TL_ERR_INVALID_ARG
    with pytest.raises(tl.TLError) as e:
        gm.prefill_lane(0, [1] * 300, 4)
    assert e.value.status == tl.TL_ERR_CONTEXT_FULL
    # a token id out of range is replaced by 0 and flagged, not trapped
    tl.tl_check_device_error(gm.handle)
    gm.score_last([1, w.shape.vocab + 5], 2)
    with pytest.raises(tl.TLError) as e:
        tl.tl_check_device_error(gm.handle)
    assert e.value.status == tl.TL_ERR_DEVICE_FLAG
    tl.tl_check_device_error(gm.handle)   # cleared


def test_tiny_bounded_wait_times_out(tiny):
    # A grid barrier made to expect one CTA more than the step launches: its
    # bounded wait (0.5 s) runs out, the step ends instead of hanging, the
    # device flag reports it, and the next steps on the same model are
    # correct again.
    import time
    w, om, gm = tiny
    gm.set_path(tl.DECODE_FUSED)
    prompt = tl_synth.make_tokens(77, w.shape.vocab, 12)
    tl.tl_check_device_error(gm.handle)
    gm.prefill_lane(9, prompt[:10], 2, logits=False)
    tl.tl_model_set_wait_test(gm.handle, 1)
    try:
        t0 = time.perf_counter()
        gm.decode([9], [int(prompt[10])], [2])
        waited = time.perf_counter() - t0
    finally:
        tl.tl_model_set_wait_test(gm.handle, 0)
    assert 0.3 < waited < 30.0, waited
    with pytest.raises(tl.TLError) as e:
        tl.tl_check_device_error(gm.handle)
    assert e.value.status == tl.TL_ERR_DEVICE_FLAG
    assert "wait" in str(e.value)
    tl.tl_check_device_error(gm.handle)   # cleared
    gm.prefill_lane(9, prompt[:10], 2, logits=False)
    cache, _ = om.prefill(prompt[:10], 2)
    for i in (10, 11):
        glg, gam = gm.decode([9], [int(prompt[i])], [2])
        expect = om.decode(cache, int(prompt[i]), 2)
        assert _max_abs(glg[0], expect) <= LOGIT_MAX_ABS
        check_argmax(int(gam[0]), expect, f"after the wait test, position {i}")
    tl.tl_check_device_error(gm.handle)


def test_tiny_context_full(tiny, path):
    w, om, gm = tiny
    _use(gm, path)
    gm.prefill_lane(6, list(range(255)), 1, logits=False)
    gm.decode([6], [1], [1])
    with pytest.raises(tl.TLError) as e:
        gm.decode([6], [1], [1])
    assert e.value.status == tl.TL_ERR_CONTEXT_FULL


# --------------------------------------------------------- the ~400M model ---

@pytest.fixture(scope="module")
def lm():
    need_gpu()
    w = tl_synth.make_model_weights(tl_synth.LOOPED_LM, tl_synth.SEED_LM)
    om = ref.LoopedModel(w)
    gm = GpuModel(w, max_loops=16, max_ctx=2048, max_lanes=16)
    om.memo = {}   # oracle results shared by the two decode paths
    yield w, om, gm
    gm.close()


def _memo(om, key, fn):
    if key not in om.memo:
        om.memo[key] = fn()
    return om.memo[key]


def test_lm_prefill_then_decode(lm, path):
    # The whole benchmarked sequence: a 128-token prompt prefilled with no
    # logits, then all 128 greedy decode steps, every step's logits and argmax
    # checked (teacher-forced with the oracle's tokens).
    w, om, gm = lm
    _use(gm, path)
    L, P, steps = 8, 128, 128
    prompt = tl_synth.make_tokens(tl_synth.SEED_LM, w.shape.vocab, P + 1)
    o_tokens, o_logits = _memo(om, "greedy", lambda: om.generate_greedy(prompt, L, steps))
    gm.prefill_lane(0, prompt[:P], L, logits=False)
    fed = int(prompt[P])
    for i in range(steps):
        glg, gam = gm.decode([0], [fed], [L])
        err = _max_abs(glg[0], o_logits[i])
        assert err <= LOGIT_MAX_ABS, (i, err)
        check_argmax(int(gam[0]), o_logits[i], f"step {i}")
        fed = o_tokens[i]


def test_lm_score_last(lm):
    w, om, gm = lm
    toks = tl_synth.make_tokens(17, w.shape.vocab, 77)
    for L in (1, 8):
        lg, am = gm.score_last(toks, L)
        expect = om.score_last(toks, L)
        assert _max_abs(lg, expect) <= LOGIT_MAX_ABS
        check_argmax(am, expect, f"L={L}")


def test_lm_lanes_per_lane_loops(lm, path):
    # Lanes with loops drawn from {4, 8, 16}, prompts of 512 ids; two lanes
    # are checked against the oracle.
    w, om, gm = lm
    _use(gm, path)
    n_lanes, P = 4, 512
    loops = [int(v) for v in tl_synth.make_lane_loops(tl_synth.SEED_LSWEEP, n_lanes)]
    prompts = tl_synth.make_lane_prompts(tl_synth.SEED_LSWEEP, w.shape.vocab, n_lanes, P + 1)
    lanes = list(range(n_lanes))
    for i in lanes:
        gm.prefill_lane(i, prompts[i, :P], loops[i], logits=False)
    together, am = gm.decode(lanes, [int(p[P]) for p in prompts], loops)
    for i in (0, n_lanes - 1):
        # = decode step at position P
        expect = _memo(om, ("lane", i), lambda: om.score_last(prompts[i, :P + 1], loops[i]))
        assert _max_abs(together[i], expect) <= LOGIT_MAX_ABS
        check_argmax(int(am[i]), expect, f"lane {i}")


def test_lm_loops_sweep(lm):
    # Loops L in {1, 2, 4, 8, 16} on one lane: a 512-token prompt prefilled
    # with last-position logits, then two cached decode steps.
    w, om, gm = lm
    gm.set_path(tl.DECODE_AUTO)
    P = 512
    prompt = tl_synth.make_tokens(tl_synth.SEED_LSWEEP, w.shape.vocab, P + 2)
    for L in (1, 2, 4, 8, 16):
        cache, o_pre = om.prefill(prompt[:P], L)
        lg, am = gm.prefill_lane(7, prompt[:P], L)
        assert _max_abs(lg, o_pre) <= LOGIT_MAX_ABS, (L, "prefill")
        check_argmax(am, o_pre, f"L={L} prefill")
        for i in range(2):
            expect = om.decode(cache, int(prompt[P + i]), L)
            glg, gam = gm.decode([7], [int(prompt[P + i])], [L])
            err = _max_abs(glg[0], expect)
            assert err <= LOGIT_MAX_ABS, (L, i, err)
            check_argmax(int(gam[0]), expect, f"L={L} step {i}")


def test_lm_sixteen_lanes_every_lane(lm):
    # All 16 lanes in one decode step, per-lane loops drawn from {4, 8, 16},
    # ragged prompt lengths; every lane is compared with its own single-lane
    # oracle run, on two consecutive steps.
    # Both per-op forms: the model's default (GEMV + split-KV: 16 lanes) and
    # the clustered kernel (eight launches of two rows per layer).
    w, om, gm = lm
    n = 16
    loops = [int(v) for v in tl_synth.make_lane_loops(tl_synth.SEED_LSWEEP + 16, n)]
    prompts = tl_synth.make_lane_prompts(tl_synth.SEED_LSWEEP + 16, w.shape.vocab, n, 100)
    lens = [40 + 4 * i for i in range(n)]       # 40 .. 100 tokens
    feeds = [[int(prompts[i, lens[i] - 1]) ^ 1 for i in range(n)]]   # any in-range ids
    feeds.append([int((t * 7 + 3) % w.shape.vocab) for t in feeds[0]])
    expects = [[], []]
    for i in range(n):
        cache = om.prefill(prompts[i, :lens[i]], loops[i])[0]
        for step in range(2):
            expects[step].append(om.decode(cache, feeds[step][i], loops[i]))
    for clustered in (False, True):
        gm.set_path(tl.DECODE_LAYERED)
        assert _set_clustered(gm, clustered) == clustered
        for i in range(n):
            gm.prefill_lane(i, prompts[i, :lens[i]], loops[i], logits=False)
        for step in range(2):
            lg, am = gm.decode(list(range(n)), feeds[step], loops)
            for i in range(n):
                err = _max_abs(lg[i], expects[step][i])
                assert err <= LOGIT_MAX_ABS, (clustered, step, i, loops[i], err)
                check_argmax(int(am[i]), expects[step][i], f"clustered {clustered} step {step} lane {i}")
    _set_clustered(gm, False)


def test_lm_long_context(lm):
    # One lane decoding at the end of the 2048-token context: a 2040-token
    # prompt at L = 2, then decode steps up to position 2047 (the last slot).
    # Both per-op forms (the clustered kernel's key split spans several
    # 64-key chunks per rank here).
    w, om, gm = lm
    L, P = 2, 2040
    prompt = tl_synth.make_tokens(tl_synth.SEED_LSWEEP + 2048, w.shape.vocab, 2048)
    cache, _ = om.prefill(prompt[:P], L)
    expects = [om.decode(cache, int(prompt[pos]), L) for pos in range(P, 2048)]
    for clustered in (False, True):
        gm.set_path(tl.DECODE_LAYERED)
        assert _set_clustered(gm, clustered) == clustered
        gm.prefill_lane(8, prompt[:P], L, logits=False)
        for pos in range(P, 2048):
            glg, gam = gm.decode([8], [int(prompt[pos])], [L])
            err = _max_abs(glg[0], expects[pos - P])
            assert err <= LOGIT_MAX_ABS, (clustered, pos, err)
            check_argmax(int(gam[0]), expects[pos - P], f"clustered {clustered} position {pos}")
    _set_clustered(gm, False)


def test_lm_benchmark_model_one_lane(lm):
    # The benchmark's own configuration: a model built for one lane (so every
    # clustered launch carries one row), the 128-token prompt prefilled with
    # no logits, then all 128 teacher-forced greedy steps (contexts 129 ..
    # 256), every step checked.
    w, om, _ = lm
    L, P, steps = 8, 128, 128
    prompt = tl_synth.make_tokens(tl_synth.SEED_LM, w.shape.vocab, P + 1)
    o_tokens, o_logits = _memo(om, "greedy", lambda: om.generate_greedy(prompt, L, steps))
    gm = GpuModel(w, max_loops=8, max_ctx=P + steps, max_lanes=1)
    try:
        gm.set_path(tl.DECODE_LAYERED)
        gm.prefill_lane(0, prompt[:P], L, logits=False)
        fed = int(prompt[P])
        for i in range(steps):
            glg, gam = gm.decode([0], [fed], [L])
            err = _max_abs(glg[0], o_logits[i])
            assert err <= LOGIT_MAX_ABS, (i, err)
            check_argmax(int(gam[0]), o_logits[i], f"step {i}")
            fed = o_tokens[i]
    finally:
        gm.close()


@pytest.mark.parametrize("kv_mode", [tl.TL_KV_FP16, tl.TL_KV_INT8])
def test_tiny_one_lane_decode_250_to_262(kv_mode):
    # A one-lane model decoding from 250 to 262 cached positions (the
    # clustered kernel's key split then changes length between steps) in
    # both cache modes, against the oracle in the same mode.
    need_gpu()
    w = tl_synth.make_model_weights(tl_synth.TINY_LM, tl_synth.SEED_TINY)
    om = ref.LoopedModel(w, kv_mode="int8" if kv_mode == tl.TL_KV_INT8 else None)
    bound = 5e-2 if kv_mode == tl.TL_KV_INT8 else LOGIT_MAX_ABS   # see test_gpu_kv8.INT8_LOGIT_MAX_ABS
    gm = GpuModel(w, max_loops=4, max_ctx=272, max_lanes=1, kv_mode=kv_mode)
    try:
        gm.set_path(tl.DECODE_LAYERED)
        L, P = 3, 250
        toks = tl_synth.make_tokens(909, w.shape.vocab, P + 12)
        cache, _ = om.prefill(toks[:P], L)
        gm.prefill_lane(0, toks[:P], L, logits=False)
        for pos in range(P, P + 12):
            expect = om.decode(cache, int(toks[pos]), L)
            glg, gam = gm.decode([0], [int(toks[pos])], [L])
            err = _max_abs(glg[0], expect)
            assert err <= bound, (kv_mode, pos, err)
            if kv_mode == tl.TL_KV_INT8:
                check_argmax(int(gam[0]), expect, f"kv {kv_mode} position {pos}", margin=bound)
            else:
                check_argmax(int(gam[0]), expect, f"kv {kv_mode} position {pos}")
    finally:
        gm.close()
