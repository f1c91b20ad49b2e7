"""Measurement helpers on the GPU: the read-bandwidth probe and the phase
timeline of the single-kernel decode step (their outputs feed bench.py's
rooflines and the trace profile, so their shapes are checked here)."""

import numpy as np
import pytest
import torch

import tl_synth
import weight_shared_looped_int4_b200 as tl
from gpu_helpers import DEV, GpuModel, need_gpu

pytestmark = pytest.mark.gpu


def test_read_probe():
    need_gpu()
    buf = torch.empty(64 << 20, dtype=torch.uint8, device=DEV)
    gbs = tl.tl_probe_read_bandwidth(buf, buf.numel(), 20)
    assert 100.0 < gbs < 100000.0
    with pytest.raises(tl.TLError) as e:
        tl.tl_probe_read_bandwidth(buf, 15, 1)   # not a multiple of 16
    assert e.value.status == tl.TL_ERR_INVALID_ARG
    with pytest.raises(tl.TLError) as e:
        tl.tl_probe_read_bandwidth(buf, 1024, 0)
    assert e.value.status == tl.TL_ERR_INVALID_ARG


def test_fused_trace_timeline_is_ordered():
    need_gpu()
    w = tl_synth.make_model_weights(tl_synth.TINY_LM, tl_synth.SEED_TINY)
    gm = GpuModel(w, max_loops=4, max_ctx=64, max_lanes=1)
    try:
        gm.set_path(tl.DECODE_FUSED)
        L = 4
        gm.prefill_lane(0, tl_synth.make_tokens(5, w.shape.vocab, 16), L, logits=False)
        G = tl.tl_model_trace_grid(gm.handle)
        assert G >= 1
        n_bar = 5 * (w.shape.n_pre + L)
        slots = 4 + 5 * n_bar
        buf = torch.zeros(slots * G, dtype=torch.int64, device=DEV)
        tl.tl_model_set_trace(gm.handle, buf, buf.numel())
        gm.decode([0], [3], [L])
        tl.tl_model_set_trace(gm.handle, None)
        t = buf.cpu().numpy().reshape(slots, G)
        start = t[0]
        assert np.all(start > 0)
        prev = start
        for k in range(n_bar):
            arr, rel = t[1 + 5 * k], t[2 + 5 * k]
            assert np.all(arr >= prev), k          # each CTA arrives after its previous release
            assert np.all(rel >= arr.max() - 1000), k   # nobody leaves before the last arrival (ns)
            prev = rel
        end = t[1 + 5 * n_bar + 2]
        assert np.all(end >= prev)
        # a step without a trace buffer leaves it untouched
        buf.zero_()
        gm.decode([0], [4], [L])
        assert int(buf.abs().sum().item()) == 0
    finally:
        gm.close()
