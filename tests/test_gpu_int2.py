"""The INT2 body (tl_config.weight_bits = 2) on the GPU against the oracle's
INT2 dequantisation.

* The linear: the sweep's (K, N) shapes at M in {1, 4, 16, 128} and ragged
  shapes on both kernel families (the GEMV reads the 2-bit layout; the
  tensor-core GEMM runs on the codes widened to its 4-bit tile layout):
  relative L2 <= 1e-3; one-hot activations return a column of W bit for bit.
* The model: the tiny LM and the 400M LM with INT2 blocks, prefill and
  teacher-forced decode steps against the INT2 oracle (logits max-abs <=
  2e-2, argmax exact unless the oracle's top-2 margin is below 1e-3); the
  single-kernel decode step is refused (INT4 only).
"""

import numpy as np
import pytest
import torch

import tl_synth
import weight_shared_looped_int4_b200 as tl
from gpu_helpers import (DEV, KERNEL_REL_L2, LOGIT_MAX_ABS, GpuModel, check_argmax, need_gpu, rel_l2,
                         to_dev)
from oracle import ref

pytestmark = pytest.mark.gpu

PATHS = [tl.TL_PATH_GEMV, tl.TL_PATH_TC]


def _run(lin, x, path):
    h = tl.tl_linear_create(lin, lin.K, lin.N, 0)
    try:
        dx = to_dev(x)
        dy = torch.empty((x.shape[0], lin.N), dtype=torch.float16, device=DEV)
        tl.tl_linear_forward(h, dx, x.shape[0], dy, path)
        torch.cuda.synchronize()
        return dy.cpu().numpy()
    finally:
        tl.tl_linear_destroy(h)


def _deq(lin):
    return ref.dequantize_int2(lin.qweight, lin.scales, lin.qzeros, lin.K)


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("kn", tl_synth.LINEAR_SWEEP_KN)
def test_int2_linear_sweep(kn, path):
    K, N = kn
    rng = np.random.default_rng(tl_synth.SEED_LINEAR + 2 * K + N)
    lin = tl_synth.make_int2_linear(rng, N, K)
    W = _deq(lin)
    for M in tl_synth.LINEAR_SWEEP_M:
        x = tl_synth.make_activations(tl_synth.SEED_LINEAR * 11 + M, M, K)
        y = _run(lin, x, path)
        err = rel_l2(y, ref.int4_linear(x, W))
        assert err <= KERNEL_REL_L2, (K, N, M, path, err)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("K,N,M", [(128, 16, 1), (384, 1000, 3), (640, 48, 17), (2176, 200, 33),
                                   (256, 33, 129)])
def test_int2_linear_ragged(K, N, M, path):
    rng = np.random.default_rng(K * 37 + N)
    lin = tl_synth.make_int2_linear(rng, N, K)
    x = tl_synth.make_activations(K + 3 * M, M, K)
    y = _run(lin, x, path)
    assert rel_l2(y, ref.int4_linear(x, _deq(lin))) <= KERNEL_REL_L2


@pytest.mark.parametrize("path", PATHS)
def test_int2_dequant_bit_exact(path):
    # one-hot activations return a column of W: (q - z) * s is exact in fp32,
    # so the fp16 output is the nearest fp16 of the oracle's exact value
    K, N = 2176, 96       # 17 groups: the zero points span two words per row
    rng = np.random.default_rng(78)
    lin = tl_synth.make_int2_linear(rng, N, K)
    W = _deq(lin)
    ks = [0, 1, 7, 8, 15, 16, 17, 31, 63, 64, 127, 128, 129, 1023, 2047, 2048, 2175]
    x = np.zeros((len(ks), K), np.float16)
    for i, k in enumerate(ks):
        x[i, k] = 1.0
    y = _run(lin, x, path)
    expect = W[:, ks].T.astype(np.float16)
    assert np.array_equal(y.view(np.uint16), expect.view(np.uint16))


def _teacher_forced(gm, om, lane, toks, P, L, steps, where):
    glg, gam = gm.prefill_lane(lane, toks[:P], L)
    cache, olg = om.prefill(toks[:P], L)
    assert np.abs(glg - olg).max() <= LOGIT_MAX_ABS, f"{where} prefill"
    check_argmax(gam, olg, f"{where} prefill")
    for i in range(P, P + steps):
        glg, gam = gm.decode([lane], [int(toks[i])], [L])
        olg = om.decode(cache, int(toks[i]), L)
        assert np.abs(glg[0] - olg).max() <= LOGIT_MAX_ABS, f"{where} step {i}"
        check_argmax(int(gam[0]), olg, f"{where} step {i}")


@pytest.mark.parametrize("P,L", [(40, 4), (9, 3)])
def test_tiny_int2_prefill_decode(P, L):
    w = tl_synth.make_model_weights(tl_synth.TINY_LM, tl_synth.SEED_TINY, bits=2)
    om = ref.LoopedModel(w)
    gm = GpuModel(w, max_loops=8, max_ctx=128, max_lanes=2, weight_bits=2)
    try:
        toks = tl_synth.make_tokens(700 + P, w.shape.vocab, P + 8)
        _teacher_forced(gm, om, 0, toks, P, L, 8, f"tiny int2 P={P} L={L}")
        with pytest.raises(tl.TLError) as e:
            gm.set_path(tl.DECODE_FUSED)
        assert e.value.status == tl.TL_ERR_UNSUPPORTED
    finally:
        gm.close()


def test_lm_int2_prefill_decode():
    w = tl_synth.make_model_weights(tl_synth.LOOPED_LM, tl_synth.SEED_LM, bits=2)
    om = ref.LoopedModel(w)
    gm = GpuModel(w, max_loops=8, max_ctx=256, max_lanes=1, weight_bits=2)
    try:
        toks = tl_synth.make_tokens(tl_synth.SEED_LM + 2, w.shape.vocab, 128 + 12)
        _teacher_forced(gm, om, 0, toks, 128, 8, 12, "LM int2")
    finally:
        gm.close()
