"""INT4 group-128 linear on the GPU against the fp64 oracle.

Workload: the INT4 dequant linear sweep, fp16 activations ~N(0,1), packed
uint4 weights with fp16 scale and 4-bit zero, M in {1, 4, 16, 128} x
(K, N) in {(2048, 3072), (2048, 2048), (2048, 11264), (5632, 2048)}, fp32
accumulate, fp16 out; plus ragged shapes and the bit-exact dequant check.
"""

import numpy as np
import pytest
import torch

import tl_synth
import weight_shared_looped_int4_b200 as tl
from gpu_helpers import DEV, KERNEL_REL_L2, f16_host, need_gpu, rel_l2, to_dev
from oracle import ref

pytestmark = pytest.mark.gpu

PATHS = [tl.TL_PATH_GEMV, tl.TL_PATH_TC]


def _run(lin, x, path):
    h = tl.tl_linear_create(lin, lin.K, lin.N, 0)
    try:
        dx = to_dev(x)
        dy = torch.empty((x.shape[0], lin.N), dtype=torch.float16, device=DEV)
        try:
            tl.tl_linear_forward(h, dx, x.shape[0], dy, path)
        except tl.TLError as e:
            if e.status == tl.TL_ERR_UNSUPPORTED:
                pytest.skip(str(e))
            raise
        torch.cuda.synchronize()
        return dy.cpu().numpy()
    finally:
        tl.tl_linear_destroy(h)


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("kn", tl_synth.LINEAR_SWEEP_KN)
def test_linear_sweep(kn, path):
    K, N = kn
    rng = np.random.default_rng(tl_synth.SEED_LINEAR + K + N)
    lin = tl_synth.make_int4_linear(rng, N, K)
    W = ref.dequantize(lin.qweight, lin.scales, lin.qzeros, K)
    for M in tl_synth.LINEAR_SWEEP_M:
        x = tl_synth.make_activations(tl_synth.SEED_LINEAR * 7 + M, M, K)
        y = _run(lin, x, path)
        expect = ref.int4_linear(x, W)
        err = rel_l2(y, expect)
        assert err <= KERNEL_REL_L2, (K, N, M, path, err)
        assert np.all(np.isfinite(y))


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("K,N,M", [(128, 16, 1), (384, 1000, 3), (640, 48, 17), (1152, 200, 33),
                                   (256, 33, 129)])
def test_linear_ragged(K, N, M, path):
    rng = np.random.default_rng(K * 31 + N)
    lin = tl_synth.make_int4_linear(rng, N, K)
    x = tl_synth.make_activations(K + M, M, K)
    y = _run(lin, x, path)
    expect = ref.int4_linear(x, ref.dequantize(lin.qweight, lin.scales, lin.qzeros, K))
    assert rel_l2(y, expect) <= KERNEL_REL_L2


@pytest.mark.parametrize("path", PATHS)
def test_dequant_bit_exact(path):
    # One-hot activations return a column of W; w = (q - z) * s is exact in
    # fp32, so the fp16 output must be the round-to-nearest fp16 of the
    # oracle's exact value, bit for bit.
    K, N = 512, 96
    rng = np.random.default_rng(77)
    lin = tl_synth.make_int4_linear(rng, N, K)
    W = ref.dequantize(lin.qweight, lin.scales, lin.qzeros, K)
    ks = [0, 1, 7, 8, 15, 16, 63, 64, 127, 128, 129, 255, 300, 383, 384, 511]
    x = np.zeros((len(ks), K), np.float16)
    for i, k in enumerate(ks):
        x[i, k] = 1.0
    y = _run(lin, x, path)
    expect = W[:, ks].T.astype(np.float16)
    assert np.array_equal(y.view(np.uint16), expect.view(np.uint16))


def test_rows_independent_of_batch():
    # A row's result is bitwise the same whatever rows share the launch.
    K, N = 2048, 512
    rng = np.random.default_rng(5)
    lin = tl_synth.make_int4_linear(rng, N, K)
    x = tl_synth.make_activations(6, 16, K)
    full = _run(lin, x, tl.TL_PATH_GEMV)
    for M in (1, 3, 8, 9):
        part = _run(lin, x[:M], tl.TL_PATH_GEMV)
        assert np.array_equal(part.view(np.uint16), full[:M].view(np.uint16))
