"""GQA attention with RoPE on Q/K, RMSNorm and RoPE ops, on the GPU against
the fp64 oracle.

Workload: D = 2048, 16 Q heads and 4 KV heads of 128, fp16 Q/K/V ~ N(0, 1),
theta 1e4; single-query cached decode over KV length {128, 1024, 4096, 8192}
and causal tiled prefill at T {128, 512, 2048}, batch 1 and 8.  RoPE is
applied on the GPU by the in-place RoPE op; the oracle rotates in fp64.
"""

import numpy as np
import pytest
import torch

import tl_synth
import weight_shared_looped_int4_b200 as tl
from gpu_helpers import DEV, KERNEL_REL_L2, need_gpu, rel_l2, to_dev
from oracle import ref

pytestmark = pytest.mark.gpu

HQ, HKV, HD, THETA = 16, 4, 128, 1e4


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def _cache(kv_btHd, ctx):
    """[B][T][Hkv][hd] host -> device plane layout [B][Hkv][ctx][hd]."""
    B, T, H, D = kv_btHd.shape
    out = torch.zeros((B, H, ctx, D), dtype=torch.float16, device=DEV)
    out[:, :, :T] = torch.from_numpy(np.ascontiguousarray(kv_btHd.transpose(0, 2, 1, 3))).to(DEV)
    return out


def _rope_cache(kc, n, ctx, hkv, hd):
    pos = torch.arange(n, dtype=torch.int32, device=DEV)
    for b in range(kc.shape[0]):
        tl.tl_op_rope(kc[b], n, hkv, hd, hd, ctx * hd, pos, THETA)


@pytest.mark.parametrize("B", [1, 8])
@pytest.mark.parametrize("S", [128, 1024, 4096, 8192])
def test_decode_attention(S, B):
    _decode_case(S, B, [S] * B, HQ, HKV, HD, seed=tl_synth.SEED_ATTN + S + B)


@pytest.mark.parametrize("hq,hkv,hd", [(16, 4, 128), (4, 2, 64), (8, 8, 64), (8, 1, 128)])
def test_decode_attention_ragged_lengths(hq, hkv, hd):
    S = 1500
    n_keys = [1, 2, 31, 32, 33, 1024, 1025, 1500]
    _decode_case(S, len(n_keys), n_keys, hq, hkv, hd, seed=9)


def _decode_case(S, B, n_keys, hq, hkv, hd, seed):
    q, k, v = tl_synth.make_qkv(seed, B, S, hq, hkv, hd, T_q=1)
    kc, vc = _cache(k, S), _cache(v, S)
    _rope_cache(kc, S, S, hkv, hd)
    qd = to_dev(np.ascontiguousarray(q[:, 0]))                       # [B][Hq][hd]
    qpos = torch.as_tensor(np.asarray(n_keys, np.int32) - 1, device=DEV)
    tl.tl_op_rope(qd, B, hq, hd, hq * hd, hd, qpos, THETA)
    out = torch.empty((B, hq, hd), dtype=torch.float16, device=DEV)
    tl.tl_op_gqa_decode(qd, kc, vc, hkv * S * hd, S, n_keys, B, hq, hkv, hd, out)
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    for b in range(B):
        n = n_keys[b]
        qr = ref.rope(q[b, :1].astype(np.float64), [n - 1], THETA)
        kr = ref.rope(k[b, :n].astype(np.float64), np.arange(n), THETA)
        expect = ref.gqa_attention(qr, kr, v[b, :n], [n - 1])[0]
        err = rel_l2(got[b], expect)
        assert err <= KERNEL_REL_L2, (S, b, n, err)


def _prefill_case(T, B, pos0, hq, hkv, hd, seed, sample=None):
    ctx = pos0 + T
    q, k, v = tl_synth.make_qkv(seed, B, ctx, hq, hkv, hd, T_q=T)
    kc, vc = _cache(k, ctx), _cache(v, ctx)
    _rope_cache(kc, ctx, ctx, hkv, hd)
    qd = to_dev(q)                                                   # [B][T][Hq][hd]
    qpos = torch.arange(pos0, pos0 + T, dtype=torch.int32, device=DEV)
    for b in range(B):
        tl.tl_op_rope(qd[b], T, hq, hd, hq * hd, hd, qpos, THETA)
    rows = np.arange(T) if sample is None else np.asarray(sample)
    expects = []
    for b in range(B):
        qr = ref.rope(q[b, rows].astype(np.float64), pos0 + rows, THETA)
        kr = ref.rope(k[b].astype(np.float64), np.arange(ctx), THETA)
        expects.append(ref.gqa_attention(qr, kr, v[b], pos0 + rows))
    # both kernels: tcgen05 (128-query tiles) and mma.sync (16-query tiles)
    try:
        for min_tc, kernel in ((1, "tcgen05"), (1 << 30, "mma.sync")):
            tl.tl_set_prefill_attention_tc_min(min_tc)
            out = torch.empty((B, T, hq, hd), dtype=torch.float16, device=DEV)
            tl.tl_op_gqa_prefill(qd, kc, vc, hkv * ctx * hd, ctx, T, pos0, B, hq, hkv, hd, out)
            torch.cuda.synchronize()
            got = out.cpu().numpy().astype(np.float64)
            for b in range(B):
                err = rel_l2(got[b, rows], expects[b])
                assert err <= KERNEL_REL_L2, (kernel, T, b, err)
    finally:
        tl.tl_set_prefill_attention_tc_min(1024)


@pytest.mark.parametrize("B", [1, 8])
@pytest.mark.parametrize("T", [128, 512, 2048])
def test_prefill_attention(T, B):
    sample = None
    if T * B > 4096:
        rng = np.random.default_rng(T + B)
        sample = np.unique(np.concatenate([[0, 1, 63, 64, 127, 128, T - 1],
                                           rng.integers(0, T, 40)]))
    _prefill_case(T, B, 0, HQ, HKV, HD, seed=tl_synth.SEED_ATTN + 7 * T + B, sample=sample)


@pytest.mark.parametrize("T,pos0,hq,hkv,hd", [(1, 0, 4, 2, 64), (17, 3, 16, 4, 128), (37, 0, 4, 2, 64),
                                              (50, 77, 16, 4, 128), (130, 5, 8, 8, 64), (65, 0, 8, 1, 128),
                                              (300, 1000, 16, 4, 128)])
def test_prefill_attention_ragged(T, pos0, hq, hkv, hd):
    # both attention kernels: ragged tiles, offsets, GQA ratios
    _prefill_case(T, 2, pos0, hq, hkv, hd, seed=T + pos0)


def test_rmsnorm_op():
    rng = np.random.default_rng(3)
    for rows, d in ((1, 256), (37, 2048), (5, 5632)):
        x = (rng.normal(size=(rows, d)) * 7).astype(np.float32)
        g = rng.uniform(0.8, 1.2, d).astype(np.float16)
        dx, dg = torch.from_numpy(x).to(DEV), to_dev(g)
        dy = torch.empty((rows, d), dtype=torch.float16, device=DEV)
        tl.tl_op_rmsnorm(dx, dg, rows, d, 1e-5, dy)
        torch.cuda.synchronize()
        expect = ref.rms_norm(x.astype(np.float64), g, 1e-5)
        assert rel_l2(dy.cpu().numpy(), expect) <= KERNEL_REL_L2


def test_rope_op():
    rng = np.random.default_rng(4)
    for T, H, hd in ((5, 3, 64), (300, 16, 128), (2, 1, 2)):
        x = rng.normal(size=(T, H, hd)).astype(np.float16)
        pos = rng.integers(0, 8192, T).astype(np.int32)
        dx = to_dev(x)
        tl.tl_op_rope(dx, T, H, hd, H * hd, hd, torch.from_numpy(pos).to(DEV), THETA)
        torch.cuda.synchronize()
        expect = ref.rope(x.astype(np.float64), pos, THETA)
        assert rel_l2(dx.cpu().numpy(), expect) <= KERNEL_REL_L2
