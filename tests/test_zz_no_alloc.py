"""The no-allocation decode attention entry point against the regular one.

tl_op_gqa_decode_noalloc serves callers that cannot call cudaMalloc: a host
that plans every device byte up front and owns the allocator, or a plug-in
running inside another runtime's memory pool.  Its scratch is a fixed array
inside the library.  It must give the same result as tl_op_gqa_decode, and
match the fp64 oracle's attention, also on a second call right after the first
(the shared scratch keeps the previous call's contents).  This file sorts last so a
run that stops at the first failure has run every other test already; it also
passes on its own in a fresh process.
"""

import numpy as np
import pytest
import torch

import tl_synth
import weight_shared_looped_int4_b200 as tl
from oracle import ref

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
KERNEL_REL_L2 = 1e-3   # the per-kernel bound the other attention tests use
THETA = 1e4


def _rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _inputs(seed, B, S, hq, hkv, hd):
    q, k, v = tl_synth.make_qkv(seed, B, S, hq, hkv, hd, T_q=1)
    kc = torch.from_numpy(np.ascontiguousarray(k.transpose(0, 2, 1, 3))).to(DEV)  # [B][Hkv][S][hd]
    vc = torch.from_numpy(np.ascontiguousarray(v.transpose(0, 2, 1, 3))).to(DEV)
    qd = torch.from_numpy(np.ascontiguousarray(q[:, 0])).to(DEV)                 # [B][Hq][hd]
    return (q, k, v), (qd, kc, vc)


def _oracle(host, n_keys):
    """fp64 attention of each query (at position n_keys[b] - 1) over its keys."""
    q, k, v = host
    out = []
    for b, n in enumerate(n_keys):
        out.append(ref.gqa_attention(q[b, :1], k[b, :n], v[b, :n], [n - 1])[0])
    return np.stack(out)


def _both(seed, n_keys, S, hq, hkv, hd):
    B = len(n_keys)
    host, (qd, kc, vc) = _inputs(seed, B, S, hq, hkv, hd)
    ref_out = torch.empty((B, hq, hd), dtype=torch.float16, device=DEV)
    new_out = torch.full((B, hq, hd), float("nan"), dtype=torch.float16, device=DEV)
    tl.tl_op_gqa_decode(qd, kc, vc, hkv * S * hd, S, n_keys, B, hq, hkv, hd, ref_out)
    tl.tl_op_gqa_decode_noalloc(qd, kc, vc, hkv * S * hd, S, n_keys, B, hq, hkv, hd, new_out)
    torch.cuda.synchronize()
    return ref_out.cpu().numpy(), new_out.cpu().numpy(), _oracle(host, n_keys)


def test_no_alloc_matches_regular_entry_point_twice():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    # first call: 8 rows over 1024 keys (32 splits each); second call right
    # after: other shapes and ragged key counts, so leftovers of the first
    # call's scratch would show.
    cases = [
        (101, [1024] * 8, 1024, 16, 4, 128),
        (202, [1, 33, 500, 64, 2, 1000], 1000, 8, 2, 64),
    ]
    for seed, n_keys, S, hq, hkv, hd in cases:
        ref_out, new_out, oracle_out = _both(seed, n_keys, S, hq, hkv, hd)
        assert np.all(np.isfinite(new_out))
        assert _rel_l2(new_out, ref_out) <= KERNEL_REL_L2
        assert _rel_l2(new_out, oracle_out) <= KERNEL_REL_L2


def test_no_alloc_rejects_oversize():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    x = torch.zeros(16, dtype=torch.float16, device=DEV)
    with pytest.raises(tl.TLError) as e:   # 33 rows: over the 32-row limit
        tl.tl_op_gqa_decode_noalloc(x, x, x, 0, 1, [1] * 33, 33, 16, 4, 128, x)
    assert e.value.status == tl.TL_ERR_UNSUPPORTED
    with pytest.raises(tl.TLError) as e:   # partials would need more than 4 MiB
        tl.tl_op_gqa_decode_noalloc(x, x, x, 0, 1, [1] * 32, 32, 64, 8, 128, x)
    assert e.value.status == tl.TL_ERR_UNSUPPORTED
