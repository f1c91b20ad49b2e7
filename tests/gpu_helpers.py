"""Shared helpers of the GPU parity tests (device buffers via torch, tolerances)."""

import numpy as np
import pytest
import torch

import weight_shared_looped_int4_b200 as tl

# Tolerances (the workload's acceptance bounds):
#   per-kernel fp16 outputs: relative L2 error <= 1e-3 against the fp64 oracle;
#   end-to-end logits: max-abs error <= 2e-2;
#   INT4 unpack and argmax indices: bit-exact (argmax may differ only where the
#   oracle's top-2 margin is below 1e-3).
KERNEL_REL_L2 = 1e-3
LOGIT_MAX_ABS = 2e-2
ARGMAX_MARGIN = 1e-3

DEV = "cuda:0"


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def rel_l2(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def to_dev(a: np.ndarray) -> torch.Tensor:
    """Host numpy array -> device tensor with the same bytes (fp16 stays fp16)."""
    if a.dtype == np.float16:
        return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    if a.dtype == np.uint32:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).to(DEV)
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def f16_host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().astype(np.float64)


def check_argmax(gpu_idx: int, oracle_logits: np.ndarray, where: str = "", margin: float = ARGMAX_MARGIN):
    """Greedy index must equal the oracle's unless its top-2 margin is below
    `margin` (1e-3; the INT8 KV tests pass their own logit bound)."""
    from oracle import ref
    o = ref.greedy(oracle_logits)
    if gpu_idx != o:
        m2 = ref.top2_margin(oracle_logits)
        assert m2 < margin, f"{where}: argmax {gpu_idx} != oracle {o} (margin {m2})"
        # the GPU's pick must be one of the near-tied leaders
        assert oracle_logits[o] - oracle_logits[gpu_idx] < margin, where


class GpuModel:
    """A tl_model built from tl_synth weights, destroyed on close()."""

    def __init__(self, weights, max_loops, max_ctx, max_lanes, device=0, kv_mode=0, weight_bits=4):
        cfg = tl.make_config(weights.shape, max_loops, max_ctx, max_lanes, kv_mode, weight_bits)
        tw, keep = tl.make_weights(weights)
        self.handle = tl.tl_model_create(cfg, tw, device)
        del keep
        self.shape = weights.shape

    def close(self):
        if self.handle:
            torch.cuda.synchronize()
            tl.tl_model_destroy(self.handle)
            self.handle = None

    def set_path(self, path):
        """Decode path of tl_decode_step (tl.DECODE_AUTO / _LAYERED / _FUSED)."""
        tl.tl_model_set_decode_path(self.handle, path)

    def score_last(self, tokens, loops):
        V = self.shape.vocab
        d_tok = torch.as_tensor(np.asarray(tokens, np.int32), device=DEV)
        lg = torch.empty(V, dtype=torch.float32, device=DEV)
        am = torch.empty(1, dtype=torch.int32, device=DEV)
        tl.tl_score_last(self.handle, d_tok, len(tokens), loops, lg, am)
        torch.cuda.synchronize()
        return lg.cpu().numpy().astype(np.float64), int(am.item())

    def prefill_lane(self, lane, tokens, loops, logits=True):
        V = self.shape.vocab
        d_tok = torch.as_tensor(np.asarray(tokens, np.int32), device=DEV)
        lg = torch.empty(V, dtype=torch.float32, device=DEV) if logits else None
        am = torch.empty(1, dtype=torch.int32, device=DEV) if logits else None
        tl.tl_prefill(self.handle, lane, d_tok, len(tokens), loops, lg, am)
        torch.cuda.synchronize()
        if not logits:
            return None, None
        return lg.cpu().numpy().astype(np.float64), int(am.item())

    def decode(self, lanes, tokens, loops):
        V = self.shape.vocab
        d_tok = torch.as_tensor(np.asarray(tokens, np.int32), device=DEV)
        lg = torch.empty((len(lanes), V), dtype=torch.float32, device=DEV)
        am = torch.empty(len(lanes), dtype=torch.int32, device=DEV)
        tl.tl_decode_step(self.handle, list(lanes), d_tok, list(loops), lg, am)
        torch.cuda.synchronize()
        return lg.cpu().numpy().astype(np.float64), am.cpu().numpy()
