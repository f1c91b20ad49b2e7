"""Python binding of the C ABI declared in ``include/tl.h``.

Argument marshalling only: every function here converts its arguments to
plain pointers / integers and calls the entry point of the same name in
``libtl_b200.so``; all computation happens in the library's CUDA kernels.
PyTorch is used for device memory and streams only.  The library is loaded on
first use; if it is not built, that first use raises ImportError (there is no
fallback of any kind).

Pointers may be given as torch tensors (their ``data_ptr()``), numpy arrays
(host pointer), ctypes pointers or plain integers.  ``stream`` may be a
``torch.cuda.Stream``, an integer ``cudaStream_t`` or None (torch's current
stream on the current device).
"""

from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_double, c_float, c_int, c_int32, c_longlong, c_size_t, c_void_p

from .build import LIB_PATH

__all__ = [
    "TLError", "lib", "load_library", "tl_config", "tl_int4_linear", "tl_block", "tl_weights",
    "TL_OK", "TL_ERR_INVALID_ARG", "TL_ERR_OOM", "TL_ERR_CUDA", "TL_ERR_CONTEXT_FULL",
    "TL_ERR_LOOPS_MISMATCH", "TL_ERR_NOT_PREFILLED", "TL_ERR_DEVICE_FLAG", "TL_ERR_UNSUPPORTED",
    "TL_PATH_AUTO", "TL_PATH_GEMV", "TL_PATH_TC",
    "tl_model_create", "tl_model_destroy", "tl_prefill", "tl_decode_step", "tl_score_last",
    "tl_lane_length", "tl_model_info", "tl_check_device_error",
    "tl_model_profile_start", "tl_model_profile_stop", "tl_kernel_launch_count", "KERNEL_CLASSES",
    "tl_model_set_graphs", "tl_model_set_decode_path", "DECODE_AUTO", "DECODE_LAYERED", "DECODE_FUSED",
    "tl_model_set_clustered_decode",
    "tl_probe_read_bandwidth", "tl_model_set_trace", "tl_model_trace_grid",
    "tl_model_set_wait_test", "tl_extend", "tl_generate_speculative", "tl_score_logit_lens",
    "tl_score_early_exit", "tl_lane_fork", "tl_spec_stats", "tl_set_prefill_attention_tc_min",
    "tl_linear_create", "tl_linear_destroy", "tl_linear_forward",
    "tl_op_rmsnorm", "tl_op_rope", "tl_op_gqa_decode", "tl_op_gqa_prefill",
    "tl_op_gqa_decode_noalloc", "tl_op_kv_quant_int8", "TL_KV_FP16", "TL_KV_INT8", "tl_lane_kv_export",
    "tl_status_string", "tl_last_error", "tl_version",
    "make_config", "make_weights", "make_int4_linear",
]

TL_OK, TL_ERR_INVALID_ARG, TL_ERR_OOM, TL_ERR_CUDA, TL_ERR_CONTEXT_FULL = 0, 1, 2, 3, 4
TL_ERR_LOOPS_MISMATCH, TL_ERR_NOT_PREFILLED, TL_ERR_DEVICE_FLAG, TL_ERR_UNSUPPORTED = 5, 6, 7, 8
TL_PATH_AUTO, TL_PATH_GEMV, TL_PATH_TC = 0, 1, 2
TL_KV_FP16, TL_KV_INT8 = 0, 1


class TLError(RuntimeError):
    """A non-OK tl_status, with the library's one-line reason."""

    def __init__(self, status: int, message: str):
        super().__init__(f"{_status_name(status)}: {message}")
        self.status = status


class tl_config(ctypes.Structure):
    _fields_ = [("d_model", c_int), ("n_q_heads", c_int), ("n_kv_heads", c_int),
                ("head_dim", c_int), ("ffn_dim", c_int), ("vocab", c_int), ("n_pre", c_int),
                ("max_loops", c_int), ("max_ctx", c_int), ("max_lanes", c_int),
                ("rms_eps", c_float), ("rope_theta", c_float), ("kv_mode", c_int), ("weight_bits", c_int)]


class tl_int4_linear(ctypes.Structure):
    _fields_ = [("qweight", c_void_p), ("scales", c_void_p), ("qzeros", c_void_p)]


class tl_block(ctypes.Structure):
    _fields_ = [("attn_norm", c_void_p), ("ffn_norm", c_void_p), ("qkv", tl_int4_linear),
                ("o", tl_int4_linear), ("gate_up", tl_int4_linear), ("down", tl_int4_linear)]


class tl_weights(ctypes.Structure):
    _fields_ = [("embed", c_void_p), ("out_norm", c_void_p), ("head", c_void_p),
                ("pre", POINTER(tl_block)), ("loop", POINTER(tl_block))]


class tl_spec_stats(ctypes.Structure):
    _fields_ = [("rounds", c_int), ("drafted", c_int), ("accepted", c_int)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is not built: run `python -m weight_shared_looped_int4_b200.build` "
            "(the CUDA library is required; there is no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    st, P = c_int, c_void_p
    sig = {
        "tl_model_create": (st, [POINTER(tl_config), POINTER(tl_weights), c_int, POINTER(c_void_p)]),
        "tl_model_destroy": (None, [P]),
        "tl_prefill": (st, [P, c_int, P, c_int, c_int, P, P, P]),
        "tl_decode_step": (st, [P, c_int, P, P, P, P, P, P]),
        "tl_score_last": (st, [P, P, c_int, c_int, P, P, P]),
        "tl_lane_length": (st, [P, c_int, POINTER(c_int)]),
        "tl_model_info": (st, [P, POINTER(c_size_t), POINTER(c_size_t), POINTER(c_size_t)]),
        "tl_check_device_error": (st, [P, P]),
        "tl_model_profile_start": (st, [P, ctypes.c_uint]),
        "tl_model_profile_stop": (st, [P, POINTER(c_int), POINTER(c_float)]),
        "tl_kernel_launch_count": (ctypes.c_ulonglong, []),
        "tl_model_set_graphs": (st, [P, c_int]),
        "tl_model_set_decode_path": (st, [P, c_int]),
        "tl_model_set_clustered_decode": (st, [P, c_int]),
        "tl_model_set_trace": (st, [P, P, c_longlong]),
        "tl_model_trace_grid": (c_int, [P]),
        "tl_model_set_wait_test": (st, [P, c_int]),
        "tl_extend": (st, [P, c_int, P, c_int, P, P, P]),
        "tl_generate_speculative": (st, [P, c_int, P, c_int, c_int, c_int, P, POINTER(tl_spec_stats), P]),
        "tl_score_logit_lens": (st, [P, P, c_int, c_int, P, P, P]),
        "tl_score_early_exit": (st, [P, P, c_int, c_int, c_int, P, P, POINTER(c_int), P]),
        "tl_lane_fork": (st, [P, c_int, c_int, c_int, P]),
        "tl_set_prefill_attention_tc_min": (st, [c_int]),
        "tl_probe_read_bandwidth": (st, [P, c_size_t, c_int, P, POINTER(c_double)]),
        "tl_linear_create": (st, [POINTER(tl_int4_linear), c_int, c_int, c_int, POINTER(c_void_p)]),
        "tl_linear_destroy": (None, [P]),
        "tl_linear_forward": (st, [P, P, c_int, P, c_int, P]),
        "tl_op_rmsnorm": (st, [P, P, c_int, c_int, c_float, P, P]),
        "tl_op_rope": (st, [P, c_int, c_int, c_int, c_longlong, c_longlong, P, c_float, P]),
        "tl_op_kv_quant_int8": (st, [P, c_int, c_int, P, P, P]),
        "tl_linear_create_int2": (st, [POINTER(tl_int4_linear), c_int, c_int, c_int, POINTER(c_void_p)]),
        "tl_lane_kv_export": (st, [P, c_int, c_int, c_int, P, P, P, P, P]),
        "tl_op_gqa_decode": (st, [P, P, P, c_longlong, c_int, P, c_int, c_int, c_int, c_int, P, P]),
        "tl_op_gqa_prefill": (st, [P, P, P, c_longlong, c_int, c_int, c_int, c_int, c_int, c_int,
                                   c_int, P, P]),
        "tl_op_gqa_decode_noalloc": (st, [P, P, P, c_longlong, c_int, P, c_int, c_int, c_int, c_int,
                                          P, P]),
        "tl_status_string": (c_char_p, [c_int]),
        "tl_last_error": (c_char_p, []),
        "tl_version": (c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


_LIB = None


def _L():
    global _LIB
    if _LIB is None:
        _LIB = _load()
    return _LIB


def __getattr__(name):
    if name == "lib":
        return _L()
    raise AttributeError(name)

# names every header declaration must have in the library (checked by tests)
EXPORTED = sorted(["tl_model_profile_start", "tl_model_profile_stop", "tl_kernel_launch_count",
                   "tl_model_set_graphs", "tl_model_set_decode_path", "tl_model_set_clustered_decode",
                   "tl_probe_read_bandwidth",
                   "tl_model_set_trace", "tl_model_trace_grid", "tl_model_set_wait_test",
                   "tl_extend", "tl_generate_speculative", "tl_score_logit_lens", "tl_score_early_exit",
                   "tl_lane_fork", "tl_set_prefill_attention_tc_min",
                   "tl_model_create", "tl_model_destroy", "tl_prefill", "tl_decode_step",
                   "tl_score_last", "tl_lane_length", "tl_model_info", "tl_check_device_error",
                   "tl_linear_create", "tl_linear_destroy", "tl_linear_forward", "tl_op_rmsnorm",
                   "tl_op_rope", "tl_op_gqa_decode", "tl_op_gqa_prefill", "tl_status_string",
                   "tl_op_gqa_decode_noalloc", "tl_op_kv_quant_int8", "tl_lane_kv_export",
                   "tl_linear_create_int2",
                   "tl_last_error", "tl_version"])


# ---------------------------------------------------------------- helpers ---

def load_library():
    """Load (once) and return the ctypes handle of libtl_b200.so."""
    return _L()


def _status_name(s: int) -> str:
    return _L().tl_status_string(int(s)).decode()


def _check(s: int):
    if s != TL_OK:
        raise TLError(s, _L().tl_last_error().decode())


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if hasattr(x, "ctypes"):
        return x.ctypes.data
    if isinstance(x, ctypes._Pointer) or isinstance(x, ctypes.Array):
        return ctypes.cast(x, c_void_p).value
    raise TypeError(f"cannot take a pointer of {type(x)}")


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _i32_host(values):
    arr = (c_int32 * len(values))(*[int(v) for v in values])
    return arr


# ------------------------------------------------------------ marshalling ---

def make_config(shape, max_loops: int, max_ctx: int, max_lanes: int, kv_mode: int = 0,
                weight_bits: int = 4) -> tl_config:
    """tl_config from an object with the ModelShape attribute names
    (kv_mode TL_KV_FP16 or TL_KV_INT8; weight_bits 4 or 2 for the INT2 body)."""
    return tl_config(shape.d_model, shape.n_q_heads, shape.n_kv_heads, shape.head_dim,
                     shape.ffn_dim, shape.vocab, shape.n_pre, max_loops, max_ctx, max_lanes,
                     float(shape.rms_eps), float(shape.rope_theta), int(kv_mode), int(weight_bits))


def make_int4_linear(lin) -> tl_int4_linear:
    """tl_int4_linear of host arrays (qweight uint32, scales fp16, qzeros uint32)."""
    for a in (lin.qweight, lin.scales, lin.qzeros):
        if not a.flags["C_CONTIGUOUS"]:
            raise ValueError("INT4 arrays must be C-contiguous")
    return tl_int4_linear(_ptr(lin.qweight), _ptr(lin.scales), _ptr(lin.qzeros))


def _block(b) -> tl_block:
    return tl_block(_ptr(b.attn_norm), _ptr(b.ffn_norm), make_int4_linear(b.qkv),
                    make_int4_linear(b.o), make_int4_linear(b.gate_up), make_int4_linear(b.down))


def make_weights(w):
    """(tl_weights, keepalive) from an object with the ModelWeights attribute
    names; keep ``keepalive`` referenced until tl_model_create returns."""
    pre = (tl_block * max(1, len(w.pre)))(*[_block(b) for b in w.pre])
    loop = _block(w.loop)
    tw = tl_weights(_ptr(w.embed), _ptr(w.out_norm), _ptr(w.head),
                    ctypes.cast(pre, POINTER(tl_block)), ctypes.pointer(loop))
    return tw, (pre, loop, w)


# ------------------------------------------------------------ entry points ---

def tl_model_create(cfg: tl_config, weights: tl_weights, device: int = 0) -> int:
    out = c_void_p()
    _check(_L().tl_model_create(ctypes.byref(cfg), ctypes.byref(weights), int(device),
                               ctypes.byref(out)))
    return out.value


def tl_model_destroy(model: int) -> None:
    _L().tl_model_destroy(model)


def tl_prefill(model, lane, d_tokens, n_tokens, loops, d_last_logits=None, d_last_argmax=None,
               stream=None) -> None:
    _check(_L().tl_prefill(model, int(lane), _ptr(d_tokens), int(n_tokens), int(loops),
                          _ptr(d_last_logits), _ptr(d_last_argmax), _stream(stream)))


def tl_decode_step(model, lane_ids, d_tokens, loops, d_logits=None, d_argmax=None,
                   stream=None) -> None:
    """lane_ids and loops are host sequences of ints."""
    n = len(lane_ids)
    if len(loops) != n:
        raise ValueError("lane_ids and loops differ in length")
    _check(_L().tl_decode_step(model, n, _i32_host(lane_ids), _ptr(d_tokens), _i32_host(loops),
                              _ptr(d_logits), _ptr(d_argmax), _stream(stream)))


def tl_score_last(model, d_tokens, n_tokens, loops, d_logits, d_argmax=None, stream=None) -> None:
    _check(_L().tl_score_last(model, _ptr(d_tokens), int(n_tokens), int(loops), _ptr(d_logits),
                             _ptr(d_argmax), _stream(stream)))


def tl_extend(model, lane, d_tokens, n_tokens, d_logits=None, d_argmax=None, stream=None) -> None:
    _check(_L().tl_extend(model, int(lane), _ptr(d_tokens), int(n_tokens), _ptr(d_logits), _ptr(d_argmax),
                         _stream(stream)))


def tl_generate_speculative(model, lane, d_first_token, max_tokens, draft_loops, draft_ahead, d_out_tokens,
                            stream=None) -> dict:
    """Returns the round counters {rounds, drafted, accepted}."""
    stats = tl_spec_stats()
    _check(_L().tl_generate_speculative(model, int(lane), _ptr(d_first_token), int(max_tokens), int(draft_loops),
                                       int(draft_ahead), _ptr(d_out_tokens), ctypes.byref(stats),
                                       _stream(stream)))
    return {"rounds": stats.rounds, "drafted": stats.drafted, "accepted": stats.accepted}


def tl_score_logit_lens(model, d_tokens, n_tokens, loops, d_logits, d_argmax=None, stream=None) -> None:
    _check(_L().tl_score_logit_lens(model, _ptr(d_tokens), int(n_tokens), int(loops), _ptr(d_logits),
                                   _ptr(d_argmax), _stream(stream)))


def tl_score_early_exit(model, d_tokens, n_tokens, max_loops, stable_n, d_logits, d_argmax=None,
                        stream=None) -> int:
    """Returns the loop iterations run."""
    used = c_int(0)
    _check(_L().tl_score_early_exit(model, _ptr(d_tokens), int(n_tokens), int(max_loops), int(stable_n),
                                   _ptr(d_logits), _ptr(d_argmax), ctypes.byref(used), _stream(stream)))
    return used.value


def tl_lane_fork(model, src_lane, dst_lane, n_tokens, stream=None) -> None:
    _check(_L().tl_lane_fork(model, int(src_lane), int(dst_lane), int(n_tokens), _stream(stream)))


def tl_set_prefill_attention_tc_min(min_queries: int) -> None:
    """Prefill attention on tcgen05 from this many queries on (default 1024)."""
    _check(_L().tl_set_prefill_attention_tc_min(int(min_queries)))


def tl_lane_length(model, lane) -> int:
    out = c_int()
    _check(_L().tl_lane_length(model, int(lane), ctypes.byref(out)))
    return out.value


def tl_model_info(model):
    w, k, s = c_size_t(), c_size_t(), c_size_t()
    _check(_L().tl_model_info(model, ctypes.byref(w), ctypes.byref(k), ctypes.byref(s)))
    return {"weight_bytes": w.value, "kv_bytes": k.value, "workspace_bytes": s.value}


def tl_check_device_error(model, stream=None) -> None:
    _check(_L().tl_check_device_error(model, _stream(stream)))


KERNEL_CLASSES = ["embed", "qkv", "attn_decode", "o_proj", "gate_up", "down", "head",
                  "attn_prefill", "gemm_tc", "norm", "setup", "decode_fused"]

# tl_decode_path
DECODE_AUTO, DECODE_LAYERED, DECODE_FUSED = 0, 1, 2


def tl_model_profile_start(model, class_mask: int = (1 << 12) - 1) -> None:
    _check(_L().tl_model_profile_start(model, int(class_mask)))


def tl_model_profile_stop(model):
    """{class name: (launches, total_ms)} for the classes that ran."""
    n = len(KERNEL_CLASSES)
    launches = (c_int * n)()
    total = (c_float * n)()
    _check(_L().tl_model_profile_stop(model, launches, total))
    return {KERNEL_CLASSES[i]: (launches[i], total[i]) for i in range(n) if launches[i]}


def tl_model_set_graphs(model, enable: bool) -> None:
    _check(_L().tl_model_set_graphs(model, 1 if enable else 0))


def tl_probe_read_bandwidth(buf, nbytes: int, reps: int = 200, stream=None) -> float:
    """GB/s of repeated 16-byte L2-path reads over `nbytes` of a device buffer."""
    out = c_double(0.0)
    _check(_L().tl_probe_read_bandwidth(_ptr(buf), int(nbytes), int(reps), _stream(stream), ctypes.byref(out)))
    return out.value


def tl_model_set_trace(model, buf=None, n_entries: int = 0) -> None:
    """Phase timeline of decode steps into a device uint64 buffer (None = off).

    Single-kernel steps stamp per-CTA phase times; per-op steps stamp, per
    layer launch, maxima over its CTAs (the caller zeroes the buffer before
    the step) after the head's per-CTA slots.  Layout in include/tl.h."""
    _check(_L().tl_model_set_trace(model, _ptr(buf) if buf is not None else None,
                                   int(n_entries if buf is not None else 0)))


def tl_model_trace_grid(model) -> int:
    return int(_L().tl_model_trace_grid(model))


def tl_model_set_wait_test(model, extra_arrivals: int) -> None:
    """Test hook: 1 makes the next single-kernel steps' grid barriers run out
    of time (see tl.h); 0 restores normal steps."""
    _check(_L().tl_model_set_wait_test(model, int(extra_arrivals)))


def tl_model_set_clustered_decode(model, enable: bool) -> None:
    """Per-op decode through the clustered QKV + attention kernel (True) or
    the QKV GEMV + split-KV attention (False); see include/tl.h."""
    _check(_L().tl_model_set_clustered_decode(model, 1 if enable else 0))


def tl_model_set_decode_path(model, path: int) -> None:
    """DECODE_AUTO (default), DECODE_LAYERED or DECODE_FUSED (see include/tl.h)."""
    _check(_L().tl_model_set_decode_path(model, int(path)))


def tl_kernel_launch_count() -> int:
    return int(_L().tl_kernel_launch_count())


def tl_linear_create(lin, K: int, N: int, device: int = 0) -> int:
    """A device linear from host storage arrays; INT2 (lin.bits == 2) goes
    through tl_linear_create_int2."""
    out = c_void_p()
    w = make_int4_linear(lin)
    fn = _L().tl_linear_create_int2 if getattr(lin, "bits", 4) == 2 else _L().tl_linear_create
    _check(fn(ctypes.byref(w), int(K), int(N), int(device), ctypes.byref(out)))
    return out.value


def tl_linear_destroy(handle) -> None:
    _L().tl_linear_destroy(handle)


def tl_linear_forward(handle, d_x, M, d_y, path=TL_PATH_AUTO, stream=None) -> None:
    _check(_L().tl_linear_forward(handle, _ptr(d_x), int(M), _ptr(d_y), int(path), _stream(stream)))


def tl_op_rmsnorm(d_x, d_g, rows, d, eps, d_y, stream=None) -> None:
    _check(_L().tl_op_rmsnorm(_ptr(d_x), _ptr(d_g), int(rows), int(d), float(eps), _ptr(d_y),
                             _stream(stream)))


def tl_op_rope(d_x, n_tokens, n_heads, head_dim, token_stride, head_stride, d_positions, theta,
               stream=None) -> None:
    _check(_L().tl_op_rope(_ptr(d_x), int(n_tokens), int(n_heads), int(head_dim), int(token_stride),
                          int(head_stride), _ptr(d_positions), float(theta), _stream(stream)))


def tl_lane_kv_export(model, lane, layer, n_tokens, d_k, d_v, d_k_scales=None, d_v_scales=None,
                      stream=None) -> None:
    _check(_L().tl_lane_kv_export(model, int(lane), int(layer), int(n_tokens), _ptr(d_k), _ptr(d_v),
                                 _ptr(d_k_scales), _ptr(d_v_scales), _stream(stream)))


def tl_op_kv_quant_int8(d_x, n, head_dim, d_codes, d_scales, stream=None) -> None:
    _check(_L().tl_op_kv_quant_int8(_ptr(d_x), int(n), int(head_dim), _ptr(d_codes), _ptr(d_scales),
                                   _stream(stream)))


def tl_op_gqa_decode(d_q, d_k, d_v, batch_stride, ctx_stride, n_keys, B, n_q_heads, n_kv_heads,
                     head_dim, d_out, stream=None) -> None:
    """n_keys is a host sequence of B ints."""
    _check(_L().tl_op_gqa_decode(_ptr(d_q), _ptr(d_k), _ptr(d_v), int(batch_stride), int(ctx_stride),
                                _i32_host(n_keys), int(B), int(n_q_heads), int(n_kv_heads),
                                int(head_dim), _ptr(d_out), _stream(stream)))


def tl_op_gqa_decode_noalloc(d_q, d_k, d_v, batch_stride, ctx_stride, n_keys, B, n_q_heads,
                             n_kv_heads, head_dim, d_out, stream=None) -> None:
    """tl_op_gqa_decode for callers that cannot allocate device memory: the
    scratch is a fixed 4 MiB array inside the library (see include/tl.h for
    the limits and the ordering rule).  n_keys is a host sequence of B ints."""
    _check(_L().tl_op_gqa_decode_noalloc(_ptr(d_q), _ptr(d_k), _ptr(d_v), int(batch_stride),
                                         int(ctx_stride), _i32_host(n_keys), int(B), int(n_q_heads),
                                         int(n_kv_heads), int(head_dim), _ptr(d_out), _stream(stream)))


def tl_op_gqa_prefill(d_q, d_k, d_v, batch_stride, ctx_stride, T, pos0, B, n_q_heads, n_kv_heads,
                      head_dim, d_out, stream=None) -> None:
    _check(_L().tl_op_gqa_prefill(_ptr(d_q), _ptr(d_k), _ptr(d_v), int(batch_stride), int(ctx_stride),
                                 int(T), int(pos0), int(B), int(n_q_heads), int(n_kv_heads),
                                 int(head_dim), _ptr(d_out), _stream(stream)))


def tl_status_string(s: int) -> str:
    return _status_name(s)


def tl_last_error() -> str:
    return _L().tl_last_error().decode()


def tl_version() -> str:
    return _L().tl_version().decode()
