#!/usr/bin/env python
"""Benchmark of the looped INT4 model on B200.

Workload (one step): the ~400M-unique-parameter looped LM (d_model 2048, 16 Q /
4 KV heads of 128, SwiGLU 5632, vocab 32000, 2 pre blocks + 1 shared loop
block, INT4 g128 body, fp16 embed/head/norms, seeded random weights) with
L = 8: prefill of a 128-token prompt with no logits, then 128 greedy decode
steps at batch 1 (the first decode step feeds prompt token 128; each later one
feeds the previous argmax, on the device).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One JSON line on rank 0.  `value` is decode tokens/s summed over ranks (each
rank runs its own replica: weak scaling, no collective on the data path);
prefill ms, roofline of the dominant decode kernel, the CPU oracle baseline,
end-to-end numbers and SM clocks are extra keys.  `--impl reference` times the
CPU oracle on this host on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "decode tok/s & prefill ms (T=128, L=8) looped INT4 model; % of roofline"
UNIT = "tokens/s"
PROMPT, STEPS_DECODE, LOOPS = 128, 128, 8
WORKLOAD = "looped INT4 LM d2048 16q/4kv hd128 F5632 V32000 n_pre2 L8; prefill 128 (no logits) + 128 greedy decode, batch 1"

# Algorithmic bytes per decode launch at batch 1 (weights + scales/zeros + the
# activations each launch must read and write), d = 2048, F = 5632, V = 32000.
D, F, V, HQ, HKV, HD = 2048, 5632, 32000, 16, 4, 128


def _int4_bytes(K, N):
    return K * N // 2 + (K // 128) * N * 5 // 2   # nibbles + fp16 scale + 4-bit zero


BYTES_PER_LAUNCH = {
    "qkv": _int4_bytes(D, (HQ + 2 * HKV) * HD) + 4 * D + 2 * D + 2 * (HQ + 2 * HKV) * HD,
    "o_proj": _int4_bytes(HQ * HD, D) + 2 * HQ * HD + 8 * D,
    "gate_up": _int4_bytes(D, 2 * F) + 4 * D + 2 * D + 2 * F,
    "down": _int4_bytes(F, D) + 2 * F + 8 * D,
    "head": V * D * 2 + 4 * D + 2 * D + 4,
}


# DRAM bytes (read + write) of one launch of each decode kernel class, from
#   ncu --clock-control none -k regex:"qkv_attn|gemv_int4|head_direct" -c 45 \
#       --metrics dram__bytes_read.sum,dram__bytes_write.sum python bench.py --ncu-case decode --decode-steps 2
# (ncu flushes the caches before every launch, so every launch reads its
# weights from DRAM; first decode step, NCU_KEYS cached keys per layer for the
# QKV + attention kernel).  Valid for the kernels as captured; the QKV
# class's cache part is rescaled to the bench's mean context.
NCU_TRAFFIC = {"qkv": 3683840, "o_proj": 2263040, "gate_up": 12307456, "down": 6179584,
               "head": 131139584 + 55552}
NCU_KEYS = PROMPT + 1



def roofline_traffic(kernel_class, mean_keys):
    """ncu DRAM bytes of one launch of a decode kernel class at the bench's
    mean context (None where no capture covers it)."""
    traffic = NCU_TRAFFIC.get(kernel_class)
    if traffic is not None and kernel_class == "qkv":
        kv = lambda n: 2 * HKV * HD * 2 * n
        traffic = traffic - kv(NCU_KEYS) + kv(mean_keys)
    return int(traffic) if traffic is not None else None


DECODE_PATHS = {"auto": 0, "layered": 1, "fused": 2}


def bench_config(world, n_dec, decode_path, graphs):
    """The `config` object of the JSON line (the same for both arms)."""
    return {"workload": WORKLOAD, "global_batch": world, "seq_len": PROMPT + n_dec,
            "decode_steps": n_dec, "decode_path": decode_path, "cuda_graphs": graphs,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "inputs larger than L2: each step streams ~333 MB of weights"}


def _attn_bytes_per_launch(mean_keys):
    return 2 * HKV * HD * 2 * mean_keys + 2 * HQ * HD * 2


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def probe_read_bandwidths(tl, torch, dev, st):
    """Measured read bandwidths: L2 (a buffer of half the L2 size, 200 sweeps
    in one launch after warm sweeps) and HBM (a 4 GiB buffer, 3 sweeps).
    Returns (l2_gbs, l2_buffer_bytes, hbm_read_gbs)."""
    l2_size = torch.cuda.get_device_properties(dev).L2_cache_size
    nbytes = (l2_size // 2) // (1 << 20) * (1 << 20)
    buf = torch.ones(nbytes, dtype=torch.uint8, device=dev)
    l2_gbs = tl.tl_probe_read_bandwidth(buf, nbytes, 200, st)
    del buf
    big = torch.ones(4 << 30, dtype=torch.uint8, device=dev)
    hbm_gbs = tl.tl_probe_read_bandwidth(big, big.numel(), 3, st)
    del big
    torch.cuda.empty_cache()
    return l2_gbs, nbytes, hbm_gbs


# ------------------------------------------------------------------ clocks ---

class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during a region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.device_index = device_index

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.device_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        if not getattr(self, "out", ""):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["no samples"]}
        loaded = [s for s in sm if mx and s > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "samples": len(sm),
                "reasons": sorted(reasons)}


# --------------------------------------------------------------- CPU oracle --

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_sample(weights, prompt, n_decode, om=None):
    """Time the oracle: prefill of the prompt, then n_decode cached greedy steps.
    Returns (prefill_s, decode_s, om)."""
    from oracle import ref
    if om is None:
        om = ref.LoopedModel(weights)
    t0 = time.perf_counter()
    cache, logits = om.prefill(prompt[:PROMPT], LOOPS)
    t1 = time.perf_counter()
    tok = int(prompt[PROMPT])
    for _ in range(n_decode):
        logits = om.decode(cache, tok, LOOPS)
        tok = ref.greedy(logits)
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1, om


# ------------------------------------------------------------------- arms ---

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(pg, values, device):
    """Element-wise maximum over all ranks of this rank's device-timed values
    (ms); `pg` is torch.distributed (every rank calls this in the same order)
    or None for one process, which returns the values unchanged."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if pg is not None:
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def whole_job_rate(world, units_per_rank, slowest_ms):
    """Units per second of the whole job: every rank's units over the slowest
    rank's time (replicas, weak scaling)."""
    return world * units_per_rank / (slowest_ms / 1e3)


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    import tl_synth
    w = tl_synth.make_model_weights(tl_synth.LOOPED_LM, tl_synth.SEED_LM)
    prompt = tl_synth.make_tokens(tl_synth.SEED_LM, tl_synth.LOOPED_LM.vocab, PROMPT + 1)
    n_dec = 2
    om = None
    pre, dec = [], []
    for i in range(args.warmup + args.steps):
        p, d, om = oracle_sample(w, prompt, n_dec, om)
        if i >= args.warmup:
            pre.append(p)
            dec.append(d)
    cores = blas_threads()
    value = n_dec * len(dec) / sum(dec)
    sample = (f"per step: oracle prefill of the 128-token prompt + {n_dec} cached greedy decode "
              f"steps at L=8 (float64 NumPy)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * (sum(pre) + sum(dec)) / len(dec),
        "prefill_ms": 1e3 * statistics.mean(pre),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded random weights and token ids)",
        "config": bench_config(world, STEPS_DECODE, "auto", True),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ncu_case(args):
    """A small eager run of the same model for kernel profilers (no timing
    output): `decode` = prefill of the prompt + --decode-steps greedy steps,
    `prefill` = two prefills of the prompt (--ncu-prompt tokens, default the
    bench's 128)."""
    import torch
    import tl_synth
    import weight_shared_looped_int4_b200 as tl
    shape = tl_synth.LOOPED_LM
    w = tl_synth.make_model_weights(shape, tl_synth.SEED_LM)
    P = args.ncu_prompt
    prompt = tl_synth.make_tokens(tl_synth.SEED_LM, shape.vocab, P + 1)
    steps = args.decode_steps
    cfg = tl.make_config(shape, max_loops=LOOPS, max_ctx=P + max(steps, 1), max_lanes=1)
    tw, keep = tl.make_weights(w)
    m = tl.tl_model_create(cfg, tw, 0)
    del keep
    tl.tl_model_set_graphs(m, False)
    tl.tl_model_set_decode_path(m, DECODE_PATHS[args.decode_path])
    d_prompt = torch.as_tensor(prompt, device="cuda:0")
    hist = torch.zeros(steps + 1, dtype=torch.int32, device="cuda:0")
    hp = hist.data_ptr()
    for _ in range(2 if args.ncu_case == "prefill" else 1):
        tl.tl_prefill(m, 0, d_prompt, P, LOOPS)
    if args.ncu_case == "decode":
        hist[0:1].copy_(d_prompt[P:P + 1])
        for i in range(steps):
            tl.tl_decode_step(m, [0], hp + 4 * i, [LOOPS], None, hp + 4 * (i + 1))
    torch.cuda.synchronize()
    tl.tl_check_device_error(m)
    tl.tl_model_destroy(m)
    print(json.dumps({"ncu_case": args.ncu_case, "decode_steps": steps, "ok": True}))
    return 0


PHASES = ["qkv", "attention", "o_proj", "gate_up", "down"]


def run_trace(args):
    """Phase timeline (globaltimer) of the single-kernel decode step at the
    workload's mid-decode context: per phase, the time from the previous
    barrier's release to the last CTA's arrival (work) and from that arrival
    to the last release (barrier), averaged over the effective layers."""
    import torch
    import tl_synth
    import weight_shared_looped_int4_b200 as tl
    shape = tl_synth.LOOPED_LM
    w = tl_synth.make_model_weights(shape, tl_synth.SEED_LM)
    prompt = tl_synth.make_tokens(tl_synth.SEED_LM, shape.vocab, PROMPT + 1)
    cfg = tl.make_config(shape, max_loops=LOOPS, max_ctx=PROMPT + 64, max_lanes=1)
    tw, keep = tl.make_weights(w)
    m = tl.tl_model_create(cfg, tw, 0)
    del keep
    tl.tl_model_set_decode_path(m, DECODE_PATHS["fused"])
    d_prompt = torch.as_tensor(prompt, device="cuda:0")
    tl.tl_prefill(m, 0, d_prompt, PROMPT, LOOPS)
    G = tl.tl_model_trace_grid(m)
    n_bar = 5 * (2 + LOOPS)
    buf = torch.zeros((4 + 5 * n_bar) * G, dtype=torch.int64, device="cuda:0")
    tok = torch.zeros(2, dtype=torch.int32, device="cuda:0")
    tok[0:1].copy_(d_prompt[PROMPT:PROMPT + 1])
    for i in range(8):   # warm, then keep the last step's timeline
        if i == 7:
            tl.tl_model_set_trace(m, buf, buf.numel())
        tl.tl_decode_step(m, [0], tok, [LOOPS], None, tok)
    torch.cuda.synchronize()
    tl.tl_check_device_error(m)
    tl.tl_model_destroy(m)
    tw, keep = tl.make_weights(w)   # for the second model below
    t = buf.cpu().numpy().reshape(-1, G).astype(np.float64)
    t0 = t[0].min()
    t = (t - t0) / 1e3   # us from the first CTA's start
    slot = lambda s: t[s]
    stats = {p: ({"load": [], "scores": [], "softmax_pv": [], "finish": []} if p == "attention" else
                 {"stage": [], "first_weights_wait": [], "items": [], "epilogue": []}) for p in PHASES}
    for p in PHASES:
        stats[p].update({"work_max": [], "work_median": []})
    barrier = []
    prev = slot(0)
    for k in range(n_bar):
        p = PHASES[k % 5]
        arr, rel = slot(1 + 5 * k), slot(2 + 5 * k)
        st = stats[p]
        st["work_max"].append(float(arr.max() - prev.max()))
        st["work_median"].append(float(np.median(arr - prev)))
        if p == "attention":
            ld, sc_, pv = slot(3 + 5 * k), slot(4 + 5 * k), slot(5 + 5 * k)
            has = ld > 0   # CTAs with an attention unit
            st["load"].append(float(np.median((ld - prev)[has])))
            st["scores"].append(float(np.median((sc_ - ld)[has])))
            st["softmax_pv"].append(float(np.median((pv - sc_)[has])))
            st["finish"].append(float(np.median((arr - pv)[has])))
        else:
            staged, ready, done = slot(3 + 5 * k), slot(4 + 5 * k), slot(5 + 5 * k)
            has = ready > 0   # CTAs with weight items in this phase
            st["stage"].append(float(np.median((staged - prev)[has])))
            st["first_weights_wait"].append(float(np.median(np.maximum(ready - staged, 0)[has])))
            st["items"].append(float(np.median((done - np.maximum(ready, staged))[has])))
            st["epilogue"].append(float(np.median((arr - done)[has])))
        barrier.append(float(rel.max() - arr.max()))
        prev = rel
    hs, hd_, end = slot(1 + 5 * n_bar), slot(2 + 5 * n_bar), slot(3 + 5 * n_bar)
    mean = lambda v: round(statistics.mean(v), 2) if v else None
    out = {"trace": "single-kernel decode step, LM L=8, context %d" % (PROMPT + 8), "grid": G,
           "total_us": round(float(end.max()), 2),
           "start_skew_us": round(float(t[0].max()), 2),
           "per_layer_us": {p: {k: mean(v) for k, v in st.items()} for p, st in stats.items()},
           "barrier_us_mean": round(statistics.mean(barrier), 3),
           "barrier_us_max": round(max(barrier), 3),
           "head_us": {"stage": round(float(np.median(hs - prev)), 2),
                       "tiles_median": round(float(np.median(hd_ - hs)), 2),
                       "tiles_max": round(float((hd_ - hs).max()), 2),
                       "total": round(float(end.max() - prev.max()), 2)},
           "layers": 2 + LOOPS, "barriers": n_bar}
    # the per-op path's head (the persistent kernel in head-only mode), in a
    # captured decode graph
    m = tl.tl_model_create(cfg, tw, 0)
    tl.tl_model_set_decode_path(m, DECODE_PATHS["layered"])
    tl.tl_prefill(m, 0, d_prompt, PROMPT, LOOPS)
    n_rec = 4 * (2 + LOOPS)   # layer launches: QKV + attention, O, gate_up, down
    hbuf = torch.zeros(4 * G + 12 * n_rec, dtype=torch.int64, device="cuda:0")
    tl.tl_model_set_trace(m, hbuf, hbuf.numel())
    tok[0:1].copy_(d_prompt[PROMPT:PROMPT + 1])
    heads, recs = [], []
    for i in range(8):
        hbuf.zero_()   # the layer records take the max over CTAs
        tl.tl_decode_step(m, [0], tok, [LOOPS], None, tok)
        torch.cuda.synchronize()
        raw = hbuf.cpu().numpy()
        h = raw[:4 * G].reshape(4, G).astype(np.float64) / 1e3
        heads.append((float(h[1].max() - h[0].min()), float(np.median(h[2] - h[1])), float(h[2].max() - h[1].min()),
                      float(h[3].max() - h[0].min())))
        last_h = h
        r = raw[4 * G:].reshape(n_rec, 12).view(np.uint64).copy()
        r[:, 0] = ~r[:, 0]   # the first start is stored complemented
        recs.append((r.astype(np.float64) / 1e3, float(h[0].min()), float(h[3].max())))
    tl.tl_model_destroy(m)
    hs = heads[2:]
    out["layered_head_us"] = {"start_to_staged": round(statistics.mean(x[0] for x in hs), 2),
                              "tiles_median": round(statistics.mean(x[1] for x in hs), 2),
                              "tiles_span": round(statistics.mean(x[2] for x in hs), 2),
                              "total": round(statistics.mean(x[3] for x in hs), 2)}
    # per layer kernel, in the captured graph: its share of the step's critical
    # path (previous launch's last CTA end -> its own last CTA end), how long
    # its CTAs waited for the previous kernel's end, and its phases after that
    names = ("qkv_attn", "o_proj", "gate_up", "down")
    acc = {n: {"critical_path": [], "started_before_prev_end": [], "release_after_prev_end": [],
               "phase1": [], "phase2": [], "phase3": [], "phase1a": [], "phase2a": []} for n in names}
    step_us, head_tail = [], []
    for r, h_start, h_end in recs[2:]:
        step_us.append(h_end - r[0, 0])
        head_tail.append(h_end - r[-1, 5])
        for i in range(1, n_rec):
            a = acc[names[i % 4]]
            prev_end = r[i - 1, 5]
            a["critical_path"].append(r[i, 5] - prev_end)
            a["started_before_prev_end"].append(prev_end - r[i, 1])
            a["release_after_prev_end"].append(r[i, 2] - prev_end)
            rel = r[i, 2]
            if i % 4 == 0:   # clustered: GEMV + exchange, attention + exchange, merge
                a["phase1"].append(r[i, 3] - rel)
                a["phase2"].append(r[i, 4] - r[i, 3])
                a["phase1a"].append(r[i, 6] - rel)        # to the last arrival at barrier 1
                a["phase2a"].append(r[i, 7] - r[i, 3])    # to the last arrival at barrier 2
                for key, v in (("norm", r[i, 8] - rel), ("weights", r[i, 9] - r[i, 8]),
                               ("gemv", r[i, 10] - r[i, 9]), ("epilogue", r[i, 6] - r[i, 10]),
                               ("keys_after_barrier1", r[i, 11] - r[i, 3])):
                    a.setdefault("p1_" + key, []).append(v)
            else:            # GEMV: weights-ready wait after release, main loop, epilogue
                a["phase1"].append(max(r[i, 3] - rel, 0.0))
                a["phase2"].append(r[i, 4] - max(r[i, 3], rel))
                a["phase1a"].append(r[i, 6] - rel)        # activations staged
                a["phase2a"].append(0.0)
            a["phase3"].append(r[i, 5] - r[i, 4])
    r, h_start, h_end = recs[-1]
    out["layered_last_step_per_launch"] = [
        [round(float(v), 2) for v in (r[i, 5] - (r[i - 1, 5] if i else r[i, 0]), r[i, 2] - r[i, 1],
                                      r[i, 3] - r[i, 2], r[i, 4] - r[i, 3], r[i, 5] - r[i, 4])]
        for i in range(n_rec)]
    out["layered_step_us"] = round(statistics.mean(step_us), 2)
    out["layered_head_after_last_down_us"] = round(statistics.mean(head_tail), 2)
    d_end = r[-1, 5]
    out["layered_head_last_step_vs_down_end_us"] = {
        "first_start": round(float(last_h[0].min() - d_end), 2), "median_start": round(float(np.median(last_h[0]) - d_end), 2),
        "last_start": round(float(last_h[0].max() - d_end), 2), "median_staged": round(float(np.median(last_h[1]) - d_end), 2),
        "last_staged": round(float(last_h[1].max() - d_end), 2), "last_end": round(float(last_h[3].max() - d_end), 2)}
    out["layered_kernels_us"] = {n: {k: round(statistics.mean(v), 2) for k, v in a.items()} for n, a in acc.items()}
    out["layered_phases"] = {"qkv_attn": "phase1 RMSNorm+QKV GEMV+RoPE+exchange (phase1a: up to the last "
                                         "arrival at its barrier), phase2 attention+exchange (phase2a: likewise), "
                                         "phase3 merge",
                             "gemv": "phase1 release to weights ready (phase1a: activations staged), "
                                     "phase2 main loop, phase3 epilogue"}
    print(json.dumps(out))
    return 0


def run_ours(args):
    import torch
    import tl_synth
    import weight_shared_looped_int4_b200 as tl

    world, rank, local = dist_env()
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
        pg = dist

    shape = tl_synth.LOOPED_LM
    w = tl_synth.make_model_weights(shape, tl_synth.SEED_LM)
    prompt = tl_synth.make_tokens(tl_synth.SEED_LM, shape.vocab, PROMPT + 1)
    n_dec = args.decode_steps
    cfg = tl.make_config(shape, max_loops=LOOPS, max_ctx=PROMPT + n_dec, max_lanes=1)
    tw, keep = tl.make_weights(w)
    m = tl.tl_model_create(cfg, tw, local)
    del keep
    if args.no_graphs:
        tl.tl_model_set_graphs(m, False)
    tl.tl_model_set_decode_path(m, DECODE_PATHS[args.decode_path])

    st = torch.cuda.Stream(device=dev)
    d_prompt = torch.as_tensor(prompt, device=dev)
    hist = torch.zeros(n_dec + 1, dtype=torch.int32, device=dev)
    hp = hist.data_ptr()

    def step(ev=None):
        with torch.cuda.stream(st):
            if ev:
                ev[0].record(st)
            tl.tl_prefill(m, 0, d_prompt, PROMPT, LOOPS, None, None, st)
            if ev:
                ev[1].record(st)
            hist[0:1].copy_(d_prompt[PROMPT:PROMPT + 1])
            for i in range(n_dec):
                tl.tl_decode_step(m, [0], hp + 4 * i, [LOOPS], None, hp + 4 * (i + 1), st)
            if ev:
                ev[2].record(st)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    launches0 = tl.tl_kernel_launch_count()
    with ClockSampler(local) as clocks:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(st)
        for i in range(args.steps):
            step(evs[i])
        t_end.record(st)
        torch.cuda.synchronize()
    launches = tl.tl_kernel_launch_count() - launches0
    if pg:
        pg.barrier()
    torch.cuda.synchronize()

    total_ms = t_start.elapsed_time(t_end)
    prefill_ms = [e[0].elapsed_time(e[1]) for e in evs]
    decode_ms = [e[1].elapsed_time(e[2]) for e in evs]
    total_ms, prefill_sum, decode_sum = max_over_ranks(pg, [total_ms, sum(prefill_ms), sum(decode_ms)], dev)
    value = whole_job_rate(world, n_dec * args.steps, decode_sum)
    generated = hist[1:].cpu().numpy().copy()

    # ---- end to end: pinned host prompt in, generated tokens out, per step --
    h_prompt = torch.from_numpy(prompt.copy()).pin_memory()
    h_out = torch.empty(n_dec, dtype=torch.int32).pin_memory()
    e2e_ms = []
    for i in range(0 if args.no_e2e else args.warmup + args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(st):
            a.record(st)
            d_prompt.copy_(h_prompt, non_blocking=True)
            step()
            h_out.copy_(hist[1:], non_blocking=True)
            b.record(st)
        b.synchronize()
        if i >= args.warmup:
            e2e_ms.append(a.elapsed_time(b))
    (e2e_slowest,) = max_over_ranks(pg, [sum(e2e_ms) if e2e_ms else float("nan")], dev)
    e2e_value = whole_job_rate(world, n_dec * args.steps, e2e_slowest) if e2e_ms else None
    if e2e_ms:
        assert np.array_equal(h_out.numpy(), generated), "end-to-end run diverged from the timed run"

    # ---- per-token byte roofline ------------------------------------------
    # HBM bytes (pre blocks, head, KV reads) at the measured HBM copy bandwidth
    # + the loop block's re-reads (L2-resident) at the measured L2 read
    # bandwidth (library probe over a buffer the size of the loop block).
    peaks = load_peaks()
    mean_keys = PROMPT + (n_dec + 1) / 2
    layer_bytes = sum(BYTES_PER_LAUNCH[k] for k in ("qkv", "o_proj", "gate_up", "down"))
    hbm_bytes = 2 * layer_bytes + BYTES_PER_LAUNCH["head"] + 10 * _attn_bytes_per_launch(mean_keys)
    l2_bytes = LOOPS * layer_bytes
    l2_gbs, l2_probe_bytes, hbm_read_gbs = probe_read_bandwidths(tl, torch, dev, st)
    t_roof_us = hbm_bytes / (peaks["hbm_gbs"] * 1e3) + l2_bytes / (l2_gbs * 1e3)
    t_tok_us = 1e3 * decode_sum / (args.steps * n_dec)
    roof_step = {"hbm_bytes_per_token": int(hbm_bytes), "l2_bytes_per_token": int(l2_bytes),
                 "hbm_gbs": peaks["hbm_gbs"], "l2_read_gbs_measured": round(l2_gbs, 1),
                 "l2_probe": f"{l2_probe_bytes >> 20} MiB buffer (half the L2), 200 sweeps in one launch",
                 "hbm_plain_read_gbs_measured": round(hbm_read_gbs, 1),
                 "roofline_us_per_token": round(t_roof_us, 2),
                 "achieved_us_per_token": round(t_tok_us, 2), "frac": round(t_roof_us / t_tok_us, 4)}

    # ---- per-kernel profile of one decode phase (separate from the timing) -
    per_class, roofline = {}, None
    if not args.no_profile:
        with torch.cuda.stream(st):
            tl.tl_prefill(m, 0, d_prompt, PROMPT, LOOPS, None, None, st)
            hist[0:1].copy_(d_prompt[PROMPT:PROMPT + 1])
            st.synchronize()
            tl.tl_model_profile_start(m)
            for i in range(n_dec):
                tl.tl_decode_step(m, [0], hp + 4 * i, [LOOPS], None, hp + 4 * (i + 1), st)
            prof = tl.tl_model_profile_stop(m)
        step_bytes = hbm_bytes + l2_bytes

        # with the clustered QKV + attention kernel (no separate attention
        # launches) the "qkv" class also reads the KV cache
        attn_in_qkv = "attn_decode" not in prof

        def bytes_of(name):
            if name == "attn_decode":
                return _attn_bytes_per_launch(mean_keys)
            if name == "decode_fused":
                return step_bytes
            if name == "qkv" and attn_in_qkv:
                return BYTES_PER_LAUNCH["qkv"] + _attn_bytes_per_launch(mean_keys)
            return BYTES_PER_LAUNCH.get(name)

        for name, (n, ms) in prof.items():
            avg_us = 1e3 * ms / n
            b = bytes_of(name)
            per_class[name] = {"launches": n, "total_ms": round(ms, 4), "avg_us": round(avg_us, 3),
                               "gbs": round(b / (avg_us * 1e3), 1) if b else None}
        dom = max(per_class, key=lambda k: per_class[k]["total_ms"])
        dom_b = bytes_of(dom)
        avg_us = per_class[dom]["avg_us"]
        if dom == "decode_fused":
            # one launch = one token: HBM and L2 bytes against the blend of the
            # two measured bandwidths (peak = bytes / roofline time)
            peak = step_bytes / (t_roof_us * 1e3)
            peak_src = (f"blend: {peaks['source']} HBM {peaks['hbm_gbs']} GB/s for {int(hbm_bytes)} B + "
                        f"measured L2 read {round(l2_gbs, 1)} GB/s for {int(l2_bytes)} B")
        else:
            peak = peaks["hbm_gbs"]
            peak_src = peaks["source"] + " HBM copy"
        achieved = dom_b / (avg_us * 1e3) if dom_b else None
        traffic = roofline_traffic(dom, mean_keys) if attn_in_qkv else None
        roofline = {
            "kernel": dom, "bound": "hbm", "achieved": round(achieved, 1) if achieved else None,
            "peak": round(peak, 1), "unit": "GB/s",
            "frac": round(achieved / peak, 4) if achieved else None,
            "traffic": traffic, "peak_source": peak_src,
            "bytes_per_launch": int(dom_b) if dom_b else None,
            "timing": "CUDA events around each launch of one extra decode phase, after the timed region",
        }
    # prefill: dense-equivalent flops of the linears + attention vs tensor peak
    per_layer_flops = 2 * PROMPT * (D * (HQ + 2 * HKV) * HD + HQ * HD * D + D * 2 * F + F * D)
    attn_flops = 4 * HQ * HD * PROMPT * (PROMPT + 1) / 2
    pf_flops = (2 + LOOPS) * (per_layer_flops + attn_flops)
    pf_ms = prefill_sum / args.steps
    roof_prefill = {"flops": int(pf_flops), "achieved_tflops": round(pf_flops / (pf_ms * 1e9), 2),
                    "peak_tflops": peaks["bf16_tflops"], "peak_source": peaks["source"] + " bf16 (fp16 assumed equal)",
                    "frac": round(pf_flops / (pf_ms * 1e9) / peaks["bf16_tflops"], 4)}

    # ---- CPU oracle baseline (rank 0, bounded sample) -----------------------
    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        n_or = 4
        p_s, d_s, om = oracle_sample(w, prompt, n_or)
        cpu = {"value": n_or / d_s, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"oracle prefill of the 128-token prompt ({p_s:.2f} s) + {n_or} cached "
                         f"greedy decode steps at L=8 ({d_s:.2f} s), float64 NumPy"}
        try:   # the same sample on one BLAS thread
            from threadpoolctl import threadpool_limits
            with threadpool_limits(limits=1, user_api="blas"):
                p1, d1, _ = oracle_sample(w, prompt, n_or, om)
            cpu["value_1thread"] = n_or / d1
            cpu["prefill_s_1thread"] = round(p1, 3)
        except ImportError:
            pass

    tl.tl_model_destroy(m)
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total_ms / args.steps, 4),
            "prefill_ms": round(prefill_sum / args.steps, 4),
            "decode_ms_per_token": round(decode_sum / (args.steps * n_dec), 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp16/fp32 (INT4 weights)",
            "data": "synthetic (seeded random weights and token ids)",
            "config": bench_config(world, n_dec, args.decode_path, not args.no_graphs),
            "roofline": roofline,
            "roofline_decode_token": roof_step,
            "roofline_prefill": roof_prefill,
            "kernels_decode": per_class,
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_value, 2) if e2e_value else None, "unit": UNIT,
                    "h2d_bytes_per_step": int(h_prompt.numel() * 4),
                    "d2h_bytes_per_step": int(h_out.numel() * 4)},
            "gpu_launches": int(launches),
            "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0


# ------------------------------------------------------- other workloads ---
# `--workload tiny|linear|attention|lsweep|peaks` times the kernels on the
# shapes of the other workloads (one JSON line each, rank 0, one GPU).  The
# headline line above stays the 400M-LM L=8 step.

def _dev_setup():
    import torch
    torch.cuda.set_device(0)
    return torch, torch.device("cuda", 0), torch.cuda.Stream(device=0)


def _l2_flusher(torch, dev):
    """Writes a buffer twice the L2 size (on the current stream): between
    timed repetitions, so each starts with a cold L2."""
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    buf = torch.empty(2 * l2 // 4, dtype=torch.float32, device=dev)
    return lambda: buf.fill_(1.0)


def _time_reps(torch, st, fn, reps, flush=None):
    """Median ms of `reps` CUDA-event-timed calls of fn() on stream st (flush()
    runs between them, outside the events)."""
    out = []
    with torch.cuda.stream(st):
        for _ in range(reps):
            if flush:
                flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            fn()
            b.record(st)
            b.synchronize()
            out.append(a.elapsed_time(b))
    return statistics.median(out)


def _time_graph(torch, st, fn, reps, launches=20):
    """Median per-call ms of fn() with the host out of the way: `launches`
    calls captured in one CUDA graph, the graph replayed `reps` times."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(st):
        fn()                       # warm (workspaces exist before the capture)
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=st):
        for _ in range(launches):
            fn()
    out = []
    with torch.cuda.stream(st):
        g.replay()
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            g.replay()
            b.record(st)
            b.synchronize()
            out.append(a.elapsed_time(b) / launches)
    del g
    return statistics.median(out)


def tensor_peak_probe(torch, dev):
    """Dense fp16 and bf16 tensor-core throughput of torch.matmul (cuBLAS) at
    8192^3, TFLOP/s, 20 timed reps after 5 warm-ups."""
    n = 8192
    res = {}
    for name, dt in (("fp16", torch.float16), ("bf16", torch.bfloat16)):
        a = torch.randn(n, n, device=dev, dtype=dt)
        b = torch.randn(n, n, device=dev, dtype=dt)
        for _ in range(5):
            torch.matmul(a, b)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(20):
            torch.matmul(a, b)
        e1.record()
        e1.synchronize()
        res[name] = round(2 * n ** 3 * 20 / (e0.elapsed_time(e1) * 1e9), 1)
        del a, b
    torch.cuda.empty_cache()
    return res


def run_workload_peaks(args):
    torch, dev, st = _dev_setup()
    import weight_shared_looped_int4_b200 as tl
    with ClockSampler(0) as clocks:
        tc = tensor_peak_probe(torch, dev)
        l2, l2_bytes, hbm = probe_read_bandwidths(tl, torch, dev, st)
    print(json.dumps({"workload": "peaks", "tensor_tflops_torch_matmul_8192": tc,
                      "l2_read_gbs": round(l2, 1), "l2_probe_bytes": l2_bytes,
                      "hbm_plain_read_gbs": round(hbm, 1), "measured_peaks_file": load_peaks(),
                      "clocks": clocks.summary()}))
    return 0


def run_workload_linear(args):
    """INT4 group-128 linear sweep: M in {1,4,16,128} x the four (K, N), the
    library's default path per M, L2-cold (flushed) and L2-warm; torch fp16
    matmul on the dequantized weight as the comparator (context only)."""
    torch, dev, st = _dev_setup()
    import tl_synth
    import weight_shared_looped_int4_b200 as tl
    peaks = load_peaks()
    flush = _l2_flusher(torch, dev)
    rows = []
    launches0 = tl.tl_kernel_launch_count()
    with ClockSampler(0) as clocks:
        tc_peak = tensor_peak_probe(torch, dev)
        for K, N in tl_synth.LINEAR_SWEEP_KN:
            rng = np.random.default_rng(tl_synth.SEED_LINEAR + K + N)
            lin = tl_synth.make_int4_linear(rng, N, K)
            h = tl.tl_linear_create(lin, K, N, 0)
            # fp16 comparator: the same weights dequantized on the device by torch
            q = torch.from_numpy(lin.qweight.view(np.int32)).to(dev)
            nib = torch.stack([(q >> (4 * j)) & 15 for j in range(8)], dim=-1).reshape(N, -1)[:, :K]
            zw = torch.from_numpy(lin.qzeros.view(np.int32)).to(dev)
            z = torch.stack([(zw >> (4 * j)) & 15 for j in range(8)], dim=-1).reshape(N, -1)[:, :K // 128]
            sc = torch.from_numpy(lin.scales.view(np.float16)).to(dev).float()
            w16 = ((nib.view(N, K // 128, 128) - z[:, :, None]).float() * sc[:, :, None]).reshape(N, K).half()
            del q, nib, zw, z, sc
            for M in tl_synth.LINEAR_SWEEP_M:
                x = torch.from_numpy(tl_synth.make_activations(tl_synth.SEED_LINEAR * 7 + M, M, K)).to(dev)
                y = torch.empty((M, N), dtype=torch.float16, device=dev)
                fn = lambda: tl.tl_linear_forward(h, x, M, y, tl.TL_PATH_AUTO, st)
                for _ in range(5):
                    fn()
                cold = _time_reps(torch, st, fn, 30, flush)
                warm = _time_graph(torch, st, fn, 10)
                tfn = lambda: torch.matmul(x, w16.t())
                for _ in range(3):
                    with torch.cuda.stream(st):
                        tfn()
                t_cold = _time_reps(torch, st, tfn, 20, flush)
                nbytes = _int4_bytes(K, N) + 2 * M * K + 2 * M * N
                flops = 2 * M * K * N
                t_hbm = nbytes / (peaks["hbm_gbs"] * 1e3)          # us
                t_tc = flops / (peaks["bf16_tflops"] * 1e6)         # us
                bound = "hbm" if t_hbm >= t_tc else "tensor"
                t_roof = max(t_hbm, t_tc)
                rows.append({"M": M, "K": K, "N": N, "path": "gemv" if M <= 16 else "tcgen05",
                             "us_l2_cold": round(1e3 * cold, 2), "us_l2_warm": round(1e3 * warm, 2),
                             "bytes": nbytes, "flops": flops, "bound": bound,
                             "achieved_cold": round(nbytes / (cold * 1e6), 1) if bound == "hbm"
                             else round(flops / (cold * 1e9), 1),
                             "unit": "GB/s" if bound == "hbm" else "TFLOP/s",
                             "roofline_us": round(t_roof, 3),
                             "frac_cold": round(t_roof / (1e3 * cold), 4),
                             "frac_warm": round(t_roof / (1e3 * warm), 4),
                             "torch_fp16_dequantized_us_l2_cold": round(1e3 * t_cold, 2)})
            tl.tl_linear_destroy(h)
            del w16
    print(json.dumps({"workload": "INT4 g128 linear sweep (fp16 x, fp32 acc, fp16 y)",
                      "metric": "per-shape us and fraction of roofline", "peaks": peaks,
                      "tensor_tflops_torch_matmul_8192": tc_peak,
                      "timing": "cold: median of 30 CUDA-event reps with a 2xL2 buffer written before each (its run hides the host's issue time); warm: 20 calls captured in one CUDA graph, median of 10 replays / 20",
                      "results": rows, "gpu_launches": tl.tl_kernel_launch_count() - launches0,
                      "clocks": clocks.summary()}))
    return 0


def run_workload_attention(args):
    """GQA attention, D 2048, 16 Q / 4 KV heads of 128: single-query decode
    over S in {128,1024,4096,8192} and causal prefill at T in {128,512,2048},
    batch 1 and 8; fp16 N(0,1) inputs; RoPE by the in-place op (timed apart)."""
    torch, dev, st = _dev_setup()
    import tl_synth
    import weight_shared_looped_int4_b200 as tl
    peaks = load_peaks()
    flush = _l2_flusher(torch, dev)
    dec, pre = [], []
    launches0 = tl.tl_kernel_launch_count()
    with ClockSampler(0) as clocks:
        for B in (1, 8):
            for S in (128, 1024, 4096, 8192):
                q, k, v = tl_synth.make_qkv(tl_synth.SEED_ATTN + S + B, B, S, HQ, HKV, HD, T_q=1)
                kc = torch.from_numpy(np.ascontiguousarray(k.transpose(0, 2, 1, 3))).to(dev)
                vc = torch.from_numpy(np.ascontiguousarray(v.transpose(0, 2, 1, 3))).to(dev)
                qd = torch.from_numpy(np.ascontiguousarray(q[:, 0])).to(dev)
                out = torch.empty((B, HQ, HD), dtype=torch.float16, device=dev)
                pos = torch.full((B,), S - 1, dtype=torch.int32, device=dev)
                fn = lambda: tl.tl_op_gqa_decode(qd, kc, vc, HKV * S * HD, S, [S] * B, B, HQ, HKV, HD, out, st)
                rope = lambda: tl.tl_op_rope(qd, B, HQ, HD, HQ * HD, HD, pos, 1e4, st)
                for _ in range(5):
                    fn()
                cold = _time_reps(torch, st, fn, 30, flush)
                warm = _time_graph(torch, st, fn, 10)
                t_rope = _time_graph(torch, st, rope, 10)
                nbytes = B * (2 * HKV * S * HD * 2 + 2 * HQ * HD * 2)
                t_roof = nbytes / (peaks["hbm_gbs"] * 1e3)
                dec.append({"B": B, "S": S, "us_l2_cold": round(1e3 * cold, 2), "us_l2_warm": round(1e3 * warm, 2),
                            "bytes": nbytes, "gbs_cold": round(nbytes / (cold * 1e6), 1),
                            "frac_cold": round(t_roof / (1e3 * cold), 4), "rope_q_us": round(1e3 * t_rope, 2)})
                del kc, vc
        for B in (1, 8):
            for T in (128, 512, 2048):
                q, k, v = tl_synth.make_qkv(tl_synth.SEED_ATTN + 7 * T + B, B, T, HQ, HKV, HD)
                kc = torch.from_numpy(np.ascontiguousarray(k.transpose(0, 2, 1, 3))).to(dev)
                vc = torch.from_numpy(np.ascontiguousarray(v.transpose(0, 2, 1, 3))).to(dev)
                qd = torch.from_numpy(np.ascontiguousarray(q)).to(dev)
                out = torch.empty((B, T, HQ, HD), dtype=torch.float16, device=dev)
                fn = lambda: tl.tl_op_gqa_prefill(qd, kc, vc, HKV * T * HD, T, T, 0, B, HQ, HKV, HD, out, st)
                flops = B * 4 * HQ * HD * T * (T + 1) / 2
                t_roof = flops / (peaks["bf16_tflops"] * 1e6)
                rec = {"B": B, "T": T, "flops": int(flops)}
                for min_tc, kname in ((1, "tcgen05"), (1 << 30, "mma_sync")):
                    tl.tl_set_prefill_attention_tc_min(min_tc)
                    for _ in range(3):
                        fn()
                    cold = _time_reps(torch, st, fn, 10, flush)
                    warm = _time_graph(torch, st, fn, 5, launches=5)
                    best = min(cold, warm)
                    rec[kname] = {"us_l2_cold": round(1e3 * cold, 2), "us_graph": round(1e3 * warm, 2),
                                  "tflops": round(flops / (best * 1e9), 2), "frac": round(t_roof / (1e3 * best), 4)}
                tl.tl_set_prefill_attention_tc_min(1024)
                pre.append(rec)
                del kc, vc, qd, out
    print(json.dumps({"workload": "GQA attention D2048 16q/4kv hd128 (fp16 KV)",
                      "metric": "per-case us and fraction of roofline", "peaks": peaks,
                      "decode": dec, "prefill": pre,
                      "context_h100_from_pages": {"decode_K128_D2048_16heads_ms": 0.092,
                                                  "prefill_T128_ms": [0.143, 0.087]},
                      "timing": "cold: median of CUDA-event reps with a 2xL2 buffer written before each; warm / graph: calls captured in one CUDA graph, per-call median of the replays",
                      "gpu_launches": tl.tl_kernel_launch_count() - launches0,
                      "clocks": clocks.summary()}))
    return 0


def _lm_model(tl, tl_synth, max_loops, max_ctx, max_lanes, kv_mode=0, bits=4):
    shape = tl_synth.LOOPED_LM
    w = tl_synth.make_model_weights(shape, tl_synth.SEED_LM, bits=bits)
    cfg = tl.make_config(shape, max_loops=max_loops, max_ctx=max_ctx, max_lanes=max_lanes, kv_mode=kv_mode,
                         weight_bits=bits)
    tw, keep = tl.make_weights(w)
    m = tl.tl_model_create(cfg, tw, 0)
    del keep
    return w, m


def _decode_roofline_us(n_rows_kv, loops_list, l2_gbs, peaks):
    """Byte roofline of one decode step (us): pre blocks + head + KV reads
    from HBM, the loop block once per iteration of the longest lane from L2."""
    layer = sum(BYTES_PER_LAUNCH[k] for k in ("qkv", "o_proj", "gate_up", "down"))
    hbm = 2 * layer + BYTES_PER_LAUNCH["head"] + n_rows_kv
    l2 = max(loops_list) * layer
    return hbm / (peaks["hbm_gbs"] * 1e3) + l2 / (l2_gbs * 1e3), hbm, l2


def run_workload_lsweep(args):
    """The 400M LM swept over loops L in {1,2,4,8,16}: prefill of a 512-token
    prompt (no logits) and 256 greedy decode steps at batch 1; then 1/4/16
    lanes with per-lane loops drawn from {4,8,16}, 512-token prompts each,
    256 decode steps (max context 2048)."""
    torch, dev, st = _dev_setup()
    import tl_synth
    import weight_shared_looped_int4_b200 as tl
    peaks = load_peaks()
    P, n_dec = 512, args.decode_steps if args.decode_steps != STEPS_DECODE else 256
    w, m = _lm_model(tl, tl_synth, 16, 2048, 16)
    l2_gbs, _, _ = probe_read_bandwidths(tl, torch, dev, st)
    prompts = tl_synth.make_lane_prompts(tl_synth.SEED_LSWEEP, w.shape.vocab, 16, P + 1)
    d_prompts = torch.as_tensor(prompts, device=dev)
    hist = torch.zeros((n_dec + 1, 16), dtype=torch.int32, device=dev)
    hp = hist.data_ptr()
    per_layer_flops = 2 * P * (D * (HQ + 2 * HKV) * HD + HQ * HD * D + D * 2 * F + F * D)
    attn_flops = 4 * HQ * HD * P * (P + 1) / 2
    sweep, lanes_res = [], []
    launches0 = tl.tl_kernel_launch_count()

    def decode_run(lanes, loops):
        n = len(lanes)
        for i, lane in enumerate(lanes):
            tl.tl_prefill(m, lane, d_prompts[lane], P, loops[i], None, None, st)
        with torch.cuda.stream(st):
            hist[0, :n].copy_(d_prompts[:n, P])
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        for i in range(n_dec):
            tl.tl_decode_step(m, lanes, hp + 64 * i, loops, None, hp + 64 * (i + 1), st)
        b.record(st)
        b.synchronize()
        return a.elapsed_time(b)

    with ClockSampler(0) as clocks:
        # batch 1: the clustered per-op form (a model built for <= 2 lanes takes
        # it by default; this one holds 16 lanes for the lane rows below)
        tl.tl_model_set_clustered_decode(m, True)
        for L in (1, 2, 4, 8, 16):
            fn = lambda: tl.tl_prefill(m, 0, d_prompts[0], P, L, None, None, st)
            for _ in range(3):
                fn()
            pf = _time_reps(torch, st, fn, 10)
            flops = (2 + L) * (per_layer_flops + attn_flops)
            decode_run([0], [L])          # warm (graph capture)
            ms = decode_run([0], [L])
            kv = (2 + L) * 2 * HKV * HD * 2 * (P + n_dec / 2)
            t_roof, _, _ = _decode_roofline_us(kv, [L], l2_gbs, peaks)
            us_tok = 1e3 * ms / n_dec
            sweep.append({"L": L, "decode_form": "clustered", "prefill_T512_ms": round(pf, 4), "prefill_flops": int(flops),
                          "prefill_tflops": round(flops / (pf * 1e9), 2),
                          "prefill_frac": round(flops / (pf * 1e9) / peaks["bf16_tflops"], 4),
                          "decode_tok_s": round(n_dec / (ms / 1e3), 1), "decode_us_per_step": round(us_tok, 2),
                          "decode_roofline_us": round(t_roof, 2), "decode_frac": round(t_roof / us_tok, 4)})
        for n in (1, 4, 16):
            # the form the library picks for a model built for n lanes
            tl.tl_model_set_clustered_decode(m, n <= 2)
            loops = [int(v) for v in tl_synth.make_lane_loops(tl_synth.SEED_LSWEEP, n)]
            lanes = list(range(n))
            decode_run(lanes, loops)      # warm (graph capture)
            ms = decode_run(lanes, loops)
            kv = sum((2 + L) * 2 * HKV * HD * 2 * (P + n_dec / 2) for L in loops)
            t_roof, _, _ = _decode_roofline_us(kv, loops, l2_gbs, peaks)
            us_step = 1e3 * ms / n_dec
            lanes_res.append({"lanes": n, "loops": loops, "decode_form": "clustered" if n <= 2 else "gemv+split-kv",
                              "decode_tok_s": round(n * n_dec / (ms / 1e3), 1),
                              "us_per_step": round(us_step, 2), "roofline_us_per_step": round(t_roof, 2),
                              "frac": round(t_roof / us_step, 4)})
    tl.tl_check_device_error(m)
    tl.tl_model_destroy(m)
    print(json.dumps({"workload": "400M looped LM, L sweep and per-lane loops (prompts 512, ctx 2048)",
                      "metric": "prefill ms (T=512) and decode tok/s per L; decode tok/s per lane count",
                      "decode_steps": n_dec, "peaks": peaks, "l2_read_gbs": round(l2_gbs, 1),
                      "loops_sweep": sweep, "lanes": lanes_res,
                      "gpu_launches": tl.tl_kernel_launch_count() - launches0,
                      "clocks": clocks.summary()}))
    return 0


def run_workload_tiny(args):
    """Tiny looped LM (d 256, 4/2 heads of 64, F 1024, V 512, 1 pre block,
    L = 4): 32-token prompt prefill, then 8 greedy decode steps, batch 1."""
    torch, dev, st = _dev_setup()
    import tl_synth
    import weight_shared_looped_int4_b200 as tl
    shape = tl_synth.TINY_LM
    w = tl_synth.make_model_weights(shape, tl_synth.SEED_TINY)
    cfg = tl.make_config(shape, max_loops=4, max_ctx=64, max_lanes=1)
    tw, keep = tl.make_weights(w)
    m = tl.tl_model_create(cfg, tw, 0)
    del keep
    P, L, n_dec = 32, 4, 8
    prompt = tl_synth.make_tokens(tl_synth.SEED_TINY, shape.vocab, P + 1)
    d_prompt = torch.as_tensor(prompt, device=dev)
    hist = torch.zeros(n_dec + 1, dtype=torch.int32, device=dev)
    hp = hist.data_ptr()
    pre_ms, dec_ms = [], []
    with ClockSampler(0) as clocks:
        for it in range(args.warmup + args.steps):
            a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            with torch.cuda.stream(st):
                a.record(st)
                tl.tl_prefill(m, 0, d_prompt, P, L, None, None, st)
                b.record(st)
                hist[0:1].copy_(d_prompt[P:P + 1])
                for i in range(n_dec):
                    tl.tl_decode_step(m, [0], hp + 4 * i, [L], None, hp + 4 * (i + 1), st)
                c.record(st)
            c.synchronize()
            if it >= args.warmup:
                pre_ms.append(a.elapsed_time(b))
                dec_ms.append(b.elapsed_time(c))
    tl.tl_model_destroy(m)
    print(json.dumps({"workload": "tiny looped LM d256 4q/2kv hd64 F1024 V512 n_pre1 L4; prompt 32 + 8 greedy steps",
                      "prefill_ms": round(statistics.median(pre_ms), 4),
                      "decode_tok_s": round(n_dec / (statistics.median(dec_ms) / 1e3), 1),
                      "decode_us_per_token": round(1e3 * statistics.median(dec_ms) / n_dec, 2),
                      "roofline": None,
                      "note": "0.51 MB per block pass: launch/latency bound, no roofline claim",
                      "clocks": clocks.summary()}))
    return 0


def run_workload_next(args):
    """The 400M LM around the forward pass: greedy self-speculative decoding
    (draft 2 or 4 loops, verify 8, look-ahead 4) against plain greedy decode,
    the logit lens and early exit against score_last, and forking a cached
    512-token prefix against prefilling it again."""
    torch, dev, st = _dev_setup()
    import tl_synth
    import weight_shared_looped_int4_b200 as tl
    peaks = load_peaks()
    w, m = _lm_model(tl, tl_synth, 16, 1024, 4)
    # single-lane decoding throughout: the clustered per-op form (the default
    # of a model built for <= 2 lanes; this one holds 4 for the prefix forks)
    tl.tl_model_set_clustered_decode(m, True)
    P, n = 128, 128
    prompt = tl_synth.make_tokens(tl_synth.SEED_LM, w.shape.vocab, 1024)
    d_prompt = torch.as_tensor(prompt, device=dev)
    out = torch.zeros(n, dtype=torch.int32, device=dev)
    hist = torch.zeros(n + 1, dtype=torch.int32, device=dev)
    hp = hist.data_ptr()
    res = {}
    launches0 = tl.tl_kernel_launch_count()

    def ev_ms(fn):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        fn()
        b.record(st)
        b.synchronize()
        return a.elapsed_time(b)

    with ClockSampler(0) as clocks:
        def plain():
            for i in range(n):
                tl.tl_decode_step(m, [0], hp + 4 * i, [LOOPS], None, hp + 4 * (i + 1), st)
        for rep in range(3):
            tl.tl_prefill(m, 0, d_prompt, P, LOOPS, None, None, st)
            with torch.cuda.stream(st):
                hist[0:1].copy_(d_prompt[P:P + 1])
            t_plain = ev_ms(plain)
        greedy_tokens = hist[1:].cpu().numpy().copy()
        res["plain_decode_tok_s"] = round(n / (t_plain / 1e3), 1)
        for draft in (2, 4):
            for rep in range(3):
                tl.tl_prefill(m, 0, d_prompt, P, LOOPS, None, None, st)
                stats = {}
                t = ev_ms(lambda: stats.update(tl.tl_generate_speculative(m, 0, d_prompt[P:], n, draft, 4, out, st)))
            same = int(np.sum(out.cpu().numpy() == greedy_tokens))
            res[f"speculative_draft{draft}_ahead4"] = {
                "tok_s": round(n / (t / 1e3), 1), "rounds": stats["rounds"], "drafted": stats["drafted"],
                "accepted": stats["accepted"], "acceptance": round(stats["accepted"] / stats["drafted"], 4),
                "tokens_equal_to_plain_greedy": same}
        d_tok = d_prompt[:P]
        lg = torch.empty((LOOPS, V), dtype=torch.float32, device=dev)
        for _ in range(3):
            tl.tl_score_last(m, d_tok, P, LOOPS, lg[0], None, st)
        t_sl = statistics.median(ev_ms(lambda: tl.tl_score_last(m, d_tok, P, LOOPS, lg[0], None, st))
                                 for _ in range(10))
        t_lens = statistics.median(ev_ms(lambda: tl.tl_score_logit_lens(m, d_tok, P, LOOPS, lg, None, st))
                                   for _ in range(10))
        used = []
        t_exit = statistics.median(ev_ms(lambda: used.append(
            tl.tl_score_early_exit(m, d_tok, P, 16, 2, lg[0], None, st))) for _ in range(10))
        res["score_last_T128_L8_ms"] = round(t_sl, 4)
        res["logit_lens_T128_L8_ms"] = round(t_lens, 4)
        res["early_exit_T128_max16_stable2"] = {"ms": round(t_exit, 4), "loops_used": used[-1]}
        PF = 512
        tl.tl_prefill(m, 1, d_prompt, PF, LOOPS, None, None, st)
        t_pf = statistics.median(ev_ms(lambda: tl.tl_prefill(m, 1, d_prompt, PF, LOOPS, None, None, st))
                                 for _ in range(5))
        for _ in range(3):
            tl.tl_lane_fork(m, 1, 2, PF, st)
        t_fork = statistics.median(ev_ms(lambda: tl.tl_lane_fork(m, 1, 2, PF, st)) for _ in range(20))
        fork_bytes = 2 * (2 + LOOPS) * 2 * HKV * PF * HD * 2    # read + write
        res["prefix_512_L8"] = {"prefill_ms": round(t_pf, 4), "fork_ms": round(t_fork, 4),
                                "fork_gbs": round(fork_bytes / (t_fork * 1e6), 1),
                                "fork_frac_of_hbm": round(fork_bytes / (t_fork * 1e6) / peaks["hbm_gbs"], 4),
                                "speedup_vs_prefill": round(t_pf / t_fork, 1)}
    tl.tl_check_device_error(m)
    tl.tl_model_destroy(m)
    print(json.dumps({"workload": "400M looped LM: speculative decode, logit lens, early exit, prefix fork",
                      "results": res, "peaks": peaks,
                      "gpu_launches": tl.tl_kernel_launch_count() - launches0, "clocks": clocks.summary()}))
    return 0


def run_workload_kv8(args):
    """FP16 against INT8 KV cache on the 400M LM where the cache's bytes
    count: 16 lanes with per-lane loops drawn from {4,8,16}, 1536-token
    prompts, 256 greedy decode steps (context up to 1792 of 2048), and the
    prefill of a 512-token prompt at L = 8.  Per mode: decode tokens/s, the
    step's byte roofline (the cache's bytes per element: 2, or 1 + 4 / hd),
    prefill ms and the cache's size."""
    torch, dev, st = _dev_setup()
    import tl_synth
    import weight_shared_looped_int4_b200 as tl
    peaks = load_peaks()
    P, n_dec, n = 1536, args.decode_steps if args.decode_steps != STEPS_DECODE else 256, 16
    l2_gbs = None
    res = []
    launches0 = tl.tl_kernel_launch_count()
    with ClockSampler(0) as clocks:
        for mode, name in ((0, "fp16"), (1, "int8")):
            w, m = _lm_model(tl, tl_synth, 16, 2048, n, kv_mode=mode)
            if l2_gbs is None:
                l2_gbs, _, _ = probe_read_bandwidths(tl, torch, dev, st)
            prompts = tl_synth.make_lane_prompts(tl_synth.SEED_LSWEEP, w.shape.vocab, n, P + 1)
            d_prompts = torch.as_tensor(prompts, device=dev)
            hist = torch.zeros((n_dec + 1, n), dtype=torch.int32, device=dev)
            hp = hist.data_ptr()
            loops = [int(v) for v in tl_synth.make_lane_loops(tl_synth.SEED_LSWEEP, n)]
            lanes = list(range(n))

            def decode_run():
                for i, lane in enumerate(lanes):
                    tl.tl_prefill(m, lane, d_prompts[lane], P, loops[i], None, None, st)
                with torch.cuda.stream(st):
                    hist[0, :n].copy_(d_prompts[:n, P])
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(st)
                for i in range(n_dec):
                    tl.tl_decode_step(m, lanes, hp + 4 * n * i, loops, None, hp + 4 * n * (i + 1), st)
                b.record(st)
                b.synchronize()
                return a.elapsed_time(b)

            decode_run()     # warm (graph capture)
            ms = decode_run()
            per_elem = 2.0 if mode == 0 else 1.0 + 4.0 / HD
            kv = sum((2 + L) * 2 * HKV * HD * per_elem * (P + n_dec / 2) for L in loops)
            t_roof, _, _ = _decode_roofline_us(kv, loops, l2_gbs, peaks)
            us_step = 1e3 * ms / n_dec
            fn = lambda: tl.tl_prefill(m, 0, d_prompts[0, :512], 512, 8, None, None, st)
            for _ in range(3):
                fn()
            pf = _time_reps(torch, st, fn, 10)
            res.append({"kv": name, "kv_cache_bytes": tl.tl_model_info(m)["kv_bytes"],
                        "decode_tok_s": round(n * n_dec / (ms / 1e3), 1), "us_per_step": round(us_step, 2),
                        "kv_bytes_per_step": int(kv), "roofline_us_per_step": round(t_roof, 2),
                        "frac": round(t_roof / us_step, 4), "prefill_T512_L8_ms": round(pf, 4)})
            tl.tl_check_device_error(m)
            tl.tl_model_destroy(m)
    print(json.dumps({"workload": "400M looped LM, FP16 vs INT8 KV cache: 16 lanes, loops from {4,8,16}, "
                                  "1536-token prompts, 256 decode steps (ctx 2048)",
                      "metric": "decode tok/s, byte roofline fraction, prefill ms (T=512, L=8), cache bytes",
                      "loops": loops, "decode_steps": n_dec, "peaks": peaks, "l2_read_gbs": round(l2_gbs, 1),
                      "results": res, "gpu_launches": tl.tl_kernel_launch_count() - launches0,
                      "clocks": clocks.summary()}))
    return 0


def run_workload_int2(args):
    """INT4 against the INT2 body on the 400M LM at the headline shape: a
    128-token no-logits prefill and 128 greedy decode steps at L = 8, batch 1
    (graph replay).  Per width: decode tokens/s, its per-token byte roofline
    (the INT2 linears read K N / 4 code bytes + a scale and a 2-bit zero per
    group and row), prefill ms and the device bytes of the weights."""
    torch, dev, st = _dev_setup()
    import tl_synth
    import weight_shared_looped_int4_b200 as tl
    peaks = load_peaks()
    n_dec = args.decode_steps
    l2_gbs = None
    res = []
    launches0 = tl.tl_kernel_launch_count()

    def lin_bytes(K, N, bits):
        return K * N * bits // 8 + (K // 128) * N * (16 + bits) // 8

    with ClockSampler(0) as clocks:
        for bits in (4, 2):
            w, m = _lm_model(tl, tl_synth, LOOPS, PROMPT + n_dec + 1, 1, bits=bits)
            if l2_gbs is None:
                l2_gbs, _, _ = probe_read_bandwidths(tl, torch, dev, st)
            prompt = tl_synth.make_tokens(tl_synth.SEED_LM, w.shape.vocab, PROMPT + 1)
            d_prompt = torch.as_tensor(prompt, device=dev)
            hist = torch.zeros(n_dec + 1, dtype=torch.int32, device=dev)
            hp = hist.data_ptr()
            fn = lambda: tl.tl_prefill(m, 0, d_prompt, PROMPT, LOOPS, None, None, st)
            for _ in range(3):
                fn()
            pf = _time_reps(torch, st, fn, 10)

            def decode_run():
                tl.tl_prefill(m, 0, d_prompt, PROMPT, LOOPS, None, None, st)
                with torch.cuda.stream(st):
                    hist[0:1].copy_(d_prompt[PROMPT:PROMPT + 1])
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(st)
                for i in range(n_dec):
                    tl.tl_decode_step(m, [0], hp + 4 * i, [LOOPS], None, hp + 4 * (i + 1), st)
                b.record(st)
                b.synchronize()
                return a.elapsed_time(b)

            decode_run()     # warm (graph capture)
            ms = decode_run()
            layer = (lin_bytes(D, (HQ + 2 * HKV) * HD, bits) + lin_bytes(HQ * HD, D, bits) +
                     lin_bytes(D, 2 * F, bits) + lin_bytes(F, D, bits))
            kv = (2 + LOOPS) * 2 * HKV * HD * 2 * (PROMPT + n_dec / 2)
            hbm = 2 * layer + BYTES_PER_LAUNCH["head"] + kv
            l2 = LOOPS * layer
            t_roof = hbm / (peaks["hbm_gbs"] * 1e3) + l2 / (l2_gbs * 1e3)
            us_tok = 1e3 * ms / n_dec
            res.append({"weight_bits": bits, "weight_bytes": tl.tl_model_info(m)["weight_bytes"],
                        "block_linear_bytes": int(layer), "decode_tok_s": round(n_dec / (ms / 1e3), 1),
                        "decode_us_per_token": round(us_tok, 2), "roofline_us_per_token": round(t_roof, 2),
                        "frac": round(t_roof / us_tok, 4), "prefill_T128_ms": round(pf, 4)})
            tl.tl_check_device_error(m)
            tl.tl_model_destroy(m)
    print(json.dumps({"workload": "400M looped LM, INT4 vs INT2 body: 128-token prefill (no logits), "
                                  "%d greedy decode steps at L = 8, batch 1" % n_dec,
                      "metric": "decode tok/s and byte roofline fraction, prefill ms, weight bytes",
                      "peaks": peaks, "l2_read_gbs": round(l2_gbs, 1), "results": res,
                      "gpu_launches": tl.tl_kernel_launch_count() - launches0, "clocks": clocks.summary()}))
    return 0


WORKLOADS = {"tiny": run_workload_tiny, "linear": run_workload_linear, "kv8": run_workload_kv8,
             "int2": run_workload_int2,
             "attention": run_workload_attention, "lsweep": run_workload_lsweep,
             "peaks": run_workload_peaks, "next": run_workload_next}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-steps", type=int, default=STEPS_DECODE,
                    help="greedy decode steps per step (the workload uses 128)")
    ap.add_argument("--no-graphs", action="store_true",
                    help="layered decode path: launch kernels one by one instead of as CUDA graphs")
    ap.add_argument("--decode-path", choices=["auto", "fused", "layered"], default="auto",
                    help="single-kernel decode step (fused), one kernel per op (layered), or the "
                         "library's default (auto)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-profile", action="store_true")
    ap.add_argument("--trace", action="store_true",
                    help="print the phase timeline of one single-kernel decode step and exit")
    ap.add_argument("--workload", choices=["lm"] + sorted(WORKLOADS), default="lm",
                    help="lm (default): the 400M-LM L=8 step; others time the kernels on the "
                         "shapes of the other workloads and print their own JSON line")
    ap.add_argument("--ncu-prompt", type=int, default=PROMPT,
                    help="prompt length of --ncu-case (e.g. 2048 for the tcgen05 prefill attention)")
    ap.add_argument("--ncu-case", choices=["none", "decode", "prefill"], default="none",
                    help="run a small eager case for kernel profilers and exit")
    args = ap.parse_args()
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)
    if args.ncu_case != "none":
        return run_ncu_case(args)
    if args.trace:
        return run_trace(args)
    if args.workload != "lm":
        return WORKLOADS[args.workload](args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
