// One decode step of the looped model as ONE persistent kernel.
//
// What it computes is the cached single-token forward of the looped model
// (TinyLoop README, "Architecture" and "Status": n_pre distinct blocks, then
// the one shared loop block applied L times, each iteration with its own KV
// slice, then the output norm, the head and the greedy argmax): per effective
// layer, RMSNorm -> QKV INT4 linear -> RoPE -> KV write -> GQA attention over
// the lane's cache slice -> O linear + residual -> RMSNorm -> gate_up INT4
// linear -> SwiGLU -> down linear + residual.  The arithmetic of every step is
// that of the per-layer kernels (exact integer q - z operands on the tensor
// cores, fp16 (hi, lo) activation pairs, fp32 scales / accumulation / residual
// stream, fp16 KV cache); only the schedule differs.
//
// Why one kernel: at batch 1 a decode step is ~50 dependent launches of
// 1-12 MB each.  Every launch boundary costs a few microseconds of drain and
// ramp-up, far more than the bytes themselves (a 3 MB projection is 0.5 us at
// HBM speed).  Here one CTA per SM runs the whole step; the phases are
// separated by a grid-wide barrier (an arrival counter in global memory,
// ~1 us), and the weights, which never depend on activations, are streamed
// into a shared-memory ring by a producer warp that runs ahead of the compute
// warps across the barriers.
//
// Layout of a CTA (16 warps):
//   warps 0..14  compute: stage activations, MMA, epilogues, attention, head
//   warp 15      producer: walks the CTA's fixed sequence of weight items and
//                bulk-copies each into the next free ring slot (mbarrier
//                full/empty pairs, bounded waits).  Loop-block items carry an
//                L2 evict_last policy, pre-block and head items evict_first,
//                so the 24 MB loop block stays in L2 across iterations and
//                steps while 130 MB of head stream past it.
// Work split: output tiles of 16 rows are dealt round-robin to the CTAs
// (RoPE pairs and gate/up pairs stay together); attention units are (row, kv
// head, key split) with a ticketed merge; head tiles are contiguous ranges.
//
// Launch: cooperative (all CTAs co-resident, 1 per SM), so the grid barrier
// cannot deadlock; every wait is bounded in time and sets kErrTimeout.
#pragma once

#include <math.h>

#include "common.cuh"
#include "misc.cuh"

namespace tl {

// 15 compute warps + 1 producer: 16 warps = 4 per SM sub-partition, so each
// thread may hold up to 128 registers (17 warps would cap it at 96).
constexpr int kFusedWarps = 15;                         // compute warps
constexpr int kFusedCompute = kFusedWarps * 32;
constexpr int kFusedThreads = kFusedCompute + 32;       // + producer warp
constexpr int kFusedMaxRows = 4;                        // activation rows (lanes)
constexpr int kFusedMaxBlocks = 9;                      // up to 8 pre blocks + the loop block
constexpr int kFusedItemK = 2048;                       // K of one INT4 ring item
constexpr int kFusedSlotW = 16384;                      // weight bytes of a slot
constexpr int kFusedSlotBytes = kFusedSlotW + 1024;     // + scales / zeros
constexpr int kFusedMaxSlots = 13;
constexpr int kFusedMaxSplits = 32;                     // key splits per (row, kv head)
constexpr int kFusedMaxKeys = 256;                      // keys per attention unit
constexpr long long kFusedWaitNs = 500LL * 1000 * 1000; // grid-barrier time limit

enum FusedPhase { FP_QKV = 0, FP_O = 1, FP_GU = 2, FP_DOWN = 3 };

struct FusedLinear {
  const uint4* w;    // GEMV tile layout [n16 tiles][K/64][32] (16 B)
  const uint2* sz;   // [n16 tiles][K/128][8]
};
struct FusedBlock {
  FusedLinear lin[4];  // qkv, o, gate_up, down
  const __half* attn_norm;
  const __half* ffn_norm;
};

struct FusedArgs {
  FusedBlock blk[kFusedMaxBlocks];  // pre blocks 0..n_pre-1, then the loop block
  int n_pre;
  int d, qdim, F, V, hd, Hkv, rep;
  float eps, theta;
  const __half* embed;
  const __half* out_norm;
  const uint4* head_w;               // head in A-fragment tiles [V/16][d/16][32] (16 B)
  __half* kv;                        // [lanes][layers][K|V][Hkv][ctx][hd]
  long long plane, layer_stride, lane_stride;
  int ctx;
  const float2* rope_tab;            // (cos, sin) [ctx][hd/2]
  // rows of this step, in decreasing loop order
  int M;
  int lane[kFusedMaxRows], pos[kFusedMaxRows], loops[kFusedMaxRows];
  int tok_index[kFusedMaxRows], out_row[kFusedMaxRows];
  const int32_t* tokens;
  float* logits;                     // [.][V] or NULL
  int32_t* argmax;                   // [.] or NULL
  // workspaces
  float* x;                          // residual stream [rows][d]
  float* q;                          // rotated queries [rows][qdim]
  float* o;                          // attention output [rows][qdim]
  float* h;                          // SwiGLU output [rows][F]
  float* attn_part;                  // [rows][Hkv][kFusedMaxSplits][rep][hd + 4]
  unsigned* attn_ticket;             // [rows][Hkv], zero between launches
  float* head_val;                   // [grid][kFusedMaxRows]
  int* head_idx;
  unsigned* head_ticket;             // zero between launches
  unsigned* bar;                     // [0] arrivals, [1] exits, [2] give-up; zero between launches
  unsigned bar_extra;                // arrivals every grid barrier expects beyond the grid (0; 1 = wait test)
  int* err_flag;
  // shared-memory plan
  int n_slots;                       // ring slots
  int area_bytes;                    // activation planes / attention scratch
  int red_bytes;                     // cross-warp reduction buffer
  // optional phase timeline (globaltimer ns, thread 0 of every CTA), NULL =
  // off.  Slot s holds entries [s grid, (s + 1) grid): 0 kernel start; for
  // grid barrier k, 1 + 5k arrival, 2 + 5k release, and for the GEMV phase
  // before it 3 + 5k activations staged, 4 + 5k first weight item arrived,
  // 5 + 5k all items consumed; after B barriers, 1 + 5B head staged, 2 + 5B
  // head tiles done, 3 + 5B end.  Entries >= trace_cap are not written.
  unsigned long long* trace;
  long long trace_cap;
  // head-only mode (no layers: output norm + head + argmax of the rows of x),
  // used by the per-layer path; outputs may come from device memory so that a
  // captured graph does not depend on them
  int head_only;
  const HeadIO* io;          // if set, logits / argmax pointers are read here
  const int* out_row_dev;    // if set, output slots are read here
};

// ---- the fixed work sequence (shared by the producer and the consumers) ----
__host__ __device__ inline int fused_k(const FusedArgs& a, int ph) {
  return ph == FP_O ? a.qdim : ph == FP_DOWN ? a.F : a.d;
}
__host__ __device__ inline int fused_tpu(int ph) { return (ph == FP_QKV || ph == FP_GU) ? 2 : 1; }
__host__ __device__ inline int fused_units(const FusedArgs& a, int ph) {
  if (ph == FP_QKV) return (a.qdim + 2 * a.Hkv * a.hd) / 32;  // RoPE pairs of 16-row tiles
  if (ph == FP_GU) return a.F / 16;                            // (gate, up) tile pairs
  return a.d / 16;
}
// 16-row tile `ti` of unit u.  QKV: tiles j and j + hd/32 of a head hold the
// rotation pairs (e, e + hd/2).  gate_up: gate tile u, up tile u + F/16.
__host__ __device__ inline int fused_tile(const FusedArgs& a, int ph, int u, int ti) {
  if (ph == FP_QKV) {
    const int hp = a.hd / 32, head = u / hp, j = u % hp;
    return head * 2 * hp + j + (ti ? hp : 0);
  }
  if (ph == FP_GU) return u + (ti ? a.F / 16 : 0);
  return u;
}
__host__ __device__ inline int fused_layers(const FusedArgs& a) { return a.head_only ? 0 : a.n_pre + a.loops[0]; }
__device__ __forceinline__ int fused_active(const FusedArgs& a, int layer) {
  int n = 0;
  while (n < a.M && a.n_pre + a.loops[n] > layer) ++n;
  return n;
}
// k columns of a head item: at most 512 and a divisor of d (d is a multiple
// of 128), so that items never run past a tile's row.
__host__ __device__ inline int fused_head_item_k(int d) {
  int k = d < 512 ? d : 512;
  while (d % k) k -= 128;
  return k;
}

// ---- attention key splits -------------------------------------------------
constexpr int kFusedChunk = 64;
constexpr int kFusedSmallKeys = 4 * kFusedChunk;   // up to here the O-phase staging merges the splits

// Key splits of a row with n keys.  Up to kFusedSmallKeys keys: one chunk per
// split (<= 4 splits), merged by the consumer.  Beyond: enough splits to fill
// the grid, at least 32 and at most kFusedMaxKeys keys each (n <= 8192 keeps
// this <= kFusedMaxSplits), merged by the last split.  The split depends only
// on the row's own key count (and the grid), so a lane's result is bitwise
// the same whichever lanes share the step.
__device__ __forceinline__ void fused_split(int n, int P, int Hkv, int& C, int& ns) {
  if (n <= kFusedSmallKeys) {
    ns = (n + kFusedChunk - 1) / kFusedChunk;
    C = (n + ns - 1) / ns;
    return;
  }
  int s = min(max(1, P / Hkv), (n + 31) / 32);
  s = max(s, (n + kFusedMaxKeys - 1) / kFusedMaxKeys);
  s = max(1, min(s, kFusedMaxSplits));
  C = (n + s - 1) / s;
  ns = (n + C - 1) / C;
}

// ---- primitives -------------------------------------------------------------
__device__ __forceinline__ void fused_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kFusedCompute) : "memory"); }
__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// Grid-wide barrier of the compute warps: a monotonic arrival counter (target
// = barriers so far x CTAs).  Bounded in time; a CTA that gives up raises the
// give-up word so the others stop waiting too.
__device__ __forceinline__ void fused_trace(const FusedArgs& a, long long slot) {
  if (a.trace) {
    const long long i = slot * gridDim.x + blockIdx.x;
    if (i < a.trace_cap) a.trace[i] = (unsigned long long)globaltimer_ns();
  }
}
__device__ __forceinline__ void fused_grid_sync(const FusedArgs& a, unsigned& target) {
  fused_sync();
  if (threadIdx.x == 0) {
    const long long k = target / gridDim.x;   // index of this barrier
    target += gridDim.x;
    fused_trace(a, 1 + 5 * k);
    // arrival with release semantics: this CTA's writes (ordered before by
    // the CTA barrier) are visible to whoever observes the new count
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(a.bar) : "memory");
    if (!*reinterpret_cast<volatile unsigned*>(a.bar + 2)) {
      const long long t0 = globaltimer_ns();
      unsigned spins = 0;
      while (ld_acquire_gpu(a.bar) < target) {
        if ((++spins & 63u) == 0) {
          if (*reinterpret_cast<volatile unsigned*>(a.bar + 2)) break;
          if (globaltimer_ns() - t0 > kFusedWaitNs) {
            atomicExch(a.bar + 2, 1u);
            atomicOr(a.err_flag, kErrTimeout);
            break;
          }
        }
      }
    }
    __threadfence();
    fused_trace(a, 2 + 5 * k);
  }
  fused_sync();
}

// ---- producer -----------------------------------------------------------------
__device__ void fused_producer(const FusedArgs& a, unsigned char* ring, uint64_t* full, uint64_t* empty,
                               int* s_fail) {
  const uint64_t keep = l2_evict_last(), stream = l2_evict_first();
  const int P = gridDim.x, c = blockIdx.x, NS = a.n_slots;
  int item = 0;
  bool ok = true;
  auto issue = [&](const unsigned char* wsrc, unsigned wbytes, const unsigned char* zsrc, unsigned zbytes,
                   uint64_t pol) {
    if (!ok) return;
    const int s = item % NS;
    if (item >= NS && !mbar_wait_or_fail(&empty[s], (unsigned)((item / NS) - 1) & 1u, s_fail)) {
      ok = false;
      return;
    }
    unsigned char* dst = ring + (size_t)s * kFusedSlotBytes;
    mbar_arrive_expect_tx(&full[s], wbytes + zbytes);
    bulk_g2s_hint(dst, wsrc, wbytes, &full[s], pol);
    if (zbytes) bulk_g2s_hint(dst + kFusedSlotW, zsrc, zbytes, &full[s], pol);
    ++item;
  };
  const int L = fused_layers(a);
  for (int layer = 0; layer < L; ++layer) {
    const FusedBlock& b = a.blk[layer < a.n_pre ? layer : a.n_pre];
    const uint64_t pol = layer < a.n_pre ? stream : keep;
    for (int ph = 0; ph < 4; ++ph) {
      const int K = fused_k(a, ph), nu = fused_units(a, ph), tpu = fused_tpu(ph);
      const size_t wt = (size_t)(K >> 6) * 512, zt = (size_t)(K >> 7) * 64;
      for (int u = c; u < nu; u += P)
        for (int ti = 0; ti < tpu; ++ti) {
          const int tile = fused_tile(a, ph, u, ti);
          const unsigned char* wb = reinterpret_cast<const unsigned char*>(b.lin[ph].w) + (size_t)tile * wt;
          const unsigned char* zb = reinterpret_cast<const unsigned char*>(b.lin[ph].sz) + (size_t)tile * zt;
          for (int kb = 0; kb < K; kb += kFusedItemK) {
            const int kn = min(kFusedItemK, K - kb);
            issue(wb + (size_t)(kb >> 6) * 512, (unsigned)(kn >> 6) * 512, zb + (size_t)(kb >> 7) * 64,
                  (unsigned)(kn >> 7) * 64, pol);
          }
        }
    }
  }
  {  // head
    const int nt = a.V >> 4, tb = (int)((long)c * nt / P), te = (int)((long)(c + 1) * nt / P);
    const int ki = fused_head_item_k(a.d);
    const size_t tile_bytes = (size_t)(a.d >> 4) * 512;
    const unsigned char* hw = reinterpret_cast<const unsigned char*>(a.head_w);
    for (int tile = tb; tile < te; ++tile)
      for (int kk = 0; kk < a.d; kk += ki)
        issue(hw + (size_t)tile * tile_bytes + (size_t)(kk >> 4) * 512, (unsigned)(ki >> 4) * 512, nullptr, 0,
              stream);
  }
  // On a give-up, wait (bounded) for the copies still in flight before the
  // CTA may exit.
  if (*reinterpret_cast<volatile int*>(s_fail)) {
    for (int i = item - NS < 0 ? 0 : item - NS; i < item; ++i) mbar_wait(&full[i % NS], (unsigned)(i / NS) & 1u);
  }
}

// ---- consumers ------------------------------------------------------------------
enum FusedStage { FS_NORM = 0, FS_EMBED = 1, FS_RAW = 2 };

// Activation rows m < Mrows into the (hi, lo) fp16 planes xs / xl [M][K + 8].
// FS_NORM / FS_EMBED apply the RMSNorm with `gain` (the row is x, or the
// embedding of the row's token); FS_RAW copies fp32 values.  Every thread
// loads all its float4 columns of every row at once (one round trip to L2),
// keeps them in registers for the norm, and writes the pair.  Values written
// by other CTAs in this launch are read through L2 (ld.global.cg).
constexpr int kFusedStageV4 = 3;   // float4 columns per thread and row: K <= 3 * 4 * 480
__device__ void fused_stage(const FusedArgs& a, int mode, const float* src, int lds, const __half* gain, int K,
                            int Mrows, __half* xs, __half* xl, float* ssq) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ldx = K + 8;
  float4 v[kFusedMaxRows][kFusedStageV4];
  uint2 gv[kFusedStageV4];   // the gains of this thread's columns, loaded with x
#pragma unroll
  for (int i = 0; i < kFusedStageV4; ++i) {
    const int k = tid * 4 + i * 4 * kFusedCompute;
    gv[i] = (mode != FS_RAW && k < K) ? *reinterpret_cast<const uint2*>(gain + k) : make_uint2(0u, 0u);
  }
  // fully unrolled with guards (no early exits) so v stays in registers
#pragma unroll
  for (int m = 0; m < kFusedMaxRows; ++m) {
    const __half* erow = a.embed;
    if (mode == FS_EMBED && m < Mrows) {
      int tok = a.tokens[a.tok_index[m]];
      if (tok < 0 || tok >= a.V) {
        if (blockIdx.x == 0 && tid == 0) atomicOr(a.err_flag, kErrToken);
        tok = 0;
      }
      erow = a.embed + (size_t)tok * a.d;
    }
#pragma unroll
    for (int i = 0; i < kFusedStageV4; ++i) {
      const int k = tid * 4 + i * 4 * kFusedCompute;
      v[m][i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (m < Mrows && k < K) {
        if (mode == FS_EMBED) {
          const uint2 u = *reinterpret_cast<const uint2*>(erow + k);
          const float2 f01 = h2_to_f2(u.x), f23 = h2_to_f2(u.y);
          v[m][i] = make_float4(f01.x, f01.y, f23.x, f23.y);
        } else {
          v[m][i] = __ldcg(reinterpret_cast<const float4*>(src + (size_t)m * lds + k));
        }
      }
    }
  }
  float rs[kFusedMaxRows] = {1.f, 1.f, 1.f, 1.f};
  if (mode != FS_RAW) {
#pragma unroll
    for (int m = 0; m < kFusedMaxRows; ++m) {
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < kFusedStageV4; ++i)
        ss += v[m][i].x * v[m][i].x + v[m][i].y * v[m][i].y + v[m][i].z * v[m][i].z + v[m][i].w * v[m][i].w;
      ss = warp_sum(ss);
      if (lane == 0 && m < Mrows) ssq[m * kFusedWarps + warp] = ss;
    }
    fused_sync();
#pragma unroll
    for (int m = 0; m < kFusedMaxRows; ++m) {
      if (m < Mrows) {
        float ss = 0.f;
#pragma unroll
        for (int w = 0; w < kFusedWarps; ++w) ss += ssq[m * kFusedWarps + w];
        rs[m] = 1.0f / sqrtf(ss / (float)K + a.eps);
      }
    }
  }
#pragma unroll
  for (int m = 0; m < kFusedMaxRows; ++m) {
#pragma unroll
    for (int i = 0; i < kFusedStageV4; ++i) {
      const int k = tid * 4 + i * 4 * kFusedCompute;
      if (m < Mrows && k < K) {
        float4 x4 = v[m][i];
        if (mode != FS_RAW) {
          const float2 g01 = h2_to_f2(gv[i].x), g23 = h2_to_f2(gv[i].y);
          x4.x = (x4.x * rs[m]) * g01.x; x4.y = (x4.y * rs[m]) * g01.y;
          x4.z = (x4.z * rs[m]) * g23.x; x4.w = (x4.w * rs[m]) * g23.y;
        }
        const __half2 h01 = __floats2half2_rn(x4.x, x4.y), h23 = __floats2half2_rn(x4.z, x4.w);
        const float2 r01 = __half22float2(h01), r23 = __half22float2(h23);
        const __half2 l01 = __floats2half2_rn(x4.x - r01.x, x4.y - r01.y);
        const __half2 l23 = __floats2half2_rn(x4.z - r23.x, x4.w - r23.y);
        uint2 ph, pl;
        ph.x = *reinterpret_cast<const uint32_t*>(&h01); ph.y = *reinterpret_cast<const uint32_t*>(&h23);
        pl.x = *reinterpret_cast<const uint32_t*>(&l01); pl.y = *reinterpret_cast<const uint32_t*>(&l23);
        *reinterpret_cast<uint2*>(xs + m * ldx + k) = ph;
        *reinterpret_cast<uint2*>(xl + m * ldx + k) = pl;
      }
    }
  }
  fused_sync();
}

// O-phase staging: the attention output of rows m < Mrows as (hi, lo) planes.
// Rows whose keys were split into <= 4 one-chunk splits are merged here from
// the partials (running max, sum of weights, unnormalised sums), in split
// order with the same formula as the in-attention merge; other rows are read
// from o.  All loads of a row are in flight at once.
__device__ void fused_stage_attn(const FusedArgs& a, int Mrows, __half* xs, __half* xl) {
  const int tid = threadIdx.x, K = a.qdim, ldx = K + 8, hd = a.hd, rep = a.rep;
  const int pstride = hd + 4;
  for (int m = 0; m < Mrows; ++m) {
    int C, ns;
    fused_split(a.pos[m] + 1, gridDim.x, a.Hkv, C, ns);
    const bool merge = ns > 1 && a.pos[m] + 1 <= kFusedSmallKeys;
    // two float4 columns per thread per round (qdim <= 3840 takes one round)
    for (int ib = 0; ib < kFusedStageV4; ib += 2) {
      float4 v[2];
      float4 part[2][4];
      float2 ml[2][4];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int k = tid * 4 + (ib + i) * 4 * kFusedCompute;
        v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (ib + i < kFusedStageV4 && k < K) {
          if (!merge) {
            v[i] = __ldcg(reinterpret_cast<const float4*>(a.o + (size_t)m * K + k));
          } else {
            const int h = k / hd, dim = k % hd, g = h / rep, hh = h % rep;
            const float* base = a.attn_part + (((size_t)m * a.Hkv + g) * kFusedMaxSplits) * rep * pstride;
#pragma unroll
            for (int sp = 0; sp < 4; ++sp) {
              if (sp < ns) {
                const float* pp = base + ((size_t)sp * rep + hh) * pstride;
                part[i][sp] = __ldcg(reinterpret_cast<const float4*>(pp + dim));
                ml[i][sp] = __ldcg(reinterpret_cast<const float2*>(pp + hd));
              }
            }
          }
        }
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int k = tid * 4 + (ib + i) * 4 * kFusedCompute;
        if (ib + i >= kFusedStageV4 || k >= K) continue;
        float4 x4 = v[i];
        if (merge) {
          float mx = -INFINITY;
#pragma unroll
          for (int sp = 0; sp < 4; ++sp)
            if (sp < ns) mx = fmaxf(mx, ml[i][sp].x);
          float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
          float den = 0.f;
#pragma unroll
          for (int sp = 0; sp < 4; ++sp) {
            if (sp < ns) {
              const float w = expf(ml[i][sp].x - mx);
              num.x = fmaf(w, part[i][sp].x, num.x);
              num.y = fmaf(w, part[i][sp].y, num.y);
              num.z = fmaf(w, part[i][sp].z, num.z);
              num.w = fmaf(w, part[i][sp].w, num.w);
              den = fmaf(w, ml[i][sp].y, den);
            }
          }
          x4 = make_float4(num.x / den, num.y / den, num.z / den, num.w / den);
        }
        const __half2 h01 = __floats2half2_rn(x4.x, x4.y), h23 = __floats2half2_rn(x4.z, x4.w);
        const float2 r01 = __half22float2(h01), r23 = __half22float2(h23);
        const __half2 l01 = __floats2half2_rn(x4.x - r01.x, x4.y - r01.y);
        const __half2 l23 = __floats2half2_rn(x4.z - r23.x, x4.w - r23.y);
        uint2 ph, pl;
        ph.x = *reinterpret_cast<const uint32_t*>(&h01); ph.y = *reinterpret_cast<const uint32_t*>(&h23);
        pl.x = *reinterpret_cast<const uint32_t*>(&l01); pl.y = *reinterpret_cast<const uint32_t*>(&l23);
        *reinterpret_cast<uint2*>(xs + m * ldx + k) = ph;
        *reinterpret_cast<uint2*>(xl + m * ldx + k) = pl;
      }
    }
  }
  fused_sync();
}

// One GEMV phase of this CTA: its units' tiles, K in ring items.  MMA columns
// are (row m, plane) = 2m + plane for m < 4, so one m16n8k16 per k16 covers
// both halves of every row.  Per-warp partial sums over the warp's K slice go
// to red[tile][warp][16][4]; the epilogue sums the 16 warps in order.
// The O and down phases deal the same tiles to the same CTAs, so a CTA owns
// its rows of the residual stream: it keeps them in shared memory (xown
// [tile][16 rows][4]) and only writes them out for the other CTAs.
__device__ void fused_gemv(const FusedArgs& a, int ph, int layer, int Ma, unsigned char* ring, uint64_t* full,
                           uint64_t* empty, int* s_fail, const __half* xs, const __half* xl, float* red,
                           float* xown, const float2* rope_s, int& item, long long trace_slot) {
  const int P = gridDim.x, c = blockIdx.x, NS = a.n_slots;
  const int K = fused_k(a, ph), nu = fused_units(a, ph), tpu = fused_tpu(ph);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int ldx = K + 8;
  const int brow = g >> 1;
  const __half* bsrc = ((g & 1) ? xl : xs) + (size_t)brow * ldx + 2 * t;
  const bool bok = brow < Ma;
  int lt = 0;
  for (int u = c; u < nu; u += P) {
    for (int ti = 0; ti < tpu; ++ti) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int kb = 0; kb < K; kb += kFusedItemK) {
        const int nck = min(kFusedItemK, K - kb) >> 6;
        const int s = item % NS;
        mbar_wait_or_fail(&full[s], (unsigned)(item / NS) & 1u, s_fail);
        if (tid == 0 && lt == 0 && kb == 0) fused_trace(a, trace_slot);   // the phase's first item arrived
        const unsigned char* wsl = ring + (size_t)s * kFusedSlotBytes;
        const unsigned char* zsl = wsl + kFusedSlotW;
        const int c0 = warp * nck / kFusedWarps, c1 = (warp + 1) * nck / kFusedWarps;
        // Two chunks per iteration, each with two accumulators (even / odd
        // k16 steps): four independent MMA chains keep the tensor pipe busy
        // instead of waiting on one chain's latency.
        auto chunk = [&](int ci, float (&t0)[4], float (&t1)[4], uint32_t& sx) {
          const uint4 wv = *reinterpret_cast<const uint4*>(wsl + (size_t)ci * 512 + lane * 16);
          const uint2 sv = *reinterpret_cast<const uint2*>(zsl + (size_t)(ci >> 1) * 64 + g * 8);
          const int kc = kb + ci * 64;
          const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t af[4];
            unpack_a_frag(words[j], sv.y, af);
            uint32_t b0 = 0, b1 = 0;
            if (bok) {
              b0 = *reinterpret_cast<const uint32_t*>(bsrc + kc + j * 16);
              b1 = *reinterpret_cast<const uint32_t*>(bsrc + kc + j * 16 + 8);
            }
            if (j & 1) mma_f16_16816(t1, af, b0, b1);
            else mma_f16_16816(t0, af, b0, b1);
          }
          sx = sv.x;
        };
        auto fold = [&](const float (&t0)[4], const float (&t1)[4], uint32_t sx) {
          const float2 sc = h2_to_f2(sx);
          acc[0] = fmaf(sc.x, t0[0] + t1[0], acc[0]);
          acc[1] = fmaf(sc.x, t0[1] + t1[1], acc[1]);
          acc[2] = fmaf(sc.y, t0[2] + t1[2], acc[2]);
          acc[3] = fmaf(sc.y, t0[3] + t1[3], acc[3]);
        };
        int ci = c0;
        for (; ci + 1 < c1; ci += 2) {
          float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
          float b0[4] = {0.f, 0.f, 0.f, 0.f}, b1[4] = {0.f, 0.f, 0.f, 0.f};
          uint32_t sa, sb;
          chunk(ci, a0, a1, sa);
          chunk(ci + 1, b0, b1, sb);
          fold(a0, a1, sa);
          fold(b0, b1, sb);
        }
        if (ci < c1) {
          float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
          uint32_t sa;
          chunk(ci, a0, a1, sa);
          fold(a0, a1, sa);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        ++item;
      }
      float* r = red + ((size_t)lt * kFusedWarps + warp) * 64;
      r[g * 4 + t] = acc[0] + acc[1];        // tile row g,     activation row t (hi + lo)
      r[(g + 8) * 4 + t] = acc[2] + acc[3];  // tile row g + 8
      ++lt;
    }
  }
  if (tid == 0) fused_trace(a, trace_slot + 1);
  fused_sync();
  if (lt == 0) return;
  const int n_local = lt / tpu;
  const int hd = a.hd;
  for (int e = tid; e < n_local * 16 * Ma; e += kFusedCompute) {
    const int ul = e / (16 * Ma), rem = e % (16 * Ma), r = rem & 15, m = rem >> 4;
    float va = 0.f, vb = 0.f;
#pragma unroll
    for (int w = 0; w < kFusedWarps; ++w) va += red[((size_t)(ul * tpu) * kFusedWarps + w) * 64 + r * 4 + m];
    if (tpu == 2) {
#pragma unroll
      for (int w = 0; w < kFusedWarps; ++w) vb += red[((size_t)(ul * tpu + 1) * kFusedWarps + w) * 64 + r * 4 + m];
    }
    const int u = c + ul * P;
    const int row0 = fused_tile(a, ph, u, 0) * 16 + r;
    if (ph == FP_QKV) {
      const int j = row0 % hd, pos = a.pos[m];
      const int kvdim = a.Hkv * hd;
      if (row0 < a.qdim) {
        const float2 cs = rope_s[m * (hd / 2) + j];
        float* qo = a.q + (size_t)m * a.qdim;
        qo[row0] = va * cs.x - vb * cs.y;
        qo[row0 + hd / 2] = vb * cs.x + va * cs.y;
      } else {
        const bool is_k = row0 < a.qdim + kvdim;
        const int kvh = (row0 - a.qdim - (is_k ? 0 : kvdim)) / hd;
        __half* dst = a.kv + a.lane[m] * a.lane_stride + layer * a.layer_stride + (is_k ? 0 : a.plane) +
                      ((size_t)kvh * a.ctx + pos) * hd;
        if (is_k) {
          const float2 cs = rope_s[m * (hd / 2) + j];
          dst[j] = __float2half_rn(va * cs.x - vb * cs.y);
          dst[j + hd / 2] = __float2half_rn(vb * cs.x + va * cs.y);
        } else {
          dst[j] = __float2half_rn(va);
          dst[j + hd / 2] = __float2half_rn(vb);
        }
      }
    } else if (ph == FP_GU) {
      a.h[(size_t)m * a.F + row0] = silu(va) * vb;
    } else {
      float* xw = xown + ((size_t)ul * 16 + r) * kFusedMaxRows + m;
      const float xv = *xw + va;
      *xw = xv;
      a.x[(size_t)m * a.d + row0] = xv;
    }
  }
}

// Single-query attention of the active rows over their lanes' slice `layer`:
// units (row, kv head, split of <= kFusedMaxKeys keys), dealt round-robin.
// A unit walks its keys in chunks of kFusedChunk: the chunk's K and V rows
// (and, with the first chunk, the group's queries) are loaded with all loads
// in flight at once into shared memory; scores are fp32 dot products (warps
// over keys, lanes over dims), the softmax is online across chunks (running
// max and sum per head), and P V runs one thread per (head, dim).  Splits
// write (unnormalised sum, max, sum of weights); the last unit of the (row,
// kv head) to finish merges them in split order.
template <int HD>
__host__ __device__ constexpr int fused_attn_bytes(int rep) {
  return 2 * kFusedChunk * HD * 2 + (rep * HD + rep * kFusedChunk + 4 * rep) * 4;
}
template <int HD>
__device__ void fused_attention(const FusedArgs& a, int layer, int Ma, unsigned char* area, int* s_last,
                                long long trace_slot) {
  constexpr int DPL = HD / 32;
  constexpr int ROW16 = HD / 8;                      // 16-byte pieces of a key row
  constexpr int NACC = (8 * HD + kFusedCompute - 1) / kFusedCompute;   // (head, dim) per thread, rep <= 8
  const int P = gridDim.x, c = blockIdx.x, rep = a.rep, Hkv = a.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  __half* ks = reinterpret_cast<__half*>(area);                 // [kFusedChunk][HD]
  __half* vs = ks + kFusedChunk * HD;                           // [kFusedChunk][HD]
  float* qs = reinterpret_cast<float*>(vs + kFusedChunk * HD);  // [rep][HD]
  float* sc = qs + rep * HD;                                    // [rep][kFusedChunk]
  float* ml = sc + rep * kFusedChunk;                           // [rep][4]: max, sum, rescale
  int ns[kFusedMaxRows], C[kFusedMaxRows];
  int total = 0;
  for (int m = 0; m < Ma; ++m) {
    fused_split(a.pos[m] + 1, P, Hkv, C[m], ns[m]);
    total += Hkv * ns[m];
  }
  const float scale = 1.0f / sqrtf((float)HD);
  for (int u = c; u < total; u += P) {
    int m = 0, r = u;
    while (r >= Hkv * ns[m]) { r -= Hkv * ns[m]; ++m; }
    const int g = r / ns[m], s = r % ns[m];
    const int n = a.pos[m] + 1, j0 = s * C[m], j1 = min(n, j0 + C[m]);
    const float* qsrc = a.q + (size_t)m * a.qdim + (size_t)g * rep * HD;
    const __half* kb = a.kv + a.lane[m] * a.lane_stride + layer * a.layer_stride + (size_t)g * a.ctx * HD;
    const __half* vb = kb + a.plane;
    float acc[NACC];                // P V sums of (head, dim) = tid + i kFusedCompute
#pragma unroll
    for (int i = 0; i < NACC; ++i) acc[i] = 0.f;
    for (int jc = j0; jc < j1; jc += kFusedChunk) {
      const int nk = min(kFusedChunk, j1 - jc);
      // ---- chunk (and queries) into shared memory, all loads in flight ----
      {
        constexpr int PER = (2 * kFusedChunk * ROW16 + kFusedCompute - 1) / kFusedCompute;
        uint4 tmp[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          const int e = tid + i * kFusedCompute;           // 16-byte piece: [K|V][key][piece]
          const int kv = e / (kFusedChunk * ROW16), rem = e % (kFusedChunk * ROW16);
          const int key = rem / ROW16, pc = rem % ROW16;
          tmp[i] = make_uint4(0, 0, 0, 0);
          if (kv < 2 && key < nk)
            tmp[i] = __ldcg(reinterpret_cast<const uint4*>((kv ? vb : kb) + (size_t)(jc + key) * HD) + pc);
        }
        float qv[NACC];
#pragma unroll
        for (int i = 0; i < NACC; ++i)
          qv[i] = (jc == j0 && tid + i * kFusedCompute < rep * HD) ? __ldcg(qsrc + tid + i * kFusedCompute) : 0.f;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          const int e = tid + i * kFusedCompute;
          if (e < 2 * kFusedChunk * ROW16) reinterpret_cast<uint4*>(ks)[e] = tmp[i];
        }
        if (jc == j0) {
#pragma unroll
          for (int i = 0; i < NACC; ++i)
            if (tid + i * kFusedCompute < rep * HD) qs[tid + i * kFusedCompute] = qv[i];
          if (tid < rep) { ml[4 * tid] = -INFINITY; ml[4 * tid + 1] = 0.f; }
        }
      }
      fused_sync();
      if (tid == 0 && u == c && jc == j0) fused_trace(a, trace_slot);       // first chunk loaded
      // ---- scores ----
      for (int jj = warp; jj < nk; jj += kFusedWarps) {
        const __half* kp = ks + jj * HD + lane * DPL;
        float kf[DPL];
        if constexpr (DPL == 4) {
          const uint2 u2 = *reinterpret_cast<const uint2*>(kp);
          const float2 f01 = h2_to_f2(u2.x), f23 = h2_to_f2(u2.y);
          kf[0] = f01.x; kf[1] = f01.y; kf[2] = f23.x; kf[3] = f23.y;
        } else {
          const float2 f01 = h2_to_f2(*reinterpret_cast<const unsigned*>(kp));
          kf[0] = f01.x; kf[1] = f01.y;
        }
        for (int h = 0; h < rep; ++h) {
          float dot = 0.f;
#pragma unroll
          for (int i = 0; i < DPL; ++i) dot = fmaf(qs[h * HD + lane * DPL + i], kf[i], dot);
          dot = warp_sum(dot);
          if (lane == 0) sc[h * kFusedChunk + jj] = dot * scale;
        }
      }
      fused_sync();
      if (tid == 0 && u == c && jc == j0) fused_trace(a, trace_slot + 1);   // its scores done
      // ---- online softmax, one warp per head ----
      if (warp < rep) {
        float* sh = sc + warp * kFusedChunk;
        float mx = -INFINITY;
        for (int jj = lane; jj < nk; jj += 32) mx = fmaxf(mx, sh[jj]);
        mx = warp_max(mx);
        const float m_old = ml[4 * warp], m_new = fmaxf(m_old, mx);
        float sum = 0.f;
        for (int jj = lane; jj < nk; jj += 32) {
          const float p = expf(sh[jj] - m_new);
          sh[jj] = p;
          sum += p;
        }
        sum = warp_sum(sum);
        if (lane == 0) {
          const float alpha = expf(m_old - m_new);   // 0 on the first chunk
          ml[4 * warp] = m_new;
          ml[4 * warp + 1] = ml[4 * warp + 1] * alpha + sum;
          ml[4 * warp + 2] = alpha;
        }
      }
      fused_sync();
      // ---- P V ----
#pragma unroll
      for (int i = 0; i < NACC; ++i) {
        const int oi = tid + i * kFusedCompute;
        if (oi < rep * HD) {
          const int h = oi / HD, dim = oi % HD;
          const float* ph = sc + h * kFusedChunk;
          float v = acc[i] * ml[4 * h + 2];
#pragma unroll 8
          for (int jj = 0; jj < nk; ++jj) v = fmaf(ph[jj], __half2float(vs[jj * HD + dim]), v);
          acc[i] = v;
        }
      }
      fused_sync();   // the chunk buffers are reused
      if (tid == 0 && u == c && jc == j0) fused_trace(a, trace_slot + 2);   // its P V done
    }
    const bool single = ns[m] == 1;
    float* pbase = a.attn_part + (((size_t)m * Hkv + g) * kFusedMaxSplits) * rep * (HD + 4);
#pragma unroll
    for (int i = 0; i < NACC; ++i) {
      const int oi = tid + i * kFusedCompute;
      if (oi < rep * HD) {
        const int h = oi / HD, dim = oi % HD;
        if (single) {
          a.o[(size_t)m * a.qdim + (size_t)(g * rep + h) * HD + dim] = acc[i] / ml[4 * h + 1];
        } else {
          float* pp = pbase + ((size_t)s * rep + h) * (HD + 4);
          pp[dim] = acc[i];
          if (dim == 0) { pp[HD] = ml[4 * h]; pp[HD + 1] = ml[4 * h + 1]; }
        }
      }
    }
    if (!single && n > kFusedSmallKeys) {   // short rows are merged by the O-phase staging
      __threadfence();
      fused_sync();
      if (tid == 0) {
        unsigned* tk = a.attn_ticket + m * Hkv + g;
        *s_last = atomicAdd(tk, 1u) == (unsigned)(ns[m] - 1);
        if (*s_last) *tk = 0u;
      }
      fused_sync();
      if (*s_last) {
        __threadfence();
        const int nsm = ns[m];
        // (max, sum) of every (split, head), all loaded in one round, into the
        // score buffer (rep * kFusedChunk >= 2 * rep * kFusedMaxSplits floats)
        float* mls = sc;
        for (int e = tid; e < nsm * rep * 2; e += kFusedCompute) {
          const int sp = e / (rep * 2), rem = e % (rep * 2);
          mls[e] = __ldcg(pbase + ((size_t)sp * rep + (rem >> 1)) * (HD + 4) + HD + (rem & 1));
        }
        fused_sync();
#pragma unroll
        for (int i = 0; i < NACC; ++i) {
          const int oi = tid + i * kFusedCompute;
          if (oi < rep * HD) {
            const int h = oi / HD, dim = oi % HD;
            float mx = -INFINITY;
            for (int sp = 0; sp < nsm; ++sp) mx = fmaxf(mx, mls[(sp * rep + h) * 2]);
            float num = 0.f, den = 0.f;
#pragma unroll 8
            for (int sp = 0; sp < nsm; ++sp) {
              const float w = expf(mls[(sp * rep + h) * 2] - mx);
              num = fmaf(w, __ldcg(pbase + ((size_t)sp * rep + h) * (HD + 4) + dim), num);
              den = fmaf(w, mls[(sp * rep + h) * 2 + 1], den);
            }
            a.o[(size_t)m * a.qdim + (size_t)(g * rep + h) * HD + dim] = num / den;
          }
        }
      }
    }
    fused_sync();
  }
}

__device__ __forceinline__ bool fused_better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

template <int HD>
__global__ void __launch_bounds__(kFusedThreads, 1) decode_fused_kernel(const __grid_constant__ FusedArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t full[kFusedMaxSlots], empty[kFusedMaxSlots];
  __shared__ float ssq[kFusedMaxRows * kFusedWarps];
  __shared__ float s_bv[kFusedMaxRows][16];
  __shared__ int s_bi[kFusedMaxRows][16];
  __shared__ float2 rope_s[kFusedMaxRows * 64];   // (cos, sin) of each row's position, hd <= 128
  __shared__ float s_wv[kFusedMaxRows][kFusedWarps];
  __shared__ int s_wi[kFusedMaxRows][kFusedWarps];
  __shared__ int s_fail, s_last;
  const int NS = a.n_slots;
  unsigned char* ring = smem;
  unsigned char* area = smem + (size_t)NS * kFusedSlotBytes;
  float* red = reinterpret_cast<float*>(area + a.area_bytes);
  float* xown = reinterpret_cast<float*>(area + a.area_bytes + a.red_bytes);   // [owned tiles][16][4]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) fused_trace(a, 0);

  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kFusedWarps);
    }
    fence_mbar_init();
    s_fail = 0;
  }
  __syncthreads();

  if (warp == kFusedWarps) {
    if (lane == 0) fused_producer(a, ring, full, empty, &s_fail);
  } else {
    const int P = gridDim.x, c = blockIdx.x;
    int item = 0;
    unsigned target = a.bar_extra;   // > 0 only under the wait test: no barrier can complete
    __half* xs = reinterpret_cast<__half*>(area);
    pdl_wait();   // head-only launches follow the kernel that wrote x
    for (int e = tid; e < (a.head_only ? 0 : a.M * (a.hd / 2)); e += kFusedCompute) {
      const int m = e / (a.hd / 2), j = e % (a.hd / 2);
      rope_s[e] = rope_cs(a.rope_tab, a.pos[m], j, a.hd, a.theta);
    }
    if (!a.head_only) {  // the residual stream of this CTA's rows starts as the tokens' embeddings
      const int n_own = (fused_units(a, FP_O) - c + P - 1) / P;
      for (int e = tid; e < n_own * 16 * a.M; e += kFusedCompute) {
        const int ul = e / (16 * a.M), rem = e % (16 * a.M), r = rem & 15, m = rem >> 4;
        int tok = a.tokens[a.tok_index[m]];
        if (tok < 0 || tok >= a.V) tok = 0;
        xown[((size_t)ul * 16 + r) * kFusedMaxRows + m] =
            __half2float(a.embed[(size_t)tok * a.d + (size_t)(c + ul * P) * 16 + r]);
      }
    }
    const int L = fused_layers(a);
    for (int layer = 0; layer < L; ++layer) {
      const int Ma = fused_active(a, layer);
      const FusedBlock& b = a.blk[layer < a.n_pre ? layer : a.n_pre];
      const long long tk = 5 * (long long)(target / P);   // trace slot base of the next barrier
      // QKV (+ RoPE, KV write)
      {
        const int K = a.d;
        __half* xl = xs + (size_t)a.M * (K + 8);
        if (c < fused_units(a, FP_QKV))
          fused_stage(a, layer == 0 ? FS_EMBED : FS_NORM, a.x, a.d, b.attn_norm, K, Ma, xs, xl, ssq);
        if (tid == 0) fused_trace(a, tk + 3);
        fused_gemv(a, FP_QKV, layer, Ma, ring, full, empty, &s_fail, xs, xl, red, xown, rope_s, item, tk + 4);
      }
      fused_grid_sync(a, target);
      fused_attention<HD>(a, layer, Ma, area, &s_last, tk + 5 + 3);
      fused_grid_sync(a, target);
      {  // O + residual
        const int K = a.qdim;
        __half* xl = xs + (size_t)a.M * (K + 8);
        if (c < fused_units(a, FP_O)) fused_stage_attn(a, Ma, xs, xl);
        if (tid == 0) fused_trace(a, tk + 10 + 3);
        fused_gemv(a, FP_O, layer, Ma, ring, full, empty, &s_fail, xs, xl, red, xown, rope_s, item, tk + 10 + 4);
      }
      fused_grid_sync(a, target);
      {  // gate_up + SwiGLU
        const int K = a.d;
        __half* xl = xs + (size_t)a.M * (K + 8);
        if (c < fused_units(a, FP_GU)) fused_stage(a, FS_NORM, a.x, a.d, b.ffn_norm, K, Ma, xs, xl, ssq);
        if (tid == 0) fused_trace(a, tk + 15 + 3);
        fused_gemv(a, FP_GU, layer, Ma, ring, full, empty, &s_fail, xs, xl, red, xown, rope_s, item, tk + 15 + 4);
      }
      fused_grid_sync(a, target);
      {  // down + residual
        const int K = a.F;
        __half* xl = xs + (size_t)a.M * (K + 8);
        if (c < fused_units(a, FP_DOWN)) fused_stage(a, FS_RAW, a.h, a.F, nullptr, K, Ma, xs, xl, ssq);
        if (tid == 0) fused_trace(a, tk + 20 + 3);
        fused_gemv(a, FP_DOWN, layer, Ma, ring, full, empty, &s_fail, xs, xl, red, xown, rope_s, item, tk + 20 + 4);
      }
      fused_grid_sync(a, target);
    }

    // ---- output norm + head + argmax --------------------------------------
    const int d = a.d, M = a.M, ldx = d + 8;
    __half* xl = xs + (size_t)M * ldx;
    fused_stage(a, FS_NORM, a.x, d, a.out_norm, d, M, xs, xl, ssq);
    const long long th = 5 * (long long)(target / P);
    if (tid == 0) fused_trace(a, th + 1);
    const int nt = a.V >> 4, tb = (int)((long)c * nt / P), te = (int)((long)(c + 1) * nt / P);
    const int ki = fused_head_item_k(d), nk16 = ki >> 4;
    const int g = lane >> 2, t = lane & 3, brow = g >> 1;
    const __half* bsrc = ((g & 1) ? xl : xs) + (size_t)brow * ldx + 2 * t;
    const bool bok = brow < M;
    const int fr = tid & 15, fm = tid >> 4;
    float best_v = -INFINITY;
    int best_i = 0x7fffffff;
    float* const logits = a.io ? a.io->logits : a.logits;
    int32_t* const argmax = a.io ? a.io->argmax : a.argmax;
    float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc2[4] = {0.f, 0.f, 0.f, 0.f};
    for (int tile = tb; tile < te; ++tile) {
      for (int kk = 0; kk < d; kk += ki) {
        const int s = item % NS;
        mbar_wait_or_fail(&full[s], (unsigned)(item / NS) & 1u, &s_fail);
        const unsigned char* wsl = ring + (size_t)s * kFusedSlotBytes;
        const int j0 = warp * nk16 / kFusedWarps, j1 = (warp + 1) * nk16 / kFusedWarps;
        for (int j = j0; j < j1; ++j) {
          const uint4 wv = *reinterpret_cast<const uint4*>(wsl + (size_t)j * 512 + lane * 16);
          const uint32_t af[4] = {wv.x, wv.y, wv.z, wv.w};
          uint32_t b0 = 0, b1 = 0;
          if (bok) {
            b0 = *reinterpret_cast<const uint32_t*>(bsrc + kk + j * 16);
            b1 = *reinterpret_cast<const uint32_t*>(bsrc + kk + j * 16 + 8);
          }
          if (j & 1) mma_f16_16816(acc2, af, b0, b1);   // two independent chains
          else mma_f16_16816(acc, af, b0, b1);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        ++item;
      }
      float* r = red + ((size_t)(tile & 1) * kFusedWarps + warp) * 64;
      r[g * 4 + t] = (acc[0] + acc2[0]) + (acc[1] + acc2[1]);
      r[(g + 8) * 4 + t] = (acc[2] + acc2[2]) + (acc[3] + acc2[3]);
      acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
      acc2[0] = acc2[1] = acc2[2] = acc2[3] = 0.f;
      fused_sync();
      if (fm < M) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kFusedWarps; ++w) v += red[((size_t)(tile & 1) * kFusedWarps + w) * 64 + fr * 4 + fm];
        const int row = tile * 16 + fr;
        if (logits) logits[(size_t)(a.out_row_dev ? a.out_row_dev[fm] : a.out_row[fm]) * a.V + row] = v;
        if (fused_better(v, row, best_v, best_i)) { best_v = v; best_i = row; }
      }
    }
    if (fm < kFusedMaxRows) { s_bv[fm][fr] = best_v; s_bi[fm][fr] = best_i; }
    if (tid == 0) fused_trace(a, th + 2);
    fused_sync();
    if (tid < M) {
      float v = s_bv[tid][0];
      int ix = s_bi[tid][0];
      for (int r = 1; r < 16; ++r)
        if (fused_better(s_bv[tid][r], s_bi[tid][r], v, ix)) { v = s_bv[tid][r]; ix = s_bi[tid][r]; }
      a.head_val[c * kFusedMaxRows + tid] = v;
      a.head_idx[c * kFusedMaxRows + tid] = ix;
    }
    __threadfence();
    fused_sync();
    if (tid == 0) s_last = atomicAdd(a.head_ticket, 1u) == (unsigned)(P - 1);
    fused_sync();
    if (s_last) {
      __threadfence();
      if (argmax) {
        // every CTA's best per row, loaded in one round, reduced by warps
        float v[kFusedMaxRows];
        int ix[kFusedMaxRows];
#pragma unroll
        for (int m = 0; m < kFusedMaxRows; ++m) {
          v[m] = -INFINITY;
          ix[m] = 0x7fffffff;
          for (int cc = tid; cc < P; cc += kFusedCompute) {
            if (m < M) {
              const float pv = __ldcg(a.head_val + cc * kFusedMaxRows + m);
              const int pi = __ldcg(a.head_idx + cc * kFusedMaxRows + m);
              if (fused_better(pv, pi, v[m], ix[m])) { v[m] = pv; ix[m] = pi; }
            }
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, v[m], o);
            const int oix = __shfl_xor_sync(0xffffffffu, ix[m], o);
            if (fused_better(ov, oix, v[m], ix[m])) { v[m] = ov; ix[m] = oix; }
          }
        }
        if (lane == 0) {
#pragma unroll
          for (int m = 0; m < kFusedMaxRows; ++m) { s_wv[m][warp] = v[m]; s_wi[m][warp] = ix[m]; }
        }
        fused_sync();
        if (tid < M) {
          float bv = s_wv[tid][0];
          int bi = s_wi[tid][0];
          for (int w = 1; w < kFusedWarps; ++w)
            if (fused_better(s_wv[tid][w], s_wi[tid][w], bv, bi)) { bv = s_wv[tid][w]; bi = s_wi[tid][w]; }
          argmax[a.out_row_dev ? a.out_row_dev[tid] : a.out_row[tid]] = bi;
        }
      }
      if (tid == 0) *a.head_ticket = 0u;
    }
  }

  __syncthreads();
  if (tid == 0) {
    fused_trace(a, 3 + 5 * (long long)(5 * fused_layers(a)));
    if (s_fail) atomicOr(a.err_flag, kErrTimeout);
    // the last CTA out resets the barrier words for the next launch
    if (atomicAdd(a.bar + 1, 1u) == gridDim.x - 1) {
      a.bar[0] = 0u;
      a.bar[2] = 0u;
      __threadfence();
      a.bar[1] = 0u;
    }
  }
}

// ---- host-side plan -------------------------------------------------------------
// Bytes of the activation planes ([hi | lo][rows][Kmax + 8] fp16) or of the
// attention scratch, whichever is larger.
__host__ inline int fused_area_bytes(int rows, int kmax, int rep, int hd) {
  const size_t act = (size_t)2 * rows * (kmax + 8) * 2;
  const size_t att = hd == 64 ? fused_attn_bytes<64>(rep) : fused_attn_bytes<128>(rep);
  const size_t b = act > att ? act : att;
  return (int)((b + 127) / 128 * 128);
}
// Residual rows a CTA owns: [ceil((d/16) / grid) tiles][16][4] floats.
__host__ inline int fused_xown_bytes(const FusedArgs& a, int grid) {
  return (fused_units(a, FP_O) + grid - 1) / grid * 16 * kFusedMaxRows * 4;
}
// Reduction buffer: the most tiles any CTA holds in one phase (>= 2 for the
// head's double buffer) x 16 warps x 16 rows x 4 columns.
__host__ inline int fused_red_bytes(const FusedArgs& a, int grid) {
  int tiles = 2;
  for (int ph = 0; ph < 4; ++ph) {
    const int per = (fused_units(a, ph) + grid - 1) / grid * fused_tpu(ph);
    if (per > tiles) tiles = per;
  }
  return tiles * kFusedWarps * 64 * 4;
}

}  // namespace tl
