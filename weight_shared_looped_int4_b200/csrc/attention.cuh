// Grouped-query attention over the fp16 KV cache.
//
// Definition: causal softmax(q k^T / sqrt(hd)) v where q head h reads kv head
// h / (Hq/Hkv) (TinyLoop README, "Status", GQA; tiny-llm feature list,
// "Grouped-Query Attention", "Causal Masking").  Keys and values sit in planes
// [Hkv][ctx][hd] per (lane, effective layer), already rotated by RoPE.
//
// Decode (one query per row): split-KV.  A CTA takes one (row, kv head, key
// split) and all Hq/Hkv query heads that share the kv head, so every key and
// value is read once.  The split length depends only on that row's key count,
// never on the batch, so a row's result does not depend on its neighbours.
// Partial (max, sum, accumulator) triples go to a scratch buffer; the last CTA
// of a (row, kv head) to finish, found by an atomic ticket, merges them in
// split order (deterministic, no spin-wait) and resets the ticket.
//
// Prefill (v1): one warp per (query, q head) with an online softmax.
#pragma once

#include "common.cuh"

namespace tl {

constexpr int kDecodeMaxSplits = 32;
constexpr int kDecodeThreads = 128;

// Keys per split: the smallest power of two >= 32 that needs at most
// kDecodeMaxSplits splits.
__host__ __device__ inline int decode_split_len(int n_keys) {
  int c = 32;
  while (c * kDecodeMaxSplits < n_keys) c <<= 1;
  return c;
}

// Queries and outputs are fp32 inside the model (no rounding between the QKV
// projection, attention and the O projection) and fp16 in the op API.
struct DecodeAttnArgs {
  const float* qf;       // [rows][Hq*hd] rotated queries (fp32), or
  const __half* qh;      // the same in fp16
  int ldq;
  const __half* k;       // K plane of lane 0 (this layer)
  const __half* v;       // V plane of lane 0
  long long lane_stride; // elements between lanes
  int ctx;
  const RowCtx* rows;    // lane and position of each row; keys 0..pos
  int Hkv;
  float* of;             // [rows][Hq*hd] output (fp32), or
  __half* oh;            // the same in fp16
  int ldo;
  float* part;           // [rows][Hkv][kDecodeMaxSplits][REP][hd+2]
  unsigned* ticket;      // [rows][Hkv], zero between launches
};

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__half>(__half v) { return __half2float(v); }
__device__ __forceinline__ void store_out(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_out(__half* p, float v) { *p = __float2half_rn(v); }

template <int HD, int REP, bool F32>
__global__ void __launch_bounds__(kDecodeThreads) decode_attn_kernel(const DecodeAttnArgs a) {
  constexpr int DPL = HD / 32;
  constexpr int CMAX = 256;  // largest split length (n_keys <= 8192)
  __shared__ float qs[REP][HD];
  __shared__ float sc[REP][CMAX];
  __shared__ float ml[REP][2];
  __shared__ int s_last;

  const int split = blockIdx.x, kvh = blockIdx.y, row = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();
  pdl_wait();

  const RowCtx rc = a.rows[row];
  const int n = rc.pos + 1;
  const int C = decode_split_len(n);
  const int nsplit = (n + C - 1) / C;
  if (split >= nsplit) return;
  const int j0 = split * C, j1 = min(n, j0 + C), nk = j1 - j0;
  const float scale = 1.0f / sqrtf((float)HD);

  const __half* kp = a.k + rc.lane * a.lane_stride + (size_t)kvh * a.ctx * HD;
  const __half* vp = a.v + rc.lane * a.lane_stride + (size_t)kvh * a.ctx * HD;
  const size_t qoff = (size_t)row * a.ldq + (size_t)kvh * REP * HD;
  for (int i = threadIdx.x; i < REP * HD; i += kDecodeThreads)
    qs[i / HD][i % HD] = F32 ? a.qf[qoff + i] : __half2float(a.qh[qoff + i]);
  __syncthreads();

  // scores
  for (int j = j0 + warp; j < j1; j += kDecodeThreads / 32) {
    const __half* kr = kp + (size_t)j * HD + lane * DPL;
    float kf[DPL];
    if constexpr (DPL == 4) {
      const uint2 raw = *reinterpret_cast<const uint2*>(kr);
      const float2 a01 = h2_to_f2(raw.x), a23 = h2_to_f2(raw.y);
      kf[0] = a01.x; kf[1] = a01.y; kf[2] = a23.x; kf[3] = a23.y;
    } else {
      const float2 a01 = h2_to_f2(*reinterpret_cast<const uint32_t*>(kr));
      kf[0] = a01.x; kf[1] = a01.y;
    }
#pragma unroll
    for (int h = 0; h < REP; ++h) {
      float p = 0.f;
#pragma unroll
      for (int d = 0; d < DPL; ++d) p = fmaf(qs[h][lane * DPL + d], kf[d], p);
      p = warp_sum(p);
      if (lane == 0) sc[h][j - j0] = p * scale;
    }
  }
  __syncthreads();

  // softmax numerators of this split
  for (int h = warp; h < REP; h += kDecodeThreads / 32) {
    float mx = -INFINITY;
    for (int j = lane; j < nk; j += 32) mx = fmaxf(mx, sc[h][j]);
    mx = warp_max(mx);
    float sum = 0.f;
    for (int j = lane; j < nk; j += 32) {
      const float e = expf(sc[h][j] - mx);
      sc[h][j] = e;
      sum += e;
    }
    sum = warp_sum(sum);
    if (lane == 0) { ml[h][0] = mx; ml[h][1] = sum; }
  }
  __syncthreads();

  // P V
  const int d = threadIdx.x;
  float acc[REP];
#pragma unroll
  for (int h = 0; h < REP; ++h) acc[h] = 0.f;
  if (d < HD) {
    for (int j = 0; j < nk; ++j) {
      const float vv = __half2float(vp[(size_t)(j0 + j) * HD + d]);
#pragma unroll
      for (int h = 0; h < REP; ++h) acc[h] = fmaf(sc[h][j], vv, acc[h]);
    }
  }

  const size_t ooff = (size_t)row * a.ldo + (size_t)kvh * REP * HD;
  if (nsplit == 1) {
    if (d < HD) {
#pragma unroll
      for (int h = 0; h < REP; ++h) {
        if (F32) store_out(a.of + ooff + h * HD + d, acc[h] / ml[h][1]);
        else store_out(a.oh + ooff + h * HD + d, acc[h] / ml[h][1]);
      }
    }
    return;
  }

  constexpr int PSTRIDE = REP * (HD + 2);
  float* pbase = a.part + ((size_t)row * a.Hkv + kvh) * kDecodeMaxSplits * PSTRIDE;
  float* pme = pbase + (size_t)split * PSTRIDE;
  if (d < HD) {
#pragma unroll
    for (int h = 0; h < REP; ++h) pme[h * (HD + 2) + d] = acc[h];
  }
  if (threadIdx.x < REP) {
    pme[threadIdx.x * (HD + 2) + HD] = ml[threadIdx.x][0];
    pme[threadIdx.x * (HD + 2) + HD + 1] = ml[threadIdx.x][1];
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned prev = atomicAdd(a.ticket + row * a.Hkv + kvh, 1u);
    s_last = (prev == (unsigned)(nsplit - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  if (d < HD) {
#pragma unroll
    for (int h = 0; h < REP; ++h) {
      float mx = -INFINITY;
      for (int s = 0; s < nsplit; ++s) mx = fmaxf(mx, __ldcg(pbase + (size_t)s * PSTRIDE + h * (HD + 2) + HD));
      float num = 0.f, den = 0.f;
      for (int s = 0; s < nsplit; ++s) {
        const float* ps = pbase + (size_t)s * PSTRIDE + h * (HD + 2);
        const float w = expf(__ldcg(ps + HD) - mx);
        den = fmaf(w, __ldcg(ps + HD + 1), den);
        num = fmaf(w, __ldcg(ps + d), num);
      }
      if (F32) store_out(a.of + ooff + h * HD + d, num / den);
      else store_out(a.oh + ooff + h * HD + d, num / den);
    }
  }
  if (threadIdx.x == 0) a.ticket[row * a.Hkv + kvh] = 0u;
}

// ---- prefill (v1: one warp per query head, online softmax) ----------------
struct PrefillAttnArgs {
  const float* qf;        // [B][T][Hq*hd] fp32 (model), or
  const __half* qh;       // fp16 (op API)
  long long q_bstride;    // elements between batch entries
  int ldq;                // elements between tokens
  const __half* k;        // K plane of batch 0: [Hkv][ctx][hd]
  const __half* v;
  long long kv_bstride;
  int ctx;
  int T, pos0;
  int Hkv;
  float* of;              // [B][T][Hq*hd] fp32 (model), or
  __half* oh;             // fp16 (op API)
  long long o_bstride;
  int ldo;
};

template <int HD, int REP, bool F32>
__global__ void __launch_bounds__(REP * 32) prefill_attn_simple_kernel(const PrefillAttnArgs a) {
  constexpr int DPL = HD / 32;
  const int t = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int h = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();
  pdl_wait();
  const int pos = a.pos0 + t;
  const float scale = 1.0f / sqrtf((float)HD);
  const size_t qoff = b * a.q_bstride + (size_t)t * a.ldq + (size_t)(kvh * REP + h) * HD + lane * DPL;
  const __half* kp = a.k + b * a.kv_bstride + (size_t)kvh * a.ctx * HD + lane * DPL;
  const __half* vp = a.v + b * a.kv_bstride + (size_t)kvh * a.ctx * HD + lane * DPL;
  float qf[DPL], acc[DPL];
#pragma unroll
  for (int d = 0; d < DPL; ++d) {
    qf[d] = (F32 ? a.qf[qoff + d] : __half2float(a.qh[qoff + d])) * scale;
    acc[d] = 0.f;
  }
  float mx = -INFINITY, l = 0.f;
  for (int j = 0; j <= pos; ++j) {
    float s = 0.f;
#pragma unroll
    for (int d = 0; d < DPL; ++d) s = fmaf(qf[d], __half2float(kp[(size_t)j * HD + d]), s);
    s = warp_sum(s);
    const float mn = fmaxf(mx, s);
    const float corr = expf(mx - mn);
    const float p = expf(s - mn);
    l = l * corr + p;
#pragma unroll
    for (int d = 0; d < DPL; ++d) acc[d] = fmaf(p, __half2float(vp[(size_t)j * HD + d]), acc[d] * corr);
    mx = mn;
  }
  const size_t ooff = b * a.o_bstride + (size_t)t * a.ldo + (size_t)(kvh * REP + h) * HD + lane * DPL;
#pragma unroll
  for (int d = 0; d < DPL; ++d) {
    if (F32) store_out(a.of + ooff + d, acc[d] / l);
    else store_out(a.oh + ooff + d, acc[d] / l);
  }
}

}  // namespace tl
