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
constexpr int kDecodeThreads = 256;
constexpr int kDecodeSub = 64;      // keys per shared-memory sub-chunk
constexpr int kKeyPad = 8;          // fp16 padding per staged key row (bank spread)

// Keys per split: 64, doubled until at most kDecodeMaxSplits splits are
// needed (so <= 8192 keys fit).  Depends only on the row's own key count.
__host__ __device__ inline int decode_split_len(int n_keys) {
  int c = kDecodeSub;
  while (c * kDecodeMaxSplits < n_keys) c <<= 1;
  return c;
}

__host__ __device__ inline size_t decode_attn_smem_bytes(int hd) {
  return (size_t)2 * 2 * kDecodeSub * (hd + kKeyPad) * 2;  // K and V, double buffered
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

// cp.async of 16 bytes into shared memory; src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, int src_bytes) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(gsrc), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// One CTA per (row, kv head, key split).  The split's keys are streamed in
// sub-chunks of kDecodeSub keys; K and V of the next sub-chunk are copied into
// shared memory (cp.async, double buffered) while the current one is used, and
// the softmax runs online across sub-chunks.  Up to 256 keys there is one
// split and no merge step.
template <int HD, int REP, bool F32>
__global__ void __launch_bounds__(kDecodeThreads) decode_attn_kernel(const DecodeAttnArgs a) {
  constexpr int DPL = HD / 32;
  constexpr int SUB = kDecodeSub;
  constexpr int NW = kDecodeThreads / 32;
  constexpr int CHUNKS = SUB * HD / 8;   // 16-byte pieces of one K (or V) sub-chunk
  constexpr int KH = kDecodeThreads / HD; // key interleave of the P V step
  constexpr int LDK = HD + kKeyPad;
  extern __shared__ __align__(128) unsigned char dsm[];
  __half (*ks)[SUB][LDK] = reinterpret_cast<__half (*)[SUB][LDK]>(dsm);
  __half (*vs)[SUB][LDK] = reinterpret_cast<__half (*)[SUB][LDK]>(dsm + (size_t)2 * SUB * LDK * 2);
  __shared__ __align__(16) float qs[REP][HD];
  __shared__ float sc[REP][SUB];
  __shared__ float s_m[REP], s_l[REP], s_corr[REP];
  __shared__ float s_acc[KH][REP][HD];
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
  const int nsub = (nk + SUB - 1) / SUB;
  const float scale = 1.0f / sqrtf((float)HD);

  const __half* kp = a.k + rc.lane * a.lane_stride + (size_t)kvh * a.ctx * HD;
  const __half* vp = a.v + rc.lane * a.lane_stride + (size_t)kvh * a.ctx * HD;

  auto issue = [&](int sb, int b) {
    const int jb = j0 + sb * SUB;
    for (int c = threadIdx.x; c < CHUNKS; c += kDecodeThreads) {
      const int key = c / (HD / 8), off = (c % (HD / 8)) * 8;
      const bool ok = jb + key < j1;
      const size_t src = ok ? (size_t)(jb + key) * HD + off : 0;
      cp_async16(&ks[b][key][off], kp + src, ok ? 16 : 0);
      cp_async16(&vs[b][key][off], vp + src, ok ? 16 : 0);
    }
    cp_async_commit();
  };
  issue(0, 0);

  const size_t qoff = (size_t)row * a.ldq + (size_t)kvh * REP * HD;
  for (int i = threadIdx.x; i < REP * HD; i += kDecodeThreads)
    qs[i / HD][i % HD] = F32 ? a.qf[qoff + i] : __half2float(a.qh[qoff + i]);
  if (threadIdx.x < REP) { s_m[threadIdx.x] = -INFINITY; s_l[threadIdx.x] = 0.f; }

  const int d = threadIdx.x % HD, kh = threadIdx.x / HD;
  float acc[REP];
#pragma unroll
  for (int h = 0; h < REP; ++h) acc[h] = 0.f;

  for (int sb = 0; sb < nsub; ++sb) {
    const int b = sb & 1;
    if (sb + 1 < nsub) {
      issue(sb + 1, b ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int kc = min(SUB, nk - sb * SUB);

    // scores of this sub-chunk: thread (key j, head h) takes one dot product
    // (K row from shared memory, q broadcast), no shuffles
    for (int item = threadIdx.x; item < REP * SUB; item += kDecodeThreads) {
      const int jj = item % SUB, h = item / SUB;
      if (jj < kc) {
        const float4* qv = reinterpret_cast<const float4*>(qs[h]);
        const uint4* kr = reinterpret_cast<const uint4*>(&ks[b][jj][0]);
        float p = 0.f;
#pragma unroll 4
        for (int c8 = 0; c8 < HD / 8; ++c8) {
          const uint4 raw = kr[c8];
          const float4 qa = qv[2 * c8], qb = qv[2 * c8 + 1];
          const float2 k01 = h2_to_f2(raw.x), k23 = h2_to_f2(raw.y);
          const float2 k45 = h2_to_f2(raw.z), k67 = h2_to_f2(raw.w);
          p = fmaf(qa.x, k01.x, p); p = fmaf(qa.y, k01.y, p);
          p = fmaf(qa.z, k23.x, p); p = fmaf(qa.w, k23.y, p);
          p = fmaf(qb.x, k45.x, p); p = fmaf(qb.y, k45.y, p);
          p = fmaf(qb.z, k67.x, p); p = fmaf(qb.w, k67.y, p);
        }
        sc[h][jj] = p * scale;
      }
    }
    __syncthreads();

    // online softmax update (one warp per head)
    for (int h = warp; h < REP; h += NW) {
      float mx = -INFINITY;
      for (int j = lane; j < kc; j += 32) mx = fmaxf(mx, sc[h][j]);
      mx = warp_max(mx);
      const float m_new = fmaxf(s_m[h], mx);
      float sum = 0.f;
      for (int j = lane; j < kc; j += 32) {
        const float e = expf(sc[h][j] - m_new);
        sc[h][j] = e;
        sum += e;
      }
      sum = warp_sum(sum);
      if (lane == 0) {
        const float corr = expf(s_m[h] - m_new);
        s_corr[h] = corr;
        s_l[h] = s_l[h] * corr + sum;
        s_m[h] = m_new;
      }
    }
    __syncthreads();

    // P V: thread (d, kh) takes keys kh, kh + KH, ...
#pragma unroll
    for (int h = 0; h < REP; ++h) acc[h] *= s_corr[h];
    for (int jj = kh; jj < kc; jj += KH) {
      const float vv = __half2float(vs[b][jj][d]);
#pragma unroll
      for (int h = 0; h < REP; ++h) acc[h] = fmaf(sc[h][jj], vv, acc[h]);
    }
    __syncthreads();
  }

  // combine the key interleave
#pragma unroll
  for (int h = 0; h < REP; ++h) s_acc[kh][h][d] = acc[h];
  __syncthreads();
  if (threadIdx.x < HD) {
#pragma unroll
    for (int h = 0; h < REP; ++h) {
      float v = 0.f;
#pragma unroll
      for (int q = 0; q < KH; ++q) v += s_acc[q][h][d];
      acc[h] = v;
    }
  }

  const size_t ooff = (size_t)row * a.ldo + (size_t)kvh * REP * HD;
  if (nsplit == 1) {
    if (threadIdx.x < HD) {
#pragma unroll
      for (int h = 0; h < REP; ++h) {
        if (F32) store_out(a.of + ooff + h * HD + d, acc[h] / s_l[h]);
        else store_out(a.oh + ooff + h * HD + d, acc[h] / s_l[h]);
      }
    }
    return;
  }

  constexpr int PSTRIDE = REP * (HD + 2);
  float* pbase = a.part + ((size_t)row * a.Hkv + kvh) * kDecodeMaxSplits * PSTRIDE;
  float* pme = pbase + (size_t)split * PSTRIDE;
  if (threadIdx.x < HD) {
#pragma unroll
    for (int h = 0; h < REP; ++h) pme[h * (HD + 2) + d] = acc[h];
  }
  if (threadIdx.x < REP) {
    pme[threadIdx.x * (HD + 2) + HD] = s_m[threadIdx.x];
    pme[threadIdx.x * (HD + 2) + HD + 1] = s_l[threadIdx.x];
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

  if (threadIdx.x < HD) {
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
