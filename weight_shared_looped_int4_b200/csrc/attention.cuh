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

// ---- prefill: tiled, tensor cores (m16n8k16), online softmax --------------
// One CTA per (16-query tile, kv head, batch entry); warp w handles q head
// kv_head * REP + w for the 16 queries, so each K/V block staged in shared
// memory serves all REP heads of the group.  S = Q K^T and O += P V run on the
// tensor cores; Q and P are split into fp16 pairs (hi, lo) and both halves are
// multiplied (K and V are fp16 already), so the result keeps ~fp32 accuracy.
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"((unsigned)__cvta_generic_to_shared(p)));
}
__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}
// (hi, lo) fp16 pairs of two floats.
__device__ __forceinline__ void split_h2(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(a, b);
  const float2 r = __half22float2(h);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = pack_h2(a - r.x, b - r.y);
}

constexpr int kPfKeys = 64;   // keys per staged block
constexpr int kPfPad = 8;     // fp16 padding per staged row

__host__ __device__ inline size_t prefill_attn_smem_bytes(int hd) {
  return (size_t)2 * kPfKeys * (hd + kPfPad) * 2;
}

template <int HD, int REP, bool F32>
__global__ void __launch_bounds__(REP * 32) prefill_attn_mma_kernel(const PrefillAttnArgs a) {
  constexpr int KC = HD / 16;        // k16 chunks of a head
  constexpr int NT = HD / 8;         // n8 tiles of the output
  constexpr int LD = HD + kPfPad;
  constexpr int NTHR = REP * 32;
  extern __shared__ __align__(128) unsigned char psm[];
  __half* ks = reinterpret_cast<__half*>(psm);             // [64][LD]
  __half* vs = ks + kPfKeys * LD;                          // [64][LD]

  const int qt = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int h = kvh * REP + warp;
  const int q0 = qt * 16;
  pdl_trigger();
  pdl_wait();

  // Q fragments (hi, lo) of rows q0+g and q0+g+8, scaled by 1/sqrt(hd)
  const float scale = 1.0f / sqrtf((float)HD);
  uint32_t qa[KC][4], ql[KC][4];
  {
    const int r0 = min(q0 + g, a.T - 1), r1 = min(q0 + g + 8, a.T - 1);
    const size_t base0 = b * a.q_bstride + (size_t)r0 * a.ldq + (size_t)h * HD;
    const size_t base1 = b * a.q_bstride + (size_t)r1 * a.ldq + (size_t)h * HD;
    auto ld2 = [&](size_t off) -> float2 {
      if (F32) return *reinterpret_cast<const float2*>(a.qf + off);
      return __half22float2(*reinterpret_cast<const __half2*>(a.qh + off));
    };
#pragma unroll
    for (int c = 0; c < KC; ++c) {
      const int d0 = c * 16 + 2 * t;
      float2 v;
      v = ld2(base0 + d0);     split_h2(v.x * scale, v.y * scale, qa[c][0], ql[c][0]);
      v = ld2(base1 + d0);     split_h2(v.x * scale, v.y * scale, qa[c][1], ql[c][1]);
      v = ld2(base0 + d0 + 8); split_h2(v.x * scale, v.y * scale, qa[c][2], ql[c][2]);
      v = ld2(base1 + d0 + 8); split_h2(v.x * scale, v.y * scale, qa[c][3], ql[c][3]);
    }
  }

  float o[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int i = 0; i < 4; ++i) o[n][i] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const int pq0 = a.pos0 + q0 + g, pq1 = pq0 + 8;   // query positions of this thread's rows
  const int last_key = a.pos0 + min(q0 + 15, a.T - 1);
  const int nblk = last_key / kPfKeys + 1;
  const __half* kp = a.k + b * a.kv_bstride + (size_t)kvh * a.ctx * HD;
  const __half* vp = a.v + b * a.kv_bstride + (size_t)kvh * a.ctx * HD;

  for (int kb = 0; kb < nblk; ++kb) {
    const int j0 = kb * kPfKeys;
    __syncthreads();  // the previous block is no longer read
    for (int c = threadIdx.x; c < kPfKeys * HD / 8; c += NTHR) {
      const int key = c / (HD / 8), off = (c % (HD / 8)) * 8;
      const bool ok = j0 + key <= last_key;
      const size_t src = ok ? (size_t)(j0 + key) * HD + off : 0;
      cp_async16(ks + key * LD + off, kp + src, ok ? 16 : 0);
      cp_async16(vs + key * LD + off, vp + src, ok ? 16 : 0);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();

    // S = Q K^T for 64 keys: 8 n8 tiles
    float sc[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) {
#pragma unroll
      for (int i = 0; i < 4; ++i) sc[n][i] = 0.f;
#pragma unroll
      for (int c = 0; c < KC; ++c) {
        const __half* kr = ks + (n * 8 + g) * LD + c * 16 + 2 * t;
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(kr);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(kr + 8);
        mma_f16_16816(sc[n], qa[c], b0, b1);
        mma_f16_16816(sc[n], ql[c], b0, b1);
      }
    }
    // causal mask and online softmax (rows g and g+8 of the tile)
    float mx0 = m0, mx1 = m1;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const int key = j0 + n * 8 + 2 * t;
      if (key > pq0) sc[n][0] = -INFINITY;
      if (key + 1 > pq0) sc[n][1] = -INFINITY;
      if (key > pq1) sc[n][2] = -INFINITY;
      if (key + 1 > pq1) sc[n][3] = -INFINITY;
      mx0 = fmaxf(mx0, fmaxf(sc[n][0], sc[n][1]));
      mx1 = fmaxf(mx1, fmaxf(sc[n][2], sc[n][3]));
    }
#pragma unroll
    for (int o_ = 1; o_ < 4; o_ <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o_));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o_));
    }
    const float c0 = (m0 == -INFINITY) ? 0.f : expf(m0 - mx0);
    const float c1 = (m1 == -INFINITY) ? 0.f : expf(m1 - mx1);
    m0 = mx0;
    m1 = mx1;
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      sc[n][0] = (mx0 == -INFINITY) ? 0.f : expf(sc[n][0] - mx0);
      sc[n][1] = (mx0 == -INFINITY) ? 0.f : expf(sc[n][1] - mx0);
      sc[n][2] = (mx1 == -INFINITY) ? 0.f : expf(sc[n][2] - mx1);
      sc[n][3] = (mx1 == -INFINITY) ? 0.f : expf(sc[n][3] - mx1);
      s0 += sc[n][0] + sc[n][1];
      s1 += sc[n][2] + sc[n][3];
    }
#pragma unroll
    for (int o_ = 1; o_ < 4; o_ <<= 1) {
      s0 += __shfl_xor_sync(0xffffffffu, s0, o_);
      s1 += __shfl_xor_sync(0xffffffffu, s1, o_);
    }
    l0 = l0 * c0 + s0;
    l1 = l1 * c1 + s1;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      o[n][0] *= c0; o[n][1] *= c0;
      o[n][2] *= c1; o[n][3] *= c1;
    }
    // O += P V: P as A fragments (hi, lo) straight from the S accumulators
#pragma unroll
    for (int kc = 0; kc < 4; ++kc) {
      uint32_t pa[4], pl[4];
      split_h2(sc[2 * kc][0], sc[2 * kc][1], pa[0], pl[0]);
      split_h2(sc[2 * kc][2], sc[2 * kc][3], pa[1], pl[1]);
      split_h2(sc[2 * kc + 1][0], sc[2 * kc + 1][1], pa[2], pl[2]);
      split_h2(sc[2 * kc + 1][2], sc[2 * kc + 1][3], pa[3], pl[3]);
#pragma unroll
      for (int n2 = 0; n2 < NT / 2; ++n2) {
        // V rows kc*16 .. +15, dims n2*16 .. +15 -> B fragments of two n8 tiles
        const int key = kc * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int dim = n2 * 16 + (lane >> 4) * 8;
        uint32_t vb[4];
        ldmatrix_x4_trans(vb, vs + key * LD + dim);
        mma_f16_16816(o[2 * n2], pa, vb[0], vb[1]);
        mma_f16_16816(o[2 * n2], pl, vb[0], vb[1]);
        mma_f16_16816(o[2 * n2 + 1], pa, vb[2], vb[3]);
        mma_f16_16816(o[2 * n2 + 1], pl, vb[2], vb[3]);
      }
    }
  }

  // normalise and store rows q0+g, q0+g+8
  const float inv0 = 1.f / l0, inv1 = 1.f / l1;
  const int r0 = q0 + g, r1 = q0 + g + 8;
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const int d = n * 8 + 2 * t;
    if (r0 < a.T) {
      const size_t off = b * a.o_bstride + (size_t)r0 * a.ldo + (size_t)h * HD + d;
      if (F32) { a.of[off] = o[n][0] * inv0; a.of[off + 1] = o[n][1] * inv0; }
      else *reinterpret_cast<uint32_t*>(a.oh + off) = pack_h2(o[n][0] * inv0, o[n][1] * inv0);
    }
    if (r1 < a.T) {
      const size_t off = b * a.o_bstride + (size_t)r1 * a.ldo + (size_t)h * HD + d;
      if (F32) { a.of[off] = o[n][2] * inv1; a.of[off + 1] = o[n][3] * inv1; }
      else *reinterpret_cast<uint32_t*>(a.oh + off) = pack_h2(o[n][2] * inv1, o[n][3] * inv1);
    }
  }
}

// ---- prefill (v1: one warp per query head, online softmax) ----------------

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
