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
#include "kv8.cuh"

namespace tl {

constexpr int kDecodeMaxSplits = 32;
constexpr int kDecodeThreads = 512;
constexpr int kDecodeSub = 256;     // largest split, staged in shared memory at once
constexpr int kKeyPad = 8;          // fp16 padding per staged key row (bank spread)

// Keys per split: kDecodeSub (256), so contexts up to 8192 keys need at most
// kDecodeMaxSplits splits and up to 256 keys need no merge.  (Splits of 64
// keys spread short contexts over more CTAs but measured slower at batch 1:
// the ticketed merge costs more than the shorter scan saves.)  The length
// depends only on the row's own key count, never on the batch.
__host__ __device__ inline int decode_split_len(int n_keys) {
  int c = kDecodeSub;
  while (c * kDecodeMaxSplits < n_keys) c <<= 1;
  return c;
}

// Tokens per tile of the tcgen05 GEMM's prepared B operand (its kTcTokens).
constexpr int kTcTokensB = 128;

// Partial results of a split: REP x (hd unnormalised sums, max, sum of
// weights, 2 pad) floats, so every head's block starts 16-byte aligned.
constexpr int kPartPad = 4;

// K and V of one split as fp16 rows; with the INT8 cache also their codes as
// copied and the split's scales
__host__ __device__ inline size_t decode_attn_smem_bytes(int hd, int rep, bool kv8 = false) {
  (void)rep;
  return (size_t)2 * kDecodeSub * (hd + kKeyPad) * 2 + (kv8 ? (size_t)2 * kDecodeSub * (hd + 4) : 0);
}

// Queries and outputs are fp32 inside the model (no rounding between the QKV
// projection, attention and the O projection) and fp16 in the op API.
struct DecodeAttnArgs {
  const float* qf;       // [rows][Hq*hd] rotated queries (fp32), or
  const __half* qh;      // the same in fp16
  int ldq;
  const __half* k;       // K plane of lane 0 (this layer); INT8 cache: int8
  const __half* v;       // codes at the same element offsets
  const float* ks;       // INT8 cache: K / V scales of lane 0 [Hkv][ctx]
  const float* vs;       // (element offset / hd); NULL for fp16
  long long lane_stride; // elements between lanes
  int ctx;
  const RowCtx* rows;    // lane and position of each row; keys 0..pos
  int Hkv;
  float* of;             // [rows][Hq*hd] output (fp32), or
  __half* oh;            // the same in fp16
  int ldo;
  float* part;           // [rows][Hkv][kDecodeMaxSplits][REP][hd + kPartPad]
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
// Arrive on `bar` once all of this thread's earlier cp.async copies landed
// (the barrier's expected count includes this arrival).
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

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

// One CTA (16 warps) per (row, kv head, split of up to 256 keys).  All keys of the
// split are copied into shared memory at once (cp.async).  On the tensor
// cores, with the REP query heads of the group as the MMA rows: warp w scores
// keys 16w..16w+15 (S = Q K^T), one warp per head takes the softmax over the
// split, then warp w computes output dims 8w..8w+7 over all keys (O = P V).
// Q and P are split into fp16 pairs (hi, lo).  Splits are merged by the last
// CTA of the (row, kv head) to finish (see above).
// KV8 (INT8 cache): the codes are copied as they are stored and widened to
// fp16 rows (exact integers) once they land; S column j is multiplied by
// key j's scale and the softmax weights by the value's scale before P V (the
// weight sums use the unscaled weights): attention over code * scale.
template <int HD, int REP, bool F32, bool KV8 = false>
__global__ void __launch_bounds__(kDecodeThreads) decode_attn_kernel(const DecodeAttnArgs a) {
  constexpr int SUB = kDecodeSub;
  constexpr int KC = HD / 16;
  constexpr int LDK = HD + kKeyPad;
  constexpr int CHUNKS = SUB * HD / 8;      // 16-byte pieces of K (or V)
  extern __shared__ __align__(128) unsigned char dsm[];
  __half* ks = reinterpret_cast<__half*>(dsm);                 // [SUB][LDK]
  __half* vs = ks + (size_t)SUB * LDK;                         // [SUB][LDK]
  int8_t* kc8 = reinterpret_cast<int8_t*>(vs + (size_t)SUB * LDK);   // KV8: codes [SUB][HD]
  int8_t* vc8 = kc8 + (size_t)SUB * HD;
  float* ksc = reinterpret_cast<float*>(vc8 + (size_t)SUB * HD);    // KV8: scales [SUB]
  float* vsc = ksc + SUB;
  __shared__ __align__(16) float sc[REP][SUB + 4];
  __shared__ float s_m[REP], s_l[REP];
  __shared__ int s_last;

  const int split = blockIdx.x, kvh = blockIdx.y, row = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  pdl_trigger();
  pdl_wait();

  const RowCtx rc = a.rows[row];
  const int n = rc.pos + 1;
  const int C = decode_split_len(n);
  const int nsplit = (n + C - 1) / C;
  if (split >= nsplit) return;
  const int j0 = split * C, j1 = min(n, j0 + C), nk = j1 - j0;
  const float scale = 1.0f / sqrtf((float)HD);

  const size_t lane_kv = (size_t)rc.lane * a.lane_stride + (size_t)kvh * a.ctx * HD;   // elements
  // keys first, values in a second group: the scores and the softmax run
  // while the values are still arriving
  if (KV8) {
    constexpr int CCH = SUB * HD / 16;   // 16-byte pieces of the codes
    const int8_t* kp8 = reinterpret_cast<const int8_t*>(a.k) + lane_kv;
    const int8_t* vp8 = reinterpret_cast<const int8_t*>(a.v) + lane_kv;
    for (int c = threadIdx.x; c < CCH; c += kDecodeThreads) {
      const int key = c / (HD / 16), off = (c % (HD / 16)) * 16;
      const bool ok = key < nk;
      cp_async16(kc8 + key * HD + off, kp8 + (ok ? (size_t)(j0 + key) * HD + off : 0), ok ? 16 : 0);
    }
    cp_async_commit();
    for (int c = threadIdx.x; c < CCH; c += kDecodeThreads) {
      const int key = c / (HD / 16), off = (c % (HD / 16)) * 16;
      const bool ok = key < nk;
      cp_async16(vc8 + key * HD + off, vp8 + (ok ? (size_t)(j0 + key) * HD + off : 0), ok ? 16 : 0);
    }
    cp_async_commit();
    const size_t s0 = lane_kv / HD + j0;
    for (int j = threadIdx.x; j < SUB; j += kDecodeThreads) {
      ksc[j] = j < nk ? __ldcg(a.ks + s0 + j) : 0.f;
      vsc[j] = j < nk ? __ldcg(a.vs + s0 + j) : 0.f;
    }
  } else {
    const __half* kp = a.k + lane_kv;
    const __half* vp = a.v + lane_kv;
    for (int c = threadIdx.x; c < CHUNKS; c += kDecodeThreads) {
      const int key = c / (HD / 8), off = (c % (HD / 8)) * 8;
      const bool ok = key < nk;
      const size_t src = ok ? (size_t)(j0 + key) * HD + off : 0;
      cp_async16(ks + key * LDK + off, kp + src, ok ? 16 : 0);
    }
    cp_async_commit();
    for (int c = threadIdx.x; c < CHUNKS; c += kDecodeThreads) {
      const int key = c / (HD / 8), off = (c % (HD / 8)) * 8;
      const bool ok = key < nk;
      const size_t src = ok ? (size_t)(j0 + key) * HD + off : 0;
      cp_async16(vs + key * LDK + off, vp + src, ok ? 16 : 0);
    }
    cp_async_commit();
  }
  // KV8: widen the landed codes of one plane to fp16 rows
  auto widen = [&](const int8_t* src8, __half* dst) {
    for (int e = threadIdx.x; e < SUB * HD / 4; e += kDecodeThreads) {
      const int key = e / (HD / 4), d4 = (e % (HD / 4)) * 4;
      __half2 c01, c23;
      kv8_codes_h2(*reinterpret_cast<const uint32_t*>(src8 + key * HD + d4), c01, c23);
      *reinterpret_cast<__half2*>(dst + key * LDK + d4) = c01;
      *reinterpret_cast<__half2*>(dst + key * LDK + d4 + 2) = c23;
    }
  };

  // Q fragments (hi, lo): MMA row g is q head g of the group (zero beyond REP)
  const size_t qoff = (size_t)row * a.ldq + (size_t)kvh * REP * HD;
  uint32_t qa[KC][2], ql[KC][2];
#pragma unroll
  for (int c = 0; c < KC; ++c) {
    float2 v0 = make_float2(0.f, 0.f), v1 = make_float2(0.f, 0.f);
    if (g < REP) {
      const size_t o = qoff + (size_t)g * HD + c * 16 + 2 * t;
      if (F32) {
        v0 = *reinterpret_cast<const float2*>(a.qf + o);
        v1 = *reinterpret_cast<const float2*>(a.qf + o + 8);
      } else {
        v0 = __half22float2(*reinterpret_cast<const __half2*>(a.qh + o));
        v1 = __half22float2(*reinterpret_cast<const __half2*>(a.qh + o + 8));
      }
    }
    split_h2(v0.x * scale, v0.y * scale, qa[c][0], ql[c][0]);
    split_h2(v1.x * scale, v1.y * scale, qa[c][1], ql[c][1]);
  }
  cp_async_wait<1>();   // the keys
  __syncthreads();
  if (KV8) {
    widen(kc8, ks);
    __syncthreads();
  }

  // S for keys kb .. kb+15 of this warp (two n8 tiles) -> shared memory
  const int kb = warp * 16;
  if (kb < nk) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < KC; ++c) {
        const __half* kr = ks + (kb + nt * 8 + g) * LDK + c * 16 + 2 * t;
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(kr);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(kr + 8);
        const uint32_t ah[4] = {qa[c][0], 0u, qa[c][1], 0u};
        const uint32_t al[4] = {ql[c][0], 0u, ql[c][1], 0u};
        mma_f16_16816(acc0, ah, b0, b1);
        mma_f16_16816(acc1, al, b0, b1);
      }
      if (g < REP) {
        const int key = kb + nt * 8 + 2 * t;
        const float f0 = KV8 ? ksc[key] : 1.f, f1 = KV8 ? ksc[key + 1] : 1.f;
        sc[g][key] = key < nk ? (acc0[0] + acc1[0]) * f0 : -INFINITY;
        sc[g][key + 1] = key + 1 < nk ? (acc0[1] + acc1[1]) * f1 : -INFINITY;
      }
    }
  }
  __syncthreads();

  // softmax over the split: warp h takes head h (unnormalised exp in place)
  if (warp < REP) {
    const int h = warp;
    float mx = -INFINITY;
    for (int j = lane; j < nk; j += 32) mx = fmaxf(mx, sc[h][j]);
    mx = warp_max(mx);
    float sum = 0.f;
    for (int j = lane; j < nk; j += 32) {
      const float e = expf(sc[h][j] - mx);
      sc[h][j] = e;
      sum += e;
    }
    // keys nk .. end of their last 16-key chunk read as zero probability
    for (int j = nk + lane; j < ((nk + 15) & ~15); j += 32) sc[h][j] = 0.f;
    sum = warp_sum(sum);
    if (lane == 0) { s_m[h] = mx; s_l[h] = sum; }
  }
  cp_async_wait<0>();   // the values
  __syncthreads();
  if (KV8) {
    widen(vc8, vs);
    __syncthreads();
  }

  // O = P V: warp w takes output dims 8w .. 8w+7 over all keys of the split
  const int dt = warp;
  float o[4] = {0.f, 0.f, 0.f, 0.f}, o2[4] = {0.f, 0.f, 0.f, 0.f};
  if (dt < HD / 8) {
    const int nch = (nk + 15) >> 4;
    for (int c = 0; c < nch; ++c) {
      uint32_t pa[4] = {0u, 0u, 0u, 0u}, pl[4] = {0u, 0u, 0u, 0u};
      if (g < REP) {
        float2 p0 = *reinterpret_cast<const float2*>(&sc[g][c * 16 + 2 * t]);
        float2 p1 = *reinterpret_cast<const float2*>(&sc[g][c * 16 + 8 + 2 * t]);
        if (KV8) {   // the values' scales (the weight sums stay unscaled)
          const float2 v0 = *reinterpret_cast<const float2*>(&vsc[c * 16 + 2 * t]);
          const float2 v1 = *reinterpret_cast<const float2*>(&vsc[c * 16 + 8 + 2 * t]);
          p0.x *= v0.x; p0.y *= v0.y; p1.x *= v1.x; p1.y *= v1.y;
        }
        split_h2(p0.x, p0.y, pa[0], pl[0]);
        split_h2(p1.x, p1.y, pa[2], pl[2]);
      }
      uint32_t vb[4];
      // rows (keys) c*16 .. +15 at dims 8 dt .. +7: two 8x8 transposed tiles
      const int key = c * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      ldmatrix_x4_trans(vb, vs + key * LDK + dt * 8);
      mma_f16_16816(o, pa, vb[0], vb[1]);
      mma_f16_16816(o2, pl, vb[0], vb[1]);
    }
  }
  const size_t ooff = (size_t)row * a.ldo + (size_t)kvh * REP * HD;
  if (nsplit == 1) {
    if (dt < HD / 8 && g < REP) {
      const float inv = 1.f / s_l[g];
      const int dd = g * HD + dt * 8 + 2 * t;
      if (F32) {
        store_out(a.of + ooff + dd, (o[0] + o2[0]) * inv);
        store_out(a.of + ooff + dd + 1, (o[1] + o2[1]) * inv);
      } else {
        store_out(a.oh + ooff + dd, (o[0] + o2[0]) * inv);
        store_out(a.oh + ooff + dd + 1, (o[1] + o2[1]) * inv);
      }
    }
    return;
  }

  constexpr int HS = HD + kPartPad;
  constexpr int PSTRIDE = REP * HS;
  float* pbase = a.part + ((size_t)row * a.Hkv + kvh) * kDecodeMaxSplits * PSTRIDE;
  float* pme = pbase + (size_t)split * PSTRIDE;
  if (dt < HD / 8 && g < REP) {
    pme[g * HS + dt * 8 + 2 * t] = o[0] + o2[0];
    pme[g * HS + dt * 8 + 2 * t + 1] = o[1] + o2[1];
  }
  if (threadIdx.x < REP) {
    pme[threadIdx.x * HS + HD] = s_m[threadIdx.x];
    pme[threadIdx.x * HS + HD + 1] = s_l[threadIdx.x];
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

  // (max, sum of weights) of every split and head in one round of loads,
  // then each (head, dim) output from independent loads in split order
  float* mls = &sc[0][0];   // >= 2 * kDecodeMaxSplits * REP floats
  for (int e = threadIdx.x; e < nsplit * REP * 2; e += kDecodeThreads) {
    const int sp = e / (REP * 2), rem = e % (REP * 2);
    mls[e] = __ldcg(pbase + (size_t)sp * PSTRIDE + (rem >> 1) * HS + HD + (rem & 1));
  }
  __syncthreads();
  for (int oi = threadIdx.x; oi < REP * HD; oi += kDecodeThreads) {
    const int h = oi / HD, d = oi % HD;
    float mx = -INFINITY;
    for (int sp = 0; sp < nsplit; ++sp) mx = fmaxf(mx, mls[(sp * REP + h) * 2]);
    float num = 0.f, den = 0.f;
#pragma unroll 8
    for (int sp = 0; sp < nsplit; ++sp) {
      const float w = expf(mls[(sp * REP + h) * 2] - mx);
      den = fmaf(w, mls[(sp * REP + h) * 2 + 1], den);
      num = fmaf(w, __ldcg(pbase + (size_t)sp * PSTRIDE + h * HS + d), num);
    }
    if (F32) store_out(a.of + ooff + h * HD + d, num / den);
    else store_out(a.oh + ooff + h * HD + d, num / den);
  }
  if (threadIdx.x == 0) a.ticket[row * a.Hkv + kvh] = 0u;
}

struct PrefillAttnArgs {
  const float* qf;        // [B][T][Hq*hd] fp32 (model), or
  const __half* qh;       // fp16 (op API)
  long long q_bstride;    // elements between batch entries
  int ldq;                // elements between tokens
  const __half* k;        // K plane of batch 0: [Hkv][ctx][hd]
  const __half* v;        // (INT8 cache: int8 codes at the same element offsets)
  const float* ks;        // INT8 cache: K / V scales of batch 0 [Hkv][ctx]
  const float* vs;        // (element offset / hd); NULL for fp16
  long long kv_bstride;
  int ctx;
  int T, pos0;
  int Hkv;
  float* of;              // [B][T][Hq*hd] fp32 (model), or
  __half* oh;             // fp16 (op API)
  long long o_bstride;
  int ldo;
  int rep;                // query heads per kv head (the kernel's REP heads are a slice of a group)
  // model prefill: the output goes straight into the O projection's prepared
  // B tiles ([token tiles][K/128][2 atoms][256 rows][128 B], fp16 hi rows
  // then lo rows, 128-byte swizzled; K = Hq * hd) instead of `of`
  uint8_t* bt;
  int bt_groups;
  int* err_flag;          // device fault flags (a bounded wait gave up), or NULL
};

// ---- prefill: tiled, tensor cores (m16n8k16), online softmax --------------
// One CTA per (16-query tile, slice of REP query heads of one kv group, batch
// entry; short prompts use smaller slices for more CTAs); warp w handles q head
// kv_head * REP + w for the 16 queries, so each K/V block staged in shared
// memory serves all REP heads of the group.  S = Q K^T and O += P V run on the
// tensor cores; Q and P are split into fp16 pairs (hi, lo) and both halves are
// multiplied (K and V are fp16 already), so the result keeps ~fp32 accuracy.
constexpr int kPfKeys = 64;   // keys per staged block
constexpr int kPfPad = 8;     // fp16 padding per staged row

__host__ __device__ inline size_t prefill_attn_smem_bytes(int hd) {
  return (size_t)2 * kPfKeys * (hd + kPfPad) * 2 + 2 * kPfKeys * 4;   // + INT8 cache scales
}

// KV8: INT8 KV cache.  The codes are staged as fp16 (exact integers) and the
// scales applied outside the MMAs: S column j times the key's scale, and the
// softmax weights times the value's scale before P V (the weight sums use
// the unscaled weights), so the result equals attention over code * scale.
template <int HD, int REP, bool F32, bool KV8>
__global__ void __launch_bounds__(REP * 32) prefill_attn_mma_kernel(const PrefillAttnArgs a) {
  constexpr int KC = HD / 16;        // k16 chunks of a head
  constexpr int NT = HD / 8;         // n8 tiles of the output
  constexpr int LD = HD + kPfPad;
  constexpr int NTHR = REP * 32;
  extern __shared__ __align__(128) unsigned char psm[];
  __half* ks = reinterpret_cast<__half*>(psm);             // [64][LD]
  __half* vs = ks + kPfKeys * LD;                          // [64][LD]
  float* sks = reinterpret_cast<float*>(vs + kPfKeys * LD);   // INT8: key / value scales [64] each
  float* svs = sks + kPfKeys;

  const int qt = blockIdx.x, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int h = blockIdx.y * REP + warp;   // REP divides the group size a.rep
  const int kvh = h / a.rep;
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
  const int8_t* kp8 = reinterpret_cast<const int8_t*>(a.k) + b * a.kv_bstride + (size_t)kvh * a.ctx * HD;
  const int8_t* vp8 = reinterpret_cast<const int8_t*>(a.v) + b * a.kv_bstride + (size_t)kvh * a.ctx * HD;
  const float* ksp = KV8 ? a.ks + (b * a.kv_bstride) / HD + (size_t)kvh * a.ctx : nullptr;
  const float* vsp = KV8 ? a.vs + (b * a.kv_bstride) / HD + (size_t)kvh * a.ctx : nullptr;

  for (int kb = 0; kb < nblk; ++kb) {
    const int j0 = kb * kPfKeys;
    __syncthreads();  // the previous block is no longer read
    if (KV8) {
      // 16 codes per load, widened to fp16 (exact), zeros past the last key
      for (int c = threadIdx.x; c < 2 * kPfKeys * HD / 16; c += NTHR) {
        const int kv = c / (kPfKeys * HD / 16), rem = c % (kPfKeys * HD / 16);
        const int key = rem / (HD / 16), off = (rem % (HD / 16)) * 16;
        uint4 w = make_uint4(0, 0, 0, 0);
        if (j0 + key <= last_key) w = __ldcg(reinterpret_cast<const uint4*>((kv ? vp8 : kp8) + (size_t)(j0 + key) * HD + off));
        __half* dst = (kv ? vs : ks) + key * LD + off;
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          __half2 c01, c23;
          kv8_codes_h2(ws[i], c01, c23);
          uint2 h;
          h.x = *reinterpret_cast<const uint32_t*>(&c01);
          h.y = *reinterpret_cast<const uint32_t*>(&c23);
          *reinterpret_cast<uint2*>(dst + 4 * i) = h;
        }
      }
      for (int c = threadIdx.x; c < 2 * kPfKeys; c += NTHR) {
        const int kv = c / kPfKeys, key = c % kPfKeys;
        sks[c] = (j0 + key <= last_key) ? __ldcg((kv ? vsp : ksp) + j0 + key) : 0.f;
      }
    } else {
      for (int c = threadIdx.x; c < kPfKeys * HD / 8; c += NTHR) {
        const int key = c / (HD / 8), off = (c % (HD / 8)) * 8;
        const bool ok = j0 + key <= last_key;
        const size_t src = ok ? (size_t)(j0 + key) * HD + off : 0;
        cp_async16(ks + key * LD + off, kp + src, ok ? 16 : 0);
        cp_async16(vs + key * LD + off, vp + src, ok ? 16 : 0);
      }
      cp_async_commit();
      cp_async_wait<0>();
    }
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
      if (KV8) {   // column j of S times key j's scale
        const float s0 = sks[n * 8 + 2 * t], s1 = sks[n * 8 + 2 * t + 1];
        sc[n][0] *= s0; sc[n][1] *= s1;
        sc[n][2] *= s0; sc[n][3] *= s1;
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
    if (KV8) {   // the weights times their value's scale (the sums above are unscaled)
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const float s0 = svs[n * 8 + 2 * t], s1 = svs[n * 8 + 2 * t + 1];
        sc[n][0] *= s0; sc[n][1] *= s1;
        sc[n][2] *= s0; sc[n][3] *= s1;
      }
    }
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
  if (F32 && a.bt) {
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int k = h * HD + n * 8 + 2 * t;     // column of the O projection's input
      const int grp = k >> 7, kg = k & 127;
#pragma unroll
      for (int half_ = 0; half_ < 2; ++half_) {
        const int r = half_ ? r1 : r0;
        if (r < a.T) {
          const float inv = half_ ? inv1 : inv0;
          uint32_t hw, lw;
          split_h2(o[n][2 * half_] * inv, o[n][2 * half_ + 1] * inv, hw, lw);
          const int tt = r / kTcTokensB, tl_ = r % kTcTokensB;
          uint8_t* blk = a.bt + ((size_t)tt * a.bt_groups + grp) * (2 * kTcTokensB * 256);
          *reinterpret_cast<uint32_t*>(blk + sw128_offset(tl_, kg, 2 * kTcTokensB)) = hw;
          *reinterpret_cast<uint32_t*>(blk + sw128_offset(kTcTokensB + tl_, kg, 2 * kTcTokensB)) = lw;
        }
      }
    }
    return;
  }
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

}  // namespace tl
