// INT4 group-wise GEMM on the 5th-generation tensor cores (tcgen05, TMEM)
// for the prefill linears: Y[t][n] = sum_k X[t][k] * (q[n][k] - z) * s, with
// groups of 128 along K (TinyLoop README, "Status": INT4 loop / pre linears
// with zero points; the workload's w = (q - z) * s).
//
// Design (ours, sm_100a):
// * One CTA owns a 128-row weight tile, a 128-token tile and a slice of the K
//   groups (split-K when the tile grid is smaller than the SM count).
// * Per K group (128 k) the tensor core computes P = A B^T with A = the exact
//   fp16 integers q - z of the tile (no scale) and B = the activations split
//   into an fp16 pair: rows 0..127 of B hold x_hi of the 128 tokens, rows
//   128..255 hold x_lo (one N = 256 MMA).  P goes to a TMEM buffer; the
//   epilogue warps read it and accumulate s[n][group] * (P_hi + P_lo) in fp32
//   registers.  So no weight is rounded and the activation keeps ~22 bits;
//   fp16 weights or activations move the looped model's logits by ~0.05.
// * Warp roles (16 warps): warp 0 allocates TMEM and one lane issues
//   tcgen05.mma; one lane of warp 1 issues the bulk asynchronous copies (raw
//   INT4 words + scales/zeros a few groups ahead, the prepared B atoms per
//   stage); warps 2-7 dequantize A from the raw ring straight into the
//   128-byte swizzled K-major layout the MMA descriptor reads (the
//   dequantisation, not the tensor core, paces this GEMM); warps 8-15 are the
//   epilogue.  Stages of 64 k (4 deep), the raw ring (3 groups) and the TMEM
//   buffers (2 groups) are handed over with mbarriers (tcgen05.commit signals
//   MMA completion).
// * Split-K partials go to a scratch buffer; a merge kernel (one CTA per 8
//   tokens of a tile, all loads in flight) adds them in split order, so the
//   result is deterministic, and applies the epilogue: residual add, raw
//   fp32, fp16 store, or RoPE with the Q output and the K/V cache write.
//   Without a split the GEMM applies the epilogue itself.
// * Every mbarrier wait is bounded; on time-out the kernel records kErrTimeout,
//   skips the rest of its work and still frees its TMEM.
#pragma once

#include "attention.cuh"
#include "common.cuh"

namespace tl {

// ---- tcgen05 wrappers ------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive on `bar` when all earlier tcgen05 operations of this thread are done.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// 32 consecutive 32-bit columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
// 16 consecutive 32-bit columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
// Named barrier among the epilogue warps only.
__device__ __forceinline__ void epi_sync(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (the canonical layout of a row-major tile whose rows are
// 128 bytes, written with the 16-byte chunk index XOR (row % 8)).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(const void* p) {
  const uint64_t addr = smem_u32(p);
  uint64_t d = (addr >> 4) & 0x3FFFull;   // start address
  d |= 1ull << 16;                         // leading byte offset (unused with swizzle)
  d |= (uint64_t)(1024 >> 4) << 32;        // stride byte offset: 8 rows x 128 B
  d |= 1ull << 46;                         // descriptor version
  d |= 2ull << 61;                         // 128-byte swizzle
  return d;
}
// Instruction descriptor of kind::f16: fp16 A and B (K-major), fp32 D.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}


// TC_SWIGLU_B: the gate_up projection with its tensor-core rows interleaved
// (tile t = gate rows 64t.. and up rows F + 64t..): silu(gate) * up is written
// straight into the down projection's prepared B tiles.
enum TcEpi { TC_RESID = 0, TC_RAW = 1, TC_STORE = 2, TC_ROPE_KV = 3, TC_SWIGLU_B = 4 };

constexpr int kTcThreads = 512;       // 16 warps
constexpr int kTcRows = 128;          // weight rows per tile (MMA M)
constexpr int kTcTokens = 128;        // tokens per tile
static_assert(kTcTokens == kTcTokensB, "the prefill attention writes B tiles of this many tokens");
static_assert(kTcTokens == kTcTokensB, "the prefill attention writes B tiles of this many tokens");
constexpr int kTcEpiThreads = 256;    // warps 8..15
constexpr int kTcUnpack = 192;        // warps 2..7
constexpr int kTcEpiWarp0 = 8;

// Original row of tensor-core row p when the layout interleaves gate / up
// (perm_F = F; 0 = no interleave).
__host__ __device__ inline int tc_row_orig(int p, int perm_F) {
  if (!perm_F) return p;
  const int rt = p / kTcRows, r = p % kTcRows;
  return r < kTcRows / 2 ? rt * (kTcRows / 2) + r : perm_F + rt * (kTcRows / 2) + r - kTcRows / 2;
}

// silu(gate) * up of token `tl_` (within token tile tt) and interleaved pair
// column j of row tile `tile`, pairs (j, j+1), as hi/lo fp16 into the down
// projection's B tile (K index 64 tile + j).
__device__ __forceinline__ void tc_swiglu_store(uint8_t* bt, int groups, int tt, int tile, int tl_, int j, float g0,
                                                float g1, float u0, float u1) {
  const float h0 = silu(g0) * u0, h1 = silu(g1) * u1;
  uint32_t hw, lw;
  const __half2 hh = __floats2half2_rn(h0, h1);
  const float2 rr = __half22float2(hh);
  const __half2 ll = __floats2half2_rn(h0 - rr.x, h1 - rr.y);
  hw = *reinterpret_cast<const uint32_t*>(&hh);
  lw = *reinterpret_cast<const uint32_t*>(&ll);
  const int k = tile * 64 + j, grp = k >> 7, kg = k & 127;
  uint8_t* blk = bt + ((size_t)tt * groups + grp) * (2 * 128 * 256);
  *reinterpret_cast<uint32_t*>(blk + sw128_offset(tl_, kg, 256)) = hw;
  *reinterpret_cast<uint32_t*>(blk + sw128_offset(128 + tl_, kg, 256)) = lw;
}


constexpr int kTcStages = 4;          // half-group (64 k) operand stages
constexpr int kTcRaw = 3;             // raw INT4 group stages
// Tensor-core weight layout, one block per (128-row tile, K group): 128 rows
// x 16 words of 8 nibbles (k = 8j .. 8j + 7 of the group, in the order
// k0 k2 k4 k6 at bits 0, 4, 8, 12 and k1 k3 k5 k7 at bits 16, 20, 24, 28, so
// that the 1024-bias unpacking yields the pairs (k0, k1) .. (k6, k7) in
// order), then 128 fp16 biased zeros 1024 + z.  Rows >= N are zero.
constexpr int kTcRawBytes = kTcRows * 64 + kTcRows * 2;   // 8448 B

__host__ __device__ inline int tc_nb(bool lo) { return lo ? 2 * kTcTokens : kTcTokens; }  // B rows (MMA N)
__host__ __device__ inline size_t tc_b_bytes(bool lo) { return (size_t)tc_nb(lo) * 256; }      // B of one group: 64 / 32 KB
// Stage = one 64-wide K atom: A 128 rows x 128 B (16 KB), B NB rows x 128 B.
__host__ __device__ inline size_t tc_smem_bytes(bool lo) {
  return (size_t)kTcStages * ((size_t)kTcRows * 128 + (size_t)tc_nb(lo) * 128) + (size_t)kTcRaw * kTcRawBytes + 1024;
}

struct TcGemmArgs {
  const uint8_t* wtc;    // INT4 weights in the tensor-core layout [N/128][K/128][kTcRawBytes]
  const uint2* sz;       // scales / biased zeros [n16 tiles][K/128][8] (GEMV layout; the epilogue's scales)
  int K, N;
  int n16_tiles;         // 16-row tiles present in w (rows beyond N are zero)
  const uint8_t* bt;     // prepared activations [token tiles][K/128][2 atoms][NB rows][128 B]
  int T;                 // tokens
  int splits;
  // outputs
  float* out_f32;        // TC_RESID (+=) / TC_RAW (=): [T][ld_out]
  __half* out_f16;       // TC_STORE: [T][ld_out]
  int ld_out;
  // TC_ROPE_KV
  float* q_out;          // [T][ldq] rotated queries
  int ldq;
  int n_q_rows, n_kv_rows, hd;
  __half* k_plane;       // K plane [Hkv][ctx][hd] of this lane and layer
  __half* v_plane;
  float* kv_stage;       // INT8 KV cache: rotated keys / values in fp32 at
                         // [token][K|V][Hkv][hd] for the quantising pass
                         // instead of the planes; NULL: fp16 cache
  int ctx, pos0;
  float theta;
  const float2* rope_tab;  // (cos, sin) [positions][hd/2], or NULL
  // split-K
  // TC_SWIGLU_B
  int perm_F;            // interleaved gate/up rows (the scales are looked up by original row)
  uint8_t* bt_out;       // the down projection's B tiles
  int bt_out_groups;     // its K / 128
  // RMSNorm hand-off between consecutive GEMMs (prefill).  Producer side
  // (TC_RESID): besides the residual, write the next GEMM's B tiles of
  // x * g_next (fp16 hi / lo) and, per token, this row tile's sum of x^2.
  uint8_t* bt_next;      // [token tiles][K/128][2 atoms][256 rows][128 B], K = N of this GEMM
  const __half* g_next;  // [N] gains of the next RMSNorm
  float* ss_out;         // [row tiles][ss_ld] sums of squares
  // Consumer side: every output of token t is scaled by
  // rsqrt(sum_p ss_in[p][t] / ss_k + eps) (the RMSNorm of its B rows).
  const float* ss_in;    // [ss_parts][ss_ld], or NULL
  int ss_parts, ss_ld;
  float ss_k, ss_eps;
  int cluster;           // 1: the splits of a tile form a thread-block cluster and
                         // reduce in distributed shared memory (no partial buffer)
  float* partial;        // [splits][row tiles][token tiles][128 tokens][128 rows]
  unsigned* tickets;     // [row tiles][token tiles], zero between launches
  int* err_flag;
};

// Key (kv = 0) or value elements j and j + hd/2 of kv head kvh for token t
// (position pos): fp16 into the cache plane, or fp32 into the INT8 mode's
// staging buffer.
__device__ __forceinline__ void tc_kv_store(const TcGemmArgs& a, int t, int kv, int kvh, int pos, int j, float e0,
                                            float e1) {
  const int hd = a.hd;
  if (a.kv_stage) {
    float* dst = a.kv_stage + ((size_t)(t * 2 + kv) * (a.n_kv_rows / hd) + kvh) * hd;
    dst[j] = e0;
    dst[j + hd / 2] = e1;
  } else {
    __half* dst = (kv ? a.v_plane : a.k_plane) + ((size_t)kvh * a.ctx + pos) * hd;
    dst[j] = __float2half_rn(e0);
    dst[j + hd / 2] = __float2half_rn(e1);
  }
}

// Final epilogue of `ntok` tokens of token tile tt (tile-local tokens tok0 ..
// tok0 + ntok - 1) of row tile `tile`, whose sums are xch[ntok][kTcRows] in
// shared memory; threads tid = 0 .. nthr - 1 share the work.
// rs_tok: per tile-local token factor applied to every value first (the
// consumer side of the RMSNorm hand-off), or NULL.
template <int EPI>
__device__ void tc_epilogue_tokens(const TcGemmArgs& a, const float* xch, int tile, int tt, int tok0, int ntok,
                                   int tid, int nthr, const float* rs_tok = nullptr) {
  if (EPI == TC_RESID && a.bt_next) {
    // one warp per token: the new residual of the tile's 128 rows, the next
    // GEMM's B tile entries of x * g_next and the token's sum of x^2 here
    const int warp = tid >> 5, lane = tid & 31, nw = nthr >> 5;
    const int grp = tile;   // this row tile is one K group of the next GEMM
    for (int ti = warp; ti < ntok; ti += nw) {
      const int tl_ = tok0 + ti, t = tt * kTcTokens + tl_;
      if (t >= a.T) continue;   // warp-uniform
      const float f = rs_tok ? rs_tok[tl_] : 1.f;
      float ss = 0.f;
      uint8_t* blk = a.bt_next + ((size_t)tt * (a.N / kTcRows) + grp) * (2 * kTcTokens * 256);
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {
        const int r = (lane + 32 * pr) * 2;   // rows r, r + 1
        const int n = tile * kTcRows + r;
        float2* xo = reinterpret_cast<float2*>(a.out_f32 + (size_t)t * a.ld_out + n);
        float2 xv = *xo;
        xv.x += xch[ti * kTcRows + r] * f;
        xv.y += xch[ti * kTcRows + r + 1] * f;
        *xo = xv;
        ss += xv.x * xv.x + xv.y * xv.y;
        const float2 gv = __half22float2(*reinterpret_cast<const __half2*>(a.g_next + n));
        uint32_t hw, lw;
        split_h2(xv.x * gv.x, xv.y * gv.y, hw, lw);
        *reinterpret_cast<uint32_t*>(blk + sw128_offset(tl_, r, 2 * kTcTokens)) = hw;
        *reinterpret_cast<uint32_t*>(blk + sw128_offset(kTcTokens + tl_, r, 2 * kTcTokens)) = lw;
      }
      ss = warp_sum(ss);
      if (lane == 0) a.ss_out[(size_t)tile * a.ss_ld + t] = ss;
    }
    return;
  }
  if (EPI == TC_RESID || EPI == TC_RAW || EPI == TC_STORE) {
    for (int item = tid; item < ntok * kTcRows; item += nthr) {
      const int ti = item / kTcRows, r = item % kTcRows;
      const int t = tt * kTcTokens + tok0 + ti, n = tile * kTcRows + r;
      if (t >= a.T || n >= a.N) continue;
      const float v = xch[ti * kTcRows + r] * (rs_tok ? rs_tok[tok0 + ti] : 1.f);
      const size_t o = (size_t)t * a.ld_out + n;
      if (EPI == TC_RESID) a.out_f32[o] += v;
      else if (EPI == TC_RAW) a.out_f32[o] = v;
      else a.out_f16[o] = __float2half_rn(v);
    }
  } else if (EPI == TC_SWIGLU_B) {
    for (int item = tid; item < ntok * 32; item += nthr) {
      const int ti = item >> 5, j = (item & 31) * 2;
      const int tq = tok0 + ti;
      if (tt * kTcTokens + tq >= a.T) continue;
      const float* xr = xch + ti * kTcRows;
      const float f = rs_tok ? rs_tok[tq] : 1.f;
      tc_swiglu_store(a.bt_out, a.bt_out_groups, tt, tile, tq, j, xr[j] * f, xr[j + 1] * f, xr[64 + j] * f,
                      xr[65 + j] * f);
    }
  } else {
    const int hd = a.hd, hh = hd / 2;
    const int pairs = kTcRows / 2;
    for (int item = tid; item < ntok * pairs; item += nthr) {
      const int ti = item / pairs, pr = item % pairs;
      const int head_local = pr / hh, j = pr % hh;
      const int r_a = head_local * hd + j, r_b = r_a + hh;
      const int t = tt * kTcTokens + tok0 + ti;
      const int na = tile * kTcRows + r_a;
      if (t >= a.T || na >= a.N) continue;
      const float f = rs_tok ? rs_tok[tok0 + ti] : 1.f;
      const float va = xch[ti * kTcRows + r_a] * f, vb = xch[ti * kTcRows + r_b] * f;
      const int pos = a.pos0 + t;
      if (na < a.n_q_rows) {
        const float2 cs = rope_cs(a.rope_tab, pos, j, hd, a.theta);
        float* qo = a.q_out + (size_t)t * a.ldq;
        qo[na] = va * cs.x - vb * cs.y;
        qo[na + hh] = vb * cs.x + va * cs.y;
      } else if (na < a.n_q_rows + a.n_kv_rows) {
        const float2 cs = rope_cs(a.rope_tab, pos, j, hd, a.theta);
        const int kvh = (na - a.n_q_rows) / hd;
        tc_kv_store(a, t, 0, kvh, pos, j, va * cs.x - vb * cs.y, vb * cs.x + va * cs.y);
      } else {
        const int kvh = (na - a.n_q_rows - a.n_kv_rows) / hd;
        tc_kv_store(a, t, 1, kvh, pos, j, va, vb);
      }
    }
  }
}

// Consumer side of the RMSNorm hand-off: rs[i] for the tile-local tokens
// i = tid, tid + nthr, ... of token tile tt (1 where no sums are given).
__device__ __forceinline__ void tc_token_scales(const TcGemmArgs& a, int tt, float* rs, int tid, int nthr) {
  for (int i = tid; i < kTcTokens; i += nthr) {
    float f = 1.f;
    const int t = tt * kTcTokens + i;
    if (a.ss_in && t < a.T) {
      float tot = 0.f;
      for (int p = 0; p < a.ss_parts; ++p) tot += a.ss_in[(size_t)p * a.ss_ld + t];
      f = 1.0f / sqrtf(tot / a.ss_k + a.ss_eps);
    }
    rs[i] = f;
  }
}

// Split-K reduction inside the thread-block cluster that holds the splits of
// one (row tile, token tile): each rank's partial tile P [128 tokens][128
// rows] fp32 sits at the start of its shared memory; rank r sums tokens
// [r * 128 / S, (r + 1) * 128 / S) over the ranks in rank (= split) order --
// deterministic -- into a slice buffer behind P and applies the epilogue.
// Called by all threads of every CTA of the cluster.
template <int EPI>
__device__ void tc_cluster_reduce(const TcGemmArgs& a, unsigned char* smem, int tile, int tt, const float* rs_tok) {
  const int S = a.splits;
  cluster_sync_all();   // every rank's partial tile is complete
  const int r = (int)cluster_rank();
  const int tok0 = r * kTcTokens / S, ntok = (r + 1) * kTcTokens / S - tok0;
  const float* P = reinterpret_cast<const float*>(smem);
  float* xs = reinterpret_cast<float*>(smem + (size_t)kTcTokens * kTcRows * 4);   // [ntok][kTcRows]
  for (int item = threadIdx.x; item < ntok * (kTcRows / 4); item += kTcThreads) {
    const int ti = item / (kTcRows / 4), r4 = (item % (kTcRows / 4)) * 4;
    const float* src = P + (size_t)(tok0 + ti) * kTcRows + r4;
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < S; s0 += 8) {
      float4 v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (s0 + i < S) v[i] = ld_cluster_f4(cluster_map(src, (unsigned)(s0 + i)));
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (s0 + i < S) { sum.x += v[i].x; sum.y += v[i].y; sum.z += v[i].z; sum.w += v[i].w; }
    }
    *reinterpret_cast<float4*>(xs + ti * kTcRows + r4) = sum;
  }
  __syncthreads();
  tc_epilogue_tokens<EPI>(a, xs, tile, tt, tok0, ntok, threadIdx.x, kTcThreads, rs_tok);
  cluster_sync_all();   // no rank leaves while another still reads its partial tile
}

template <int EPI, bool LO>
__global__ void __launch_bounds__(kTcThreads, 1) gemm_int4_tc_kernel(const TcGemmArgs a) {
  constexpr int NB = LO ? 2 * kTcTokens : kTcTokens;
  constexpr uint32_t NCOL = NB;                    // TMEM columns per buffer
  constexpr uint32_t A_BYTES = kTcRows * 128;      // one 64-k atom of A
  constexpr uint32_t B_BYTES = NB * 128;           // one 64-k atom of B
  extern __shared__ __align__(128) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  auto sA = [&](int st) { return smem + st * A_BYTES; };
  auto sB = [&](int st) { return smem + kTcStages * A_BYTES + st * B_BYTES; };
  auto sR = [&](int r) { return smem + kTcStages * (A_BYTES + B_BYTES) + r * kTcRawBytes; };
  __shared__ __align__(8) uint64_t bar_full[kTcStages], bar_empty[kTcStages], bar_tfull[2], bar_tempty[2];
  __shared__ __align__(8) uint64_t raw_full[kTcRaw], raw_empty[kTcRaw];
  __shared__ uint32_t s_tmem;
  __shared__ int s_last;
  __shared__ int s_fail;
  __shared__ float s_rs[kTcTokens];   // per-token factor (RMSNorm hand-off), 1 without it

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, tt = blockIdx.y, split = blockIdx.z;
  const int G = a.K >> 7;
  const int g_begin = split * G / a.splits, g_end = (split + 1) * G / a.splits;
  const int ng = g_end - g_begin;
  const int nh = 2 * ng;                             // half-group steps
  const int row_tiles = gridDim.x, tok_tiles = gridDim.y;
  // CTAs walk their K groups from different starting points so that they do
  // not all fetch the same activation atom at the same time (the epilogue
  // adds the groups in this fixed order: deterministic)
  const int rot = ng > 0 ? tile % ng : 0;
  auto gmap = [&](int it) { return g_begin + (it + rot) % ng; };

  if (warp == 0) {
    tmem_alloc(&s_tmem, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    for (int i = 0; i < kTcStages; ++i) {
      mbar_init(&bar_full[i], kTcUnpack + 1);   // + the copy lane's arrive with the B bytes
      mbar_init(&bar_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_tfull[i], 1);
      mbar_init(&bar_tempty[i], kTcEpiThreads);
    }
    for (int i = 0; i < kTcRaw; ++i) {
      mbar_init(&raw_full[i], 1);
      mbar_init(&raw_empty[i], kTcUnpack);
    }
    fence_mbar_init();
    s_fail = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  pdl_trigger();

  if (warp == 0) {
    pdl_wait();
    // ---- MMA issue: 4 k16 steps per 64-k stage, a group = 2 stages into one
    // TMEM buffer (double-buffered across groups) ----------------------------
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(kTcRows, NB);
      for (int h = 0; h < nh; ++h) {
        const int s = h % kTcStages, it = h >> 1, half = h & 1, b = it & 1;
        if (!mbar_wait_or_fail(&bar_full[s], (unsigned)(h / kTcStages) & 1u, &s_fail)) break;
        if (half == 0 && it >= 2 && !mbar_wait_or_fail(&bar_tempty[b], (unsigned)((it - 2) >> 1) & 1u, &s_fail))
          break;
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t ad = sw128_kmajor_desc(sA(s) + j * 32);
          const uint64_t bd = sw128_kmajor_desc(sB(s) + j * 32);
          tc_mma_f16(tmem + b * NCOL, ad, bd, idesc, (half | j) ? 1u : 0u);
        }
        tc_commit(&bar_empty[s]);
        if (half) tc_commit(&bar_tfull[b]);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---- copy issuer (one lane) ----------------------------------------------
    // Keeps kTcRaw groups of raw INT4 words and scales/zeros in flight (bulk
    // copies; the weights do not depend on earlier kernels, so the first ones
    // go out before the dependency wait) and issues each stage's B atom as
    // soon as the MMA has released the stage.
    if (lane == 0) {
      int g_issued = 0;
      auto issue_raw = [&](int it) {
        const int r = it % kTcRaw, g = gmap(it);
        mbar_arrive_expect_tx(&raw_full[r], kTcRawBytes);
        bulk_g2s(sR(r), a.wtc + ((size_t)tile * G + g) * kTcRawBytes, kTcRawBytes, &raw_full[r]);
      };
      for (; g_issued < ng && g_issued < kTcRaw; ++g_issued) issue_raw(g_issued);
      pdl_wait();
      for (int h = 0; h < nh; ++h) {
        const int s = h % kTcStages, it = h >> 1, half = h & 1, g = gmap(it);
        if (h >= kTcStages && !mbar_wait_or_fail(&bar_empty[s], (unsigned)((h / kTcStages) - 1) & 1u, &s_fail))
          break;
        // arrive with the expected bytes: the stage cannot complete before
        // this arrival, so the unpackers' arrivals cannot race past the copy
        mbar_arrive_expect_tx(&bar_full[s], B_BYTES);
        bulk_g2s(sB(s), a.bt + (((size_t)tt * G + g) * 2 + half) * B_BYTES, B_BYTES, &bar_full[s]);
        if (half) {
          // top up the raw ring: group g_issued reuses the slot of g_issued - kTcRaw
          for (; g_issued < ng && g_issued < it + kTcRaw; ++g_issued)
            if (mbar_wait_or_fail(&raw_empty[g_issued % kTcRaw], (unsigned)((g_issued / kTcRaw) - 1) & 1u,
                                  &s_fail))
              issue_raw(g_issued);
        }
      }
      // a CTA that gave up waits (bounded) for its raw copies still in flight
      if (*reinterpret_cast<volatile int*>(&s_fail))
        for (int it = g_issued - kTcRaw < 0 ? 0 : g_issued - kTcRaw; it < g_issued; ++it)
          mbar_wait(&raw_full[it % kTcRaw], (unsigned)(it / kTcRaw) & 1u);
    }
    __syncwarp();
  } else if (warp < kTcEpiWarp0) {
    // ---- unpackers: A from the raw ring into the 128-byte swizzled K-major
    // layout the MMA descriptor reads --------------------------------------------
    const int p = threadIdx.x - 64;
    for (int h = 0; h < nh; ++h) {
      const int s = h % kTcStages, it = h >> 1, half = h & 1, r = it % kTcRaw;
      if (h >= kTcStages && !mbar_wait_or_fail(&bar_empty[s], (unsigned)((h / kTcStages) - 1) & 1u, &s_fail))
        break;
      if (!mbar_wait_or_fail(&raw_full[r], (unsigned)(it / kTcRaw) & 1u, &s_fail)) break;
      const unsigned char* raw = sR(r);
      unsigned char* A = sA(s);
      // item = (row, 4 consecutive 8-k chunks of this 64-k atom): one 16-byte
      // load of 32 nibbles, four 16-byte stores of exact fp16 q - z
      for (int wi = p; wi < 2 * kTcRows; wi += kTcUnpack) {
        const int row = wi >> 1, qd = wi & 1;
        const uint4 wv = *reinterpret_cast<const uint4*>(raw + row * 64 + (half * 8 + qd * 4) * 4);
        const uint32_t zb = *reinterpret_cast<const uint16_t*>(raw + kTcRows * 64 + row * 2);
        const uint32_t zz = zb | (zb << 16);
        const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t w = words[i];
          uint4 o;
          o.x = h2_sub(nib_pair_to_h2_biased(w), zz);
          o.y = h2_sub(nib_pair_to_h2_biased(w >> 4), zz);
          o.z = h2_sub(nib_pair_to_h2_biased(w >> 8), zz);
          o.w = h2_sub(nib_pair_to_h2_biased(w >> 12), zz);
          const int c = qd * 4 + i;   // 16-byte chunk (8 k) within the 128-byte row
          *reinterpret_cast<uint4*>(A + row * 128 + ((c ^ (row & 7)) << 4)) = o;
        }
      }
      if (half) mbar_arrive(&raw_empty[r]);
      fence_proxy_async_smem();
      mbar_arrive(&bar_full[s]);
    }
  } else {
    // ---- epilogue: accumulate s * (P_hi + P_lo) per group --------------
    pdl_wait();   // it reads / writes what earlier kernels wrote
    const int e = warp - kTcEpiWarp0;
    const int quad = warp & 3;                 // TMEM lanes this warp may access
    const int half = e >> 2;                   // tokens [64 half, 64 half + 64)
    const int row = quad * 32 + lane;          // weight row within the tile
    const int orow = tc_row_orig(tile * kTcRows + row, a.perm_F);   // row in the GEMV layout
    const int gt = orow >> 4;
    const bool row_ok = gt < a.n16_tiles;
    float acc[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) acc[i] = 0.f;
    auto scale_of = [&](int g) -> float {
      if (!row_ok) return 0.f;
      const uint32_t sp = __ldg(&a.sz[((size_t)gt * G + g) * 8 + (orow & 7)]).x;
      const float2 f = h2_to_f2(sp);
      return (orow & 8) ? f.y : f.x;
    };
    float s_next = ng > 0 ? scale_of(gmap(0)) : 0.f;
    for (int it = 0; it < ng; ++it) {
      const int b = it & 1;
      const float sc = s_next;
      if (it + 1 < ng) s_next = scale_of(gmap(it + 1));
      // on a time-out the loop keeps its shape (no further waits) so the
      // epilogue barriers below still match across the epilogue warps
      mbar_wait_or_fail(&bar_tfull[b], (it >> 1) & 1, &s_fail);
      tc_fence_after();
      const uint32_t base = tmem + ((uint32_t)(quad * 32) << 16) + b * NCOL + half * 64;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t hi[16];
        tmem_ld16(base + c * 16, hi);
        if (LO) {
          uint32_t lo[16];
          tmem_ld16(base + kTcTokens + c * 16, lo);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            acc[c * 16 + i] = fmaf(sc, __uint_as_float(hi[i]) + __uint_as_float(lo[i]), acc[c * 16 + i]);
        } else {
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) acc[c * 16 + i] = fmaf(sc, __uint_as_float(hi[i]), acc[c * 16 + i]);
        }
      }
      tc_fence_before();
      mbar_arrive(&bar_tempty[b]);
    }

    // ---- split-K: partial sums to scratch, merged by tc_merge_kernel --------
    const int n = tile * kTcRows + row;
    const int t0 = tt * kTcTokens + half * 64;
    const int etid = threadIdx.x - kTcEpiWarp0 * 32;
    tc_token_scales(a, tt, s_rs, etid, kTcEpiThreads);
    epi_sync(kTcEpiThreads);
    const bool failed = s_fail != 0;
    // the direct epilogue below writes from registers; the hand-off needs
    // whole token rows, so it goes through shared memory like RoPE / SwiGLU
    const bool via_smem = a.bt_next || a.ss_in;
    if (a.splits > 1 && a.cluster) {
      // partial tile into this CTA's shared memory (the operand stages are
      // idle: the last MMA has completed), reduced across the cluster below
      float* P = reinterpret_cast<float*>(smem);   // [128 tokens][128 rows]
#pragma unroll
      for (int i = 0; i < 64; ++i) P[(half * 64 + i) * kTcRows + row] = acc[i];
      if (e == 0 && lane == 0) s_last = 0;
    } else if (a.splits > 1) {
      float* mine = a.partial + (((size_t)split * row_tiles + tile) * tok_tiles + tt) * (kTcTokens * kTcRows);
#pragma unroll
      for (int i = 0; i < 64; ++i) mine[(size_t)(half * 64 + i) * kTcRows + row] = acc[i];
      if (e == 0 && lane == 0) s_last = 0;
    } else {
      if (e == 0 && lane == 0) s_last = 1;
    }
    epi_sync(kTcEpiThreads);

    // ---- final epilogue -----------------------------------------------------
    if (!failed && s_last && via_smem) {
      float* xch = reinterpret_cast<float*>(smem);   // [128 tokens][128 rows]
#pragma unroll
      for (int i = 0; i < 64; ++i) xch[(half * 64 + i) * kTcRows + row] = acc[i];
      epi_sync(kTcEpiThreads);
      tc_epilogue_tokens<EPI>(a, xch, tile, tt, 0, kTcTokens, etid, kTcEpiThreads, s_rs);
    } else if (!failed && s_last) {
      if (EPI == TC_RESID || EPI == TC_RAW || EPI == TC_STORE) {
        if (n < a.N) {
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const int t = t0 + i;
            if (t < a.T) {
              const size_t o = (size_t)t * a.ld_out + n;
              if (EPI == TC_RESID) a.out_f32[o] += acc[i];
              else if (EPI == TC_RAW) a.out_f32[o] = acc[i];
              else a.out_f16[o] = __float2half_rn(acc[i]);
            }
          }
        }
      } else if (EPI == TC_SWIGLU_B) {
        // gate rows 0..63 and up rows 64..127 of the tile: exchange through
        // shared memory, then write pairs of SwiGLU outputs
        float* xch = reinterpret_cast<float*>(smem);   // [128 tokens][128 rows]
#pragma unroll
        for (int i = 0; i < 64; ++i) xch[(half * 64 + i) * kTcRows + row] = acc[i];
        epi_sync(kTcEpiThreads);
        for (int item = threadIdx.x - kTcEpiWarp0 * 32; item < kTcTokens * 32; item += kTcEpiThreads) {
          const int tl_ = item >> 5, j = (item & 31) * 2;
          if (tt * kTcTokens + tl_ >= a.T) continue;
          const float* xr = xch + tl_ * kTcRows;
          tc_swiglu_store(a.bt_out, a.bt_out_groups, tt, tile, tl_, j, xr[j], xr[j + 1], xr[64 + j], xr[65 + j]);
        }
      } else {
        // RoPE pairs (j, j + hd/2) sit in different rows of the tile: exchange
        // through shared memory (the stages are idle now).
        float* xch = reinterpret_cast<float*>(smem);   // [128 tokens][128 rows]
#pragma unroll
        for (int i = 0; i < 64; ++i) xch[(half * 64 + i) * kTcRows + row] = acc[i];
        epi_sync(kTcEpiThreads);
        const int hd = a.hd, hh = hd / 2;
        const int pairs_per_tok = kTcRows / 2;         // 64 (j < hd/2 of each head in the tile)
        for (int item = threadIdx.x - kTcEpiWarp0 * 32; item < kTcTokens * pairs_per_tok; item += kTcEpiThreads) {
          const int tl_ = item / pairs_per_tok, pr = item % pairs_per_tok;
          const int head_local = pr / hh, j = pr % hh;
          const int r_a = head_local * hd + j, r_b = r_a + hh;
          const int t = tt * kTcTokens + tl_;
          const int na = tile * kTcRows + r_a;
          if (t >= a.T || na >= a.N) continue;
          const float va = xch[tl_ * kTcRows + r_a], vb = xch[tl_ * kTcRows + r_b];
          const int pos = a.pos0 + t;
          if (na < a.n_q_rows) {
            const float2 cs = rope_cs(a.rope_tab, pos, j, hd, a.theta);
            float* qo = a.q_out + (size_t)t * a.ldq;
            qo[na] = va * cs.x - vb * cs.y;
            qo[na + hh] = vb * cs.x + va * cs.y;
          } else if (na < a.n_q_rows + a.n_kv_rows) {
            const float2 cs = rope_cs(a.rope_tab, pos, j, hd, a.theta);
            const int kvh = (na - a.n_q_rows) / hd;
            tc_kv_store(a, t, 0, kvh, pos, j, va * cs.x - vb * cs.y, vb * cs.x + va * cs.y);
          } else {
            const int kvh = (na - a.n_q_rows - a.n_kv_rows) / hd;
            tc_kv_store(a, t, 1, kvh, pos, j, va, vb);
          }
        }
      }
    }
    if (failed && e == 0 && lane == 0) atomicOr(a.err_flag, kErrTimeout);
  }

  // ---- teardown: every role reaches here; TMEM is always freed -----------
  tc_fence_before();
  __syncthreads();
  if (a.splits > 1 && a.cluster) tc_cluster_reduce<EPI>(a, smem, tile, tt, s_rs);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---- load-time re-layout for the tensor-core path -------------------------------
// One thread per 8-nibble word (and, for j == 0, the row's biased zero) of
// the tensor-core layout, from the storage format (qweight [N][K/8] words,
// element k in bits 4 (k % 8); qzeros [N][ceil(G/8)] words).  perm_F != 0
// interleaves gate and up rows per 128-row tile (see tc_row_orig).
// bits = 2: the INT2 body's storage (element k in bits 2 (k % 16) of word
// k / 16, 16 zero points per word), widened to the same nibble layout.
__global__ void repack_int4_tc_kernel(const uint32_t* __restrict__ qweight, const uint32_t* __restrict__ qzeros,
                                      int K, int N, int perm_F, uint8_t* __restrict__ out, int bits) {
  const int G = K >> 7, zw = bits == 2 ? (G + 15) >> 4 : (G + 7) >> 3;
  const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int row_tiles = (N + kTcRows - 1) / kTcRows;
  const size_t total = (size_t)row_tiles * G * kTcRows * 16;
  if (idx >= total) return;
  const int j = (int)(idx & 15);
  const int r = (int)((idx >> 4) % kTcRows);
  const size_t blk = (idx >> 4) / kTcRows;          // rt * G + g
  const int g = (int)(blk % G), rt = (int)(blk / G);
  const int n = tc_row_orig(rt * kTcRows + r, perm_F);
  uint8_t* base = out + blk * kTcRawBytes;
  uint32_t word = 0, z = 0;
  if (n < N) {
    // k = 128 g + 8 j + i; destination nibble slot of k_i: i even -> 4 (i / 2),
    // i odd -> 16 + 4 (i / 2)
    if (bits == 2) {
      const uint32_t src = qweight[(size_t)n * (K >> 4) + g * 8 + (j >> 1)];   // k_i at bits 2 (8 (j & 1) + i)
#pragma unroll
      for (int i = 0; i < 8; ++i)
        word |= ((src >> (2 * (8 * (j & 1) + i))) & 0x3u) << ((i & 1) * 16 + 4 * (i >> 1));
      z = (qzeros[(size_t)n * zw + (g >> 4)] >> (2 * (g & 15))) & 0x3u;
    } else {
      const uint32_t src = qweight[(size_t)n * (K >> 3) + g * 16 + j];   // k_i at bits 4 i
#pragma unroll
      for (int i = 0; i < 8; ++i) word |= ((src >> (4 * i)) & 0xFu) << ((i & 1) * 16 + 4 * (i >> 1));
      z = (qzeros[(size_t)n * zw + (g >> 3)] >> (4 * (g & 7))) & 0xFu;
    }
  }
  reinterpret_cast<uint32_t*>(base)[r * 16 + j] = word;
  if (j == 0) reinterpret_cast<uint16_t*>(base + kTcRows * 64)[r] = (uint16_t)(0x6400u + z);
}

// ---- split-K merge + epilogue ------------------------------------------------
// One CTA per (row tile, token tile, 8-token slice): sums the split partials
// of its 8 x 128 outputs in split order (all loads of a batch of 8 splits in
// flight), then applies the GEMM's epilogue.  Deterministic; the partials
// are [split][row tile][token tile][128 tokens][128 rows].
constexpr int kTcMergeTok = 8;
template <int EPI>
__global__ void __launch_bounds__(256) tc_merge_kernel(const TcGemmArgs a) {
  __shared__ __align__(16) float xch[kTcMergeTok][kTcRows];
  __shared__ float s_rs[kTcTokens];
  const int tile = blockIdx.x, tt = blockIdx.y, slice = blockIdx.z;
  const int row_tiles = gridDim.x, tok_tiles = gridDim.y;
  const int tl_ = threadIdx.x >> 5, r4 = (threadIdx.x & 31) * 4;   // token in the slice, 4 rows
  const int tok = slice * kTcMergeTok + tl_;                       // token within the tile
  pdl_trigger();
  pdl_wait();
  tc_token_scales(a, tt, s_rs, threadIdx.x, 256);
  float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
  const size_t split_stride = (size_t)row_tiles * tok_tiles * kTcTokens * kTcRows;
  const float* base = a.partial + ((size_t)tile * tok_tiles + tt) * (kTcTokens * kTcRows) + (size_t)tok * kTcRows + r4;
  for (int sp0 = 0; sp0 < a.splits; sp0 += 8) {
    float4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      v[i] = sp0 + i < a.splits ? __ldcg(reinterpret_cast<const float4*>(base + (size_t)(sp0 + i) * split_stride))
                                : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (sp0 + i < a.splits) {
        sum.x += v[i].x; sum.y += v[i].y; sum.z += v[i].z; sum.w += v[i].w;
      }
    }
  }
  *reinterpret_cast<float4*>(&xch[tl_][r4]) = sum;
  __syncthreads();
  tc_epilogue_tokens<EPI>(a, &xch[0][0], tile, tt, slice * kTcMergeTok, kTcMergeTok, threadIdx.x, 256, s_rs);
}

// ---- activation preparation ---------------------------------------------
// B tile of token tile tt and K group g: rows 0..127 = fp16 hi of the tokens,
// rows 128..255 = fp16 lo (when LO), each row 128 k in two 64-wide atoms,
// 128-byte swizzled; tokens >= T are zero.
// PREP_NONE: the B tiles were written by the producing kernel (the prefill
// attention writes the O projection's, the gate_up epilogue the down
// projection's).
enum PrepMode { PREP_NORM = 0, PREP_F16 = 3, PREP_NONE = 4 };

struct PrepArgs {
  const float* x;        // PREP_NORM: fp32 [T][ldx]
  const __half* xh;      // PREP_F16: fp16 [T][ldx]
  int ldx;
  const __half* gain;    // PREP_NORM
  float eps;
  int K, T;
  uint8_t* bt;
};

template <int MODE>
__global__ void __launch_bounds__(256) prep_b_kernel(const PrepArgs a) {
  constexpr bool LO = MODE != PREP_F16;
  constexpr int NB = LO ? 2 * kTcTokens : kTcTokens;
  __shared__ float s_ss[8];
  const int tok = blockIdx.x;                    // token index, padded to whole tiles
  const int tt = tok / kTcTokens, tl_ = tok % kTcTokens;
  const int G = a.K >> 7;
  const bool valid = tok < a.T;
  pdl_trigger();
  pdl_wait();
  float rs = 1.f;
  if (MODE == PREP_NORM && valid) {
    const float* src = a.x + (size_t)tok * a.ldx;
    float ss = 0.f;
    for (int k = threadIdx.x * 4; k < a.K; k += 1024) {
      const float4 v = *reinterpret_cast<const float4*>(src + k);
      ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) s_ss[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) tot += s_ss[w];
    rs = 1.0f / sqrtf(tot / (float)a.K + a.eps);
  }
  for (int c8 = threadIdx.x; c8 < a.K / 8; c8 += 256) {
    const int k = c8 * 8;
    float v[8];
    if (!valid) {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.f;
    } else if (MODE == PREP_F16) {
      const uint4 raw = *reinterpret_cast<const uint4*>(a.xh + (size_t)tok * a.ldx + k);
      const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = h2_to_f2(w4[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
      }
    } else {
      const float* src = a.x + (size_t)tok * a.ldx;
      const float4 x0 = *reinterpret_cast<const float4*>(src + k), x1 = *reinterpret_cast<const float4*>(src + k + 4);
      v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w; v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
      if (MODE == PREP_NORM) {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = (v[i] * rs) * __half2float(a.gain[k + i]);
      }
    }
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2 h = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
      const float2 r = __half22float2(h);
      const __half2 l = __floats2half2_rn(v[2 * i] - r.x, v[2 * i + 1] - r.y);
      hw[i] = *reinterpret_cast<const uint32_t*>(&h);
      lw[i] = *reinterpret_cast<const uint32_t*>(&l);
    }
    const int g = k >> 7, kg = k & 127;
    uint8_t* blk = a.bt + ((size_t)tt * G + g) * (NB * 256);
    *reinterpret_cast<uint4*>(blk + sw128_offset(tl_, kg, NB)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    if (LO)
      *reinterpret_cast<uint4*>(blk + sw128_offset(kTcTokens + tl_, kg, NB)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
}

}  // namespace tl
