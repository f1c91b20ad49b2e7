// Decode: RMSNorm + QKV INT4 linear + RoPE + KV write + GQA attention of one
// effective layer in ONE kernel, one thread-block cluster per kv head.
//
// What it computes is steps a2-a5 of a decode step (TinyLoop README,
// "Status": fused RMSNorm + RoPE, GQA with a per-layer KV cache): the same
// arithmetic as gemv_int4_kernel<.., IN_NORM, EPI_ROPE_KV> followed by
// decode_attn_kernel (exact integer q - z MMA operands with (hi, lo) fp16
// activations, fp32 scales and q, fp16 keys/values, fp32 softmax).
//
// Why a cluster: attention for kv head g needs exactly the QKV rows of its
// group (rep query heads, the key head and the value head: (rep + 2) hd
// rows).  A cluster of kQaCluster CTAs computes those rows, exchanges q and
// the new key/value through distributed shared memory, synchronises with the
// hardware cluster barrier and runs the attention over the lane's cache with
// the keys split across its CTAs.  Each rank sends its split's running max
// and weight sum to every rank and each slice of its weighted value sums to
// the rank that owns that slice of the head dimension, so after the second
// cluster barrier every rank merges hd / kQaCluster dimensions of every head.
// That removes a kernel boundary (and its global round trips) per layer.
//
// The lane's cached keys and values (positions before the new one) do not
// depend on this step: once the weights have landed, one thread bulk-copies
// the first chunk of the rank's key split into shared memory, and the copy
// runs under the GEMV and the first exchange.
//
// CTA c of cluster g: GEMV of the group's 16-row tiles c, c + kQaCluster, ...
// ((rep + 2) hd / 16 tiles, 3 per rank for 4 query heads of 128), weights
// bulk-copied into shared memory before the programmatic-launch wait; 8 warps
// split K, each warp's B fragments are loaded once per chunk and reused for
// every tile.  The raw projections go to every rank; RoPE (whose pairs j,
// j + hd/2 sit in different tiles, often on different ranks) is applied by
// every rank to its own copy after the exchange, and each rank writes its
// hd / kQaCluster elements of the new key and value to the cache.
#pragma once

#include "attention.cuh"
#include "common.cuh"
#include "kv8.cuh"

namespace tl {

constexpr int kQaCluster = 16;         // non-portable cluster size (B200 GPCs hold 16 CTAs of this size)
constexpr int kQaThreads = 256;
constexpr int kQaWarps = kQaThreads / 32;
constexpr int kQaMaxRows = 2;
constexpr int kQaMaxTiles = 4;        // 16-row QKV tiles per CTA
constexpr int kQaChunk = 64;          // keys per staged chunk
static_assert(kQaMaxTiles * 16 * kQaMaxRows <= kQaThreads, "one epilogue element per thread");
static_assert(kQaMaxRows * 8 * 8 <= kQaThreads, "one merged (row, head, dimension) per thread");

struct QkvAttnArgs {
  const uint4* w;        // QKV weights, GEMV tile layout [n16 tiles][K/64][32]
  const uint2* sz;       // [n16 tiles][K/128][8]
  int K;                 // d_model
  const float* x;        // residual stream [M][K]
  const __half* gain;    // attention RMSNorm gains
  float eps;
  int M;                 // rows (lanes), <= kQaMaxRows
  const RowCtx* rows;    // lane and position of each row
  int hd, rep, Hkv;
  const float2* rope_tab;
  float theta;
  __half* k_plane;       // this layer's K plane of lane 0 [Hkv][ctx][hd]
  __half* v_plane;       // (INT8 cache: int8 codes at the same element offsets)
  float* k_scale;        // INT8 cache: this layer's K / V scales of lane 0
  float* v_scale;        // [Hkv][ctx] (element offset / hd)
  long long lane_stride;
  int ctx;
  float* o;              // attention output [M][Hq*hd] fp32
  int l2_keep;           // 1: loop-block weights (L2 evict-last), else evict-first
  int* err_flag;
  unsigned long long* trace;  // launch timeline (kTraceEvents entries) or NULL:
                              // released, q/k/v exchanged, partials exchanged,
                              // (6, 7) arrival at the two exchange barriers,
                              // (8) rows normalised, (9) weights arrived,
                              // (10) GEMV reduced, (11) key prefetch arrived
};

__host__ __device__ inline int qa_tiles(int rep, int hd) { return (rep + 2) * hd / 16; }
__host__ __device__ inline int qa_tiles_per_cta(int rep, int hd) {
  return (qa_tiles(rep, hd) + kQaCluster - 1) / kQaCluster;
}
// Shared memory: weight tiles, one key/value chunk per row (the prefetched
// first chunk, then later chunks), the partials this rank merges, activation
// planes, reduction buffer, q and the new key/value of every row, scores.
struct QaLayout {
  size_t w, kvc, pml, pv, act, red, q, kv, kvs, cs, total;
};
// bits: 4 (INT4 weights) or 2 (the INT2 body's half-size tiles)
__host__ __device__ inline QaLayout qa_layout(int K, int M, int rep, int hd, int bits = 4) {
  QaLayout L;
  const size_t tile = (size_t)(K / 64) * (bits == 2 ? 256 : 512) + (size_t)(K / 128) * 64;
  const size_t wbytes = (size_t)qa_tiles_per_cta(rep, hd) * tile;
  const size_t chunk = (size_t)2 * kQaChunk * hd * 2;   // keys then values, fp16
  L.w = 0;
  L.kvc = (wbytes + 127) / 128 * 128;
  L.pml = L.kvc + (size_t)M * chunk;
  L.pv = L.pml + ((size_t)kQaCluster * M * rep * 8 + 127) / 128 * 128;
  L.act = L.pv + ((size_t)kQaCluster * M * rep * (hd / kQaCluster) * 4 + 127) / 128 * 128;
  L.red = L.act + ((size_t)M * (K + 8) * 2 * 2 + 127) / 128 * 128;
  L.q = L.red + (size_t)kQaWarps * kQaMaxTiles * 64 * 4;
  L.kv = L.q + (size_t)M * rep * hd * 4;
  L.kvs = L.kv + (size_t)2 * M * hd * 4;             // INT8 cache: the chunk's scales [m][K|V][kQaChunk]
  L.total = L.kvs + (size_t)M * 2 * kQaChunk * 4 + 128;   // + scores and softmax state
  L.total += (size_t)(rep * kQaChunk + 4 * rep) * 4;
  L.cs = (L.total + 15) / 16 * 16;                    // RoPE (cos, sin) [m][hd / 2]
  L.total = L.cs + (size_t)M * (hd / 2) * 8;
  return L;
}

__device__ __forceinline__ unsigned qa_cluster_rank() {
  unsigned r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void qa_cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Shared-memory address of `p` in the CTA of cluster rank `rank`.
__device__ __forceinline__ unsigned qa_peer(const void* p, unsigned rank) {
  unsigned out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(smem_u32(p)), "r"(rank));
  return out;
}
__device__ __forceinline__ void qa_st_peer(unsigned addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void qa_st_peer2(unsigned addr, float x, float y) {
  asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(x), "f"(y) : "memory");
}

// KV8: INT8 KV cache (kv8.cuh): the new key / value are quantised by every
// rank alike after the first exchange (rank 0 stores them) and the cached
// keys / values are read as codes times their vector's scale.
// BITS: 4 (INT4 weights) or 2 (INT2 body, unpack_a_frag2).
template <int HD, bool KV8, int BITS = 4>
__global__ void __launch_bounds__(kQaThreads, 1) qkv_attn_kernel(const QkvAttnArgs a) {
  constexpr int DPL = HD / 32;
  constexpr int ROW16 = HD / 8;
  constexpr int SW = HD / kQaCluster;   // head dimensions merged by each rank
  extern __shared__ __align__(128) unsigned char qsm[];
  __shared__ __align__(8) uint64_t wbar, kvbar;
  __shared__ int s_ok;
  __shared__ float s_ss[kQaMaxRows][kQaWarps];
  const int K = a.K, M = a.M, rep = a.rep;
  const QaLayout L = qa_layout(K, M, rep, HD, BITS);
  unsigned char* wsm = qsm + L.w;
  __half* kvc = reinterpret_cast<__half*>(qsm + L.kvc);     // [m][keys, values][kQaChunk][hd]
  float2* pml = reinterpret_cast<float2*>(qsm + L.pml);     // [rank][m][h]: (max, sum of weights)
  float* pv = reinterpret_cast<float*>(qsm + L.pv);         // [rank][m][h][SW]: this rank's dims
  __half* xs = reinterpret_cast<__half*>(qsm + L.act);
  __half* xl = xs + (size_t)M * (K + 8);
  float* red = reinterpret_cast<float*>(qsm + L.red);       // [warp][tile][16][4]
  float* qb = reinterpret_cast<float*>(qsm + L.q);          // [m][rep * hd]
  float* knew = reinterpret_cast<float*>(qsm + L.kv);       // [m][hd]
  float* vnew = knew + (size_t)M * HD;                       // [m][hd]
  float* kvs = reinterpret_cast<float*>(qsm + L.kvs);      // INT8: [m][K|V][kQaChunk] scales
  float* sc = kvs + (size_t)M * 2 * kQaChunk;                // [rep][kQaChunk]
  float2* cst = reinterpret_cast<float2*>(qsm + L.cs);       // RoPE (cos, sin) [m][hd / 2]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g8 = lane >> 2, t4 = lane & 3;
  const unsigned crank = qa_cluster_rank();
  const int c = (int)crank, grp = blockIdx.y;
  const int TG = qa_tiles(rep, HD), hpt = HD / 16;
  const int qdim = a.Hkv * rep * HD, kvdim = a.Hkv * HD;
  constexpr int LANE_B = BITS == 2 ? 8 : 16;   // weight bytes per lane per 64-k chunk
  const size_t wt_bytes = (size_t)(K / 64) * 32 * LANE_B, sz_bytes = (size_t)(K / 128) * 64;
  // this CTA's group tiles: c, c + kQaCluster, ... (nt of them)
  const int nt = c < TG ? min(kQaMaxTiles, (TG - 1 - c) / kQaCluster + 1) : 0;
  // group tile -> global 16-row tile of the QKV output: group heads are rep
  // query heads, then the key head, then the value head
  auto group_tile = [&](int tau) -> int {
    const int hh = tau / hpt, j = tau % hpt;
    const int row_base = hh < rep ? (grp * rep + hh) * HD : (hh == rep ? qdim + grp * HD : qdim + kvdim + grp * HD);
    return row_base / 16 + j;
  };

  trace_start(a.trace);
  // No early trigger: the next kernel (the O projection) launches when this
  // one completes.  Launched early, its CTAs and, through its own trigger,
  // gate_up's crowd onto the SMs this kernel leaves free; the decode step
  // measured faster without.
  if (tid == 0) {
    mbar_init(&wbar, 1);
    mbar_init(&kvbar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&wbar, (unsigned)(nt * (wt_bytes + sz_bytes)));
    const uint64_t pol = a.l2_keep ? l2_evict_last() : l2_evict_first();
    for (int i = 0; i < nt; ++i) {
      const int tile = group_tile(c + i * kQaCluster);
      const unsigned char* src = reinterpret_cast<const unsigned char*>(a.w) + (size_t)tile * wt_bytes;
      for (size_t off = 0; off < wt_bytes; off += 32768) {
        const unsigned n = (unsigned)((wt_bytes - off) < 32768 ? (wt_bytes - off) : 32768);
        bulk_g2s_hint(wsm + i * wt_bytes + off, src + off, n, &wbar, pol);
      }
      bulk_g2s_hint(wsm + nt * wt_bytes + i * sz_bytes,
                    reinterpret_cast<const unsigned char*>(a.sz) + (size_t)tile * sz_bytes, (unsigned)sz_bytes, &wbar,
                    pol);
    }
  }
  // every rank of the cluster must be running before any distributed
  // shared-memory write reaches it (the first ones come after the GEMV)
  qa_cluster_sync();
  pdl_wait();
  trace_mark(a.trace, 2);
  RowCtx rcs[kQaMaxRows];
#pragma unroll
  for (int m = 0; m < kQaMaxRows; ++m) rcs[m] = m < M ? a.rows[m] : RowCtx{0, 0};
  // ---- RMSNorm of the rows into the (hi, lo) planes: every thread loads its
  // columns of every row (and the gains) at once and keeps them in registers
  constexpr int V4 = 4;                       // float4 columns per thread and row: K <= 4096
  float4 xv[kQaMaxRows][V4];
  uint2 gv[V4];
#pragma unroll
  for (int i = 0; i < V4; ++i) {
    const int k = tid * 4 + i * 4 * kQaThreads;
    gv[i] = k < K ? *reinterpret_cast<const uint2*>(a.gain + k) : make_uint2(0u, 0u);
#pragma unroll
    for (int m = 0; m < kQaMaxRows; ++m)
      xv[m][i] = (m < M && k < K) ? *reinterpret_cast<const float4*>(a.x + (size_t)m * K + k)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // INT8: the first chunk's scales (their offsets are not 16-byte aligned,
  // so plain loads) by warp 1, under the GEMV like the codes' bulk copies
  if (KV8 && warp == 1) {
    for (int m = 0; m < M; ++m) {
      RowCtx rc = rcs[0];
#pragma unroll
      for (int q = 1; q < kQaMaxRows; ++q)
        if (m == q) rc = rcs[q];
      const int n = rc.pos + 1, C = (n + kQaCluster - 1) / kQaCluster;
      const int j0 = min(n, c * C), j1 = min(n, j0 + C), nk = min(kQaChunk, j1 - j0);
      float* ssk0 = kvs + (size_t)m * 2 * kQaChunk;
      const float* ksb = a.k_scale + (rc.lane * a.lane_stride) / HD + (size_t)grp * a.ctx;
      const float* vsb = a.v_scale + (rc.lane * a.lane_stride) / HD + (size_t)grp * a.ctx;
      for (int e = lane; e < 2 * kQaChunk; e += 32) {
        const int kv = e / kQaChunk, key = e % kQaChunk, jj = j0 + key;
        ssk0[e] = (key < nk && jj != rc.pos) ? __ldcg((kv ? vsb : ksb) + jj) : 0.f;
      }
    }
  }
  // RoPE (cos, sin) of every row's position, applied after the exchange
  // (published before the GEMV's block barrier)
  for (int e = tid; e < M * (HD / 2); e += kQaThreads) {
    const int m = e / (HD / 2), j = e % (HD / 2);
    RowCtx rc = rcs[0];
#pragma unroll
    for (int q = 1; q < kQaMaxRows; ++q)
      if (m == q) rc = rcs[q];
    cst[e] = rope_cs(a.rope_tab, rc.pos, j, HD, a.theta);
  }

#pragma unroll
  for (int m = 0; m < kQaMaxRows; ++m) {
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < V4; ++i)
      ss += xv[m][i].x * xv[m][i].x + xv[m][i].y * xv[m][i].y + xv[m][i].z * xv[m][i].z + xv[m][i].w * xv[m][i].w;
    ss = warp_sum(ss);
    if (lane == 0) s_ss[m][warp] = ss;
  }
  __syncthreads();
#pragma unroll
  for (int m = 0; m < kQaMaxRows; ++m) {
    if (m >= M) continue;
    float ss = 0.f;
#pragma unroll
    for (int w = 0; w < kQaWarps; ++w) ss += s_ss[m][w];
    const float rs = 1.0f / sqrtf(ss / (float)K + a.eps);
#pragma unroll
    for (int i = 0; i < V4; ++i) {
      const int k = tid * 4 + i * 4 * kQaThreads;
      if (k >= K) continue;
      float4 v = xv[m][i];
      const float2 g01 = h2_to_f2(gv[i].x), g23 = h2_to_f2(gv[i].y);
      v.x = (v.x * rs) * g01.x; v.y = (v.y * rs) * g01.y;
      v.z = (v.z * rs) * g23.x; v.w = (v.w * rs) * g23.y;
      const __half2 h01 = __floats2half2_rn(v.x, v.y), h23 = __floats2half2_rn(v.z, v.w);
      const float2 r01 = __half22float2(h01), r23 = __half22float2(h23);
      const __half2 l01 = __floats2half2_rn(v.x - r01.x, v.y - r01.y);
      const __half2 l23 = __floats2half2_rn(v.z - r23.x, v.w - r23.y);
      uint2 ph, pl;
      ph.x = *reinterpret_cast<const uint32_t*>(&h01); ph.y = *reinterpret_cast<const uint32_t*>(&h23);
      pl.x = *reinterpret_cast<const uint32_t*>(&l01); pl.y = *reinterpret_cast<const uint32_t*>(&l23);
      *reinterpret_cast<uint2*>(xs + (size_t)m * (K + 8) + k) = ph;
      *reinterpret_cast<uint2*>(xl + (size_t)m * (K + 8) + k) = pl;
    }
  }
  if (tid == 0) {
    trace_mark(a.trace, 8);
    s_ok = mbar_wait(&wbar, 0) ? 1 : 0;
    if (!s_ok) atomicOr(a.err_flag, kErrTimeout);
    trace_mark(a.trace, 9);
  }
  // The first chunk of this rank's key split of every row, minus the new key,
  // goes out once the weights have landed, under the GEMV (issued during the
  // RMSNorm it delayed the norm's block barrier by more than it saved).
  if (tid == 0) {
    unsigned bytes = 0;
    int lo[kQaMaxRows], cnt[kQaMaxRows];
#pragma unroll
    for (int m = 0; m < kQaMaxRows; ++m) {
      cnt[m] = 0;
      lo[m] = 0;
      if (m < M) {
        const int n = rcs[m].pos + 1, C = (n + kQaCluster - 1) / kQaCluster;
        lo[m] = min(n, c * C);
        const int hi = min(min(n, lo[m] + C), lo[m] + kQaChunk);
        cnt[m] = max(0, min(hi, rcs[m].pos) - lo[m]);
        bytes += 2u * (unsigned)cnt[m] * HD * (KV8 ? 1u : 2u);
      }
    }
    mbar_arrive_expect_tx(&kvbar, bytes);
#pragma unroll
    for (int m = 0; m < kQaMaxRows; ++m) {
      if (cnt[m] > 0) {
        const size_t src = (size_t)rcs[m].lane * a.lane_stride + ((size_t)grp * a.ctx + lo[m]) * HD;
        __half* dst = kvc + (size_t)m * 2 * kQaChunk * HD;
        if (KV8) {   // codes only, staged in the V half (their scales follow with plain loads below)
          int8_t* d8 = reinterpret_cast<int8_t*>(dst + kQaChunk * HD);
          bulk_g2s(d8, reinterpret_cast<const int8_t*>(a.k_plane) + src, (unsigned)cnt[m] * HD, &kvbar);
          bulk_g2s(d8 + kQaChunk * HD, reinterpret_cast<const int8_t*>(a.v_plane) + src, (unsigned)cnt[m] * HD,
                   &kvbar);
        } else {
          bulk_g2s(dst, a.k_plane + src, (unsigned)cnt[m] * HD * 2u, &kvbar);
          bulk_g2s(dst + kQaChunk * HD, a.v_plane + src, (unsigned)cnt[m] * HD * 2u, &kvbar);
        }
      }
    }
  }
  __syncthreads();
  const bool ok = s_ok != 0;   // on a time-out the control flow stays the same (cluster barriers)

  // ---- GEMV of this CTA's tiles: warps split K, B fragments shared --------
  {
    const int nck = K / 64;
    const int c0 = warp * nck / kQaWarps, c1 = (warp + 1) * nck / kQaWarps;
    const int brow = g8 >> 1;
    const __half* bsrc = ((g8 & 1) ? xl : xs) + (size_t)brow * (K + 8) + 2 * t4;
    const bool bok = brow < M;
    float acc[kQaMaxTiles][4];
#pragma unroll
    for (int i = 0; i < kQaMaxTiles; ++i)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[i][q] = 0.f;
    for (int ci = c0; ok && ci < c1; ++ci) {
      uint32_t bf[4][2];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        bf[j][0] = bok ? *reinterpret_cast<const uint32_t*>(bsrc + ci * 64 + j * 16) : 0u;
        bf[j][1] = bok ? *reinterpret_cast<const uint32_t*>(bsrc + ci * 64 + j * 16 + 8) : 0u;
      }
#pragma unroll
      for (int i = 0; i < kQaMaxTiles; ++i) {
        if (i < nt) {
          uint32_t words[4];
          if (BITS == 2) {
            const uint2 w2 = *reinterpret_cast<const uint2*>(wsm + i * wt_bytes + (size_t)ci * 32 * LANE_B + lane * LANE_B);
            words[0] = w2.x; words[1] = w2.y; words[2] = 0u; words[3] = 0u;
          } else {
            const uint4 wv = *reinterpret_cast<const uint4*>(wsm + i * wt_bytes + (size_t)ci * 32 * LANE_B + lane * LANE_B);
            words[0] = wv.x; words[1] = wv.y; words[2] = wv.z; words[3] = wv.w;
          }
          const uint2 sv =
              *reinterpret_cast<const uint2*>(wsm + nt * wt_bytes + i * sz_bytes + (size_t)(ci >> 1) * 64 + g8 * 8);
          float t0[4] = {0.f, 0.f, 0.f, 0.f}, t1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t af[4];
            if (BITS == 2) unpack_a_frag2(words[j >> 1], j & 1, sv.y, af);
            else unpack_a_frag(words[j], sv.y, af);
            if (j & 1) mma_f16_16816(t1, af, bf[j][0], bf[j][1]);
            else mma_f16_16816(t0, af, bf[j][0], bf[j][1]);
          }
          const float2 s2 = h2_to_f2(sv.x);
          acc[i][0] = fmaf(s2.x, t0[0] + t1[0], acc[i][0]);
          acc[i][1] = fmaf(s2.x, t0[1] + t1[1], acc[i][1]);
          acc[i][2] = fmaf(s2.y, t0[2] + t1[2], acc[i][2]);
          acc[i][3] = fmaf(s2.y, t0[3] + t1[3], acc[i][3]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kQaMaxTiles; ++i) {
      if (i < nt) {
        float* r = red + ((size_t)warp * kQaMaxTiles + i) * 64;
        r[g8 * 4 + t4] = acc[i][0] + acc[i][1];        // tile row g8, activation row t4 (hi + lo)
        r[(g8 + 8) * 4 + t4] = acc[i][2] + acc[i][3];  // tile row g8 + 8
      }
    }
  }
  __syncthreads();
  trace_mark(a.trace, 10);

  // ---- epilogue: the raw projections of this rank's tiles to every rank ----
  if (tid < nt * 16 * M) {   // nt * 16 * M <= 128: one element per thread
    const int ti = tid / (16 * M), rem = tid % (16 * M), r = rem & 15, m = rem >> 4;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kQaWarps; ++w) v += red[((size_t)w * kQaMaxTiles + ti) * 64 + r * 4 + m];
    const int gr = (c + ti * kQaCluster) * 16 + r;   // row of the group: q heads, key, value
    float* dst_s = gr < rep * HD ? qb + (size_t)m * rep * HD + gr
                                 : (gr < (rep + 1) * HD ? knew + (size_t)m * HD + (gr - rep * HD)
                                                        : vnew + (size_t)m * HD + (gr - (rep + 1) * HD));
    for (unsigned rk = 0; rk < kQaCluster; ++rk) qa_st_peer(qa_peer(dst_s, rk), v);
  }
  trace_mark(a.trace, 6);
  qa_cluster_sync();   // #1: q and the new key / value are in every rank
  trace_mark(a.trace, 3);
  // RoPE on every query head and the key: pairs (j, j + hd/2); with an fp16
  // cache the key and value become the fp16 values the cache stores (the
  // attention reads the new position like any cached one)
  for (int e = tid; e < M * (rep + 1) * (HD / 2); e += kQaThreads) {
    const int m = e / ((rep + 1) * (HD / 2)), rem = e % ((rep + 1) * (HD / 2));
    const int hh = rem / (HD / 2), j = rem % (HD / 2);
    float* base = hh < rep ? qb + (size_t)m * rep * HD + hh * HD : knew + (size_t)m * HD;
    const float va = base[j], vb = base[j + HD / 2];
    const float2 cs = cst[m * (HD / 2) + j];
    float e0 = va * cs.x - vb * cs.y, e1 = vb * cs.x + va * cs.y;
    if (!KV8 && hh == rep) {
      e0 = __half2float(__float2half_rn(e0));
      e1 = __half2float(__float2half_rn(e1));
    }
    base[j] = e0;
    base[j + HD / 2] = e1;
  }
  if (!KV8)
    for (int e = tid; e < M * HD; e += kQaThreads) vnew[e] = __half2float(__float2half_rn(vnew[e]));
  __syncthreads();
  if (!KV8 && ok) {
    // this rank's hd / kQaCluster elements of each row's new key and value
    constexpr int PER = HD / kQaCluster;
    if (tid < M * 2 * PER) {
      const int m = tid / (2 * PER), kv = (tid / PER) & 1, j = c * PER + tid % PER;
      RowCtx rc = rcs[0];
#pragma unroll
      for (int q = 1; q < kQaMaxRows; ++q)
        if (m == q) rc = rcs[q];
      __half* cache = (kv ? a.v_plane : a.k_plane) + rc.lane * a.lane_stride + ((size_t)grp * a.ctx + rc.pos) * HD;
      cache[j] = __float2half_rn((kv ? vnew : knew)[(size_t)m * HD + j]);
    }
  }
  if (KV8) {
    // INT8 cache: warp 2m + kv quantises row m's new key (kv = 0) or value;
    // every rank computes the same codes, rank 0 stores them, and attention
    // reads code * scale like any cached position
    if (warp < 2 * M) {
      const int m = warp >> 1, kv = warp & 1;
      float* vec = (kv ? vnew : knew) + (size_t)m * HD;
      float xv[DPL];
      int qc[DPL];
#pragma unroll
      for (int i = 0; i < DPL; ++i) xv[i] = vec[lane * DPL + i];
      const float sc8 = kv8_quant_warp<DPL>(xv, qc);
#pragma unroll
      for (int i = 0; i < DPL; ++i) vec[lane * DPL + i] = (float)qc[i] * sc8;
      if (c == 0 && ok) {
        RowCtx rc = rcs[0];
#pragma unroll
        for (int q = 1; q < kQaMaxRows; ++q)
          if (m == q) rc = rcs[q];
        const size_t e = (size_t)rc.lane * a.lane_stride + ((size_t)grp * a.ctx + rc.pos) * HD;
        int8_t* dst = reinterpret_cast<int8_t*>(kv ? a.v_plane : a.k_plane) + e;
        uint32_t w = 0;
#pragma unroll
        for (int i = 0; i < DPL; ++i) w |= ((uint32_t)qc[i] & 0xffu) << (8 * i);
        if (DPL == 4) *reinterpret_cast<uint32_t*>(dst + lane * 4) = w;
        else *reinterpret_cast<uint16_t*>(dst + lane * 2) = (uint16_t)w;
        if (lane == 0) (kv ? a.v_scale : a.k_scale)[e / HD] = sc8;
      }
    }
    __syncthreads();
  }

  // ---- attention over this rank's key split, per row: warp h < rep takes
  // query head h (scores, online softmax and P V stay inside the warp) ------
  const float scale = 1.0f / sqrtf((float)HD);
  const bool head_warp = warp < rep;
  float* sh = sc + (head_warp ? warp : 0) * kQaChunk;   // this warp's scores / weights
  for (int m = 0; m < M; ++m) {
    RowCtx rc = rcs[0];
#pragma unroll
    for (int q = 1; q < kQaMaxRows; ++q)
      if (m == q) rc = rcs[q];
    const int n = rc.pos + 1;
    const int C = (n + kQaCluster - 1) / kQaCluster;
    const int j0 = min(n, c * C), j1 = min(n, j0 + C);
    const __half* kb = a.k_plane + rc.lane * a.lane_stride + (size_t)grp * a.ctx * HD;
    const __half* vb = a.v_plane + rc.lane * a.lane_stride + (size_t)grp * a.ctx * HD;
    __half* ks = kvc + (size_t)m * 2 * kQaChunk * HD;      // [kQaChunk][HD]
    __half* vs = ks + kQaChunk * HD;
    // INT8 cache: each chunk's codes are widened once into the fp16 layout
    // above (exact integers; the first chunk's bulk copy lands as int8 in the
    // V half first), its scales go to ssk / ssv and are applied per key
    const int8_t* kb8 = reinterpret_cast<const int8_t*>(a.k_plane) + rc.lane * a.lane_stride + (size_t)grp * a.ctx * HD;
    const int8_t* vb8 = reinterpret_cast<const int8_t*>(a.v_plane) + rc.lane * a.lane_stride + (size_t)grp * a.ctx * HD;
    const float* ksb = KV8 ? a.k_scale + (rc.lane * a.lane_stride) / HD + (size_t)grp * a.ctx : nullptr;
    const float* vsb = KV8 ? a.v_scale + (rc.lane * a.lane_stride) / HD + (size_t)grp * a.ctx : nullptr;
    const int8_t* stage8 = reinterpret_cast<const int8_t*>(vs);   // [K|V][kQaChunk][HD] codes of the first chunk
    float* ssk = kvs + (size_t)m * 2 * kQaChunk;                  // [kQaChunk]
    float* ssv = ssk + kQaChunk;
    // this lane's DPL dimensions of q (head `warp`) and of the new key / value
    float qv[DPL], kn[DPL], vn[DPL], o[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      qv[i] = head_warp ? qb[((size_t)m * rep + warp) * HD + lane * DPL + i] : 0.f;
      kn[i] = knew[(size_t)m * HD + lane * DPL + i];
      vn[i] = vnew[(size_t)m * HD + lane * DPL + i];
      o[i] = 0.f;
    }
    float m_run = -INFINITY, l_run = 0.f;
    if (head_warp && j0 < j1 && !mbar_wait(&kvbar, 0) && lane == 0) atomicOr(a.err_flag, kErrTimeout);
    trace_mark(a.trace, 11);
    for (int jc = j0; jc < j1; jc += kQaChunk) {
      const int nk = min(kQaChunk, j1 - jc);
      if (KV8) {
        // codes into registers (16 per load): the first chunk from its staged
        // bulk copy, later ones from the cache; then widened to fp16 in the
        // chunk layout; the new key is read from registers, not from here
        constexpr int ROW16B = HD / 16;
        constexpr int PER = 2 * kQaChunk * ROW16B / kQaThreads;
        static_assert(PER * kQaThreads == 2 * kQaChunk * ROW16B, "whole chunk per pass");
        const bool first = jc == j0;
        if (first && !mbar_wait(&kvbar, 0) && tid == 0) atomicOr(a.err_flag, kErrTimeout);
        __syncthreads();   // the previous chunk is consumed
        uint4 cv[PER];
#pragma unroll
        for (int u = 0; u < PER; ++u) {
          const int e = tid + u * kQaThreads;
          const int kv = e / (kQaChunk * ROW16B), rem = e % (kQaChunk * ROW16B);
          const int key = rem / ROW16B, pc = rem % ROW16B, jj = jc + key;
          cv[u] = make_uint4(0, 0, 0, 0);
          if (key < nk && jj != rc.pos)
            cv[u] = first ? reinterpret_cast<const uint4*>(stage8)[e]
                          : __ldcg(reinterpret_cast<const uint4*>((kv ? vb8 : kb8) + (size_t)jj * HD) + pc);
        }
        if (!first)
          for (int e = tid; e < 2 * kQaChunk; e += kQaThreads) {
            const int kv = e / kQaChunk, key = e % kQaChunk, jj = jc + key;
            ssk[e] = (key < nk && jj != rc.pos) ? __ldcg((kv ? vsb : ksb) + jj) : 0.f;
          }
        __syncthreads();   // the staged codes are read
#pragma unroll
        for (int u = 0; u < PER; ++u) {
          const int e = tid + u * kQaThreads;   // 16 codes -> 16 fp16 at element 16 e of [K|V][kQaChunk][HD]
          const uint32_t ws[4] = {cv[u].x, cv[u].y, cv[u].z, cv[u].w};
          uint4 h0, h1;
          __half2 c01, c23;
          kv8_codes_h2(ws[0], c01, c23); h0.x = *reinterpret_cast<uint32_t*>(&c01); h0.y = *reinterpret_cast<uint32_t*>(&c23);
          kv8_codes_h2(ws[1], c01, c23); h0.z = *reinterpret_cast<uint32_t*>(&c01); h0.w = *reinterpret_cast<uint32_t*>(&c23);
          kv8_codes_h2(ws[2], c01, c23); h1.x = *reinterpret_cast<uint32_t*>(&c01); h1.y = *reinterpret_cast<uint32_t*>(&c23);
          kv8_codes_h2(ws[3], c01, c23); h1.z = *reinterpret_cast<uint32_t*>(&c01); h1.w = *reinterpret_cast<uint32_t*>(&c23);
          reinterpret_cast<uint4*>(ks)[2 * e] = h0;
          reinterpret_cast<uint4*>(ks)[2 * e + 1] = h1;
        }
        __syncthreads();
      } else if (jc != j0) {
        // later chunks (splits longer than kQaChunk keys): plain loads by
        // every thread; the new key is read from registers, not from here
        __syncthreads();   // the previous chunk is consumed
        for (int e = tid; e < 2 * kQaChunk * ROW16; e += kQaThreads) {
          const int kv = e / (kQaChunk * ROW16), rem = e % (kQaChunk * ROW16);
          const int key = rem / ROW16, pc = rem % ROW16, jj = jc + key;
          uint4 val = make_uint4(0, 0, 0, 0);
          if (key < nk && jj != rc.pos) val = __ldcg(reinterpret_cast<const uint4*>((kv ? vb : kb) + (size_t)jj * HD) + pc);
          reinterpret_cast<uint4*>(ks)[e] = val;
        }
        __syncthreads();
      }
      if (head_warp) {
        // scores, eight keys at a time (independent butterfly reductions)
        for (int j8 = 0; j8 < nk; j8 += 8) {
          float p[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int jj = j8 + u;
            float d = 0.f;
            if (jj < nk) {
              float kf[DPL];
              if (jc + jj == rc.pos) {
#pragma unroll
                for (int i = 0; i < DPL; ++i) kf[i] = kn[i];
              } else if constexpr (DPL == 4) {   // (INT8: the codes; the key's scale after the sum)
                const uint2 u2 = *reinterpret_cast<const uint2*>(ks + jj * HD + lane * 4);
                const float2 f01 = h2_to_f2(u2.x), f23 = h2_to_f2(u2.y);
                kf[0] = f01.x; kf[1] = f01.y; kf[2] = f23.x; kf[3] = f23.y;
              } else {
                const float2 f01 = h2_to_f2(*reinterpret_cast<const unsigned*>(ks + jj * HD + lane * 2));
                kf[0] = f01.x; kf[1] = f01.y;
              }
#pragma unroll
              for (int i = 0; i < DPL; ++i) d = fmaf(qv[i], kf[i], d);
            }
            p[u] = d;
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1)
#pragma unroll
            for (int u = 0; u < 8; ++u) p[u] += __shfl_xor_sync(0xffffffffu, p[u], off);
#pragma unroll
          for (int u = 0; u < 8; ++u)
            if (lane == u && j8 + u < nk)
              sh[j8 + u] = p[u] * scale * ((KV8 && jc + j8 + u != rc.pos) ? ssk[j8 + u] : 1.f);
        }
        __syncwarp();
        // online softmax over the chunk
        float mx = -INFINITY;
        for (int jj = lane; jj < nk; jj += 32) mx = fmaxf(mx, sh[jj]);
        mx = warp_max(mx);
        const float m_new = fmaxf(m_run, mx);
        float sum = 0.f;
        for (int jj = lane; jj < nk; jj += 32) {
          const float e = expf(sh[jj] - m_new);
          sh[jj] = e;
          sum += e;
        }
        sum = warp_sum(sum);
        const float alpha = expf(m_run - m_new);
        l_run = l_run * alpha + sum;
        m_run = m_new;
        __syncwarp();
        // P V over the lane's dimensions
#pragma unroll
        for (int i = 0; i < DPL; ++i) o[i] *= alpha;
#pragma unroll 4
        for (int jj = 0; jj < nk; ++jj) {
          float pj = sh[jj];
          float vf[DPL];
          if (jc + jj == rc.pos) {
#pragma unroll
            for (int i = 0; i < DPL; ++i) vf[i] = vn[i];
          } else if constexpr (DPL == 4) {
            if (KV8) pj *= ssv[jj];   // INT8: the codes; the weight carries the value's scale
            const uint2 u2 = *reinterpret_cast<const uint2*>(vs + jj * HD + lane * 4);
            const float2 f01 = h2_to_f2(u2.x), f23 = h2_to_f2(u2.y);
            vf[0] = f01.x; vf[1] = f01.y; vf[2] = f23.x; vf[3] = f23.y;
          } else {
            if (KV8) pj *= ssv[jj];
            const float2 f01 = h2_to_f2(*reinterpret_cast<const unsigned*>(vs + jj * HD + lane * 2));
            vf[0] = f01.x; vf[1] = f01.y;
          }
#pragma unroll
          for (int i = 0; i < DPL; ++i) o[i] = fmaf(pj, vf[i], o[i]);
        }
        __syncwarp();   // sh is rewritten by the next chunk
      }
    }
    // this split's (max, sum of weights) to every rank, each slice of its
    // weighted value sums to the rank that merges those dimensions
    if (head_warp) {
      if (lane < kQaCluster)
        qa_st_peer2(qa_peer(pml + ((size_t)c * M + m) * rep + warp, (unsigned)lane), m_run, l_run);
#pragma unroll
      for (int i = 0; i < DPL; ++i) {
        const int dim = lane * DPL + i;
        qa_st_peer(qa_peer(pv + (((size_t)c * M + m) * rep + warp) * SW + dim % SW, (unsigned)(dim / SW)), o[i]);
      }
    }
  }
  trace_mark(a.trace, 7);
  qa_cluster_sync();   // #2: every rank holds every split's partials of its dimensions
  trace_mark(a.trace, 4);

  // ---- each rank merges its SW dimensions of every (row, head), ranks in order
  if (tid < M * rep * SW) {
    const int m = tid / (rep * SW), rem = tid % (rep * SW), h = rem / SW, dd = rem % SW;
    float mx = -INFINITY;
#pragma unroll
    for (int rk = 0; rk < kQaCluster; ++rk) mx = fmaxf(mx, pml[((size_t)rk * M + m) * rep + h].x);
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int rk = 0; rk < kQaCluster; ++rk) {
      const float2 st = pml[((size_t)rk * M + m) * rep + h];
      if (st.y > 0.f) {   // ranks without keys contribute nothing
        const float w = expf(st.x - mx);
        num = fmaf(w, pv[(((size_t)rk * M + m) * rep + h) * SW + dd], num);
        den = fmaf(w, st.y, den);
      }
    }
    if (ok)
      a.o[(size_t)m * (a.Hkv * rep * HD) + (size_t)(grp * rep + h) * HD + c * SW + dd] = num / den;
  }
  trace_mark(a.trace, 5);
}

}  // namespace tl
