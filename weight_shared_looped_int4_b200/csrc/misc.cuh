// Embedding gather, stand-alone RMSNorm and RoPE, and the output head with
// the greedy argmax.
#pragma once

#include "common.cuh"

namespace tl {

// ---- embedding: x[row] = E[token] widened to fp32 -------------------------
// A token outside [0, vocab) is replaced by 0 and recorded in *err_flag.
__global__ void embed_kernel(const __half* __restrict__ E, int d, int vocab,
                             const int32_t* __restrict__ tokens, const int* __restrict__ tok_index,
                             float* __restrict__ x, int* err_flag) {
  const int row = blockIdx.x;
  pdl_trigger();
  pdl_wait();
  const int src = tok_index ? tok_index[row] : row;
  int tok = tokens[src];
  if (tok < 0 || tok >= vocab) {
    if (threadIdx.x == 0) atomicOr(err_flag, kErrToken);
    tok = 0;
  }
  const __half* e = E + (size_t)tok * d;
  float* xr = x + (size_t)row * d;
  for (int k = threadIdx.x * 2; k < d; k += blockDim.x * 2) {
    const float2 v = __half22float2(*reinterpret_cast<const __half2*>(e + k));
    *reinterpret_cast<float2*>(xr + k) = v;
  }
}

// ---- RMSNorm: y = fp16(x / sqrt(mean(x^2) + eps) * g), one warp per row ---
// Same arithmetic order as the norm fused into the GEMV prologue.
__global__ void rmsnorm_kernel(const float* __restrict__ x, const __half* __restrict__ gain,
                               int rows, int d, float eps, __half* __restrict__ y) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  pdl_trigger();
  pdl_wait();
  if (row >= rows) return;
  const float* src = x + (size_t)row * d;
  float ss = 0.f;
  for (int k = lane * 4; k < d; k += 128) {
    const float4 v = *reinterpret_cast<const float4*>(src + k);
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = warp_sum(ss);
  const float rs = 1.0f / sqrtf(ss / (float)d + eps);
  __half* dst = y + (size_t)row * d;
  for (int k = lane * 4; k < d; k += 128) {
    const float4 v = *reinterpret_cast<const float4*>(src + k);
    const float2 g01 = __half22float2(*reinterpret_cast<const __half2*>(gain + k));
    const float2 g23 = __half22float2(*reinterpret_cast<const __half2*>(gain + k + 2));
    *reinterpret_cast<__half2*>(dst + k) = __floats2half2_rn((v.x * rs) * g01.x, (v.y * rs) * g01.y);
    *reinterpret_cast<__half2*>(dst + k + 2) = __floats2half2_rn((v.z * rs) * g23.x, (v.w * rs) * g23.y);
  }
}

// ---- RoPE table of a model: (cos, sin) [positions][hd/2] --------------------
__global__ void rope_table_kernel(float2* tab, int n_pos, int hd, float theta) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int half = hd >> 1;
  if (i < n_pos * half) tab[i] = rope_cos_sin(i / half, i % half, hd, theta);
}

// ---- RoPE in place: one thread per (token, head, pair) ---------------------
__global__ void rope_inplace_kernel(__half* x, int n_tokens, int n_heads, int hd,
                                    long long token_stride, long long head_stride,
                                    const int32_t* __restrict__ positions, float theta) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int half = hd >> 1;
  pdl_trigger();
  pdl_wait();
  if (idx >= (long long)n_tokens * n_heads * half) return;
  const int j = (int)(idx % half);
  const long long th = idx / half;
  const int h = (int)(th % n_heads);
  const int t = (int)(th / n_heads);
  __half* p = x + t * token_stride + h * head_stride;
  const float2 cs = rope_cos_sin(positions[t], j, hd, theta);
  const float a = __half2float(p[j]), b = __half2float(p[j + half]);
  p[j] = __float2half_rn(a * cs.x - b * cs.y);
  p[j + half] = __float2half_rn(b * cs.x + a * cs.y);
}

// ---- output head -------------------------------------------------------------
// The fp16 head [V][d] is re-laid out at load time so that one 16-byte load of
// a lane is the A fragment of one m16n8k16 MMA: for 16-row tile T, 16-wide K
// tile kk and lane l = 4g + t, the four fp16 pairs are
//   (r0, kb+2t..), (r0+8, kb+2t..), (r0, kb+2t+8..), (r0+8, kb+2t+8..)
// with r0 = 16T + g, kb = 16 kk.
__global__ void repack_head_kernel(const uint32_t* __restrict__ head, int V, int d,
                                   uint4* __restrict__ out) {
  const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int nk = d >> 4;
  const size_t total = (size_t)(V >> 4) * nk * 32;
  if (idx >= total) return;
  const int l = (int)(idx & 31);
  const size_t rest = idx >> 5;
  const int kk = (int)(rest % nk);
  const int T = (int)(rest / nk);
  const int g = l >> 2, t = l & 3;
  const size_t r0 = (size_t)T * 16 + g, r1 = r0 + 8;
  const int kb = kk * 16 + 2 * t;
  const size_t dw = (size_t)d >> 1;  // u32 words per row
  out[idx] = make_uint4(head[r0 * dw + (kb >> 1)], head[r1 * dw + (kb >> 1)],
                        head[r0 * dw + ((kb + 8) >> 1)], head[r1 * dw + ((kb + 8) >> 1)]);
}

// Output pointers of a decode step, read by the head kernel from device
// memory so that a captured CUDA graph of the step is independent of them.
struct HeadIO {
  float* logits;
  int32_t* argmax;
};

struct HeadArgs {
  const HeadIO* io;     // if set, logits / argmax come from here
  const uint4* w;       // re-laid-out head
  int V, d;
  const float* x;       // final residual stream, fp32 [M][d]
  const __half* gain;   // output norm gains
  float eps;
  int M;                // rows (<= 16)
  const int* out_row;   // output slot of row m (NULL = m)
  float* logits;        // [.][V] or NULL
  int32_t* argmax;      // [.] or NULL
  float* part_val;      // [gridDim][16] per-CTA best value
  int* part_idx;        // [gridDim][16] per-CTA best index
  unsigned* ticket;     // zero between launches
  int* err_flag;        // device fault flags
};

constexpr int kHeadWarps = 8;                      // compute warps
constexpr int kHeadThreads = (kHeadWarps + 1) * 32;  // + one producer warp
constexpr int kHeadStageMax = 16384;                  // bytes per bulk-copy stage
constexpr size_t kHeadSmemBudget = 200 * 1024;

__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

// Stage size: 16 KB, or one whole row tile when the tile is smaller.
// Bytes per stage: at most kHeadStageMax, a divisor of the tile's bytes and a
// multiple of kHeadWarps k16 blocks (the tile, 32 d bytes, is a multiple of
// 4096 since d is a multiple of 128).
__host__ __device__ inline int head_stage_bytes(int d) {
  const int tile = (d / 16) * 512;
  int sb = tile < kHeadStageMax ? tile : kHeadStageMax;
  while (tile % sb) sb -= 512 * kHeadWarps;
  return sb;
}
__host__ __device__ inline size_t head_act_bytes(int d, int M) { return (size_t)M * (d + 8) * 2 * 2; }
__host__ __device__ inline int head_stages(int d, int M) {
  const size_t rest = kHeadSmemBudget - head_act_bytes(d, M);
  int s = (int)(rest / head_stage_bytes(d));
  return s > 12 ? 12 : s;
}
// Dynamic shared memory: the stage ring, the activation planes (hi, lo), the
// cross-warp reduction buffer.
__host__ __device__ inline size_t head_smem_bytes(int d, int M) {
  return (size_t)head_stages(d, M) * head_stage_bytes(d) + head_act_bytes(d, M) +
         (size_t)kHeadWarps * 16 * 16 * 4;
}

// One CTA per SM takes a contiguous range of 16-row tiles (balanced to +-1
// tile).  A producer warp streams the range through a ring of shared-memory
// stages with bulk asynchronous copies (the TMA engine), so up to ~190 KB per
// SM is in flight without spending registers; the first stages are requested
// before griddepcontrol.wait.  The 8 compute warps split each stage along K
// (MMA with the fp16 pair of the normalised activations) and combine at the
// end of every tile through shared memory, in warp order.  The output norm is
// computed by every CTA in the prologue.  Each row keeps its best (value,
// index); the last CTA to finish (atomic ticket) combines the CTAs.  Ties go
// to the lowest index.  Every wait is bounded (kErrTimeout on give-up).
template <int NT>
__global__ void __launch_bounds__(kHeadThreads, 1) head_argmax_kernel(const HeadArgs a) {
  constexpr int NC = NT * 8;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t full[12], empty[12];
  __shared__ float s_ss[16][kHeadWarps];
  __shared__ float s_val[16][16];
  __shared__ int s_idx[16][16];
  __shared__ int s_last, s_fail;
  const int d = a.d, ldxs = d + 8, M = a.M;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int SB = head_stage_bytes(d);
  const int S = head_stages(d, M);
  const int nk = d >> 4;                      // k16-tiles per row tile
  const int spt = (nk * 512) / SB;            // stages per row tile
  const int k16_per_stage = SB / 512;
  const int k16_per_warp = k16_per_stage / kHeadWarps;
  unsigned char* ring = smem;
  __half* xs = reinterpret_cast<__half*>(smem + (size_t)S * SB);
  __half* xl = xs + (size_t)M * ldxs;
  float* red = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(xs) + head_act_bytes(d, M));
  const int n_tiles = a.V >> 4;
  const int tb = (int)((long)blockIdx.x * n_tiles / gridDim.x);
  const int te = (int)((long)(blockIdx.x + 1) * n_tiles / gridDim.x);
  const int nf = (te - tb) * spt;             // stages this CTA streams

  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kHeadWarps);
    }
    fence_mbar_init();
    s_fail = 0;
  }
  __syncthreads();
  const unsigned char* wsrc = reinterpret_cast<const unsigned char*>(a.w) + (size_t)tb * spt * SB;
  if (warp == kHeadWarps && lane == 0) {  // first stages before the dependency wait
    for (int f = 0; f < S && f < nf; ++f) {
      mbar_arrive_expect_tx(&full[f], SB);
      bulk_g2s(ring + (size_t)f * SB, wsrc + (size_t)f * SB, SB, &full[f]);
    }
  }
  pdl_wait();

  // output RMSNorm of every row into shared memory as an fp16 pair
  for (int m = 0; m < M; ++m) {
    const float* src = a.x + (size_t)m * d;
    float ss = 0.f;
    if (warp < kHeadWarps) {
      for (int k = threadIdx.x * 4; k < d; k += 4 * kHeadWarps * 32) {
        const float4 v = *reinterpret_cast<const float4*>(src + k);
        ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
      }
      ss = warp_sum(ss);
      if (lane == 0) s_ss[m][warp] = ss;
    }
  }
  __syncthreads();
  for (int m = 0; m < M && warp < kHeadWarps; ++m) {
    const float* src = a.x + (size_t)m * d;
    float ss = 0.f;
#pragma unroll
    for (int w = 0; w < kHeadWarps; ++w) ss += s_ss[m][w];
    const float rs = 1.0f / sqrtf(ss / (float)d + a.eps);
    for (int k = threadIdx.x * 4; k < d; k += 4 * kHeadWarps * 32) {
      float4 v = *reinterpret_cast<const float4*>(src + k);
      const float2 g01 = __half22float2(*reinterpret_cast<const __half2*>(a.gain + k));
      const float2 g23 = __half22float2(*reinterpret_cast<const __half2*>(a.gain + k + 2));
      v.x = (v.x * rs) * g01.x; v.y = (v.y * rs) * g01.y;
      v.z = (v.z * rs) * g23.x; v.w = (v.w * rs) * g23.y;
      const __half2 h01 = __floats2half2_rn(v.x, v.y), h23 = __floats2half2_rn(v.z, v.w);
      const float2 r01 = __half22float2(h01), r23 = __half22float2(h23);
      *reinterpret_cast<__half2*>(xs + m * ldxs + k) = h01;
      *reinterpret_cast<__half2*>(xs + m * ldxs + k + 2) = h23;
      *reinterpret_cast<__half2*>(xl + m * ldxs + k) = __floats2half2_rn(v.x - r01.x, v.y - r01.y);
      *reinterpret_cast<__half2*>(xl + m * ldxs + k + 2) = __floats2half2_rn(v.z - r23.x, v.w - r23.y);
    }
  }
  __syncthreads();

  float* const logits = a.io ? a.io->logits : a.logits;
  int32_t* const argmax = a.io ? a.io->argmax : a.argmax;

  if (warp == kHeadWarps) {
    // ---- producer: refill each stage once all compute warps released it ----
    if (lane == 0) {
      int s = 0;
      unsigned par = 0;   // parity of the release being waited for
      for (int f = S; f < nf; ++f) {
        if (!mbar_wait_or_fail(&empty[s], par, &s_fail)) break;
        mbar_arrive_expect_tx(&full[s], SB);
        bulk_g2s(ring + (size_t)s * SB, wsrc + (size_t)f * SB, SB, &full[s]);
        if (++s == S) { s = 0; par ^= 1u; }
      }
    }
  } else {
    // ---- compute warps ------------------------------------------------------
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
    // rows of the logits this thread finalises: (r, m) = (tid % 16, tid / 16)
    const int fr = threadIdx.x & 15, fm = threadIdx.x >> 4;
    float best_v = -INFINITY;
    int best_i = 0x7fffffff;
    int s = 0, part = 0, tile = tb;
    unsigned par = 0;
    for (int f = 0; f < nf; ++f) {
      // on a time-out the loop keeps its shape (no further waits) so the
      // tile-end barriers below still match across the compute warps
      mbar_wait_or_fail(&full[s], par, &s_fail);
      const unsigned char* stage = ring + (size_t)s * SB;
      for (int jj = 0; jj < k16_per_warp; ++jj) {
        const int j = warp * k16_per_warp + jj;          // k16-tile within the stage
        const int kk = part * k16_per_stage + j;         // k16-tile within the row tile
        const uint4 wv = *reinterpret_cast<const uint4*>(stage + (size_t)(j * 32 + lane) * 16);
        const uint32_t af[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int row = nt * 8 + g;
          uint32_t b0 = 0, b1 = 0, c0 = 0, c1 = 0;
          if (row < M) {
            const size_t off = (size_t)row * ldxs + kk * 16 + 2 * t;
            b0 = *reinterpret_cast<const uint32_t*>(xs + off);
            b1 = *reinterpret_cast<const uint32_t*>(xs + off + 8);
            c0 = *reinterpret_cast<const uint32_t*>(xl + off);
            c1 = *reinterpret_cast<const uint32_t*>(xl + off + 8);
          }
          mma_f16_16816(acc[nt], af, b0, b1);
          mma_f16_16816(acc[nt], af, c0, c1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (++s == S) { s = 0; par ^= 1u; }
      if (part == spt - 1) {  // row tile done: combine the warps, logits, best
        float* myred = red + warp * 16 * 16;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int col = nt * 8 + 2 * t;
          myred[g * 16 + col] = acc[nt][0];
          myred[g * 16 + col + 1] = acc[nt][1];
          myred[(g + 8) * 16 + col] = acc[nt][2];
          myred[(g + 8) * 16 + col + 1] = acc[nt][3];
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
        }
        asm volatile("bar.sync 1, %0;" ::"r"(kHeadWarps * 32) : "memory");
        if (fm < M && fm < NC) {
          float v = 0.f;
#pragma unroll
          for (int w = 0; w < kHeadWarps; ++w) v += red[w * 256 + fr * 16 + fm];
          const int row = tile * 16 + fr;
          if (logits) logits[(size_t)(a.out_row ? a.out_row[fm] : fm) * a.V + row] = v;
          if (better(v, row, best_v, best_i)) { best_v = v; best_i = row; }
        }
        asm volatile("bar.sync 1, %0;" ::"r"(kHeadWarps * 32) : "memory");
        part = 0;
        ++tile;
      } else {
        ++part;
      }
    }
    if (fm < 16) { s_val[fm][fr] = best_v; s_idx[fm][fr] = best_i; }
  }
  __syncthreads();
  if (s_fail) {
    if (threadIdx.x == 0) atomicOr(a.err_flag, kErrTimeout);
    return;
  }
  if (!argmax) return;
  if (threadIdx.x < M) {
    const int m = threadIdx.x;
    float v = s_val[m][0];
    int ix = s_idx[m][0];
    for (int r = 1; r < 16; ++r)
      if (better(s_val[m][r], s_idx[m][r], v, ix)) { v = s_val[m][r]; ix = s_idx[m][r]; }
    a.part_val[blockIdx.x * 16 + m] = v;
    a.part_idx[blockIdx.x * 16 + m] = ix;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(a.ticket, 1u) == gridDim.x - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (threadIdx.x < M) {
    const int m = threadIdx.x;
    float v = -INFINITY;
    int ix = 0x7fffffff;
    for (int c = 0; c < (int)gridDim.x; ++c) {
      const float pv = __ldcg(a.part_val + c * 16 + m);
      const int pi = __ldcg(a.part_idx + c * 16 + m);
      if (better(pv, pi, v, ix)) { v = pv; ix = pi; }
    }
    argmax[a.out_row ? a.out_row[m] : m] = ix;
  }
  if (threadIdx.x == 0) *a.ticket = 0u;
}

// ---- output norm + head + argmax for up to 4 rows, direct loads -----------
// One CTA per SM, 16 warps.  Warp w of CTA c owns the 16-row head tiles
// w * P + c, then every P * 16 after that, and streams each whole tile
// (64 KB at d = 2048, in A-fragment order: lane l's 16-byte word of k16
// chunk j is exactly its m16n8k16 A operand) with plain 16-byte loads in
// batches of eight per lane, two batches in flight, marked L2 evict-first (the head is read once per token
// and must not push the loop block out of L2).  The first loads go out
// before the wait on the previous kernel.  The B operand is the normalised
// activation as fp16 (hi, lo) pairs from shared memory (columns 2t / 2t + 1
// = hi / lo of row t), so lane (g, t) ends a tile holding the logits of
// vocabulary rows g and g + 8 for row t: no cross-warp reduction per tile.
// The greedy argmax (lowest index on ties) is reduced per warp, per CTA and
// by the last CTA (ticket).  Timeline (when `trace` is set, G = grid entries
// per slot): slot 0 start, 1 activations staged, 2 tiles done, 3 end.
constexpr int kHdWarps = 16;
constexpr int kHdThreads = kHdWarps * 32;
constexpr int kHdMaxRows = 4;
constexpr int kHdUnroll = 8;
constexpr int kHdXChunks = 4;   // float4 columns per thread and row: d <= 8192

__host__ __device__ inline size_t head_direct_smem(int d) { return (size_t)2 * kHdMaxRows * (d + 8) * 2; }

__device__ __forceinline__ uint4 ldg_evict_first(const uint4* p, uint64_t pol) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p), "l"(pol));
  return r;
}

__global__ void __launch_bounds__(kHdThreads, 1) head_direct_kernel(const HeadArgs a, unsigned long long* trace,
                                                                    long long trace_cap) {
  extern __shared__ __align__(16) unsigned char hsm[];
  __shared__ float s_ss[kHdMaxRows][kHdWarps];
  __shared__ float s_bv[kHdMaxRows][kHdWarps];
  __shared__ int s_bi[kHdMaxRows][kHdWarps];
  __shared__ int s_last;
  const int d = a.d, M = a.M, ldx = d + 8;
  __half* xs = reinterpret_cast<__half*>(hsm);      // hi [kHdMaxRows][ldx]
  __half* xl = xs + (size_t)kHdMaxRows * ldx;       // lo
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x, P = gridDim.x;
  const int g = lane >> 2, t = lane & 3;
  const int nt = a.V >> 4, nk16 = d >> 4;
  auto stamp = [&](int slot) {
    if (trace && threadIdx.x == 0) {
      const long long i = (long long)slot * P + c;
      if (i < trace_cap) trace[i] = (unsigned long long)globaltimer_ns();
    }
  };
  stamp(0);
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  // warp-major order: every CTA gets a tile for its warp w before any CTA's
  // warp w + 1 does, so all SMs stream (+-1 tile) even when the tiles do not
  // fill every warp
  const int stride = P * kHdWarps;
  int tile = warp * P + c;
  uint4 wv[kHdUnroll];
  if (tile < nt) {   // the weights do not depend on earlier kernels
    const uint4* wt = a.w + (size_t)tile * nk16 * 32 + lane;
#pragma unroll
    for (int u = 0; u < kHdUnroll; ++u) wv[u] = ldg_evict_first(wt + u * 32, pol);
  }
  // the gains of this thread's columns and the zero rows >= M do not depend
  // on earlier kernels either; each thread owns columns 4 * (tid + i * T) ..
  // + 3 of every row (d <= kHdXChunks * 4 * T)
  uint2 gr[kHdXChunks];
#pragma unroll
  for (int i = 0; i < kHdXChunks; ++i) {
    const int k = (threadIdx.x + i * kHdThreads) * 4;
    gr[i] = k < d ? *reinterpret_cast<const uint2*>(a.gain + k) : make_uint2(0u, 0u);
  }
  for (int e = threadIdx.x; e < (kHdMaxRows - M) * (d / 2); e += kHdThreads) {
    const int m = M + e / (d / 2), k = (e % (d / 2)) * 2;
    *reinterpret_cast<uint32_t*>(xs + (size_t)m * ldx + k) = 0u;
    *reinterpret_cast<uint32_t*>(xl + (size_t)m * ldx + k) = 0u;
  }
  pdl_trigger();
  pdl_wait();
  float* const logits = a.io ? a.io->logits : a.logits;
  int32_t* const argmax = a.io ? a.io->argmax : a.argmax;

  // RMSNorm of the M rows, staged as fp16 (hi, lo): every row's loads go out
  // together, then one block reduction of the sums of squares
  float4 xr[kHdMaxRows][kHdXChunks];
#pragma unroll
  for (int m = 0; m < kHdMaxRows; ++m) {
#pragma unroll
    for (int i = 0; i < kHdXChunks; ++i) {
      const int k = (threadIdx.x + i * kHdThreads) * 4;
      xr[m][i] = (m < M && k < d) ? *reinterpret_cast<const float4*>(a.x + (size_t)m * d + k)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
#pragma unroll
  for (int m = 0; m < kHdMaxRows; ++m) {
    if (m < M) {
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < kHdXChunks; ++i) {
        const float4 v = xr[m][i];
        ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
      }
      ss = warp_sum(ss);
      if (lane == 0) s_ss[m][warp] = ss;
    }
  }
  __syncthreads();
#pragma unroll
  for (int m = 0; m < kHdMaxRows; ++m) {
    if (m < M) {
      float tot = 0.f;
#pragma unroll
      for (int w = 0; w < kHdWarps; ++w) tot += s_ss[m][w];
      const float rs = 1.0f / sqrtf(tot / (float)d + a.eps);
#pragma unroll
      for (int i = 0; i < kHdXChunks; ++i) {
        const int k = (threadIdx.x + i * kHdThreads) * 4;
        if (k < d) {
          const float xv[4] = {xr[m][i].x, xr[m][i].y, xr[m][i].z, xr[m][i].w};
          const uint32_t gw[2] = {gr[i].x, gr[i].y};
          uint32_t hw[2], lw[2];
#pragma unroll
          for (int p = 0; p < 2; ++p) {
            const float2 gv = __half22float2(*reinterpret_cast<const __half2*>(&gw[p]));
            const float y0 = xv[2 * p] * rs * gv.x, y1 = xv[2 * p + 1] * rs * gv.y;
            const __half2 h = __floats2half2_rn(y0, y1);
            const float2 r = __half22float2(h);
            const __half2 l = __floats2half2_rn(y0 - r.x, y1 - r.y);
            hw[p] = *reinterpret_cast<const uint32_t*>(&h);
            lw[p] = *reinterpret_cast<const uint32_t*>(&l);
          }
          *reinterpret_cast<uint2*>(xs + (size_t)m * ldx + k) = make_uint2(hw[0], hw[1]);
          *reinterpret_cast<uint2*>(xl + (size_t)m * ldx + k) = make_uint2(lw[0], lw[1]);
        }
      }
    }
  }
  __syncthreads();
  stamp(1);

  const __half* bsrc = ((g & 1) ? xl : xs) + (size_t)(g >> 1) * ldx + 2 * t;
  float best_v = -INFINITY;
  int best_i = 0x7fffffff;
  bool have = tile < nt;   // wv holds the first batch of `tile`
  // batches of kHdUnroll k16 chunks in two register sets used in turn (no
  // copies between them, which would wait for the loads): while one set
  // multiplies, the other set's loads are in flight
  const int nb = nk16 / kHdUnroll;   // d is a multiple of 128
  for (; tile < nt; tile += stride) {
    const uint4* wt = a.w + (size_t)tile * nk16 * 32 + lane;
    float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc2[4] = {0.f, 0.f, 0.f, 0.f};
    auto load = [&](uint4 (&v)[kHdUnroll], int b) {
#pragma unroll
      for (int u = 0; u < kHdUnroll; ++u) v[u] = ldg_evict_first(wt + (size_t)(b * kHdUnroll + u) * 32, pol);
    };
    auto mul = [&](const uint4 (&v)[kHdUnroll], int b) {
#pragma unroll
      for (int u = 0; u < kHdUnroll; ++u) {
        const int j = b * kHdUnroll + u;
        const uint32_t af[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(bsrc + j * 16);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(bsrc + j * 16 + 8);
        if (u & 1) mma_f16_16816(acc2, af, b0, b1);
        else mma_f16_16816(acc, af, b0, b1);
      }
    };
    if (!have) load(wv, 0);
    have = false;
    uint4 nv[kHdUnroll];
    for (int b = 0; b < nb; b += 2) {
      if (b + 1 < nb) load(nv, b + 1);
      mul(wv, b);
      if (b + 2 < nb) load(wv, b + 2);
      if (b + 1 < nb) mul(nv, b + 1);
    }
    // lane (g, t): columns 2t (hi) and 2t + 1 (lo) of row t
    const float v0 = (acc[0] + acc2[0]) + (acc[1] + acc2[1]);
    const float v1 = (acc[2] + acc2[2]) + (acc[3] + acc2[3]);
    if (t < M) {
      const int r0 = tile * 16 + g, r1 = r0 + 8;
      if (logits) {
        const size_t o = (size_t)(a.out_row ? a.out_row[t] : t) * a.V;
        logits[o + r0] = v0;
        logits[o + r1] = v1;
      }
      if (better(v0, r0, best_v, best_i)) { best_v = v0; best_i = r0; }
      if (better(v1, r1, best_v, best_i)) { best_v = v1; best_i = r1; }
    }
  }
  // best per row: lanes of equal t, then warps, then CTAs
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, best_v, o);
    const int oi = __shfl_xor_sync(0xffffffffu, best_i, o);
    if (better(ov, oi, best_v, best_i)) { best_v = ov; best_i = oi; }
  }
  if (lane < kHdMaxRows) { s_bv[lane][warp] = best_v; s_bi[lane][warp] = best_i; }
  __syncthreads();
  stamp(2);
  if (threadIdx.x < M) {
    const int m = threadIdx.x;
    float v = s_bv[m][0];
    int ix = s_bi[m][0];
    for (int w = 1; w < kHdWarps; ++w)
      if (better(s_bv[m][w], s_bi[m][w], v, ix)) { v = s_bv[m][w]; ix = s_bi[m][w]; }
    a.part_val[c * 16 + m] = v;
    a.part_idx[c * 16 + m] = ix;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(a.ticket, 1u) == (unsigned)(P - 1);
  __syncthreads();
  if (s_last) {
    __threadfence();
    if (argmax && warp < M) {
      float v = -INFINITY;
      int ix = 0x7fffffff;
      for (int cc = lane; cc < P; cc += 32) {
        const float pv = __ldcg(a.part_val + cc * 16 + warp);
        const int pi = __ldcg(a.part_idx + cc * 16 + warp);
        if (better(pv, pi, v, ix)) { v = pv; ix = pi; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, o);
        const int oi = __shfl_xor_sync(0xffffffffu, ix, o);
        if (better(ov, oi, v, ix)) { v = ov; ix = oi; }
      }
      if (lane == 0) argmax[a.out_row ? a.out_row[warp] : warp] = ix;
    }
    if (threadIdx.x == 0) *a.ticket = 0u;
  }
  stamp(3);
}

}  // namespace tl
