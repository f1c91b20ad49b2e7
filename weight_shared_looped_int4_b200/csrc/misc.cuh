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

constexpr int kHeadThreads = 256;
constexpr int kHeadChunk = 4096;   // bytes per bulk copy: 8 k16-tiles of one 16-row tile

__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

// Ring stages per warp: deeper when the activation planes are small.
__host__ __device__ inline int head_stages(int M) { return M <= 8 ? 4 : 2; }

// Dynamic shared memory: per-warp rings, then the activation planes (hi, lo).
__host__ __device__ inline size_t head_smem_bytes(int d, int M) {
  return (size_t)8 * head_stages(M) * kHeadChunk + (size_t)M * (d + 8) * 2 * 2;
}

// One CTA per SM.  Global warp w takes 16-row tiles w, w + W, w + 2W, ...
// (W = warps in the grid) over all of K.  Its tiles stream through a private
// ring of S shared-memory stages, each filled by one 4 KB bulk asynchronous
// copy (the TMA engine) that completes on an mbarrier, so a warp keeps S * 4 KB
// in flight without spending registers on it; the first copies are issued
// before griddepcontrol.wait.  The output norm is computed by every CTA in the
// prologue and kept as an fp16 pair (hi, lo) like the INT4 GEMV's activations.
// Each warp keeps its best (value, index) per row; CTAs combine warps, and the
// last CTA to finish (atomic ticket) combines CTAs.  Ties go to the lowest
// index, so the result does not depend on the order of combination.  Every
// wait is bounded: on time-out the kernel sets kErrTimeout and stops.
template <int NT>
__global__ void __launch_bounds__(kHeadThreads, 1) head_argmax_kernel(const HeadArgs a) {
  constexpr int S = NT == 1 ? 4 : 2;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t bars[8][4];
  __shared__ float s_val[8][16];
  __shared__ int s_idx[8][16];
  __shared__ float s_ss[16][8];
  __shared__ int s_last;
  const int d = a.d, ldxs = d + 8, M = a.M;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  unsigned char* ring = smem + (size_t)warp * S * kHeadChunk;
  __half* xs = reinterpret_cast<__half*>(smem + (size_t)8 * S * kHeadChunk);
  __half* xl = xs + (size_t)M * ldxs;
  const int n_tiles = a.V >> 4;
  const int nk = d >> 4;                      // k16-tiles per row tile
  const int cpt = nk / 8;                     // 4 KB chunks per row tile
  const int GW = gridDim.x * 8;
  const int gw = blockIdx.x * 8 + warp;
  const int my_tiles = gw < n_tiles ? (n_tiles - 1 - gw) / GW + 1 : 0;
  const int nf = my_tiles * cpt;              // chunks this warp streams
  uint64_t* bar = bars[warp];
  auto chunk_src = [&](int f) {
    const int tile = gw + (f / cpt) * GW;
    return reinterpret_cast<const unsigned char*>(a.w) + ((size_t)tile * cpt + (f % cpt)) * kHeadChunk;
  };

  pdl_trigger();
  if (lane == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&bar[s], 1);
    fence_mbar_init();
    for (int s = 0; s < S && s < nf; ++s) {
      mbar_arrive_expect_tx(&bar[s], kHeadChunk);
      bulk_g2s(ring + s * kHeadChunk, chunk_src(s), kHeadChunk, &bar[s]);
    }
  }
  __syncwarp();
  pdl_wait();

  // output RMSNorm of every row into shared memory as an fp16 pair
  for (int m = 0; m < M; ++m) {
    const float* src = a.x + (size_t)m * d;
    float ss = 0.f;
#pragma unroll 4
    for (int k = threadIdx.x * 4; k < d; k += 4 * kHeadThreads) {
      const float4 v = *reinterpret_cast<const float4*>(src + k);
      ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
    ss = warp_sum(ss);
    if (lane == 0) s_ss[m][warp] = ss;
  }
  __syncthreads();
  for (int m = 0; m < M; ++m) {
    const float* src = a.x + (size_t)m * d;
    float ss = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) ss += s_ss[m][w];
    const float rs = 1.0f / sqrtf(ss / (float)d + a.eps);
#pragma unroll 4
    for (int k = threadIdx.x * 4; k < d; k += 4 * kHeadThreads) {
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

  float acc[NT][4];
  float bv[NT][2];
  int bi[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
    bv[nt][0] = bv[nt][1] = -INFINITY;
    bi[nt][0] = bi[nt][1] = 0x7fffffff;
  }

  float* const logits = a.io ? a.io->logits : a.logits;
  int32_t* const argmax = a.io ? a.io->argmax : a.argmax;
  bool ok = true;
  for (int f = 0; f < nf && ok; ++f) {
    const int s = f % S;
    if (!mbar_wait(&bar[s], (unsigned)((f / S) & 1))) {
      ok = false;
      if (lane == 0) atomicOr(a.err_flag, kErrTimeout);
      break;
    }
    const unsigned char* stage = ring + s * kHeadChunk;
    const int kk0 = (f % cpt) * 8;   // first k16-tile of this chunk within the row tile
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint4 wv = *reinterpret_cast<const uint4*>(stage + (j * 32 + lane) * 16);
      const uint32_t af[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int row = nt * 8 + g;
        uint32_t b0 = 0, b1 = 0, c0 = 0, c1 = 0;
        if (row < M) {
          const size_t off = (size_t)row * ldxs + (kk0 + j) * 16 + 2 * t;
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
    if (lane == 0 && f + S < nf) {  // refill this stage
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&bar[s], kHeadChunk);
      bulk_g2s(ring + s * kHeadChunk, chunk_src(f + S), kHeadChunk, &bar[s]);
    }
    if ((f + 1) % cpt == 0) {  // row tile done: logits and running best
      const int tile = gw + (f / cpt) * GW;
      const int ra = tile * 16 + g, rb = ra + 8;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int m = nt * 8 + 2 * t + c;
          const float va = acc[nt][c], vb = acc[nt][2 + c];
          if (m < M && logits) {
            const int orow = a.out_row ? a.out_row[m] : m;
            logits[(size_t)orow * a.V + ra] = va;
            logits[(size_t)orow * a.V + rb] = vb;
          }
          if (better(va, ra, bv[nt][c], bi[nt][c])) { bv[nt][c] = va; bi[nt][c] = ra; }
          if (better(vb, rb, bv[nt][c], bi[nt][c])) { bv[nt][c] = vb; bi[nt][c] = rb; }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[nt][q] = 0.f;
      }
    }
  }
  if (!ok) {  // drain the copies still in flight (bounded), then stop
    if (lane == 0)
      for (int s = 0; s < S; ++s) (void)mbar_try_wait(&bar[s], 0);
    return;
  }

  // best per row across the lanes of the warp, then across warps
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      float v = bv[nt][c];
      int ix = bi[nt][c];
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, o);
        const int oi = __shfl_xor_sync(0xffffffffu, ix, o);
        if (better(ov, oi, v, ix)) { v = ov; ix = oi; }
      }
      if (g == 0) { s_val[warp][nt * 8 + 2 * t + c] = v; s_idx[warp][nt * 8 + 2 * t + c] = ix; }
    }
  }
  __syncthreads();

  if (!argmax) return;
  if (threadIdx.x < M) {
    const int m = threadIdx.x;
    float v = s_val[0][m];
    int ix = s_idx[0][m];
    for (int w = 1; w < 8; ++w)
      if (better(s_val[w][m], s_idx[w][m], v, ix)) { v = s_val[w][m]; ix = s_idx[w][m]; }
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

}  // namespace tl
