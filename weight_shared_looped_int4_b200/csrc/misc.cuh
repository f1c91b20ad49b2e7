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
    if (threadIdx.x == 0) atomicOr(err_flag, 1);
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

struct HeadArgs {
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
};

constexpr int kHeadThreads = 256;
constexpr int kGemvPrefetchHead = 8;  // 16-byte loads in flight per lane

__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

// Activation planes (hi, lo) of M rows.
__host__ __device__ inline size_t head_smem_bytes(int d, int M) {
  return (size_t)M * (d + 8) * 2 * 2;
}

// One warp per 16-row tile over all of K; the CTA's 8 warps take 8
// consecutive tiles.  The output norm is computed per CTA in the prologue and
// kept as an fp16 pair (hi, lo) like the INT4 GEMV's activations.
template <int NT>
__global__ void __launch_bounds__(kHeadThreads) head_argmax_kernel(const HeadArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ float s_val[8][16];
  __shared__ int s_idx[8][16];
  __shared__ int s_last;
  const int d = a.d, ldxs = d + 8, M = a.M;
  __half* xs = reinterpret_cast<__half*>(smem);
  __half* xl = xs + (size_t)M * ldxs;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int n_tiles = a.V >> 4;
  const int tile = blockIdx.x * 8 + warp;
  const int nk = d >> 4;
  const uint4* wp = a.w + (size_t)tile * nk * 32 + lane;
  const bool has_tile = tile < n_tiles;

  pdl_trigger();
  uint4 buf[kGemvPrefetchHead];
#pragma unroll
  for (int i = 0; i < kGemvPrefetchHead; ++i)
    if (has_tile && i < nk) buf[i] = ldg_stream(wp + (size_t)i * 32);
  pdl_wait();

  // output RMSNorm of every row into shared memory as an fp16 pair
  for (int m = warp; m < M; m += 8) {
    const float* src = a.x + (size_t)m * d;
    float ss = 0.f;
    for (int k = lane * 4; k < d; k += 128) {
      const float4 v = *reinterpret_cast<const float4*>(src + k);
      ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
    ss = warp_sum(ss);
    const float rs = 1.0f / sqrtf(ss / (float)d + a.eps);
    for (int k = lane * 4; k < d; k += 128) {
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
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;

  if (has_tile) {
    for (int base = 0; base < nk; base += kGemvPrefetchHead) {
#pragma unroll
      for (int i = 0; i < kGemvPrefetchHead; ++i) {
        const int kk = base + i;
        if (kk < nk) {
          const uint4 wv = buf[i];
          if (kk + kGemvPrefetchHead < nk) buf[i] = ldg_stream(wp + (size_t)(kk + kGemvPrefetchHead) * 32);
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
      }
    }
  }

  // logits and per-warp best per row (column of the MMA output)
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int m = nt * 8 + 2 * t + c;
      const int ra = tile * 16 + g, rb = ra + 8;
      const float va = acc[nt][c], vb = acc[nt][2 + c];
      if (has_tile && m < M && a.logits) {
        const int orow = a.out_row ? a.out_row[m] : m;
        a.logits[(size_t)orow * a.V + ra] = va;
        a.logits[(size_t)orow * a.V + rb] = vb;
      }
      float bv = va;
      int bi = ra;
      if (better(vb, rb, bv, bi)) { bv = vb; bi = rb; }
      if (!has_tile) { bv = -INFINITY; bi = 0x7fffffff; }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
      }
      if (g == 0) { s_val[warp][m] = bv; s_idx[warp][m] = bi; }
    }
  }
  __syncthreads();

  if (!a.argmax) return;
  if (threadIdx.x < M) {
    const int m = threadIdx.x;
    float bv = s_val[0][m];
    int bi = s_idx[0][m];
    for (int w = 1; w < 8; ++w)
      if (better(s_val[w][m], s_idx[w][m], bv, bi)) { bv = s_val[w][m]; bi = s_idx[w][m]; }
    a.part_val[blockIdx.x * 16 + m] = bv;
    a.part_idx[blockIdx.x * 16 + m] = bi;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(a.ticket, 1u) == gridDim.x - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (threadIdx.x < a.M) {
    const int m = threadIdx.x;
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int c = 0; c < (int)gridDim.x; ++c) {
      const float v = __ldcg(a.part_val + c * 16 + m);
      const int i = __ldcg(a.part_idx + c * 16 + m);
      if (better(v, i, bv, bi)) { bv = v; bi = i; }
    }
    a.argmax[a.out_row ? a.out_row[m] : m] = bi;
  }
  if (threadIdx.x == 0) *a.ticket = 0u;
}

}  // namespace tl
