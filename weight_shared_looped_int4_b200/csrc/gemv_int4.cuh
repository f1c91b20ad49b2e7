// INT4 group-wise dequant GEMV for the decode path (and short prefill chunks):
// y[m][n] = sum_k x[m][k] * (q[n][k] - z[n][k/128]) * s[n][k/128], m < 16.
//
// Definition: TinyLoop README, "Status" (INT4 loop / pre linears with zero
// points); the group size, fp16 scale and 4-bit zero are the workload's
// w = (q - z) * s.  The kernel design is ours, for sm_100a:
//
// * Weights are re-laid out at load time so that one 16-byte load of a lane
//   holds the A fragments of four m16n8k16 MMAs (64 consecutive k of rows g
//   and g+8 of a 16-row tile).  A warp load is 512 contiguous bytes.
// * Unpacking is a LOP3 per nibble pair (the 1024-bias trick) and one fp16
//   subtract of the biased zero point; q - z is an exact small integer in fp16,
//   so the tensor-core product with the fp16 activation is exact and the MMA
//   accumulates in fp32.  The fp16 scale is applied in fp32 once per 64-wide
//   K chunk, so no weight is ever rounded.
// * A CTA owns TPC 16-row tiles and all of K.  With TPC = 2 the two tiles are
//   the pair an epilogue needs (RoPE halves of one head, gate/up rows of
//   SwiGLU) and the 8 warps split (tile, K quarter); with TPC = 1 (residual
//   and plain outputs) the 8 warps split K eight ways, which doubles the CTA
//   count of the small projections.  Partial sums are reduced through shared
//   memory in a fixed order, so results are deterministic and each activation
//   row's result does not depend on how many rows share the launch.
// * Weight prefetch is issued before griddepcontrol.wait, so it overlaps the
//   tail of the previous kernel under programmatic dependent launch (the
//   caller picks where the kernel releases its own dependent: PdlTrigger).
// * fp32 activations are split into an fp16 pair x = hi + lo (lo is the fp16
//   rounding of x - hi) and both halves go through the MMA, so the product
//   keeps about 22 bits of the activation instead of fp16's 11.  The looped
//   model amplifies rounding across iterations, and fp16 activations alone
//   move its logits by several 1e-2.
// * The prologue can fuse the block's RMSNorm (fp32 residual in, fp16 pair
//   out into shared memory); the epilogue fuses RoPE + KV-cache write, SwiGLU,
//   or the residual add.
#pragma once

#include "common.cuh"

namespace tl {

// IN_F32W: IN_F32 for long rows (the down projection's input), staged with
// every load of a row in flight at once; its extra registers would keep the
// dependent kernel's CTAs off the SMs if the O projection used it too.
enum GemvIn { IN_NORM = 0, IN_F16 = 1, IN_F32 = 2, IN_F32W = 3 };
enum GemvEpi { EPI_STORE = 0, EPI_RESID = 1, EPI_SWIGLU = 2, EPI_ROPE_KV = 3 };
enum PairMode { PAIR_NEIGHBOUR = 0, PAIR_OFFSET = 1, PAIR_ROPE = 2 };
// When the kernel lets the next kernel of the stream launch (programmatic
// dependent launch).  A dependent launched early prefetches its weights
// during this kernel, but its CTAs land wherever this kernel's leave room,
// several on one SM at times; measured on the decode step, the gate_up ->
// down hand-off is faster with the trigger after the main loop.
enum PdlTrigger { TRIGGER_AT_START = 0, TRIGGER_AFTER_LOOP = 1 };

struct GemvArgs {
  const uint4* w;      // tiled weights  [n_tiles][K/64][32] (see repack)
  const uint2* sz;     // scales / zeros [n_tiles][K/128][8]
  int K;               // multiple of 128
  int n_rows;          // valid output rows N
  int M;               // activation rows, 1..16
  // input
  const float* x;      // IN_NORM / IN_F32: fp32 [M][ldx]
  const __half* xh;    // IN_F16:  fp16 [M][ldx]
  int ldx;
  const __half* gain;  // IN_NORM: RMSNorm gains [K]
  float eps;
  // tile pairing
  int pair_mode;
  int pair_off;        // PAIR_OFFSET: tiles between the two; PAIR_ROPE: hd/32
  // outputs
  __half* y;           // EPI_STORE: fp16 [M][ldy]
  float* yf;           // EPI_SWIGLU: fp32 [M][ldy]
  int ldy;
  float* resid;        // EPI_RESID: fp32 [M][ldr] += y
  int ldr;
  // EPI_ROPE_KV
  float* q_out;        // fp32 [M][ldq], rows < n_q_rows
  int ldq;
  int n_q_rows;        // Hq * hd
  int n_kv_rows;       // Hkv * hd
  int hd;
  __half* k_plane;     // K plane of this layer for lane 0: [Hkv][ctx][hd]
  __half* v_plane;     // V plane of this layer for lane 0
  float* kv_stage;     // INT8 KV cache: the rotated keys and the values go here
                       // in fp32, [row][K|V][Hkv][hd], for the quantising pass
                       // (k_plane / v_plane unused); NULL: fp16 cache
  long long lane_stride;
  int ctx;
  const RowCtx* rows;  // per activation row
  float theta;
  const float2* rope_tab;  // (cos, sin) [positions][hd/2], or NULL
  int* err_flag;       // device fault flags (a bounded wait gave up)
  unsigned long long* trace;  // launch timeline (kTraceEvents entries) or NULL:
                              // released, weights arrived, main loop done,
                              // (6) activations staged
  int trigger;                // PdlTrigger
  int l2_keep;                // 1: the weights are the loop block's (L2 evict-last), else evict-first
  int bits;                   // 4, or 2: INT2 weights (selects gemv_int4_kernel<.., 2>)
  // L2 prefetch issued at the start (pf NULL: none): pf_count pieces of
  // pf_piece bytes (a multiple of 16, at most 32 KB) at pf + i * pf_stride,
  // dealt over the CTAs -- the start of every head tile, read from HBM while
  // the loop block runs from L2 and HBM is otherwise idle
  const unsigned char* pf;
  int pf_count;
  unsigned pf_piece;
  size_t pf_stride;
};

constexpr int kGemvThreads = 256;

// Shared memory of a CTA: its weight tiles and scales (bulk-copied), the
// activation planes (hi, and lo unless IN_F16) of M rows, the K-slice
// reduction buffer and the RMSNorm partial sums.
__host__ __device__ inline size_t gemv_act_bytes(int K, int M, bool lo) {
  return (((size_t)M * (K + 8) * 2 * (lo ? 2 : 1)) + 15) / 16 * 16;
}
// INT4: 16 bytes per lane per 64-k chunk; INT2: 8
__host__ __device__ inline size_t gemv_w_bytes(int K, int bits = 4) { return (size_t)(K >> 6) * (bits == 2 ? 256 : 512); }
__host__ __device__ inline size_t gemv_sz_bytes(int K) { return (size_t)(K >> 7) * 64; }
// Activation planes of gemv_rows_kernel: kGemvPhaseK columns per phase.
constexpr int kGemvPhaseK = 512;
__host__ __device__ inline size_t gemv_rows_act_bytes(int M, bool lo) {
  return (((size_t)M * (kGemvPhaseK + 8) * 2 * (lo ? 2 : 1)) + 15) / 16 * 16;
}
__host__ __device__ inline int gemv_nt(int M, bool lo);
__host__ __device__ inline size_t gemv_smem_bytes(int K, int M, bool lo, int tpc) {
  const int nc = M <= 8 ? 8 : 16;
  const size_t act = gemv_nt(M, lo) == 0 ? gemv_act_bytes(K, M, lo) : gemv_rows_act_bytes(M, lo);
  return (size_t)tpc * (gemv_w_bytes(K) + gemv_sz_bytes(K)) + act + (size_t)8 * 16 * nc * 4 + 16 * 8 * 4;
}

// Tiles per CTA of each epilogue.
__host__ __device__ constexpr int gemv_tpc(int epi) {
  return (epi == EPI_ROPE_KV || epi == EPI_SWIGLU) ? 2 : 1;
}

// MMA column layouts.  NT = 0: one MMA per k16 tile; with the fp16 pair the
// B columns are (row m hi, row m lo) for m < 4, otherwise columns are rows
// m < 8.  NT = 1: rows m < 8, hi and lo in two MMAs.  NT = 2: rows m < 16.
__host__ __device__ inline int gemv_nt(int M, bool lo) {
  if (M <= (lo ? 4 : 8)) return 0;
  return M <= 8 ? 1 : 2;
}

// BITS: 4 (INT4 weights) or 2 (INT2 body: half the weight bytes, the A
// fragments of two k16 steps per 32-bit word, unpack_a_frag2).
template <int NT, int IN, int EPI, int BITS = 4>
__global__ void __launch_bounds__(kGemvThreads) gemv_int4_kernel(const GemvArgs a) {
  constexpr bool LO = (IN != IN_F16);
  constexpr int TPC = gemv_tpc(EPI);
  constexpr int KS = 8 / TPC;                 // K slices
  constexpr int NC = NT == 2 ? 16 : 8;        // reduction columns
  constexpr int NTILES = NT == 2 ? 2 : 1;     // n8 tiles of the MMA
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t wbar;
  __shared__ int s_ok;
  const int K = a.K;
  const int M = a.M;
  const int ldxs = K + 8;
  const int n_chunks = K >> 6;
  const size_t wt_bytes = gemv_w_bytes(K, BITS), sz_bytes = gemv_sz_bytes(K);
  unsigned char* sw = smem;                                       // [TPC][chunks][32][16 B]
  unsigned char* ssz = smem + TPC * wt_bytes;                     // [TPC][groups][8][8 B]
  __half* xs = reinterpret_cast<__half*>(ssz + TPC * sz_bytes);   // hi plane [M][ldxs]
  __half* xl = xs + (size_t)M * ldxs;                             // lo plane [M][ldxs]
  float* red = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(xs) + gemv_act_bytes(K, M, LO));
  float* ssq = red + 8 * 16 * NC;                                 // [16 rows][8 warps]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int tsel = TPC == 2 ? (warp & 1) : 0;
  const int kq = TPC == 2 ? (warp >> 1) : warp;

  int t0, t1;
  if (TPC == 1) {
    t0 = blockIdx.x;
    t1 = t0;
  } else if (a.pair_mode == PAIR_OFFSET) {
    t0 = blockIdx.x;
    t1 = t0 + a.pair_off;
  } else {
    const int head = blockIdx.x / a.pair_off, j16 = blockIdx.x % a.pair_off;
    t0 = head * 2 * a.pair_off + j16;
    t1 = t0 + a.pair_off;
  }

  trace_start(a.trace);
  if (a.trigger == TRIGGER_AT_START) pdl_trigger();
  // The weights do not depend on earlier kernels: start their bulk copies
  // before waiting for the previous kernel.
  if (threadIdx.x == 0) {
    mbar_init(&wbar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&wbar, (unsigned)(TPC * (wt_bytes + sz_bytes)));
    const uint64_t pol = a.l2_keep ? l2_evict_last() : l2_evict_first();
    for (int ts = 0; ts < TPC; ++ts) {
      const int tile = ts ? t1 : t0;
      const unsigned char* src = reinterpret_cast<const unsigned char*>(a.w) + (size_t)tile * wt_bytes;
      for (size_t off = 0; off < wt_bytes; off += 32768) {
        const unsigned n = (unsigned)((wt_bytes - off) < 32768 ? (wt_bytes - off) : 32768);
        bulk_g2s_hint(sw + ts * wt_bytes + off, src + off, n, &wbar, pol);
      }
      bulk_g2s_hint(ssz + ts * sz_bytes, reinterpret_cast<const unsigned char*>(a.sz) + (size_t)tile * sz_bytes,
                    (unsigned)sz_bytes, &wbar, pol);
    }
  }

  if (a.pf && threadIdx.x == 32)
    for (int i = blockIdx.x; i < a.pf_count; i += gridDim.x) bulk_prefetch_l2(a.pf + i * a.pf_stride, a.pf_piece);

  pdl_wait();
  trace_mark(a.trace, 2);

  // ---- stage the activations: fp16 pair (hi, lo) of the fp32 input --------
  if (IN == IN_F16) {
    for (int m = 0; m < M; ++m) {
      __half* dst = xs + m * ldxs;
      const __half* src = a.xh + (size_t)m * a.ldx;
#pragma unroll 4
      for (int k = threadIdx.x * 8; k < K; k += 8 * kGemvThreads)
        *reinterpret_cast<uint4*>(dst + k) = *reinterpret_cast<const uint4*>(src + k);
    }
  } else if (IN == IN_NORM && M <= 4 && K <= 8 * kGemvThreads) {
    // few short rows: one pass, the row values and gains stay in registers
    // (one round trip to L2 instead of two)
    float4 xv[4][2];
    uint2 gv[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int k = threadIdx.x * 4 + i * 4 * kGemvThreads;
      gv[i] = k < K ? *reinterpret_cast<const uint2*>(a.gain + k) : make_uint2(0u, 0u);
#pragma unroll
      for (int m = 0; m < 4; ++m)
        xv[m][i] = (m < M && k < K) ? *reinterpret_cast<const float4*>(a.x + (size_t)m * a.ldx + k)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < 2; ++i)
        ss += xv[m][i].x * xv[m][i].x + xv[m][i].y * xv[m][i].y + xv[m][i].z * xv[m][i].z + xv[m][i].w * xv[m][i].w;
      ss = warp_sum(ss);
      if (lane == 0 && m < M) ssq[m * 8 + warp] = ss;
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      if (m >= M) continue;
      float ss = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) ss += ssq[m * 8 + w];
      const float rs = 1.0f / sqrtf(ss / (float)K + a.eps);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int k = threadIdx.x * 4 + i * 4 * kGemvThreads;
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
        *reinterpret_cast<uint2*>(xs + m * ldxs + k) = ph;
        *reinterpret_cast<uint2*>(xl + m * ldxs + k) = pl;
      }
    }
  } else if (IN == IN_F32W && M <= 2 && K <= 8 * 4 * kGemvThreads) {
    // fp32 rows of up to 8 float4 per thread (the down input of a decode
    // step): every load of a row is issued before the first conversion, one
    // round trip to L2 instead of two
    constexpr int R = 8;
    for (int m = 0; m < M; ++m) {
      const float* src = a.x + (size_t)m * a.ldx;
      float4 v[R];
#pragma unroll
      for (int j = 0; j < R; ++j) {
        const int k = threadIdx.x * 4 + j * 4 * kGemvThreads;
        v[j] = k < K ? *reinterpret_cast<const float4*>(src + k) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int j = 0; j < R; ++j) {
        const int k = threadIdx.x * 4 + j * 4 * kGemvThreads;
        if (k >= K) continue;
        const __half2 h01 = __floats2half2_rn(v[j].x, v[j].y), h23 = __floats2half2_rn(v[j].z, v[j].w);
        const float2 r01 = __half22float2(h01), r23 = __half22float2(h23);
        const __half2 l01 = __floats2half2_rn(v[j].x - r01.x, v[j].y - r01.y);
        const __half2 l23 = __floats2half2_rn(v[j].z - r23.x, v[j].w - r23.y);
        uint2 ph, pl;
        ph.x = *reinterpret_cast<const uint32_t*>(&h01); ph.y = *reinterpret_cast<const uint32_t*>(&h23);
        pl.x = *reinterpret_cast<const uint32_t*>(&l01); pl.y = *reinterpret_cast<const uint32_t*>(&l23);
        *reinterpret_cast<uint2*>(xs + m * ldxs + k) = ph;
        *reinterpret_cast<uint2*>(xl + m * ldxs + k) = pl;
      }
    }
  } else {
    // every thread takes float4 columns tid*4 + 1024 i of every row
    if (IN == IN_NORM) {
      for (int m = 0; m < M; ++m) {
        const float* src = a.x + (size_t)m * a.ldx;
        float ss = 0.f;
#pragma unroll 4
        for (int k = threadIdx.x * 4; k < K; k += 4 * kGemvThreads) {
          const float4 v = *reinterpret_cast<const float4*>(src + k);
          ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
        }
        ss = warp_sum(ss);
        if (lane == 0) ssq[m * 8 + warp] = ss;
      }
      __syncthreads();
    }
    for (int m = 0; m < M; ++m) {
      const float* src = a.x + (size_t)m * a.ldx;
      float rs = 1.f;
      if (IN == IN_NORM) {
        float ss = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) ss += ssq[m * 8 + w];
        rs = 1.0f / sqrtf(ss / (float)K + a.eps);
      }
#pragma unroll 4
      for (int k = threadIdx.x * 4; k < K; k += 4 * kGemvThreads) {
        float4 v = *reinterpret_cast<const float4*>(src + k);
        if (IN == IN_NORM) {
          const float2 g01 = __half22float2(*reinterpret_cast<const __half2*>(a.gain + k));
          const float2 g23 = __half22float2(*reinterpret_cast<const __half2*>(a.gain + k + 2));
          v.x = (v.x * rs) * g01.x; v.y = (v.y * rs) * g01.y;
          v.z = (v.z * rs) * g23.x; v.w = (v.w * rs) * g23.y;
        }
        const __half2 h01 = __floats2half2_rn(v.x, v.y), h23 = __floats2half2_rn(v.z, v.w);
        const float2 r01 = __half22float2(h01), r23 = __half22float2(h23);
        const __half2 l01 = __floats2half2_rn(v.x - r01.x, v.y - r01.y);
        const __half2 l23 = __floats2half2_rn(v.z - r23.x, v.w - r23.y);
        uint2 ph, pl;
        ph.x = *reinterpret_cast<const uint32_t*>(&h01); ph.y = *reinterpret_cast<const uint32_t*>(&h23);
        pl.x = *reinterpret_cast<const uint32_t*>(&l01); pl.y = *reinterpret_cast<const uint32_t*>(&l23);
        *reinterpret_cast<uint2*>(xs + m * ldxs + k) = ph;
        *reinterpret_cast<uint2*>(xl + m * ldxs + k) = pl;
      }
    }
  }
  if (threadIdx.x == 0) {
    trace_mark(a.trace, 6);
    s_ok = mbar_wait(&wbar, 0) ? 1 : 0;
    if (!s_ok) atomicOr(a.err_flag, kErrTimeout);
    trace_mark(a.trace, 3);
  }
  __syncthreads();
  if (!s_ok) return;  // uniform: every thread read the same flag after the barrier

  // ---- main loop: 64-wide K chunks from shared memory, 4 k16 tiles each ----
  const int c_begin = (n_chunks * kq) / KS;
  const int nc = (n_chunks * (kq + 1)) / KS - c_begin;
  constexpr int LANE_B = BITS == 2 ? 8 : 16;    // weight bytes per lane per chunk
  const unsigned char* wbase = sw + tsel * wt_bytes + (size_t)lane * LANE_B;
  const unsigned char* sbase = ssz + tsel * sz_bytes + (size_t)g * 8;
  // B-fragment source of this lane: activation row and plane
  int brow, bplane;
  if (NT == 0 && LO) { brow = g >> 1; bplane = g & 1; }
  else { brow = g; bplane = 0; }
  const __half* bsrc = (bplane ? xl : xs) + (size_t)brow * ldxs + 2 * t;

  float acc[NTILES][4];
#pragma unroll
  for (int nt = 0; nt < NTILES; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;

#pragma unroll 2
  for (int ci = 0; ci < nc; ++ci) {
    const int c = c_begin + ci;
    uint32_t words[4];
    if (BITS == 2) {
      const uint2 w2 = *reinterpret_cast<const uint2*>(wbase + (size_t)c * 32 * LANE_B);
      words[0] = w2.x; words[1] = w2.y; words[2] = 0u; words[3] = 0u;
    } else {
      const uint4 wv = *reinterpret_cast<const uint4*>(wbase + (size_t)c * 32 * LANE_B);
      words[0] = wv.x; words[1] = wv.y; words[2] = wv.z; words[3] = wv.w;
    }
    const uint2 sv = *reinterpret_cast<const uint2*>(sbase + (size_t)(c >> 1) * 64);
    const int kc = c * 64;
    float tmp[NTILES][4];
#pragma unroll
    for (int nt = 0; nt < NTILES; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) tmp[nt][q] = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t af[4];
      if (BITS == 2) unpack_a_frag2(words[j >> 1], j & 1, sv.y, af);
      else unpack_a_frag(words[j], sv.y, af);
      const int ko = kc + j * 16;
      if (NT == 0) {
        uint32_t b0 = 0, b1 = 0;
        if (brow < M) {
          b0 = *reinterpret_cast<const uint32_t*>(bsrc + ko);
          b1 = *reinterpret_cast<const uint32_t*>(bsrc + ko + 8);
        }
        mma_f16_16816(tmp[0], af, b0, b1);
      } else {
#pragma unroll
        for (int nt = 0; nt < NTILES; ++nt) {
          const int row = nt * 8 + g;
          uint32_t b0 = 0, b1 = 0, c0 = 0, c1 = 0;
          if (row < M) {
            const size_t off = (size_t)row * ldxs + ko + 2 * t;
            b0 = *reinterpret_cast<const uint32_t*>(xs + off);
            b1 = *reinterpret_cast<const uint32_t*>(xs + off + 8);
            if (LO) {
              c0 = *reinterpret_cast<const uint32_t*>(xl + off);
              c1 = *reinterpret_cast<const uint32_t*>(xl + off + 8);
            }
          }
          mma_f16_16816(tmp[nt], af, b0, b1);
          if (LO) mma_f16_16816(tmp[nt], af, c0, c1);
        }
      }
    }
    const float2 s = h2_to_f2(sv.x);
#pragma unroll
    for (int nt = 0; nt < NTILES; ++nt) {
      acc[nt][0] = fmaf(s.x, tmp[nt][0], acc[nt][0]);
      acc[nt][1] = fmaf(s.x, tmp[nt][1], acc[nt][1]);
      acc[nt][2] = fmaf(s.y, tmp[nt][2], acc[nt][2]);
      acc[nt][3] = fmaf(s.y, tmp[nt][3], acc[nt][3]);
    }
  }

  trace_mark(a.trace, 4);
  if (a.trigger == TRIGGER_AFTER_LOOP) pdl_trigger();
  // ---- reduce the K slices (fixed order) ---------------------------------
  float* myred = red + (kq * TPC + tsel) * 16 * NC;
  if (NT == 0 && LO) {  // columns (2m, 2m+1) = (hi, lo) parts of row m = t
    myred[g * NC + t] = acc[0][0] + acc[0][1];
    myred[(g + 8) * NC + t] = acc[0][2] + acc[0][3];
  } else {
#pragma unroll
    for (int nt = 0; nt < NTILES; ++nt) {
      const int col = nt * 8 + 2 * t;
      myred[g * NC + col] = acc[nt][0];
      myred[g * NC + col + 1] = acc[nt][1];
      myred[(g + 8) * NC + col] = acc[nt][2];
      myred[(g + 8) * NC + col + 1] = acc[nt][3];
    }
  }
  __syncthreads();

  const int r = threadIdx.x & 15, m = threadIdx.x >> 4;
  if (m >= M || m >= NC) return;
  float va = 0.f, vb = 0.f;
#pragma unroll
  for (int q = 0; q < KS; ++q) {
    va += red[(q * TPC + 0) * 16 * NC + r * NC + m];
    if (TPC == 2) vb += red[(q * TPC + 1) * 16 * NC + r * NC + m];
  }
  const int row0 = t0 * 16 + r, row1 = t1 * 16 + r;

  if (EPI == EPI_STORE) {
    if (row0 < a.n_rows) a.y[(size_t)m * a.ldy + row0] = __float2half_rn(va);
  } else if (EPI == EPI_RESID) {
    if (row0 < a.n_rows) a.resid[(size_t)m * a.ldr + row0] += va;
  } else if (EPI == EPI_SWIGLU) {
    a.yf[(size_t)m * a.ldy + row0] = silu(va) * vb;
  } else {  // EPI_ROPE_KV: row0 is element j < hd/2 of a head, row1 = row0 + hd/2
    const int hd = a.hd;
    const int j = row0 % hd;
    const RowCtx rc = a.rows[m];
    if (row0 < a.n_q_rows) {
      const float2 cs = rope_cs(a.rope_tab, rc.pos, j, hd, a.theta);
      float* qo = a.q_out + (size_t)m * a.ldq;
      qo[row0] = va * cs.x - vb * cs.y;
      qo[row1] = vb * cs.x + va * cs.y;
    } else if (row0 < a.n_q_rows + a.n_kv_rows) {
      const float2 cs = rope_cs(a.rope_tab, rc.pos, j, hd, a.theta);
      const int kvh = (row0 - a.n_q_rows) / hd;
      const float k0 = va * cs.x - vb * cs.y, k1 = vb * cs.x + va * cs.y;
      if (a.kv_stage) {
        float* dst = a.kv_stage + ((size_t)(m * 2) * (a.n_kv_rows / hd) + kvh) * hd;
        dst[j] = k0;
        dst[j + hd / 2] = k1;
      } else {
        __half* dst = a.k_plane + rc.lane * a.lane_stride + ((size_t)kvh * a.ctx + rc.pos) * hd;
        dst[j] = __float2half_rn(k0);
        dst[j + hd / 2] = __float2half_rn(k1);
      }
    } else {
      const int kvh = (row0 - a.n_q_rows - a.n_kv_rows) / hd;
      if (a.kv_stage) {
        float* dst = a.kv_stage + ((size_t)(m * 2 + 1) * (a.n_kv_rows / hd) + kvh) * hd;
        dst[j] = va;
        dst[j + hd / 2] = vb;
      } else {
        __half* dst = a.v_plane + rc.lane * a.lane_stride + ((size_t)kvh * a.ctx + rc.pos) * hd;
        dst[j] = __float2half_rn(va);
        dst[j + hd / 2] = __float2half_rn(vb);
      }
    }
  }
  trace_mark(a.trace, 5);
}

// The same GEMV for 5..16 activation rows (NT = 1, 2): the activation planes
// hold K in phases of kGemvPhaseK columns, a share of every warp's K slice
// each, so a CTA's planes stay small and several CTAs share an SM (whole
// 16-row planes held one CTA per SM and spread a 352-CTA grid over 2.4
// waves).  Every warp keeps its contiguous K slice, chunk order and
// accumulation, so a row's result equals what the one-pass layout gives.
template <int NT, int IN, int EPI, int BITS = 4>
__global__ void __launch_bounds__(kGemvThreads) gemv_rows_kernel(const GemvArgs a) {
  static_assert(NT != 0, "the one-pass layout is gemv_int4_kernel");
  constexpr bool LO = (IN != IN_F16);
  constexpr int TPC = gemv_tpc(EPI);
  constexpr int KS = 8 / TPC;                 // K slices
  constexpr int NC = NT == 2 ? 16 : 8;        // reduction columns
  constexpr int NTILES = NT == 2 ? 2 : 1;     // n8 tiles of the MMA
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t wbar;
  __shared__ int s_ok;
  const int K = a.K;
  const int M = a.M;
  const int ldxs = kGemvPhaseK + 8;
  const int n_chunks = K >> 6;
  const size_t wt_bytes = gemv_w_bytes(K, BITS), sz_bytes = gemv_sz_bytes(K);
  unsigned char* sw = smem;                                       // [TPC][chunks][32][16 B]
  unsigned char* ssz = smem + TPC * wt_bytes;                     // [TPC][groups][8][8 B]
  __half* xs = reinterpret_cast<__half*>(ssz + TPC * sz_bytes);   // hi plane [M][ldxs]
  __half* xl = xs + (size_t)M * ldxs;                             // lo plane [M][ldxs]
  float* red = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(xs) + gemv_rows_act_bytes(M, LO));
  float* ssq = red + 8 * 16 * NC;                                 // [16 rows][8 warps]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int tsel = TPC == 2 ? (warp & 1) : 0;
  const int kq = TPC == 2 ? (warp >> 1) : warp;

  int t0, t1;
  if (TPC == 1) {
    t0 = blockIdx.x;
    t1 = t0;
  } else if (a.pair_mode == PAIR_OFFSET) {
    t0 = blockIdx.x;
    t1 = t0 + a.pair_off;
  } else {
    const int head = blockIdx.x / a.pair_off, j16 = blockIdx.x % a.pair_off;
    t0 = head * 2 * a.pair_off + j16;
    t1 = t0 + a.pair_off;
  }

  trace_start(a.trace);
  if (a.trigger == TRIGGER_AT_START) pdl_trigger();
  // The weights do not depend on earlier kernels: start their bulk copies
  // before waiting for the previous kernel.
  if (threadIdx.x == 0) {
    mbar_init(&wbar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&wbar, (unsigned)(TPC * (wt_bytes + sz_bytes)));
    const uint64_t pol = a.l2_keep ? l2_evict_last() : l2_evict_first();
    for (int ts = 0; ts < TPC; ++ts) {
      const int tile = ts ? t1 : t0;
      const unsigned char* src = reinterpret_cast<const unsigned char*>(a.w) + (size_t)tile * wt_bytes;
      for (size_t off = 0; off < wt_bytes; off += 32768) {
        const unsigned n = (unsigned)((wt_bytes - off) < 32768 ? (wt_bytes - off) : 32768);
        bulk_g2s_hint(sw + ts * wt_bytes + off, src + off, n, &wbar, pol);
      }
      bulk_g2s_hint(ssz + ts * sz_bytes, reinterpret_cast<const unsigned char*>(a.sz) + (size_t)tile * sz_bytes,
                    (unsigned)sz_bytes, &wbar, pol);
    }
  }

  pdl_wait();
  trace_mark(a.trace, 2);

  float acc[NTILES][4];
  // ---- many rows: the planes hold K in phases of kGemvPhaseK columns -------
  // a phase stages the next CPW chunks of every warp's K slice
  constexpr int CPW = kGemvPhaseK / 64 / KS;   // chunks per slice and phase
  constexpr int LANE_B = BITS == 2 ? 8 : 16;    // weight bytes per lane per chunk
  const unsigned char* wbase = sw + tsel * wt_bytes + (size_t)lane * LANE_B;
  const unsigned char* sbase = ssz + tsel * sz_bytes + (size_t)g * 8;
  const int c_begin = (n_chunks * kq) / KS;
  const int nc = (n_chunks * (kq + 1)) / KS - c_begin;
  const int n_ph = ((n_chunks + KS - 1) / KS + CPW - 1) / CPW;   // phases of the longest slice
#pragma unroll
  for (int nt = 0; nt < NTILES; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
  __shared__ float s_rs[16];
  if (IN == IN_NORM) {   // every row's RMS factor over the whole row first
    for (int m = 0; m < M; ++m) {
      const float* src = a.x + (size_t)m * a.ldx;
      float ss = 0.f;
      for (int k = threadIdx.x * 4; k < K; k += 4 * kGemvThreads) {
        const float4 v = *reinterpret_cast<const float4*>(src + k);
        ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
      }
      ss = warp_sum(ss);
      if (lane == 0) ssq[m * 8 + warp] = ss;
    }
    __syncthreads();
    if (threadIdx.x < M) {
      float ss = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) ss += ssq[threadIdx.x * 8 + w];
      s_rs[threadIdx.x] = 1.0f / sqrtf(ss / (float)K + a.eps);
    }
    __syncthreads();
  }
  for (int ph = 0; ph < n_ph; ++ph) {
    // stage chunk l < CPW of phase ph of every slice q at plane column
    // (q * CPW + l) * 64; chunks past a slice's end are not staged
    constexpr int G4 = 16;   // 4-column groups per chunk
    for (int e = threadIdx.x; e < M * KS * CPW * G4; e += kGemvThreads) {
      const int m = e / (KS * CPW * G4), rem = e % (KS * CPW * G4);
      const int q = rem / (CPW * G4), l = (rem / G4) % CPW, k4 = (rem % G4) * 4;
      const int qb = (n_chunks * q) / KS, qe = (n_chunks * (q + 1)) / KS;
      const int c = qb + ph * CPW + l;
      if (c >= qe) continue;
      const int kg = c * 64 + k4, col = (q * CPW + l) * 64 + k4;
      if (IN == IN_F16) {
        *reinterpret_cast<uint2*>(xs + m * ldxs + col) =
            *reinterpret_cast<const uint2*>(a.xh + (size_t)m * a.ldx + kg);
      } else {
        float4 v = *reinterpret_cast<const float4*>(a.x + (size_t)m * a.ldx + kg);
        if (IN == IN_NORM) {
          const float rs = s_rs[m];
          const float2 g01 = __half22float2(*reinterpret_cast<const __half2*>(a.gain + kg));
          const float2 g23 = __half22float2(*reinterpret_cast<const __half2*>(a.gain + kg + 2));
          v.x = (v.x * rs) * g01.x; v.y = (v.y * rs) * g01.y;
          v.z = (v.z * rs) * g23.x; v.w = (v.w * rs) * g23.y;
        }
        const __half2 h01 = __floats2half2_rn(v.x, v.y), h23 = __floats2half2_rn(v.z, v.w);
        const float2 r01 = __half22float2(h01), r23 = __half22float2(h23);
        const __half2 l01 = __floats2half2_rn(v.x - r01.x, v.y - r01.y);
        const __half2 l23 = __floats2half2_rn(v.z - r23.x, v.w - r23.y);
        uint2 ph2, pl2;
        ph2.x = *reinterpret_cast<const uint32_t*>(&h01); ph2.y = *reinterpret_cast<const uint32_t*>(&h23);
        pl2.x = *reinterpret_cast<const uint32_t*>(&l01); pl2.y = *reinterpret_cast<const uint32_t*>(&l23);
        *reinterpret_cast<uint2*>(xs + m * ldxs + col) = ph2;
        *reinterpret_cast<uint2*>(xl + m * ldxs + col) = pl2;
      }
    }
    if (ph == 0 && threadIdx.x == 0) {
      trace_mark(a.trace, 6);
      s_ok = mbar_wait(&wbar, 0) ? 1 : 0;
      if (!s_ok) atomicOr(a.err_flag, kErrTimeout);
      trace_mark(a.trace, 3);
    }
    __syncthreads();
    if (!s_ok) return;  // uniform: every thread read the same flag after the barrier
    for (int l = 0; l < CPW; ++l) {
      const int ci = ph * CPW + l;
      if (ci >= nc) break;
      const int c = c_begin + ci;
      uint32_t words[4];
      if (BITS == 2) {
        const uint2 w2 = *reinterpret_cast<const uint2*>(wbase + (size_t)c * 32 * LANE_B);
        words[0] = w2.x; words[1] = w2.y; words[2] = 0u; words[3] = 0u;
      } else {
        const uint4 wv = *reinterpret_cast<const uint4*>(wbase + (size_t)c * 32 * LANE_B);
        words[0] = wv.x; words[1] = wv.y; words[2] = wv.z; words[3] = wv.w;
      }
      const uint2 sv = *reinterpret_cast<const uint2*>(sbase + (size_t)(c >> 1) * 64);
      float tmp[NTILES][4];
#pragma unroll
      for (int nt = 0; nt < NTILES; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) tmp[nt][q] = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t af[4];
        if (BITS == 2) unpack_a_frag2(words[j >> 1], j & 1, sv.y, af);
        else unpack_a_frag(words[j], sv.y, af);
        const int ko = (kq * CPW + l) * 64 + j * 16;   // column within the staged phase
#pragma unroll
        for (int nt = 0; nt < NTILES; ++nt) {
          const int row = nt * 8 + g;
          uint32_t b0 = 0, b1 = 0, c0 = 0, c1 = 0;
          if (row < M) {
            const size_t off = (size_t)row * ldxs + ko + 2 * t;
            b0 = *reinterpret_cast<const uint32_t*>(xs + off);
            b1 = *reinterpret_cast<const uint32_t*>(xs + off + 8);
            if (LO) {
              c0 = *reinterpret_cast<const uint32_t*>(xl + off);
              c1 = *reinterpret_cast<const uint32_t*>(xl + off + 8);
            }
          }
          mma_f16_16816(tmp[nt], af, b0, b1);
          if (LO) mma_f16_16816(tmp[nt], af, c0, c1);
        }
      }
      const float2 sc2 = h2_to_f2(sv.x);
#pragma unroll
      for (int nt = 0; nt < NTILES; ++nt) {
        acc[nt][0] = fmaf(sc2.x, tmp[nt][0], acc[nt][0]);
        acc[nt][1] = fmaf(sc2.x, tmp[nt][1], acc[nt][1]);
        acc[nt][2] = fmaf(sc2.y, tmp[nt][2], acc[nt][2]);
        acc[nt][3] = fmaf(sc2.y, tmp[nt][3], acc[nt][3]);
      }
    }
    __syncthreads();   // the planes are restaged for the next phase
  }

  trace_mark(a.trace, 4);
  if (a.trigger == TRIGGER_AFTER_LOOP) pdl_trigger();
  // ---- reduce the K slices (fixed order) ---------------------------------
  float* myred = red + (kq * TPC + tsel) * 16 * NC;
  if (NT == 0 && LO) {  // columns (2m, 2m+1) = (hi, lo) parts of row m = t
    myred[g * NC + t] = acc[0][0] + acc[0][1];
    myred[(g + 8) * NC + t] = acc[0][2] + acc[0][3];
  } else {
#pragma unroll
    for (int nt = 0; nt < NTILES; ++nt) {
      const int col = nt * 8 + 2 * t;
      myred[g * NC + col] = acc[nt][0];
      myred[g * NC + col + 1] = acc[nt][1];
      myred[(g + 8) * NC + col] = acc[nt][2];
      myred[(g + 8) * NC + col + 1] = acc[nt][3];
    }
  }
  __syncthreads();

  const int r = threadIdx.x & 15, m = threadIdx.x >> 4;
  if (m >= M || m >= NC) return;
  float va = 0.f, vb = 0.f;
#pragma unroll
  for (int q = 0; q < KS; ++q) {
    va += red[(q * TPC + 0) * 16 * NC + r * NC + m];
    if (TPC == 2) vb += red[(q * TPC + 1) * 16 * NC + r * NC + m];
  }
  const int row0 = t0 * 16 + r, row1 = t1 * 16 + r;

  if (EPI == EPI_STORE) {
    if (row0 < a.n_rows) a.y[(size_t)m * a.ldy + row0] = __float2half_rn(va);
  } else if (EPI == EPI_RESID) {
    if (row0 < a.n_rows) a.resid[(size_t)m * a.ldr + row0] += va;
  } else if (EPI == EPI_SWIGLU) {
    a.yf[(size_t)m * a.ldy + row0] = silu(va) * vb;
  } else {  // EPI_ROPE_KV: row0 is element j < hd/2 of a head, row1 = row0 + hd/2
    const int hd = a.hd;
    const int j = row0 % hd;
    const RowCtx rc = a.rows[m];
    if (row0 < a.n_q_rows) {
      const float2 cs = rope_cs(a.rope_tab, rc.pos, j, hd, a.theta);
      float* qo = a.q_out + (size_t)m * a.ldq;
      qo[row0] = va * cs.x - vb * cs.y;
      qo[row1] = vb * cs.x + va * cs.y;
    } else if (row0 < a.n_q_rows + a.n_kv_rows) {
      const float2 cs = rope_cs(a.rope_tab, rc.pos, j, hd, a.theta);
      const int kvh = (row0 - a.n_q_rows) / hd;
      const float k0 = va * cs.x - vb * cs.y, k1 = vb * cs.x + va * cs.y;
      if (a.kv_stage) {
        float* dst = a.kv_stage + ((size_t)(m * 2) * (a.n_kv_rows / hd) + kvh) * hd;
        dst[j] = k0;
        dst[j + hd / 2] = k1;
      } else {
        __half* dst = a.k_plane + rc.lane * a.lane_stride + ((size_t)kvh * a.ctx + rc.pos) * hd;
        dst[j] = __float2half_rn(k0);
        dst[j + hd / 2] = __float2half_rn(k1);
      }
    } else {
      const int kvh = (row0 - a.n_q_rows - a.n_kv_rows) / hd;
      if (a.kv_stage) {
        float* dst = a.kv_stage + ((size_t)(m * 2 + 1) * (a.n_kv_rows / hd) + kvh) * hd;
        dst[j] = va;
        dst[j + hd / 2] = vb;
      } else {
        __half* dst = a.v_plane + rc.lane * a.lane_stride + ((size_t)kvh * a.ctx + rc.pos) * hd;
        dst[j] = __float2half_rn(va);
        dst[j + hd / 2] = __float2half_rn(vb);
      }
    }
  }
  trace_mark(a.trace, 5);
}

// ---- load-time re-layout ----------------------------------------------------
// Nibble i of packed word j for (tile T, chunk c, lane l = 4g + t) holds, with
// r0 = 16T + g, r1 = r0 + 8, kb = 64c + 16j:
//   0:(r0,kb+2t) 1:(r1,kb+2t) 2:(r0,kb+2t+8) 3:(r1,kb+2t+8)
//   4:(r0,kb+2t+1) 5:(r1,kb+2t+1) 6:(r0,kb+2t+9) 7:(r1,kb+2t+9)
// so that unpack_a_frag yields the m16n8k16 A fragment.  Rows >= N are zero.
__global__ void repack_int4_weights_kernel(const uint32_t* __restrict__ qweight, int K, int N,
                                           int n_tiles, uint4* __restrict__ out) {
  const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int n_chunks = K >> 6;
  const size_t total = (size_t)n_tiles * n_chunks * 32;
  if (idx >= total) return;
  const int l = (int)(idx & 31);
  const size_t rest = idx >> 5;
  const int c = (int)(rest % n_chunks);
  const int T = (int)(rest / n_chunks);
  const int g = l >> 2, t = l & 3;
  const int r0 = T * 16 + g, r1 = r0 + 8;
  const int kw = K >> 3;
  auto q = [&](int r, int k) -> uint32_t {
    if (r >= N) return 0u;
    return (qweight[(size_t)r * kw + (k >> 3)] >> (4 * (k & 7))) & 0xFu;
  };
  uint32_t wd[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int kb = c * 64 + j * 16 + 2 * t;
    wd[j] = q(r0, kb) | (q(r1, kb) << 4) | (q(r0, kb + 8) << 8) | (q(r1, kb + 8) << 12) |
            (q(r0, kb + 1) << 16) | (q(r1, kb + 1) << 20) | (q(r0, kb + 9) << 24) |
            (q(r1, kb + 9) << 28);
  }
  out[idx] = make_uint4(wd[0], wd[1], wd[2], wd[3]);
}

// INT2 body: for (tile T, chunk c, lane l) two words; word j2 holds k16
// steps 2 j2 and 2 j2 + 1, step s's slots in the order above at fields
// 4s + r (first element of the pair) and 8 + 4s + r (second), field f at bits
// 2f, so that unpack_a_frag2 yields the A fragment.  Storage: element k of
// row n in bits 2 (k % 16) of word k / 16.
__global__ void repack_int2_weights_kernel(const uint32_t* __restrict__ qweight, int K, int N,
                                           int n_tiles, uint2* __restrict__ out) {
  const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int n_chunks = K >> 6;
  const size_t total = (size_t)n_tiles * n_chunks * 32;
  if (idx >= total) return;
  const int l = (int)(idx & 31);
  const size_t rest = idx >> 5;
  const int c = (int)(rest % n_chunks);
  const int T = (int)(rest / n_chunks);
  const int g = l >> 2, t = l & 3;
  const int r0 = T * 16 + g, r1 = r0 + 8;
  const int kw = K >> 4;
  auto q = [&](int r, int k) -> uint32_t {
    if (r >= N) return 0u;
    return (qweight[(size_t)r * kw + (k >> 4)] >> (2 * (k & 15))) & 0x3u;
  };
  uint32_t wd[2];
#pragma unroll
  for (int j2 = 0; j2 < 2; ++j2) {
    uint32_t w = 0;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int kb = c * 64 + (2 * j2 + s) * 16 + 2 * t;
      const uint32_t v[8] = {q(r0, kb), q(r1, kb), q(r0, kb + 8), q(r1, kb + 8),
                             q(r0, kb + 1), q(r1, kb + 1), q(r0, kb + 9), q(r1, kb + 9)};
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        w |= v[r] << (2 * (4 * s + r));
        w |= v[4 + r] << (2 * (8 + 4 * s + r));
      }
    }
    wd[j2] = w;
  }
  out[idx] = make_uint2(wd[0], wd[1]);
}

// sz[T][group][g] = {(s[r0], s[r1]) fp16 pair, (1024 + z[r0], 1024 + z[r1]) fp16 pair};
// the zero points are 4-bit (bits = 4) or 2-bit (bits = 2) fields
__global__ void repack_int4_scales_kernel(const uint16_t* __restrict__ scales,
                                          const uint32_t* __restrict__ qzeros, int K, int N,
                                          int n_tiles, uint2* __restrict__ out, int bits) {
  const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int G = K >> 7;
  const int epw = 32 / bits;   // zero points per word
  const int zw = (G + epw - 1) / epw;
  const size_t total = (size_t)n_tiles * G * 8;
  if (idx >= total) return;
  const int g = (int)(idx & 7);
  const size_t rest = idx >> 3;
  const int gr = (int)(rest % G);
  const int T = (int)(rest / G);
  const int r0 = T * 16 + g, r1 = r0 + 8;
  auto sc = [&](int r) -> uint32_t { return r < N ? (uint32_t)scales[(size_t)r * G + gr] : 0u; };
  auto zb = [&](int r) -> uint32_t {
    const uint32_t z = r < N ? (qzeros[(size_t)r * zw + gr / epw] >> (bits * (gr % epw))) & ((1u << bits) - 1u) : 0u;
    return 0x6400u + z;  // fp16 bits of 1024 + z
  };
  out[idx] = make_uint2(sc(r0) | (sc(r1) << 16), zb(r0) | (zb(r1) << 16));
}

}  // namespace tl
