// Causal tiled prefill GQA attention on the 5th-generation tensor cores
// (tcgen05, TMEM accumulators) -- the tiled prefill path of TinyLoop README,
// "Current Runtime Snapshot" (full prefill attention, tiled), with the GQA
// head mapping of "Status" and the tiled online softmax / causal masking of
// the tiny-llm feature list.
//
// Design (ours, sm_100a):
// * One CTA per (128-query tile, query head, batch entry).  The queries are
//   the MMA rows (M = 128): S = Q K^T over a block of 64 keys (N = 64) and
//   O_j = P_j V_j (N = head_dim), both in TMEM, double-buffered.
// * Q (fp32 or fp16 in memory) is scaled by log2(e)/sqrt(hd) (the softmax
//   runs in base 2) and split into an fp16 pair (hi, lo); S accumulates
//   Q_hi K^T + Q_lo K^T.  P is split the same
//   way and O_j accumulates P_hi V + P_lo V.  K and V are fp16 already, so
//   the products keep ~fp32 accuracy (as the other attention kernels).
// * Operands in shared memory, 128-byte swizzled: Q and P K-major, K K-major
//   (a key's head dims are the MMA's K), V MN-major (a key's head dims are
//   the MMA's N: 64-wide dim chunks LBO apart, groups of 8 keys SBO apart),
//   so K and V rows are copied as they lie in the cache.
// * Warp roles, all handing over through mbarriers, so loads, MMAs, softmax
//   and the output update of different key blocks overlap:
//     warp 0       one lane issues the MMAs: S_j, then O_{j-1} (the softmax of
//                  block j runs while O_{j-1} is computed);
//     warp 1       loads K/V blocks (cp.async, completion tracked by an
//                  mbarrier), two blocks ahead;
//     warps 2-9    softmax: two threads per query row (32 of its 64 scores
//                  each, max and sum exchanged through shared memory) read
//                  the scores from TMEM, mask, keep the running max / sum,
//                  write P (hi, lo) and the rescale factor of the block;
//     warps 10-17  output: two threads per query row (half of the head dims
//                  each) keep O in registers and apply O = O c_j + O_j as
//                  each O_j lands in TMEM.
// * Every mbarrier wait is bounded; a CTA that gives up records kErrTimeout
//   and still frees its TMEM.
#pragma once

#include "attention.cuh"
#include "common.cuh"
#include "gemm_tc.cuh"

namespace tl {

constexpr int kAtQ = 128;        // queries per CTA (MMA M)
constexpr int kAtKeys = 64;      // keys per block (MMA N of S, K of P V)
constexpr int kAtWarps = 18;
constexpr int kAtThreads = kAtWarps * 32;
constexpr int kAtSoftWarp0 = 2, kAtOutWarp0 = 10;   // 8 softmax warps, 8 output warps

// Shared-memory plan (bytes) for head_dim HD.
template <int HD>
struct AtLayout {
  static constexpr int KA = HD / 64;                       // 64-wide atoms of a head
  static constexpr int Q_BYTES = KA * kAtQ * 128;          // one of hi / lo
  static constexpr int K_BYTES = KA * kAtKeys * 128;       // one key block
  static constexpr int V_BYTES = KA * kAtKeys * 128;
  static constexpr int P_BYTES = kAtQ * 128;               // one of hi / lo (64 keys)
  static constexpr int q_hi = 0, q_lo = Q_BYTES;
  static constexpr int k0 = 2 * Q_BYTES;                   // [2 buffers]
  static constexpr int v0 = k0 + 2 * K_BYTES;              // [2 buffers]
  static constexpr int p0 = v0 + 2 * V_BYTES;              // [2 buffers][hi, lo]
  static constexpr int total = p0 + 4 * P_BYTES;
};
template <int HD>
__host__ __device__ constexpr size_t attn_tc_smem_bytes() {
  return (size_t)AtLayout<HD>::total + 1024;   // + alignment slack
}

// Shared-memory descriptor of an MN-major operand, 128-byte swizzle: rows of
// 64 consecutive N elements (128 B), 8 rows (8 consecutive K) per 1024-byte
// swizzle atom; `lbo` bytes between 64-wide N chunks, `sbo` bytes between
// groups of 8 K.
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(const void* p, uint32_t lbo, uint32_t sbo) {
  const uint64_t addr = smem_u32(p);
  uint64_t d = (addr >> 4) & 0x3FFFull;
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= 1ull << 46;
  d |= 2ull << 61;
  return d;
}
// kind::f16 instruction descriptor with B MN-major (bit 16).
__host__ __device__ constexpr uint32_t idesc_f16_f32_bmn(int M, int N) {
  return idesc_f16_f32(M, N) | (1u << 16);
}

template <int HD, bool F32>
__global__ void __launch_bounds__(kAtThreads, 1) prefill_attn_tc_kernel(const PrefillAttnArgs a) {
  using Lay = AtLayout<HD>;
  constexpr int KA = Lay::KA;
  extern __shared__ __align__(128) unsigned char at_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(at_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t kv_full[2], s_full[2], p_full[2], o_full[2], o_empty[2], blk_done[2];
  __shared__ uint32_t s_tmem;
  __shared__ int s_fail;
  __shared__ float cfac[2][kAtQ];   // rescale factor of block j for each row
  __shared__ float lfin[kAtQ];      // final row sums
  __shared__ float xmax[2][kAtQ], xsum[2][kAtQ];   // the two softmax halves of a row

  // grid (heads, query tiles, batch): the last (longest, causal) query tiles
  // are scheduled first so that the short ones fill the tail of the grid
  const int qt = gridDim.y - 1 - blockIdx.y, h = blockIdx.x, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kvh = h / a.rep;
  const int q0 = qt * kAtQ;
  const int last_key = a.pos0 + min(q0 + kAtQ - 1, a.T - 1);
  const int nblk = last_key / kAtKeys + 1;
  const __half* kp = a.k + b * a.kv_bstride + (size_t)kvh * a.ctx * HD;
  const __half* vp = a.v + b * a.kv_bstride + (size_t)kvh * a.ctx * HD;

  if (warp == 0) {
    tmem_alloc(&s_tmem, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 32);          // the loader warp's lanes (cp.async completion)
      mbar_init(&s_full[i], 1);            // tcgen05.commit
      mbar_init(&p_full[i], 256);          // softmax threads
      mbar_init(&o_full[i], 1);
      mbar_init(&o_empty[i], 256);         // output threads
      mbar_init(&blk_done[i], 1);
    }
    fence_mbar_init();
    s_fail = 0;
  }
  pdl_trigger();
  pdl_wait();
  __syncthreads();   // barriers initialised before the loader arrives on them

  // ---- K / V block j into buffer j % 2 (cp.async, zeros past last_key) ----
  auto load_kv = [&](int j) {
    const int bb = j & 1;
    unsigned char* ks = sm + Lay::k0 + bb * Lay::K_BYTES;
    unsigned char* vs = sm + Lay::v0 + bb * Lay::V_BYTES;
    const int j0 = j * kAtKeys;
    for (int c = lane; c < kAtKeys * HD / 8; c += 32) {
      const int key = c / (HD / 8), c16 = c % (HD / 8);
      const bool ok = j0 + key <= last_key;
      const size_t src = ok ? (size_t)(j0 + key) * HD + c16 * 8 : 0;
      const int atom = c16 >> 3, j16 = c16 & 7;
      cp_async16(ks + atom * kAtKeys * 128 + key * 128 + ((j16 ^ (key & 7)) << 4), kp + src, ok ? 16 : 0);
      cp_async16(vs + atom * (kAtKeys * 128) + (key >> 3) * 1024 + (key & 7) * 128 + ((j16 ^ (key & 7)) << 4),
                 vp + src, ok ? 16 : 0);
    }
    cp_async_mbar_arrive_noinc(&kv_full[bb]);
  };
  // the first two blocks go out before the Q tile is staged
  if (warp == 1)
    for (int j = 0; j < 2 && j < nblk; ++j) load_kv(j);

  // ---- Q tile (all threads): scale by log2(e) / sqrt(hd) (the softmax works
  // in base 2), split into (hi, lo), K-major swizzled; every load of a thread
  // is issued before any is used ------------------------------------------
  {
    constexpr int NQ = (kAtQ * HD / 8 + kAtThreads - 1) / kAtThreads;
    const float scale = 1.4426950408889634f / sqrtf((float)HD);
    float4 xv[NQ][2];
#pragma unroll
    for (int u = 0; u < NQ; ++u) {
      const int c = threadIdx.x + u * kAtThreads;
      const int row = c / (HD / 8), c16 = c % (HD / 8);
      const int t = q0 + row;
      xv[u][0] = xv[u][1] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c < kAtQ * HD / 8 && t < a.T) {
        const size_t off = b * a.q_bstride + (size_t)t * a.ldq + (size_t)h * HD + c16 * 8;
        if (F32) {
          xv[u][0] = *reinterpret_cast<const float4*>(a.qf + off);
          xv[u][1] = *reinterpret_cast<const float4*>(a.qf + off + 4);
        } else {
          const uint4 raw = *reinterpret_cast<const uint4*>(a.qh + off);
          xv[u][0] = *reinterpret_cast<const float4*>(&raw);   // raw fp16 bits, widened below
        }
      }
    }
#pragma unroll
    for (int u = 0; u < NQ; ++u) {
      const int c = threadIdx.x + u * kAtThreads;
      if (c >= kAtQ * HD / 8) continue;
      const int row = c / (HD / 8), c16 = c % (HD / 8);
      float v[8];
      if (F32) {
        v[0] = xv[u][0].x; v[1] = xv[u][0].y; v[2] = xv[u][0].z; v[3] = xv[u][0].w;
        v[4] = xv[u][1].x; v[5] = xv[u][1].y; v[6] = xv[u][1].z; v[7] = xv[u][1].w;
      } else {
        const uint32_t w4[4] = {__float_as_uint(xv[u][0].x), __float_as_uint(xv[u][0].y),
                                __float_as_uint(xv[u][0].z), __float_as_uint(xv[u][0].w)};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = h2_to_f2(w4[i]);
          v[2 * i] = f.x;
          v[2 * i + 1] = f.y;
        }
      }
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) split_h2(v[2 * i] * scale, v[2 * i + 1] * scale, hw[i], lw[i]);
      const int atom = c16 >> 3, j16 = c16 & 7;
      const int o = atom * kAtQ * 128 + row * 128 + ((j16 ^ (row & 7)) << 4);
      *reinterpret_cast<uint4*>(sm + Lay::q_hi + o) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(sm + Lay::q_lo + o) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
  }
  fence_proxy_async_smem();   // Q (st.shared) -> the tensor core's reads
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  auto t_s = [&](int buf) { return tmem + (uint32_t)(buf * 64); };          // S_j: 64 columns
  auto t_o = [&](int buf) { return tmem + 128u + (uint32_t)(buf * 128); };  // O_j: HD columns

  if (warp == 0) {
    // ---- MMA issue --------------------------------------------------------
    if (lane == 0) {
      const uint32_t idesc_s = idesc_f16_f32(kAtQ, kAtKeys);
      const uint32_t idesc_o = idesc_f16_f32_bmn(kAtQ, HD);
      auto issue_o = [&](int j) {   // O_j = P_j V_j into O buffer j % 2
        const int bb = j & 1;
        mbar_wait_or_fail(&p_full[bb], (unsigned)(j >> 1) & 1u, &s_fail);
        if (j >= 2) mbar_wait_or_fail(&o_empty[bb], (unsigned)((j - 2) >> 1) & 1u, &s_fail);
        tc_fence_after();
        const unsigned char* vs = sm + Lay::v0 + bb * Lay::V_BYTES;
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
          const unsigned char* ps = sm + Lay::p0 + (bb * 2 + pass) * Lay::P_BYTES;
#pragma unroll
          for (int kk = 0; kk < kAtKeys / 16; ++kk) {
            const uint64_t ad = sw128_kmajor_desc(ps + kk * 32);
            const uint64_t bd = sw128_mnmajor_desc(vs + kk * 2 * 1024, kAtKeys * 128, 1024);
            tc_mma_f16(t_o(bb), ad, bd, idesc_o, (pass | kk) ? 1u : 0u);
          }
        }
        tc_commit(&o_full[bb]);
        tc_commit(&blk_done[bb]);   // K_j, V_j and P_j are no longer read
      };
      for (int j = 0; j < nblk; ++j) {
        const int bb = j & 1;
        mbar_wait_or_fail(&kv_full[bb], (unsigned)(j >> 1) & 1u, &s_fail);
        fence_proxy_async_smem();   // the cp.async data -> the tensor core's reads
        // S buffer bb was last read by the softmax of block j - 2
        if (j >= 2) mbar_wait_or_fail(&p_full[bb], (unsigned)((j - 2) >> 1) & 1u, &s_fail);
        tc_fence_after();
        const unsigned char* ks = sm + Lay::k0 + bb * Lay::K_BYTES;
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
          const unsigned char* qs = sm + (pass ? Lay::q_lo : Lay::q_hi);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const int atom = kk >> 2, within = (kk & 3) * 32;
            const uint64_t ad = sw128_kmajor_desc(qs + atom * kAtQ * 128 + within);
            const uint64_t bd = sw128_kmajor_desc(ks + atom * kAtKeys * 128 + within);
            tc_mma_f16(t_s(bb), ad, bd, idesc_s, (pass | kk) ? 1u : 0u);
          }
        }
        tc_commit(&s_full[bb]);
        if (j >= 1) issue_o(j - 1);
      }
      issue_o(nblk - 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---- K / V loader: blocks 2 .. into the buffer block j - 2 released ----
    for (int j = 2; j < nblk; ++j) {
      mbar_wait_or_fail(&blk_done[j & 1], (unsigned)((j - 2) >> 1) & 1u, &s_fail);
      load_kv(j);
    }
    cp_async_wait<0>();   // nothing of this warp in flight at exit
  } else if (warp < kAtOutWarp0) {
    // ---- softmax: two threads per query row r, 32 scores each ---------------
    const int quad = warp & 3, half = (warp - kAtSoftWarp0) >> 2, r = quad * 32 + lane;
    const int pos = a.pos0 + q0 + r;
    float m_run = -INFINITY, l_run = 0.f;
    for (int j = 0; j < nblk; ++j) {
      const int bb = j & 1;
      mbar_wait_or_fail(&s_full[bb], (unsigned)(j >> 1) & 1u, &s_fail);
      tc_fence_after();
      float s[32];
      {
        uint32_t raw[32];
        const int k0 = j * kAtKeys + half * 32;
        tmem_ld32(t_s(bb) + ((uint32_t)(quad * 32) << 16) + half * 32, raw);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) s[i] = (k0 + i <= pos) ? __uint_as_float(raw[i]) : -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 32; ++i) mx = fmaxf(mx, s[i]);
      xmax[half][r] = mx;
      asm volatile("bar.sync 2, 256;" ::: "memory");   // the 8 softmax warps
      // scores are in base 2 (Q carries log2(e)): weights 2^(s - m)
      const float m_new = fmaxf(m_run, fmaxf(mx, xmax[half ^ 1][r]));
      const float c = (m_run == -INFINITY) ? 0.f : exp2f(m_run - m_new);
      float sum = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        s[i] = (m_new == -INFINITY) ? 0.f : exp2f(s[i] - m_new);   // 2^-inf = 0 for masked keys
        sum += s[i];
      }
      m_run = m_new;
      xsum[half][r] = sum;
      // P buffer bb was last read by O_{j-2}, cfac[bb] by the output warps'
      // update of block j - 2
      if (j >= 2) {
        mbar_wait_or_fail(&blk_done[bb], (unsigned)((j - 2) >> 1) & 1u, &s_fail);
        mbar_wait_or_fail(&o_empty[bb], (unsigned)((j - 2) >> 1) & 1u, &s_fail);
      }
      unsigned char* ph = sm + Lay::p0 + (bb * 2) * Lay::P_BYTES;
      unsigned char* pl = ph + Lay::P_BYTES;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) split_h2(s[q * 8 + 2 * i], s[q * 8 + 2 * i + 1], hw[i], lw[i]);
        const int j16 = half * 4 + q;
        const int o = r * 128 + ((j16 ^ (r & 7)) << 4);
        *reinterpret_cast<uint4*>(ph + o) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(pl + o) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      if (half == 0) cfac[bb][r] = c;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[bb]);
      asm volatile("bar.sync 2, 256;" ::: "memory");
      l_run = l_run * c + xsum[0][r] + xsum[1][r];
    }
    if (half == 0) lfin[r] = l_run;
  } else {
    // ---- output: two threads per query row r, O (HD / 2 columns each) kept
    // in registers ---------------------------------------------------------------
    constexpr int HO = HD / 2;
    const int quad = warp & 3, half = (warp - kAtOutWarp0) >> 2, r = quad * 32 + lane;
    float o_acc[HO];
#pragma unroll
    for (int i = 0; i < HO; ++i) o_acc[i] = 0.f;
    for (int j = 0; j < nblk; ++j) {
      const int bb = j & 1;
      // cfac of block j first: p_full cannot move on to block j + 2 before
      // these warps release o_empty for block j, so the phase is unambiguous
      mbar_wait_or_fail(&p_full[bb], (unsigned)(j >> 1) & 1u, &s_fail);
      mbar_wait_or_fail(&o_full[bb], (unsigned)(j >> 1) & 1u, &s_fail);
      tc_fence_after();
      const float c = cfac[bb][r];
#pragma unroll
      for (int c0 = 0; c0 < HO; c0 += 16) {
        uint32_t raw[16];
        tmem_ld16(t_o(bb) + ((uint32_t)(quad * 32) << 16) + half * HO + c0, raw);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) o_acc[c0 + i] = fmaf(o_acc[c0 + i], c, __uint_as_float(raw[i]));
      }
      tc_fence_before();
      mbar_arrive(&o_empty[bb]);
    }
    asm volatile("bar.sync 1, 512;" ::: "memory");   // softmax (lfin) and output warps
    const int t_row = q0 + r;
    if (t_row < a.T) {
      const float inv = 1.f / lfin[r];
      if (F32 && a.bt) {
        const int tt = t_row / kTcTokensB, tl_ = t_row % kTcTokensB;
#pragma unroll
        for (int i = 0; i < HO; i += 2) {
          const int k = h * HD + half * HO + i;   // column of the O projection's input
          const int grp = k >> 7, kg = k & 127;
          uint32_t hw, lw;
          split_h2(o_acc[i] * inv, o_acc[i + 1] * inv, hw, lw);
          uint8_t* blk = a.bt + ((size_t)tt * a.bt_groups + grp) * (2 * kTcTokensB * 256);
          *reinterpret_cast<uint32_t*>(blk + sw128_offset(tl_, kg, 2 * kTcTokensB)) = hw;
          *reinterpret_cast<uint32_t*>(blk + sw128_offset(kTcTokensB + tl_, kg, 2 * kTcTokensB)) = lw;
        }
      } else {
        const size_t off = b * a.o_bstride + (size_t)t_row * a.ldo + (size_t)h * HD + half * HO;
#pragma unroll
        for (int i = 0; i < HO; i += 2) {
          if (F32) *reinterpret_cast<float2*>(a.of + off + i) = make_float2(o_acc[i] * inv, o_acc[i + 1] * inv);
          else *reinterpret_cast<uint32_t*>(a.oh + off + i) = pack_h2(o_acc[i] * inv, o_acc[i + 1] * inv);
        }
      }
    }
  }
  if (warp >= kAtSoftWarp0 && warp < kAtOutWarp0) asm volatile("bar.arrive 1, 512;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && s_fail && a.err_flag) atomicOr(a.err_flag, kErrTimeout);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tl
