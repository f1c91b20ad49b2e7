// Device helpers shared by the sm_100a kernels: PTX wrappers for programmatic
// dependent launch, streaming loads, the m16n8k16 fp16 MMA and INT4 unpacking.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tl {

constexpr int kGroup = 128;      // INT4 group size along K
constexpr int kMaxLanes = 16;    // rows of activations a GEMV launch handles

// Per activation row: which KV-cache lane it reads / writes and at what
// position.
struct RowCtx {
  int lane;
  int pos;
};

// ---- programmatic dependent launch -------------------------------------
// Kernels of the forward pass call pdl_trigger() (most at their start, so the
// next kernel may start its weight prefetch; the decode GEMVs where their
// caller says, the clustered QKV + attention kernel never) and pdl_wait()
// before they read anything an earlier kernel wrote.  Every kernel waits, so
// completion is transitive along the stream.
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- loads ---------------------------------------------------------------
// Weights are read once per pass: do not keep them in L1.
__device__ __forceinline__ uint4 ldg_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}
__device__ __forceinline__ uint2 ldg_stream2(const uint2* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
               : "=r"(r.x), "=r"(r.y)
               : "l"(p));
  return r;
}

// ---- launch timeline ---------------------------------------------------------
__device__ __forceinline__ long long globaltimer_ns() {
  long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Per-launch timeline of a layer kernel: `tr` holds kTraceEvents entries of
// one launch (zeroed by the caller), or is NULL.  Thread 0 of every CTA
// stamps event e >= 1 as the latest %globaltimer over the CTAs; event 0 holds
// the earliest start, complemented (so that both use atomicMax).
constexpr int kTraceEvents = 12;  // first start, last start, released, mid 1, mid 2, end, extra 6 .. 11
__device__ __forceinline__ void trace_start(unsigned long long* tr) {
  if (tr && threadIdx.x == 0) {
    const unsigned long long t = (unsigned long long)globaltimer_ns();
    atomicMax(tr, ~t);
    atomicMax(tr + 1, t);
  }
}
__device__ __forceinline__ void trace_mark(unsigned long long* tr, int e) {
  if (tr && threadIdx.x == 0) atomicMax(tr + e, (unsigned long long)globaltimer_ns());
}

// ---- bulk asynchronous copies (TMA engine) with mbarrier completion --------
__device__ __forceinline__ unsigned smem_u32(const void* p) {
  return (unsigned)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
// Make mbarrier initialisation visible to the asynchronous (copy) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Order this thread's earlier shared-memory accesses before later writes of
// the asynchronous proxy (a bulk copy into a buffer just read).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for phase `parity` of an mbarrier; false if it gave up.
constexpr long kMaxSpin = 1L << 22;
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity) {
  for (long i = 0; i < kMaxSpin; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}
// Bounded wait that gives up at once when another thread of the CTA already
// gave up (*fail != 0), so a stuck pipeline costs at most one time-out per
// thread and threads that share later barriers keep the same control flow.
__device__ __forceinline__ bool mbar_wait_or_fail(uint64_t* bar, unsigned parity, int* fail) {
  if (*reinterpret_cast<volatile int*>(fail)) return false;
  if (mbar_wait(bar, parity)) return true;
  atomicOr(fail, 1);
  return false;
}
// Bulk prefetch of `bytes` (a multiple of 16, 16-byte aligned) into L2.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, unsigned bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
// Global -> shared bulk copy of `bytes` (multiple of 16, both addresses 16-byte
// aligned); completion is signalled on `bar` as transaction bytes.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// L2 eviction-priority policies for loads and bulk copies: the loop block's
// weights are re-read every iteration (keep them), everything else is read
// once per token (stream it).
__device__ __forceinline__ uint64_t l2_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, unsigned bytes, uint64_t* bar,
                                              uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

// Device fault flag bits.
constexpr int kErrToken = 1;    // a token id outside [0, vocab) was replaced by 0
constexpr int kErrTimeout = 2;  // a bounded wait gave up

// ---- tensor-core MMA (m16n8k16, fp16 in, fp32 accumulate) ----------------
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4],
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ---- INT4 unpacking -------------------------------------------------------
// (w & mask) | 0x64006400 turns the two nibbles at bits 0..3 and 16..19 into
// the fp16 pair (1024 + n_lo, 1024 + n_hi): 0x6400 is 1024 and one unit in the
// last place of that binade is 1, so the nibble lands in the integer part.
__device__ __forceinline__ uint32_t nib_pair_to_h2_biased(uint32_t w) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(w), "r"(0x000F000Fu), "r"(0x64006400u));
  return r;
}

__device__ __forceinline__ uint32_t h2_sub(uint32_t a, uint32_t b) {
  __half2 r = __hsub2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t h2_mul(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
// Broadcast the low / high half of a pair into both halves.
__device__ __forceinline__ uint32_t h2_lo_lo(uint32_t a) { return __byte_perm(a, 0, 0x1010); }
__device__ __forceinline__ uint32_t h2_hi_hi(uint32_t a) { return __byte_perm(a, 0, 0x3232); }

__device__ __forceinline__ float2 h2_to_f2(uint32_t a) {
  return __half22float2(*reinterpret_cast<__half2*>(&a));
}

// Unpack one packed word of the tiled INT4 layout into the A fragment of an
// m16n8k16 MMA, with the zero point already removed: every element is the
// exact small integer q - z in fp16.
//   zz = (1024 + z_row_g, 1024 + z_row_g+8) as an fp16 pair.
__device__ __forceinline__ void unpack_a_frag(uint32_t w, uint32_t zz, uint32_t (&a)[4]) {
  const uint32_t zlo = h2_lo_lo(zz), zhi = h2_hi_hi(zz);
  a[0] = h2_sub(nib_pair_to_h2_biased(w), zlo);        // row g,   k 2t..2t+1
  a[1] = h2_sub(nib_pair_to_h2_biased(w >> 4), zhi);   // row g+8, k 2t..2t+1
  a[2] = h2_sub(nib_pair_to_h2_biased(w >> 8), zlo);   // row g,   k 2t+8..2t+9
  a[3] = h2_sub(nib_pair_to_h2_biased(w >> 12), zhi);  // row g+8, k 2t+8..2t+9
}

// INT2 weights: two 2-bit fields (bits 0..1 and 16..17 of w) as an fp16 pair
// biased by 1024, exact.
__device__ __forceinline__ uint32_t crumb_pair_to_h2_biased(uint32_t w) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(w), "r"(0x00030003u), "r"(0x64006400u));
  return r;
}
// The m16n8k16 A fragment of k16 step s (0 or 1) held by one INT2 word: the
// fields of step s sit at bits 8s + 2r (pair r, first element) and
// 16 + 8s + 2r (second element), r = 0..3 in the order of unpack_a_frag.
__device__ __forceinline__ void unpack_a_frag2(uint32_t w, int s, uint32_t zz, uint32_t (&a)[4]) {
  const uint32_t zlo = h2_lo_lo(zz), zhi = h2_hi_hi(zz);
  const uint32_t ws = w >> (8 * s);
  a[0] = h2_sub(crumb_pair_to_h2_biased(ws), zlo);        // row g,   k 2t..2t+1
  a[1] = h2_sub(crumb_pair_to_h2_biased(ws >> 2), zhi);   // row g+8, k 2t..2t+1
  a[2] = h2_sub(crumb_pair_to_h2_biased(ws >> 4), zlo);   // row g,   k 2t+8..2t+9
  a[3] = h2_sub(crumb_pair_to_h2_biased(ws >> 6), zhi);   // row g+8, k 2t+8..2t+9
}

// Byte offset of element pair (row, k..k+1), k even, in a 128-byte-swizzled
// K-major tile of `rows` rows and 128 k (two 64-wide atoms): the operand
// layout of the tcgen05 GEMM's B tiles and A stages.
__host__ __device__ inline uint32_t sw128_offset(int row, int k, int rows) {
  const int atom = k >> 6, kin = k & 63;
  const int chunk = kin >> 3, within = (kin & 7) * 2;
  return (uint32_t)(atom * rows * 128 + row * 128 + ((chunk ^ (row & 7)) << 4) + within);
}

// ---- thread-block clusters -------------------------------------------------
__device__ __forceinline__ unsigned cluster_rank() {
  unsigned r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Every thread of every CTA of the cluster arrives; release / acquire order
// shared-memory writes before the barrier with reads after it.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Distributed shared-memory address of `p` in the CTA of cluster rank `rank`.
__device__ __forceinline__ unsigned cluster_map(const void* p, unsigned rank) {
  unsigned out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(smem_u32(p)), "r"(rank));
  return out;
}
__device__ __forceinline__ float4 ld_cluster_f4(unsigned addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// ---- reductions -----------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float silu(float u) { return u / (1.0f + expf(-u)); }

// RoPE angle of pair j at position p: p * theta^(-2j/hd), evaluated in double
// precision and returned as (cos, sin) in float.  The model keeps a table of
// these values per (position, j), built once at load.
__device__ __forceinline__ float2 rope_cos_sin(int pos, int j, int hd, float theta) {
  const double inv_freq = exp(-(2.0 * (double)j / (double)hd) * log((double)theta));
  double s, c;
  sincos((double)pos * inv_freq, &s, &c);
  return make_float2((float)c, (float)s);
}

// (cos, sin) of pair j at position p from a [positions][hd/2] table when
// given, else computed.
__device__ __forceinline__ float2 rope_cs(const float2* tab, int pos, int j, int hd, float theta) {
  return tab ? tab[(size_t)pos * (hd >> 1) + j] : rope_cos_sin(pos, j, hd, theta);
}

}  // namespace tl
