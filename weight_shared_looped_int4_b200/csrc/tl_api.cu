// Host runtime behind the C ABI (include/tl.h): model creation and weight
// re-layout, the KV cache, the prefill / decode / score drivers with the loop
// over the shared block, and the op entry points.
//
// The forward pass follows TinyLoop README, "Why TinyLoop Exists":
// tokens -> embed -> pre blocks -> shared loop block x L -> output norm -> head.
// Effective layer l uses pre[l] for l < n_pre and the one loop block after
// that; its keys and values go to cache slice l of the lane.

#include "../../include/tl.h"
#include "internal.h"

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <tuple>
#include <vector>

#include "attention.cuh"
#include "attn_tc.cuh"
#include "common.cuh"
#include "decode_fused.cuh"
#include "gemm_tc.cuh"
#include "gemv_int4.cuh"
#include "misc.cuh"
#include "qkv_attn.cuh"

using namespace tl;

// ============================================================================
// errors
// ============================================================================
namespace {

thread_local std::string g_err;

tl_status fail(tl_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

tl_status cuda_fail(cudaError_t e, const char* what) {
  cudaGetLastError();  // clear a sticky-free launch error
  return fail(e == cudaErrorMemoryAllocation ? TL_ERR_OOM : TL_ERR_CUDA, "%s: %s", what,
              cudaGetErrorString(e));
}

#define TL_CUDA(call)                                   \
  do {                                                  \
    cudaError_t e_ = (call);                            \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
  } while (0)

struct DeviceGuard {
  int prev = -1;
  bool ok = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) == cudaSuccess && cudaSetDevice(dev) == cudaSuccess) ok = true;
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

// ============================================================================
// per-kernel event profiler and launch counter
// ============================================================================
struct Profiler {
  unsigned mask = 0;                 // classes being timed (0 = off)
  std::vector<cudaEvent_t> ev;       // begin/end pairs
  std::vector<int> cls;              // class of each pair
  int used = 0;
  static constexpr int kCapacity = 16384;
  void destroy() {
    for (cudaEvent_t e : ev) cudaEventDestroy(e);
    ev.clear();
    cls.clear();
    used = 0;
    mask = 0;
  }
};

thread_local Profiler* g_prof = nullptr;  // profiler of the model in the current call
thread_local int g_cls = -1;              // class of the next launch
// L2 access-policy window of the next launches (the loop block's weights while
// a loop iteration runs; num_bytes == 0 means none).
thread_local cudaAccessPolicyWindow g_window = {};
std::atomic<unsigned long long> g_launches{0};

struct ProfScope {  // installs a model's profiler for the duration of one API call
  Profiler* prev;
  explicit ProfScope(Profiler* p) : prev(g_prof) { g_prof = p; g_cls = -1; }
  ~ProfScope() { g_prof = prev; g_cls = -1; }
};

inline void kclass(int c) { g_cls = c; }

// ============================================================================
// launches (programmatic dependent launch on every kernel of the pass)
// ============================================================================
// Launch with event profiling and launch counting.  Ordinary kernels get
// programmatic dependent launch (and the current L2 access-policy window);
// `coop` launches are cooperative (all CTAs co-resident) and get neither.
template <typename... KArgs, typename... Args>
cudaError_t launch_impl(bool coop, dim3 cluster, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                        cudaStream_t st, Args&&... args) {
  Profiler* pr = g_prof;
  const bool timed = pr && g_cls >= 0 && (pr->mask & (1u << g_cls)) && pr->used < Profiler::kCapacity;
  if (timed) {
    if ((int)pr->ev.size() < 2 * (pr->used + 1)) {
      cudaEvent_t a, b;
      if (cudaEventCreate(&a) != cudaSuccess) return cudaErrorMemoryAllocation;
      if (cudaEventCreate(&b) != cudaSuccess) return cudaErrorMemoryAllocation;
      pr->ev.push_back(a);
      pr->ev.push_back(b);
      pr->cls.push_back(-1);
    }
    cudaEventRecord(pr->ev[2 * pr->used], st);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[3];
  if (coop) {
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
  } else {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
  }
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (!coop && g_window.num_bytes) {
    attr[cfg.numAttrs].id = cudaLaunchAttributeAccessPolicyWindow;
    attr[cfg.numAttrs].val.accessPolicyWindow = g_window;
    ++cfg.numAttrs;
  }
  if (cluster.x * cluster.y * cluster.z > 1) {
    attr[cfg.numAttrs].id = cudaLaunchAttributeClusterDimension;
    attr[cfg.numAttrs].val.clusterDim.x = cluster.x;
    attr[cfg.numAttrs].val.clusterDim.y = cluster.y;
    attr[cfg.numAttrs].val.clusterDim.z = cluster.z;
    ++cfg.numAttrs;
  }
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  if (e == cudaSuccess) g_launches.fetch_add(1, std::memory_order_relaxed);
  if (timed) {
    cudaEventRecord(pr->ev[2 * pr->used + 1], st);
    pr->cls[pr->used] = g_cls;
    ++pr->used;
  }
  return e;
}

template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                   Args&&... args) {
  return launch_impl(false, dim3(1, 1, 1), kern, grid, block, smem, st, std::forward<Args>(args)...);
}

constexpr size_t kMaxDynSmem = 220 * 1024;  // budget for dynamic smem per CTA

// One-time per-device attribute setup for kernels with large dynamic smem.
std::mutex g_init_mu;
std::map<int, bool> g_dev_init;

// Allow a kernel the opt-in shared memory of the device minus its static part.
template <typename K>
cudaError_t allow_max_smem(K* kern, int dev) {
  int optin = 0;
  cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              optin - (int)fa.sharedSizeBytes);
}

template <int NT, int IN, int EPI>
cudaError_t set_gemv_attr(int dev) {
  if constexpr (NT == 0) {
    const cudaError_t e = allow_max_smem(gemv_int4_kernel<NT, IN, EPI, 4>, dev);
    return e == cudaSuccess ? allow_max_smem(gemv_int4_kernel<NT, IN, EPI, 2>, dev) : e;
  } else {
    const cudaError_t e = allow_max_smem(gemv_rows_kernel<NT, IN, EPI, 4>, dev);
    return e == cudaSuccess ? allow_max_smem(gemv_rows_kernel<NT, IN, EPI, 2>, dev) : e;
  }
}

cudaError_t init_device_kernels(int dev) {
  std::lock_guard<std::mutex> lk(g_init_mu);
  if (g_dev_init[dev]) return cudaSuccess;
  cudaError_t e = cudaSuccess;
#define SET(NT, IN, EPI) \
  if (e == cudaSuccess) e = set_gemv_attr<NT, IN, EPI>(dev);
#define SET3(IN, EPI) SET(0, IN, EPI) SET(1, IN, EPI) SET(2, IN, EPI)
  SET3(IN_F16, EPI_STORE) SET3(IN_F32, EPI_RESID) SET3(IN_F32W, EPI_RESID) SET3(IN_NORM, EPI_SWIGLU) SET3(IN_NORM, EPI_ROPE_KV)
#undef SET3
#undef SET
  if (e == cudaSuccess) e = allow_max_smem(qkv_attn_kernel<64, false>, dev);
  if (e == cudaSuccess) e = allow_max_smem(qkv_attn_kernel<128, false>, dev);
  if (e == cudaSuccess) e = allow_max_smem(qkv_attn_kernel<64, true>, dev);
  if (e == cudaSuccess) e = allow_max_smem(qkv_attn_kernel<128, true>, dev);
  if (e == cudaSuccess) e = allow_max_smem(qkv_attn_kernel<64, false, 2>, dev);
  if (e == cudaSuccess) e = allow_max_smem(qkv_attn_kernel<128, false, 2>, dev);
  if (e == cudaSuccess) e = allow_max_smem(qkv_attn_kernel<64, true, 2>, dev);
  if (e == cudaSuccess) e = allow_max_smem(qkv_attn_kernel<128, true, 2>, dev);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(qkv_attn_kernel<64, false>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(qkv_attn_kernel<64, true>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(qkv_attn_kernel<128, true>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(qkv_attn_kernel<64, false, 2>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(qkv_attn_kernel<128, false, 2>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(qkv_attn_kernel<64, true, 2>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(qkv_attn_kernel<128, true, 2>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(qkv_attn_kernel<128, false>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess) e = allow_max_smem(decode_fused_kernel<64>, dev);
  if (e == cudaSuccess) e = allow_max_smem(decode_fused_kernel<128>, dev);
  if (e == cudaSuccess) e = allow_max_smem(head_argmax_kernel<1>, dev);
  if (e == cudaSuccess) e = allow_max_smem(head_argmax_kernel<2>, dev);
  if (e == cudaSuccess) e = allow_max_smem(gemm_int4_tc_kernel<TC_RESID, true>, dev);
  if (e == cudaSuccess) e = allow_max_smem(gemm_int4_tc_kernel<TC_RAW, true>, dev);
  if (e == cudaSuccess) e = allow_max_smem(gemm_int4_tc_kernel<TC_ROPE_KV, true>, dev);
  if (e == cudaSuccess) e = allow_max_smem(gemm_int4_tc_kernel<TC_STORE, false>, dev);
  if (e == cudaSuccess) e = allow_max_smem(gemm_int4_tc_kernel<TC_SWIGLU_B, true>, dev);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(prefill_attn_tc_kernel<128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)attn_tc_smem_bytes<128>());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(prefill_attn_tc_kernel<128, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)attn_tc_smem_bytes<128>());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(prefill_attn_tc_kernel<64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)attn_tc_smem_bytes<64>());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(prefill_attn_tc_kernel<64, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)attn_tc_smem_bytes<64>());
  if (e == cudaSuccess) e = allow_max_smem(head_direct_kernel, dev);
  // split-K clusters of up to 16 CTAs
#define NP(EPI, LO)   \
  if (e == cudaSuccess) \
    e = cudaFuncSetAttribute(gemm_int4_tc_kernel<EPI, LO>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  NP(TC_RESID, true) NP(TC_RAW, true) NP(TC_ROPE_KV, true) NP(TC_STORE, false) NP(TC_SWIGLU_B, true)
#undef NP
#define ATT(HD, REP)                                                                  \
  if (e == cudaSuccess) e = allow_max_smem(decode_attn_kernel<HD, REP, true>, dev);   \
  if (e == cudaSuccess) e = allow_max_smem(decode_attn_kernel<HD, REP, true, true>, dev);   \
  if (e == cudaSuccess) e = allow_max_smem(decode_attn_kernel<HD, REP, false>, dev);  \
  if (e == cudaSuccess) e = allow_max_smem(prefill_attn_mma_kernel<HD, REP, true, false>, dev); \
  if (e == cudaSuccess) e = allow_max_smem(prefill_attn_mma_kernel<HD, REP, false, false>, dev); \
  if (e == cudaSuccess) e = allow_max_smem(prefill_attn_mma_kernel<HD, REP, true, true>, dev);
  ATT(64, 1) ATT(64, 2) ATT(64, 4) ATT(64, 8) ATT(128, 1) ATT(128, 2) ATT(128, 4) ATT(128, 8)
#undef ATT
  if (e == cudaSuccess) g_dev_init[dev] = true;
  return e;
}

// Largest activation-row count (<= 16) per GEMV launch that fits shared memory.
int gemv_rows_per_launch(int K, bool lo, int tpc) {
  int M = kMaxLanes;
  while (M > 0 && gemv_smem_bytes(K, M, lo, tpc) > kMaxDynSmem) --M;
  return M;
}

cudaError_t launch_gemv(const GemvArgs& a, int grid, int in_mode, int epi, cudaStream_t st) {
  const bool lo = in_mode != IN_F16;
  const int nt = gemv_nt(a.M, lo);
  const size_t smem = gemv_smem_bytes(a.K, a.M, lo, gemv_tpc(epi));
  const dim3 g(grid), b(kGemvThreads);
#define CASE(NT, IN, EPI, KERN)                                                                       \
  if (nt == NT && in_mode == IN && epi == EPI)                                                        \
    return a.bits == 2 ? launch(KERN<NT, IN, EPI, 2>, g, b, smem, st, a)                              \
                       : launch(KERN<NT, IN, EPI, 4>, g, b, smem, st, a);
  // one row pass for <= 4 rows (8 without the lo plane), phases of K above
#define CASE3(IN, EPI) CASE(0, IN, EPI, gemv_int4_kernel) CASE(1, IN, EPI, gemv_rows_kernel) CASE(2, IN, EPI, gemv_rows_kernel)
  CASE3(IN_F16, EPI_STORE) CASE3(IN_F32, EPI_RESID) CASE3(IN_F32W, EPI_RESID) CASE3(IN_NORM, EPI_SWIGLU) CASE3(IN_NORM, EPI_ROPE_KV)
#undef CASE3
#undef CASE
  return cudaErrorInvalidValue;
}

// Launch a GEMV over `total` activation rows, in chunks of as many rows as
// fit shared memory; every row-indexed pointer advances with the chunk.
cudaError_t launch_gemv_rows(GemvArgs a, int total, int in_mode, int epi, int grid, cudaStream_t st) {
  const int per = gemv_rows_per_launch(a.K, in_mode != IN_F16, gemv_tpc(epi));
  if (per < 1) return cudaErrorInvalidValue;
  for (int r0 = 0; r0 < total; r0 += per) {
    GemvArgs c = a;
    c.M = std::min(per, total - r0);
    if (c.x) c.x += (size_t)r0 * a.ldx;
    if (c.xh) c.xh += (size_t)r0 * a.ldx;
    if (c.rows) c.rows += r0;
    if (c.q_out) c.q_out += (size_t)r0 * a.ldq;
    if (c.y) c.y += (size_t)r0 * a.ldy;
    if (c.yf) c.yf += (size_t)r0 * a.ldy;
    if (c.resid) c.resid += (size_t)r0 * a.ldr;
    if (c.kv_stage) c.kv_stage += (size_t)r0 * 2 * a.n_kv_rows;   // [row][K|V][Hkv * hd]
    const cudaError_t e = launch_gemv(c, grid, in_mode, epi, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// ============================================================================
// INT4 weights on the device
// ============================================================================
struct Int4Dev {
  int K = 0, N = 0, n_tiles = 0;
  int bits = 4;            // 4, or 2 for the INT2 body (w then holds uint2 per lane and chunk)
  uint4* w = nullptr;
  uint2* sz = nullptr;
  uint8_t* tc = nullptr;   // tensor-core layout (prefill), always owned
  bool owned = true;   // false when w / sz live in a block's arena
  static size_t tc_bytes(int K, int N) { return (size_t)((N + kTcRows - 1) / kTcRows) * (K / 128) * kTcRawBytes; }
  static size_t w_bytes(int K, int N, int bits = 4) {
    return (size_t)(((N + 31) / 32) * 2) * (K / 64) * 32 * (bits == 2 ? sizeof(uint2) : sizeof(uint4));
  }
  static size_t sz_bytes(int K, int N) { return (size_t)(((N + 31) / 32) * 2) * (K / 128) * 8 * sizeof(uint2); }
  size_t bytes() const { return w_bytes(K, N, bits) + sz_bytes(K, N) + (tc ? tc_bytes(K, N) : 0); }
  void free_all() {
    if (owned) {
      if (w) cudaFree(w);
      if (sz) cudaFree(sz);
    }
    if (tc) cudaFree(tc);
    w = nullptr;
    sz = nullptr;
    tc = nullptr;
  }
};

// A bump allocator over one device allocation (256-byte aligned pieces).
struct Arena {
  char* base = nullptr;
  size_t size = 0, used = 0;
  void* take(size_t bytes) {
    const size_t off = (used + 255) & ~size_t(255);
    if (off + bytes > size) return nullptr;
    used = off + bytes;
    return base + off;
  }
};

// Copy one linear in the storage format to the device and re-lay it out.
// N is padded to whole pairs of 16-row tiles with zero weights.
// perm_F != 0: the tensor-core copy interleaves gate rows [0, F) and up rows
// [F, 2F) per 128-row tile (for the fused SwiGLU epilogue).
tl_status upload_int4(const tl_int4_linear& h, int K, int N, Int4Dev* out, cudaStream_t st, Arena* arena = nullptr,
                      int perm_F = 0, int bits = 4) {
  if (!h.qweight || !h.scales || !h.qzeros) return fail(TL_ERR_INVALID_ARG, "null INT4 array");
  const int epw = 32 / bits;   // fields per storage word
  const int G = K / 128, zw = (G + epw - 1) / epw;
  out->K = K;
  out->N = N;
  out->bits = bits;
  out->n_tiles = ((N + 31) / 32) * 2;
  const size_t qb = (size_t)N * (K / epw) * 4, sb = (size_t)N * G * 2, zb = (size_t)N * zw * 4;
  void *dq = nullptr, *ds = nullptr, *dz = nullptr;
  tl_status rc = TL_OK;
  cudaError_t e = cudaMalloc(&dq, qb);
  if (e == cudaSuccess) e = cudaMalloc(&ds, sb);
  if (e == cudaSuccess) e = cudaMalloc(&dz, zb);
  if (arena) {
    out->owned = false;
    out->w = (uint4*)arena->take(Int4Dev::w_bytes(K, N, bits));
    out->sz = (uint2*)arena->take(Int4Dev::sz_bytes(K, N));
    if (e == cudaSuccess && (!out->w || !out->sz)) e = cudaErrorMemoryAllocation;
  } else {
    if (e == cudaSuccess) e = cudaMalloc(&out->w, Int4Dev::w_bytes(K, N, bits));
    if (e == cudaSuccess) e = cudaMalloc(&out->sz, Int4Dev::sz_bytes(K, N));
  }
  if (e == cudaSuccess) e = cudaMalloc(&out->tc, Int4Dev::tc_bytes(K, N));
  if (e == cudaSuccess) e = cudaMemcpyAsync(dq, h.qweight, qb, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(ds, h.scales, sb, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dz, h.qzeros, zb, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) {
    const size_t tw = (size_t)out->n_tiles * (K / 64) * 32;
    if (bits == 2)
      repack_int2_weights_kernel<<<(unsigned)((tw + 255) / 256), 256, 0, st>>>(
          (const uint32_t*)dq, K, N, out->n_tiles, reinterpret_cast<uint2*>(out->w));
    else
      repack_int4_weights_kernel<<<(unsigned)((tw + 255) / 256), 256, 0, st>>>(
          (const uint32_t*)dq, K, N, out->n_tiles, out->w);
    const size_t ts = (size_t)out->n_tiles * G * 8;
    repack_int4_scales_kernel<<<(unsigned)((ts + 255) / 256), 256, 0, st>>>(
        (const uint16_t*)ds, (const uint32_t*)dz, K, N, out->n_tiles, out->sz, bits);
    const size_t tt = (size_t)((N + kTcRows - 1) / kTcRows) * G * kTcRows * 16;
    repack_int4_tc_kernel<<<(unsigned)((tt + 255) / 256), 256, 0, st>>>((const uint32_t*)dq, (const uint32_t*)dz, K,
                                                                       N, perm_F, out->tc, bits);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) {
    rc = cuda_fail(e, "upload INT4 linear");
    out->free_all();
  }
  if (dq) cudaFree(dq);
  if (ds) cudaFree(ds);
  if (dz) cudaFree(dz);
  return rc;
}

tl_status upload_f16(const uint16_t* h, size_t n, __half** out, cudaStream_t st) {
  if (!h) return fail(TL_ERR_INVALID_ARG, "null fp16 array");
  TL_CUDA(cudaMalloc(out, n * 2));
  TL_CUDA(cudaMemcpyAsync(*out, h, n * 2, cudaMemcpyHostToDevice, st));
  return TL_OK;
}

struct BlockDev {
  __half* attn_norm = nullptr;
  __half* ffn_norm = nullptr;
  Int4Dev qkv, o, gate_up, down;
  Arena arena;   // one allocation holding the four linears (an L2 window)
  void free_all() {
    if (attn_norm) cudaFree(attn_norm);
    if (ffn_norm) cudaFree(ffn_norm);
    attn_norm = ffn_norm = nullptr;
    qkv.free_all();
    o.free_all();
    gate_up.free_all();
    down.free_all();
    if (arena.base) cudaFree(arena.base);
    arena = Arena{};
  }
  size_t bytes(int d) const { return qkv.bytes() + o.bytes() + gate_up.bytes() + down.bytes() + 4 * (size_t)d; }
};

// Per-step row description, passed by value to the step's first kernel (so
// no host buffer has to outlive the call).  Rows are the step's lanes in
// decreasing loop order.
struct StepDesc {
  int n;
  int lane[kMaxLanes];
  int pos[kMaxLanes];
  int tok_index[kMaxLanes];
  int out_row[kMaxLanes];
  const int32_t* tokens;
  float* logits;
  int32_t* argmax;
};

// First kernel of a decode step: publishes the rows' lanes / positions and
// the output pointers to device memory, then gathers the embeddings.
__global__ void step_embed_kernel(StepDesc s, const __half* __restrict__ E, int d, int vocab, RowCtx* rows,
                                  int* out_row, HeadIO* io, float* __restrict__ x, int* err_flag) {
  const int row = blockIdx.x;
  pdl_trigger();
  pdl_wait();
  if (row == 0) {
    if (threadIdx.x < s.n) {
      rows[threadIdx.x].lane = s.lane[threadIdx.x];
      rows[threadIdx.x].pos = s.pos[threadIdx.x];
      out_row[threadIdx.x] = s.out_row[threadIdx.x];
    }
    if (threadIdx.x == 0) {
      io->logits = s.logits;
      io->argmax = s.argmax;
    }
  }
  int tok = s.tokens[s.tok_index[row]];
  if (tok < 0 || tok >= vocab) {
    if (threadIdx.x == 0) atomicOr(err_flag, kErrToken);
    tok = 0;
  }
  const __half* e = E + (size_t)tok * d;
  float* xr = x + (size_t)row * d;
  for (int k = threadIdx.x * 2; k < d; k += blockDim.x * 2)
    *reinterpret_cast<float2*>(xr + k) = __half22float2(*reinterpret_cast<const __half2*>(e + k));
}

__global__ void fill_rows_kernel(RowCtx* rows, int n, int lane, int pos0) {
  pdl_trigger();
  pdl_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    rows[i].lane = lane;
    rows[i].pos = pos0 + i;
  }
}


// ---- tensor-core INT4 GEMM (prefill / large M) ------------------------------
struct TcScratch {
  uint8_t* bt = nullptr;       // prepared activation tiles
  uint8_t* bt2 = nullptr;      // the down projection's tiles, written by the gate_up epilogue
  uint8_t* bt3 = nullptr;      // gate_up's tiles (x * ffn gains), written by the O epilogue
  float* ss_attn = nullptr;    // per (d row tile, token) sums of x^2 for the next attention RMSNorm
  float* ss_ffn = nullptr;     // ... for the FFN RMSNorm
  int ss_ld = 0;               // tokens per row of ss_*
  size_t bt_bytes = 0;
  float* partial = nullptr;    // split-K partial tiles
  size_t partial_bytes = 0;
  unsigned* tickets = nullptr; // >= 4096 entries, zero between launches
  int* err_flag = nullptr;
  int n_sm = 148;
};

constexpr int kTcMinTokens = 32;   // below this the GEMV path is used

size_t tc_bt_bytes(int T, int K, bool lo) {
  return (size_t)((T + kTcTokens - 1) / kTcTokens) * (K / 128) * tc_b_bytes(lo);
}

using TcKernel = void (*)(const TcGemmArgs);
constexpr int kTcMaxCluster = 16;   // non-portable cluster size limit

// Whether `clusters` clusters of S CTAs of a GEMM variant can be resident on
// the current device at once (cached per device, kernel and S).
bool tc_clusters_fit(TcKernel kern, int S, int clusters, size_t smem) {
  static std::mutex mu;
  static std::map<std::tuple<int, const void*, int>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  const auto key = std::make_tuple(dev, (const void*)kern, S);
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(key);
  if (it == cache.end()) {
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(1, 1, S);
    lc.blockDim = dim3(kTcThreads);
    lc.dynamicSmemBytes = smem;
    cudaLaunchAttribute la[1];
    la[0].id = cudaLaunchAttributeClusterDimension;
    la[0].val.clusterDim.x = 1;
    la[0].val.clusterDim.y = 1;
    la[0].val.clusterDim.z = S;
    lc.attrs = la;
    lc.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &lc) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    it = cache.emplace(key, n).first;
  }
  return it->second >= clusters;
}

cudaError_t launch_prep(int mode, const PrepArgs& p, cudaStream_t st) {
  if (mode == PREP_NONE) return cudaSuccess;
  const dim3 g(((p.T + kTcTokens - 1) / kTcTokens) * kTcTokens), b(256);
  switch (mode) {
    case PREP_NORM: return launch(prep_b_kernel<PREP_NORM>, g, b, 0, st, p);
    case PREP_F16: return launch(prep_b_kernel<PREP_F16>, g, b, 0, st, p);
  }
  return cudaErrorInvalidValue;
}

// Runs prep + GEMM for T tokens.  `ta` carries the epilogue outputs; the
// weight, activation and scratch fields are filled here.
// `b_tiles`: where the GEMM reads its prepared B tiles (default: the scratch
// the prep kernel writes).
cudaError_t launch_tc_linear(const uint8_t* wtc, const uint2* sz, int K, int N, int n16_tiles, int prep_mode,
                             PrepArgs pa, TcGemmArgs ta, int epi, int T, const TcScratch& sc, cudaStream_t st,
                             const uint8_t* b_tiles = nullptr) {
  const bool lo = prep_mode != PREP_F16;
  if (tc_bt_bytes(T, K, lo) > sc.bt_bytes) return cudaErrorInvalidValue;
  pa.K = K;
  pa.T = T;
  pa.bt = sc.bt;
  cudaError_t e = launch_prep(prep_mode, pa, st);
  if (e != cudaSuccess) return e;
  const int G = K / 128;
  const int row_tiles = (N + kTcRows - 1) / kTcRows, tok_tiles = (T + kTcTokens - 1) / kTcTokens;
  if (row_tiles * tok_tiles > 4096) return cudaErrorInvalidValue;
  TcKernel kern = nullptr;
  if (epi == TC_RESID && lo) kern = gemm_int4_tc_kernel<TC_RESID, true>;
  else if (epi == TC_RAW && lo) kern = gemm_int4_tc_kernel<TC_RAW, true>;
  else if (epi == TC_ROPE_KV && lo) kern = gemm_int4_tc_kernel<TC_ROPE_KV, true>;
  else if (epi == TC_STORE && !lo) kern = gemm_int4_tc_kernel<TC_STORE, false>;
  else if (epi == TC_SWIGLU_B && lo) kern = gemm_int4_tc_kernel<TC_SWIGLU_B, true>;
  else return cudaErrorInvalidValue;
  const size_t smem = tc_smem_bytes(lo);
  // Split K when the tiles alone leave SMs idle.  Preferred: the splits of a
  // tile run as one thread-block cluster and reduce in distributed shared
  // memory (as many splits as keep every cluster resident in one wave);
  // otherwise partial sums go to global scratch and a merge kernel adds them.
  // (measured on the 400M model: a cluster reduction with fewer splits is
  // slower than the partial buffer + merge kernel with more, so the cluster
  // form is taken only where it keeps every split)
  int splits = std::max(1, std::min(G, sc.n_sm / (row_tiles * tok_tiles)));
  while (splits > 1 && (size_t)splits * row_tiles * tok_tiles * kTcRows * kTcTokens * 4 > sc.partial_bytes) --splits;
  bool cluster = false;
  if (splits > 1 && splits <= kTcMaxCluster && tc_clusters_fit(kern, splits, row_tiles * tok_tiles, smem))
    cluster = true;
  ta.wtc = wtc; ta.sz = sz; ta.K = K; ta.N = N; ta.n16_tiles = n16_tiles;
  ta.bt = b_tiles ? b_tiles : sc.bt; ta.T = T; ta.splits = splits; ta.cluster = cluster ? 1 : 0;
  ta.partial = sc.partial; ta.tickets = sc.tickets; ta.err_flag = sc.err_flag;
  const dim3 g(row_tiles, tok_tiles, splits), b(kTcThreads);
  e = launch_impl(false, cluster ? dim3(1, 1, splits) : dim3(1, 1, 1), kern, g, b, smem, st, ta);
  if (e != cudaSuccess || splits == 1 || cluster) return e;
  const dim3 mg(row_tiles, tok_tiles, kTcTokens / kTcMergeTok);
  if (epi == TC_RESID) return launch(tc_merge_kernel<TC_RESID>, mg, dim3(256), 0, st, ta);
  if (epi == TC_RAW) return launch(tc_merge_kernel<TC_RAW>, mg, dim3(256), 0, st, ta);
  if (epi == TC_ROPE_KV) return launch(tc_merge_kernel<TC_ROPE_KV>, mg, dim3(256), 0, st, ta);
  if (epi == TC_SWIGLU_B) return launch(tc_merge_kernel<TC_SWIGLU_B>, mg, dim3(256), 0, st, ta);
  return launch(tc_merge_kernel<TC_STORE>, mg, dim3(256), 0, st, ta);
}

template <int HD, int REP, bool F32>
cudaError_t launch_decode_attn_t(const DecodeAttnArgs& a, int rows, cudaStream_t st) {
  if (a.ks)   // INT8 cache (fp32 queries)
    return F32 ? launch(decode_attn_kernel<HD, REP, true, true>, dim3(kDecodeMaxSplits, a.Hkv, rows), dim3(kDecodeThreads),
                        decode_attn_smem_bytes(HD, REP, true), st, a)
               : cudaErrorInvalidValue;
  return launch(decode_attn_kernel<HD, REP, F32>, dim3(kDecodeMaxSplits, a.Hkv, rows), dim3(kDecodeThreads), decode_attn_smem_bytes(HD, REP),
                st, a);
}

cudaError_t launch_decode_attn(const DecodeAttnArgs& a, int rows, int hd, int rep, bool f32, cudaStream_t st) {
#define C(HD, REP)                                                                                   \
  if (hd == HD && rep == REP)                                                                        \
    return f32 ? launch_decode_attn_t<HD, REP, true>(a, rows, st) : launch_decode_attn_t<HD, REP, false>(a, rows, st);
  C(64, 1) C(64, 2) C(64, 4) C(64, 8) C(128, 1) C(128, 2) C(128, 4) C(128, 8)
#undef C
  return cudaErrorInvalidValue;
}

// Prefill attention runs on tcgen05 from this many queries on, below it on
// 16-query mma.sync tiles (tl_set_prefill_attention_tc_min).
std::atomic<int> g_at_min_tokens{1024};

cudaError_t launch_prefill_attn(PrefillAttnArgs a, int B, int hd, int rep, bool f32, cudaStream_t st) {
  a.rep = rep;
  const bool kv8 = a.ks != nullptr;   // INT8 KV cache: the 16-query tile kernel, fp32 queries
  if (kv8 && !f32) return cudaErrorInvalidValue;
  if (!kv8 && a.T >= g_at_min_tokens.load(std::memory_order_relaxed)) {
    // tensor cores (tcgen05): one CTA per (query head, 128-query tile, batch entry)
    const dim3 grid(a.Hkv * rep, (a.T + kAtQ - 1) / kAtQ, B);   // heads fastest, longest tiles first
    if (hd == 128)
      return f32 ? launch(prefill_attn_tc_kernel<128, true>, grid, dim3(kAtThreads), attn_tc_smem_bytes<128>(), st, a)
                 : launch(prefill_attn_tc_kernel<128, false>, grid, dim3(kAtThreads), attn_tc_smem_bytes<128>(), st, a);
    if (hd == 64)
      return f32 ? launch(prefill_attn_tc_kernel<64, true>, grid, dim3(kAtThreads), attn_tc_smem_bytes<64>(), st, a)
                 : launch(prefill_attn_tc_kernel<64, false>, grid, dim3(kAtThreads), attn_tc_smem_bytes<64>(), st, a);
    return cudaErrorInvalidValue;
  }
  // short passes (decode-sized verify / append chunks): 16-query tiles on
  // mma.sync; query heads per CTA: the whole group, halved while the grid
  // would leave SMs idle; each CTA stages its kv head's keys itself
  int hpc = rep;
  const int qtiles = (a.T + 15) / 16;
  while (hpc > 1 && (long)qtiles * (a.Hkv * rep / hpc) * B < 148) hpc /= 2;
  const dim3 grid(qtiles, a.Hkv * rep / hpc, B);
  const size_t smem = prefill_attn_smem_bytes(hd);
#define C(HD, REP)                                                                                       \
  if (hd == HD && hpc == REP)                                                                            \
    return kv8 ? launch(prefill_attn_mma_kernel<HD, REP, true, true>, grid, dim3(REP * 32), smem, st, a)  \
               : f32 ? launch(prefill_attn_mma_kernel<HD, REP, true, false>, grid, dim3(REP * 32), smem, st, a) \
                     : launch(prefill_attn_mma_kernel<HD, REP, false, false>, grid, dim3(REP * 32), smem, st, a);
  C(64, 1) C(64, 2) C(64, 4) C(64, 8) C(128, 1) C(128, 2) C(128, 4) C(128, 8)
#undef C
  return cudaErrorInvalidValue;
}

bool rep_ok(int rep) { return rep == 1 || rep == 2 || rep == 4 || rep == 8; }

// The clustered QKV + attention kernel for a head size, KV cache mode and
// weight width.
using QaKernel = void (*)(QkvAttnArgs);
QaKernel qa_kernel(int hd, bool kv8, int bits) {
  if (bits == 2)
    return hd == 64 ? (kv8 ? qkv_attn_kernel<64, true, 2> : qkv_attn_kernel<64, false, 2>)
                    : (kv8 ? qkv_attn_kernel<128, true, 2> : qkv_attn_kernel<128, false, 2>);
  return hd == 64 ? (kv8 ? qkv_attn_kernel<64, true, 4> : qkv_attn_kernel<64, false, 4>)
                  : (kv8 ? qkv_attn_kernel<128, true, 4> : qkv_attn_kernel<128, false, 4>);
}

}  // namespace

// ============================================================================
// model
// ============================================================================
struct tl_model {
  tl_config cfg{};
  int device = 0;
  int n_layers_max = 0;
  std::vector<BlockDev> pre;
  BlockDev loop;
  __half* embed = nullptr;
  __half* out_norm = nullptr;
  uint4* head_w = nullptr;
  int head_pf_layer = -1;         // decode step: the layer whose O projection prefetches the head
  // KV cache: [max_lanes + 1][n_layers_max][2][Hkv][max_ctx][hd] fp16, or
  // with kv_int8 the same element layout in int8 codes (kv points at them)
  // plus the scales kvs with the head dimension collapsed (kv8.cuh)
  __half* kv = nullptr;
  float* kvs = nullptr;
  float* kv_stage = nullptr;   // INT8: a pass's fp32 keys / values [rows][2][Hkv][hd]
  bool kv_int8 = false;
  long long plane = 0, layer_stride = 0, lane_stride = 0;
  // workspaces
  float* x = nullptr;   // residual stream [rows][d]
  float* q = nullptr;   // rotated queries [rows][Hq*hd]
  float* o = nullptr;   // attention output [rows][Hq*hd]
  float* h = nullptr;   // SwiGLU output [rows][F]
  RowCtx* rows = nullptr;
  int* tok_index = nullptr;
  int* out_row = nullptr;
  float* attn_part = nullptr;
  unsigned* tickets = nullptr;  // attention [16][Hkv] then head [1]
  float* head_val = nullptr;
  int* head_idx = nullptr;
  int* err_flag = nullptr;
  int32_t* spec_tok = nullptr;    // speculative decode / early exit tokens [2 kMaxLanes + 2]
  int head_grid = 0;
  int hd_grid = 0;                // CTAs of the direct-load head (one per SM)
  HeadIO* io = nullptr;          // output pointers of the current decode step
  TcScratch tc;                  // tensor-core GEMM scratch (prefill)
  cudaAccessPolicyWindow loop_window = {};  // keeps the loop block's weights in L2
  size_t l2_persist_bytes = 0;
  float2* rope_tab = nullptr;    // RoPE (cos, sin) [max_ctx][hd/2]
  cudaStream_t setup_stream = nullptr;
  cudaStream_t cap_stream = nullptr;   // stream used to capture decode graphs
  struct Graph {
    cudaGraphExec_t exec = nullptr;
    int kernels = 0;
  };
  std::map<std::string, Graph> graphs;   // decode step graphs by row pattern
  bool use_graphs = true;
  bool use_qkv_attn = true;       // the clustered QKV + attention kernel fits the device
  bool qa_select = true;          // decode steps take it (set at creation from max_lanes,
                                  // tl_model_set_clustered_decode)
  int qa_smem_max = 0;            // dynamic shared memory it may use
  int decode_path = TL_DECODE_AUTO;
  // single-kernel decode step
  bool fused_ok = false;          // the model's shapes and the device allow it
  int fused_grid = 0;             // one CTA per SM
  int fused_smem_max = 0;         // dynamic shared memory the kernel may use
  FusedArgs fused{};              // model part of the arguments
  unsigned* fused_bar = nullptr;  // grid-barrier words [4]
  float* fused_val = nullptr;     // per-CTA best logit [grid][4]
  int* fused_idx = nullptr;
  unsigned long long* trace = nullptr;  // caller's phase-timeline buffer (device), or NULL
  long long trace_cap = 0;
  long long trace_i = -1;         // next layer-launch record of a layered decode step (-1: none)
  std::vector<int> lane_len, lane_loops;
  size_t weight_bytes = 0, kv_bytes = 0, ws_bytes = 0;
  Profiler prof;

  unsigned* attn_tickets() const { return tickets; }
  unsigned* head_ticket() const { return tickets + kMaxLanes * cfg.n_kv_heads; }
  // element pointers of lane 0's planes (int8 codes when kv_int8: same
  // element offsets, reinterpreted by the kernels)
  __half* k_plane(int layer) const {
    return kv_int8 ? reinterpret_cast<__half*>(reinterpret_cast<int8_t*>(kv) + layer * layer_stride)
                   : kv + layer * layer_stride;
  }
  __half* v_plane(int layer) const {
    return kv_int8 ? reinterpret_cast<__half*>(reinterpret_cast<int8_t*>(kv) + layer * layer_stride + plane)
                   : kv + layer * layer_stride + plane;
  }
  // INT8 scales of lane 0's planes (NULL for fp16); lane l adds l * lane_stride / hd
  float* ks_plane(int layer) const { return kv_int8 ? kvs + layer * layer_stride / cfg.head_dim : nullptr; }
  float* vs_plane(int layer) const {
    return kv_int8 ? kvs + (layer * layer_stride + plane) / cfg.head_dim : nullptr;
  }
  // an element offset within the cache as a pointer into it (int8 or fp16)
  __half* kv_at(long long e) const {
    return kv_int8 ? reinterpret_cast<__half*>(reinterpret_cast<int8_t*>(kv) + e) : kv + e;
  }
  // planes and scales of one lane
  __half* k_lane(int layer, int lane) const { return kv_at(layer * layer_stride + lane * lane_stride); }
  __half* v_lane(int layer, int lane) const { return kv_at(layer * layer_stride + plane + lane * lane_stride); }
  float* ks_lane(int layer, int lane) const {
    return kv_int8 ? kvs + (layer * layer_stride + lane * lane_stride) / cfg.head_dim : nullptr;
  }
  float* vs_lane(int layer, int lane) const {
    return kv_int8 ? kvs + (layer * layer_stride + plane + lane * lane_stride) / cfg.head_dim : nullptr;
  }
  const BlockDev& block(int layer) const { return layer < cfg.n_pre ? pre[layer] : loop; }

  void free_all() {
    for (auto& b : pre) b.free_all();
    loop.free_all();
    for (auto& kv_ : graphs)
      if (kv_.second.exec) cudaGraphExecDestroy(kv_.second.exec);
    graphs.clear();
    if (cap_stream) cudaStreamDestroy(cap_stream);
    void* ptrs[] = {embed, out_norm, head_w, kv, kvs, kv_stage, x, q, o, h, rows, tok_index, out_row, spec_tok,
                    attn_part, tickets, head_val, head_idx, err_flag, io, tc.bt, tc.bt2, tc.bt3, tc.ss_attn,
                    tc.ss_ffn, tc.partial, tc.tickets,
                    rope_tab, fused_bar, fused_val, fused_idx};
    for (void* p : ptrs)
      if (p) cudaFree(p);
    if (setup_stream) cudaStreamDestroy(setup_stream);
    prof.destroy();
  }
};

namespace {

// Shared-memory plan of the single-kernel decode step for `rows` rows: the
// largest ring (<= kFusedMaxSlots slots) that fits beside the activation
// planes and the reduction buffer.  False if not even two slots fit.
// Head-only launches need only the d-wide activation planes and the head's
// double reduction buffer, which leaves room for more ring slots.
bool fused_plan(const tl_model* m, int rows, FusedArgs* f, size_t* smem) {
  const tl_config& c = m->cfg;
  const int qdim = c.n_q_heads * c.head_dim;
  const int kmax = f->head_only ? c.d_model : std::max(std::max(c.d_model, qdim), c.ffn_dim);
  if (kmax > kFusedStageV4 * 4 * kFusedCompute) return false;
  const int area = f->head_only ? (2 * rows * (c.d_model + 8) * 2 + 127) / 128 * 128
                                : fused_area_bytes(rows, kmax, c.n_q_heads / c.n_kv_heads, c.head_dim);
  const int red = f->head_only ? 2 * kFusedWarps * 64 * 4 : fused_red_bytes(*f, m->fused_grid);
  const int xown = f->head_only ? 0 : fused_xown_bytes(*f, m->fused_grid);
  const long avail = (long)m->fused_smem_max - area - red - xown;
  const long ns = std::min<long>(kFusedMaxSlots, avail / kFusedSlotBytes);
  if (ns < 2) return false;
  f->n_slots = (int)ns;
  f->area_bytes = area;
  f->red_bytes = red;
  *smem = (size_t)ns * kFusedSlotBytes + area + red + xown;
  return true;
}

tl_status validate_config(const tl_config* c) {
  if (!c) return fail(TL_ERR_INVALID_ARG, "null config");
  if (c->d_model < 128 || c->d_model % 128 || c->d_model > 8192)
    return fail(TL_ERR_UNSUPPORTED, "d_model must be a multiple of 128 in [128, 8192]");
  if (c->head_dim != 64 && c->head_dim != 128) return fail(TL_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (c->n_q_heads < 1 || c->n_kv_heads < 1 || c->n_q_heads % c->n_kv_heads)
    return fail(TL_ERR_INVALID_ARG, "n_q_heads must be a positive multiple of n_kv_heads");
  if (!rep_ok(c->n_q_heads / c->n_kv_heads)) return fail(TL_ERR_UNSUPPORTED, "n_q_heads/n_kv_heads must be 1, 2, 4 or 8");
  if ((c->n_q_heads * c->head_dim) % 128 || c->n_q_heads * c->head_dim > 8192)
    return fail(TL_ERR_UNSUPPORTED, "n_q_heads*head_dim must be a multiple of 128, <= 8192");
  if (c->ffn_dim < 128 || c->ffn_dim % 128 || c->ffn_dim > 12288)
    return fail(TL_ERR_UNSUPPORTED, "ffn_dim must be a multiple of 128 in [128, 12288]");
  if (c->vocab < 16 || c->vocab % 16) return fail(TL_ERR_UNSUPPORTED, "vocab must be a positive multiple of 16");
  if (c->n_pre < 0 || c->n_pre > 64) return fail(TL_ERR_INVALID_ARG, "n_pre out of range");
  if (c->max_loops < 1 || c->max_loops > 256) return fail(TL_ERR_INVALID_ARG, "max_loops out of range");
  if (c->max_ctx < 1 || c->max_ctx > 8192) return fail(TL_ERR_INVALID_ARG, "max_ctx must be in [1, 8192]");
  if (c->max_lanes < 1 || c->max_lanes > kMaxLanes) return fail(TL_ERR_INVALID_ARG, "max_lanes must be in [1, 16]");
  if (!(c->rms_eps >= 0.f) || !(c->rope_theta > 0.f)) return fail(TL_ERR_INVALID_ARG, "bad eps or theta");
  if (c->kv_mode != TL_KV_FP16 && c->kv_mode != TL_KV_INT8) return fail(TL_ERR_INVALID_ARG, "kv_mode must be TL_KV_FP16 or TL_KV_INT8");
  if (c->weight_bits != 0 && c->weight_bits != 4 && c->weight_bits != 2)
    return fail(TL_ERR_INVALID_ARG, "weight_bits must be 4 (or 0) or 2");
  return TL_OK;
}

tl_status upload_block(const tl_config& c, const tl_block& hb, BlockDev* b, cudaStream_t st) {
  const int d = c.d_model, hd = c.head_dim;
  const int qkv_rows = (c.n_q_heads + 2 * c.n_kv_heads) * hd;
  tl_status rc;
  if ((rc = upload_f16(hb.attn_norm, d, &b->attn_norm, st)) != TL_OK) return rc;
  if ((rc = upload_f16(hb.ffn_norm, d, &b->ffn_norm, st)) != TL_OK) return rc;
  const int qdim = c.n_q_heads * hd;
  size_t total = 0;
  const int shapes[4][2] = {{d, qkv_rows}, {qdim, d}, {d, 2 * c.ffn_dim}, {c.ffn_dim, d}};
  const int bits = c.weight_bits == 2 ? 2 : 4;
  for (auto& sh : shapes) total += Int4Dev::w_bytes(sh[0], sh[1], bits) + Int4Dev::sz_bytes(sh[0], sh[1]) + 512;
  if (cudaMalloc(&b->arena.base, total) != cudaSuccess) return fail(TL_ERR_OOM, "block weights (%zu bytes)", total);
  b->arena.size = total;
  if ((rc = upload_int4(hb.qkv, d, qkv_rows, &b->qkv, st, &b->arena, 0, bits)) != TL_OK) return rc;
  if ((rc = upload_int4(hb.o, qdim, d, &b->o, st, &b->arena, 0, bits)) != TL_OK) return rc;
  if ((rc = upload_int4(hb.gate_up, d, 2 * c.ffn_dim, &b->gate_up, st, &b->arena, c.ffn_dim, bits)) != TL_OK) return rc;
  if ((rc = upload_int4(hb.down, c.ffn_dim, d, &b->down, st, &b->arena, 0, bits)) != TL_OK) return rc;
  return TL_OK;
}

// Launches of a loop-block layer carry the L2 window of the loop weights.
struct WindowScope {
  cudaAccessPolicyWindow prev;
  WindowScope(const tl_model* m, int layer) : prev(g_window) {
    if (layer >= m->cfg.n_pre) g_window = m->loop_window;
  }
  ~WindowScope() { g_window = prev; }
};

// Timeline entries of the next layer launch of a traced layered decode step
// (kTraceEvents per launch after the head-only launch's 4 slots), or NULL.
unsigned long long* next_trace(tl_model* m) {
  if (!m->trace || m->trace_i < 0) return nullptr;
  const long long base = 4LL * m->fused_grid + (long long)kTraceEvents * m->trace_i++;
  return base + kTraceEvents <= m->trace_cap ? m->trace + base : nullptr;
}

// ---- one effective layer ------------------------------------------------------
// QKV projection of `M` rows of the residual stream x (RMSNorm fused), RoPE on
// q and k, k and v written to cache slice `layer` at each row's (lane, pos).
tl_status run_qkv(tl_model* m, int layer, int M, float* x, const RowCtx* rows, float* q, cudaStream_t st) {
  WindowScope window_scope(m, layer);
  const tl_config& c = m->cfg;
  const BlockDev& b = m->block(layer);
  const int hd = c.head_dim, qdim = c.n_q_heads * hd;
  GemvArgs a{};
  a.eps = c.rms_eps;
  a.theta = c.rope_theta;
  a.rows = rows;
  a.hd = hd;
  a.w = b.qkv.w; a.sz = b.qkv.sz; a.K = c.d_model; a.n_rows = b.qkv.N; a.bits = b.qkv.bits;
  a.x = x; a.ldx = c.d_model; a.gain = b.attn_norm;
  a.pair_mode = PAIR_ROPE; a.pair_off = hd / 32;
  a.q_out = q; a.ldq = qdim; a.n_q_rows = qdim; a.n_kv_rows = c.n_kv_heads * hd;
  a.k_plane = m->k_plane(layer); a.v_plane = m->v_plane(layer);
  a.kv_stage = m->kv_stage;   // INT8: quantised by run_kv8 after this launch
  a.lane_stride = m->lane_stride; a.ctx = c.max_ctx;
  a.rope_tab = m->rope_tab;
  a.err_flag = m->err_flag;
  a.trace = next_trace(m);
  a.l2_keep = layer >= c.n_pre;
  kclass(TL_KERNEL_QKV);
  TL_CUDA(launch_gemv_rows(a, M, IN_NORM, EPI_ROPE_KV, (c.n_q_heads + 2 * c.n_kv_heads) * hd / 32, st));
  return TL_OK;
}

// Single-query attention of M decode rows over their lanes' slice `layer`.
tl_status run_decode_attn(tl_model* m, int layer, int M, const RowCtx* rows, const float* q, float* o,
                          cudaStream_t st) {
  const tl_config& c = m->cfg;
  const int qdim = c.n_q_heads * c.head_dim;
  DecodeAttnArgs da{};
  da.qf = q; da.ldq = qdim;
  da.k = m->k_plane(layer); da.v = m->v_plane(layer);
  da.ks = m->ks_plane(layer); da.vs = m->vs_plane(layer);   // NULL for fp16
  da.lane_stride = m->lane_stride; da.ctx = c.max_ctx;
  da.rows = rows; da.Hkv = c.n_kv_heads;
  da.of = o; da.ldo = qdim;
  da.part = m->attn_part; da.ticket = m->attn_tickets();
  kclass(TL_KERNEL_ATTN_DECODE);
  TL_CUDA(launch_decode_attn(da, M, c.head_dim, c.n_q_heads / c.n_kv_heads, true, st));
  return TL_OK;
}

// QKV projection + RoPE + KV write + attention of M <= kQaMaxRows decode rows
// in one clustered kernel (see qkv_attn.cuh), when the shapes allow it.
// A model-level choice (shapes and device only, never the row count), so a
// lane's arithmetic does not depend on which lanes share the step.
bool qkv_attn_ok(const tl_model* m) {
  const tl_config& c = m->cfg;
  const int rep = c.n_q_heads / c.n_kv_heads;
  if (!m->use_qkv_attn || (c.head_dim != 64 && c.head_dim != 128) || c.d_model > 4 * 4 * kQaThreads) return false;
  if (qa_tiles_per_cta(rep, c.head_dim) > kQaMaxTiles || rep * c.head_dim > 4 * kQaThreads) return false;
  return qa_layout(c.d_model, kQaMaxRows, rep, c.head_dim).total <= (size_t)m->qa_smem_max;
}

// Rows are taken kQaMaxRows per launch; each row's result is independent of
// the others in its launch.
tl_status run_qkv_attn(tl_model* m, int layer, int M, const RowCtx* rows, cudaStream_t st) {
  WindowScope window_scope(m, layer);
  const tl_config& c = m->cfg;
  const BlockDev& b = m->block(layer);
  const int qdim = c.n_q_heads * c.head_dim;
  kclass(TL_KERNEL_QKV);
  for (int r0 = 0; r0 < M; r0 += kQaMaxRows) {
    QkvAttnArgs a{};
    a.w = b.qkv.w; a.sz = b.qkv.sz; a.K = c.d_model;
    a.x = m->x + (size_t)r0 * c.d_model; a.gain = b.attn_norm; a.eps = c.rms_eps;
    a.M = std::min(kQaMaxRows, M - r0); a.rows = rows + r0;
    a.hd = c.head_dim; a.rep = c.n_q_heads / c.n_kv_heads; a.Hkv = c.n_kv_heads;
    a.rope_tab = m->rope_tab; a.theta = c.rope_theta;
    a.k_plane = m->k_plane(layer); a.v_plane = m->v_plane(layer);
    a.lane_stride = m->lane_stride; a.ctx = c.max_ctx;
    a.o = m->o + (size_t)r0 * qdim; a.err_flag = m->err_flag;
    a.trace = next_trace(m);
    a.l2_keep = layer >= c.n_pre;
    const size_t smem = qa_layout(c.d_model, a.M, a.rep, c.head_dim).total;
    const dim3 grid(kQaCluster, c.n_kv_heads);
    if (m->kv_int8) {
      a.k_scale = m->ks_plane(layer);
      a.v_scale = m->vs_plane(layer);
    }
    auto kern = qa_kernel(c.head_dim, m->kv_int8, b.qkv.bits);
    TL_CUDA(launch_impl(false, dim3(kQaCluster, 1, 1), kern, grid, dim3(kQaThreads), smem, st, a));
  }
  return TL_OK;
}

// Bytes of every head tile prefetched into L2 during a decode step's last
// layer (the loop block runs from L2 then, and HBM is otherwise idle).
constexpr unsigned kHeadPfPiece = 24576;

// O projection + residual, RMSNorm + gate_up + SwiGLU, down + residual.
tl_status run_ffn(tl_model* m, int layer, int M, float* x, const float* o, float* h, cudaStream_t st) {
  WindowScope window_scope(m, layer);
  const tl_config& c = m->cfg;
  const BlockDev& b = m->block(layer);
  const int d = c.d_model, F = c.ffn_dim, qdim = c.n_q_heads * c.head_dim;
  GemvArgs a{};
  a.eps = c.rms_eps;
  a.w = b.o.w; a.sz = b.o.sz; a.K = qdim; a.n_rows = d; a.bits = b.o.bits;
  a.x = o; a.ldx = qdim;
  a.pair_mode = PAIR_NEIGHBOUR;
  a.resid = x; a.ldr = d;
  a.err_flag = m->err_flag;
  a.trace = next_trace(m);
  a.trigger = TRIGGER_AT_START;
  a.l2_keep = layer >= c.n_pre;
  if (layer == m->head_pf_layer) {
    // the start of every 16-row head tile into L2 while the last layer runs
    // from it: each warp of the head then begins its tile from L2
    const size_t tile_bytes = (size_t)16 * c.d_model * 2;
    a.pf = reinterpret_cast<const unsigned char*>(m->head_w);
    a.pf_count = c.vocab / 16;
    a.pf_stride = tile_bytes;
    a.pf_piece = (unsigned)std::min<size_t>(kHeadPfPiece, tile_bytes);
  }
  kclass(TL_KERNEL_O_PROJ);
  TL_CUDA(launch_gemv_rows(a, M, IN_F32, EPI_RESID, (b.o.N + 15) / 16, st));
  GemvArgs g{};
  g.eps = c.rms_eps;
  g.w = b.gate_up.w; g.sz = b.gate_up.sz; g.K = d; g.n_rows = 2 * F; g.bits = b.gate_up.bits;
  g.x = x; g.ldx = d; g.gain = b.ffn_norm;
  g.pair_mode = PAIR_OFFSET; g.pair_off = F / 16;
  g.yf = h; g.ldy = F;
  g.err_flag = m->err_flag;
  g.trace = next_trace(m);
  g.trigger = TRIGGER_AFTER_LOOP;
  g.l2_keep = layer >= c.n_pre;
  kclass(TL_KERNEL_GATE_UP);
  TL_CUDA(launch_gemv_rows(g, M, IN_NORM, EPI_SWIGLU, F / 16, st));
  GemvArgs dn{};
  dn.w = b.down.w; dn.sz = b.down.sz; dn.K = F; dn.n_rows = d; dn.bits = b.down.bits;
  dn.x = h; dn.ldx = F;
  dn.pair_mode = PAIR_NEIGHBOUR;
  dn.resid = x; dn.ldr = d;
  dn.err_flag = m->err_flag;
  dn.trace = next_trace(m);
  dn.trigger = TRIGGER_AT_START;
  dn.l2_keep = layer >= c.n_pre;
  kclass(TL_KERNEL_DOWN);
  TL_CUDA(launch_gemv_rows(dn, M, IN_F32W, EPI_RESID, (b.down.N + 15) / 16, st));
  return TL_OK;
}

// Prefill forms of run_qkv / run_ffn on the tensor cores (positions
// pos0..pos0+T-1 of one lane).
// RMSNorm hand-off: for layer > 0 the previous layer's down projection has
// already written this layer's B tiles (x * attn gains) and the per-token
// sums of squares, so the QKV GEMM scales each token by its norm factor in
// the epilogue instead of running a prep kernel; the O projection does the
// same for the FFN's norm.
tl_status run_qkv_tc(tl_model* m, int layer, int lane, int T, int pos0, cudaStream_t st) {
  WindowScope window_scope(m, layer);
  const tl_config& c = m->cfg;
  const BlockDev& b = m->block(layer);
  const int hd = c.head_dim, qdim = c.n_q_heads * hd;
  const bool handed = layer > 0;
  PrepArgs pa{};
  pa.x = m->x; pa.ldx = c.d_model; pa.gain = b.attn_norm; pa.eps = c.rms_eps;
  TcGemmArgs ta{};
  if (handed) {
    ta.ss_in = m->tc.ss_attn; ta.ss_parts = c.d_model / kTcRows; ta.ss_ld = m->tc.ss_ld;
    ta.ss_k = (float)c.d_model; ta.ss_eps = c.rms_eps;
  }
  ta.q_out = m->q; ta.ldq = qdim; ta.n_q_rows = qdim; ta.n_kv_rows = c.n_kv_heads * hd; ta.hd = hd;
  ta.k_plane = m->k_lane(layer, lane);
  ta.v_plane = m->v_lane(layer, lane);
  ta.kv_stage = m->kv_stage;   // INT8: quantised by run_kv8 after the GEMM
  ta.ctx = c.max_ctx; ta.pos0 = pos0; ta.theta = c.rope_theta; ta.rope_tab = m->rope_tab;
  kclass(TL_KERNEL_GEMM_TC);
  TL_CUDA(launch_tc_linear(b.qkv.tc, b.qkv.sz, c.d_model, b.qkv.N, b.qkv.n_tiles, handed ? PREP_NONE : PREP_NORM,
                           pa, ta, TC_ROPE_KV, T, m->tc, st));
  return TL_OK;
}

// INT8 KV cache: quantise the pass's staged keys and values (T tokens at
// positions pos0.. of `lane`) into the lane's slice `layer`.
tl_status run_kv8(tl_model* m, int layer, int lane, int T, int pos0, cudaStream_t st) {
  const tl_config& c = m->cfg;
  Kv8QuantArgs ka{};
  ka.x = m->kv_stage;
  ka.n = T * 2 * c.n_kv_heads;
  ka.k8 = reinterpret_cast<int8_t*>(m->k_lane(layer, lane));
  ka.v8 = reinterpret_cast<int8_t*>(m->v_lane(layer, lane));
  ka.ks = m->ks_lane(layer, lane);
  ka.vs = m->vs_lane(layer, lane);
  ka.Hkv = c.n_kv_heads; ka.ctx = c.max_ctx; ka.pos0 = pos0;
  const dim3 grid((ka.n + kKv8Warps - 1) / kKv8Warps);
  kclass(TL_KERNEL_SETUP);
  if (c.head_dim == 64) TL_CUDA(launch(kv8_quant_kernel<64>, grid, dim3(kKv8Warps * 32), 0, st, ka));
  else TL_CUDA(launch(kv8_quant_kernel<128>, grid, dim3(kKv8Warps * 32), 0, st, ka));
  return TL_OK;
}

// INT8 KV cache, decode: quantise the new keys and values of M decode rows
// (staged by the QKV GEMV) into each row's lane at its position, slice `layer`.
tl_status run_kv8_rows(tl_model* m, int layer, int M, const RowCtx* rows, cudaStream_t st) {
  const tl_config& c = m->cfg;
  Kv8QuantArgs ka{};
  ka.x = m->kv_stage;
  ka.n = M * 2 * c.n_kv_heads;
  ka.k8 = reinterpret_cast<int8_t*>(m->k_plane(layer));
  ka.v8 = reinterpret_cast<int8_t*>(m->v_plane(layer));
  ka.ks = m->ks_plane(layer);
  ka.vs = m->vs_plane(layer);
  ka.Hkv = c.n_kv_heads; ka.ctx = c.max_ctx;
  ka.rows = rows; ka.lane_stride = m->lane_stride;
  const dim3 grid((ka.n + kKv8Warps - 1) / kKv8Warps);
  kclass(TL_KERNEL_SETUP);
  if (c.head_dim == 64) TL_CUDA(launch(kv8_quant_kernel<64>, grid, dim3(kKv8Warps * 32), 0, st, ka));
  else TL_CUDA(launch(kv8_quant_kernel<128>, grid, dim3(kKv8Warps * 32), 0, st, ka));
  return TL_OK;
}

// O + residual, gate_up + SwiGLU, down + residual of `layer`; the down
// projection also hands the next layer's attention RMSNorm over when
// `next_layer` >= 0 (its gains).
tl_status run_ffn_tc(tl_model* m, int layer, int T, int next_layer, cudaStream_t st) {
  WindowScope window_scope(m, layer);
  const tl_config& c = m->cfg;
  const BlockDev& b = m->block(layer);
  const int d = c.d_model, F = c.ffn_dim, qdim = c.n_q_heads * c.head_dim;
  kclass(TL_KERNEL_GEMM_TC);
  {  // O projection + residual (the prefill attention wrote its B tiles);
     // hands the FFN RMSNorm over to gate_up
    PrepArgs pa{};
    TcGemmArgs ta{};
    ta.out_f32 = m->x; ta.ld_out = d;
    ta.bt_next = m->tc.bt3; ta.g_next = b.ffn_norm; ta.ss_out = m->tc.ss_ffn; ta.ss_ld = m->tc.ss_ld;
    TL_CUDA(launch_tc_linear(b.o.tc, b.o.sz, qdim, d, b.o.n_tiles, PREP_NONE, pa, ta, TC_RESID, T, m->tc, st));
  }
  {  // gate_up (B = x * ffn gains, each token scaled by its norm factor);
     // its epilogue writes silu(gate) * up as the down projection's B tiles
     // (the tensor-core rows interleave gate and up)
    PrepArgs pa{};
    TcGemmArgs ta{};
    ta.ss_in = m->tc.ss_ffn; ta.ss_parts = d / kTcRows; ta.ss_ld = m->tc.ss_ld;
    ta.ss_k = (float)d; ta.ss_eps = c.rms_eps;
    ta.perm_F = F; ta.bt_out = m->tc.bt2; ta.bt_out_groups = F / 128;
    TL_CUDA(launch_tc_linear(b.gate_up.tc, b.gate_up.sz, d, 2 * F, b.gate_up.n_tiles, PREP_NONE, pa, ta,
                             TC_SWIGLU_B, T, m->tc, st, m->tc.bt3));
  }
  {  // down + residual (+ the next layer's attention RMSNorm hand-off)
    PrepArgs pa{};
    TcGemmArgs ta{};
    ta.out_f32 = m->x; ta.ld_out = d;
    if (next_layer >= 0) {
      ta.bt_next = m->tc.bt; ta.g_next = m->block(next_layer).attn_norm; ta.ss_out = m->tc.ss_attn;
      ta.ss_ld = m->tc.ss_ld;
    }
    TL_CUDA(launch_tc_linear(b.down.tc, b.down.sz, F, d, b.down.n_tiles, PREP_NONE, pa, ta, TC_RESID, T, m->tc, st,
                             m->tc.bt2));
  }
  return TL_OK;
}

tl_status launch_head(tl_model* m, const float* x, int M, const int* out_row, float* logits,
                      int32_t* argmax, cudaStream_t st, const HeadIO* io = nullptr) {
  const tl_config& c = m->cfg;
  if (M <= kHdMaxRows) {
    // one CTA per SM; each warp streams whole head tiles with direct loads
    HeadArgs ha{};
    ha.io = io;
    ha.w = m->head_w; ha.V = c.vocab; ha.d = c.d_model;
    ha.x = x; ha.gain = m->out_norm; ha.eps = c.rms_eps; ha.M = M;
    ha.out_row = out_row; ha.logits = logits; ha.argmax = argmax;
    ha.part_val = m->head_val; ha.part_idx = m->head_idx; ha.ticket = m->head_ticket();
    ha.err_flag = m->err_flag;
    kclass(TL_KERNEL_HEAD);
    TL_CUDA(launch(head_direct_kernel, dim3(m->hd_grid), dim3(kHdThreads), head_direct_smem(c.d_model), st, ha,
                   m->trace, m->trace_cap));
    return TL_OK;
  }
  HeadArgs ha{};
  ha.io = io;
  ha.w = m->head_w; ha.V = c.vocab; ha.d = c.d_model;
  ha.x = x; ha.gain = m->out_norm; ha.eps = c.rms_eps; ha.M = M;
  ha.out_row = out_row; ha.logits = logits; ha.argmax = argmax;
  ha.part_val = m->head_val; ha.part_idx = m->head_idx; ha.ticket = m->head_ticket();
  ha.err_flag = m->err_flag;
  const int nt = M <= 8 ? 1 : 2;
  const size_t smem = head_smem_bytes(c.d_model, M);
  kclass(TL_KERNEL_HEAD);
  if (nt == 1) TL_CUDA(launch(head_argmax_kernel<1>, dim3(m->head_grid), dim3(kHeadThreads), smem, st, ha));
  else TL_CUDA(launch(head_argmax_kernel<2>, dim3(m->head_grid), dim3(kHeadThreads), smem, st, ha));
  return TL_OK;
}

// What a forward pass over a lane's tokens produces besides the KV cache.
struct FwdOut {
  float* logits = nullptr;       // last position [V] (or every position [T][V] with all_rows)
  int32_t* argmax = nullptr;     // last position [1] (or [T])
  bool all_rows = false;         // head on every position (T <= kMaxLanes)
  float* lens_logits = nullptr;  // logit lens: last position after each loop iteration [loops][V]
  int32_t* lens_argmax = nullptr;
};

// Forward of T tokens on one lane at positions pos0..pos0+T-1 through
// n_pre + loops effective layers, attending to the lane's cached keys
// 0..pos0+t (a whole prompt when pos0 = 0, an appended chunk otherwise).
tl_status forward_tokens(tl_model* m, int lane, const int32_t* d_tokens, int T, int loops, int pos0,
                         const FwdOut& out, cudaStream_t st) {
  const tl_config& c = m->cfg;
  const int d = c.d_model, qdim = c.n_q_heads * c.head_dim;
  const int n_layers = c.n_pre + loops;
  kclass(TL_KERNEL_SETUP);
  TL_CUDA(launch(fill_rows_kernel, dim3((T + 255) / 256), dim3(256), 0, st, m->rows, T, lane, pos0));
  kclass(TL_KERNEL_EMBED);
  TL_CUDA(launch(embed_kernel, dim3(T), dim3(256), 0, st, (const __half*)m->embed, d, c.vocab,
                 d_tokens, (const int*)nullptr, m->x, m->err_flag));
  const bool tc = T >= kTcMinTokens;
  for (int layer = 0; layer < n_layers; ++layer) {
    tl_status rc = tc ? run_qkv_tc(m, layer, lane, T, pos0, st) : run_qkv(m, layer, T, m->x, m->rows, m->q, st);
    if (rc == TL_OK && m->kv_int8) rc = run_kv8(m, layer, lane, T, pos0, st);
    if (rc != TL_OK) return rc;
    PrefillAttnArgs pa{};
    pa.qf = m->q; pa.q_bstride = 0; pa.ldq = qdim;
    pa.k = m->k_lane(layer, lane);
    pa.v = m->v_lane(layer, lane);
    pa.ks = m->ks_lane(layer, lane);
    pa.vs = m->vs_lane(layer, lane);
    pa.kv_bstride = 0; pa.ctx = c.max_ctx;
    pa.T = T; pa.pos0 = pos0; pa.Hkv = c.n_kv_heads;
    pa.of = m->o; pa.o_bstride = 0; pa.ldo = qdim;
    pa.err_flag = m->err_flag;
    if (tc) {   // straight into the O projection's B tiles
      pa.bt = m->tc.bt;
      pa.bt_groups = qdim / 128;
    }
    kclass(TL_KERNEL_ATTN_PREFILL);
    TL_CUDA(launch_prefill_attn(pa, 1, c.head_dim, c.n_q_heads / c.n_kv_heads, true, st));
    rc = tc ? run_ffn_tc(m, layer, T, layer + 1 < n_layers ? layer + 1 : -1, st)
            : run_ffn(m, layer, T, m->x, m->o, m->h, st);
    if (rc != TL_OK) return rc;
    if ((out.lens_logits || out.lens_argmax) && layer >= c.n_pre) {
      const int i = layer - c.n_pre;   // loop iteration i + 1 done
      rc = launch_head(m, m->x + (size_t)(T - 1) * d, 1, nullptr,
                       out.lens_logits ? out.lens_logits + (size_t)i * c.vocab : nullptr,
                       out.lens_argmax ? out.lens_argmax + i : nullptr, st);
      if (rc != TL_OK) return rc;
    }
  }
  if (out.logits || out.argmax) {
    if (out.all_rows) return launch_head(m, m->x, T, nullptr, out.logits, out.argmax, st);
    return launch_head(m, m->x + (size_t)(T - 1) * d, 1, nullptr, out.logits, out.argmax, st);
  }
  return TL_OK;
}

tl_status decode_impl(tl_model* m, int n_lanes, const int32_t* h_lane_ids, const int32_t* d_tokens,
                      const int32_t* h_loops, float* d_logits, int32_t* d_argmax, cudaStream_t st);

// Copy positions [0, n) of every KV slice of `layers` layers from one lane to
// another: runs of n * head_dim elements of `esz` bytes (fp16 or int8 codes)
// per (layer, K|V, kv head), 16 bytes per thread, one CTA row per run
// (grid.y), the positions of a run over grid.x; with an INT8 cache also the
// run's n scales (scales != NULL, their offsets are the codes' / hd).
__global__ void kv_copy_kernel(unsigned char* __restrict__ kv, int esz, float* __restrict__ scales,
                               long long lane_stride, long long layer_stride, long long plane, int Hkv, int ctx,
                               int hd, int src, int dst, int n) {
  pdl_trigger();
  pdl_wait();
  const int run = blockIdx.y;                  // (layer * 2 + kv) * Hkv + head
  const int head = run % Hkv, kvsel = (run / Hkv) & 1, layer = run / (2 * Hkv);
  const size_t off = (size_t)layer * layer_stride + (size_t)kvsel * plane + (size_t)head * ctx * hd;
  const uint4* s4 = reinterpret_cast<const uint4*>(kv + ((size_t)src * lane_stride + off) * esz);
  uint4* d4 = reinterpret_cast<uint4*>(kv + ((size_t)dst * lane_stride + off) * esz);
  const size_t n16 = (size_t)n * hd * esz / 16;
  const size_t i0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x, step = (size_t)gridDim.x * blockDim.x;
  for (size_t i = i0; i < n16; i += step) d4[i] = __ldcs(s4 + i);
  if (scales) {
    const float* ss = scales + ((size_t)src * lane_stride + off) / hd;
    float* ds = scales + ((size_t)dst * lane_stride + off) / hd;
    for (size_t i = i0; i < (size_t)n; i += step) ds[i] = __ldcs(ss + i);
  }
}

}  // namespace

extern "C" {

tl_status tl_model_create(const tl_config* cfg, const tl_weights* w, int device, tl_model** out) {
  if (!out) return fail(TL_ERR_INVALID_ARG, "null out");
  *out = nullptr;
  tl_status rc = validate_config(cfg);
  if (rc != TL_OK) return rc;
  if (!w || !w->embed || !w->out_norm || !w->head || !w->loop || (cfg->n_pre > 0 && !w->pre))
    return fail(TL_ERR_INVALID_ARG, "null weight pointer");
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev)
    return fail(TL_ERR_INVALID_ARG, "device %d not available", device);
  DeviceGuard guard(device);
  if (!guard.ok) return fail(TL_ERR_CUDA, "cannot select device %d", device);
  TL_CUDA(init_device_kernels(device));

  tl_model* m = new tl_model();
  m->cfg = *cfg;
  m->device = device;
  m->n_layers_max = cfg->n_pre + cfg->max_loops;
  const tl_config& c = m->cfg;
  const int d = c.d_model, hd = c.head_dim, qdim = c.n_q_heads * hd;
  auto bail = [&](tl_status s) {
    m->free_all();
    delete m;
    return s;
  };
  if (cudaStreamCreateWithFlags(&m->setup_stream, cudaStreamNonBlocking) != cudaSuccess ||
      cudaStreamCreateWithFlags(&m->cap_stream, cudaStreamNonBlocking) != cudaSuccess)
    return bail(fail(TL_ERR_CUDA, "stream create failed"));
  cudaStream_t st = m->setup_stream;

  m->pre.resize(c.n_pre);
  for (int i = 0; i < c.n_pre; ++i)
    if ((rc = upload_block(c, w->pre[i], &m->pre[i], st)) != TL_OK) return bail(rc);
  if ((rc = upload_block(c, *w->loop, &m->loop, st)) != TL_OK) return bail(rc);
  if ((rc = upload_f16(w->embed, (size_t)c.vocab * d, &m->embed, st)) != TL_OK) return bail(rc);
  if ((rc = upload_f16(w->out_norm, d, &m->out_norm, st)) != TL_OK) return bail(rc);
  {
    __half* raw = nullptr;
    if ((rc = upload_f16(w->head, (size_t)c.vocab * d, &raw, st)) != TL_OK) return bail(rc);
    const size_t n = (size_t)(c.vocab / 16) * (d / 16) * 32;
    if (cudaMalloc(&m->head_w, n * sizeof(uint4)) != cudaSuccess) {
      cudaFree(raw);
      return bail(fail(TL_ERR_OOM, "head allocation"));
    }
    repack_head_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>((const uint32_t*)raw, c.vocab, d, m->head_w);
    cudaError_t e = cudaStreamSynchronize(st);
    cudaFree(raw);
    if (e != cudaSuccess) return bail(cuda_fail(e, "head repack"));
  }
  {  // L2 residency of the loop block: persisting window over its arena
    int max_persist = 0, max_window = 0;
    cudaDeviceGetAttribute(&max_persist, cudaDevAttrMaxPersistingL2CacheSize, device);
    cudaDeviceGetAttribute(&max_window, cudaDevAttrMaxAccessPolicyWindowSize, device);
    const size_t want = m->loop.arena.used;
    if (max_persist > 0 && max_window > 0 && want > 0) {
      const size_t carve = std::min((size_t)max_persist, want);
      size_t cur = 0;
      cudaDeviceGetLimit(&cur, cudaLimitPersistingL2CacheSize);
      if (cur < carve) cudaDeviceSetLimit(cudaLimitPersistingL2CacheSize, carve);
      cudaDeviceGetLimit(&cur, cudaLimitPersistingL2CacheSize);
      const size_t win = std::min(want, (size_t)max_window);
      m->loop_window.base_ptr = m->loop.arena.base;
      m->loop_window.num_bytes = win;
      m->loop_window.hitRatio = std::min(1.0f, (float)cur / (float)win);
      m->loop_window.hitProp = cudaAccessPropertyPersisting;
      m->loop_window.missProp = cudaAccessPropertyStreaming;
      m->l2_persist_bytes = cur;
    }
    cudaGetLastError();
  }
  m->weight_bytes = m->loop.bytes(d) + (size_t)c.vocab * d * 4 + 2 * (size_t)d;
  for (auto& b : m->pre) m->weight_bytes += b.bytes(d);

  // KV cache (one extra private lane for tl_score_last)
  m->plane = (long long)c.n_kv_heads * c.max_ctx * hd;
  m->layer_stride = 2 * m->plane;
  m->lane_stride = (long long)m->n_layers_max * m->layer_stride;
  m->kv_int8 = c.kv_mode == TL_KV_INT8;
  if (m->kv_int8) {   // one byte per element, then one fp32 scale per vector
    const size_t codes = (size_t)(c.max_lanes + 1) * m->lane_stride;
    const size_t scales = codes / hd * 4;
    m->kv_bytes = codes + scales;
    if (cudaMalloc(&m->kv, codes) != cudaSuccess || cudaMalloc(&m->kvs, scales) != cudaSuccess)
      return bail(fail(TL_ERR_OOM, "KV cache (%zu bytes)", m->kv_bytes));
  } else {
    m->kv_bytes = (size_t)(c.max_lanes + 1) * m->lane_stride * 2;
    if (cudaMalloc(&m->kv, m->kv_bytes) != cudaSuccess) return bail(fail(TL_ERR_OOM, "KV cache (%zu bytes)", m->kv_bytes));
  }

  // workspaces
  const int rows = std::max(c.max_ctx, kMaxLanes);
  const int rep = c.n_q_heads / c.n_kv_heads;
  {
    int n_sm = 0;
    if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || n_sm < 1) n_sm = 148;
    // one CTA per SM, never more CTAs than head tiles
    m->head_grid = std::min(n_sm, c.vocab / 16);
    m->hd_grid = n_sm;
    m->fused_grid = n_sm;   // one CTA per SM; also the timeline's entries per slot
    m->tc.n_sm = n_sm;
  }
  size_t ws = 0;
  auto alloc = [&](void** p, size_t bytes) -> bool {
    ws += bytes;
    if (cudaMalloc(p, bytes) != cudaSuccess) return false;
    return cudaMemsetAsync(*p, 0, bytes, st) == cudaSuccess;
  };
  bool ok = alloc((void**)&m->x, (size_t)rows * d * 4) && alloc((void**)&m->q, (size_t)rows * qdim * 4) &&
            alloc((void**)&m->o, (size_t)rows * qdim * 4) && alloc((void**)&m->h, (size_t)rows * c.ffn_dim * 4) &&
            alloc((void**)&m->rows, (size_t)rows * sizeof(RowCtx)) &&
            alloc((void**)&m->tok_index, kMaxLanes * 4) && alloc((void**)&m->out_row, kMaxLanes * 4) &&
            alloc((void**)&m->attn_part, (size_t)kMaxLanes * c.n_kv_heads * kDecodeMaxSplits * rep * (hd + kPartPad) * 4) &&
            alloc((void**)&m->tickets, (size_t)(kMaxLanes * c.n_kv_heads + 1) * 4) &&
            alloc((void**)&m->head_val, (size_t)std::max(m->head_grid, m->hd_grid) * 16 * 4) &&
            alloc((void**)&m->head_idx, (size_t)std::max(m->head_grid, m->hd_grid) * 16 * 4) &&
            alloc((void**)&m->err_flag, 4) &&
            alloc((void**)&m->spec_tok, (2 * kMaxLanes + 2) * 4) &&
            alloc((void**)&m->io, sizeof(HeadIO)) &&
            (!m->kv_int8 || alloc((void**)&m->kv_stage, (size_t)rows * 2 * c.n_kv_heads * hd * 4));
  if (ok) {
    const int kmax = std::max(std::max(d, qdim), c.ffn_dim);
    m->tc.bt_bytes = tc_bt_bytes(rows, kmax, true);
    m->tc.partial_bytes = (size_t)160 * kTcRows * kTcTokens * 4;
    m->tc.err_flag = m->err_flag;
    m->tc.ss_ld = (rows + kTcTokens - 1) / kTcTokens * kTcTokens;
    const size_t ss_bytes = (size_t)(d / kTcRows) * m->tc.ss_ld * 4;
    ok = alloc((void**)&m->tc.bt, m->tc.bt_bytes) && alloc((void**)&m->tc.bt2, m->tc.bt_bytes) &&
         alloc((void**)&m->tc.bt3, m->tc.bt_bytes) && alloc((void**)&m->tc.ss_attn, ss_bytes) &&
         alloc((void**)&m->tc.ss_ffn, ss_bytes) &&
         alloc((void**)&m->tc.partial, m->tc.partial_bytes) &&
         alloc((void**)&m->tc.tickets, 4096 * sizeof(unsigned)) &&
         alloc((void**)&m->rope_tab, (size_t)c.max_ctx * (hd / 2) * sizeof(float2));
    if (ok) {
      const int n = c.max_ctx * (hd / 2);
      rope_table_kernel<<<(n + 255) / 256, 256, 0, st>>>(m->rope_tab, c.max_ctx, hd, c.rope_theta);
      ok = cudaGetLastError() == cudaSuccess;
    }
  }
  if (!ok) return bail(fail(TL_ERR_OOM, "workspace allocation"));
  {  // single-kernel decode step: shapes, device support, resources
    // attention partials share the layered path's buffer, which holds
    // kMaxLanes x Hkv x kDecodeMaxSplits x rep x (hd + kPartPad) floats
    static_assert(kFusedMaxSplits == kDecodeMaxSplits && 2 * kFusedMaxRows <= kMaxLanes,
                  "fused partials ([4 rows][..][hd + 4]) must fit the layered path's buffer");
    int coop = 0;
    cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, device);
    // (the single-kernel step keeps an fp16 cache and INT4 weights only)
    if (coop && !m->kv_int8 && c.weight_bits != 2 && (hd == 64 || hd == 128) && c.n_pre < kFusedMaxBlocks &&
        rep_ok(rep)) {
      FusedArgs& f = m->fused;
      for (int i = 0; i <= c.n_pre; ++i) {
        const BlockDev& b = i < c.n_pre ? m->pre[i] : m->loop;
        f.blk[i].lin[FP_QKV] = {b.qkv.w, b.qkv.sz};
        f.blk[i].lin[FP_O] = {b.o.w, b.o.sz};
        f.blk[i].lin[FP_GU] = {b.gate_up.w, b.gate_up.sz};
        f.blk[i].lin[FP_DOWN] = {b.down.w, b.down.sz};
        f.blk[i].attn_norm = b.attn_norm;
        f.blk[i].ffn_norm = b.ffn_norm;
      }
      f.n_pre = c.n_pre;
      f.d = d; f.qdim = qdim; f.F = c.ffn_dim; f.V = c.vocab; f.hd = hd; f.Hkv = c.n_kv_heads; f.rep = rep;
      f.eps = c.rms_eps; f.theta = c.rope_theta;
      f.embed = m->embed; f.out_norm = m->out_norm; f.head_w = m->head_w;
      f.kv = m->kv; f.plane = m->plane; f.layer_stride = m->layer_stride; f.lane_stride = m->lane_stride;
      f.ctx = c.max_ctx; f.rope_tab = m->rope_tab;
      f.x = m->x; f.q = m->q; f.o = m->o; f.h = m->h;
      f.attn_part = m->attn_part; f.attn_ticket = m->attn_tickets(); f.head_ticket = m->head_ticket();
      f.err_flag = m->err_flag;
      m->fused_grid = m->tc.n_sm;
      ok = alloc((void**)&m->fused_bar, 4 * sizeof(unsigned)) &&
           alloc((void**)&m->fused_val, (size_t)m->fused_grid * kFusedMaxRows * 4) &&
           alloc((void**)&m->fused_idx, (size_t)m->fused_grid * kFusedMaxRows * 4);
      if (!ok) return bail(fail(TL_ERR_OOM, "workspace allocation"));
      f.bar = m->fused_bar; f.head_val = m->fused_val; f.head_idx = m->fused_idx;
      void (*kern)(const FusedArgs) = hd == 64 ? decode_fused_kernel<64> : decode_fused_kernel<128>;
      cudaFuncAttributes fa{};
      int optin = 0, nb = 0;
      size_t smem = 0;
      FusedArgs probe = f;
      if (cudaFuncGetAttributes(&fa, kern) == cudaSuccess &&
          cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device) == cudaSuccess) {
        m->fused_smem_max = optin - (int)fa.sharedSizeBytes;
        if (fused_plan(m, kFusedMaxRows, &probe, &smem) &&
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, kFusedThreads, smem) == cudaSuccess)
          m->fused_ok = nb >= 1;
      }
    }
    cudaGetLastError();
  }
  {
    cudaFuncAttributes fa{};
    int optin = 0;
    auto qa_kern = qa_kernel(hd, m->kv_int8, m->loop.qkv.bits);
    if (cudaFuncGetAttributes(&fa, qa_kern) == cudaSuccess &&
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device) == cudaSuccess)
      m->qa_smem_max = optin - (int)fa.sharedSizeBytes;
    // the clustered kernel is used only if a cluster of its size fits the GPU
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(kQaCluster, c.n_kv_heads);
    lc.blockDim = dim3(kQaThreads);
    lc.dynamicSmemBytes = qa_layout(d, kQaMaxRows, rep, hd).total;
    cudaLaunchAttribute la[1];
    la[0].id = cudaLaunchAttributeClusterDimension;
    la[0].val.clusterDim.x = kQaCluster;
    la[0].val.clusterDim.y = 1;
    la[0].val.clusterDim.z = 1;
    lc.attrs = la;
    lc.numAttrs = 1;
    int n_clusters = 0;
    if (lc.dynamicSmemBytes > (size_t)m->qa_smem_max ||
        cudaOccupancyMaxActiveClusters(&n_clusters, qa_kern, &lc) !=
            cudaSuccess ||
        n_clusters < 1)
      m->use_qkv_attn = false;
    cudaGetLastError();
  }
  // The clustered kernel takes kQaMaxRows rows per launch; a model built for
  // more lanes decodes through the QKV GEMV + split-KV attention instead
  // (measured on the 400M model: 1.6x the clustered path's tokens/s at 16
  // lanes, 1.08x at 4, 0.82x at 1).  A model-level choice, so a lane's
  // arithmetic never depends on which lanes share a step.
  m->qa_select = c.max_lanes <= kQaMaxRows;
  m->ws_bytes = ws;
  if (cudaStreamSynchronize(st) != cudaSuccess) return bail(fail(TL_ERR_CUDA, "setup sync"));
  m->lane_len.assign(c.max_lanes + 1, 0);
  m->lane_loops.assign(c.max_lanes + 1, 0);
  *out = m;
  return TL_OK;
}

void tl_model_destroy(tl_model* m) {
  if (!m) return;
  DeviceGuard guard(m->device);
  cudaDeviceSynchronize();
  if (m->loop_window.num_bytes) cudaCtxResetPersistingL2Cache();
  m->free_all();
  delete m;
}

tl_status tl_prefill(tl_model* m, int lane, const int32_t* d_tokens, int n_tokens, int loops,
                     float* d_last_logits, int32_t* d_last_argmax, void* stream) {
  if (!m) return fail(TL_ERR_INVALID_ARG, "null model");
  const tl_config& c = m->cfg;
  if (lane < 0 || lane >= c.max_lanes) return fail(TL_ERR_INVALID_ARG, "lane %d out of range", lane);
  if (!d_tokens) return fail(TL_ERR_INVALID_ARG, "null tokens");
  if (n_tokens < 1 || n_tokens > c.max_ctx) return fail(TL_ERR_CONTEXT_FULL, "n_tokens %d not in [1, max_ctx]", n_tokens);
  if (loops < 1 || loops > c.max_loops) return fail(TL_ERR_INVALID_ARG, "loops %d not in [1, max_loops]", loops);
  DeviceGuard guard(m->device);
  if (!guard.ok) return fail(TL_ERR_CUDA, "cannot select device");
  ProfScope prof_scope(&m->prof);
  FwdOut out;
  out.logits = d_last_logits;
  out.argmax = d_last_argmax;
  tl_status rc = forward_tokens(m, lane, d_tokens, n_tokens, loops, 0, out, (cudaStream_t)stream);
  if (rc != TL_OK) {
    m->lane_len[lane] = 0;
    return rc;
  }
  m->lane_len[lane] = n_tokens;
  m->lane_loops[lane] = loops;
  return TL_OK;
}

tl_status tl_score_last(tl_model* m, const int32_t* d_tokens, int n_tokens, int loops, float* d_logits,
                        int32_t* d_argmax, void* stream) {
  if (!m) return fail(TL_ERR_INVALID_ARG, "null model");
  const tl_config& c = m->cfg;
  if (!d_tokens || !d_logits) return fail(TL_ERR_INVALID_ARG, "null tokens or logits");
  if (n_tokens < 1 || n_tokens > c.max_ctx) return fail(TL_ERR_CONTEXT_FULL, "n_tokens %d not in [1, max_ctx]", n_tokens);
  if (loops < 1 || loops > c.max_loops) return fail(TL_ERR_INVALID_ARG, "loops %d not in [1, max_loops]", loops);
  DeviceGuard guard(m->device);
  if (!guard.ok) return fail(TL_ERR_CUDA, "cannot select device");
  ProfScope prof_scope(&m->prof);
  FwdOut out;
  out.logits = d_logits;
  out.argmax = d_argmax;
  return forward_tokens(m, c.max_lanes, d_tokens, n_tokens, loops, 0, out, (cudaStream_t)stream);
}

tl_status tl_decode_step(tl_model* m, int n_lanes, const int32_t* h_lane_ids, const int32_t* d_tokens,
                         const int32_t* h_loops, float* d_logits, int32_t* d_argmax, void* stream) {
  if (!m) return fail(TL_ERR_INVALID_ARG, "null model");
  const tl_config& c = m->cfg;
  if (n_lanes < 1 || n_lanes > c.max_lanes) return fail(TL_ERR_INVALID_ARG, "n_lanes %d not in [1, max_lanes]", n_lanes);
  if (!h_lane_ids || !d_tokens || !h_loops) return fail(TL_ERR_INVALID_ARG, "null argument");
  for (int i = 0; i < n_lanes; ++i) {
    const int lane = h_lane_ids[i];
    if (lane < 0 || lane >= c.max_lanes) return fail(TL_ERR_INVALID_ARG, "lane %d out of range", lane);
    for (int j = 0; j < i; ++j)
      if (h_lane_ids[j] == lane) return fail(TL_ERR_INVALID_ARG, "lane %d listed twice", lane);
    if (m->lane_len[lane] == 0) return fail(TL_ERR_NOT_PREFILLED, "lane %d holds no prompt", lane);
    if (h_loops[i] != m->lane_loops[lane])
      return fail(TL_ERR_LOOPS_MISMATCH, "lane %d was prefilled with loops=%d, step asks %d", lane,
                  m->lane_loops[lane], h_loops[i]);
    if (m->lane_len[lane] >= c.max_ctx) return fail(TL_ERR_CONTEXT_FULL, "lane %d is full", lane);
  }
  DeviceGuard guard(m->device);
  if (!guard.ok) return fail(TL_ERR_CUDA, "cannot select device");
  ProfScope prof_scope(&m->prof);
  return decode_impl(m, n_lanes, h_lane_ids, d_tokens, h_loops, d_logits, d_argmax, (cudaStream_t)stream);
}

}  // extern "C"

namespace {

// One decode step of validated rows: lane h_lane_ids[i] feeds d_tokens[i] at
// its current length through n_pre + h_loops[i] layers (h_loops[i] may be
// below the lane's prefill loops: a draft step reads and writes only the
// first slices, which a longer pass computes identically); each lane's
// length grows by one.
tl_status decode_impl(tl_model* m, int n_lanes, const int32_t* h_lane_ids, const int32_t* d_tokens,
                      const int32_t* h_loops, float* d_logits, int32_t* d_argmax, cudaStream_t st) {
  const tl_config& c = m->cfg;
  std::vector<int> order(n_lanes);
  for (int i = 0; i < n_lanes; ++i) order[i] = i;
  // Rows sorted by loop count (descending): the rows still running at layer l
  // are then a prefix.
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return h_loops[a] > h_loops[b]; });
  StepDesc sd{};
  sd.n = n_lanes;
  for (int s = 0; s < n_lanes; ++s) {
    const int i = order[s];
    sd.lane[s] = h_lane_ids[i];
    sd.pos[s] = m->lane_len[h_lane_ids[i]];
    sd.tok_index[s] = i;
    sd.out_row[s] = i;
  }
  sd.tokens = d_tokens;
  sd.logits = d_logits;
  sd.argmax = d_argmax;
  // AUTO takes the layered path: on the 400M model at batch 1 its graph
  // replay currently measures faster than the single-kernel step.
  const bool fused = m->decode_path == TL_DECODE_FUSED;
  if (fused) {
    if (!m->fused_ok || n_lanes > kFusedMaxRows)
      return fail(TL_ERR_UNSUPPORTED, "single-kernel decode needs <= %d lanes and a supported model/device",
                  kFusedMaxRows);
    FusedArgs f = m->fused;
    f.M = n_lanes;
    for (int s = 0; s < n_lanes; ++s) {
      f.lane[s] = sd.lane[s];
      f.pos[s] = sd.pos[s];
      f.loops[s] = h_loops[order[s]];
      f.tok_index[s] = sd.tok_index[s];
      f.out_row[s] = sd.out_row[s];
    }
    f.tokens = d_tokens;
    f.logits = d_logits;
    f.argmax = d_argmax;
    f.trace = m->trace;
    f.trace_cap = m->trace_cap;
    size_t smem = 0;
    if (!fused_plan(m, n_lanes, &f, &smem)) return fail(TL_ERR_UNSUPPORTED, "single-kernel decode: no shared-memory plan");
    kclass(TL_KERNEL_DECODE_FUSED);
    if (c.head_dim == 64)
      TL_CUDA(launch_impl(true, dim3(1, 1, 1), decode_fused_kernel<64>, dim3(m->fused_grid), dim3(kFusedThreads), smem, st, f));
    else
      TL_CUDA(launch_impl(true, dim3(1, 1, 1), decode_fused_kernel<128>, dim3(m->fused_grid), dim3(kFusedThreads), smem, st, f));
    for (int i = 0; i < n_lanes; ++i) m->lane_len[h_lane_ids[i]] += 1;
    return TL_OK;
  }
  kclass(TL_KERNEL_EMBED);
  TL_CUDA(launch(step_embed_kernel, dim3(n_lanes), dim3(256), 0, st, sd, (const __half*)m->embed, c.d_model,
                 c.vocab, m->rows, m->out_row, m->io, m->x, m->err_flag));
  // rows still running at each effective layer
  const int max_layers = c.n_pre + h_loops[order[0]];
  std::vector<int> active(max_layers);
  for (int layer = 0; layer < max_layers; ++layer) {
    int M = 0;
    while (M < n_lanes && c.n_pre + h_loops[order[M]] > layer) ++M;
    active[layer] = M;
  }
  auto body = [&](cudaStream_t s) -> tl_status {
    m->trace_i = 0;   // layer launches of this step take timeline records 0, 1, ...
    m->head_pf_layer = max_layers - 1;
    struct TraceOff { tl_model* m; ~TraceOff() { m->trace_i = -1; m->head_pf_layer = -1; } } trace_off{m};
    for (int layer = 0; layer < max_layers; ++layer) {
      const int M = active[layer];
      tl_status rc = TL_OK;
      if (m->qa_select && qkv_attn_ok(m)) {
        rc = run_qkv_attn(m, layer, M, m->rows, s);
      } else {
        rc = run_qkv(m, layer, M, m->x, m->rows, m->q, s);
        if (rc == TL_OK && m->kv_int8) rc = run_kv8_rows(m, layer, M, m->rows, s);
        if (rc == TL_OK) rc = run_decode_attn(m, layer, M, m->rows, m->q, m->o, s);
      }
      if (rc == TL_OK) rc = run_ffn(m, layer, M, m->x, m->o, m->h, s);
      if (rc != TL_OK) return rc;
    }
    return launch_head(m, m->x, n_lanes, m->out_row, nullptr, nullptr, s, m->io);
  };
  if (m->prof.mask || !m->use_graphs) {  // profiling times every launch: run eagerly
    tl_status rc = body(st);
    if (rc != TL_OK) return rc;
  } else {
    std::string key = std::to_string(n_lanes);
    for (int a : active) key += "," + std::to_string(a);
    auto it = m->graphs.find(key);
    if (it == m->graphs.end()) {
      // capture the layers and the head once for this row pattern
      tl_model::Graph gr;
      const unsigned long long before = g_launches.load();
      Profiler* saved = g_prof;
      g_prof = nullptr;
      cudaError_t e = cudaStreamBeginCapture(m->cap_stream, cudaStreamCaptureModeThreadLocal);
      if (e != cudaSuccess) { g_prof = saved; return cuda_fail(e, "cudaStreamBeginCapture"); }
      tl_status rc = body(m->cap_stream);
      cudaGraph_t graph = nullptr;
      e = cudaStreamEndCapture(m->cap_stream, &graph);
      g_prof = saved;
      gr.kernels = (int)(g_launches.load() - before);
      g_launches.fetch_sub(gr.kernels);   // counted when the graph runs
      if (rc != TL_OK) { if (graph) cudaGraphDestroy(graph); return rc; }
      if (e != cudaSuccess) { if (graph) cudaGraphDestroy(graph); return cuda_fail(e, "cudaStreamEndCapture"); }
      e = cudaGraphInstantiate(&gr.exec, graph, 0);
      cudaGraphDestroy(graph);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGraphInstantiate");
      it = m->graphs.emplace(key, gr).first;
    }
    TL_CUDA(cudaGraphLaunch(it->second.exec, st));
    g_launches.fetch_add(it->second.kernels);
  }
  for (int i = 0; i < n_lanes; ++i) m->lane_len[h_lane_ids[i]] += 1;
  return TL_OK;
}

}  // namespace

extern "C" {

tl_status tl_extend(tl_model* m, int lane, const int32_t* d_tokens, int n_tokens, float* d_logits,
                    int32_t* d_argmax, void* stream) {
  if (!m) return fail(TL_ERR_INVALID_ARG, "null model");
  const tl_config& c = m->cfg;
  if (lane < 0 || lane >= c.max_lanes) return fail(TL_ERR_INVALID_ARG, "lane %d out of range", lane);
  if (!d_tokens) return fail(TL_ERR_INVALID_ARG, "null tokens");
  if (m->lane_len[lane] == 0) return fail(TL_ERR_NOT_PREFILLED, "lane %d holds no prompt", lane);
  if (n_tokens < 1) return fail(TL_ERR_INVALID_ARG, "n_tokens must be >= 1");
  if ((d_logits || d_argmax) && n_tokens > kMaxLanes)
    return fail(TL_ERR_UNSUPPORTED, "per-position logits need n_tokens <= %d", kMaxLanes);
  const int pos0 = m->lane_len[lane];
  if (n_tokens > c.max_ctx - pos0) return fail(TL_ERR_CONTEXT_FULL, "lane %d: %d + %d tokens exceed max_ctx", lane,
                                               pos0, n_tokens);
  DeviceGuard guard(m->device);
  if (!guard.ok) return fail(TL_ERR_CUDA, "cannot select device");
  ProfScope prof_scope(&m->prof);
  FwdOut out;
  out.logits = d_logits;
  out.argmax = d_argmax;
  out.all_rows = true;
  tl_status rc = forward_tokens(m, lane, d_tokens, n_tokens, m->lane_loops[lane], pos0, out, (cudaStream_t)stream);
  if (rc != TL_OK) return rc;
  m->lane_len[lane] = pos0 + n_tokens;
  return TL_OK;
}

tl_status tl_generate_speculative(tl_model* m, int lane, const int32_t* d_first_token, int max_tokens,
                                  int draft_loops, int draft_ahead, int32_t* d_out_tokens, tl_spec_stats* h_stats,
                                  void* stream) {
  if (!m) return fail(TL_ERR_INVALID_ARG, "null model");
  const tl_config& c = m->cfg;
  if (lane < 0 || lane >= c.max_lanes) return fail(TL_ERR_INVALID_ARG, "lane %d out of range", lane);
  if (!d_first_token || !d_out_tokens) return fail(TL_ERR_INVALID_ARG, "null argument");
  if (m->lane_len[lane] == 0) return fail(TL_ERR_NOT_PREFILLED, "lane %d holds no prompt", lane);
  const int verify_loops = m->lane_loops[lane];
  if (draft_loops < 1 || draft_loops > verify_loops)
    return fail(TL_ERR_INVALID_ARG, "draft_loops %d not in [1, the lane's loops %d]", draft_loops, verify_loops);
  if (draft_ahead < 1 || draft_ahead > kMaxLanes)
    return fail(TL_ERR_INVALID_ARG, "draft_ahead %d not in [1, %d]", draft_ahead, kMaxLanes);
  if (max_tokens < 1) return fail(TL_ERR_INVALID_ARG, "max_tokens must be >= 1");
  const int p_start = m->lane_len[lane];
  if (max_tokens > c.max_ctx - p_start)
    return fail(TL_ERR_CONTEXT_FULL, "lane %d: %d + %d tokens exceed max_ctx", lane, p_start, max_tokens);
  DeviceGuard guard(m->device);
  if (!guard.ok) return fail(TL_ERR_CUDA, "cannot select device");
  ProfScope prof_scope(&m->prof);
  cudaStream_t st = (cudaStream_t)stream;
  // Per round on the device: seq = [next input, draft 1 .. draft k] and the
  // verifier's greedy tokens ver[0 .. k-1] (ver[i] follows seq[0..i]).
  int32_t* seq = m->spec_tok;
  int32_t* ver = m->spec_tok + kMaxLanes + 1;
  TL_CUDA(cudaMemcpyAsync(seq, d_first_token, 4, cudaMemcpyDeviceToDevice, st));
  tl_spec_stats stats{};
  int produced = 0;
  std::vector<int32_t> h(2 * kMaxLanes + 2);
  while (produced < max_tokens) {
    const int p = m->lane_len[lane];
    const int k = std::min(draft_ahead, max_tokens - produced);
    // draft: k cached greedy steps with draft_loops (first slices only)
    const int32_t lane_id = lane, dl = draft_loops;
    for (int i = 0; i < k; ++i) {
      tl_status rc = decode_impl(m, 1, &lane_id, seq + i, &dl, nullptr, seq + i + 1, st);
      if (rc != TL_OK) return rc;
    }
    // verify: the k inputs seq[0..k-1] at positions p..p+k-1 with the
    // lane's loops, one greedy token per position
    FwdOut out;
    out.argmax = ver;
    out.all_rows = true;
    tl_status rc = forward_tokens(m, lane, seq, k, verify_loops, p, out, st);
    if (rc != TL_OK) return rc;
    TL_CUDA(cudaMemcpyAsync(h.data(), seq, (size_t)(2 * kMaxLanes + 2) * 4, cudaMemcpyDeviceToHost, st));
    TL_CUDA(cudaStreamSynchronize(st));
    // accept drafts while they equal the verifier's tokens; the verifier's
    // token at the first mismatch is emitted in place of the draft
    int acc = 0;
    while (acc < k && h[1 + acc] == h[kMaxLanes + 1 + acc]) ++acc;
    const int emit = std::min(acc + 1, k);
    TL_CUDA(cudaMemcpyAsync(d_out_tokens + produced, ver, (size_t)emit * 4, cudaMemcpyDeviceToDevice, st));
    TL_CUDA(cudaMemcpyAsync(seq, ver + emit - 1, 4, cudaMemcpyDeviceToDevice, st));
    produced += emit;
    m->lane_len[lane] = p + emit;   // roll back the rejected drafts' positions
    stats.rounds += 1;
    stats.drafted += k;
    stats.accepted += acc;
  }
  if (h_stats) *h_stats = stats;
  return TL_OK;
}

tl_status tl_score_logit_lens(tl_model* m, const int32_t* d_tokens, int n_tokens, int loops, float* d_logits,
                              int32_t* d_argmax, void* stream) {
  if (!m) return fail(TL_ERR_INVALID_ARG, "null model");
  const tl_config& c = m->cfg;
  if (!d_tokens || !d_logits) return fail(TL_ERR_INVALID_ARG, "null tokens or logits");
  if (n_tokens < 1 || n_tokens > c.max_ctx) return fail(TL_ERR_CONTEXT_FULL, "n_tokens %d not in [1, max_ctx]", n_tokens);
  if (loops < 1 || loops > c.max_loops) return fail(TL_ERR_INVALID_ARG, "loops %d not in [1, max_loops]", loops);
  DeviceGuard guard(m->device);
  if (!guard.ok) return fail(TL_ERR_CUDA, "cannot select device");
  ProfScope prof_scope(&m->prof);
  FwdOut out;
  out.lens_logits = d_logits;
  out.lens_argmax = d_argmax;
  return forward_tokens(m, c.max_lanes, d_tokens, n_tokens, loops, 0, out, (cudaStream_t)stream);
}

tl_status tl_score_early_exit(tl_model* m, const int32_t* d_tokens, int n_tokens, int max_loops, int stable_n,
                              float* d_logits, int32_t* d_argmax, int* h_loops_used, void* stream) {
  if (!m) return fail(TL_ERR_INVALID_ARG, "null model");
  const tl_config& c = m->cfg;
  if (!d_tokens || !d_logits || !h_loops_used) return fail(TL_ERR_INVALID_ARG, "null argument");
  if (n_tokens < 1 || n_tokens > c.max_ctx) return fail(TL_ERR_CONTEXT_FULL, "n_tokens %d not in [1, max_ctx]", n_tokens);
  if (max_loops < 1 || max_loops > c.max_loops) return fail(TL_ERR_INVALID_ARG, "max_loops %d not in [1, max_loops]", max_loops);
  if (stable_n < 1) return fail(TL_ERR_INVALID_ARG, "stable_n must be >= 1");
  DeviceGuard guard(m->device);
  if (!guard.ok) return fail(TL_ERR_CUDA, "cannot select device");
  ProfScope prof_scope(&m->prof);
  cudaStream_t st = (cudaStream_t)stream;
  const int lane = c.max_lanes;   // the private scratch lane, as tl_score_last
  const int d = c.d_model, qdim = c.n_q_heads * c.head_dim, T = n_tokens;
  const bool tc = T >= kTcMinTokens;
  kclass(TL_KERNEL_SETUP);
  TL_CUDA(launch(fill_rows_kernel, dim3((T + 255) / 256), dim3(256), 0, st, m->rows, T, lane, 0));
  kclass(TL_KERNEL_EMBED);
  TL_CUDA(launch(embed_kernel, dim3(T), dim3(256), 0, st, (const __half*)m->embed, d, c.vocab, d_tokens,
                 (const int*)nullptr, m->x, m->err_flag));
  int32_t* am = m->spec_tok;   // device argmax of the current iteration
  int prev = -1, run = 0;
  for (int layer = 0; layer < c.n_pre + max_loops; ++layer) {
    tl_status rc = tc ? run_qkv_tc(m, layer, lane, T, 0, st) : run_qkv(m, layer, T, m->x, m->rows, m->q, st);
    if (rc == TL_OK && m->kv_int8) rc = run_kv8(m, layer, lane, T, 0, st);
    if (rc != TL_OK) return rc;
    PrefillAttnArgs pa{};
    pa.qf = m->q; pa.q_bstride = 0; pa.ldq = qdim;
    pa.k = m->k_lane(layer, lane);
    pa.v = m->v_lane(layer, lane);
    pa.ks = m->ks_lane(layer, lane);
    pa.vs = m->vs_lane(layer, lane);
    pa.kv_bstride = 0; pa.ctx = c.max_ctx;
    pa.T = T; pa.pos0 = 0; pa.Hkv = c.n_kv_heads;
    pa.of = m->o; pa.o_bstride = 0; pa.ldo = qdim;
    pa.err_flag = m->err_flag;
    if (tc) {
      pa.bt = m->tc.bt;
      pa.bt_groups = qdim / 128;
    }
    kclass(TL_KERNEL_ATTN_PREFILL);
    TL_CUDA(launch_prefill_attn(pa, 1, c.head_dim, c.n_q_heads / c.n_kv_heads, true, st));
    rc = tc ? run_ffn_tc(m, layer, T, layer + 1 < c.n_pre + max_loops ? layer + 1 : -1, st)
            : run_ffn(m, layer, T, m->x, m->o, m->h, st);
    if (rc != TL_OK) return rc;
    if (layer < c.n_pre) continue;
    // output norm + head after this iteration; stop once the greedy token
    // has been the same for stable_n consecutive iterations
    rc = launch_head(m, m->x + (size_t)(T - 1) * d, 1, nullptr, d_logits, am, st);
    if (rc != TL_OK) return rc;
    int32_t tok = 0;
    TL_CUDA(cudaMemcpyAsync(&tok, am, 4, cudaMemcpyDeviceToHost, st));
    TL_CUDA(cudaStreamSynchronize(st));
    run = tok == prev ? run + 1 : 1;
    prev = tok;
    *h_loops_used = layer - c.n_pre + 1;
    if (run >= stable_n) break;
  }
  if (d_argmax) TL_CUDA(cudaMemcpyAsync(d_argmax, am, 4, cudaMemcpyDeviceToDevice, st));
  return TL_OK;
}

tl_status tl_lane_fork(tl_model* m, int src_lane, int dst_lane, int n_tokens, void* stream) {
  if (!m) return fail(TL_ERR_INVALID_ARG, "null model");
  const tl_config& c = m->cfg;
  if (src_lane < 0 || src_lane >= c.max_lanes || dst_lane < 0 || dst_lane >= c.max_lanes)
    return fail(TL_ERR_INVALID_ARG, "lane out of range");
  if (src_lane == dst_lane) return fail(TL_ERR_INVALID_ARG, "source and destination lanes are the same");
  if (m->lane_len[src_lane] == 0) return fail(TL_ERR_NOT_PREFILLED, "lane %d holds no prompt", src_lane);
  if (n_tokens < 1 || n_tokens > m->lane_len[src_lane])
    return fail(TL_ERR_INVALID_ARG, "n_tokens %d not in [1, length of lane %d = %d]", n_tokens, src_lane,
                m->lane_len[src_lane]);
  DeviceGuard guard(m->device);
  if (!guard.ok) return fail(TL_ERR_CUDA, "cannot select device");
  ProfScope prof_scope(&m->prof);
  const int layers = c.n_pre + m->lane_loops[src_lane];
  const int runs = layers * 2 * c.n_kv_heads;
  const int per_run16 = n_tokens * c.head_dim / 8;
  const int gx = std::max(1, std::min((per_run16 + 255) / 256, std::max(1, 4 * m->tc.n_sm / runs)));
  kclass(TL_KERNEL_SETUP);
  TL_CUDA(launch(kv_copy_kernel, dim3(gx, runs), dim3(256), 0, (cudaStream_t)stream,
                 reinterpret_cast<unsigned char*>(m->kv), m->kv_int8 ? 1 : 2, m->kvs, m->lane_stride,
                 m->layer_stride, m->plane, c.n_kv_heads, c.max_ctx, c.head_dim, src_lane, dst_lane, n_tokens));
  m->lane_len[dst_lane] = n_tokens;
  m->lane_loops[dst_lane] = m->lane_loops[src_lane];
  return TL_OK;
}

tl_status tl_lane_kv_export(const tl_model* m, int lane, int layer, int n_tokens, void* d_k, void* d_v,
                            float* d_k_scales, float* d_v_scales, void* stream) {
  if (!m) return fail(TL_ERR_INVALID_ARG, "null model");
  const tl_config& c = m->cfg;
  if (lane < 0 || lane >= c.max_lanes) return fail(TL_ERR_INVALID_ARG, "lane %d out of range", lane);
  if (m->lane_len[lane] == 0) return fail(TL_ERR_NOT_PREFILLED, "lane %d holds no prompt", lane);
  if (layer < 0 || layer >= c.n_pre + m->lane_loops[lane])
    return fail(TL_ERR_INVALID_ARG, "layer %d not in [0, %d)", layer, c.n_pre + m->lane_loops[lane]);
  if (n_tokens < 1 || n_tokens > m->lane_len[lane])
    return fail(TL_ERR_INVALID_ARG, "n_tokens %d not in [1, length of lane %d]", n_tokens, lane);
  if (!d_k || !d_v || (m->kv_int8 && (!d_k_scales || !d_v_scales))) return fail(TL_ERR_INVALID_ARG, "null argument");
  DeviceGuard guard(m->device);
  if (!guard.ok) return fail(TL_ERR_CUDA, "cannot select device");
  cudaStream_t st = (cudaStream_t)stream;
  const size_t esz = m->kv_int8 ? 1 : 2, hd = c.head_dim;
  for (int kv = 0; kv < 2; ++kv) {
    const void* src = kv ? m->v_lane(layer, lane) : m->k_lane(layer, lane);
    TL_CUDA(cudaMemcpy2DAsync(kv ? d_v : d_k, (size_t)n_tokens * hd * esz, src, (size_t)c.max_ctx * hd * esz,
                              (size_t)n_tokens * hd * esz, c.n_kv_heads, cudaMemcpyDeviceToDevice, st));
    if (m->kv_int8) {
      const float* ssrc = kv ? m->vs_lane(layer, lane) : m->ks_lane(layer, lane);
      TL_CUDA(cudaMemcpy2DAsync(kv ? d_v_scales : d_k_scales, (size_t)n_tokens * 4, ssrc, (size_t)c.max_ctx * 4,
                                (size_t)n_tokens * 4, c.n_kv_heads, cudaMemcpyDeviceToDevice, st));
    }
  }
  return TL_OK;
}

tl_status tl_model_profile_start(tl_model* m, unsigned class_mask) {
  if (!m) return fail(TL_ERR_INVALID_ARG, "null model");
  m->prof.mask = class_mask;
  m->prof.used = 0;
  return TL_OK;
}

tl_status tl_model_profile_stop(tl_model* m, int* h_launches, float* h_total_ms) {
  if (!m) return fail(TL_ERR_INVALID_ARG, "null model");
  DeviceGuard guard(m->device);
  for (int c = 0; c < TL_KERNEL_CLASSES; ++c) {
    if (h_launches) h_launches[c] = 0;
    if (h_total_ms) h_total_ms[c] = 0.f;
  }
  for (int i = 0; i < m->prof.used; ++i) {
    TL_CUDA(cudaEventSynchronize(m->prof.ev[2 * i + 1]));
    float ms = 0.f;
    TL_CUDA(cudaEventElapsedTime(&ms, m->prof.ev[2 * i], m->prof.ev[2 * i + 1]));
    const int c = m->prof.cls[i];
    if (c < 0 || c >= TL_KERNEL_CLASSES) continue;
    if (h_launches) h_launches[c] += 1;
    if (h_total_ms) h_total_ms[c] += ms;
  }
  m->prof.mask = 0;
  m->prof.used = 0;
  return TL_OK;
}

unsigned long long tl_kernel_launch_count(void) { return g_launches.load(); }

tl_status tl_model_set_graphs(tl_model* m, int enable) {
  if (!m) return fail(TL_ERR_INVALID_ARG, "null model");
  m->use_graphs = enable != 0;
  return TL_OK;
}

tl_status tl_model_set_clustered_decode(tl_model* m, int enable) {
  if (!m) return fail(TL_ERR_INVALID_ARG, "null model");
  if (enable && !qkv_attn_ok(m)) return fail(TL_ERR_UNSUPPORTED, "the clustered decode kernel does not fit this model/device");
  if (m->qa_select != (enable != 0)) {
    DeviceGuard guard(m->device);
    if (cudaDeviceSynchronize() != cudaSuccess) return fail(TL_ERR_CUDA, "device sync");
    for (auto& kv_ : m->graphs)
      if (kv_.second.exec) cudaGraphExecDestroy(kv_.second.exec);
    m->graphs.clear();   // captured with the other path
    m->qa_select = enable != 0;
  }
  return TL_OK;
}

tl_status tl_model_set_decode_path(tl_model* m, int path) {
  if (!m) return fail(TL_ERR_INVALID_ARG, "null model");
  if (path != TL_DECODE_AUTO && path != TL_DECODE_LAYERED && path != TL_DECODE_FUSED)
    return fail(TL_ERR_INVALID_ARG, "unknown decode path %d", path);
  if (path == TL_DECODE_FUSED && !m->fused_ok)
    return fail(TL_ERR_UNSUPPORTED, "single-kernel decode is not available for this model/device");
  m->decode_path = path;
  return TL_OK;
}

tl_status tl_model_set_trace(tl_model* m, unsigned long long* d_buf, long long n_entries) {
  if (!m) return fail(TL_ERR_INVALID_ARG, "null model");
  if (d_buf && n_entries < 1) return fail(TL_ERR_INVALID_ARG, "n_entries must be >= 1");
  m->trace = d_buf;
  m->trace_cap = d_buf ? n_entries : 0;
  return TL_OK;
}

int tl_model_trace_grid(const tl_model* m) { return m ? m->fused_grid : 0; }

tl_status tl_set_prefill_attention_tc_min(int min_queries) {
  if (min_queries < 1) return fail(TL_ERR_INVALID_ARG, "min_queries must be >= 1");
  g_at_min_tokens.store(min_queries, std::memory_order_relaxed);
  return TL_OK;
}

tl_status tl_model_set_wait_test(tl_model* m, int extra_arrivals) {
  if (!m) return fail(TL_ERR_INVALID_ARG, "null model");
  if (extra_arrivals < 0 || extra_arrivals > 1) return fail(TL_ERR_INVALID_ARG, "extra_arrivals must be 0 or 1");
  m->fused.bar_extra = (unsigned)extra_arrivals;
  return TL_OK;
}

tl_status tl_lane_length(const tl_model* m, int lane, int* h_length) {
  if (!m || !h_length) return fail(TL_ERR_INVALID_ARG, "null argument");
  if (lane < 0 || lane >= m->cfg.max_lanes) return fail(TL_ERR_INVALID_ARG, "lane %d out of range", lane);
  *h_length = m->lane_len[lane];
  return TL_OK;
}

tl_status tl_model_info(const tl_model* m, size_t* weight_bytes, size_t* kv_bytes, size_t* workspace_bytes) {
  if (!m) return fail(TL_ERR_INVALID_ARG, "null model");
  if (weight_bytes) *weight_bytes = m->weight_bytes;
  if (kv_bytes) *kv_bytes = m->kv_bytes;
  if (workspace_bytes) *workspace_bytes = m->ws_bytes;
  return TL_OK;
}

tl_status tl_check_device_error(tl_model* m, void* stream) {
  if (!m) return fail(TL_ERR_INVALID_ARG, "null model");
  DeviceGuard guard(m->device);
  TL_CUDA(cudaStreamSynchronize((cudaStream_t)stream));
  int flag = 0;
  TL_CUDA(cudaMemcpy(&flag, m->err_flag, 4, cudaMemcpyDeviceToHost));
  if (flag) {
    TL_CUDA(cudaMemset(m->err_flag, 0, 4));
    if (flag & kErrTimeout) return fail(TL_ERR_DEVICE_FLAG, "a kernel's bounded wait gave up (results invalid)");
    return fail(TL_ERR_DEVICE_FLAG, "a token id outside [0, vocab) was replaced by 0");
  }
  return TL_OK;
}

// ============================================================================
// op API
// ============================================================================
}  // extern "C"

struct tl_linear {
  int device = 0;
  Int4Dev w;
};

namespace {
// Library-owned per-device workspace of the op entry points: a grow-only
// scratch buffer (row descriptors, split-KV partials) and a fixed array of
// tickets that is zeroed once and that every kernel leaves zeroed.
constexpr int kOpTickets = 65536;
struct OpWorkspace {
  void* buf = nullptr;
  size_t bytes = 0;
  unsigned* tickets = nullptr;
};
std::mutex g_ws_mu;
std::map<int, OpWorkspace> g_ws;

// A zeroed per-device fault flag for the op entry points.
std::map<int, int*> g_op_err;
// Row descriptors of an op call, passed by value.
constexpr int kOpRowsPerSetup = 128;
struct OpRows {
  int n;
  RowCtx rows[kOpRowsPerSetup];
};
__global__ void op_rows_kernel(OpRows r, RowCtx* out) {
  pdl_trigger();
  pdl_wait();
  if ((int)threadIdx.x < r.n) out[threadIdx.x] = r.rows[threadIdx.x];
}

int* op_err_flag(int dev) {
  std::lock_guard<std::mutex> lk(g_ws_mu);
  int*& f = g_op_err[dev];
  if (!f) {
    if (cudaMalloc(&f, sizeof(int)) != cudaSuccess) { f = nullptr; return nullptr; }
    if (cudaMemset(f, 0, sizeof(int)) != cudaSuccess) return nullptr;
  }
  return f;
}

// Scratch of at least `bytes` (contents undefined) and the ticket array.
// Growing the scratch synchronises the device.
tl_status op_workspace(int dev, size_t bytes, void** out, unsigned** tickets) {
  std::lock_guard<std::mutex> lk(g_ws_mu);
  OpWorkspace& w = g_ws[dev];
  if (!w.tickets) {
    TL_CUDA(cudaMalloc(&w.tickets, kOpTickets * sizeof(unsigned)));
    TL_CUDA(cudaMemset(w.tickets, 0, kOpTickets * sizeof(unsigned)));
  }
  if (w.bytes < bytes) {
    if (w.buf) {
      cudaDeviceSynchronize();
      cudaFree(w.buf);
      w.buf = nullptr;
      w.bytes = 0;
    }
    const size_t nb = std::max(bytes, (size_t)1 << 20);
    TL_CUDA(cudaMalloc(&w.buf, nb));
    w.bytes = nb;
  }
  *out = w.buf;
  *tickets = w.tickets;
  return TL_OK;
}
}  // namespace

extern "C" {

static tl_status linear_create(const tl_int4_linear* w, int K, int N, int bits, int device, tl_linear** out) {
  if (!out || !w) return fail(TL_ERR_INVALID_ARG, "null argument");
  *out = nullptr;
  if (K < 128 || K % 128 || K > 12288) return fail(TL_ERR_UNSUPPORTED, "K must be a multiple of 128 in [128, 12288]");
  if (N < 1 || N > 65536) return fail(TL_ERR_INVALID_ARG, "N must be in [1, 65536]");
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev)
    return fail(TL_ERR_INVALID_ARG, "device %d not available", device);
  DeviceGuard guard(device);
  TL_CUDA(init_device_kernels(device));
  tl_linear* l = new tl_linear();
  l->device = device;
  cudaStream_t st;
  TL_CUDA(cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking));
  tl_status rc = upload_int4(*w, K, N, &l->w, st, nullptr, 0, bits);
  cudaStreamDestroy(st);
  if (rc != TL_OK) {
    delete l;
    return rc;
  }
  *out = l;
  return TL_OK;
}

tl_status tl_linear_create(const tl_int4_linear* w, int K, int N, int device, tl_linear** out) {
  return linear_create(w, K, N, 4, device, out);
}

tl_status tl_linear_create_int2(const tl_int4_linear* w, int K, int N, int device, tl_linear** out) {
  return linear_create(w, K, N, 2, device, out);
}

void tl_linear_destroy(tl_linear* l) {
  if (!l) return;
  DeviceGuard guard(l->device);
  cudaDeviceSynchronize();
  l->w.free_all();
  delete l;
}

tl_status tl_linear_forward(tl_linear* l, const uint16_t* d_x, int M, uint16_t* d_y, int path, void* stream) {
  if (!l || !d_x || !d_y) return fail(TL_ERR_INVALID_ARG, "null argument");
  if (M < 1) return fail(TL_ERR_INVALID_ARG, "M must be >= 1");
  if (path == TL_PATH_AUTO) path = M <= kMaxLanes ? TL_PATH_GEMV : TL_PATH_TC;
  if (path != TL_PATH_GEMV && path != TL_PATH_TC) return fail(TL_ERR_INVALID_ARG, "unknown path %d", path);
  DeviceGuard guard(l->device);
  if (!guard.ok) return fail(TL_ERR_CUDA, "cannot select device");
  const int K = l->w.K, N = l->w.N;
  if (path == TL_PATH_TC) {
    if ((N + kTcRows - 1) / kTcRows * ((M + kTcTokens - 1) / kTcTokens) > 4096)
      return fail(TL_ERR_UNSUPPORTED, "too many tiles for the tensor-core path");
    TcScratch sc;
    const size_t bt = tc_bt_bytes(M, K, false), part = (size_t)160 * kTcRows * kTcTokens * 4;
    void* ws = nullptr;
    unsigned* tick = nullptr;
    tl_status rc = op_workspace(l->device, bt + part + 256, &ws, &tick);
    if (rc != TL_OK) return rc;
    sc.bt = (uint8_t*)ws;
    sc.bt_bytes = bt;
    sc.partial = (float*)((char*)ws + ((bt + 255) / 256) * 256);
    sc.partial_bytes = part;
    sc.tickets = tick + kOpTickets / 2;    // the second half of the op tickets
    sc.err_flag = op_err_flag(l->device);
    if (!sc.err_flag) return fail(TL_ERR_OOM, "op error flag");
    int n_sm = 148;
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, l->device);
    sc.n_sm = n_sm;
    PrepArgs pa{};
    pa.xh = reinterpret_cast<const __half*>(d_x); pa.ldx = K;
    TcGemmArgs ta{};
    ta.out_f16 = reinterpret_cast<__half*>(d_y); ta.ld_out = N;
    TL_CUDA(launch_tc_linear(l->w.tc, l->w.sz, K, N, l->w.n_tiles, PREP_F16, pa, ta, TC_STORE, M, sc,
                             (cudaStream_t)stream));
    return TL_OK;
  }
  if (gemv_rows_per_launch(K, false, gemv_tpc(EPI_STORE)) < 1) return fail(TL_ERR_UNSUPPORTED, "K too large for the GEMV");
  GemvArgs a{};
  a.err_flag = op_err_flag(l->device);
  if (!a.err_flag) return fail(TL_ERR_OOM, "op error flag");
  a.w = l->w.w; a.sz = l->w.sz; a.K = K; a.n_rows = N; a.bits = l->w.bits;
  a.xh = reinterpret_cast<const __half*>(d_x); a.ldx = K;
  a.pair_mode = PAIR_NEIGHBOUR;
  a.y = reinterpret_cast<__half*>(d_y); a.ldy = N;
  TL_CUDA(launch_gemv_rows(a, M, IN_F16, EPI_STORE, (N + 15) / 16, (cudaStream_t)stream));
  return TL_OK;
}

tl_status tl_op_rmsnorm(const float* d_x, const uint16_t* d_g, int rows, int d, float eps, uint16_t* d_y,
                        void* stream) {
  if (!d_x || !d_g || !d_y) return fail(TL_ERR_INVALID_ARG, "null argument");
  if (rows < 1 || d < 4 || d % 4) return fail(TL_ERR_INVALID_ARG, "rows >= 1 and d a multiple of 4 required");
  TL_CUDA(launch(rmsnorm_kernel, dim3((rows + 7) / 8), dim3(256), 0, (cudaStream_t)stream, d_x,
                 reinterpret_cast<const __half*>(d_g), rows, d, eps, reinterpret_cast<__half*>(d_y)));
  return TL_OK;
}

tl_status tl_op_rope(uint16_t* d_x, int n_tokens, int n_heads, int head_dim, long long token_stride,
                     long long head_stride, const int32_t* d_positions, float theta, void* stream) {
  if (!d_x || !d_positions) return fail(TL_ERR_INVALID_ARG, "null argument");
  if (n_tokens < 1 || n_heads < 1 || head_dim < 2 || head_dim % 2 || head_dim > 256 || !(theta > 0.f))
    return fail(TL_ERR_INVALID_ARG, "bad RoPE shape");
  const long long n = (long long)n_tokens * n_heads * (head_dim / 2);
  TL_CUDA(launch(rope_inplace_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, (cudaStream_t)stream,
                 reinterpret_cast<__half*>(d_x), n_tokens, n_heads, head_dim, token_stride, head_stride,
                 d_positions, theta));
  return TL_OK;
}

tl_status tl_op_kv_quant_int8(const float* d_x, int n, int head_dim, int8_t* d_codes, float* d_scales,
                              void* stream) {
  if (!d_x || !d_codes || !d_scales || n < 0) return fail(TL_ERR_INVALID_ARG, "null argument or n < 0");
  if (head_dim != 64 && head_dim != 128) return fail(TL_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (n == 0) return TL_OK;
  Kv8QuantArgs ka{};
  ka.x = d_x; ka.n = n; ka.codes = d_codes; ka.scales = d_scales;
  const dim3 grid((unsigned)((n + kKv8Warps - 1) / kKv8Warps));
  if (head_dim == 64) TL_CUDA(launch(kv8_quant_kernel<64>, grid, dim3(kKv8Warps * 32), 0, (cudaStream_t)stream, ka));
  else TL_CUDA(launch(kv8_quant_kernel<128>, grid, dim3(kKv8Warps * 32), 0, (cudaStream_t)stream, ka));
  return TL_OK;
}

tl_status tl_op_gqa_decode(const uint16_t* d_q, const uint16_t* d_k, const uint16_t* d_v, long long batch_stride,
                           int ctx_stride, const int32_t* h_n_keys, int B, int n_q_heads, int n_kv_heads,
                           int head_dim, uint16_t* d_out, void* stream) {
  if (!d_q || !d_k || !d_v || !h_n_keys || !d_out) return fail(TL_ERR_INVALID_ARG, "null argument");
  if (B < 1 || n_kv_heads < 1 || n_q_heads % n_kv_heads || !rep_ok(n_q_heads / n_kv_heads) ||
      (head_dim != 64 && head_dim != 128))
    return fail(TL_ERR_UNSUPPORTED, "unsupported attention shape");
  if (ctx_stride < 1 || ctx_stride > 8192) return fail(TL_ERR_INVALID_ARG, "ctx_stride must be in [1, 8192]");
  std::vector<RowCtx> rows(B);
  for (int b = 0; b < B; ++b) {
    if (h_n_keys[b] < 1 || h_n_keys[b] > ctx_stride) return fail(TL_ERR_INVALID_ARG, "n_keys[%d] out of range", b);
    rows[b].lane = b;
    rows[b].pos = h_n_keys[b] - 1;
  }
  int dev = 0;
  TL_CUDA(cudaGetDevice(&dev));
  TL_CUDA(init_device_kernels(dev));
  const int rep = n_q_heads / n_kv_heads;
  const size_t rows_b = (size_t)B * sizeof(RowCtx);
  const size_t part_b = (size_t)B * n_kv_heads * kDecodeMaxSplits * rep * (head_dim + kPartPad) * 4;
  if ((long long)B * n_kv_heads > kOpTickets) return fail(TL_ERR_UNSUPPORTED, "B * n_kv_heads > %d", kOpTickets);
  void* ws = nullptr;
  unsigned* tick = nullptr;
  tl_status rc = op_workspace(dev, ((rows_b + 255) / 256) * 256 + part_b, &ws, &tick);
  if (rc != TL_OK) return rc;
  char* base = (char*)ws;
  RowCtx* d_rows = (RowCtx*)base;
  float* part = (float*)(base + ((rows_b + 255) / 256) * 256);
  cudaStream_t st = (cudaStream_t)stream;
  // the row descriptors travel as kernel arguments (no copy from host memory
  // that a captured graph would read again, after this call, at replay)
  for (int b0 = 0; b0 < B; b0 += kOpRowsPerSetup) {
    OpRows r{};
    r.n = std::min(kOpRowsPerSetup, B - b0);
    for (int i = 0; i < r.n; ++i) r.rows[i] = rows[b0 + i];
    kclass(TL_KERNEL_SETUP);
    TL_CUDA(launch(op_rows_kernel, dim3(1), dim3(kOpRowsPerSetup), 0, st, r, d_rows + b0));
  }
  DecodeAttnArgs a{};
  a.qh = reinterpret_cast<const __half*>(d_q);
  a.ldq = n_q_heads * head_dim;
  a.k = reinterpret_cast<const __half*>(d_k);
  a.v = reinterpret_cast<const __half*>(d_v);
  a.lane_stride = batch_stride;
  a.ctx = ctx_stride;
  a.rows = d_rows;
  a.Hkv = n_kv_heads;
  a.oh = reinterpret_cast<__half*>(d_out);
  a.ldo = n_q_heads * head_dim;
  a.part = part;
  a.ticket = tick;
  TL_CUDA(launch_decode_attn(a, B, head_dim, rep, false, st));
  return TL_OK;
}

tl_status tl_op_gqa_prefill(const uint16_t* d_q, const uint16_t* d_k, const uint16_t* d_v, long long batch_stride,
                            int ctx_stride, int T, int pos0, int B, int n_q_heads, int n_kv_heads, int head_dim,
                            uint16_t* d_out, void* stream) {
  if (!d_q || !d_k || !d_v || !d_out) return fail(TL_ERR_INVALID_ARG, "null argument");
  if (B < 1 || T < 1 || pos0 < 0 || n_kv_heads < 1 || n_q_heads % n_kv_heads || !rep_ok(n_q_heads / n_kv_heads) ||
      (head_dim != 64 && head_dim != 128))
    return fail(TL_ERR_UNSUPPORTED, "unsupported attention shape");
  if (pos0 + T > ctx_stride) return fail(TL_ERR_INVALID_ARG, "pos0 + T exceeds ctx_stride");
  int dev = 0;
  TL_CUDA(cudaGetDevice(&dev));
  TL_CUDA(init_device_kernels(dev));
  const int qdim = n_q_heads * head_dim;
  PrefillAttnArgs a{};
  a.qh = reinterpret_cast<const __half*>(d_q);
  a.q_bstride = (long long)T * qdim;
  a.ldq = qdim;
  a.k = reinterpret_cast<const __half*>(d_k);
  a.v = reinterpret_cast<const __half*>(d_v);
  a.kv_bstride = batch_stride;
  a.ctx = ctx_stride;
  a.T = T;
  a.pos0 = pos0;
  a.Hkv = n_kv_heads;
  a.oh = reinterpret_cast<__half*>(d_out);
  a.o_bstride = (long long)T * qdim;
  a.ldo = qdim;
  a.err_flag = op_err_flag(dev);
  TL_CUDA(launch_prefill_attn(a, B, head_dim, n_q_heads / n_kv_heads, false, (cudaStream_t)stream));
  return TL_OK;
}

const char* tl_status_string(tl_status s) {
  switch (s) {
    case TL_OK: return "TL_OK";
    case TL_ERR_INVALID_ARG: return "TL_ERR_INVALID_ARG";
    case TL_ERR_OOM: return "TL_ERR_OOM";
    case TL_ERR_CUDA: return "TL_ERR_CUDA";
    case TL_ERR_CONTEXT_FULL: return "TL_ERR_CONTEXT_FULL";
    case TL_ERR_LOOPS_MISMATCH: return "TL_ERR_LOOPS_MISMATCH";
    case TL_ERR_NOT_PREFILLED: return "TL_ERR_NOT_PREFILLED";
    case TL_ERR_DEVICE_FLAG: return "TL_ERR_DEVICE_FLAG";
    case TL_ERR_UNSUPPORTED: return "TL_ERR_UNSUPPORTED";
  }
  return "TL_ERR_UNKNOWN";
}

const char* tl_last_error(void) { return g_err.c_str(); }

}  // extern "C"

// Sets the calling thread's last-error text for other translation units of
// the library (not exported).
__attribute__((visibility("hidden"))) tl_status tl_internal_set_error(tl_status s, const char* msg) {
  g_err = msg;
  return s;
}

namespace {
// Read-bandwidth probe: `passes` sweeps over the buffer inside one launch, 8
// independent 16-byte loads in flight per thread.  The loads are volatile
// (ld.global.cg: L2, not L1), so no pass can be folded into another.
__device__ __forceinline__ uint4 probe_ld(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__global__ void __launch_bounds__(512) read_probe_kernel(const uint4* __restrict__ p, size_t n16, int passes,
                                                         unsigned* __restrict__ sink) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  const size_t i0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  unsigned acc = 0;
  for (int pass = 0; pass < passes; ++pass) {
    size_t i = i0;
    for (; i + 7 * stride < n16; i += 8 * stride) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = probe_ld(p + i + u * stride);
#pragma unroll
      for (int u = 0; u < 8; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
    }
    for (; i < n16; i += stride) {
      const uint4 a = probe_ld(p + i);
      acc ^= a.x ^ a.y ^ a.z ^ a.w;
    }
  }
  if (acc == 0x9E3779B9u) *sink = acc;  // keeps the loads; practically never taken
}
}  // namespace

extern "C" {

const char* tl_version(void) { return "0.2.0"; }

tl_status tl_probe_read_bandwidth(const void* d_buf, size_t bytes, int reps, void* stream, double* h_gbs) {
  if (!d_buf || !h_gbs) return fail(TL_ERR_INVALID_ARG, "null argument");
  if (bytes < 16 || bytes % 16 || ((uintptr_t)d_buf & 15))
    return fail(TL_ERR_INVALID_ARG, "bytes must be a positive multiple of 16 on a 16-byte boundary");
  if (reps < 1 || reps > 100000) return fail(TL_ERR_INVALID_ARG, "reps must be in [1, 100000]");
  cudaPointerAttributes pa{};
  if (cudaPointerGetAttributes(&pa, d_buf) != cudaSuccess || pa.type != cudaMemoryTypeDevice) {
    cudaGetLastError();
    return fail(TL_ERR_INVALID_ARG, "d_buf is not device memory");
  }
  DeviceGuard guard(pa.device);
  if (!guard.ok) return fail(TL_ERR_CUDA, "cannot select device");
  int n_sm = 0;
  TL_CUDA(cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, pa.device));
  cudaStream_t st = (cudaStream_t)stream;
  unsigned* sink = nullptr;
  TL_CUDA(cudaMalloc(&sink, sizeof(unsigned)));
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  cudaError_t e = cudaEventCreate(&e0);
  if (e == cudaSuccess) e = cudaEventCreate(&e1);
  const dim3 grid(n_sm * 4), block(512);
  const uint4* p = (const uint4*)d_buf;
  const size_t n16 = bytes / 16;
  // warm: 3 untimed passes (brings an L2-sized buffer into L2)
  if (e == cudaSuccess) {
    read_probe_kernel<<<grid, block, 0, st>>>(p, n16, 3, sink);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaEventRecord(e0, st);
  if (e == cudaSuccess) {
    read_probe_kernel<<<grid, block, 0, st>>>(p, n16, reps, sink);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaEventRecord(e1, st);
  if (e == cudaSuccess) e = cudaEventSynchronize(e1);
  float ms = 0.f;
  if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, e0, e1);
  if (e0) cudaEventDestroy(e0);
  if (e1) cudaEventDestroy(e1);
  cudaFree(sink);
  if (e != cudaSuccess) return cuda_fail(e, "read probe");
  *h_gbs = (double)bytes * reps / ((double)ms * 1e6);
  return TL_OK;
}

}  // extern "C"
