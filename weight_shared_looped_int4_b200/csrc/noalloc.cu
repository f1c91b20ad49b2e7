// tl_op_gqa_decode_noalloc: the split-KV decode attention with its scratch in
// a fixed block of device memory that the library owns from load time, so the
// call itself allocates nothing.
//
// Who needs it: callers that must not call cudaMalloc from inside their own
// code, e.g. a host that pre-plans every device byte before serving starts,
// or a plug-in running inside another runtime whose allocator owns the
// device memory and must not be bypassed.  tl_op_gqa_decode allocates (and
// may grow) its workspace on first use; this variant never does.
//
// The scratch is the file-scope array below.  Every GPU that loads this
// library reserves it for the life of the process.  In host code the name
// g_noalloc_scratch is only a stand-in for the device array, not a device
// address: the device address is looked up once per device with
// cudaGetSymbolAddress (with that device current) and cached for the life of
// the process.  The cache is not refreshed if the device's context is torn
// down (cudaDeviceReset): a call after that would use a stale address.
#include <mutex>
#include <string>

#include "../../include/tl.h"
#include "attention.cuh"
#include "internal.h"

using namespace tl;

namespace {

// Scratch layout: [tickets][row descriptors][split-KV partial results].
constexpr size_t kNoAllocScratchBytes = 4u << 20;   // 4 MiB per device
constexpr int kNoAllocMaxRows = 32;                  // B limit per call
constexpr int kNoAllocTickets = 4096;                // B * n_kv_heads limit
constexpr size_t kTicketBytes = kNoAllocTickets * sizeof(unsigned);
constexpr size_t kRowsBytes = 1024;                  // >= kNoAllocMaxRows * sizeof(RowCtx)
constexpr size_t kPartOffset = kTicketBytes + kRowsBytes;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

struct NoAllocRows {
  int n;
  int n_kv_heads;
  RowCtx rows[kNoAllocMaxRows];
};

// Writes this call's row descriptors into the scratch and zeroes the tickets
// the attention kernel will count on (the array keeps the previous call's
// contents, so nothing may be assumed zero).
__global__ void noalloc_setup_kernel(NoAllocRows r, unsigned char* scratch) {
  unsigned* tickets = reinterpret_cast<unsigned*>(scratch);
  RowCtx* rows = reinterpret_cast<RowCtx*>(scratch + kTicketBytes);
  const int n_tick = r.n * r.n_kv_heads;
  for (int i = threadIdx.x; i < n_tick; i += blockDim.x) tickets[i] = 0u;
  for (int i = threadIdx.x; i < r.n; i += blockDim.x) rows[i] = r.rows[i];
}

tl_status err(tl_status s, const std::string& m) { return tl_internal_set_error(s, m.c_str()); }

// Allow the attention kernels their dynamic shared memory (once per device,
// with the scratch address lookup).
cudaError_t allow_attn_smem() {
  cudaError_t e = cudaSuccess;
#define A(HD, REP)                                                                               \
  if (e == cudaSuccess)                                                                          \
    e = cudaFuncSetAttribute(decode_attn_kernel<HD, REP, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             (int)decode_attn_smem_bytes(HD, REP));
  A(64, 1) A(64, 2) A(64, 4) A(64, 8) A(128, 1) A(128, 2) A(128, 4) A(128, 8)
#undef A
  return e;
}

// Device address of the scratch on the current device (looked up once).
tl_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return err(TL_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return err(TL_ERR_UNSUPPORTED, "device index beyond 63");
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return err(TL_ERR_CUDA, std::string("cudaGetSymbolAddress(scratch): ") + cudaGetErrorString(e));
    e = allow_attn_smem();
    if (e != cudaSuccess) return err(TL_ERR_CUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return TL_OK;
}

template <int HD, int REP>
cudaError_t launch_attn(const DecodeAttnArgs& a, int rows, cudaStream_t st) {
  decode_attn_kernel<HD, REP, false><<<dim3(kDecodeMaxSplits, a.Hkv, rows), kDecodeThreads, decode_attn_smem_bytes(HD, REP), st>>>(a);
  return cudaGetLastError();
}

}  // namespace

extern "C" tl_status tl_op_gqa_decode_noalloc(const uint16_t* d_q, const uint16_t* d_k, const uint16_t* d_v,
                                              long long batch_stride, int ctx_stride, const int32_t* h_n_keys,
                                              int B, int n_q_heads, int n_kv_heads, int head_dim,
                                              uint16_t* d_out, void* stream) {
  if (!d_q || !d_k || !d_v || !h_n_keys || !d_out) return err(TL_ERR_INVALID_ARG, "null argument");
  if (n_kv_heads < 1 || n_q_heads % n_kv_heads || (head_dim != 64 && head_dim != 128))
    return err(TL_ERR_UNSUPPORTED, "unsupported attention shape");
  const int rep = n_q_heads / n_kv_heads;
  if (rep != 1 && rep != 2 && rep != 4 && rep != 8) return err(TL_ERR_UNSUPPORTED, "n_q_heads/n_kv_heads must be 1, 2, 4 or 8");
  if (ctx_stride < 1 || ctx_stride > 8192) return err(TL_ERR_INVALID_ARG, "ctx_stride must be in [1, 8192]");
  if (B < 1 || B > kNoAllocMaxRows)
    return err(TL_ERR_UNSUPPORTED, "B must be in [1, 32] for the no-allocation variant");
  if ((long long)B * n_kv_heads > kNoAllocTickets) return err(TL_ERR_UNSUPPORTED, "B * n_kv_heads exceeds 4096");
  const size_t part_bytes = (size_t)B * n_kv_heads * kDecodeMaxSplits * rep * (head_dim + kPartPad) * sizeof(float);
  if (kPartOffset + part_bytes > kNoAllocScratchBytes)
    return err(TL_ERR_UNSUPPORTED,
               "shape needs " + std::to_string(kPartOffset + part_bytes) +
                   " bytes of scratch; the no-allocation variant has 4 MiB (use tl_op_gqa_decode)");
  NoAllocRows r{};
  r.n = B;
  r.n_kv_heads = n_kv_heads;
  for (int b = 0; b < B; ++b) {
    if (h_n_keys[b] < 1 || h_n_keys[b] > ctx_stride) return err(TL_ERR_INVALID_ARG, "n_keys out of range");
    r.rows[b].lane = b;
    r.rows[b].pos = h_n_keys[b] - 1;
  }
  void* base = nullptr;
  tl_status rc = scratch_address(&base);
  if (rc != TL_OK) return rc;
  unsigned char* scratch = static_cast<unsigned char*>(base);
  cudaStream_t st = (cudaStream_t)stream;
  noalloc_setup_kernel<<<1, 256, 0, st>>>(r, scratch);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return err(TL_ERR_CUDA, std::string("setup launch: ") + cudaGetErrorString(e));

  DecodeAttnArgs a{};
  a.qh = reinterpret_cast<const __half*>(d_q);
  a.ldq = n_q_heads * head_dim;
  a.k = reinterpret_cast<const __half*>(d_k);
  a.v = reinterpret_cast<const __half*>(d_v);
  a.lane_stride = batch_stride;
  a.ctx = ctx_stride;
  a.rows = reinterpret_cast<const RowCtx*>(scratch + kTicketBytes);
  a.Hkv = n_kv_heads;
  a.oh = reinterpret_cast<__half*>(d_out);
  a.ldo = n_q_heads * head_dim;
  a.part = reinterpret_cast<float*>(scratch + kPartOffset);
  a.ticket = reinterpret_cast<unsigned*>(scratch);
  e = cudaErrorInvalidValue;
#define C(HD, REP) \
  if (head_dim == HD && rep == REP) e = launch_attn<HD, REP>(a, B, st);
  C(64, 1) C(64, 2) C(64, 4) C(64, 8) C(128, 1) C(128, 2) C(128, 4) C(128, 8)
#undef C
  if (e != cudaSuccess) return err(TL_ERR_CUDA, std::string("attention launch: ") + cudaGetErrorString(e));
  return TL_OK;
}
