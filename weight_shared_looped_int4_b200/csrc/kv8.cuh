// INT8 KV cache storage: one fp32 scale per stored key or value vector (one
// position, one kv head, HD elements), scale = max|x| / 127 and code =
// round-half-even(x / scale), both decisions in fp32; an all-zero vector has
// scale 0 and codes 0; the cache holds code * scale.  (TinyLoop README,
// "Python API reference", KV cache modes: INT8 KV; the format is this
// library's reading, the pages give none.)
//
// Layout: the int8 planes mirror the fp16 ones element for element
// ([lanes][layers][K|V][Hkv][ctx][hd] at one byte per element); the scales
// mirror them with the head dimension collapsed, so the scale of the vector
// whose codes start at element offset e is at offset e / hd.
#pragma once

#include "common.cuh"

namespace tl {

// Quantise one vector held by a warp, E consecutive elements per lane: the
// warp's max |x| gives the scale; q receives the codes.  Every lane returns
// the scale.
template <int E>
__device__ __forceinline__ float kv8_quant_warp(const float (&x)[E], int (&q)[E]) {
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < E; ++i) m = fmaxf(m, fabsf(x[i]));
  m = warp_max(m);
  const float scale = m / 127.0f;   // IEEE division: the same fp32 value as the oracle's
#pragma unroll
  for (int i = 0; i < E; ++i) {
    int c = 0;
    if (scale > 0.f) c = __float2int_rn(x[i] / scale);   // ties to even
    q[i] = max(-127, min(127, c));
  }
  return scale;
}

// Four codes (one 32-bit word, lowest byte first) as two fp16 pairs, exact:
// the biased byte code + 128 goes into the mantissa of 1024 (fp16 0x6400)
// and 1152 = 1024 + 128 is subtracted.
__device__ __forceinline__ void kv8_codes_h2(uint32_t w, __half2& c01, __half2& c23) {
  const uint32_t u = w ^ 0x80808080u;                       // code + 128, per byte
  const uint32_t lo = __byte_perm(u, 0x64646464u, 0x4140);  // (1024 + u0, 1024 + u1)
  const uint32_t hi = __byte_perm(u, 0x64646464u, 0x4342);  // (1024 + u2, 1024 + u3)
  const __half2 bias = __halves2half2(__ushort_as_half((unsigned short)0x6480), __ushort_as_half((unsigned short)0x6480));
  c01 = __hsub2(*reinterpret_cast<const __half2*>(&lo), bias);
  c23 = __hsub2(*reinterpret_cast<const __half2*>(&hi), bias);
}
struct Kv8QuantArgs {
  const float* x;     // [n][HD] fp32
  int n;
  // flat output (op API): codes [n][HD], scales [n]
  int8_t* codes;
  float* scales;
  // model staging (codes == NULL): vector v = (t * 2 + kv) * Hkv + head of a
  // pass of tokens at positions pos0 + t goes to this layer's K (kv = 0) or V
  // plane of the lane: codes at ((head * ctx + pos0 + t) * HD), scale at
  // (head * ctx + pos0 + t)
  int8_t* k8;
  int8_t* v8;
  float* ks;
  float* vs;
  int Hkv, ctx, pos0;
  // decode rows (rows != NULL): t indexes the step's rows, each at its own
  // lane and position; k8 .. vs are lane 0's planes and lane l's start
  // lane_stride elements (codes) further
  const RowCtx* rows;
  long long lane_stride;
};

constexpr int kKv8Warps = 8;

// One warp per vector.
template <int HD>
__global__ void __launch_bounds__(kKv8Warps * 32) kv8_quant_kernel(const Kv8QuantArgs a) {
  constexpr int E = HD / 32;
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int v = blockIdx.x * kKv8Warps + (threadIdx.x >> 5);
  if (v >= a.n) return;   // warp-uniform
  float x[E];
  const float* src = a.x + (size_t)v * HD + lane * E;
#pragma unroll
  for (int i = 0; i < E; ++i) x[i] = src[i];
  int q[E];
  const float scale = kv8_quant_warp<E>(x, q);
  int8_t* dst;
  float* sdst;
  if (a.codes) {
    dst = a.codes + (size_t)v * HD;
    sdst = a.scales + v;
  } else {
    const int head = v % a.Hkv, kv = (v / a.Hkv) & 1, t = v / (2 * a.Hkv);
    size_t lane_off = 0;
    int pos = a.pos0 + t;
    if (a.rows) {
      const RowCtx rc = a.rows[t];
      lane_off = (size_t)rc.lane * a.lane_stride;
      pos = rc.pos;
    }
    const size_t row = (size_t)head * a.ctx + pos;
    dst = (kv ? a.v8 : a.k8) + lane_off + row * HD;
    sdst = (kv ? a.vs : a.ks) + lane_off / HD + row;
  }
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < E; ++i) w |= ((uint32_t)q[i] & 0xffu) << (8 * i);
  if (E == 4) *reinterpret_cast<uint32_t*>(dst + lane * E) = w;
  else *reinterpret_cast<uint16_t*>(dst + lane * E) = (uint16_t)w;
  if (lane == 0) *sdst = scale;
}

}  // namespace tl
