// pi_device.cuh -- device helpers shared by the sparse-FFN kernels (sm_100a).
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#define PI_DEV __device__ __forceinline__

namespace pi {

enum WType { W_F32 = 0, W_F16 = 1, W_INT4 = 2 };
enum Act { ACT_RELU = 0, ACT_SWIGLU = 1 };

// status word codes (same values as pi_status)
constexpr int kStatusTimeout = 5;
constexpr int kStatusDeviceArg = 6;

PI_DEV void set_status(int *status, int code) { atomicCAS(status, 0, code); }

// ---------------------------------------------------------------- PDL
PI_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
PI_DEV void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// ---------------------------------------------------------------- loads
// Weights are streamed once per step: bypass L1, read-only path.
PI_DEV uint4 ld_stream16(const void *p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
PI_DEV uint32_t ld_stream4(const void *p) {
  uint32_t v;
  asm("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
// Small vectors reused by every warp of an SM (u, h): keep them in L1.
PI_DEV uint4 ld_keep16(const void *p) { return __ldg(reinterpret_cast<const uint4 *>(p)); }
PI_DEV float4 ld_keep_f4(const float *p) { return __ldg(reinterpret_cast<const float4 *>(p)); }

PI_DEV void l2_prefetch(const void *p) { asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(p)); }

// ---------------------------------------------------------------- conversions
PI_DEV void h8_to_f8(const uint4 &v, float o[8]) {
  const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float2 t = __half22float2(h[k]);
    o[2 * k] = t.x;
    o[2 * k + 1] = t.y;
  }
}

// 8 nibbles of one 32-bit word -> (q - 8) as floats, element order low nibble first
PI_DEV void q8_to_f8(uint32_t w, float o[8]) {
#pragma unroll
  for (int k = 0; k < 8; ++k) o[k] = (float)((int)((w >> (4 * k)) & 15u) - 8);
}

PI_DEV float silu(float z) { return z / (1.0f + expf(-z)); }

// ---------------------------------------------------------------- reductions
PI_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

PI_DEV double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------- row chunks
// A "chunk" is 16 bytes of one weight row: 4 fp32, 8 fp16 or 32 int4 values.
template <int WT> struct Chunk;
template <> struct Chunk<W_F32> { static constexpr int elems = 4; };
template <> struct Chunk<W_F16> { static constexpr int elems = 8; };
template <> struct Chunk<W_INT4> { static constexpr int elems = 32; };

// Bytes of one weight row of d elements (int4: packed nibbles only).
PI_DEV size_t row_bytes(int wt, int d) { return wt == W_F32 ? (size_t)d * 4 : wt == W_F16 ? (size_t)d * 2 : (size_t)d / 2; }

// dot of one 16-byte weight chunk at element column c0 with token vector u
// (fp32 when WT == W_F32, fp16 otherwise).  For int4 the scale is applied by
// the caller per chunk (one chunk = one 32-element group).
template <int WT>
PI_DEV float chunk_dot(const uint4 &w, const void *u, int c0);

template <>
PI_DEV float chunk_dot<W_F32>(const uint4 &w, const void *u, int c0) {
  float4 uv = ld_keep_f4(reinterpret_cast<const float *>(u) + c0);
  float4 wv = *reinterpret_cast<const float4 *>(&w);
  float a = wv.x * uv.x;
  a = fmaf(wv.y, uv.y, a);
  a = fmaf(wv.z, uv.z, a);
  a = fmaf(wv.w, uv.w, a);
  return a;
}

template <>
PI_DEV float chunk_dot<W_F16>(const uint4 &w, const void *u, int c0) {
  float wf[8], uf[8];
  h8_to_f8(w, wf);
  h8_to_f8(ld_keep16(reinterpret_cast<const __half *>(u) + c0), uf);
  float a = wf[0] * uf[0];
#pragma unroll
  for (int k = 1; k < 8; ++k) a = fmaf(wf[k], uf[k], a);
  return a;
}

template <>
PI_DEV float chunk_dot<W_INT4>(const uint4 &w, const void *u, int c0) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  float a = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float wf[8], uf[8];
    q8_to_f8(ws[j], wf);
    h8_to_f8(ld_keep16(reinterpret_cast<const __half *>(u) + c0 + 8 * j), uf);
#pragma unroll
    for (int k = 0; k < 8; ++k) a = fmaf(wf[k], uf[k], a);
  }
  return a;
}

}  // namespace pi
