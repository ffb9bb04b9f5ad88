// Shared device helpers for the CSA / HCA kernels (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/csa.h"

namespace csa {

// Counts the kernels the library enqueues (defined in api.cu; read by csa_launch_count).
void note_launch();
// SMs of the current device (148 on B200), read once; 148 when no device answers (the
// host-only size queries of a machine without a GPU).  Grids are planned in its units.
int num_sms();

// Error bits are OR-ed into a per-device word owned by api.cu; kernels get its address.
__device__ __forceinline__ void raise_err(unsigned* err, unsigned bit) {
  if (err) atomicOr(err, bit);
}

// ---- element access for the two latent storage types --------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float ld(const float* p) { return *p; }
  static __device__ __forceinline__ void st(float* p, float v) { *p = v; }
  // 16-byte vector: 4 floats
  static constexpr int VEC = 4;
  static __device__ __forceinline__ void ld_vec(const float* p, float* out) {
    float4 v = *reinterpret_cast<const float4*>(p);
    out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
  }
  static __device__ __forceinline__ void st_vec(float* p, const float* in) {
    *reinterpret_cast<float4*>(p) = make_float4(in[0], in[1], in[2], in[3]);
  }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void st(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
  static constexpr int VEC = 8;
  static __device__ __forceinline__ void ld_vec(const __nv_bfloat16* p, float* out) {
    uint4 v = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      out[2 * i] = __uint_as_float(w[i] << 16);
      out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  static __device__ __forceinline__ void st_vec(__nv_bfloat16* p, const float* in) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(in[2 * i], in[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  }
};

// ---- FP8 e4m3 / e2m1 / ue8m0 decoding (exact, from the format definitions) -----------------
// e4m3: sign | 4-bit exponent (bias 7) | 3-bit mantissa; exponent 0 is subnormal (mant/8 * 2^-6).
__device__ __forceinline__ float e4m3_to_float(uint32_t c) {
  const uint32_t s = (c & 0x80u) << 24;
  const uint32_t e = (c >> 3) & 0xFu;
  const uint32_t mnt = c & 0x7u;
  float mag;
  if (e == 0) mag = (float)mnt * 0.001953125f;                       // mant * 2^-9
  else mag = __uint_as_float(((e + 120u) << 23) | (mnt << 20));       // (1+mant/8) * 2^(e-7)
  return __uint_as_float(__float_as_uint(mag) | s);
}
__device__ __forceinline__ double e4m3_to_double(uint32_t c) { return (double)e4m3_to_float(c); }

// e2m1 magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6; sign in bit 3.
__device__ __forceinline__ float e2m1_to_float(uint32_t c) {
  const uint32_t e = (c >> 1) & 0x3u, mnt = c & 0x1u;
  float mag = (e == 0) ? 0.5f * (float)mnt : (1.0f + 0.5f * (float)mnt) * (float)(1u << (e - 1));
  return (c & 0x8u) ? -mag : mag;
}
__device__ __forceinline__ float ue8m0_to_float(uint32_t c) {
  // 2^(c-127); c == 0 is 2^-127 (subnormal in fp32)
  return c == 0 ? 5.877471754111438e-39f : __uint_as_float(c << 23);
}

// Monotone key for fp32 ordering: larger float -> larger key; NaN -> 0 (below everything).
__device__ __forceinline__ uint32_t f32_order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u & 0x7fffffffu) > 0x7f800000u) return 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float f32_from_order_key(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}

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
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace csa
