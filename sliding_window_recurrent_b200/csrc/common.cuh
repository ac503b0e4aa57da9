// Device helpers shared by the kernels of libmaglev (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace maglev {

typedef __nv_bfloat16 bf16;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(bf16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }

// 8 consecutive elements (16 bytes of bf16, 32 of fp32) to / from fp32 registers.
__device__ __forceinline__ void load8f(const bf16* p, float* x) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8f(const float* p, float* x) {
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ void store8f(bf16* p, const float* x) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void store8f(float* p, const float* x) {
  *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(x[4], x[5], x[6], x[7]);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// g = 2*sigmoid(a); finite for a = +-inf.
__device__ __forceinline__ float gate_value(float a) { return 2.0f / (1.0f + expf(-a)); }
// dg/da = 2 s (1 - s).
__device__ __forceinline__ float gate_slope(float a) {
  float s = 1.0f / (1.0f + expf(-a));
  return 2.0f * s * (1.0f - s);
}

// RoPE angle of pair c at absolute position p: p * base^(-2c/hd). The product
// is formed in double and reduced to [-pi, pi] before the float sincos, so
// positions in the thousands keep full float accuracy.
__device__ __forceinline__ void rope_cos_sin(int64_t p, int c, int hd, double log2_base,
                                             float* cs, float* sn) {
  const double two_pi = 6.283185307179586476925286766559;
  double inv_freq = exp2(-(2.0 * (double)c / (double)hd) * log2_base);
  double ang = (double)p * inv_freq;
  ang -= two_pi * rint(ang / two_pi);
  sincosf((float)ang, sn, cs);
}

// Device status word (per device, defined in api.cu); kernels receive its address.
enum { DEV_OK = 0, DEV_TIMEOUT = 4, DEV_BOUNDS = 5 };

__device__ __forceinline__ void record_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// Index checks of the debug build (compiled with -DMAGLEV_DEBUG): a false
// condition records MAGLEV_ERR_BOUNDS in the status word and the caller skips
// the access; nothing traps. In the release build the check is `true`.
#ifdef MAGLEV_DEBUG
__device__ __forceinline__ bool debug_check(int* err, bool cond) {
  if (!cond) record_error(err, DEV_BOUNDS);
  return cond;
}
#define MAGLEV_CHECK(err, cond) ::maglev::debug_check((err), (cond))
#else
#define MAGLEV_CHECK(err, cond) true
#endif

}  // namespace maglev
