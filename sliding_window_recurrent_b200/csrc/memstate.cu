// Memory state of a decoder stack and its shifted copy.
//
// "Maglev: Sliding Recurrent Memory", paper.rainbus.top, 方法步骤详情: m_t is the
// stack's final post-RMSNorm state; the next segment reads the shifted memory
// m_{t-1}, with m_0 = 0. Reading: RMSNorm over the d channels of a row, no
// weight, eps added to the mean square.
//   forward:  m[b,t] = o[b,t] * rstd[b,t],  rstd = 1/sqrt(mean(o^2) + eps);
//             m_shift[b,0] = 0, m_shift[b,t] = m[b,t-1].
//   backward: dy[b,t] = dm[b,t] + dm_shift[b,t+1] (terms absent when NULL or
//             past the end), do = dout_in + rstd * (dy - m * mean(m * dy)),
//             dout_in optional (it may alias do).
// One warp per row; 8-element (16 or 32 byte) vector accesses when d % 8 == 0.
#include "common.cuh"
#include "launchers.h"

namespace maglev {
namespace {

constexpr int MS_THREADS = 256;
constexpr int MS_WARPS = MS_THREADS / 32;

__device__ __forceinline__ void ld8(const bf16* p, float* x) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void ld8(const float* p, float* x) {
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ void st8(bf16* p, const float* x) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void st8(float* p, const float* x) {
  *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(x[4], x[5], x[6], x[7]);
}

template <typename T>
__global__ void __launch_bounds__(MS_THREADS) memstate_fwd_kernel(const T* __restrict__ o, T* __restrict__ m,
                                                                  T* __restrict__ m_shift, float* __restrict__ rstd,
                                                                  int64_t rows, int T_len, int d, float eps) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * MS_WARPS + threadIdx.x / 32;
  if (row >= rows) return;
  const int t = (int)(row % T_len);
  const T* x = o + row * d;
  T* y = m + row * d;
  T* ys = (m_shift && t + 1 < T_len) ? m_shift + (row + 1) * d : nullptr;
  const bool vec = (d & 7) == 0;
  float ss = 0.f;
  if (vec) {
    for (int c = 8 * lane; c < d; c += 256) {
      float v[8];
      ld8(x + c, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(v[e], v[e], ss);
    }
  } else {
    for (int c = lane; c < d; c += 32) {
      const float v = to_f(x[c]);
      ss = fmaf(v, v, ss);
    }
  }
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / (float)d + eps);
  if (lane == 0) rstd[row] = r;
  if (vec) {
    for (int c = 8 * lane; c < d; c += 256) {
      float v[8];
      ld8(x + c, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] *= r;
      st8(y + c, v);
      if (ys) st8(ys + c, v);
    }
  } else {
    for (int c = lane; c < d; c += 32) {
      const T v = from_f<T>(to_f(x[c]) * r);
      y[c] = v;
      if (ys) ys[c] = v;
    }
  }
  if (m_shift && t == 0) {
    T* z = m_shift + row * d;
    for (int c = lane; c < d; c += 32) z[c] = from_f<T>(0.f);
  }
}

template <typename T>
__global__ void __launch_bounds__(MS_THREADS) memstate_bwd_kernel(const T* __restrict__ o, const float* __restrict__ rstd,
                                                                  const T* __restrict__ dm, const T* __restrict__ dms,
                                                                  const T* din, T* dout, int64_t rows, int T_len,
                                                                  int d) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * MS_WARPS + threadIdx.x / 32;
  if (row >= rows) return;
  const int t = (int)(row % T_len);
  const T* x = o + row * d;
  const T* g1 = dm ? dm + row * d : nullptr;
  const T* g2 = (dms && t + 1 < T_len) ? dms + (row + 1) * d : nullptr;
  T* dx = dout + row * d;
  const T* base = din ? din + row * d : nullptr;  // may alias dx: each element is read before it is written
  const float r = rstd[row];
  // m = o * r is recomputed in fp32 from o (the stored m is rounded)
  const bool vec = (d & 7) == 0;
  float dot = 0.f;
  if (vec) {
    for (int c = 8 * lane; c < d; c += 256) {
      float v[8], a[8] = {0, 0, 0, 0, 0, 0, 0, 0}, b[8];
      ld8(x + c, v);
      if (g1) ld8(g1 + c, a);
      if (g2) {
        ld8(g2 + c, b);
#pragma unroll
        for (int e = 0; e < 8; ++e) a[e] += b[e];
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) dot = fmaf(v[e] * r, a[e], dot);
    }
  } else {
    for (int c = lane; c < d; c += 32) {
      const float g = (g1 ? to_f(g1[c]) : 0.f) + (g2 ? to_f(g2[c]) : 0.f);
      dot = fmaf(to_f(x[c]) * r, g, dot);
    }
  }
  dot = warp_sum(dot) / (float)d;
  if (vec) {
    for (int c = 8 * lane; c < d; c += 256) {
      float v[8], a[8] = {0, 0, 0, 0, 0, 0, 0, 0}, b[8], prev[8];
      ld8(x + c, v);
      if (g1) ld8(g1 + c, a);
      if (g2) {
        ld8(g2 + c, b);
#pragma unroll
        for (int e = 0; e < 8; ++e) a[e] += b[e];
      }
      if (base) ld8(base + c, prev);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float g = r * (a[e] - v[e] * r * dot);
        a[e] = base ? prev[e] + g : g;
      }
      st8(dx + c, a);
    }
  } else {
    for (int c = lane; c < d; c += 32) {
      const float gsum = (g1 ? to_f(g1[c]) : 0.f) + (g2 ? to_f(g2[c]) : 0.f);
      const float g = r * (gsum - to_f(x[c]) * r * dot);
      dx[c] = from_f<T>(base ? to_f(base[c]) + g : g);
    }
  }
}

}  // namespace

cudaError_t launch_memstate_fwd(const void* o, void* m, void* m_shift, float* rstd, int B, int T, int d,
                                float eps, int dtype, cudaStream_t st) {
  const int64_t rows = (int64_t)B * T;
  if (rows == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((rows + MS_WARPS - 1) / MS_WARPS);
  if (dtype == DT_BF16)
    memstate_fwd_kernel<bf16><<<grid, MS_THREADS, 0, st>>>(static_cast<const bf16*>(o), static_cast<bf16*>(m),
                                                           static_cast<bf16*>(m_shift), rstd, rows, T, d, eps);
  else
    memstate_fwd_kernel<float><<<grid, MS_THREADS, 0, st>>>(static_cast<const float*>(o), static_cast<float*>(m),
                                                            static_cast<float*>(m_shift), rstd, rows, T, d, eps);
  return cudaGetLastError();
}

cudaError_t launch_memstate_bwd(const void* o, const float* rstd, const void* dm, const void* dm_shift,
                                const void* dout_in, void* dout, int B, int T, int d, int dtype, cudaStream_t st) {
  const int64_t rows = (int64_t)B * T;
  if (rows == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((rows + MS_WARPS - 1) / MS_WARPS);
  if (dtype == DT_BF16)
    memstate_bwd_kernel<bf16><<<grid, MS_THREADS, 0, st>>>(static_cast<const bf16*>(o), rstd,
                                                           static_cast<const bf16*>(dm),
                                                           static_cast<const bf16*>(dm_shift),
                                                           static_cast<const bf16*>(dout_in),
                                                           static_cast<bf16*>(dout), rows, T, d);
  else
    memstate_bwd_kernel<float><<<grid, MS_THREADS, 0, st>>>(static_cast<const float*>(o), rstd,
                                                            static_cast<const float*>(dm),
                                                            static_cast<const float*>(dm_shift),
                                                            static_cast<const float*>(dout_in),
                                                            static_cast<float*>(dout), rows, T, d);
  return cudaGetLastError();
}

}  // namespace maglev
