// a7: consistency loss lambda * inv_count * sum_t ||m_t - m'_t||^2 / sqrt(d)
// ("Maglev: Sliding Recurrent Memory", paper.rainbus.top, 方法步骤详情), with its
// gradients. The sum is reduced in a fixed order (per-block partials, then one
// block over the partials), so the loss is bitwise reproducible run to run.
#include "common.cuh"
#include "launchers.h"

namespace maglev {
namespace {

constexpr int LOSS_THREADS = 256;
constexpr int LOSS_U = 2;             // 8-element vectors per thread per round
constexpr int LOSS_MAX_BLOCKS = 592;  // persistent grid: 4 blocks on each of 148 SMs

// 8 elements in their stored form, so that a thread puts all its loads of a
// round in flight before any arithmetic.
template <typename T>
struct Raw8L;
template <>
struct Raw8L<bf16> {
  uint4 u;
  __device__ __forceinline__ void load(const bf16* p) { u = *reinterpret_cast<const uint4*>(p); }
  __device__ __forceinline__ void load_from(const float* x) {  // rounded as store8f rounds
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
  }
  __device__ __forceinline__ void to(float* x) const {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
};
template <>
struct Raw8L<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = *reinterpret_cast<const float4*>(p);
    b = *reinterpret_cast<const float4*>(p + 4);
  }
  __device__ __forceinline__ void load_from(const float* x) {
    a = make_float4(x[0], x[1], x[2], x[3]);
    b = make_float4(x[4], x[5], x[6], x[7]);
  }
  __device__ __forceinline__ void to(float* x) const {
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
};

// Block b walks rounds r = b, b + G, ... (G blocks); round r covers vectors
// [r * 256 * U, (r + 1) * 256 * U). Each thread loads all U vectors of m, m'
// and, when accumulating, dm of its round before any arithmetic, then writes
// dm, dm' and adds its squares; the block's partial is the sum over its rounds
// in a fixed order, so the loss is bitwise reproducible for a given size.
template <typename T>
__global__ void __launch_bounds__(LOSS_THREADS, sizeof(T) == 2 ? 4 : 2) loss_partial_kernel(
    const T* __restrict__ m, const T* __restrict__ mt, int64_t n, float scale_grad,
    T* __restrict__ dm, T* __restrict__ dmt, int accumulate, float* __restrict__ partials) {
  __shared__ float red[LOSS_THREADS / 32];
  float acc = 0.f;
  if ((n & 7) == 0) {
    const int64_t nv = n >> 3;
    const bool rd = dm != nullptr && accumulate;
    for (int64_t r0 = (int64_t)blockIdx.x * LOSS_THREADS * LOSS_U; r0 < nv;
         r0 += (int64_t)gridDim.x * LOSS_THREADS * LOSS_U) {
      Raw8L<T> a[LOSS_U], b[LOSS_U], d[LOSS_U];
#pragma unroll
      for (int u = 0; u < LOSS_U; ++u) {
        const int64_t i = r0 + (int64_t)u * LOSS_THREADS + threadIdx.x;
        if (i < nv) {
          a[u].load(m + 8 * i);
          b[u].load(mt + 8 * i);
          if (rd) d[u].load(dm + 8 * i);
        }
      }
#pragma unroll
      for (int u = 0; u < LOSS_U; ++u) {
        const int64_t i = r0 + (int64_t)u * LOSS_THREADS + threadIdx.x;
        if (i >= nv) continue;
        float x[8], y[8], z[8];
        a[u].to(x);
        b[u].to(y);
        if (rd) d[u].to(z);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float diff = x[e] - y[e];
          acc = fmaf(diff, diff, acc);
          // product and sum rounded separately (no contraction): loss_prep_partial_kernel
          // forms the same dm bit for bit
          const float g = __fmul_rn(scale_grad, diff);
          x[e] = rd ? __fadd_rn(z[e], g) : g;
          y[e] = -g;
        }
        if (dm) store8f(dm + 8 * i, x);
        if (dmt) store8f(dmt + 8 * i, y);
      }
    }
  } else {
    for (int64_t i = (int64_t)blockIdx.x * LOSS_THREADS + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * LOSS_THREADS) {
      const float diff = to_f(m[i]) - to_f(mt[i]);
      acc = fmaf(diff, diff, acc);
      const float g = scale_grad * diff;
      if (dm) dm[i] = from_f<T>(accumulate ? to_f(dm[i]) + g : g);
      if (dmt) dmt[i] = from_f<T>(-g);
    }
  }
  acc = warp_sum(acc);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    float x = threadIdx.x < LOSS_THREADS / 32 ? red[threadIdx.x] : 0.f;
    x = warp_sum(x);
    if (threadIdx.x == 0) partials[blockIdx.x] = x;
  }
}

// The loss of a layer's own output fused with the first pass of that layer's
// attention backward ("Maglev: Sliding Recurrent Memory", paper.rainbus.top,
// 方法步骤详情: the consistency loss; the backward of the banded attention
// needs Delta = rowsum(out * dO) per query row and head). m = out, dm = dO
// (updated in place, as loss_partial_kernel with accumulate); besides the
// squares, each 8-element vector adds out * (the stored dO) to its head's Delta
// (HDV vectors per head, aligned lane groups of a warp) and zeroes its part of
// the fp32 dQ accumulator. The squares are summed in loss_partial_kernel's
// order on the same grid, so the loss is the same, bit for bit.
template <typename T, int HDV>
__global__ void __launch_bounds__(LOSS_THREADS, sizeof(T) == 2 ? 4 : 2) loss_prep_partial_kernel(
    const T* __restrict__ m, const T* __restrict__ mt, int64_t n, float scale_grad, T* __restrict__ dm,
    float* __restrict__ partials, float* __restrict__ delta, float* __restrict__ dq_acc, int seq, int heads) {
  __shared__ float red[LOSS_THREADS / 32];
  float acc = 0.f;
  const int64_t nv = n >> 3;                      // whole heads: a multiple of HDV
  const int64_t vrow = (int64_t)heads * HDV;      // vectors per token row
  for (int64_t r0 = (int64_t)blockIdx.x * LOSS_THREADS * LOSS_U; r0 < nv;
       r0 += (int64_t)gridDim.x * LOSS_THREADS * LOSS_U) {
    Raw8L<T> a[LOSS_U], b[LOSS_U], d[LOSS_U];
#pragma unroll
    for (int u = 0; u < LOSS_U; ++u) {
      const int64_t i = r0 + (int64_t)u * LOSS_THREADS + threadIdx.x;
      if (i < nv) {
        a[u].load(m + 8 * i);
        b[u].load(mt + 8 * i);
        d[u].load(dm + 8 * i);
      }
    }
#pragma unroll
    for (int u = 0; u < LOSS_U; ++u) {
      const int64_t i = r0 + (int64_t)u * LOSS_THREADS + threadIdx.x;
      float dl = 0.f;
      if (i < nv) {
        float x[8], y[8], z[8];
        a[u].to(x);
        b[u].to(y);
        d[u].to(z);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float diff = x[e] - y[e];
          acc = fmaf(diff, diff, acc);
          z[e] = __fadd_rn(z[e], __fmul_rn(scale_grad, diff));  // as loss_partial_kernel
        }
        store8f(dm + 8 * i, z);
        Raw8L<T> w;  // the dO just stored, read back in registers in its stored precision
        w.load_from(z);
        w.to(z);
#pragma unroll
        for (int e = 0; e < 8; ++e) dl = fmaf(x[e], z[e], dl);
        if (dq_acc) {
          *reinterpret_cast<float4*>(dq_acc + 8 * i) = make_float4(0.f, 0.f, 0.f, 0.f);
          *reinterpret_cast<float4*>(dq_acc + 8 * i + 4) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      // a head's HDV vectors are an aligned lane group, all in range or all out
#pragma unroll
      for (int o = HDV / 2; o > 0; o >>= 1) dl += __shfl_xor_sync(0xffffffffu, dl, o);
      if (i < nv && (threadIdx.x % HDV) == 0) {
        const int64_t row = i / vrow;
        const int h = (int)((i % vrow) / HDV);
        const int t = (int)(row % seq);
        const int64_t bb = row / seq;
        delta[(bb * heads + h) * seq + t] = dl;
      }
    }
  }
  acc = warp_sum(acc);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    float x = threadIdx.x < LOSS_THREADS / 32 ? red[threadIdx.x] : 0.f;
    x = warp_sum(x);
    if (threadIdx.x == 0) partials[blockIdx.x] = x;
  }
}

__global__ void __launch_bounds__(LOSS_THREADS) loss_final_kernel(const float* __restrict__ partials,
                                                                  int nblk, float scale_loss,
                                                                  float* __restrict__ loss) {
  __shared__ float red[LOSS_THREADS / 32];
  float acc = 0.f;
  for (int i = threadIdx.x; i < nblk; i += LOSS_THREADS) acc += partials[i];
  acc = warp_sum(acc);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    float x = threadIdx.x < LOSS_THREADS / 32 ? red[threadIdx.x] : 0.f;
    x = warp_sum(x);
    if (threadIdx.x == 0) *loss = x * scale_loss;
  }
}

}  // namespace

int loss_partial_blocks(int64_t n) {
  const int64_t per = (n & 7) == 0 ? 8 * LOSS_THREADS * LOSS_U : LOSS_THREADS;  // elements per round
  const int64_t b = (n + per - 1) / per;
  return (int)(b < 1 ? 1 : (b > LOSS_MAX_BLOCKS ? LOSS_MAX_BLOCKS : b));
}

cudaError_t launch_consistency_loss(const void* m, const void* mt, int64_t rows, int d, int dtype,
                                    float scale_loss, float scale_grad, float* loss, void* dm,
                                    void* dmt, int accumulate, float* partials, cudaStream_t st) {
  const int64_t n = rows * (int64_t)d;
  const int nblk = loss_partial_blocks(n);
  if (dtype == 1)
    loss_partial_kernel<bf16><<<nblk, LOSS_THREADS, 0, st>>>(
        (const bf16*)m, (const bf16*)mt, n, scale_grad, (bf16*)dm, (bf16*)dmt, accumulate, partials);
  else
    loss_partial_kernel<float><<<nblk, LOSS_THREADS, 0, st>>>(
        (const float*)m, (const float*)mt, n, scale_grad, (float*)dm, (float*)dmt, accumulate, partials);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  loss_final_kernel<<<1, LOSS_THREADS, 0, st>>>(partials, nblk, scale_loss, loss);
  return cudaGetLastError();
}

// The loss of out [rows, H*hd] against mt, accumulated into dout, plus the
// attention backward's Delta [B, H, seq] and zeroed dq_acc (nullable) — see
// loss_prep_partial_kernel. hd is 64 or 128.
cudaError_t launch_consistency_loss_prep(const void* out, const void* mt, int64_t rows, int H, int hd, int seq,
                                         int dtype, float scale_loss, float scale_grad, float* loss, void* dout,
                                         float* delta, float* dq_acc, float* partials, cudaStream_t st) {
  const int64_t n = rows * (int64_t)H * hd;
  const int nblk = loss_partial_blocks(n);
#define MAGLEV_LOSS_PREP(TT, HDV)                                                                         \
  loss_prep_partial_kernel<TT, HDV><<<nblk, LOSS_THREADS, 0, st>>>((const TT*)out, (const TT*)mt, n,         \
                                                                   scale_grad, (TT*)dout, partials, delta,  \
                                                                   dq_acc, seq, H)
  if (dtype == 1 && hd == 128) MAGLEV_LOSS_PREP(bf16, 16);
  else if (dtype == 1 && hd == 64) MAGLEV_LOSS_PREP(bf16, 8);
  else if (dtype == 0 && hd == 128) MAGLEV_LOSS_PREP(float, 16);
  else if (dtype == 0 && hd == 64) MAGLEV_LOSS_PREP(float, 8);
  else return cudaErrorInvalidValue;
#undef MAGLEV_LOSS_PREP
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  loss_final_kernel<<<1, LOSS_THREADS, 0, st>>>(partials, nblk, scale_loss, loss);
  return cudaGetLastError();
}

}  // namespace maglev
