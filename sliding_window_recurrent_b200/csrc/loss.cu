// a7: consistency loss lambda * inv_count * sum_t ||m_t - m'_t||^2 / sqrt(d)
// ("Maglev: Sliding Recurrent Memory", paper.rainbus.top, 方法步骤详情), with its
// gradients. The sum is reduced in a fixed order (per-block partials, then one
// block over the partials), so the loss is bitwise reproducible run to run.
#include "common.cuh"
#include "launchers.h"

namespace maglev {
namespace {

constexpr int LOSS_THREADS = 256;
constexpr int LOSS_MAX_BLOCKS = 1184;  // 8 x 148 SMs

template <typename T>
__global__ void __launch_bounds__(LOSS_THREADS) loss_partial_kernel(
    const T* __restrict__ m, const T* __restrict__ mt, int64_t n, int64_t chunk, float scale_grad,
    T* __restrict__ dm, T* __restrict__ dmt, int accumulate, float* __restrict__ partials) {
  __shared__ float red[LOSS_THREADS / 32];
  const int64_t lo = (int64_t)blockIdx.x * chunk;
  const int64_t hi = min(n, lo + chunk);
  float acc = 0.f;
  if ((chunk & 7) == 0 && (n & 7) == 0) {
    // 8 elements (16 or 32 bytes) per step; chunk boundaries stay 8-aligned
    for (int64_t i = lo + 8 * threadIdx.x; i < hi; i += 8 * LOSS_THREADS) {
      float a[8], b[8], d[8];
      load8f(m + i, a);
      load8f(mt + i, b);
      if (dm && accumulate) load8f(dm + i, d);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float diff = a[e] - b[e];
        acc = fmaf(diff, diff, acc);
        const float g = scale_grad * diff;
        a[e] = (dm && accumulate) ? d[e] + g : g;
        b[e] = -g;
      }
      if (dm) store8f(dm + i, a);
      if (dmt) store8f(dmt + i, b);
    }
  } else {
    for (int64_t i = lo + threadIdx.x; i < hi; i += LOSS_THREADS) {
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
  int64_t b = (n + 8 * LOSS_THREADS - 1) / (8 * LOSS_THREADS);
  if (b < 1) b = 1;
  if (b > LOSS_MAX_BLOCKS) b = LOSS_MAX_BLOCKS;
  return (int)b;
}

cudaError_t launch_consistency_loss(const void* m, const void* mt, int64_t rows, int d, int dtype,
                                    float scale_loss, float scale_grad, float* loss, void* dm,
                                    void* dmt, int accumulate, float* partials, cudaStream_t st) {
  const int64_t n = rows * (int64_t)d;
  const int nblk = loss_partial_blocks(n);
  const int64_t chunk = (((n + nblk - 1) / nblk) + 7) & ~(int64_t)7;
  if (dtype == 1)
    loss_partial_kernel<bf16><<<nblk, LOSS_THREADS, 0, st>>>(
        (const bf16*)m, (const bf16*)mt, n, chunk, scale_grad, (bf16*)dm, (bf16*)dmt, accumulate,
        partials);
  else
    loss_partial_kernel<float><<<nblk, LOSS_THREADS, 0, st>>>(
        (const float*)m, (const float*)mt, n, chunk, scale_grad, (float*)dm, (float*)dmt,
        accumulate, partials);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  loss_final_kernel<<<1, LOSS_THREADS, 0, st>>>(partials, nblk, scale_loss, loss);
  return cudaGetLastError();
}

}  // namespace maglev
