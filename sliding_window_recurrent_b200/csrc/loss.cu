// a7: consistency loss lambda * inv_count * sum_t ||m_t - m'_t||^2 / sqrt(d)
// ("Maglev: Sliding Recurrent Memory", paper.rainbus.top, 方法步骤详情), with its
// gradients. The sum is reduced in a fixed order (per-block partials, then one
// block over the partials), so the loss is bitwise reproducible run to run.
#include "common.cuh"
#include "launchers.h"

namespace maglev {
namespace {

constexpr int LOSS_THREADS = 256;
constexpr int LOSS_U = 4;                                 // 8-element vectors per thread
constexpr int64_t LOSS_CHUNK = 8 * LOSS_THREADS * LOSS_U;  // elements per block

// Block b covers elements [b * LOSS_CHUNK, (b + 1) * LOSS_CHUNK): each thread
// puts all of its loads (LOSS_U vectors of m, m' and, when accumulating, dm)
// in flight before any arithmetic, then writes dm, dm' and adds its squares.
template <typename T>
__global__ void __launch_bounds__(LOSS_THREADS) loss_partial_kernel(
    const T* __restrict__ m, const T* __restrict__ mt, int64_t n, float scale_grad,
    T* __restrict__ dm, T* __restrict__ dmt, int accumulate, float* __restrict__ partials) {
  __shared__ float red[LOSS_THREADS / 32];
  const int64_t lo = (int64_t)blockIdx.x * LOSS_CHUNK;
  float acc = 0.f;
  if ((n & 7) == 0) {
    float a[LOSS_U][8], b[LOSS_U][8], d[LOSS_U][8];
    const bool rd = dm != nullptr && accumulate;
#pragma unroll
    for (int u = 0; u < LOSS_U; ++u) {
      const int64_t i = lo + 8 * ((int64_t)u * LOSS_THREADS + threadIdx.x);
      if (i < n) {
        load8f(m + i, a[u]);
        load8f(mt + i, b[u]);
        if (rd) load8f(dm + i, d[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < LOSS_U; ++u) {
      const int64_t i = lo + 8 * ((int64_t)u * LOSS_THREADS + threadIdx.x);
      if (i >= n) continue;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float diff = a[u][e] - b[u][e];
        acc = fmaf(diff, diff, acc);
        const float g = scale_grad * diff;
        a[u][e] = rd ? d[u][e] + g : g;
        b[u][e] = -g;
      }
      if (dm) store8f(dm + i, a[u]);
      if (dmt) store8f(dmt + i, b[u]);
    }
  } else {
    const int64_t hi = min(n, lo + LOSS_CHUNK);
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
  const int64_t b = (n + LOSS_CHUNK - 1) / LOSS_CHUNK;
  return (int)(b < 1 ? 1 : b);
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

}  // namespace maglev
