// CUDA-core GEMM with arbitrary element strides: the fp32 path's projection
// GEMMs (d20 layer: [B*T, d] x [d, 2D] forward, dR^T m and dR W backward).
#include "common.cuh"
#include "launchers.h"

namespace maglev {
namespace {

constexpr int BM = 64, BN = 64, BK = 16;

template <typename T>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmArgs g) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const T* A1 = static_cast<const T*>(g.A1);
  const T* B1 = static_cast<const T*>(g.B1);
  const T* A2 = static_cast<const T*>(g.A2);
  const T* B2 = static_cast<const T*>(g.B2);
  T* C = static_cast<T*>(g.C);
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int64_t m0 = (int64_t)blockIdx.y * BM, n0 = (int64_t)blockIdx.x * BN;
  const int64_t K = g.K1 + g.K2;
  float acc[4][4] = {};
  for (int64_t k0 = 0; k0 < K; k0 += BK) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      int e = tid + 256 * r;
      // A tile: (m, k) = (e / BK, e % BK)
      int am = e / BK, ak = e % BK;
      int64_t gm = m0 + am, gk = k0 + ak;
      float a = 0.f;
      if (gm < g.M && gk < K)
        a = gk < g.K1 ? to_f(A1[gm * g.sa1m + gk * g.sa1k])
                      : to_f(A2[gm * g.sa2m + (gk - g.K1) * g.sa2k]);
      As[ak][am] = a;
      // B tile: (k, n) = (e / BN, e % BN)
      int bk = e / BN, bn = e % BN;
      int64_t gk2 = k0 + bk, gn = n0 + bn;
      float b = 0.f;
      if (gn < g.N && gk2 < K)
        b = gk2 < g.K1 ? to_f(B1[gk2 * g.sb1k + gn * g.sb1n])
                       : to_f(B2[(gk2 - g.K1) * g.sb2k + gn * g.sb2n]);
      Bs[bk][bn] = b;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int64_t gm = m0 + ty * 4 + i;
    if (gm >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int64_t gn = n0 + tx * 4 + j;
      if (gn >= g.N) continue;
      int64_t off = gm * g.scm + gn * g.scn;
      float x = acc[i][j];
      if (g.accumulate) x += to_f(C[off]);
      C[off] = from_f<T>(x);
    }
  }
}

}  // namespace

cudaError_t launch_gemm_simt(const GemmArgs& g, cudaStream_t s) {
  if (g.M == 0 || g.N == 0) return cudaSuccess;
  dim3 grid((unsigned)((g.N + BN - 1) / BN), (unsigned)((g.M + BM - 1) / BM));
  if (g.dtype == 1)
    gemm_simt_kernel<bf16><<<grid, 256, 0, s>>>(g);
  else
    gemm_simt_kernel<float><<<grid, 256, 0, s>>>(g);
  return cudaGetLastError();
}

}  // namespace maglev
