// LM head with softcapped logits and cross-entropy over the memory state
// ("Maglev: Sliding Recurrent Memory", paper.rainbus.top, 方法步骤详情:
// p(x_{t+1} | x_<=t) = softmax(15 tanh(U m_t / 15)); the loss averages the
// per-token CE over the positions in I). The logits GEMM and its fused
// epilogue (capped logits, per-tile row max / sum of exponentials, target
// logit) are in tc_gemm.cu; here:
//   finish  per row: LSE = log-sum-exp merged over the tiles' partials,
//           CE_t = LSE_t - c_t[y_t]
//   sum     loss = inv_count * sum_t CE_t in a fixed order (bitwise repeatable)
//   grad    dz = inv_count (exp(c - LSE) - onehot(y)) (1 - (c / softcap)^2),
//           bf16, the A operand of the dm and dU GEMMs
#include <cmath>

#include "common.cuh"
#include "launchers.h"

namespace maglev {
namespace {

constexpr float LOG2E_F = 1.4426950408889634f;

// One warp per row: merge the row's (max, sum) pairs of its N tiles.
__global__ void __launch_bounds__(256) lm_ce_finish_kernel(int64_t N, int V, int tiles, const float2* __restrict__ part,
                                                           const float* __restrict__ tgt,
                                                           const int64_t* __restrict__ targets,
                                                           float* __restrict__ lse, float* __restrict__ ce) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + threadIdx.x / 32;
  if (row >= N) return;
  const float2* pr = part + row * tiles;
  float mx = -INFINITY;
  for (int i = lane; i < tiles; i += 32) mx = fmaxf(mx, pr[i].x);
  mx = warp_max(mx);
  float sm = 0.f;
  for (int i = lane; i < tiles; i += 32) sm += pr[i].y * exp2f((pr[i].x - mx) * LOG2E_F);
  sm = warp_sum(sm);
  if (lane == 0) {
    const float l = mx + logf(sm);
    lse[row] = l;
    const int64_t y = targets[row];
    ce[row] = (y >= 0 && y < V) ? l - tgt[row] : NAN;
  }
}

// loss = inv_count * sum of ce[0..N) in a fixed order (one block).
__global__ void __launch_bounds__(1024) lm_ce_sum_kernel(int64_t N, float inv_count, const float* __restrict__ ce,
                                                         float* __restrict__ loss) {
  __shared__ float red[32];
  float acc = 0.f;
  for (int64_t i = threadIdx.x; i < N; i += 1024) acc += ce[i];
  acc = warp_sum(acc);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    float x = red[threadIdx.x];
    x = warp_sum(x);
    if (threadIdx.x == 0) *loss = x * inv_count;
  }
}

// dz for 8 consecutive columns of one row per thread (V % 8 == 0).
__global__ void __launch_bounds__(256) lm_ce_grad_kernel(int64_t N, int V, float inv_count, float inv_cap,
                                                         const float* __restrict__ c, const float* __restrict__ lse,
                                                         const int64_t* __restrict__ targets, bf16* __restrict__ dz) {
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int vpr = V / 8;
  if (gid >= N * vpr) return;
  const int64_t row = gid / vpr;
  const int col0 = (int)(gid % vpr) * 8;
  const int64_t off = row * V + col0;
  float x[8];
  load8f(c + off, x);
  const float l = lse[row];
  const int64_t y = targets[row];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float pe = exp2f((x[e] - l) * LOG2E_F);
    const float t = x[e] * inv_cap;
    x[e] = inv_count * (pe - (col0 + e == y ? 1.0f : 0.0f)) * (1.0f - t * t);
  }
  store8f(dz + off, x);
}

}  // namespace

cudaError_t launch_lm_ce_finish(int64_t N, int V, int tiles, float inv_count, float softcap, const float2* part,
                                const float* tgt, const int64_t* targets, const float* c, float* lse, float* ce,
                                float* loss, void* dz, cudaStream_t st) {
  lm_ce_finish_kernel<<<(unsigned)((N + 7) / 8), 256, 0, st>>>(N, V, tiles, part, tgt, targets, lse, ce);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  lm_ce_sum_kernel<<<1, 1024, 0, st>>>(N, inv_count, ce, loss);
  if ((e = cudaGetLastError()) != cudaSuccess || dz == nullptr) return e;
  const int64_t n = N * (V / 8);
  lm_ce_grad_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(N, V, inv_count, 1.0f / softcap, c, lse, targets,
                                                                 static_cast<bf16*>(dz));
  return cudaGetLastError();
}

}  // namespace maglev
