// Scratch-free variant of the consistency loss, for callers that cannot
// allocate device memory: for example a plugin or custom-op interface that
// hands the library its input and output tensors but no workspace, or a
// latency-critical loop in which cudaMalloc (which may synchronise the
// device) is not allowed. It computes exactly what maglev_consistency_loss
// computes; its per-block partial sums live in a file-scope device array
// instead of a caller-provided workspace.
//
// The array holds NOALLOC_PARTIALS fp32 partial sums (128 KiB). Every device
// that loads the library keeps it until the process exits. Each partial
// covers NOALLOC_CHUNK elements, so one call handles at most
// NOALLOC_PARTIALS * NOALLOC_CHUNK = 67,108,864 elements (rows * d).
//
// All calls share the one array. A call writes every partial it later reads,
// so nothing has to start at zero; but calls that overlap on the GPU (for
// example on two streams) race on the array and must be serialised.
#include <cmath>
#include <mutex>

#include "common.cuh"
#include "launchers.h"
#include "maglev.h"

namespace maglev {
namespace {

constexpr int NOALLOC_THREADS = 256;
constexpr int NOALLOC_PARTIALS = 32768;
constexpr int64_t NOALLOC_CHUNK = 2048;
constexpr int64_t NOALLOC_MAX_ELEMS = (int64_t)NOALLOC_PARTIALS * NOALLOC_CHUNK;

static __device__ __align__(256) float g_loss_scratch[NOALLOC_PARTIALS];

template <typename T>
__global__ void __launch_bounds__(NOALLOC_THREADS) noalloc_partial_kernel(
    const T* __restrict__ m, const T* __restrict__ mt, int64_t n, float scale_grad,
    T* __restrict__ dm, T* __restrict__ dmt, int accumulate, float* __restrict__ partials) {
  __shared__ float red[NOALLOC_THREADS / 32];
  const int64_t lo = (int64_t)blockIdx.x * NOALLOC_CHUNK;
  const int64_t hi = min(n, lo + NOALLOC_CHUNK);
  float acc = 0.f;
  if ((n & 7) == 0) {
    // 8 elements (16 or 32 bytes) per thread and step; NOALLOC_CHUNK is a
    // multiple of 8, so every vector lies inside one chunk
    for (int64_t i = lo + 8 * threadIdx.x; i < hi; i += 8 * NOALLOC_THREADS) {
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
    for (int64_t i = lo + threadIdx.x; i < hi; i += NOALLOC_THREADS) {
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
    float x = threadIdx.x < NOALLOC_THREADS / 32 ? red[threadIdx.x] : 0.f;
    x = warp_sum(x);
    if (threadIdx.x == 0) partials[blockIdx.x] = x;
  }
}

__global__ void __launch_bounds__(NOALLOC_THREADS) noalloc_final_kernel(
    const float* __restrict__ partials, int nblk, float scale_loss, float* __restrict__ loss) {
  __shared__ float red[NOALLOC_THREADS / 32];
  float acc = 0.f;
  for (int i = threadIdx.x; i < nblk; i += NOALLOC_THREADS) acc += partials[i];
  acc = warp_sum(acc);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    float x = threadIdx.x < NOALLOC_THREADS / 32 ? red[threadIdx.x] : 0.f;
    x = warp_sum(x);
    if (threadIdx.x == 0) *loss = x * scale_loss;
  }
}

// Device address of g_loss_scratch on the current device. In host code the
// symbol itself is only a host-side stand-in and must never be handed to a
// kernel. The address is looked up with the device current on the first call
// and again on every call whose stream is not being captured (a device reset
// reloads the module, possibly at another address); a call made during stream
// capture uses the address cached by an earlier call on that device.
std::mutex g_scratch_mu;
float* g_scratch_addr[128];

cudaError_t scratch_address(cudaStream_t s, float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  const bool capturing = cudaStreamIsCapturing(s, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!capturing || !g_scratch_addr[dev]) {
    if (capturing) return cudaErrorStreamCaptureUnsupported;  // first call on this device inside a capture
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_loss_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

maglev_status fail_msg(maglev_status st, const char* msg) {
  set_last_error(msg);
  return st;
}

}  // namespace
}  // namespace maglev

using namespace maglev;

extern "C" maglev_status maglev_consistency_loss_noalloc(const void* m, const void* m_target,
                                                         int64_t rows, int d, int dtype,
                                                         float lambda, float inv_count,
                                                         float* loss, void* dm, void* dm_target,
                                                         int accumulate_dm, void* stream) {
  auto misaligned = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
  if (rows < 0) return fail_msg(MAGLEV_ERR_INVALID_ARG, "rows must be >= 0");
  if (d < 1) return fail_msg(MAGLEV_ERR_INVALID_ARG, "d must be >= 1");
  if (dtype != MAGLEV_F32 && dtype != MAGLEV_BF16)
    return fail_msg(MAGLEV_ERR_INVALID_ARG, "dtype must be MAGLEV_F32 or MAGLEV_BF16");
  if (!std::isfinite(lambda) || !std::isfinite(inv_count) || inv_count < 0)
    return fail_msg(MAGLEV_ERR_INVALID_ARG, "lambda and inv_count must be finite, inv_count >= 0");
  if (!loss || misaligned(loss)) return fail_msg(MAGLEV_ERR_INVALID_ARG, "loss must be a 16-byte aligned pointer");
  if (misaligned(dm) || misaligned(dm_target))
    return fail_msg(MAGLEV_ERR_INVALID_ARG, "dm and dm_target must be 16-byte aligned");
  if (rows == 0) return MAGLEV_OK;
  if (!m || !m_target || misaligned(m) || misaligned(m_target))
    return fail_msg(MAGLEV_ERR_INVALID_ARG, "m and m_target must be 16-byte aligned pointers");
  const int64_t n = rows * (int64_t)d;
  if (n > NOALLOC_MAX_ELEMS)
    return fail_msg(MAGLEV_ERR_UNSUPPORTED,
                    "maglev_consistency_loss_noalloc handles at most 67108864 elements (rows * d); "
                    "use maglev_consistency_loss with a workspace for larger inputs");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* partials = nullptr;
  cudaError_t e = scratch_address(s, &partials);
  if (e == cudaErrorStreamCaptureUnsupported)
    return fail_msg(MAGLEV_ERR_CUDA,
                    "maglev_consistency_loss_noalloc: the first call on a device must come before any stream capture");
  if (e != cudaSuccess) return fail_msg(MAGLEV_ERR_CUDA, cudaGetErrorString(e));
  const double ic = inv_count == 0.0f ? 1.0 / (double)rows : (double)inv_count;
  const double sl = (double)lambda * ic / std::sqrt((double)d);
  const int nblk = (int)((n + NOALLOC_CHUNK - 1) / NOALLOC_CHUNK);
  if (dtype == MAGLEV_BF16)
    noalloc_partial_kernel<bf16><<<nblk, NOALLOC_THREADS, 0, s>>>(
        (const bf16*)m, (const bf16*)m_target, n, (float)(2.0 * sl), (bf16*)dm, (bf16*)dm_target,
        accumulate_dm ? 1 : 0, partials);
  else
    noalloc_partial_kernel<float><<<nblk, NOALLOC_THREADS, 0, s>>>(
        (const float*)m, (const float*)m_target, n, (float)(2.0 * sl), (float*)dm,
        (float*)dm_target, accumulate_dm ? 1 : 0, partials);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail_msg(MAGLEV_ERR_CUDA, cudaGetErrorString(e));
  noalloc_final_kernel<<<1, NOALLOC_THREADS, 0, s>>>(partials, nblk, (float)sl, loss);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail_msg(MAGLEV_ERR_CUDA, cudaGetErrorString(e));
  return MAGLEV_OK;
}
