// CUDA-core kernels of the injected sliding-window attention layer for the
// fp32 path: banded attention forward and backward (dq, dk_bar / dv_bar) on
// the saved rotated / mixed entries. The element-wise injection and un-mix
// live in ew.cu.
//
// Source: "Maglev: Sliding Recurrent Memory", paper.rainbus.top, sections
// 前置知识 (SWA over the most recent W tokens; RoPE rotation of q and k) and
// 方法步骤详情 (k_rec = RMSNorm(W_k^rec m'_{t-1}), v_rec = W_v^rec m'_{t-1},
// k_bar = g_loc k + g_rec k_rec with g = 2 sigmoid(a), v_bar likewise; both keys
// rotated before the mix).
//
// Layout: activations [B,T,H,hd] (row (b,t,h) holds hd contiguous values);
// R_k, R_v [B,T,H*hd] share that flat layout; lse and delta are [B,H,T].
#include "common.cuh"
#include "launchers.h"

namespace maglev {
namespace {

constexpr unsigned FULL = 0xffffffffu;

// ---------------------------------------------------------------------------
// a5 forward: one warp per query row i, 8 rows per block sharing 32-key tiles
// of the window [i0-W+1, i0+7] in shared memory; online softmax in fp32.
// ---------------------------------------------------------------------------
template <typename T, int HD>
__global__ void __launch_bounds__(256) attn_fwd_kernel(SwaShape s, const T* __restrict__ qr,
                                                       const T* __restrict__ kb,
                                                       const T* __restrict__ vb,
                                                       T* __restrict__ out,
                                                       float* __restrict__ lse, float scale) {
  constexpr int NC = HD / 32;
  __shared__ float Ks[32][HD + 1];
  __shared__ float Vs[32][HD + 1];
  __shared__ float Qs[8][HD];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.y, b = blockIdx.z;
  const int T_ = s.T, H = s.H, W = s.W;
  const int i0 = blockIdx.x * 8, i = i0 + warp;
  const int lo = max(0, i0 - W + 1), hi = min(T_, i0 + 8) - 1;
  auto rowp = [&](int t) { return (((int64_t)b * T_ + t) * H + h) * HD; };
  if (i < T_)
    for (int c = lane; c < HD; c += 32) Qs[warp][c] = to_f(qr[rowp(i) + c]);
  float m = -INFINITY, l = 0.f, acc[NC];
#pragma unroll
  for (int r = 0; r < NC; ++r) acc[r] = 0.f;
  for (int j0 = lo; j0 <= hi; j0 += 32) {
    __syncthreads();
    for (int e = threadIdx.x; e < 32 * HD; e += 256) {
      const int jj = e / HD, c = e % HD, j = j0 + jj;
      float kv = 0.f, vv = 0.f;
      if (j <= hi) {
        kv = to_f(kb[rowp(j) + c]);
        vv = to_f(vb[rowp(j) + c]);
      }
      Ks[jj][c] = kv;
      Vs[jj][c] = vv;
    }
    __syncthreads();
    if (i < T_) {
      const int j = j0 + lane;
      const bool valid = j <= hi && j <= i && j >= i - W + 1;
      float sc = -INFINITY;
      if (valid) {
        float d = 0.f;
#pragma unroll 16
        for (int c = 0; c < HD; ++c) d = fmaf(Qs[warp][c], Ks[lane][c], d);
        sc = d * scale;
      }
      const float m_new = fmaxf(m, warp_max(sc));
      if (m_new != -INFINITY) {
        const float corr = expf(m - m_new);
        const float pv = valid ? expf(sc - m_new) : 0.f;
        l = l * corr + warp_sum(pv);
#pragma unroll
        for (int r = 0; r < NC; ++r) acc[r] *= corr;
#pragma unroll 4
        for (int jj = 0; jj < 32; ++jj) {
          const float pj = __shfl_sync(FULL, pv, jj);
#pragma unroll
          for (int r = 0; r < NC; ++r) acc[r] = fmaf(pj, Vs[jj][lane + 32 * r], acc[r]);
        }
        m = m_new;
      }
    }
  }
  if (i < T_) {
    const float inv = 1.f / l;
#pragma unroll
    for (int r = 0; r < NC; ++r) out[rowp(i) + lane + 32 * r] = from_f<T>(acc[r] * inv);
    if (lane == 0) lse[((int64_t)b * H + h) * T_ + i] = m + logf(l);
  }
}

// ---------------------------------------------------------------------------
// a6 backward, dq: warp per query row (same tiling as the forward); the
// result is rotated back by RoPE^T and written as dq.
// ---------------------------------------------------------------------------
template <typename T, int HD>
__global__ void __launch_bounds__(256) attn_bwd_dq_kernel(
    SwaShape s, const T* __restrict__ qr, const T* __restrict__ kb, const T* __restrict__ vb,
    const T* __restrict__ dout, const float* __restrict__ lse, const float* __restrict__ delta,
    T* __restrict__ dq, float scale) {
  constexpr int NC = HD / 32;
  __shared__ float Ks[32][HD + 1];
  __shared__ float Vs[32][HD + 1];
  __shared__ float Qs[8][HD];
  __shared__ float Gs[8][HD];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.y, b = blockIdx.z;
  const int T_ = s.T, H = s.H, W = s.W;
  const int i0 = blockIdx.x * 8, i = i0 + warp;
  const int lo = max(0, i0 - W + 1), hi = min(T_, i0 + 8) - 1;
  auto rowp = [&](int t) { return (((int64_t)b * T_ + t) * H + h) * HD; };
  float lse_i = 0.f, d_i = 0.f;
  if (i < T_) {
    for (int c = lane; c < HD; c += 32) {
      Qs[warp][c] = to_f(qr[rowp(i) + c]);
      Gs[warp][c] = to_f(dout[rowp(i) + c]);
    }
    lse_i = lse[((int64_t)b * H + h) * T_ + i];
    d_i = delta[((int64_t)b * H + h) * T_ + i];
  }
  float acc[NC];
#pragma unroll
  for (int r = 0; r < NC; ++r) acc[r] = 0.f;
  for (int j0 = lo; j0 <= hi; j0 += 32) {
    __syncthreads();
    for (int e = threadIdx.x; e < 32 * HD; e += 256) {
      const int jj = e / HD, c = e % HD, j = j0 + jj;
      float kv = 0.f, vv = 0.f;
      if (j <= hi) {
        kv = to_f(kb[rowp(j) + c]);
        vv = to_f(vb[rowp(j) + c]);
      }
      Ks[jj][c] = kv;
      Vs[jj][c] = vv;
    }
    __syncthreads();
    if (i < T_) {
      const int j = j0 + lane;
      const bool valid = j <= hi && j <= i && j >= i - W + 1;
      float ds = 0.f;
      if (valid) {
        float d = 0.f, dp = 0.f;
#pragma unroll 16
        for (int c = 0; c < HD; ++c) {
          d = fmaf(Qs[warp][c], Ks[lane][c], d);
          dp = fmaf(Gs[warp][c], Vs[lane][c], dp);
        }
        const float p = expf(d * scale - lse_i);
        ds = p * (dp - d_i);
      }
#pragma unroll 4
      for (int jj = 0; jj < 32; ++jj) {
        const float dsj = __shfl_sync(FULL, ds, jj);
#pragma unroll
        for (int r = 0; r < NC; ++r) acc[r] = fmaf(dsj, Ks[jj][lane + 32 * r], acc[r]);
      }
    }
  }
  if (i < T_) {
    const int64_t p = (int64_t)s.pos0 + i;
#pragma unroll
    for (int r = 0; r < NC / 2; ++r) {
      const int c = lane + 32 * r;
      float cs, sn;
      rope_cos_sin(p, c, HD, s.log2_base, &cs, &sn);
      const float x1 = acc[r] * scale, x2 = acc[r + NC / 2] * scale;
      dq[rowp(i) + c] = from_f<T>(x1 * cs + x2 * sn);
      dq[rowp(i) + c + HD / 2] = from_f<T>(-x1 * sn + x2 * cs);
    }
  }
}

// ---------------------------------------------------------------------------
// a6 backward, dk_bar and dv_bar: warp per key row j, 8 keys per block sharing
// 32-query tiles of [j0, j0+7+W-1]; results in the activation type for the un-mix.
// ---------------------------------------------------------------------------
template <typename T, int HD>
__global__ void __launch_bounds__(256) attn_bwd_dkdv_kernel(
    SwaShape s, const T* __restrict__ qr, const T* __restrict__ kb, const T* __restrict__ vb,
    const T* __restrict__ dout, const float* __restrict__ lse, const float* __restrict__ delta,
    T* __restrict__ dkb, T* __restrict__ dvb, float scale) {
  constexpr int NC = HD / 32;
  __shared__ float Qs[32][HD + 1];
  __shared__ float Gs[32][HD + 1];
  __shared__ float Kr[8][HD];
  __shared__ float Vr[8][HD];
  __shared__ float Ls[32], Dl[32];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.y, b = blockIdx.z;
  const int T_ = s.T, H = s.H, W = s.W;
  const int j0 = blockIdx.x * 8, j = j0 + warp;
  const int lo = j0;
  const int hi = (int)min((int64_t)T_ - 1, (int64_t)j0 + 7 + W - 1);
  auto rowp = [&](int t) { return (((int64_t)b * T_ + t) * H + h) * HD; };
  if (j < T_)
    for (int c = lane; c < HD; c += 32) {
      Kr[warp][c] = to_f(kb[rowp(j) + c]);
      Vr[warp][c] = to_f(vb[rowp(j) + c]);
    }
  float ak[NC], av[NC];
#pragma unroll
  for (int r = 0; r < NC; ++r) ak[r] = av[r] = 0.f;
  for (int q0 = lo; q0 <= hi; q0 += 32) {
    __syncthreads();
    for (int e = threadIdx.x; e < 32 * HD; e += 256) {
      const int ii = e / HD, c = e % HD, i = q0 + ii;
      float qv = 0.f, gv = 0.f;
      if (i <= hi) {
        qv = to_f(qr[rowp(i) + c]);
        gv = to_f(dout[rowp(i) + c]);
      }
      Qs[ii][c] = qv;
      Gs[ii][c] = gv;
    }
    if (threadIdx.x < 32) {
      const int i = q0 + threadIdx.x;
      Ls[threadIdx.x] = i <= hi ? lse[((int64_t)b * H + h) * T_ + i] : 0.f;
      Dl[threadIdx.x] = i <= hi ? delta[((int64_t)b * H + h) * T_ + i] : 0.f;
    }
    __syncthreads();
    if (j < T_) {
      const int i = q0 + lane;
      const bool valid = i <= hi && i >= j && i <= j + W - 1;
      float p = 0.f, ds = 0.f;
      if (valid) {
        float d = 0.f, dp = 0.f;
#pragma unroll 16
        for (int c = 0; c < HD; ++c) {
          d = fmaf(Qs[lane][c], Kr[warp][c], d);
          dp = fmaf(Gs[lane][c], Vr[warp][c], dp);
        }
        p = expf(d * scale - Ls[lane]);
        ds = p * (dp - Dl[lane]);
      }
#pragma unroll 4
      for (int ii = 0; ii < 32; ++ii) {
        const float pi = __shfl_sync(FULL, p, ii);
        const float dsi = __shfl_sync(FULL, ds, ii);
#pragma unroll
        for (int r = 0; r < NC; ++r) {
          av[r] = fmaf(pi, Gs[ii][lane + 32 * r], av[r]);
          ak[r] = fmaf(dsi, Qs[ii][lane + 32 * r], ak[r]);
        }
      }
    }
  }
  if (j < T_) {
#pragma unroll
    for (int r = 0; r < NC; ++r) {
      dkb[rowp(j) + lane + 32 * r] = from_f<T>(ak[r] * scale);
      dvb[rowp(j) + lane + 32 * r] = from_f<T>(av[r]);
    }
  }
}

}  // namespace

#define MAGLEV_DISPATCH(DT, HDV, ...)                                 \
  do {                                                                \
    if ((DT) == 1 && (HDV) == 128) { using T = bf16; constexpr int HD = 128; __VA_ARGS__; } \
    else if ((DT) == 1 && (HDV) == 64) { using T = bf16; constexpr int HD = 64; __VA_ARGS__; } \
    else if ((DT) == 0 && (HDV) == 128) { using T = float; constexpr int HD = 128; __VA_ARGS__; } \
    else if ((DT) == 0 && (HDV) == 64) { using T = float; constexpr int HD = 64; __VA_ARGS__; } \
    else return cudaErrorInvalidValue;                                \
  } while (0)


cudaError_t launch_attn_fwd_simt(const SwaShape& s, const void* q_rot, const void* k_bar,
                                 const void* v_bar, void* out, float* lse, cudaStream_t st) {
  dim3 grid((unsigned)((s.T + 7) / 8), (unsigned)s.H, (unsigned)s.B);
  const float scale = 1.0f / sqrtf((float)s.hd);
  MAGLEV_DISPATCH(s.dtype, s.hd,
                  attn_fwd_kernel<T, HD><<<grid, 256, 0, st>>>(s, (const T*)q_rot, (const T*)k_bar,
                                                               (const T*)v_bar, (T*)out, lse,
                                                               scale));
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd_dq_simt(const SwaShape& s, const void* q_rot, const void* k_bar,
                                    const void* v_bar, const void* dout, const float* lse,
                                    const float* delta, void* dq, cudaStream_t st) {
  dim3 grid((unsigned)((s.T + 7) / 8), (unsigned)s.H, (unsigned)s.B);
  const float scale = 1.0f / sqrtf((float)s.hd);
  MAGLEV_DISPATCH(s.dtype, s.hd,
                  attn_bwd_dq_kernel<T, HD><<<grid, 256, 0, st>>>(
                      s, (const T*)q_rot, (const T*)k_bar, (const T*)v_bar, (const T*)dout, lse,
                      delta, (T*)dq, scale));
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd_dkdv_simt(const SwaShape& s, const void* q_rot, const void* k_bar,
                                      const void* v_bar, const void* dout, const float* lse,
                                      const float* delta, void* dk_bar, void* dv_bar,
                                      cudaStream_t st) {
  dim3 grid((unsigned)((s.T + 7) / 8), (unsigned)s.H, (unsigned)s.B);
  const float scale = 1.0f / sqrtf((float)s.hd);
  MAGLEV_DISPATCH(s.dtype, s.hd,
                  attn_bwd_dkdv_kernel<T, HD><<<grid, 256, 0, st>>>(
                      s, (const T*)q_rot, (const T*)k_bar, (const T*)v_bar, (const T*)dout, lse,
                      delta, (T*)dk_bar, (T*)dv_bar, scale));
  return cudaGetLastError();
}

}  // namespace maglev
