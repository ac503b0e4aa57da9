// a8: recurrent decode over a rolling W-entry K/V ring.
//
// Source: "Maglev: Sliding Recurrent Memory", paper.rainbus.top, 研究动机 (at
// inference m_t = P(x_{t-W+1:t}, M_{t-1}); the token window and the memory window
// stay fixed) and 前置知识 (the cache equals that of plain SWA: the memory is
// carried inside the existing K/V entries); gist.science, Inferentiemechanisme
// (injection through the learned projections and gates, no extra slot).
//
// Ring layout [B,H,W,hd]: the entry of absolute position j lives in slot j mod W,
// stored after RoPE and after the gated mix. A step writes slot p mod W, then
// attends over the live slots (positions max(0, p-W+1)..p).
#include "common.cuh"
#include "launchers.h"

namespace maglev {
namespace {

// In place: x[b,h,:] <- RoPE_{pos[b]}(RMSNorm(x[b,h,:])); one warp per (b,h).
template <typename T, int HD>
__global__ void __launch_bounds__(256) rmsnorm_rope_rows_kernel(DecShape s,
                                                                const int64_t* __restrict__ pos,
                                                                T* __restrict__ x) {
  constexpr int NP = HD / 64, HALF = HD / 2;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t row = (int64_t)blockIdx.x * 8 + warp;
  if (row >= (int64_t)s.B * s.H) return;
  const int b = (int)(row / s.H);
  const int64_t p = pos[b] < 0 ? 0 : pos[b];
  const int64_t base = row * HD;
  float x1[NP], x2[NP], ss = 0.f;
#pragma unroll
  for (int r = 0; r < NP; ++r) {
    x1[r] = to_f(x[base + lane + 32 * r]);
    x2[r] = to_f(x[base + lane + 32 * r + HALF]);
    ss += x1[r] * x1[r] + x2[r] * x2[r];
  }
  const float rinv = rsqrtf(warp_sum(ss) / HD + s.eps);
#pragma unroll
  for (int r = 0; r < NP; ++r) {
    const int c = lane + 32 * r;
    float cs, sn;
    rope_cos_sin(p, c, HD, s.log2_base, &cs, &sn);
    const float n1 = x1[r] * rinv, n2 = x2[r] * rinv;
    x[base + c] = from_f<T>(n1 * cs - n2 * sn);
    x[base + c + HALF] = from_f<T>(n1 * sn + n2 * cs);
  }
}

// One block per (b,h): build the new entry, write it to slot p mod W, then
// softmax-attend q_rot over the live slots. Scores live in shared memory.
template <typename T, int HD>
__global__ void __launch_bounds__(256) decode_step_kernel(
    DecShape s, const int64_t* __restrict__ pos, const T* __restrict__ q, const T* __restrict__ k,
    const T* __restrict__ v, const T* __restrict__ krec, const T* __restrict__ vrec,
    const float* __restrict__ gates, T* __restrict__ kring, T* __restrict__ vring,
    T* __restrict__ out, float scale) {
  constexpr int HALF = HD / 2, PARTS = 256 / HD;
  extern __shared__ float sc[];  // [W]
  __shared__ float qs[HD], kn[HD], vn[HD];
  __shared__ float red[32];
  __shared__ float pacc[PARTS][HD];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int bh = blockIdx.x, b = bh / s.H, h = bh % s.H;
  const int W = s.W;
  const int64_t p = pos[b];
  const int64_t tok = (int64_t)bh * HD;
  if (p < 0) {  // invalid position: the ring is left untouched, the output is zero
    if (tid < HD) out[tok + tid] = from_f<T>(0.f);
    return;
  }
  const int slot = (int)(p % W);
  const int nlive = p >= W - 1 ? W : (int)p + 1;
  const int64_t ring = (int64_t)bh * W * HD;
  if (tid < HALF) {
    const int c = tid;
    float cs, sn;
    rope_cos_sin(p, c, HD, s.log2_base, &cs, &sn);
    const float q1 = to_f(q[tok + c]), q2 = to_f(q[tok + c + HALF]);
    qs[c] = q1 * cs - q2 * sn;
    qs[c + HALF] = q1 * sn + q2 * cs;
    const float k1 = to_f(k[tok + c]), k2 = to_f(k[tok + c + HALF]);
    float a1 = k1 * cs - k2 * sn, a2 = k1 * sn + k2 * cs;
    float v1 = to_f(v[tok + c]), v2 = to_f(v[tok + c + HALF]);
    if (s.inject) {
      const float gkl = gate_value(gates[0 * s.H + h]), gkr = gate_value(gates[1 * s.H + h]);
      const float gvl = gate_value(gates[2 * s.H + h]), gvr = gate_value(gates[3 * s.H + h]);
      a1 = gkl * a1 + gkr * to_f(krec[tok + c]);
      a2 = gkl * a2 + gkr * to_f(krec[tok + c + HALF]);
      v1 = gvl * v1 + gvr * to_f(vrec[tok + c]);
      v2 = gvl * v2 + gvr * to_f(vrec[tok + c + HALF]);
    }
    // the step attends to exactly the values it stores in the ring
    kn[c] = to_f(from_f<T>(a1));
    kn[c + HALF] = to_f(from_f<T>(a2));
    vn[c] = to_f(from_f<T>(v1));
    vn[c + HALF] = to_f(from_f<T>(v2));
  }
  __syncthreads();
  if (tid < HD) {
    kring[ring + (int64_t)slot * HD + tid] = from_f<T>(kn[tid]);
    vring[ring + (int64_t)slot * HD + tid] = from_f<T>(vn[tid]);
  }
  for (int j = warp; j < W; j += 8) {
    float d = -INFINITY;
    if (j < nlive) {
      float acc = 0.f;
      if (j == slot) {
        for (int c = lane; c < HD; c += 32) acc = fmaf(qs[c], kn[c], acc);
      } else {
        for (int c = lane; c < HD; c += 32) acc = fmaf(qs[c], to_f(kring[ring + (int64_t)j * HD + c]), acc);
      }
      d = warp_sum(acc) * scale;
    }
    if (lane == 0) sc[j] = d;
  }
  __syncthreads();
  float mx = -INFINITY;
  for (int j = tid; j < nlive; j += 256) mx = fmaxf(mx, sc[j]);
  mx = warp_max(mx);
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  mx = red[0];
  for (int w = 1; w < 8; ++w) mx = fmaxf(mx, red[w]);
  __syncthreads();
  float l = 0.f;
  for (int j = tid; j < nlive; j += 256) {
    const float e = expf(sc[j] - mx);
    sc[j] = e;
    l += e;
  }
  l = warp_sum(l);
  if (lane == 0) red[warp] = l;
  __syncthreads();
  l = 0.f;
  for (int w = 0; w < 8; ++w) l += red[w];
  const int c = tid % HD, part = tid / HD;
  float acc = 0.f;
  for (int j = part; j < nlive; j += PARTS) {
    const float vv = j == slot ? vn[c] : to_f(vring[ring + (int64_t)j * HD + c]);
    acc = fmaf(sc[j], vv, acc);
  }
  pacc[part][c] = acc;
  __syncthreads();
  if (tid < HD) {
    float o = 0.f;
    for (int u = 0; u < PARTS; ++u) o += pacc[u][tid];
    out[tok + tid] = from_f<T>(o / l);
  }
}

}  // namespace

#define MAGLEV_DISPATCH2(DT, HDV, ...)                                                        \
  do {                                                                                       \
    if ((DT) == 1 && (HDV) == 128) { using T = bf16; constexpr int HD = 128; __VA_ARGS__; }   \
    else if ((DT) == 1 && (HDV) == 64) { using T = bf16; constexpr int HD = 64; __VA_ARGS__; } \
    else if ((DT) == 0 && (HDV) == 128) { using T = float; constexpr int HD = 128; __VA_ARGS__; } \
    else if ((DT) == 0 && (HDV) == 64) { using T = float; constexpr int HD = 64; __VA_ARGS__; } \
    else return cudaErrorInvalidValue;                                                       \
  } while (0)

cudaError_t launch_rmsnorm_rope_rows(const DecShape& s, const int64_t* pos, void* x,
                                     cudaStream_t st) {
  const unsigned blocks = (unsigned)(((int64_t)s.B * s.H + 7) / 8);
  MAGLEV_DISPATCH2(s.dtype, s.hd,
                   rmsnorm_rope_rows_kernel<T, HD><<<blocks, 256, 0, st>>>(s, pos, (T*)x));
  return cudaGetLastError();
}

cudaError_t launch_decode_step(const DecShape& s, const int64_t* pos, const void* q, const void* k,
                               const void* v, const void* krec, const void* vrec,
                               const float* gates, void* k_ring, void* v_ring, void* out,
                               cudaStream_t st) {
  const float scale = 1.0f / sqrtf((float)s.hd);
  const size_t smem = (size_t)s.W * sizeof(float);
  MAGLEV_DISPATCH2(s.dtype, s.hd, {
    if (smem > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(decode_step_kernel<T, HD>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    decode_step_kernel<T, HD><<<s.B * s.H, 256, smem, st>>>(
        s, pos, (const T*)q, (const T*)k, (const T*)v, (const T*)krec, (const T*)vrec, gates,
        (T*)k_ring, (T*)v_ring, (T*)out, scale);
  });
  return cudaGetLastError();
}

}  // namespace maglev
