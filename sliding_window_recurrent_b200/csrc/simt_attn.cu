// CUDA-core kernels of the injected sliding-window attention layer: the
// element-wise injection (RoPE of both keys, RMSNorm of the memory key, gated
// mix), the fp32 attention forward/backward, and the un-mix of the gradients.
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
// a2-a4: q_rot = RoPE(q); k_bar = g_kl RoPE(k) + g_kr RoPE(RMSNorm(R_k));
// v_bar = g_vl v + g_vr R_v. One warp per (b,t,h); lane owns pairs
// (c, c + hd/2) for c = lane + 32 r.
// ---------------------------------------------------------------------------
template <typename T, int HD>
__global__ void __launch_bounds__(256) prep_kernel(SwaShape s, const T* __restrict__ q,
                                                   const T* __restrict__ k,
                                                   const T* __restrict__ v,
                                                   const T* __restrict__ Rk,
                                                   const T* __restrict__ Rv,
                                                   const float* __restrict__ gates,
                                                   T* __restrict__ qr, T* __restrict__ kb,
                                                   T* __restrict__ vb) {
  constexpr int NP = HD / 64, HALF = HD / 2;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t row = (int64_t)blockIdx.x * 8 + warp;
  if (row >= (int64_t)s.B * s.T * s.H) return;
  const int h = (int)(row % s.H);
  const int t = (int)((row / s.H) % s.T);
  const int64_t p = (int64_t)s.pos0 + t;
  const int64_t base = row * HD;
  float cs[NP], sn[NP];
#pragma unroll
  for (int r = 0; r < NP; ++r) rope_cos_sin(p, lane + 32 * r, HD, s.log2_base, &cs[r], &sn[r]);
#pragma unroll
  for (int r = 0; r < NP; ++r) {
    const int c = lane + 32 * r;
    float x1 = to_f(q[base + c]), x2 = to_f(q[base + c + HALF]);
    qr[base + c] = from_f<T>(x1 * cs[r] - x2 * sn[r]);
    qr[base + c + HALF] = from_f<T>(x1 * sn[r] + x2 * cs[r]);
  }
  float kl1[NP], kl2[NP];
#pragma unroll
  for (int r = 0; r < NP; ++r) {
    const int c = lane + 32 * r;
    float x1 = to_f(k[base + c]), x2 = to_f(k[base + c + HALF]);
    kl1[r] = x1 * cs[r] - x2 * sn[r];
    kl2[r] = x1 * sn[r] + x2 * cs[r];
  }
  if (!s.inject) {
#pragma unroll
    for (int r = 0; r < NP; ++r) {
      const int c = lane + 32 * r;
      kb[base + c] = from_f<T>(kl1[r]);
      kb[base + c + HALF] = from_f<T>(kl2[r]);
      vb[base + c] = v[base + c];
      vb[base + c + HALF] = v[base + c + HALF];
    }
    return;
  }
  const float gkl = gate_value(gates[0 * s.H + h]), gkr = gate_value(gates[1 * s.H + h]);
  const float gvl = gate_value(gates[2 * s.H + h]), gvr = gate_value(gates[3 * s.H + h]);
  float r1[NP], r2[NP], ss = 0.f;
#pragma unroll
  for (int r = 0; r < NP; ++r) {
    const int c = lane + 32 * r;
    r1[r] = to_f(Rk[base + c]);
    r2[r] = to_f(Rk[base + c + HALF]);
    ss += r1[r] * r1[r] + r2[r] * r2[r];
  }
  const float rinv = rsqrtf(warp_sum(ss) / HD + s.eps);
#pragma unroll
  for (int r = 0; r < NP; ++r) {
    const int c = lane + 32 * r;
    const float n1 = r1[r] * rinv, n2 = r2[r] * rinv;
    const float kr1 = n1 * cs[r] - n2 * sn[r], kr2 = n1 * sn[r] + n2 * cs[r];
    kb[base + c] = from_f<T>(gkl * kl1[r] + gkr * kr1);
    kb[base + c + HALF] = from_f<T>(gkl * kl2[r] + gkr * kr2);
    vb[base + c] = from_f<T>(gvl * to_f(v[base + c]) + gvr * to_f(Rv[base + c]));
    vb[base + c + HALF] = from_f<T>(gvl * to_f(v[base + c + HALF]) + gvr * to_f(Rv[base + c + HALF]));
  }
}

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

// delta[b,h,i] = sum_c dout[b,i,h,c] * out[b,i,h,c]
template <typename T>
__global__ void __launch_bounds__(256) delta_kernel(SwaShape s, const T* __restrict__ out,
                                                    const T* __restrict__ dout,
                                                    float* __restrict__ delta) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t row = (int64_t)blockIdx.x * 8 + warp;
  if (row >= (int64_t)s.B * s.T * s.H) return;
  const int h = (int)(row % s.H);
  const int64_t bt = row / s.H;
  const int t = (int)(bt % s.T), b = (int)(bt / s.T);
  float acc = 0.f;
  for (int c = lane; c < s.hd; c += 32) acc += to_f(out[row * s.hd + c]) * to_f(dout[row * s.hd + c]);
  acc = warp_sum(acc);
  if (lane == 0) delta[((int64_t)b * s.H + h) * s.T + t] = acc;
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
// 32-query tiles of [j0, j0+7+W-1]; fp32 results for the un-mix.
// ---------------------------------------------------------------------------
template <typename T, int HD>
__global__ void __launch_bounds__(256) attn_bwd_dkdv_kernel(
    SwaShape s, const T* __restrict__ qr, const T* __restrict__ kb, const T* __restrict__ vb,
    const T* __restrict__ dout, const float* __restrict__ lse, const float* __restrict__ delta,
    float* __restrict__ dkb, float* __restrict__ dvb, float scale) {
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
      dkb[rowp(j) + lane + 32 * r] = ak[r] * scale;
      dvb[rowp(j) + lane + 32 * r] = av[r];
    }
  }
}

// ---------------------------------------------------------------------------
// a6 un-mix: from dk_bar, dv_bar to dk, dv, dR_k (through RoPE^T and the
// RMSNorm backward), dR_v, and per-row partial sums of the gate gradients.
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ void store_acc(T* p, int64_t i, float x, int accumulate) {
  if (accumulate) x += to_f(p[i]);
  p[i] = from_f<T>(x);
}

template <typename T, int HD>
__global__ void __launch_bounds__(256) unmix_kernel(
    SwaShape s, const float* __restrict__ dkb, const float* __restrict__ dvb,
    const T* __restrict__ k, const T* __restrict__ v, const T* __restrict__ Rk,
    const T* __restrict__ Rv, const float* __restrict__ gates, T* __restrict__ dk,
    T* __restrict__ dv, T* __restrict__ dRk, T* __restrict__ dRv, int accumulate,
    float* __restrict__ gpart, const float* __restrict__ dq_acc, T* __restrict__ dq) {
  constexpr int NP = HD / 64, HALF = HD / 2;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t row = (int64_t)blockIdx.x * 8 + warp;
  if (row >= (int64_t)s.B * s.T * s.H) return;
  const int h = (int)(row % s.H);
  const int64_t bt = row / s.H;
  const int t = (int)(bt % s.T);
  const int64_t p = (int64_t)s.pos0 + t;
  const int64_t base = row * HD;
  float cs[NP], sn[NP];
#pragma unroll
  for (int r = 0; r < NP; ++r) rope_cos_sin(p, lane + 32 * r, HD, s.log2_base, &cs[r], &sn[r]);
  if (dq_acc) {  // dq = RoPE^T(dq_rot), dq_rot accumulated in fp32 by the attention backward
#pragma unroll
    for (int r = 0; r < NP; ++r) {
      const int c = lane + 32 * r;
      const float x1 = dq_acc[base + c], x2 = dq_acc[base + c + HALF];
      dq[base + c] = from_f<T>(x1 * cs[r] + x2 * sn[r]);
      dq[base + c + HALF] = from_f<T>(-x1 * sn[r] + x2 * cs[r]);
    }
  }
  float d1[NP], d2[NP];  // dk_bar pairs
#pragma unroll
  for (int r = 0; r < NP; ++r) {
    d1[r] = dkb[base + lane + 32 * r];
    d2[r] = dkb[base + lane + 32 * r + HALF];
  }
  if (!s.inject) {
#pragma unroll
    for (int r = 0; r < NP; ++r) {
      const int c = lane + 32 * r;
      dk[base + c] = from_f<T>(d1[r] * cs[r] + d2[r] * sn[r]);
      dk[base + c + HALF] = from_f<T>(-d1[r] * sn[r] + d2[r] * cs[r]);
      dv[base + c] = from_f<T>(dvb[base + c]);
      dv[base + c + HALF] = from_f<T>(dvb[base + c + HALF]);
    }
    return;
  }
  const float gkl = gate_value(gates[0 * s.H + h]), gkr = gate_value(gates[1 * s.H + h]);
  const float gvl = gate_value(gates[2 * s.H + h]), gvr = gate_value(gates[3 * s.H + h]);
  float r1[NP], r2[NP], ss = 0.f;
#pragma unroll
  for (int r = 0; r < NP; ++r) {
    r1[r] = to_f(Rk[base + lane + 32 * r]);
    r2[r] = to_f(Rk[base + lane + 32 * r + HALF]);
    ss += r1[r] * r1[r] + r2[r] * r2[r];
  }
  const float rinv = rsqrtf(warp_sum(ss) / HD + s.eps);
  float s_kl = 0.f, s_kr = 0.f, s_vl = 0.f, s_vr = 0.f, s_ndn = 0.f;
  float n1[NP], n2[NP], dn1[NP], dn2[NP];
#pragma unroll
  for (int r = 0; r < NP; ++r) {
    const int c = lane + 32 * r;
    // local key and its gradient
    const float k1 = to_f(k[base + c]), k2 = to_f(k[base + c + HALF]);
    const float kl1 = k1 * cs[r] - k2 * sn[r], kl2 = k1 * sn[r] + k2 * cs[r];
    s_kl += d1[r] * kl1 + d2[r] * kl2;
    const float bk1 = d1[r] * cs[r] + d2[r] * sn[r];   // RoPE^T dk_bar
    const float bk2 = -d1[r] * sn[r] + d2[r] * cs[r];
    dk[base + c] = from_f<T>(gkl * bk1);
    dk[base + c + HALF] = from_f<T>(gkl * bk2);
    // memory key
    n1[r] = r1[r] * rinv;
    n2[r] = r2[r] * rinv;
    const float kr1 = n1[r] * cs[r] - n2[r] * sn[r], kr2 = n1[r] * sn[r] + n2[r] * cs[r];
    s_kr += d1[r] * kr1 + d2[r] * kr2;
    dn1[r] = gkr * bk1;
    dn2[r] = gkr * bk2;
    s_ndn += n1[r] * dn1[r] + n2[r] * dn2[r];
    // values
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int cc = c + u * HALF;
      const float dvv = dvb[base + cc];
      s_vl += dvv * to_f(v[base + cc]);
      s_vr += dvv * to_f(Rv[base + cc]);
      store_acc(dv, base + cc, gvl * dvv, 0);
      store_acc(dRv, base + cc, gvr * dvv, accumulate);
    }
  }
  const float mean_ndn = warp_sum(s_ndn) / HD;
#pragma unroll
  for (int r = 0; r < NP; ++r) {
    const int c = lane + 32 * r;
    store_acc(dRk, base + c, (dn1[r] - n1[r] * mean_ndn) * rinv, accumulate);
    store_acc(dRk, base + c + HALF, (dn2[r] - n2[r] * mean_ndn) * rinv, accumulate);
  }
  s_kl = warp_sum(s_kl);
  s_kr = warp_sum(s_kr);
  s_vl = warp_sum(s_vl);
  s_vr = warp_sum(s_vr);
  if (lane == 0) {
    float* g = gpart + bt * 4 * s.H;
    g[0 * s.H + h] = s_kl;
    g[1 * s.H + h] = s_kr;
    g[2 * s.H + h] = s_vl;
    g[3 * s.H + h] = s_vr;
  }
}

// dgate[g,h] = (sum over rows of gpart[row][g][h]) * dg/da, in a fixed order.
__global__ void __launch_bounds__(256) gate_reduce_kernel(int rows, int H,
                                                          const float* __restrict__ gpart,
                                                          const float* __restrict__ gates,
                                                          float* __restrict__ dgate) {
  __shared__ float red[256];
  const int col = blockIdx.x;  // g * H + h
  float acc = 0.f;
  for (int r = threadIdx.x; r < rows; r += 256) acc += gpart[(int64_t)r * 4 * H + col];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) dgate[col] = red[0] * gate_slope(gates[col]);
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

static inline unsigned rows_blocks(const SwaShape& s) {
  return (unsigned)(((int64_t)s.B * s.T * s.H + 7) / 8);
}

cudaError_t launch_prep(const SwaShape& s, const void* q, const void* k, const void* v,
                        const void* Rk, const void* Rv, const float* gates, void* q_rot,
                        void* k_bar, void* v_bar, cudaStream_t st) {
  MAGLEV_DISPATCH(s.dtype, s.hd,
                  prep_kernel<T, HD><<<rows_blocks(s), 256, 0, st>>>(
                      s, (const T*)q, (const T*)k, (const T*)v, (const T*)Rk, (const T*)Rv, gates,
                      (T*)q_rot, (T*)k_bar, (T*)v_bar));
  return cudaGetLastError();
}

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

cudaError_t launch_attn_delta(const SwaShape& s, const void* out, const void* dout, float* delta,
                              cudaStream_t st) {
  if (s.dtype == 1)
    delta_kernel<bf16><<<rows_blocks(s), 256, 0, st>>>(s, (const bf16*)out, (const bf16*)dout, delta);
  else
    delta_kernel<float><<<rows_blocks(s), 256, 0, st>>>(s, (const float*)out, (const float*)dout, delta);
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
                                      const float* delta, float* dk_bar, float* dv_bar,
                                      cudaStream_t st) {
  dim3 grid((unsigned)((s.T + 7) / 8), (unsigned)s.H, (unsigned)s.B);
  const float scale = 1.0f / sqrtf((float)s.hd);
  MAGLEV_DISPATCH(s.dtype, s.hd,
                  attn_bwd_dkdv_kernel<T, HD><<<grid, 256, 0, st>>>(
                      s, (const T*)q_rot, (const T*)k_bar, (const T*)v_bar, (const T*)dout, lse,
                      delta, dk_bar, dv_bar, scale));
  return cudaGetLastError();
}

cudaError_t launch_unmix(const SwaShape& s, const float* dk_bar, const float* dv_bar,
                         const void* k, const void* v, const void* Rk, const void* Rv,
                         const float* gates, void* dk, void* dv, void* dRk, void* dRv,
                         int accumulate, float* gpart, const float* dq_acc, void* dq,
                         cudaStream_t st) {
  MAGLEV_DISPATCH(s.dtype, s.hd,
                  unmix_kernel<T, HD><<<rows_blocks(s), 256, 0, st>>>(
                      s, dk_bar, dv_bar, (const T*)k, (const T*)v, (const T*)Rk, (const T*)Rv,
                      gates, (T*)dk, (T*)dv, (T*)dRk, (T*)dRv, accumulate, gpart, dq_acc, (T*)dq));
  return cudaGetLastError();
}

cudaError_t launch_gate_reduce(int rows, int H, const float* gpart, const float* gates,
                               float* dgate, cudaStream_t st) {
  gate_reduce_kernel<<<4 * H, 256, 0, st>>>(rows, H, gpart, gates, dgate);
  return cudaGetLastError();
}

}  // namespace maglev
