// Element-wise kernels of the injected attention layer, vectorised for HBM:
//   prep   q_rot = RoPE(q); k_bar = g_kl RoPE(k) + g_kr RoPE(RMSNorm_head(R_k));
//          v_bar = g_vl v + g_vr R_v                       (forward, a2-a4)
//   unmix  dq = RoPE^T(dq_rot); dk = g_kl RoPE^T(dk_bar);
//          dR_k = RMSNorm'(R_k, RoPE^T(g_kr dk_bar)); dv = g_vl dv_bar;
//          dR_v = g_vr dv_bar; per-row partial sums of the four gate gradients.
//          dR is written in the activation type, or summed over the layers
//          that share W^rec in fp32 running sums (rounded once, by the last)
//   delta  Delta_i = dout_i . out_i (and zeroes the dq accumulator)
//   gate   dgate[g,h] = sum over rows of the partials * dg/da
// Source: "Maglev: Sliding Recurrent Memory", paper.rainbus.top, 方法步骤详情
// (k_rec = RMSNorm(W_k^rec m'_{t-1}), v_rec = W_v^rec m'_{t-1}, gates
// g = 2 sigmoid(a), both keys RoPE-rotated before the mix) and 前置知识 (RoPE).
//
// A thread owns 8 RoPE pairs of one (b,t,h) row: channels [8u, 8u+8) and
// [hd/2 + 8u, hd/2 + 8u + 8), loaded and stored 16 bytes at a time; hd/16
// threads cover a row and reduce its RMS / gate sums with shuffles.
#include <cmath>

#include "common.cuh"
#include "launchers.h"

namespace maglev {
namespace {

struct V8 {
  float x[8];
};

__device__ __forceinline__ V8 load8(const bf16* p) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
  V8 r;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    r.x[2 * i] = f.x;
    r.x[2 * i + 1] = f.y;
  }
  return r;
}
__device__ __forceinline__ V8 load8(const float* p) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  V8 r;
  r.x[0] = a.x; r.x[1] = a.y; r.x[2] = a.z; r.x[3] = a.w;
  r.x[4] = b.x; r.x[5] = b.y; r.x[6] = b.z; r.x[7] = b.w;
  return r;
}
__device__ __forceinline__ void store8(bf16* p, const V8& v) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v.x[2 * i], v.x[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void store8(float* p, const V8& v) {
  *reinterpret_cast<float4*>(p) = make_float4(v.x[0], v.x[1], v.x[2], v.x[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(v.x[4], v.x[5], v.x[6], v.x[7]);
}
// A 16-byte (bf16) or 32-byte (fp32) load kept in its stored form until used,
// so that a thread can put all its loads in flight before any arithmetic.
template <typename T>
struct Raw8;
template <>
struct Raw8<bf16> {
  uint4 u;
};
template <>
struct Raw8<float> {
  float4 a, b;
};
__device__ __forceinline__ Raw8<bf16> raw8(const bf16* p) { return {*reinterpret_cast<const uint4*>(p)}; }
__device__ __forceinline__ Raw8<float> raw8(const float* p) {
  return {*reinterpret_cast<const float4*>(p), *reinterpret_cast<const float4*>(p + 4)};
}
__device__ __forceinline__ V8 cvt8(const Raw8<bf16>& r) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r.u);
  V8 x;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    x.x[2 * i] = f.x;
    x.x[2 * i + 1] = f.y;
  }
  return x;
}
__device__ __forceinline__ V8 cvt8(const Raw8<float>& r) {
  V8 x;
  x.x[0] = r.a.x; x.x[1] = r.a.y; x.x[2] = r.a.z; x.x[3] = r.a.w;
  x.x[4] = r.b.x; x.x[5] = r.b.y; x.x[6] = r.b.z; x.x[7] = r.b.w;
  return x;
}

// Sum over the TPR lanes that share a row (TPR a power of two <= 32, aligned).
template <int TPR>
__device__ __forceinline__ float row_sum(float x) {
#pragma unroll
  for (int o = TPR / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// cos / sin of position p times inv_freq (double) for 8 pairs, reduced to
// [-pi, pi] in double before the hardware sin / cos (__sincosf: absolute error
// about 2^-21 on [-pi, pi], far below the bf16 and fp32 tolerances of the
// rotated values, and two special-function instructions instead of a full
// range-reduced sincosf per pair).
__device__ __forceinline__ void rope8(int64_t p, const double* inv_freq, int c0, float* cs, float* sn) {
  const double two_pi = 6.283185307179586476925286766559;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    double ang = (double)p * inv_freq[c0 + e];
    ang -= two_pi * rint(ang * 0.15915494309189533577);
    __sincosf((float)ang, &sn[e], &cs[e]);
  }
}

struct RopeTable {
  double inv_freq[64];  // base^(-2c/hd), c < hd/2
};

// One (row, u) item of prep: thread gid of a grid that covers B*T*H rows with
// hd/16 threads each (gid past the end: a thread that only joins the row sums).
template <typename T, int HD>
__device__ __forceinline__ void prep_item(int64_t gid, const SwaShape& s, const RopeTable& rt,
                                          const T* __restrict__ q, const T* __restrict__ k,
                                          const T* __restrict__ v, const T* __restrict__ Rk,
                                          const T* __restrict__ Rv, const float* __restrict__ gates,
                                          T* __restrict__ qr, T* __restrict__ kb, T* __restrict__ vb) {
  constexpr int HALF = HD / 2, TPR = HD / 16;
  const int64_t row = gid / TPR;
  const int u = (int)(gid % TPR);
  const int64_t nrows = (int64_t)s.B * s.T * s.H;
  const bool live = row < nrows;
  const int64_t rr = live ? row : 0;
  const int h = (int)(rr % s.H);
  const int t = (int)((rr / s.H) % s.T);
  const int64_t p = (int64_t)s.pos0 + t;
  const int64_t b1 = rr * HD + 8 * u, b2 = b1 + HALF;
  // every load first; the RoPE angles are computed while they are in flight
  Raw8<T> q1r{}, q2r{}, k1r{}, k2r{}, v1r{}, v2r{}, r1r{}, r2r{}, w1r{}, w2r{};
  if (live) {
    q1r = raw8(q + b1);
    q2r = raw8(q + b2);
    k1r = raw8(k + b1);
    k2r = raw8(k + b2);
    v1r = raw8(v + b1);
    v2r = raw8(v + b2);
    if (s.inject) {
      r1r = raw8(Rk + b1);
      r2r = raw8(Rk + b2);
      w1r = raw8(Rv + b1);
      w2r = raw8(Rv + b2);
    }
  }
  float cs[8], sn[8];
  rope8(p, rt.inv_freq, 8 * u, cs, sn);
  if (live) {
    const V8 q1 = cvt8(q1r), q2 = cvt8(q2r);
    V8 o1, o2;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      o1.x[e] = q1.x[e] * cs[e] - q2.x[e] * sn[e];
      o2.x[e] = q1.x[e] * sn[e] + q2.x[e] * cs[e];
    }
    store8(qr + b1, o1);
    store8(qr + b2, o2);
  }
  V8 k1, k2;
  {
    const V8 a = cvt8(k1r), c = cvt8(k2r);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      k1.x[e] = a.x[e] * cs[e] - c.x[e] * sn[e];
      k2.x[e] = a.x[e] * sn[e] + c.x[e] * cs[e];
    }
  }
  if (!s.inject) {
    if (live) {
      store8(kb + b1, k1);
      store8(kb + b2, k2);
      store8(vb + b1, cvt8(v1r));
      store8(vb + b2, cvt8(v2r));
    }
    return;
  }
  const V8 r1 = cvt8(r1r), r2 = cvt8(r2r);
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) ss += r1.x[e] * r1.x[e] + r2.x[e] * r2.x[e];
  ss = row_sum<TPR>(ss);
  if (!live) return;
  const float rinv = rsqrtf(ss / HD + s.eps);
  const float gkl = gate_value(gates[0 * s.H + h]), gkr = gate_value(gates[1 * s.H + h]);
  const float gvl = gate_value(gates[(s.vg + 0) * s.H + h]), gvr = gate_value(gates[(s.vg + 1) * s.H + h]);
  V8 o1, o2;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float n1 = r1.x[e] * rinv, n2 = r2.x[e] * rinv;
    o1.x[e] = gkl * k1.x[e] + gkr * (n1 * cs[e] - n2 * sn[e]);
    o2.x[e] = gkl * k2.x[e] + gkr * (n1 * sn[e] + n2 * cs[e]);
  }
  store8(kb + b1, o1);
  store8(kb + b2, o2);
  const V8 va = cvt8(v1r), vc = cvt8(v2r), ra = cvt8(w1r), rc = cvt8(w2r);
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    o1.x[e] = gvl * va.x[e] + gvr * ra.x[e];
    o2.x[e] = gvl * vc.x[e] + gvr * rc.x[e];
  }
  store8(vb + b1, o1);
  store8(vb + b2, o2);
}

// Persistent: the grid fills the SMs once and each thread strides over the
// items (the stride is a multiple of the block, so a warp's lanes stay in
// step and its row sums see whole rows).
template <typename T, int HD>
__global__ void __launch_bounds__(256) prep_vec_kernel(SwaShape s, RopeTable rt, const T* __restrict__ q,
                                                       const T* __restrict__ k, const T* __restrict__ v,
                                                       const T* __restrict__ Rk, const T* __restrict__ Rv,
                                                       const float* __restrict__ gates, T* __restrict__ qr,
                                                       T* __restrict__ kb, T* __restrict__ vb) {
  const int64_t total = (int64_t)s.B * s.T * s.H * (HD / 16);
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x; base < total; base += stride)
    prep_item<T, HD>(base + threadIdx.x, s, rt, q, k, v, Rk, Rv, gates, qr, kb, vb);
}

// One (row, u) item of unmix (as prep_item).
template <typename T, int HD>
__device__ __forceinline__ void unmix_item(
    int64_t gid, const SwaShape& s, const RopeTable& rt, const T* __restrict__ dkb, const T* __restrict__ dvb,
    const T* __restrict__ k, const T* __restrict__ v, const T* __restrict__ Rk, const T* __restrict__ Rv,
    const float* __restrict__ gates, T* __restrict__ dk, T* __restrict__ dv, T* __restrict__ dRk,
    T* __restrict__ dRv, float* __restrict__ accRk, float* __restrict__ accRv, int dr_mode,
    float* __restrict__ gpart, const float* __restrict__ dq_acc, T* __restrict__ dq) {
  constexpr int HALF = HD / 2, TPR = HD / 16;
  const int64_t row = gid / TPR;
  const int u = (int)(gid % TPR);
  const int64_t nrows = (int64_t)s.B * s.T * s.H;
  const bool live = row < nrows;
  const int64_t rr = live ? row : 0;
  const int h = (int)(rr % s.H);
  const int64_t bt = rr / s.H;
  const int t = (int)(bt % s.T);
  const int64_t p = (int64_t)s.pos0 + t;
  const int64_t b1 = rr * HD + 8 * u, b2 = b1 + HALF;
  // every load first; the RoPE angles are computed while they are in flight
  Raw8<T> d1r{}, d2r{}, e1r{}, e2r{}, k1r{}, k2r{}, r1r{}, r2r{}, v1r{}, v2r{}, w1r{}, w2r{};
  Raw8<float> pk1{}, pk2{}, pv1{}, pv2{};  // fp32 running sums of dR over earlier layers
  Raw8<float> x1r{}, x2r{};
  const bool read_acc = dr_mode == DR_ADD || dr_mode == DR_LAST;
  const bool with_dq = dq_acc != nullptr;
  if (live) {
    d1r = raw8(dkb + b1);
    d2r = raw8(dkb + b2);
    e1r = raw8(dvb + b1);
    e2r = raw8(dvb + b2);
    if (with_dq) {
      x1r = raw8(dq_acc + b1);
      x2r = raw8(dq_acc + b2);
    }
    if (s.inject) {
      k1r = raw8(k + b1);
      k2r = raw8(k + b2);
      r1r = raw8(Rk + b1);
      r2r = raw8(Rk + b2);
      v1r = raw8(v + b1);
      v2r = raw8(v + b2);
      w1r = raw8(Rv + b1);
      w2r = raw8(Rv + b2);
      if (read_acc) {
        pk1 = raw8(accRk + b1);
        pk2 = raw8(accRk + b2);
        pv1 = raw8(accRv + b1);
        pv2 = raw8(accRv + b2);
      }
    }
  }
  float cs[8], sn[8];
  rope8(p, rt.inv_freq, 8 * u, cs, sn);
  if (live && with_dq) {  // dq = RoPE^T(dq_rot)
    const V8 x1 = cvt8(x1r), x2 = cvt8(x2r);
    V8 o1, o2;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      o1.x[e] = x1.x[e] * cs[e] + x2.x[e] * sn[e];
      o2.x[e] = -x1.x[e] * sn[e] + x2.x[e] * cs[e];
    }
    store8(dq + b1, o1);
    store8(dq + b2, o2);
  }
  const V8 d1 = cvt8(d1r), d2 = cvt8(d2r);
  // RoPE^T of dk_bar
  V8 bk1, bk2;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    bk1.x[e] = d1.x[e] * cs[e] + d2.x[e] * sn[e];
    bk2.x[e] = -d1.x[e] * sn[e] + d2.x[e] * cs[e];
  }
  if (!s.inject) {
    if (live) {
      store8(dk + b1, bk1);
      store8(dk + b2, bk2);
      store8(dv + b1, cvt8(e1r));
      store8(dv + b2, cvt8(e2r));
    }
    return;
  }
  const float gkl = gate_value(gates[0 * s.H + h]), gkr = gate_value(gates[1 * s.H + h]);
  const float gvl = gate_value(gates[(s.vg + 0) * s.H + h]), gvr = gate_value(gates[(s.vg + 1) * s.H + h]);
  const V8 r1 = cvt8(r1r), r2 = cvt8(r2r), k1 = cvt8(k1r), k2 = cvt8(k2r);
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) ss += r1.x[e] * r1.x[e] + r2.x[e] * r2.x[e];
  ss = row_sum<TPR>(ss);
  const float rinv = rsqrtf(ss / HD + s.eps);
  float s_kl = 0.f, s_kr = 0.f, s_ndn = 0.f;
  V8 n1, n2, dn1, dn2;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float kl1 = k1.x[e] * cs[e] - k2.x[e] * sn[e], kl2 = k1.x[e] * sn[e] + k2.x[e] * cs[e];
    s_kl += d1.x[e] * kl1 + d2.x[e] * kl2;
    n1.x[e] = r1.x[e] * rinv;
    n2.x[e] = r2.x[e] * rinv;
    const float kr1 = n1.x[e] * cs[e] - n2.x[e] * sn[e], kr2 = n1.x[e] * sn[e] + n2.x[e] * cs[e];
    s_kr += d1.x[e] * kr1 + d2.x[e] * kr2;
    dn1.x[e] = gkr * bk1.x[e];
    dn2.x[e] = gkr * bk2.x[e];
    s_ndn += n1.x[e] * dn1.x[e] + n2.x[e] * dn2.x[e];
  }
  const float mean_ndn = row_sum<TPR>(s_ndn) / HD;
  const V8 dv1 = cvt8(e1r), dv2 = cvt8(e2r), va = cvt8(v1r), vc = cvt8(v2r), ra = cvt8(w1r), rc = cvt8(w2r);
  float s_vl = 0.f, s_vr = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    s_vl += dv1.x[e] * va.x[e] + dv2.x[e] * vc.x[e];
    s_vr += dv1.x[e] * ra.x[e] + dv2.x[e] * rc.x[e];
  }
  s_kl = row_sum<TPR>(s_kl);
  s_kr = row_sum<TPR>(s_kr);
  s_vl = row_sum<TPR>(s_vl);
  s_vr = row_sum<TPR>(s_vr);
  if (!live) return;
  V8 o1, o2;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    o1.x[e] = gkl * bk1.x[e];
    o2.x[e] = gkl * bk2.x[e];
  }
  store8(dk + b1, o1);
  store8(dk + b2, o2);
  const bool to_acc = dr_mode == DR_FIRST || dr_mode == DR_ADD;
  {
    const V8 a1 = cvt8(pk1), a2 = cvt8(pk2);  // zero unless a running sum is read
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      o1.x[e] = (dn1.x[e] - n1.x[e] * mean_ndn) * rinv + a1.x[e];
      o2.x[e] = (dn2.x[e] - n2.x[e] * mean_ndn) * rinv + a2.x[e];
    }
  }
  if (to_acc) {
    store8(accRk + b1, o1);
    store8(accRk + b2, o2);
  } else {
    store8(dRk + b1, o1);
    store8(dRk + b2, o2);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    o1.x[e] = gvl * dv1.x[e];
    o2.x[e] = gvl * dv2.x[e];
  }
  store8(dv + b1, o1);
  store8(dv + b2, o2);
  {
    const V8 a1 = cvt8(pv1), a2 = cvt8(pv2);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      o1.x[e] = gvr * dv1.x[e] + a1.x[e];
      o2.x[e] = gvr * dv2.x[e] + a2.x[e];
    }
  }
  if (to_acc) {
    store8(accRv + b1, o1);
    store8(accRv + b2, o2);
  } else {
    store8(dRv + b1, o1);
    store8(dRv + b2, o2);
  }
  if (u == 0) {  // column-contiguous partials: gpart[(g*H + h) * rows + bt]
    const int64_t rows = (int64_t)s.B * s.T;
    gpart[(0 * s.H + h) * rows + bt] = s_kl;
    gpart[(1 * s.H + h) * rows + bt] = s_kr;
    gpart[(2 * s.H + h) * rows + bt] = s_vl;
    gpart[(3 * s.H + h) * rows + bt] = s_vr;
  }
}

// Persistent, as prep_vec_kernel; two blocks per SM for bf16 (measured: one
// block at up to 255 registers without spills ran 6% slower, and a version
// whose 128 registers spilled freshly loaded values ran 20% slower).
template <typename T, int HD>
__global__ void __launch_bounds__(256, sizeof(T) == 2 ? 2 : 1) unmix_vec_kernel(
    SwaShape s, RopeTable rt, const T* __restrict__ dkb, const T* __restrict__ dvb,
    const T* __restrict__ k, const T* __restrict__ v, const T* __restrict__ Rk, const T* __restrict__ Rv,
    const float* __restrict__ gates, T* __restrict__ dk, T* __restrict__ dv, T* __restrict__ dRk,
    T* __restrict__ dRv, float* __restrict__ accRk, float* __restrict__ accRv, int dr_mode,
    float* __restrict__ gpart, const float* __restrict__ dq_acc, T* __restrict__ dq) {
  const int64_t total = (int64_t)s.B * s.T * s.H * (HD / 16);
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x; base < total; base += stride)
    unmix_item<T, HD>(base + threadIdx.x, s, rt, dkb, dvb, k, v, Rk, Rv, gates, dk, dv, dRk, dRv, accRk, accRv,
                      dr_mode, gpart, dq_acc, dq);
}

// Delta[b,h,t] = dout . out over hd; also zeroes the fp32 dq accumulator rows.
template <typename T, int HD>
__global__ void __launch_bounds__(256) delta_vec_kernel(SwaShape s, const T* __restrict__ out,
                                                        const T* __restrict__ dout, float* __restrict__ delta,
                                                        float* __restrict__ dq_acc) {
  constexpr int TPR = HD / 16;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t row = gid / TPR;
  const int u = (int)(gid % TPR);
  const int64_t nrows = (int64_t)s.B * s.T * s.H;
  const bool live = row < nrows;
  float acc = 0.f;
  if (live) {
    const int64_t b0 = row * HD + 16 * u;
    const V8 a1 = load8(out + b0), a2 = load8(out + b0 + 8);
    const V8 g1 = load8(dout + b0), g2 = load8(dout + b0 + 8);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc += a1.x[e] * g1.x[e] + a2.x[e] * g2.x[e];
    if (dq_acc) {
      V8 z = {};
      store8(dq_acc + b0, z);
      store8(dq_acc + b0 + 8, z);
    }
  }
  acc = row_sum<TPR>(acc);
  if (live && u == 0) {
    const int h = (int)(row % s.H);
    const int64_t bt = row / s.H;
    const int t = (int)(bt % s.T), b = (int)(bt / s.T);
    delta[((int64_t)b * s.H + h) * s.T + t] = acc;
  }
}

// dgate[col] = sum_r gpart[col * rows + r] * dg/da, fixed reduction order.
// With gates shared by K and V (fold = 2H) the value's partials of the same
// gate, column col + 2H, are added to the key's: dgate is [2, H].
__global__ void __launch_bounds__(512) gate_reduce_vec_kernel(int64_t rows, int fold, const float* __restrict__ gpart,
                                                              const float* __restrict__ gates,
                                                              float* __restrict__ dgate) {
  __shared__ float red[16];
  const int col = blockIdx.x;
  const float* g = gpart + (int64_t)col * rows;
  const float* g2 = fold ? gpart + (int64_t)(col + fold) * rows : nullptr;
  float acc = 0.f;
  for (int64_t r = threadIdx.x; r < rows; r += 512) acc += g2 ? g[r] + g2[r] : g[r];
  acc = warp_sum(acc);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    float x = threadIdx.x < 16 ? red[threadIdx.x] : 0.f;
    x = warp_sum(x);
    if (threadIdx.x == 0) dgate[col] = x * gate_slope(gates[col]);
  }
}

RopeTable rope_table(const SwaShape& s) {
  RopeTable t{};
  const double base = std::exp2(s.log2_base);
  for (int c = 0; c < s.hd / 2 && c < 64; ++c) t.inv_freq[c] = std::pow(base, -2.0 * c / s.hd);
  return t;
}

inline unsigned blocks_for(const SwaShape& s, int tpr) {
  const int64_t threads = (int64_t)s.B * s.T * s.H * tpr;
  return (unsigned)((threads + 255) / 256);
}

// Grid of a persistent element-wise kernel: as many 256-thread blocks as are
// resident on all SMs at once (cached per kernel), or fewer if the items run out.
template <typename Kern>
unsigned persistent_blocks(Kern kern, int& cached_per_sm, const SwaShape& s, int tpr) {
  if (cached_per_sm < 1) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 256, 0) != cudaSuccess || n < 1) n = 1;
    (void)cudaGetLastError();
    cached_per_sm = n;
  }
  const unsigned cap = (unsigned)(num_sms() * cached_per_sm);
  const unsigned want = blocks_for(s, tpr);
  return want < cap ? want : cap;
}
template <typename T, int HD>
unsigned prep_blocks(const SwaShape& s) {
  static int per_sm = 0;
  return persistent_blocks(prep_vec_kernel<T, HD>, per_sm, s, HD / 16);
}
template <typename T, int HD>
unsigned unmix_blocks(const SwaShape& s) {
  static int per_sm = 0;
  return persistent_blocks(unmix_vec_kernel<T, HD>, per_sm, s, HD / 16);
}

}  // namespace

#define MAGLEV_EW_DISPATCH(DT, HDV, ...)                                                        \
  do {                                                                                         \
    if ((DT) == 1 && (HDV) == 128) { using T = bf16; constexpr int HD = 128; __VA_ARGS__; }     \
    else if ((DT) == 1 && (HDV) == 64) { using T = bf16; constexpr int HD = 64; __VA_ARGS__; }  \
    else if ((DT) == 0 && (HDV) == 128) { using T = float; constexpr int HD = 128; __VA_ARGS__; } \
    else if ((DT) == 0 && (HDV) == 64) { using T = float; constexpr int HD = 64; __VA_ARGS__; } \
    else return cudaErrorInvalidValue;                                                         \
  } while (0)

cudaError_t launch_prep(const SwaShape& s, const void* q, const void* k, const void* v, const void* Rk,
                        const void* Rv, const float* gates, void* q_rot, void* k_bar, void* v_bar,
                        cudaStream_t st) {
  const RopeTable rt = rope_table(s);
  MAGLEV_EW_DISPATCH(s.dtype, s.hd,
                     prep_vec_kernel<T, HD><<<prep_blocks<T, HD>(s), 256, 0, st>>>(
                         s, rt, (const T*)q, (const T*)k, (const T*)v, (const T*)Rk, (const T*)Rv, gates,
                         (T*)q_rot, (T*)k_bar, (T*)v_bar));
  return cudaGetLastError();
}

cudaError_t launch_unmix(const SwaShape& s, const void* dk_bar, const void* dv_bar, const void* k,
                         const void* v, const void* Rk, const void* Rv, const float* gates, void* dk, void* dv,
                         void* dRk, void* dRv, float* accRk, float* accRv, int dr_mode, float* gpart,
                         const float* dq_acc, void* dq, cudaStream_t st) {
  const RopeTable rt = rope_table(s);
  MAGLEV_EW_DISPATCH(s.dtype, s.hd,
                     unmix_vec_kernel<T, HD><<<unmix_blocks<T, HD>(s), 256, 0, st>>>(
                         s, rt, (const T*)dk_bar, (const T*)dv_bar, (const T*)k, (const T*)v, (const T*)Rk, (const T*)Rv, gates,
                         (T*)dk, (T*)dv, (T*)dRk, (T*)dRv, accRk, accRv, dr_mode, gpart, dq_acc, (T*)dq));
  return cudaGetLastError();
}

cudaError_t launch_attn_delta(const SwaShape& s, const void* out, const void* dout, float* delta,
                              float* dq_acc, cudaStream_t st) {
  MAGLEV_EW_DISPATCH(s.dtype, s.hd,
                     delta_vec_kernel<T, HD><<<blocks_for(s, HD / 16), 256, 0, st>>>(
                         s, (const T*)out, (const T*)dout, delta, dq_acc));
  return cudaGetLastError();
}

cudaError_t launch_gate_reduce(int64_t rows, int H, int shared_kv, const float* gpart, const float* gates,
                               float* dgate, cudaStream_t st) {
  const int cols = shared_kv ? 2 * H : 4 * H;
  gate_reduce_vec_kernel<<<cols, 512, 0, st>>>(rows, shared_kv ? 2 * H : 0, gpart, gates, dgate);
  return cudaGetLastError();
}

}  // namespace maglev
