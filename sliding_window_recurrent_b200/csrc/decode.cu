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
#include <cooperative_groups.h>

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

// ---------------------------------------------------------------------------
// Ring attention for bf16 rings, one thread-block cluster of NS CTAs per (b,h).
// CTA `rank` owns slots [rank*C, rank*C + C), C <= 128; warp w owns 32 of
// them. Each lane loads 16-byte pieces of its K rows straight into registers
// (all issued before any is used, so many bytes are in flight per SM), forms
// partial dot products reduced over the lanes of a row, then does the same
// for its V rows while the chunk softmax is formed. Four 128-thread CTAs fit
// per SM (128 registers per thread), which overlaps one CTA's loads with
// another's arithmetic. Rank 0 merges the NS partial
// (max, sum, o) triples through distributed shared memory. The CTA whose
// chunk holds slot p mod W writes the new entry to the ring and uses it in
// place of the stale slot.
// ---------------------------------------------------------------------------
constexpr int RING_ROWS = 128;  // slots per CTA at most
constexpr int RING_THREADS = 128;
constexpr int RING_WARPS = RING_THREADS / 32;
constexpr int ROWS_PER_WARP = RING_ROWS / RING_WARPS;

template <int HD>
__global__ void __launch_bounds__(RING_THREADS) decode_ring_kernel(
    DecShape s, int ns, int chunk, const int64_t* __restrict__ pos, const bf16* __restrict__ q,
    const bf16* __restrict__ k, const bf16* __restrict__ v, const bf16* __restrict__ krec,
    const bf16* __restrict__ vrec, const float* __restrict__ gates, bf16* __restrict__ kring,
    bf16* __restrict__ vring, bf16* __restrict__ out, float scale) {
  namespace cg = cooperative_groups;
  constexpr int HALF = HD / 2;
  constexpr int LPR = HD / 8;     // lanes per row (16 B each)
  constexpr int RPW = 32 / LPR;   // rows per warp load step
  constexpr int STEPS = ROWS_PER_WARP / RPW;  // load steps for the warp's rows
  __shared__ float qs[HD], kn[HD], vn[HD];
  __shared__ float sc[RING_ROWS];
  __shared__ float part_o[RING_WARPS][HD];
  __shared__ float stat[2];  // chunk max, chunk sum
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int bh = blockIdx.x / ns, b = bh / s.H, h = bh % s.H;
  const int W = s.W;
  const int64_t p = pos[b];
  const int64_t tok = (int64_t)bh * HD;
  const int64_t ring = (int64_t)bh * W * HD;
  const int r0 = rank * chunk;
  const int rows = max(0, min(W, r0 + chunk) - r0);
  const bool valid_pos = p >= 0;
  const int slot = valid_pos ? (int)(p % W) : -1;
  const int nlive = !valid_pos ? 0 : (p >= W - 1 ? W : (int)p + 1);
  const int live_rows = max(0, min(rows, nlive - r0));
  const int sub = lane / LPR, cl = (lane % LPR) * 8;

  // K rows of this warp -> registers (issued first, consumed after the new entry)
  uint4 kv[STEPS];
#pragma unroll
  for (int i = 0; i < STEPS; ++i) {
    const int r = warp * ROWS_PER_WARP + i * RPW + sub;
    kv[i] = r < live_rows ? __ldg(reinterpret_cast<const uint4*>(kring + ring + (int64_t)(r0 + r) * HD + cl))
                          : make_uint4(0, 0, 0, 0);
  }
  if (tid < HALF && valid_pos) {
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
    kn[c] = to_f(from_f<bf16>(a1));  // the step attends to exactly what it stores
    kn[c + HALF] = to_f(from_f<bf16>(a2));
    vn[c] = to_f(from_f<bf16>(v1));
    vn[c + HALF] = to_f(from_f<bf16>(v2));
  }
  __syncthreads();
  const bool owner = valid_pos && slot >= r0 && slot < r0 + rows;
  if (owner && tid < HD) {
    kring[ring + (int64_t)slot * HD + tid] = from_f<bf16>(kn[tid]);
    vring[ring + (int64_t)slot * HD + tid] = from_f<bf16>(vn[tid]);
  }
  float qv[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) qv[e] = qs[cl + e];
#pragma unroll
  for (int i = 0; i < STEPS; ++i) {
    const int r = warp * ROWS_PER_WARP + i * RPW + sub;
    float d = 0.f;
    if (r0 + r == slot) {
#pragma unroll
      for (int e = 0; e < 8; ++e) d = fmaf(qv[e], kn[cl + e], d);
    } else {
      const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&kv[i]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(hv[e]);
        d = fmaf(qv[2 * e], f.x, d);
        d = fmaf(qv[2 * e + 1], f.y, d);
      }
    }
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
    if ((lane % LPR) == 0) sc[r] = r < live_rows ? d * scale : -INFINITY;
  }
  // V rows of this warp -> registers while the chunk softmax is formed
#pragma unroll
  for (int i = 0; i < STEPS; ++i) {
    const int r = warp * ROWS_PER_WARP + i * RPW + sub;
    kv[i] = r < live_rows ? __ldg(reinterpret_cast<const uint4*>(vring + ring + (int64_t)(r0 + r) * HD + cl))
                          : make_uint4(0, 0, 0, 0);
  }
  __syncthreads();
  if (warp == 0) {
    float mx = -INFINITY;
    for (int r = lane; r < RING_ROWS; r += 32) mx = fmaxf(mx, sc[r]);
    mx = warp_max(mx);
    float l = 0.f;
    for (int r = lane; r < RING_ROWS; r += 32) {
      const float e = mx == -INFINITY ? 0.f : expf(sc[r] - mx);
      sc[r] = e;
      l += e;
    }
    l = warp_sum(l);
    if (lane == 0) {
      stat[0] = mx;
      stat[1] = l;
    }
  }
  __syncthreads();
  float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < STEPS; ++i) {
    const int r = warp * ROWS_PER_WARP + i * RPW + sub;
    const float pr = r < live_rows ? sc[r] : 0.f;
    if (r0 + r == slot) {
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = fmaf(pr, vn[cl + e], o[e]);
    } else {
      const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&kv[i]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(hv[e]);
        o[2 * e] = fmaf(pr, f.x, o[2 * e]);
        o[2 * e + 1] = fmaf(pr, f.y, o[2 * e + 1]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e)
#pragma unroll
    for (int off = 16; off >= LPR; off >>= 1) o[e] += __shfl_xor_sync(0xffffffffu, o[e], off);
  if (lane < LPR) {
#pragma unroll
    for (int e = 0; e < 8; ++e) part_o[warp][cl + e] = o[e];
  }
  __syncthreads();
  if (tid < HD) {
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < RING_WARPS; ++w) acc += part_o[w][tid];
    part_o[0][tid] = acc;
  }
  cluster.sync();
  if (rank == 0 && tid < HD) {
    float M = -INFINITY;
    for (int r = 0; r < ns; ++r) M = fmaxf(M, cluster.map_shared_rank(stat, r)[0]);
    float L = 0.f, O = 0.f;
    for (int r = 0; r < ns; ++r) {
      const float mr = cluster.map_shared_rank(stat, r)[0];
      const float w = mr == -INFINITY ? 0.f : expf(mr - M);
      L += w * cluster.map_shared_rank(stat, r)[1];
      O += w * cluster.map_shared_rank(&part_o[0][0], r)[tid];
    }
    out[tok + tid] = from_f<bf16>(valid_pos ? O / L : 0.f);
  }
  cluster.sync();  // remote reads done before any CTA of the cluster exits
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
                               int64_t limit_us, int* err, cudaStream_t st) {
  const float scale = 1.0f / sqrtf((float)s.hd);
  if (s.dtype == 1 && (s.hd == 128 || s.hd == 64) && s.W <= 8 * RING_ROWS) {
    (void)limit_us;  // the ring kernel has no asynchronous waits
    (void)err;
    const int ns = (s.W + RING_ROWS - 1) / RING_ROWS;
    const int chunk = (s.W + ns - 1) / ns;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(s.B * s.H * ns));
    cfg.blockDim = dim3(RING_THREADS);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)ns;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (s.hd == 128)
      return cudaLaunchKernelEx(&cfg, decode_ring_kernel<128>, s, ns, chunk, pos, (const bf16*)q, (const bf16*)k,
                                (const bf16*)v, (const bf16*)krec, (const bf16*)vrec, gates, (bf16*)k_ring,
                                (bf16*)v_ring, (bf16*)out, scale);
    return cudaLaunchKernelEx(&cfg, decode_ring_kernel<64>, s, ns, chunk, pos, (const bf16*)q, (const bf16*)k,
                              (const bf16*)v, (const bf16*)krec, (const bf16*)vrec, gates, (bf16*)k_ring,
                              (bf16*)v_ring, (bf16*)out, scale);
  }
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
