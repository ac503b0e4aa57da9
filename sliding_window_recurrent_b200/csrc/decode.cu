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

#include <cmath>

#include "common.cuh"
#include "launchers.h"
#include "tc_common.cuh"

namespace maglev {

cudaError_t make_tmap_bf16_2d_plain(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                                    uint32_t box_inner, uint32_t box_rows);
int num_sms();

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
      const float gvl = gate_value(gates[(s.vg + 0) * s.H + h]), gvr = gate_value(gates[(s.vg + 1) * s.H + h]);
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
// Streaming ring attention for bf16 rings: persistent, one CTA per SM walks
// (b,h) pairs with a stride of the grid and reads each window once. A
// producer warp streams 128-slot chunks of K and V through a ring of
// shared-memory stages with tiled TMA copies (a 2-D view of the ring, boxes of
// 64 channels x 128 slots, alternating K_c, V_c), running on into the next
// pair while the current one finishes; sixteen compute warps each own 8 rows
// of every chunk and keep an online softmax (running max, sum and output,
// log2 units) over their rows, merged at the end of the pair. A prep warp
// forms each pair's rotated q and new entry one pair ahead, into a double
// buffer, so the compute warps never wait on that arithmetic; the new entry
// is used in place of slot p mod W and written to the ring after the pair's
// copies have landed.
// ---------------------------------------------------------------------------
// x[c0 .. c0+N) and x[c0+half .. c0+half+N) of one bf16 row, as floats
// (one 4-byte load per half when N == 2).
template <int N>
__device__ __forceinline__ void load_pairs(const bf16* x, int c0, int half, float* a, float* b) {
  if constexpr (N == 2) {
    const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(x + c0));
    const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(x + c0 + half));
    a[0] = fa.x; a[1] = fa.y;
    b[0] = fb.x; b[1] = fb.y;
  } else {
#pragma unroll
    for (int e = 0; e < N; ++e) {
      a[e] = to_f(x[c0 + e]);
      b[e] = to_f(x[c0 + half + e]);
    }
  }
}

// RoPE frequencies base^(-2c/hd), computed once on the host (double).
struct RopeFreq {
  double inv_freq[64];
};

constexpr int ST_ROWS = 128;          // slots per chunk
constexpr int ST_WARPS = 16;          // compute warps
constexpr int ST_THREADS = 32 * (ST_WARPS + 2);  // + producer warp + prep warp

template <int HD>
struct StreamCfg {
  static constexpr int CH = HD / 64;                         // 64-channel boxes per row
  static constexpr int BOX_BYTES = ST_ROWS * 64 * 2;         // 16 KiB
  static constexpr int CHUNK_BYTES = CH * BOX_BYTES;         // one K or V chunk
  static constexpr int NSTAGE = HD == 128 ? 6 : 12;          // 192 KiB
  static constexpr int OFF_BAR = NSTAGE * CHUNK_BYTES;
  static constexpr size_t SMEM = OFF_BAR + 256;
};

// Each (sequence, head) pair's ring is split into ST_SPLIT work units of
// consecutive 128-slot chunks; units u = pair * ST_SPLIT + part are dealt to
// the persistent CTAs with a stride of the grid, so that every SM streams about
// the same number of chunks (whole pairs left the last of five waves 29% full
// at 64 x 10 pairs on 148 SMs). A unit writes its partial softmax state (max
// and sum in log2 units, unnormalised output) to the workspace and counts
// itself in the pair's counter; the last unit of the pair merges the partials
// into the output and resets the counter to zero, so the workspace is all
// zero again when the call ends. The unit that holds slot p mod W also writes
// the new entry to the ring.
constexpr int ST_SPLIT = 2;  // the most units per pair (workspace size)

template <int HD>
__global__ void __launch_bounds__(ST_THREADS, 1) decode_stream_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, DecShape s,
    const int64_t* __restrict__ pos, const bf16* __restrict__ q, const bf16* __restrict__ k,
    const bf16* __restrict__ v, const bf16* __restrict__ krec, const bf16* __restrict__ vrec,
    const float* __restrict__ gates, bf16* __restrict__ kring, bf16* __restrict__ vring,
    float* __restrict__ part, int* __restrict__ counters, bf16* __restrict__ out, int split, int cpu_chunks,
    float scale_log2, int64_t limit_ns, int* err, const __grid_constant__ RopeFreq rf) {
  using C = StreamCfg<HD>;
  constexpr int HALF = HD / 2;
  constexpr int LPR = HD / 8;                // lanes per row (16 B each)
  constexpr int RPS = 32 / LPR;              // rows per warp step
  constexpr int WROWS = ST_ROWS / ST_WARPS;  // rows of a chunk per warp
  constexpr int STEPS = WROWS / RPS;
  constexpr int CT = 32 * ST_WARPS;          // compute threads
  extern __shared__ __align__(1024) uint8_t dsm[];
  uint64_t* full = reinterpret_cast<uint64_t*>(dsm + C::OFF_BAR);   // [NSTAGE]
  uint64_t* empty = full + C::NSTAGE;                                 // [NSTAGE]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + C::NSTAGE);
  uint64_t* prep_full = empty + C::NSTAGE + 1;  // [2]
  uint64_t* prep_empty = prep_full + 2;         // [2]
  __shared__ float qs[2][HD], kn[2][HD], vn[2][HD];  // per pair, double-buffered
  __shared__ long long ppos[2];
  __shared__ float wm[ST_WARPS], wl[ST_WARPS];
  __shared__ float wo[ST_WARPS][HD];
  __shared__ int last_unit;  // this unit completes its pair
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int W = s.W;
  const int nunits = s.B * s.H * split;
  const tc::Abort ab{abort_flag, err, limit_ns};
  // live slots of pair bh: positions max(0, p-W+1)..p
  auto live_of = [&](int bh) -> int {
    const int64_t p = pos[bh / s.H];
    return p < 0 ? 0 : (p >= W - 1 ? W : (int)p + 1);
  };
  // chunks [c0, c1) of unit u (cpu_chunks chunks per unit; may be empty)
  auto range_of = [&](int u, int nchunks, int* c0, int* c1) {
    *c0 = min(nchunks, (u % split) * cpu_chunks);
    *c1 = min(nchunks, *c0 + cpu_chunks);
  };

  if (tid == 0) {
    for (int i = 0; i < C::NSTAGE; ++i) {
      tc::mbar_init(&full[i], 1);
      tc::mbar_init(&empty[i], ST_WARPS);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&prep_full[i], 32);
      tc::mbar_init(&prep_empty[i], 1);
    }
    *abort_flag = 0;
    tc::fence_mbar_init();
    tc::tma_prefetch_desc(&tmK);
    tc::tma_prefetch_desc(&tmV);
  }
  __syncthreads();

  if (warp == ST_WARPS) {
    // ------------------------------------------------------------ producer
    // streams K_c, V_c of every chunk of every pair of this CTA, in order
    if (lane == 0) {
      uint32_t armed = 0, par = 0;
      int L = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
        const int bh = u / split;
        int cb, ce;
        range_of(u, (live_of(bh) + ST_ROWS - 1) / ST_ROWS, &cb, &ce);
        for (int j = 2 * cb; j < 2 * ce; ++j, ++L) {  // j = 2c: K_c, j = 2c+1: V_c
          const int st = L % C::NSTAGE;
          const uint32_t ph = (uint32_t)(L / C::NSTAGE) & 1u;
          if (!MAGLEV_CHECK(err, (j >> 1) * ST_ROWS < W && bh < s.B * s.H)) {  // every role stops
            *abort_flag = 1;
            ok = false;
            break;
          }
          if (!tc::mbar_wait(&empty[st], ph ^ 1u, ab)) {
            ok = false;
            break;
          }
          tc::mbar_arrive_expect_tx(&full[st], C::CHUNK_BYTES);
          armed |= 1u << st;
          par = (par & ~(1u << st)) | (ph << st);
          const int row = bh * W + (j >> 1) * ST_ROWS;  // rows past the tensor arrive as zeros
#pragma unroll
          for (int c = 0; c < C::CH; ++c)
            tc::tma_load_2d(dsm + st * C::CHUNK_BYTES + c * C::BOX_BYTES, (j & 1) ? &tmV : &tmK, &full[st], 64 * c,
                            row);
        }
      }
      // copies in flight land before the CTA leaves (needed only after an abort)
      for (int st = 0; st < C::NSTAGE; ++st)
        if (armed & (1u << st)) tc::mbar_drain(&full[st], (par >> st) & 1u, tc::DRAIN_LIMIT_NS);
    }
    return;  // takes no part in the compute warps' barriers
  }
  if (warp == ST_WARPS + 1) {
    // ------------------------------------------------------------ prep
    // pair i's position, q rotated and scaled to log2 units, and its new K/V
    // entry (RoPE of the local key, gated mix), into buffer i&1 once the
    // compute warps are done with pair i-2
    int i = 0;
    for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++i) {
      const int bh = u / split;
      const int buf = i & 1;
      if (i >= 2 && !tc::warp_wait(&prep_empty[buf], (uint32_t)((i - 2) >> 1) & 1u, ab)) break;
      const int h = bh % s.H;
      const int64_t tok = (int64_t)bh * HD;
      // every load of the pair at once (none depends on p): at kernel start they
      // queue behind the ring fill of every SM, so one round trip, not three
      constexpr int NPL = HALF / 32;  // channel pairs per lane (2 or 1), contiguous
      const int c0 = lane * NPL;
      float qa[NPL], qb[NPL], ka[NPL], kb[NPL], va[NPL], vb[NPL], ra[NPL], rb[NPL], wa[NPL], wb[NPL];
      load_pairs<NPL>(q + tok, c0, HALF, qa, qb);
      load_pairs<NPL>(k + tok, c0, HALF, ka, kb);
      load_pairs<NPL>(v + tok, c0, HALF, va, vb);
      float ga = 0.f, gb = 0.f, gc = 0.f, gd = 0.f;
      if (s.inject) {  // the memory inputs and gates may be NULL without injection
        load_pairs<NPL>(krec + tok, c0, HALF, ra, rb);
        load_pairs<NPL>(vrec + tok, c0, HALF, wa, wb);
        ga = gates[0 * s.H + h];
        gb = gates[1 * s.H + h];
        gc = gates[(s.vg + 0) * s.H + h];
        gd = gates[(s.vg + 1) * s.H + h];
      }
      const int64_t p = pos[bh / s.H];
      if (p >= 0) {
        const float gkl = gate_value(ga), gkr = gate_value(gb), gvl = gate_value(gc), gvr = gate_value(gd);
#pragma unroll
        for (int e = 0; e < NPL; ++e) {
          const int c = c0 + e;
          // angle p * theta_c reduced to [-pi, pi] in double before the float sincos
          double ang = (double)p * rf.inv_freq[c];
          ang -= 6.283185307179586476925286766559 * rint(ang * 0.15915494309189533577);
          float cs, sn;
          sincosf((float)ang, &sn, &cs);
          qs[buf][c] = (qa[e] * cs - qb[e] * sn) * scale_log2;  // scores come out in log2 units
          qs[buf][c + HALF] = (qa[e] * sn + qb[e] * cs) * scale_log2;
          float a1 = ka[e] * cs - kb[e] * sn, a2 = ka[e] * sn + kb[e] * cs;
          float v1 = va[e], v2 = vb[e];
          if (s.inject) {
            a1 = gkl * a1 + gkr * ra[e];
            a2 = gkl * a2 + gkr * rb[e];
            v1 = gvl * v1 + gvr * wa[e];
            v2 = gvl * v2 + gvr * wb[e];
          }
          kn[buf][c] = to_f(from_f<bf16>(a1));  // the step attends to exactly what it stores
          kn[buf][c + HALF] = to_f(from_f<bf16>(a2));
          vn[buf][c] = to_f(from_f<bf16>(v1));
          vn[buf][c + HALF] = to_f(from_f<bf16>(v2));
        }
      }
      if (lane == 0) ppos[buf] = p;
      tc::mbar_arrive(&prep_full[buf]);  // each lane releases its own writes
    }
    return;  // takes no part in the compute warps' barriers
  }
  // ------------------------------------------------------------ compute warps
  const int sub = lane / LPR, cl = (lane % LPR) * 8;
  const int boff = (cl / 64) * C::BOX_BYTES + (cl % 64) * 2;  // byte offset of this lane's piece in a row
  int L = 0;
  bool ok = true;
  int i = 0;
  for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++i) {
    const int bh = u / split;
    const int buf = i & 1;
    // the pair's q and new entry are ready (after an abort the unit is skipped)
    ok = ok && tc::mbar_wait(&prep_full[buf], (uint32_t)(i >> 1) & 1u, ab);
    const int64_t p = ok ? (int64_t)ppos[buf] : -1;
    const int64_t ring = (int64_t)bh * W * HD;
    const bool valid_pos = p >= 0;
    const int slot = valid_pos ? (int)(p % W) : -1;
    const int nlive = valid_pos ? (p >= W - 1 ? W : (int)p + 1) : 0;
    int cb, ce;  // this unit's chunks, as the producer counts them
    range_of(u, (nlive + ST_ROWS - 1) / ST_ROWS, &cb, &ce);
    const float* kn_b = kn[buf];
    const float* vn_b = vn[buf];
    float qv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) qv[e] = qs[buf][cl + e];
    float m = -INFINITY, l = 0.f;  // log2 units, over the rows this lane-group has seen
    float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int c = cb; c < ce; ++c, L += 2) {
      if (!ok) continue;  // after an abort the remaining chunks are skipped
      const int sk = L % C::NSTAGE, sv = (L + 1) % C::NSTAGE;
      if (!tc::mbar_wait(&full[sk], (uint32_t)(L / C::NSTAGE) & 1u, ab)) {
        ok = false;
        continue;
      }
      const uint8_t* kc = dsm + sk * C::CHUNK_BYTES + boff;
      float sc[STEPS];
      float cmax = -INFINITY;
#pragma unroll
      for (int i = 0; i < STEPS; ++i) {
        const int r = warp * WROWS + i * RPS + sub;  // row within the chunk
        const int gr = c * ST_ROWS + r;              // ring slot
        float d0 = 0.f, d1 = 0.f;
        if (gr == slot) {
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            d0 = fmaf(qv[e], kn_b[cl + e], d0);
            d1 = fmaf(qv[e + 1], kn_b[cl + e + 1], d1);
          }
        } else {
          const uint4 u = *reinterpret_cast<const uint4*>(kc + r * 128);
          const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(hv[e]);
            d0 = fmaf(qv[2 * e], f.x, d0);
            d1 = fmaf(qv[2 * e + 1], f.y, d1);
          }
        }
        float d = d0 + d1;
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
        sc[i] = gr < nlive ? d : -INFINITY;
        cmax = fmaxf(cmax, sc[i]);
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&empty[sk]);  // K_c read by this warp
      // online softmax over this lane-group's rows (log2 units)
      const float mn = fmaxf(m, cmax);
      const float alpha = (m == -INFINITY) ? 0.f : tc::ex2_fast(m - mn);
      const float nm = mn == -INFINITY ? 0.f : -mn;
      float pr[STEPS];
      float ps = 0.f;
#pragma unroll
      for (int i = 0; i < STEPS; ++i) {
        pr[i] = tc::ex2_fast(sc[i] + nm);  // -inf gives 0
        ps += pr[i];
      }
      l = l * alpha + ps;
      m = mn;
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] *= alpha;
      if (!tc::mbar_wait(&full[sv], (uint32_t)((L + 1) / C::NSTAGE) & 1u, ab)) {
        ok = false;
        continue;
      }
      const uint8_t* vc = dsm + sv * C::CHUNK_BYTES + boff;
#pragma unroll
      for (int i = 0; i < STEPS; ++i) {
        const int r = warp * WROWS + i * RPS + sub;
        const int gr = c * ST_ROWS + r;
        if (gr == slot) {
#pragma unroll
          for (int e = 0; e < 8; ++e) o[e] = fmaf(pr[i], vn_b[cl + e], o[e]);
        } else if (gr < nlive) {  // dead slots may hold anything, NaN included
          const uint4 u = *reinterpret_cast<const uint4*>(vc + r * 128);
          const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(hv[e]);
            o[2 * e] = fmaf(pr[i], f.x, o[2 * e]);
            o[2 * e + 1] = fmaf(pr[i], f.y, o[2 * e + 1]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&empty[sv]);  // V_c read by this warp
    }
    // merge the RPS lane-groups of the warp (same channels, different rows)
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
      const float l2 = __shfl_xor_sync(0xffffffffu, l, off);
      const float mn = fmaxf(m, m2);
      const float a1 = m == -INFINITY ? 0.f : tc::ex2_fast(m - mn);
      const float a2 = m2 == -INFINITY ? 0.f : tc::ex2_fast(m2 - mn);
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = o[e] * a1 + __shfl_xor_sync(0xffffffffu, o[e], off) * a2;
      l = l * a1 + l2 * a2;
      m = mn;
    }
    if (lane < LPR) {
#pragma unroll
      for (int e = 0; e < 8; ++e) wo[warp][cl + e] = o[e];
    }
    if (lane == 0) {
      wm[warp] = ok ? m : -INFINITY;
      wl[warp] = ok ? l : 0.f;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(CT) : "memory");  // every warp's partial is in
    // merge the warps into the unit's partial; the unit that holds the slot
    // writes the new entry now that its copies have landed
    if (tid < HD) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < ST_WARPS; ++w) M = fmaxf(M, wm[w]);
      float Ls = 0.f, O = 0.f;
#pragma unroll
      for (int w = 0; w < ST_WARPS; ++w) {
        const float a = wm[w] == -INFINITY ? 0.f : tc::ex2_fast(wm[w] - M);
        Ls += a * wl[w];
        O += a * wo[w][tid];
      }
      if (split == 1) {  // the unit is the whole pair
        out[(int64_t)bh * HD + tid] = from_f<bf16>(valid_pos && Ls > 0.f ? O / Ls : 0.f);
      } else {
        float* pu = part + (int64_t)u * (HD + 2);
        pu[2 + tid] = O;
        if (tid == 0) {
          pu[0] = M;
          pu[1] = Ls;
        }
      }
      const bool has_slot = valid_pos && slot / ST_ROWS >= cb && slot / ST_ROWS < ce;
      if (has_slot && ok && MAGLEV_CHECK(err, slot >= 0 && slot < W && bh < s.B * s.H)) {
        kring[ring + (int64_t)slot * HD + tid] = from_f<bf16>(kn_b[tid]);
        vring[ring + (int64_t)slot * HD + tid] = from_f<bf16>(vn_b[tid]);
      }
    }
    if (split > 1) {
    asm volatile("bar.sync 1, %0;" ::"n"(CT) : "memory");  // the unit's partial is written
    if (tid == 0) {
      // release: the fence is cumulative, so it orders the CTA's partial (seen
      // through the barrier) before the count; acquire on the last unit's side
      __threadfence();
      last_unit = atomicAdd(&counters[bh], 1) == split - 1;
      if (last_unit) __threadfence();
    }
    asm volatile("bar.sync 1, %0;" ::"n"(CT) : "memory");
    if (last_unit) {  // every unit of the pair has counted itself: merge the partials
      if (tid < HD) {
        const float* pp = part + (int64_t)bh * split * (HD + 2);
        float M = -INFINITY;
#pragma unroll
        for (int k2 = 0; k2 < split; ++k2) M = fmaxf(M, __ldcg(pp + k2 * (HD + 2)));
        float Ls = 0.f, O = 0.f;
#pragma unroll
        for (int k2 = 0; k2 < split; ++k2) {
          const float m2 = __ldcg(pp + k2 * (HD + 2));
          const float a = m2 == -INFINITY ? 0.f : tc::ex2_fast(m2 - M);
          Ls += a * __ldcg(pp + k2 * (HD + 2) + 1);
          O += a * __ldcg(pp + k2 * (HD + 2) + 2 + tid);
        }
        out[(int64_t)bh * HD + tid] = from_f<bf16>(valid_pos && Ls > 0.f ? O / Ls : 0.f);
      }
      if (tid == 0) counters[bh] = 0;  // ready for the next call
    }
    }  // split > 1
    asm volatile("bar.sync 1, %0;" ::"n"(CT) : "memory");  // q, new entry, partials free again
    if (tid == 0) tc::mbar_arrive(&prep_empty[buf]);           // the prep warp may refill buffer buf
  }
}

}  // namespace

// Work units per (sequence, head) pair.
static int decode_split() { return 1; }

// [B*H*ST_SPLIT][hd + 2] fp32 partials, then [B*H] int pair counters.
static size_t decode_part_bytes(const DecShape& s) {
  return ((size_t)s.B * s.H * ST_SPLIT * (s.hd + 2) * sizeof(float) + 255) & ~(size_t)255;
}
size_t decode_workspace_bytes(const DecShape& s) {
  if (s.dtype != 1 || (s.hd != 128 && s.hd != 64)) return 0;
  return decode_part_bytes(s) + (size_t)s.B * s.H * sizeof(int);
}

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
                               const float* gates, void* k_ring, void* v_ring, void* out, void* workspace,
                               int64_t limit_us, int* err, cudaStream_t st) {
  const float scale = 1.0f / sqrtf((float)s.hd);
  if (s.dtype == 1 && (s.hd == 128 || s.hd == 64)) {
    const int64_t limit_ns = (limit_us > 0 ? limit_us : DEFAULT_SPIN_LIMIT) * 1000;
    if (s.B * s.H == 0) return cudaSuccess;
    // the rings as 2-D [B*H*W, hd] tensors, boxes of 64 channels x 128 slots
    CUtensorMap tk, tv;
    const uint64_t nrows = (uint64_t)s.B * s.H * s.W;
    cudaError_t te = make_tmap_bf16_2d_plain(&tk, k_ring, (uint64_t)s.hd, nrows, 64, ST_ROWS);
    if (te != cudaSuccess) return te;
    te = make_tmap_bf16_2d_plain(&tv, v_ring, (uint64_t)s.hd, nrows, 64, ST_ROWS);
    if (te != cudaSuccess) return te;
    const float scale_log2 = 1.4426950408889634f * scale;
    RopeFreq rf{};
    const double base = std::exp2(s.log2_base);
    for (int c = 0; c < s.hd / 2 && c < 64; ++c) rf.inv_freq[c] = std::pow(base, -2.0 * c / s.hd);
    const int split = decode_split();
    const int nunits = s.B * s.H * split;
    const unsigned grid = (unsigned)(nunits < num_sms() ? nunits : num_sms());  // persistent
    const int cpu_chunks = ((s.W + ST_ROWS - 1) / ST_ROWS + split - 1) / split;
    float* part = static_cast<float*>(workspace);
    int* counters = reinterpret_cast<int*>(static_cast<char*>(workspace) + decode_part_bytes(s));
    if (s.hd == 128) {
      auto kern = decode_stream_kernel<128>;
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)StreamCfg<128>::SMEM);
      if (e != cudaSuccess) return e;
      kern<<<grid, ST_THREADS, StreamCfg<128>::SMEM, st>>>(tk, tv, s, pos, (const bf16*)q, (const bf16*)k,
                                                               (const bf16*)v, (const bf16*)krec, (const bf16*)vrec,
                                                               gates, (bf16*)k_ring, (bf16*)v_ring, part, counters,
                                                               (bf16*)out, split, cpu_chunks, scale_log2, limit_ns, err, rf);
    } else {
      auto kern = decode_stream_kernel<64>;
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)StreamCfg<64>::SMEM);
      if (e != cudaSuccess) return e;
      kern<<<grid, ST_THREADS, StreamCfg<64>::SMEM, st>>>(tk, tv, s, pos, (const bf16*)q, (const bf16*)k,
                                                              (const bf16*)v, (const bf16*)krec, (const bf16*)vrec,
                                                              gates, (bf16*)k_ring, (bf16*)v_ring, part, counters,
                                                              (bf16*)out, split, cpu_chunks, scale_log2, limit_ns, err, rf);
    }
    return cudaGetLastError();
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
