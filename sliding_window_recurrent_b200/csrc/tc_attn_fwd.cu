// tcgen05 banded attention forward over the injected K/V entries.
//
// Source: "Maglev: Sliding Recurrent Memory", paper.rainbus.top, 前置知识
// (sliding-window attention: each position attends to the most recent W
// tokens) and 方法步骤详情 (the attention runs over the mixed entries
// k_bar, v_bar). Reading: keys j in [i-W+1, i], scale 1/sqrt(hd).
//
// One CTA per (128-query tile, head, batch row); two CTAs share an SM (about
// 112 KiB of shared memory and 256 TMEM columns each) so that one CTA's loads
// and set-up overlap the other's arithmetic. Only the 64-key half-tiles that
// meet the band [i0-W+1, i0+127] are visited (at most 10 for W = 512).
//   warp 0     TMA: Q once, K/V half-tiles into a 2-deep ring
//   warp 1     tcgen05.mma: S_j = Q K_j^T (128 x 64) into one of two TMEM S
//              buffers, issued one half-tile ahead; O += P_j V_j
//   warps 2-5  one query row per thread: masked online softmax in log2 units
//              (no masks on half-tiles inside every row's window), P_j (bf16)
//              into 128B-swizzled shared memory, lazy O rescale in TMEM,
//              final O / l and LSE.
// Inputs are the saved q_rot / k_bar / v_bar ([B,T,H,hd] bf16), read through
// 4-D tensor maps {hd, H, T, B} so rows past T arrive zero-filled.
#include <cuda.h>

#include "launchers.h"
#include "tc_common.cuh"

namespace maglev {

cudaError_t make_tmap_tokens(CUtensorMap* m, const void* base, int B, int T, int H, int hd, uint32_t box_rows);

namespace {

using namespace tc;

constexpr int NUM_THREADS = 192;
constexpr float LOG2E = 1.4426950408889634f;

template <int HD>
struct FwdCfg {
  static constexpr int CH = HD / 64;        // 64-wide swizzle chunks per row
  static constexpr int QCHUNK = 128 * 128;  // 128 rows x 64 bf16
  static constexpr int KCHUNK = 64 * 128;   // 64 rows x 64 bf16
  static constexpr int Q_BYTES = 128 * HD * 2;
  static constexpr int KH = 64 * HD * 2;    // one 64-key half-tile of K (or V)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = Q_BYTES;            // [2]
  static constexpr int OFF_V = OFF_K + 2 * KH;     // [2]
  static constexpr int OFF_P = OFF_V + 2 * KH;     // [128 queries x 64 keys] bf16
  static constexpr int P_BYTES = 128 * 64 * 2;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr size_t SMEM = OFF_BAR + 128;  // base is 1024-aligned (checked in the kernel)
  static constexpr uint32_t T_O = 0, T_S = 128;  // S buffers at 128 and 192 (64 columns each)
};

struct FwdParams {
  int B, T, H, W;
  float scale_log2;
  void* out;
  float* lse;
  int64_t spin_limit;
  int* err;
};

template <int HD>
__global__ void __launch_bounds__(NUM_THREADS, 2)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, FwdParams p) {
  using C = FwdCfg<HD>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  if (smem_u32(smem) & 1023u) {  // the swizzled tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) record_error(p.err, DEV_TIMEOUT);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;   // [2]
  uint64_t* kv_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;    // [2]
  uint64_t* p_full = bars + 7;
  uint64_t* pv_done = bars + 8;   // PV_j done: P buffer free, O updated
  uint64_t* drain = bars + 9;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 10);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const Abort ab{abort_flag, p.err, p.spin_limit * 1000};
  const int i0 = blockIdx.x * 128, h = blockIdx.y, b = blockIdx.z;
  const int first_key = max(0, i0 - p.W + 1);
  const int last_key = min(p.T - 1, i0 + 127);
  const int kh0 = first_key & ~63;
  const int n_half = ((last_key & ~63) - kh0) / 64 + 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
      mbar_init(&s_full[s], 1);
    }
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) tmem_alloc(tmem_slot, 256);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      uint32_t armed = 0, par = 0;
      mbar_arrive_expect_tx(q_full, C::Q_BYTES);
#pragma unroll
      for (int c = 0; c < C::CH; ++c) tma_load_4d(smem + C::OFF_Q + c * C::QCHUNK, &tmQ, q_full, 64 * c, h, i0, b);
      for (int j = 0; j < n_half; ++j) {
        const int s = j & 1;
        const uint32_t ph = (uint32_t)(j >> 1) & 1u;
        if (!mbar_wait(&kv_empty[s], ph ^ 1u, ab)) break;
        mbar_arrive_expect_tx(&kv_full[s], 2 * C::KH);
        armed |= 1u << s;
        par = (par & ~(1u << s)) | (ph << s);
        const int kh = kh0 + 64 * j;
#pragma unroll
        for (int c = 0; c < C::CH; ++c) {
          tma_load_4d(smem + C::OFF_K + s * C::KH + c * C::KCHUNK, &tmK, &kv_full[s], 64 * c, h, kh, b);
          tma_load_4d(smem + C::OFF_V + s * C::KH + c * C::KCHUNK, &tmV, &kv_full[s], 64 * c, h, kh, b);
        }
      }
      mbar_drain(q_full, 0, DRAIN_LIMIT_NS);
      for (int s = 0; s < 2; ++s)
        if (armed & (1u << s)) mbar_drain(&kv_full[s], (par >> s) & 1u, DRAIN_LIMIT_NS);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t ID_S = idesc_bf16(128, 64, false, false);  // 128 queries x 64 keys
      constexpr uint32_t ID_O = idesc_bf16(128, HD, false, true);   // 128 queries x hd
      const uint32_t q_addr = smem_u32(smem + C::OFF_Q);
      const uint32_t p_addr = smem_u32(smem + C::OFF_P);
      auto issue_s = [&](int j) {
        const int s = j & 1;
        const uint32_t k_addr = smem_u32(smem + C::OFF_K + s * C::KH);
#pragma unroll
        for (int k16 = 0; k16 < HD / 16; ++k16) {
          mma_ss(tmem + C::T_S + 64u * (uint32_t)s, kmajor_desc(q_addr + (uint32_t)(k16 >> 2) * C::QCHUNK, k16 & 3),
                 kmajor_desc(k_addr + (uint32_t)(k16 >> 2) * C::KCHUNK, k16 & 3), ID_S, k16 > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[s]);
      };
      bool ok = mbar_wait(q_full, 0, ab) && mbar_wait(&kv_full[0], 0, ab);
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      for (int j = 0; j < n_half && ok; ++j) {
        if (j + 1 < n_half) {  // S buffer (j+1)&1 was read by softmax j-1 (p_full waited last round)
          if (!mbar_wait(&kv_full[(j + 1) & 1], (uint32_t)((j + 1) >> 1) & 1u, ab)) break;
          tc_fence_after();
          issue_s(j + 1);
        }
        if (!mbar_wait(p_full, (uint32_t)j & 1u, ab)) break;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(smem + C::OFF_V + (j & 1) * C::KH);
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16) {  // K = 64 keys
          mma_ss(tmem + C::T_O, kmajor_desc(p_addr, k16),
                 sw128_desc(v_addr + (uint32_t)k16 * 2048u, (uint32_t)C::KCHUNK, 1024u), ID_O,
                 (j > 0 || k16 > 0) ? 1u : 0u);
        }
        mma_commit(&kv_empty[j & 1]);
        mma_commit(pv_done);
      }
      mma_commit(drain);
      mbar_drain(drain, 0, DRAIN_LIMIT_NS);
    }
  } else {
    // -------------------------------------------------------------- softmax / epilogue
    // The running max m_ref is only raised when a half-tile's max exceeds it by
    // more than 8 (log2 units), so P stays <= 2^8 and O is rescaled rarely; l
    // and the final LSE use the same reference, so the result is unchanged.
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int i = i0 + r;
    const int i_lo = i0 + 32 * q;  // first row of this warp
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    uint8_t* sP = smem + C::OFF_P;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_half; ++j) {
      const int s = j & 1;
      if (!warp_wait(&s_full[s], (uint32_t)(j >> 1) & 1u, ab)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t va[32], vb[32];
      tmem_ld32(tmem + lane_off + C::T_S + 64u * (uint32_t)s, va);
      tmem_ld32(tmem + lane_off + C::T_S + 64u * (uint32_t)s + 32u, vb);
      tmem_wait_ld();
      const int kh = kh0 + 64 * j;
      const int lo = max(i - p.W + 1, 0) - kh;  // first valid column
      const int hi = min(i, p.T - 1) - kh;      // last valid column
      // every key of the half-tile inside the window of every row of this warp
      const bool full = kh >= i_lo + 31 - p.W + 1 && kh + 63 <= i_lo && kh + 63 <= p.T - 1;
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (full) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          mx[e & 1] = fmaxf(mx[e & 1], __uint_as_float(va[e]));
          mx[2 + (e & 1)] = fmaxf(mx[2 + (e & 1)], __uint_as_float(vb[e]));
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          if (e >= lo && e <= hi) mx[e & 1] = fmaxf(mx[e & 1], __uint_as_float(va[e]));
          if (32 + e >= lo && 32 + e <= hi) mx[2 + (e & 1)] = fmaxf(mx[2 + (e & 1)], __uint_as_float(vb[e]));
        }
      }
      const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.scale_log2;
      float alpha = 1.f;
      bool rescale = false;
      if (mt != -INFINITY && (m_ref == -INFINITY || mt > m_ref + 8.f)) {
        if (m_ref != -INFINITY) {
          alpha = ex2_fast(m_ref - mt);
          rescale = true;
        }
        m_ref = mt;
      }
      const bool live = m_ref != -INFINITY;
      const float sl = p.scale_log2, nmr = -m_ref;
      float pr[64];
      float rs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float ya = ex2_fast(fmaf(__uint_as_float(va[e]), sl, nmr));
        const float yb = ex2_fast(fmaf(__uint_as_float(vb[e]), sl, nmr));
        pr[e] = full ? ya : ((live && e >= lo && e <= hi) ? ya : 0.f);
        pr[32 + e] = full ? yb : ((live && 32 + e >= lo && 32 + e <= hi) ? yb : 0.f);
        rs[e & 1] += pr[e];
        rs[2 + (e & 1)] += pr[32 + e];
      }
      l = l * alpha + ((rs[0] + rs[1]) + (rs[2] + rs[3]));
      if (j >= 1) {  // P buffer and O: PV_{j-1} must be complete
        if (!warp_wait(pv_done, (uint32_t)(j - 1) & 1u, ab)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        uint4 w;
        w.x = pack_bf16(pr[8 * g + 0], pr[8 * g + 1]);
        w.y = pack_bf16(pr[8 * g + 2], pr[8 * g + 3]);
        w.z = pack_bf16(pr[8 * g + 4], pr[8 * g + 5]);
        w.w = pack_bf16(pr[8 * g + 6], pr[8 * g + 7]);
        *reinterpret_cast<uint4*>(sP + r * 128 + ((g ^ (r & 7)) << 4)) = w;
      }
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + C::T_O + 32u * (uint32_t)c, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
          tmem_st32(tmem + lane_off + C::T_O + 32u * (uint32_t)c, v);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    const int last = n_half - 1;
    if (__all_sync(0xffffffffu, ok) && n_half > 0 && warp_wait(pv_done, (uint32_t)last & 1u, ab)) {
      tc_fence_after();
      const float inv = 1.f / l;
      bf16* dst = static_cast<bf16*>(p.out) + (((int64_t)b * p.T + i) * p.H + h) * HD;
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + C::T_O + 32u * (uint32_t)c, v);
        tmem_wait_ld();
        if (i < p.T) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            uint4 o;
            o.x = pack_bf16(__uint_as_float(v[8 * g + 0]) * inv, __uint_as_float(v[8 * g + 1]) * inv);
            o.y = pack_bf16(__uint_as_float(v[8 * g + 2]) * inv, __uint_as_float(v[8 * g + 3]) * inv);
            o.z = pack_bf16(__uint_as_float(v[8 * g + 4]) * inv, __uint_as_float(v[8 * g + 5]) * inv);
            o.w = pack_bf16(__uint_as_float(v[8 * g + 6]) * inv, __uint_as_float(v[8 * g + 7]) * inv);
            *reinterpret_cast<uint4*>(dst + 32 * c + 8 * g) = o;
          }
        }
      }
      if (i < p.T) p.lse[((int64_t)b * p.H + h) * p.T + i] = (m_ref + log2f(l)) * 0.69314718055994531f;
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace

cudaError_t launch_attn_fwd_tc(const SwaShape& s, const void* q_rot, const void* k_bar, const void* v_bar,
                               void* out, float* lse, int64_t spin_limit, int* err, cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  cudaError_t e;
  if ((e = make_tmap_tokens(&tq, q_rot, s.B, s.T, s.H, s.hd, 128)) != cudaSuccess) return e;
  if ((e = make_tmap_tokens(&tk, k_bar, s.B, s.T, s.H, s.hd, 64)) != cudaSuccess) return e;
  if ((e = make_tmap_tokens(&tv, v_bar, s.B, s.T, s.H, s.hd, 64)) != cudaSuccess) return e;
  FwdParams p;
  p.B = s.B;
  p.T = s.T;
  p.H = s.H;
  p.W = s.W;
  p.scale_log2 = LOG2E / sqrtf((float)s.hd);
  p.out = out;
  p.lse = lse;
  p.spin_limit = spin_limit;
  p.err = err;
  dim3 grid((unsigned)((s.T + 127) / 128), (unsigned)s.H, (unsigned)s.B);
  if (s.hd == 128) {
    auto k = attn_fwd_tc_kernel<128>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FwdCfg<128>::SMEM);
    if (e != cudaSuccess) return e;
    k<<<grid, NUM_THREADS, FwdCfg<128>::SMEM, st>>>(tq, tk, tv, p);
  } else if (s.hd == 64) {
    auto k = attn_fwd_tc_kernel<64>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FwdCfg<64>::SMEM);
    if (e != cudaSuccess) return e;
    k<<<grid, NUM_THREADS, FwdCfg<64>::SMEM, st>>>(tq, tk, tv, p);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace maglev
