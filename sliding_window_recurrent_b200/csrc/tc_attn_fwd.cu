// tcgen05 banded attention forward over the injected K/V entries.
//
// Source: "Maglev: Sliding Recurrent Memory", paper.rainbus.top, 前置知识
// (sliding-window attention: each position attends to the most recent W
// tokens) and 方法步骤详情 (the attention runs over the mixed entries
// k_bar, v_bar). Reading: keys j in [i-W+1, i], scale 1/sqrt(hd).
//
// Persistent, two CTAs per SM (about 113 KiB of shared memory and 256 TMEM
// columns each): every CTA walks work units (128-query tile, head, batch row)
// with a stride of the grid, so set-up is paid once per CTA and the next
// unit's Q and K/V stream in while the current unit finishes. Only the 64-key
// half-tiles that meet the band [i0-W+1, i0+127] are visited (at most 10 for
// W = 512). K and V have separate 2-deep rings: a K slot frees as soon as its
// S MMA completes, a V slot when its PV MMA completes.
//   warp 0     TMA producer: Q per unit, K one half-tile ahead of V
//   warp 1     tcgen05.mma: S_g = Q K_g^T (128 x 64) into one of two TMEM S
//              buffers, issued one half-tile ahead; O += P_g V_g
//   warps 2-5  one query row per thread: online softmax in log2 units
//              (masked scores set to -inf in one pass on half-tiles that
//              cross the band's edge), P (bf16) into 128B-swizzled shared
//              memory, lazy O rescale in TMEM, final O / l and LSE per unit.
// Inputs are the saved q_rot / k_bar / v_bar ([B,T,H,hd] bf16), read through
// 4-D tensor maps {hd, H, T, B} so rows past T arrive zero-filled.
#include <cuda.h>

#include "launchers.h"
#include "tc_common.cuh"

namespace maglev {

cudaError_t make_tmap_tokens(CUtensorMap* m, const void* base, int B, int T, int H, int hd, uint32_t box_rows);
int num_sms();

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
  static constexpr size_t SMEM = OFF_BAR + 256;    // base is 1024-aligned (checked in the kernel)
  static constexpr uint32_t T_O = 0, T_S = 128;    // S buffers at 128 and 192 (64 columns each)
};

struct FwdParams {
  int B, T, H, W;
  int n_qtiles, n_units;
  float scale_log2;
  void* out;
  float* lse;
  int64_t spin_limit;
  int* err;
};

struct Unit {
  int i0, h, b, kh0, n_half;
};

// Work order: units ranked by decreasing cost (query tiles from the last one
// down; the first tiles see fewer keys), dealt to the CTAs in a snake (pass k
// runs over the CTAs forwards when k is even, backwards when odd), so every
// CTA ends up with about the same number of half-tiles. Returns -1 past the end.
__device__ __forceinline__ int unit_rank(const FwdParams& p, int k) {
  const int G = (int)gridDim.x, c = (int)blockIdx.x;
  const int r = k * G + ((k & 1) ? G - 1 - c : c);
  return r < p.n_units ? r : -1;
}

__device__ __forceinline__ Unit unit_of(const FwdParams& p, int r) {
  Unit x;
  const int hb = p.H * p.B;
  x.i0 = (p.n_qtiles - 1 - r / hb) * 128;
  x.h = (r % hb) % p.H;
  x.b = (r % hb) / p.H;
  const int first_key = max(0, x.i0 - p.W + 1);
  const int last_key = min(p.T - 1, x.i0 + 127);
  x.kh0 = first_key & ~63;
  x.n_half = ((last_key & ~63) - x.kh0) / 64 + 1;
  return x;
}

template <int HD>
__global__ void __launch_bounds__(NUM_THREADS, 2)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, FwdParams p) {
  using C = FwdCfg<HD>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {  // the swizzled tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) record_error(p.err, DEV_TIMEOUT);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;    // [2]
  uint64_t* k_empty = bars + 4;   // [2]
  uint64_t* v_full = bars + 6;    // [2]
  uint64_t* v_empty = bars + 8;   // [2]
  uint64_t* s_full = bars + 10;   // [2]
  uint64_t* p_full = bars + 12;
  uint64_t* pv_done = bars + 13;  // PV_g done: P buffer free, O updated
  uint64_t* o_empty = bars + 14;  // the unit's O has been read out of TMEM
  uint64_t* drain = bars + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const Abort ab{abort_flag, p.err, p.spin_limit * 1000};

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
    }
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(o_empty, 128);
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
      // Global half-tile counter g over this CTA's units. Step g loads K_g and
      // then V_{g-1}, so a K load never queues behind a V slot that is still
      // waiting for its PV.
      uint32_t q_armed = 0, q_par = 0, k_armed = 0, k_par = 0, v_armed = 0, v_par = 0;
      int g = 0, n = 0, kh_prev = 0, h_prev = 0, b_prev = 0;
      bool ok = true;
      auto load_v = [&](int gv, int kh, int hh, int bb) -> bool {
        const int s = gv & 1;
        const uint32_t ph = (uint32_t)(gv >> 1) & 1u;
        if (!mbar_wait(&v_empty[s], ph ^ 1u, ab)) return false;
        mbar_arrive_expect_tx(&v_full[s], C::KH);
        v_armed |= 1u << s;
        v_par = (v_par & ~(1u << s)) | (ph << s);
#pragma unroll
        for (int c = 0; c < C::CH; ++c)
          tma_load_4d(smem + C::OFF_V + s * C::KH + c * C::KCHUNK, &tmV, &v_full[s], 64 * c, hh, kh, bb);
        return true;
      };
      for (int u = unit_rank(p, 0); u >= 0 && ok; u = unit_rank(p, ++n)) {
        const Unit x = unit_of(p, u);
        const uint32_t qph = (uint32_t)n & 1u;
        if (!mbar_wait(q_empty, qph ^ 1u, ab)) break;
        mbar_arrive_expect_tx(q_full, C::Q_BYTES);
        q_armed = 1;
        q_par = qph;
#pragma unroll
        for (int c = 0; c < C::CH; ++c) tma_load_4d(smem + C::OFF_Q + c * C::QCHUNK, &tmQ, q_full, 64 * c, x.h, x.i0, x.b);
        for (int j = 0; j < x.n_half; ++j, ++g) {
          const int s = g & 1;
          const uint32_t ph = (uint32_t)(g >> 1) & 1u;
          const int kh = x.kh0 + 64 * j;
          if (!mbar_wait(&k_empty[s], ph ^ 1u, ab)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&k_full[s], C::KH);
          k_armed |= 1u << s;
          k_par = (k_par & ~(1u << s)) | (ph << s);
#pragma unroll
          for (int c = 0; c < C::CH; ++c)
            tma_load_4d(smem + C::OFF_K + s * C::KH + c * C::KCHUNK, &tmK, &k_full[s], 64 * c, x.h, kh, x.b);
          if (g > 0 && !load_v(g - 1, kh_prev, h_prev, b_prev)) {
            ok = false;
            break;
          }
          kh_prev = kh;
          h_prev = x.h;
          b_prev = x.b;
        }
      }
      if (ok && g > 0) load_v(g - 1, kh_prev, h_prev, b_prev);
      if (q_armed) mbar_drain(q_full, q_par, DRAIN_LIMIT_NS);
      for (int s = 0; s < 2; ++s) {
        if (k_armed & (1u << s)) mbar_drain(&k_full[s], (k_par >> s) & 1u, DRAIN_LIMIT_NS);
        if (v_armed & (1u << s)) mbar_drain(&v_full[s], (v_par >> s) & 1u, DRAIN_LIMIT_NS);
      }
    }
  } else if (warp == 1) {
    {
      // ------------------------------------------------------------ MMA issuer
      // Every lane runs the loop and the waits (warp-uniform descriptors and
      // counters); the elected lane issues each batch of MMAs and commits.
      constexpr uint32_t ID_S = idesc_bf16(128, 64, false, false);  // 128 queries x 64 keys
      constexpr uint32_t ID_O = idesc_bf16(128, HD, false, true);   // 128 queries x hd
      // base descriptors: each MMA's operand is a constant offset from these
      const uint64_t qd = kmajor_desc(smem_u32(smem + C::OFF_Q), 0);
      const uint64_t pd = kmajor_desc(smem_u32(smem + C::OFF_P), 0);
      // S_gs = Q K_gs^T into S buffer gs&1; the K slot is released when it completes
      auto issue_s = [&](int gs) -> bool {
        const int s = gs & 1;
        if (!warp_wait(&k_full[s], (uint32_t)(gs >> 1) & 1u, ab)) return false;
        tc_fence_after();
        const uint64_t kd = kmajor_desc(smem_u32(smem + C::OFF_K + s * C::KH), 0);
        if (elect_one()) {
#pragma unroll
          for (int k16 = 0; k16 < HD / 16; ++k16) {
            mma_ss(tmem + C::T_S + 64u * (uint32_t)s,
                   desc_at(qd, (uint32_t)(k16 >> 2) * C::QCHUNK + (k16 & 3) * 32u),
                   desc_at(kd, (uint32_t)(k16 >> 2) * C::KCHUNK + (k16 & 3) * 32u), ID_S, k16 > 0 ? 1u : 0u);
          }
          mma_commit(&s_full[s]);
          mma_commit(&k_empty[s]);
        }
        __syncwarp();
        return true;
      };
      int g = 0, n = 0;
      bool ok = true;
      for (int u = unit_rank(p, 0); u >= 0 && ok; u = unit_rank(p, ++n)) {
        const Unit x = unit_of(p, u);
        // S buffer g&1 was last read by the softmax of half-tile g-2, whose
        // p_full this thread has waited for
        if (!warp_wait(q_full, (uint32_t)n & 1u, ab) || !issue_s(g)) break;
        for (int j = 0; j < x.n_half; ++j, ++g) {
          if (j + 1 < x.n_half) {
            if (!issue_s(g + 1)) {
              ok = false;
              break;
            }
          } else {
            if (elect_one()) mma_commit(q_empty);  // every S of this unit has been issued
            __syncwarp();
          }
          if (!warp_wait(p_full, (uint32_t)g & 1u, ab)) {
            ok = false;
            break;
          }
          // the first PV of a unit overwrites O: the previous unit's epilogue must be done
          if (j == 0 && !warp_wait(o_empty, ((uint32_t)n & 1u) ^ 1u, ab)) {
            ok = false;
            break;
          }
          if (!warp_wait(&v_full[g & 1], (uint32_t)(g >> 1) & 1u, ab)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t vmn = sw128_desc(smem_u32(smem + C::OFF_V + (g & 1) * C::KH), (uint32_t)C::KCHUNK, 1024u);
          if (elect_one()) {
#pragma unroll
            for (int k16 = 0; k16 < 4; ++k16)  // K = 64 keys
              mma_ss(tmem + C::T_O, desc_at(pd, k16 * 32u), desc_at(vmn, k16 * 2048u), ID_O,
                     (j > 0 || k16 > 0) ? 1u : 0u);
            mma_commit(&v_empty[g & 1]);
            mma_commit(pv_done);
          }
          __syncwarp();
        }
      }
      if (elect_one()) {  // the issuing lane's MMAs complete before TMEM is released
        mma_commit(drain);
        mbar_drain(drain, 0, DRAIN_LIMIT_NS);
      }
      __syncwarp();
    }
  } else {
    // -------------------------------------------------------------- softmax / epilogue
    // The running max m_ref is only raised when a half-tile's max exceeds it by
    // more than 8 (log2 units), so P stays <= 2^8 and O is rescaled rarely; l
    // and the final LSE use the same reference, so the result is unchanged.
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    uint8_t* sP = smem + C::OFF_P;
    const uint32_t NEG_INF = 0xff800000u;
    int g = 0, n = 0;
    bool ok = true;
    for (int u = unit_rank(p, 0); u >= 0 && ok; u = unit_rank(p, ++n)) {
      const Unit x = unit_of(p, u);
      const int i = x.i0 + r;
      const int i_lo = x.i0 + 32 * q;  // first row of this warp
      float m_ref = -INFINITY, l = 0.f;
      for (int j = 0; j < x.n_half; ++j, ++g) {
        const int s = g & 1;
        if (!warp_wait(&s_full[s], (uint32_t)(g >> 1) & 1u, ab)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t v2[2][32];
        tmem_ld32(tmem + lane_off + C::T_S + 64u * (uint32_t)s, v2[0]);
        tmem_ld32(tmem + lane_off + C::T_S + 64u * (uint32_t)s + 32u, v2[1]);
        tmem_wait_ld();
        uint32_t* v = &v2[0][0];  // 64 scores, indexed with compile-time constants
        const int kh = x.kh0 + 64 * j;
        // every key of the half-tile inside the window of every row of this warp
        const bool full = kh >= i_lo + 31 - p.W + 1 && kh + 63 <= i_lo && kh + 63 <= p.T - 1;
        if (!full) {  // columns outside [lo, hi] become -inf (exp2 gives 0)
          const int lo = max(i - p.W + 1, 0) - kh;
          const int hi = min(i, p.T - 1) - kh;
          const uint32_t span = hi >= lo ? (uint32_t)(hi - lo) : 0u;
          const bool none = hi < lo;
#pragma unroll
          for (int e = 0; e < 64; ++e)
            v[e] = (!none && (uint32_t)(e - lo) <= span) ? v[e] : NEG_INF;
        }
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int e = 0; e < 64; ++e) mx[e & 3] = fmaxf(mx[e & 3], __uint_as_float(v[e]));
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
        // a row with no valid key yet keeps m_ref = -inf; its scores are all -inf
        const float sl = p.scale_log2, nmr = m_ref == -INFINITY ? 0.f : -m_ref;
        float rs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          const float y = ex2_fast(fmaf(__uint_as_float(v[e]), sl, nmr));
          v[e] = __float_as_uint(y);
          rs[e & 3] += y;
        }
        l = l * alpha + ((rs[0] + rs[1]) + (rs[2] + rs[3]));
        if (g >= 1) {  // the P buffer (and, within a unit, O) wait for the previous PV
          if (!warp_wait(pv_done, (uint32_t)(g - 1) & 1u, ab)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          uint4 w;
          w.x = pack_bf16(__uint_as_float(v[8 * c8 + 0]), __uint_as_float(v[8 * c8 + 1]));
          w.y = pack_bf16(__uint_as_float(v[8 * c8 + 2]), __uint_as_float(v[8 * c8 + 3]));
          w.z = pack_bf16(__uint_as_float(v[8 * c8 + 4]), __uint_as_float(v[8 * c8 + 5]));
          w.w = pack_bf16(__uint_as_float(v[8 * c8 + 6]), __uint_as_float(v[8 * c8 + 7]));
          *reinterpret_cast<uint4*>(sP + r * 128 + ((c8 ^ (r & 7)) << 4)) = w;
        }
        if (__any_sync(0xffffffffu, rescale)) {  // rescale only happens for j >= 1
#pragma unroll 1
          for (int c = 0; c < HD / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_off + C::T_O + 32u * (uint32_t)c, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tmem + lane_off + C::T_O + 32u * (uint32_t)c, o);
          }
          tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(p_full);
      }
      if (!ok) break;
      // epilogue of the unit: its last PV is half-tile g-1
      if (!warp_wait(pv_done, (uint32_t)(g - 1) & 1u, ab)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float inv = 1.f / l;
      // 64 columns at a time through this warp's own 32 rows of the P buffer
      // (free: the unit's last PV has completed; only this warp writes them
      // next), read back so that each warp-wide store covers four whole
      // 128-byte row pieces
      uint8_t* stg = sP + q * 4096;
      const int64_t tstride = (int64_t)p.H * HD;  // elements between consecutive tokens
      bf16* obase = static_cast<bf16*>(p.out) + ((int64_t)x.b * p.T + i_lo) * tstride + (int64_t)x.h * HD;
#pragma unroll 1
      for (int c = 0; c < HD / 64; ++c) {
        uint32_t o2[2][32];
        tmem_ld32(tmem + lane_off + C::T_O + 64u * (uint32_t)c, o2[0]);
        tmem_ld32(tmem + lane_off + C::T_O + 64u * (uint32_t)c + 32u, o2[1]);
        tmem_wait_ld();
        const uint32_t* o = &o2[0][0];
        if (c == HD / 64 - 1) {  // O is in registers: the next unit's first PV may overwrite it
          tc_fence_before();
          mbar_arrive(o_empty);
        }
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          uint4 w;
          w.x = pack_bf16(__uint_as_float(o[8 * c8 + 0]) * inv, __uint_as_float(o[8 * c8 + 1]) * inv);
          w.y = pack_bf16(__uint_as_float(o[8 * c8 + 2]) * inv, __uint_as_float(o[8 * c8 + 3]) * inv);
          w.z = pack_bf16(__uint_as_float(o[8 * c8 + 4]) * inv, __uint_as_float(o[8 * c8 + 5]) * inv);
          w.w = pack_bf16(__uint_as_float(o[8 * c8 + 6]) * inv, __uint_as_float(o[8 * c8 + 7]) * inv);
          *reinterpret_cast<uint4*>(stg + lane * 128 + ((c8 ^ (lane & 7)) << 4)) = w;
        }
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int rr = 4 * k + (lane >> 3), j = lane & 7;  // row of the warp's 32, 16-byte chunk
          const uint4 w = *reinterpret_cast<const uint4*>(stg + rr * 128 + ((j ^ (rr & 7)) << 4));
          if (i_lo + rr < p.T && MAGLEV_CHECK(p.err, i_lo + rr >= 0 && x.b < p.B && x.h < p.H))
            *reinterpret_cast<uint4*>(obase + rr * tstride + 64 * c + 8 * j) = w;
        }
        __syncwarp();
      }
      if (i < p.T) p.lse[((int64_t)x.b * p.H + x.h) * p.T + i] = (m_ref + log2f(l)) * 0.69314718055994531f;
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
  p.n_qtiles = (s.T + 127) / 128;
  p.n_units = p.n_qtiles * s.H * s.B;
  p.scale_log2 = LOG2E / sqrtf((float)s.hd);
  p.out = out;
  p.lse = lse;
  p.spin_limit = spin_limit;
  p.err = err;
  const int slots = 2 * num_sms();  // two CTAs per SM
  const unsigned grid = (unsigned)(p.n_units < slots ? p.n_units : slots);
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
