// tcgen05 banded attention forward over the injected K/V entries.
//
// Source: "Maglev: Sliding Recurrent Memory", paper.rainbus.top, 前置知识
// (sliding-window attention: each position attends to the most recent W
// tokens) and 方法步骤详情 (the attention runs over the mixed entries
// k_bar, v_bar). Reading: keys j in [i-W+1, i], scale 1/sqrt(hd).
//
// One CTA per (128-query tile, head, batch row). Only the 128-key tiles that
// intersect the band [i0-W+1, i0+127] are visited (at most 5 for W = 512).
//   warp 0     TMA: Q once, K/V tiles into a 2-deep ring
//   warp 1     tcgen05.mma: S_j = Q K_j^T into one of two TMEM S buffers
//              (issued one tile ahead), then O += P_j V_j once P_j is ready
//   warps 2-5  one query row per thread: masked online softmax in log2 units,
//              P_j (bf16) into 128B-swizzled shared memory, O rescaled in
//              TMEM when the running max grows, final O / l and LSE.
// Inputs are the saved q_rot / k_bar / v_bar ([B,T,H,hd] bf16), read through
// 4-D tensor maps {hd, H, T, B} so rows past T arrive zero-filled.
#include <cuda.h>

#include "launchers.h"
#include "tc_common.cuh"

namespace maglev {

cudaError_t make_tmap_bf16_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                              uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer);
cudaError_t make_tmap_tokens(CUtensorMap* m, const void* base, int B, int T, int H, int hd, uint32_t box_rows);

namespace {

using namespace tc;

constexpr int NUM_THREADS = 192;
constexpr float LOG2E = 1.4426950408889634f;

template <int HD>
struct FwdCfg {
  static constexpr int CH = HD / 64;          // 64-wide swizzle chunks per row
  static constexpr int TILE = 128 * HD * 2;   // one 128-row operand tile
  static constexpr int CHUNK = 128 * 128;     // bytes of one 128-row x 64-col chunk
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = TILE;
  static constexpr int OFF_V = 3 * TILE;
  static constexpr int OFF_P = 5 * TILE;
  static constexpr int P_BYTES = 128 * 128 * 2;  // one P tile; two are kept
  static constexpr int OFF_BAR = OFF_P + 2 * P_BYTES;
  static constexpr size_t SMEM = 1024 + OFF_BAR + 256;
  static constexpr uint32_t S_COL = 128;      // S buffers at columns 128 and 256
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
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, FwdParams p) {
  using C = FwdCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;   // [2]
  uint64_t* kv_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;    // [2]
  uint64_t* p_full = bars + 7;
  uint64_t* pv_done = bars + 8;   // [2]: PV_j done (P buffer j%2 free, O updated)
  uint64_t* drain = bars + 10;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const Abort ab{abort_flag, p.err, p.spin_limit * 1000};
  const int i0 = blockIdx.x * 128, h = blockIdx.y, b = blockIdx.z;
  const int first_key = max(0, i0 - p.W + 1);
  const int last_key = min(p.T - 1, i0 + 127);
  const int kt_first = first_key & ~127;
  const int n_tiles = ((last_key & ~127) - kt_first) / 128 + 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
      mbar_init(&s_full[s], 1);
    }
    mbar_init(p_full, 128);
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      uint32_t armed_q = 0, armed_kv = 0, par_kv = 0;
      mbar_arrive_expect_tx(q_full, C::TILE);
      armed_q = 1;
#pragma unroll
      for (int c = 0; c < C::CH; ++c) tma_load_4d(smem + C::OFF_Q + c * C::CHUNK, &tmQ, q_full, 64 * c, h, i0, b);
      for (int j = 0; j < n_tiles; ++j) {
        const int buf = j & 1;
        const uint32_t ph = (uint32_t)(j >> 1) & 1u;
        if (!mbar_wait(&kv_empty[buf], ph ^ 1u, ab)) break;
        mbar_arrive_expect_tx(&kv_full[buf], 2 * C::TILE);
        armed_kv |= 1u << buf;
        par_kv = (par_kv & ~(1u << buf)) | (ph << buf);
        const int kt = kt_first + 128 * j;
#pragma unroll
        for (int c = 0; c < C::CH; ++c) {
          tma_load_4d(smem + C::OFF_K + buf * C::TILE + c * C::CHUNK, &tmK, &kv_full[buf], 64 * c, h, kt, b);
          tma_load_4d(smem + C::OFF_V + buf * C::TILE + c * C::CHUNK, &tmV, &kv_full[buf], 64 * c, h, kt, b);
        }
      }
      if (armed_q) mbar_drain(q_full, 0, DRAIN_LIMIT_NS);
      for (int s = 0; s < 2; ++s)
        if (armed_kv & (1u << s)) mbar_drain(&kv_full[s], (par_kv >> s) & 1u, DRAIN_LIMIT_NS);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false, false);
      constexpr uint32_t IDESC_O = idesc_bf16(128, HD, false, true);
      const uint32_t q_addr = smem_u32(smem + C::OFF_Q);
      const uint32_t p_addr = smem_u32(smem + C::OFF_P);
      auto issue_s = [&](int j) {
        const int buf = j & 1;
        const uint32_t k_addr = smem_u32(smem + C::OFF_K + buf * C::TILE);
        const uint32_t d = tmem + C::S_COL + 128u * (uint32_t)buf;
#pragma unroll
        for (int k16 = 0; k16 < HD / 16; ++k16) {
          const uint32_t off = (uint32_t)(k16 >> 2) * C::CHUNK;
          mma_ss(d, kmajor_desc(q_addr + off, k16 & 3), kmajor_desc(k_addr + off, k16 & 3), IDESC_S,
                 k16 > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[buf]);
      };
      bool ok = mbar_wait(q_full, 0, ab);
      if (ok && n_tiles > 0) {
        ok = mbar_wait(&kv_full[0], 0, ab);
        if (ok) {
          tc_fence_after();
          issue_s(0);
        }
      }
      for (int j = 0; j < n_tiles && ok; ++j) {
        if (j + 1 < n_tiles) {
          if (!mbar_wait(&kv_full[(j + 1) & 1], (uint32_t)((j + 1) >> 1) & 1u, ab)) break;
          tc_fence_after();
          issue_s(j + 1);
        }
        if (!mbar_wait(p_full, (uint32_t)j & 1u, ab)) break;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(smem + C::OFF_V + (j & 1) * C::TILE);
        const uint32_t pj_addr = p_addr + (uint32_t)((j & 1) * C::P_BYTES);
#pragma unroll
        for (int k16 = 0; k16 < 8; ++k16) {  // K = 128 keys
          const uint64_t ad = kmajor_desc(pj_addr + (uint32_t)(k16 >> 2) * C::CHUNK, k16 & 3);
          const uint64_t bd = sw128_desc(v_addr + (uint32_t)k16 * 2048u, (uint32_t)C::CHUNK, 1024u);
          mma_ss(tmem, ad, bd, IDESC_O, (j > 0 || k16 > 0) ? 1u : 0u);
        }
        mma_commit(&kv_empty[j & 1]);
        mma_commit(&pv_done[j & 1]);
      }
      mma_commit(drain);
      mbar_drain(drain, 0, DRAIN_LIMIT_NS);
    }
  } else {
    // -------------------------------------------------------------- softmax / epilogue
    // The running max m_ref is only raised when a tile's max exceeds it by more
    // than 8 (log2 units), so P stays <= 2^8 and O is rescaled rarely; l and the
    // final LSE use the same reference, so the result is unchanged.
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int i = i0 + r;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int buf = j & 1;
      if (!warp_wait(&s_full[buf], (uint32_t)(j >> 1) & 1u, ab)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t s_addr = tmem + lane_off + C::S_COL + 128u * (uint32_t)buf;
      const int kt = kt_first + 128 * j;
      const int lo = max(i - p.W + 1, 0) - kt;  // first valid column
      const int hi = min(i, p.T - 1) - kt;      // last valid column
      float mt = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        tmem_ld32(s_addr + 32u * (uint32_t)c, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int col = 32 * c + e;
          if (col >= lo && col <= hi) mt = fmaxf(mt, __uint_as_float(v[e]));
        }
      }
      mt *= p.scale_log2;
      float alpha = 1.f;
      bool rescale = false;
      if (mt != -INFINITY && (m_ref == -INFINITY || mt > m_ref + 8.f)) {
        if (m_ref != -INFINITY) {
          alpha = exp2f(m_ref - mt);
          rescale = true;
        }
        m_ref = mt;
      }
      if (j >= 2) {  // P buffer `buf` was read by PV_{j-2}
        if (!warp_wait(&pv_done[buf], (uint32_t)((j - 2) >> 1) & 1u, ab)) {
          ok = false;
          break;
        }
      }
      uint8_t* sP = smem + C::OFF_P + buf * C::P_BYTES;
      float rs = 0.f;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        tmem_ld32(s_addr + 32u * (uint32_t)c, v);
        tmem_wait_ld();
        float pv[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int col = 32 * c + e;
          const float x = exp2f(__uint_as_float(v[e]) * p.scale_log2 - m_ref);
          pv[e] = (col >= lo && col <= hi && m_ref != -INFINITY) ? x : 0.f;
          rs += pv[e];
        }
        const int ch = c >> 1;
#pragma unroll
        for (int gg = 0; gg < 4; ++gg) {
          const int g = (c & 1) * 4 + gg;
          uint4 w;
          w.x = pack_bf16(pv[8 * gg + 0], pv[8 * gg + 1]);
          w.y = pack_bf16(pv[8 * gg + 2], pv[8 * gg + 3]);
          w.z = pack_bf16(pv[8 * gg + 4], pv[8 * gg + 5]);
          w.w = pack_bf16(pv[8 * gg + 6], pv[8 * gg + 7]);
          *reinterpret_cast<uint4*>(sP + ch * C::CHUNK + r * 128 + ((g ^ (r & 7)) << 4)) = w;
        }
      }
      l = l * alpha + rs;
      if (__any_sync(0xffffffffu, rescale)) {  // O must hold PV_{j-1} before it is scaled
        if (!warp_wait(&pv_done[buf ^ 1], (uint32_t)((j - 1) >> 1) & 1u, ab)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + 32u * (uint32_t)c, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
          tmem_st32(tmem + lane_off + 32u * (uint32_t)c, v);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    const int last = n_tiles - 1;
    if (__all_sync(0xffffffffu, ok) && n_tiles > 0 && warp_wait(&pv_done[last & 1], (uint32_t)(last >> 1) & 1u, ab)) {
      tc_fence_after();
      const float inv = 1.f / l;
      bf16* dst = static_cast<bf16*>(p.out) + (((int64_t)b * p.T + i) * p.H + h) * HD;
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + 32u * (uint32_t)c, v);
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
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

// Tensor map over a [B,T,H,hd] bf16 token-major tensor: dims {hd, H, T, B},
// box {64, 1, box_rows, 1} (one head, box_rows positions), 128B swizzle.
cudaError_t make_tmap_tokens(CUtensorMap* m, const void* base, int B, int T, int H, int hd, uint32_t box_rows);

cudaError_t launch_attn_fwd_tc(const SwaShape& s, const void* q_rot, const void* k_bar, const void* v_bar,
                               void* out, float* lse, int64_t spin_limit, int* err, cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  cudaError_t e;
  if ((e = make_tmap_tokens(&tq, q_rot, s.B, s.T, s.H, s.hd, 128)) != cudaSuccess) return e;
  if ((e = make_tmap_tokens(&tk, k_bar, s.B, s.T, s.H, s.hd, 128)) != cudaSuccess) return e;
  if ((e = make_tmap_tokens(&tv, v_bar, s.B, s.T, s.H, s.hd, 128)) != cudaSuccess) return e;
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
