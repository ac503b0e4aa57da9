// tcgen05 banded attention backward over the injected K/V entries: the chain
// rule of the forward in tc_attn_fwd.cu ("Maglev: Sliding Recurrent Memory",
// paper.rainbus.top, 方法步骤详情; window of W keys, self included).
//
// Head dim 64: one CTA per (128-key tile, head, batch row), looping over the
// 128-query tiles that see those keys (at most 5 for W = 512); head dim 128
// uses the persistent pipelined kernel further down.
//   S^T  = K Q^T,  dP^T = V dO^T                    (TMEM, fp32)
//   P^T  = exp(S^T * scale - LSE),  dS^T = P^T (dP^T - Delta) * scale
//   dV  += P^T dO,  dK += dS^T Q                    (TMEM accumulators)
//   dQ_i = dS K -> staged in shared memory, reduce-added (TMA, fp32) into a
//                  zeroed dQ accumulator
//   warp 0     TMA: K, V once; Q_i, dO_i per query tile
//   warp 1     tcgen05.mma issue
//   warps 2-9  two warps per TMEM lane quarter, each taking half of the 128
//              query columns of a key row: masked P^T and dS^T in registers,
//              written bf16 128B-swizzled into shared memory (K-major for the
//              dV / dK MMAs, read back MN-major as dS for the dQ MMA); then
//              half of the dQ drain: TMEM -> registers (R_S released at
//              once) -> the warp's own 4 KiB slices of the P^T / dS^T
//              buffers (free once the dQ MMA completed) -> one TMA
//              reduce-add per 32x32 fp32 block; finally dK, dV rows, rounded
//              to bf16.
//              Half-tiles inside every row's window skip the band mask.
//              LSE and Delta of each query tile are staged in shared memory.
// Delta = rowsum(dO * O) comes from the delta kernel. Every wait is bounded.
#include <cuda.h>

#include "launchers.h"
#include "tc_common.cuh"

namespace maglev {

cudaError_t make_tmap_tokens(CUtensorMap* m, const void* base, int B, int T, int H, int hd, uint32_t box_rows);
cudaError_t make_tmap_f32_tokens(CUtensorMap* m, void* base, int B, int T, int H, int hd, uint32_t box_rows);
int num_sms();

namespace {

using namespace tc;

constexpr int NUM_THREADS = 320;  // producer, MMA, 8 softmax warps
constexpr int SOFT_THREADS = 256;
constexpr float LOG2E = 1.4426950408889634f;

template <int HD>
struct BwdCfg {
  static constexpr int CH = HD / 64;
  static constexpr int TILE = 128 * HD * 2;  // 128 rows x hd bf16
  static constexpr int CHUNK = 128 * 128;    // 128 rows x 64 bf16
  static constexpr int PT = 128 * 128 * 2;   // 128 x 128 bf16 (P^T or dS^T)
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = TILE;
  static constexpr int OFF_Q = 2 * TILE;
  static constexpr int OFF_DO = 3 * TILE;
  static constexpr int OFF_P = 4 * TILE;
  static constexpr int OFF_DS = 4 * TILE + PT;
  static constexpr int OFF_LD = 4 * TILE + 2 * PT;  // [2][2][128] floats: LSE*log2e, Delta
  static constexpr int OFF_BAR = OFF_LD + 2 * 2 * 128 * 4;
  static constexpr size_t SMEM = 1024 + OFF_BAR + 256;
  // TMEM columns
  static constexpr uint32_t R_S = 0;     // S^T, later dQ_i
  static constexpr uint32_t R_DP = 128;  // dP^T
  static constexpr uint32_t R_DV = 256;
  static constexpr uint32_t R_DK = 384;
};

struct BwdParams {
  int B, T, H, W;
  float scale, scale_log2;
  const float* lse;    // [B,H,T] natural log
  const float* delta;  // [B,H,T]
  float* dq_acc;       // [B,T,H,hd] fp32, zeroed, rotated frame (written through tmDQ)
  bf16* dk_bar;        // [B,T,H,hd] bf16 (rounded from the fp32 accumulators)
  bf16* dv_bar;        // [B,T,H,hd] bf16
  int64_t spin_limit;
  int* err;
};

__device__ __forceinline__ void store_row_swizzled(uint8_t* tile, int r, const float* x, int c) {
  // 32 consecutive values x (columns 32c..32c+31) of row r into a 128B-swizzled
  // [128 rows x 128 cols] bf16 tile made of two 64-column chunks.
  const int ch = c >> 1;
#pragma unroll
  for (int gg = 0; gg < 4; ++gg) {
    const int g = (c & 1) * 4 + gg;
    uint4 w;
    w.x = pack_bf16(x[8 * gg + 0], x[8 * gg + 1]);
    w.y = pack_bf16(x[8 * gg + 2], x[8 * gg + 3]);
    w.z = pack_bf16(x[8 * gg + 4], x[8 * gg + 5]);
    w.w = pack_bf16(x[8 * gg + 6], x[8 * gg + 7]);
    *reinterpret_cast<uint4*>(tile + ch * 16384 + r * 128 + ((g ^ (r & 7)) << 4)) = w;
  }
}

template <int HD>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                       const __grid_constant__ CUtensorMap tmDQ, BwdParams p) {
  using C = BwdCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* qdo_full = bars + 1;
  uint64_t* qdo_empty = bars + 2;
  uint64_t* s_full = bars + 3;
  uint64_t* ds_full = bars + 4;
  uint64_t* dq_full = bars + 5;
  uint64_t* dq_empty = bars + 6;
  uint64_t* drain = bars + 7;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const Abort ab{abort_flag, p.err, p.spin_limit * 1000};
  const int kt = blockIdx.x * 128, h = blockIdx.y, b = blockIdx.z;
  const int last_q = min(p.T - 1, kt + 127 + p.W - 1);
  const int n_q = ((last_q & ~127) - kt) / 128 + 1;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(qdo_full, 1);
    mbar_init(qdo_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(ds_full, SOFT_THREADS);
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, SOFT_THREADS);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmDO);
    tma_prefetch_desc(&tmDQ);
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      mbar_arrive_expect_tx(kv_full, 2 * C::TILE);
#pragma unroll
      for (int c = 0; c < C::CH; ++c) {
        tma_load_4d(smem + C::OFF_K + c * C::CHUNK, &tmK, kv_full, 64 * c, h, kt, b);
        tma_load_4d(smem + C::OFF_V + c * C::CHUNK, &tmV, kv_full, 64 * c, h, kt, b);
      }
      bool armed = false;
      uint32_t last_par = 0;
      for (int i = 0; i < n_q; ++i) {
        if (!mbar_wait(qdo_empty, ((uint32_t)i & 1u) ^ 1u, ab)) break;
        mbar_arrive_expect_tx(qdo_full, 2 * C::TILE);
        armed = true;
        last_par = (uint32_t)i & 1u;
        const int qt = kt + 128 * i;
#pragma unroll
        for (int c = 0; c < C::CH; ++c) {
          tma_load_4d(smem + C::OFF_Q + c * C::CHUNK, &tmQ, qdo_full, 64 * c, h, qt, b);
          tma_load_4d(smem + C::OFF_DO + c * C::CHUNK, &tmDO, qdo_full, 64 * c, h, qt, b);
        }
      }
      mbar_drain(kv_full, 0, DRAIN_LIMIT_NS);
      if (armed) mbar_drain(qdo_full, last_par, DRAIN_LIMIT_NS);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t ID_S = idesc_bf16(128, 128, false, false);   // S^T, dP^T
      constexpr uint32_t ID_KV = idesc_bf16(128, HD, false, true);    // dV, dK
      constexpr uint32_t ID_Q = idesc_bf16(128, HD, true, true);      // dQ (A = dS, MN-major)
      const uint32_t k_addr = smem_u32(smem + C::OFF_K);
      const uint32_t v_addr = smem_u32(smem + C::OFF_V);
      const uint32_t q_addr = smem_u32(smem + C::OFF_Q);
      const uint32_t do_addr = smem_u32(smem + C::OFF_DO);
      const uint32_t pt_addr = smem_u32(smem + C::OFF_P);
      const uint32_t ds_addr = smem_u32(smem + C::OFF_DS);
      bool ok = mbar_wait(kv_full, 0, ab);
      for (int i = 0; i < n_q && ok; ++i) {
        const uint32_t par = (uint32_t)i & 1u;
        if (!mbar_wait(qdo_full, par, ab)) break;
        if (!mbar_wait(dq_empty, par ^ 1u, ab)) break;  // dQ_{i-1} drained from R_S
        tc_fence_after();
#pragma unroll
        for (int k16 = 0; k16 < HD / 16; ++k16) {
          const uint32_t off = (uint32_t)(k16 >> 2) * C::CHUNK;
          mma_ss(tmem + C::R_S, kmajor_desc(k_addr + off, k16 & 3), kmajor_desc(q_addr + off, k16 & 3), ID_S,
                 k16 > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int k16 = 0; k16 < HD / 16; ++k16) {
          const uint32_t off = (uint32_t)(k16 >> 2) * C::CHUNK;
          mma_ss(tmem + C::R_DP, kmajor_desc(v_addr + off, k16 & 3), kmajor_desc(do_addr + off, k16 & 3), ID_S,
                 k16 > 0 ? 1u : 0u);
        }
        mma_commit(s_full);
        if (!mbar_wait(ds_full, par, ab)) break;
        tc_fence_after();
        const uint32_t acc = i > 0 ? 1u : 0u;
#pragma unroll
        for (int k16 = 0; k16 < 8; ++k16) {  // K = 128 queries
          const uint64_t a = kmajor_desc(pt_addr + (uint32_t)(k16 >> 2) * C::CHUNK, k16 & 3);
          const uint64_t bq = sw128_desc(do_addr + (uint32_t)k16 * 2048u, (uint32_t)C::CHUNK, 1024u);
          mma_ss(tmem + C::R_DV, a, bq, ID_KV, (acc || k16 > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int k16 = 0; k16 < 8; ++k16) {
          const uint64_t a = kmajor_desc(ds_addr + (uint32_t)(k16 >> 2) * C::CHUNK, k16 & 3);
          const uint64_t bq = sw128_desc(q_addr + (uint32_t)k16 * 2048u, (uint32_t)C::CHUNK, 1024u);
          mma_ss(tmem + C::R_DK, a, bq, ID_KV, (acc || k16 > 0) ? 1u : 0u);
        }
        mma_commit(qdo_empty);
#pragma unroll
        for (int k16 = 0; k16 < 8; ++k16) {  // K = 128 keys
          const uint64_t a = sw128_desc(ds_addr + (uint32_t)k16 * 2048u, (uint32_t)C::CHUNK, 1024u);
          const uint64_t bk = sw128_desc(k_addr + (uint32_t)k16 * 2048u, (uint32_t)C::CHUNK, 1024u);
          mma_ss(tmem + C::R_S, a, bk, ID_Q, k16 > 0 ? 1u : 0u);
        }
        mma_commit(dq_full);
      }
      mma_commit(drain);
      mbar_drain(drain, 0, DRAIN_LIMIT_NS);
    }
  } else {
    // -------------------------------------------------------------- softmax-backward / drains
    const int q4 = warp & 3;
    const int half = (warp - 2) >> 2;  // which 64 of the 128 columns this warp takes
    const int r = q4 * 32 + lane;      // TMEM lane: key row (S^T, dV, dK) / query row (dQ)
    const int st = threadIdx.x - 64;   // 0..255 among the softmax threads
    const int kj = kt + r;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const int64_t lrow = ((int64_t)b * p.H + h) * p.T;
    float* sLD = reinterpret_cast<float*>(smem + C::OFF_LD);
    uint8_t* sPT = smem + C::OFF_P;
    uint8_t* sDS = smem + C::OFF_DS;
    bool ok = true;
    float pre_l = 0.f, pre_d = 0.f;  // this thread's LSE / Delta entry of the next tile
    auto fetch = [&](int i) {
      const int qi = kt + 128 * i + (st & 127);
      const bool in = qi < p.T;
      pre_l = in ? p.lse[lrow + qi] * LOG2E : 0.f;
      pre_d = in ? p.delta[lrow + qi] : 0.f;
    };
    fetch(0);
    for (int i = 0; i < n_q; ++i) {
      const uint32_t par = (uint32_t)i & 1u;
      const int qt = kt + 128 * i;
      float* lds = sLD + (i & 1) * 256;  // [0,128): LSE*log2e, [128,256): Delta
      if (st < 128) lds[st] = pre_l;
      else lds[st] = pre_d;
      // every softmax thread reaches this barrier on every tile, aborted or not
      asm volatile("bar.sync 1, %0;" ::"n"(SOFT_THREADS) : "memory");
      if (i + 1 < n_q) fetch(i + 1);
      ok = ok && warp_wait(s_full, par, ab);
      if (!ok) continue;
      tc_fence_after();
      if (i > 0) {  // the previous tile's dQ reduce has read its staging (our P^T / dS^T slices)
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
      }
      const int lo = kj - qt;  // first valid column (query >= key)
      const int hi = min(kj + p.W - 1, p.T - 1) - qt;
      const int kw = kt + 32 * q4;  // first key row of this warp
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * half + cc;  // 32-column chunk index
        uint32_t sv[32], dv[32];
        tmem_ld32(tmem + lane_off + C::R_S + 32u * (uint32_t)c, sv);
        tmem_ld32(tmem + lane_off + C::R_DP + 32u * (uint32_t)c, dv);
        tmem_wait_ld();
        // queries qt+32c .. +31 inside the window of each of this warp's keys
        const int q0 = qt + 32 * c;
        const bool full = q0 >= kw + 31 && q0 + 31 <= kw + p.W - 1 && q0 + 31 <= p.T - 1 && kw + 31 < p.T;
        float pt[32], ds[32];
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 L = *reinterpret_cast<const float4*>(lds + 32 * c + 4 * e4);
          const float4 D = *reinterpret_cast<const float4*>(lds + 128 + 32 * c + 4 * e4);
          const float Ls[4] = {L.x, L.y, L.z, L.w};
          const float Ds[4] = {D.x, D.y, D.z, D.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int e = 4 * e4 + u;
            const int col = 32 * c + e;
            const float y = ex2_fast(fmaf(__uint_as_float(sv[e]), p.scale_log2, -Ls[u]));
            const float pe = (full || (col >= lo && col <= hi && kj < p.T)) ? y : 0.f;
            pt[e] = pe;
            ds[e] = pe * (__uint_as_float(dv[e]) - Ds[u]) * p.scale;
          }
        }
        store_row_swizzled(sPT, r, pt, c);
        store_row_swizzled(sDS, r, ds, c);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(ds_full);
      // dQ_i = dS K: lane r is query qt + r; this warp drains hd columns [64*half, 64*half+64)
      ok = warp_wait(dq_full, par, ab);
      if (!ok) continue;
      tc_fence_after();
      // this warp's dQ block: query rows qt+32*q4 .. +31, channels [32*c0, 32*c0 + 32*NC)
      constexpr int NC = HD / 64;
      const int c0 = half * NC;
      uint32_t v[NC][32];
#pragma unroll
      for (int cc = 0; cc < NC; ++cc) tmem_ld32(tmem + lane_off + C::R_S + 32u * (uint32_t)(c0 + cc), v[cc]);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(dq_empty);  // R_S may take S^T of the next tile
      // stage each 32x32 fp32 block in this warp's slice of P^T (cc = 0) / dS^T
      // (cc = 1): rows of 128 B, 16-byte chunks swizzled by row (TMA 128B swizzle)
#pragma unroll
      for (int cc = 0; cc < NC; ++cc) {
        uint8_t* stage = (cc == 0 ? sPT : sDS) + half * 16384 + q4 * 4096;
#pragma unroll
        for (int g = 0; g < 8; ++g)
          *reinterpret_cast<uint4*>(stage + lane * 128 + ((g ^ (lane & 7)) << 4)) =
              make_uint4(v[cc][4 * g], v[cc][4 * g + 1], v[cc][4 * g + 2], v[cc][4 * g + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && qt + 32 * q4 < p.T) {
#pragma unroll
        for (int cc = 0; cc < NC; ++cc)
          tma_reduce_add_4d(&tmDQ, (cc == 0 ? sPT : sDS) + half * 16384 + q4 * 4096, 32 * (c0 + cc), h,
                            qt + 32 * q4, b);
        bulk_commit();
      }
    }
    if (lane == 0) bulk_wait_all();  // dQ reductions complete before the CTA leaves
    __syncwarp();
    if (__all_sync(0xffffffffu, ok) && n_q > 0) {
      // all MMAs are complete (dq_full of the last tile was waited): dK, dV rows
      tc_fence_after();
      // tcgen05.ld is warp-collective: every lane loads, only rows < T store
      const bool row_ok = kj < p.T;
      const int64_t row = (((int64_t)b * p.T + (row_ok ? kj : 0)) * p.H + h) * HD;
#pragma unroll 1
      for (int c = half * (HD / 64); c < (half + 1) * (HD / 64); ++c) {
        uint32_t v[32];
#pragma unroll
        for (int t = 0; t < 2; ++t) {  // dK, then dV
          tmem_ld32(tmem + lane_off + (t == 0 ? C::R_DK : C::R_DV) + 32u * (uint32_t)c, v);
          tmem_wait_ld();
          bf16* dst = (t == 0 ? p.dk_bar : p.dv_bar) + row + 32 * c;
          if (row_ok) {
#pragma unroll
            for (int g = 0; g < 4; ++g)
              *reinterpret_cast<uint4*>(dst + 8 * g) = make_uint4(
                  pack_bf16(__uint_as_float(v[8 * g + 0]), __uint_as_float(v[8 * g + 1])),
                  pack_bf16(__uint_as_float(v[8 * g + 2]), __uint_as_float(v[8 * g + 3])),
                  pack_bf16(__uint_as_float(v[8 * g + 4]), __uint_as_float(v[8 * g + 5])),
                  pack_bf16(__uint_as_float(v[8 * g + 6]), __uint_as_float(v[8 * g + 7])));
          }
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}


// =========================================================================== pipelined, hd = 128
// Persistent: one CTA per SM walks units (128-key tile, head, batch row),
// ranked by decreasing cost and dealt in a snake order. A unit visits the
// 64-query half-tiles that see its keys (at most 10 for W = 512); g counts
// half-tiles over all of the CTA's units.
//   S^T_g  = K Q_g^T, dP^T_g = V dO_g^T   128 keys x 64 queries, TMEM S, DP (one each)
//   P^T_g                                  bf16, TMEM PT[g&1] (the A operand of dV)
//   dS^T_g                                 bf16, shared memory buffer g&1
//   dV += P^T_g dO_g, dK += dS^T_g Q_g     TMEM accumulators (whole unit)
//   dQ^T_g = K^T dS^T_g                    128 channels x 64 queries, TMEM DQ
// The softmax warps release S / dP as soon as their tcgen05.ld of half-tile g
// has completed, so the MMA warp issues S/dP of g+1 at once and the tensor
// core computes it (and then dV/dK/dQ of g) while the softmax warps turn g's
// scores into P and dS. After storing P/dS of g the softmax warps drain
// dQ^T_{g-1}: TMEM -> registers (DQ released at once) -> the warp's 2 KiB
// slice of a staging buffer of its own -> one 16 x 32 fp32 TMA reduce-add per
// warp. An SM's reductions to global memory drain at only ~25 B/clk (the 32
// KiB of a half-tile take ~1300 cycles); a slice is next written a whole
// half-tile later. Q/dO arrive through a 3-deep ring; K/V once per unit.
constexpr int PIPE_SOFT_WARPS = 16;                  // 4 per TMEM lane quarter
constexpr int PIPE_SOFT_THREADS = 32 * PIPE_SOFT_WARPS;
constexpr int PIPE_THREADS = 64 + PIPE_SOFT_THREADS;  // producer, MMA, softmax warps

template <int HD>
struct PipeCfg {
  static_assert(HD == 128, "pipelined backward is written for 128 channels");
  static constexpr int CH = HD / 64;
  static constexpr int KV_TILE = 128 * HD * 2;  // 128 keys
  static constexpr int KCHUNK = 128 * 128;      // 128 rows x 64 bf16
  static constexpr int QH = 64 * HD * 2;        // 64 queries
  static constexpr int QCHUNK = 64 * 128;       // 64 rows x 64 bf16
  static constexpr int NQ = 3;                  // Q / dO ring depth
  static constexpr int PH = 128 * 64 * 2;       // [128 keys x 64 queries] bf16
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = KV_TILE;
  static constexpr int OFF_Q = 2 * KV_TILE;
  static constexpr int OFF_DO = OFF_Q + NQ * QH;
  static constexpr int OFF_X = OFF_DO + NQ * QH;  // dQ^T staging: 16 slices of 16 queries x 32 channels fp32
  static constexpr int OFF_DS = OFF_X + 2 * PH;   // [2]
  static constexpr int OFF_LD = OFF_DS + 2 * PH;  // [16 warps][32] floats: LSE*log2e (16), Delta (16)
  static constexpr int OFF_BAR = OFF_LD + 16 * 32 * 4;
  static constexpr size_t SMEM = OFF_BAR + 256;   // base is 1024-aligned (checked in the kernel)
  // TMEM columns: S 64, dP 64, dQ 64, P^T 2 x 32 (bf16 pairs), dV 128, dK 128
  static constexpr uint32_t T_S = 0, T_DP = 64, T_DQ = 128, T_PT = 192, T_DV = 256, T_DK = 384;
};

struct PipeParams {
  BwdParams b;
  int n_ktiles, n_units;
};

struct KUnit {
  int kt, h, b, nh;
};

// Rank r in decreasing cost: key tiles from the first (the last tiles see
// fewer queries); snake over the CTAs per pass. -1 past the end.
__device__ __forceinline__ int kunit_rank(const PipeParams& p, int k) {
  const int G = (int)gridDim.x, c = (int)blockIdx.x;
  const int r = k * G + ((k & 1) ? G - 1 - c : c);
  return r < p.n_units ? r : -1;
}

__device__ __forceinline__ KUnit kunit_of(const PipeParams& p, int r) {
  KUnit x;
  const int hb = p.b.H * p.b.B;
  x.kt = (r / hb) * 128;
  x.h = (r % hb) % p.b.H;
  x.b = (r % hb) / p.b.H;
  const int last_q = min(p.b.T - 1, x.kt + 127 + p.b.W - 1);
  x.nh = ((last_q & ~63) - x.kt) / 64 + 1;
  return x;
}

template <int HD>
__global__ void __launch_bounds__(PIPE_THREADS, 1)
    attn_bwd_pipe_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                         const __grid_constant__ CUtensorMap tmDQ, PipeParams pp) {
  using C = PipeCfg<HD>;
  const BwdParams& p = pp.b;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {  // the swizzled tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) record_error(p.err, DEV_TIMEOUT);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;
  uint64_t* q_full = bars + 2;     // [3]
  uint64_t* q_empty = bars + 5;    // [3]
  uint64_t* s_full = bars + 8;     // S / dP of the current half-tile computed
  uint64_t* s_free = bars + 9;     // ... and loaded by every softmax thread
  uint64_t* p_full = bars + 10;    // [2]
  uint64_t* dq_full = bars + 12;
  uint64_t* dq_empty = bars + 14;
  uint64_t* acc_full = bars + 16;
  uint64_t* acc_empty = bars + 17;
  uint64_t* drain = bars + 18;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 19);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const Abort ab{abort_flag, p.err, p.spin_limit * 1000};

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int s = 0; s < 3; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, PIPE_SOFT_THREADS);
    for (int s = 0; s < 2; ++s) mbar_init(&p_full[s], PIPE_SOFT_THREADS);
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, PIPE_SOFT_THREADS);
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, PIPE_SOFT_THREADS);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmDO);
    tma_prefetch_desc(&tmDQ);
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      uint32_t kv_armed = 0, kv_par = 0, q_armed = 0, q_par = 0;
      int g = 0, n = 0;
      bool ok = true;
      for (int u = kunit_rank(pp, 0); u >= 0 && ok; u = kunit_rank(pp, ++n)) {
        const KUnit x = kunit_of(pp, u);
        for (int j = 0; j < x.nh; ++j, ++g) {
          const int s = g % 3;
          const uint32_t ph = (uint32_t)(g / 3) & 1u;
          if (!mbar_wait(&q_empty[s], ph ^ 1u, ab)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&q_full[s], 2 * C::QH);
          q_armed |= 1u << s;
          q_par = (q_par & ~(1u << s)) | (ph << s);
          const int qt = x.kt + 64 * j;
#pragma unroll
          for (int c = 0; c < C::CH; ++c) {
            tma_load_4d(smem + C::OFF_Q + s * C::QH + c * C::QCHUNK, &tmQ, &q_full[s], 64 * c, x.h, qt, x.b);
            tma_load_4d(smem + C::OFF_DO + s * C::QH + c * C::QCHUNK, &tmDO, &q_full[s], 64 * c, x.h, qt, x.b);
          }
          if (j == 0) {  // the unit's K/V, once the previous unit's MMAs are done with them
            const uint32_t kph = (uint32_t)n & 1u;
            if (!mbar_wait(kv_empty, kph ^ 1u, ab)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(kv_full, 2 * C::KV_TILE);
            kv_armed = 1;
            kv_par = kph;
#pragma unroll
            for (int c = 0; c < C::CH; ++c) {
              tma_load_4d(smem + C::OFF_K + c * C::KCHUNK, &tmK, kv_full, 64 * c, x.h, x.kt, x.b);
              tma_load_4d(smem + C::OFF_V + c * C::KCHUNK, &tmV, kv_full, 64 * c, x.h, x.kt, x.b);
            }
          }
        }
      }
      if (kv_armed) mbar_drain(kv_full, kv_par, DRAIN_LIMIT_NS);
      for (int s = 0; s < 3; ++s)
        if (q_armed & (1u << s)) mbar_drain(&q_full[s], (q_par >> s) & 1u, DRAIN_LIMIT_NS);
    }
  } else if (warp == 1) {
    {
      // ------------------------------------------------------------ MMA issuer
      // Every lane runs the loop and the waits, so descriptors and counters are
      // warp-uniform; the elected lane issues each batch of MMAs and commits.
      constexpr uint32_t ID_S = idesc_bf16(128, 64, false, false);  // S^T, dP^T: 128 keys x 64 queries
      constexpr uint32_t ID_KV = idesc_bf16(128, HD, false, true);  // dV, dK: 128 keys x hd
      constexpr uint32_t ID_DQ = idesc_bf16(HD, 64, true, true);    // dQ^T: hd x 64 queries
      const uint32_t k_addr = smem_u32(smem + C::OFF_K);
      // base descriptors: each MMA's operand is a constant offset from these
      const uint64_t kd0 = kmajor_desc(k_addr, 0), vd0 = kmajor_desc(smem_u32(smem + C::OFF_V), 0);
      const uint64_t kmn = sw128_desc(k_addr, (uint32_t)C::KCHUNK, 1024u);  // K read MN-major (dQ^T)
      // S^T_gs, dP^T_gs, once Q/dO have arrived and the softmax warps have
      // loaded S/dP of half-tile gs-1
      auto issue_sdp = [&](int gs) -> bool {
        const int s = gs % 3;
        if (!warp_wait(&q_full[s], (uint32_t)(gs / 3) & 1u, ab)) return false;
        if (gs >= 1 && !warp_wait(s_free, (uint32_t)(gs - 1) & 1u, ab)) return false;
        tc_fence_after();
        const uint64_t qd = kmajor_desc(smem_u32(smem + C::OFF_Q + s * C::QH), 0);
        const uint64_t dod = kmajor_desc(smem_u32(smem + C::OFF_DO + s * C::QH), 0);
        if (elect_one()) {
#pragma unroll
          for (int k16 = 0; k16 < HD / 16; ++k16) {
            const uint32_t ka = (uint32_t)(k16 >> 2) * C::KCHUNK + (k16 & 3) * 32u;
            const uint32_t qa = (uint32_t)(k16 >> 2) * C::QCHUNK + (k16 & 3) * 32u;
            mma_ss(tmem + C::T_S, desc_at(kd0, ka), desc_at(qd, qa), ID_S, k16 > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int k16 = 0; k16 < HD / 16; ++k16) {
            const uint32_t ka = (uint32_t)(k16 >> 2) * C::KCHUNK + (k16 & 3) * 32u;
            const uint32_t qa = (uint32_t)(k16 >> 2) * C::QCHUNK + (k16 & 3) * 32u;
            mma_ss(tmem + C::T_DP, desc_at(vd0, ka), desc_at(dod, qa), ID_S, k16 > 0 ? 1u : 0u);
          }
          mma_commit(s_full);
        }
        __syncwarp();
        return true;
      };
      // dV, dK and dQ^T of half-tile gr (local index jr of unit nr), once the
      // softmax warps have stored its P^T (TMEM) / dS^T (shared memory)
      auto issue_rest = [&](int gr, int jr, int nr) -> bool {
        const int s = gr % 3, buf = gr & 1;
        if (!warp_wait(&p_full[buf], (uint32_t)(gr >> 1) & 1u, ab)) return false;
        // the first dV/dK of a unit overwrites the accumulators: the previous
        // unit's epilogue must have read them
        if (jr == 0 && !warp_wait(acc_empty, ((uint32_t)nr & 1u) ^ 1u, ab)) return false;
        tc_fence_after();
        const uint32_t ds_addr = smem_u32(smem + C::OFF_DS + buf * C::PH);
        const uint32_t pt = tmem + C::T_PT + 32u * (uint32_t)buf;
        const uint64_t dsd = kmajor_desc(ds_addr, 0);
        const uint64_t domn = sw128_desc(smem_u32(smem + C::OFF_DO + s * C::QH), (uint32_t)C::QCHUNK, 1024u);
        const uint64_t qmn = sw128_desc(smem_u32(smem + C::OFF_Q + s * C::QH), (uint32_t)C::QCHUNK, 1024u);
        const uint64_t dsmn = sw128_desc(ds_addr, (uint32_t)C::PH, 1024u);
        if (elect_one()) {
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16)  // K = 64 queries, 8 TMEM columns each
            mma_ts(tmem + C::T_DV, pt + 8u * (uint32_t)k16, desc_at(domn, k16 * 2048u), ID_KV,
                   (jr > 0 || k16 > 0) ? 1u : 0u);
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16)
            mma_ss(tmem + C::T_DK, desc_at(dsd, k16 * 32u), desc_at(qmn, k16 * 2048u), ID_KV,
                   (jr > 0 || k16 > 0) ? 1u : 0u);
          mma_commit(&q_empty[s]);
        }
        __syncwarp();
        // DQ held dQ^T of half-tile gr-1, drained while dV / dK of gr run
        if (gr >= 1 && !warp_wait(dq_empty, (uint32_t)(gr - 1) & 1u, ab)) return false;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int k16 = 0; k16 < 8; ++k16)  // K = 128 keys
            mma_ss(tmem + C::T_DQ, desc_at(kmn, k16 * 2048u), desc_at(dsmn, k16 * 2048u), ID_DQ,
                   k16 > 0 ? 1u : 0u);
          mma_commit(dq_full);
        }
        __syncwarp();
        return true;
      };
      int g = 0, n = 0;
      bool ok = true;
      for (int u = kunit_rank(pp, 0); u >= 0 && ok; u = kunit_rank(pp, ++n)) {
        const KUnit x = kunit_of(pp, u);
        if (!warp_wait(kv_full, (uint32_t)n & 1u, ab)) break;
        // S/dP of g+1 go to the tensor core ahead of dV/dK/dQ of g
        for (int j = 0; j < x.nh; ++j, ++g) {
          if (!issue_sdp(g) || (j > 0 && !issue_rest(g - 1, j - 1, n))) {
            ok = false;
            break;
          }
        }
        if (!ok || !issue_rest(g - 1, x.nh - 1, n)) break;
        if (elect_one()) {
          mma_commit(acc_full);
          mma_commit(kv_empty);  // the next unit's K/V may overwrite this one's
        }
        __syncwarp();
      }
      if (elect_one()) {  // the issuing lane's MMAs complete before TMEM is released
        mma_commit(drain);
        mbar_drain(drain, 0, DRAIN_LIMIT_NS);
      }
      __syncwarp();
    }
  } else {
    // -------------------------------------------------------------- softmax-backward / drains
    // 16 warps: warp w reads TMEM lane quarter q4 = w % 4 (key rows / dQ^T
    // channels 32*q4 ..) and owns the 16 query columns [16*cs, 16*cs + 16) of
    // each 64-query half-tile, cs = (w - 2) / 4.
    const int q4 = warp & 3;
    const int cs = (warp - 2) >> 2;
    const int r = q4 * 32 + lane;      // TMEM lane: key row (S^T, dV, dK) / channel (dQ^T)
    const int w16 = q4 + 4 * cs;       // this warp's 2 KiB staging slice
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    // This warp's LSE (log2 units) and Delta of its 16 query columns of the
    // current half-tile: lane l < 16 holds column l's LSE, lane 16 + l its Delta.
    float* lds = reinterpret_cast<float*>(smem + C::OFF_LD) + 32 * w16;
    bool ok = true;
    // Each lane loads its value of the next half-tile one half-tile ahead and
    // touches it only after the current half-tile's math, so no thread stalls
    // on the load's latency and no warp waits for another.
    float pre = 0.f;
    auto fetch = [&](const KUnit& x, int j) {
      const int qi = x.kt + 64 * j + 16 * cs + (lane & 15);
      const int64_t lrow = ((int64_t)x.b * p.H + x.h) * p.T;
      pre = 0.f;
      if (qi < p.T) pre = __ldg((lane < 16 ? p.lse : p.delta) + lrow + qi);
    };
    auto publish = [&]() {  // every lane of the warp has finished reading the previous values
      __syncwarp();
      lds[lane] = lane < 16 ? pre * LOG2E : pre;
      __syncwarp();
    };
    // dQ^T of half-tile gd (unit xd, its local index jd): lanes are channels,
    // this warp's 16 columns are queries xd.kt + 64*jd + 16*cs ...
    auto drain_dq = [&](int gd, const KUnit& xd, int jd) {
      ok = ok && warp_wait(dq_full, (uint32_t)gd & 1u, ab);
      if (!ok) return;
      tc_fence_after();
      uint32_t v[16];
      tmem_ld16(tmem + lane_off + C::T_DQ + 16u * (uint32_t)cs, v);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(dq_empty);  // DQ may take dQ^T of half-tile gd + 1
      // the warp's reduce-add of half-tile gd-1 has read its slice
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
      // box of 16 query rows x 32 channels (128 B rows, 16-byte chunks swizzled by row)
      uint8_t* slice = smem + C::OFF_X + w16 * 2048;
#pragma unroll
      for (int c = 0; c < 16; ++c)
        *reinterpret_cast<uint32_t*>(slice + c * 128 + ((((lane >> 2) ^ (c & 7))) << 4) + (lane & 3) * 4) = v[c];
      fence_proxy_async_smem();
      __syncwarp();
      const int q0 = xd.kt + 64 * jd + 16 * cs;
      if (lane == 0 && q0 < p.T && MAGLEV_CHECK(p.err, q0 >= 0 && xd.h < p.H && xd.b < p.B)) {  // none past the end
        tma_reduce_add_4d(&tmDQ, slice, 32 * q4, xd.h, q0, xd.b);
        bulk_commit();
      }
    };
    int g = 0, n = 0;
    KUnit xp{0, 0, 0, 0};  // unit of half-tile g-1
    int jp = 0;            // its local index
    {
      const int u0 = kunit_rank(pp, 0);
      if (u0 >= 0) fetch(kunit_of(pp, u0), 0);
      publish();  // LSE / Delta of half-tile 0
    }
    for (int u = kunit_rank(pp, 0); u >= 0; u = kunit_rank(pp, ++n)) {
      const KUnit x = kunit_of(pp, u);
      const int kj = x.kt + r;
      const int kw = x.kt + 32 * q4;  // first key row of this warp
      for (int j = 0; j < x.nh; ++j, ++g) {
        const int buf = g & 1;
        const int qt = x.kt + 64 * j;
        if (j + 1 < x.nh) {  // LSE / Delta of half-tile g+1, stored below
          fetch(x, j + 1);
        } else {
          const int un = kunit_rank(pp, n + 1);
          if (un >= 0) fetch(kunit_of(pp, un), 0);
        }
        ok = ok && warp_wait(s_full, (uint32_t)g & 1u, ab);
        float pt[16], ds[16];
        if (ok) {
          tc_fence_after();
          uint32_t sv[16], dv[16];
          tmem_ld16(tmem + lane_off + C::T_S + 16u * cs, sv);
          tmem_ld16(tmem + lane_off + C::T_DP + 16u * cs, dv);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(s_free);  // S / dP may take half-tile g + 1
          const int q0 = qt + 16 * cs;  // first query column of this warp
          // every (key, query) of this warp's 32 x 16 block inside the window
          const bool full = q0 >= kw + 31 && q0 + 15 <= kw + p.W - 1 && q0 + 15 <= p.T - 1 && kw + 31 < p.T;
          if (full) {
#pragma unroll
            for (int e4 = 0; e4 < 4; ++e4) {
              const float4 L = *reinterpret_cast<const float4*>(lds + 4 * e4);
              const float4 D = *reinterpret_cast<const float4*>(lds + 16 + 4 * e4);
              const float Ls[4] = {L.x, L.y, L.z, L.w};
              const float Ds[4] = {D.x, D.y, D.z, D.w};
#pragma unroll
              for (int uu = 0; uu < 4; ++uu) {
                const int e = 4 * e4 + uu;
                const float pe = ex2_fast(fmaf(__uint_as_float(sv[e]), p.scale_log2, -Ls[uu]));
                pt[e] = pe;
                ds[e] = pe * (__uint_as_float(dv[e]) - Ds[uu]) * p.scale;
              }
            }
          } else {
            const int lo = kj - q0;  // query >= key
            const int hi = min(kj + p.W - 1, p.T - 1) - q0;
#pragma unroll
            for (int e4 = 0; e4 < 4; ++e4) {
              const float4 L = *reinterpret_cast<const float4*>(lds + 4 * e4);
              const float4 D = *reinterpret_cast<const float4*>(lds + 16 + 4 * e4);
              const float Ls[4] = {L.x, L.y, L.z, L.w};
              const float Ds[4] = {D.x, D.y, D.z, D.w};
#pragma unroll
              for (int uu = 0; uu < 4; ++uu) {
                const int e = 4 * e4 + uu;
                const float y = ex2_fast(fmaf(__uint_as_float(sv[e]), p.scale_log2, -Ls[uu]));
                const float pe = (e >= lo && e <= hi && kj < p.T) ? y : 0.f;
                pt[e] = pe;
                ds[e] = pe * (__uint_as_float(dv[e]) - Ds[uu]) * p.scale;
              }
            }
          }
        }
        publish();  // LSE / Delta of half-tile g+1
        // Buffers g&1 (P^T in TMEM, dS^T in shared memory) held half-tile
        // g-2, whose MMAs completed before this warp drained dQ^T_{g-2}.
        if (ok) {
          // P^T row r (this lane's key), queries 16*cs .. +15 as 8 bf16 pairs
          // in TMEM columns PT[buf] + 8*cs ..; dS^T into shared memory: 16-byte
          // chunks 2*cs and 2*cs + 1 of the 128 B row.
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) pk[i] = pack_bf16(pt[2 * i], pt[2 * i + 1]);
          tmem_st8(tmem + lane_off + C::T_PT + 32u * (uint32_t)buf + 8u * (uint32_t)cs, pk);
          uint8_t* drow = smem + C::OFF_DS + buf * C::PH + r * 128;
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int chunk = ((2 * cs + h2) ^ (r & 7)) << 4;
            *reinterpret_cast<uint4*>(drow + chunk) =
                make_uint4(pack_bf16(ds[8 * h2 + 0], ds[8 * h2 + 1]), pack_bf16(ds[8 * h2 + 2], ds[8 * h2 + 3]),
                           pack_bf16(ds[8 * h2 + 4], ds[8 * h2 + 5]), pack_bf16(ds[8 * h2 + 6], ds[8 * h2 + 7]));
          }
          tmem_wait_st();
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(&p_full[buf]);
        }
        if (g >= 1) drain_dq(g - 1, xp, jp);
        xp = x;
        jp = j;
      }
      // epilogue of the unit: dK, dV rows, rounded to bf16. Each warp's 32 rows
      // x 32 columns go through its own 2 KiB of the dS^T buffers (free: the
      // unit's MMAs are complete), so that every global store covers whole
      // 64-byte row pieces.
      ok = ok && warp_wait(acc_full, (uint32_t)n & 1u, ab);
      if (ok) {
        tc_fence_after();
        uint8_t* stg = smem + C::OFF_DS + w16 * 2048;       // [32 rows][32 bf16], 16-byte chunks swizzled
        const int64_t tstride = (int64_t)p.H * HD;          // elements between consecutive tokens
        const int64_t col0 = (int64_t)x.h * HD + 32 * cs;
#pragma unroll
        for (int t = 0; t < 2; ++t) {  // dK, then dV
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + (t == 0 ? C::T_DK : C::T_DV) + 32u * (uint32_t)cs, v);
          tmem_wait_ld();
          if (t == 1) {  // both accumulators are in registers or stored: the next unit may overwrite them
            tc_fence_before();
            mbar_arrive(acc_empty);
          }
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4)
            *reinterpret_cast<uint4*>(stg + lane * 64 + ((c4 ^ ((lane >> 1) & 3)) << 4)) = make_uint4(
                pack_bf16(__uint_as_float(v[8 * c4 + 0]), __uint_as_float(v[8 * c4 + 1])),
                pack_bf16(__uint_as_float(v[8 * c4 + 2]), __uint_as_float(v[8 * c4 + 3])),
                pack_bf16(__uint_as_float(v[8 * c4 + 4]), __uint_as_float(v[8 * c4 + 5])),
                pack_bf16(__uint_as_float(v[8 * c4 + 6]), __uint_as_float(v[8 * c4 + 7])));
          __syncwarp();
          bf16* dst = t == 0 ? p.dk_bar : p.dv_bar;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int rr = 8 * i + (lane >> 2), ch = lane & 3;  // row of the warp's 32, 16-byte chunk
            const uint4 w = *reinterpret_cast<const uint4*>(stg + rr * 64 + ((ch ^ ((rr >> 1) & 3)) << 4));
            const int key = x.kt + 32 * q4 + rr;
            if (key < p.T && MAGLEV_CHECK(p.err, x.b < p.B && col0 + 8 * ch + 8 <= tstride))
              *reinterpret_cast<uint4*>(dst + ((int64_t)x.b * p.T + key) * tstride + col0 + 8 * ch) = w;
          }
          __syncwarp();
        }
      }
      // the next unit's dS^T rows overwrite other warps' staging: every warp is
      // past its epilogue first (reached by every softmax thread, aborted or not)
      asm volatile("bar.sync 1, %0;" ::"n"(PIPE_SOFT_THREADS) : "memory");
    }
    if (g >= 1) drain_dq(g - 1, xp, jp);
    if (lane == 0) bulk_wait_all();  // dQ reductions complete before the CTA leaves
    __syncwarp();
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_attn_bwd_tc(const SwaShape& s, const void* q_rot, const void* k_bar, const void* v_bar,
                               const void* dout, const float* lse, const float* delta, float* dq_acc,
                               void* dk_bar, void* dv_bar, int64_t spin_limit, int* err, cudaStream_t st) {
  CUtensorMap tq, tk, tv, tdo;
  cudaError_t e;
  if ((e = make_tmap_tokens(&tq, q_rot, s.B, s.T, s.H, s.hd, 128)) != cudaSuccess) return e;
  if ((e = make_tmap_tokens(&tk, k_bar, s.B, s.T, s.H, s.hd, 128)) != cudaSuccess) return e;
  if ((e = make_tmap_tokens(&tv, v_bar, s.B, s.T, s.H, s.hd, 128)) != cudaSuccess) return e;
  if ((e = make_tmap_tokens(&tdo, dout, s.B, s.T, s.H, s.hd, 128)) != cudaSuccess) return e;
  CUtensorMap tdq;  // dQ reduce-add boxes: 32 query rows (head dim 64), 16 (pipelined kernel)
  if ((e = make_tmap_f32_tokens(&tdq, dq_acc, s.B, s.T, s.H, s.hd, s.hd == 128 ? 16 : 32)) != cudaSuccess) return e;
  BwdParams p;
  p.B = s.B;
  p.T = s.T;
  p.H = s.H;
  p.W = s.W;
  p.scale = 1.0f / sqrtf((float)s.hd);
  p.scale_log2 = LOG2E * p.scale;
  p.lse = lse;
  p.delta = delta;
  p.dq_acc = dq_acc;
  p.dk_bar = static_cast<bf16*>(dk_bar);
  p.dv_bar = static_cast<bf16*>(dv_bar);
  p.spin_limit = spin_limit;
  p.err = err;
  dim3 grid((unsigned)((s.T + 127) / 128), (unsigned)s.H, (unsigned)s.B);
  if (s.hd == 128) {
    CUtensorMap tq64, tdo64;  // Q / dO in 64-row boxes for the half-tiles
    if ((e = make_tmap_tokens(&tq64, q_rot, s.B, s.T, s.H, s.hd, 64)) != cudaSuccess) return e;
    if ((e = make_tmap_tokens(&tdo64, dout, s.B, s.T, s.H, s.hd, 64)) != cudaSuccess) return e;
    PipeParams pp;
    pp.b = p;
    pp.n_ktiles = (s.T + 127) / 128;
    pp.n_units = pp.n_ktiles * s.H * s.B;
    const unsigned pgrid = (unsigned)(pp.n_units < num_sms() ? pp.n_units : num_sms());
    auto k = attn_bwd_pipe_kernel<128>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PipeCfg<128>::SMEM);
    if (e != cudaSuccess) return e;
    k<<<pgrid, PIPE_THREADS, PipeCfg<128>::SMEM, st>>>(tq64, tk, tv, tdo64, tdq, pp);
  } else if (s.hd == 64) {
    auto k = attn_bwd_tc_kernel<64>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)BwdCfg<64>::SMEM);
    if (e != cudaSuccess) return e;
    k<<<grid, NUM_THREADS, BwdCfg<64>::SMEM, st>>>(tq, tk, tv, tdo, tdq, p);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace maglev
