// tcgen05 banded attention backward over the injected K/V entries: the chain
// rule of the forward in tc_attn_fwd.cu ("Maglev: Sliding Recurrent Memory",
// paper.rainbus.top, 方法步骤详情; window of W keys, self included).
//
// One CTA per (128-key tile, head, batch row), looping over the 128-query
// tiles that see those keys (at most 5 for W = 512):
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
//              reduce-add per 32x32 fp32 block; finally dK, dV rows in fp32.
//              Half-tiles inside every row's window skip the band mask.
//              LSE and Delta of each query tile are staged in shared memory.
// Delta = rowsum(dO * O) comes from the delta kernel. Every wait is bounded.
#include <cuda.h>

#include "launchers.h"
#include "tc_common.cuh"

namespace maglev {

cudaError_t make_tmap_tokens(CUtensorMap* m, const void* base, int B, int T, int H, int hd, uint32_t box_rows);
cudaError_t make_tmap_f32_tokens(CUtensorMap* m, void* base, int B, int T, int H, int hd);

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
  float* dk_bar;       // [B,T,H,hd] fp32
  float* dv_bar;       // [B,T,H,hd] fp32
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
        tmem_ld32(tmem + lane_off + C::R_DK + 32u * (uint32_t)c, v);
        tmem_wait_ld();
        if (row_ok) {
#pragma unroll
          for (int g = 0; g < 8; ++g)
            *reinterpret_cast<float4*>(p.dk_bar + row + 32 * c + 4 * g) =
                make_float4(__uint_as_float(v[4 * g]), __uint_as_float(v[4 * g + 1]),
                            __uint_as_float(v[4 * g + 2]), __uint_as_float(v[4 * g + 3]));
        }
        tmem_ld32(tmem + lane_off + C::R_DV + 32u * (uint32_t)c, v);
        tmem_wait_ld();
        if (row_ok) {
#pragma unroll
          for (int g = 0; g < 8; ++g)
            *reinterpret_cast<float4*>(p.dv_bar + row + 32 * c + 4 * g) =
                make_float4(__uint_as_float(v[4 * g]), __uint_as_float(v[4 * g + 1]),
                            __uint_as_float(v[4 * g + 2]), __uint_as_float(v[4 * g + 3]));
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

}  // namespace

cudaError_t launch_attn_bwd_tc(const SwaShape& s, const void* q_rot, const void* k_bar, const void* v_bar,
                               const void* dout, const float* lse, const float* delta, float* dq_acc,
                               float* dk_bar, float* dv_bar, int64_t spin_limit, int* err, cudaStream_t st) {
  CUtensorMap tq, tk, tv, tdo;
  cudaError_t e;
  if ((e = make_tmap_tokens(&tq, q_rot, s.B, s.T, s.H, s.hd, 128)) != cudaSuccess) return e;
  if ((e = make_tmap_tokens(&tk, k_bar, s.B, s.T, s.H, s.hd, 128)) != cudaSuccess) return e;
  if ((e = make_tmap_tokens(&tv, v_bar, s.B, s.T, s.H, s.hd, 128)) != cudaSuccess) return e;
  if ((e = make_tmap_tokens(&tdo, dout, s.B, s.T, s.H, s.hd, 128)) != cudaSuccess) return e;
  CUtensorMap tdq;
  if ((e = make_tmap_f32_tokens(&tdq, dq_acc, s.B, s.T, s.H, s.hd)) != cudaSuccess) return e;
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
  p.dk_bar = dk_bar;
  p.dv_bar = dv_bar;
  p.spin_limit = spin_limit;
  p.err = err;
  dim3 grid((unsigned)((s.T + 127) / 128), (unsigned)s.H, (unsigned)s.B);
  if (s.hd == 128) {
    auto k = attn_bwd_tc_kernel<128>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)BwdCfg<128>::SMEM);
    if (e != cudaSuccess) return e;
    k<<<grid, NUM_THREADS, BwdCfg<128>::SMEM, st>>>(tq, tk, tv, tdo, tdq, p);
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
