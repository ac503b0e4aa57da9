// Two-SM tcgen05 GEMM for the shared memory projection of Maglev's recurrent
// K/V injection and its backward ("Maglev: Sliding Recurrent Memory",
// paper.rainbus.top, 方法步骤详情: k_rec and v_rec come from the projections
// W_k^rec, W_v^rec shared by all layers):
//   forward  R = m_shift [B*T, d] x [W_mk; W_mv]^T           -> R_k | R_v
//   backward dm = [dR_k | dR_v] x [W_mk; W_mv]                (K = 2D)
//            dW = [dR_k | dR_v]^T x m_shift                   (M = 2D)
// and the per-layer projection's dm over layer-strided operands.
//
// A cluster of two CTAs on two SMs owns a 256 x 256 output tile: each CTA
// TMA-loads its 128 rows of A and its 128 columns of B per K block into its
// own shared memory (no multicast), and the leader (even) CTA issues
// tcgen05.mma.cta_group::2 (256 x 256 x 16), which reads both CTAs' operands
// and accumulates each CTA's 128 rows in that CTA's TMEM. Per SM that is 64 KiB
// of operands per 1024 MMA cycles (a one-SM 128 x 256 tile needs 1.5x that
// per flop and is fed-bound at ~70%). Every operand arrives in 16 KiB boxes
// ({64, 128}): L2 -> SM TMA throughput with 8 KiB boxes is a third lower.
// Two TMEM accumulators per CTA let the epilogue of one tile run under the
// next tile's MMAs.
//
// One launch may carry two GEMMs (the backward's dm and dW both read dR, and
// neither fills the 74 SM pairs of a B200 evenly on its own: dm is 160 tiles
// of 20 K blocks, 2.16 waves; dW 50 tiles of 64 K blocks). The host then
// deals the tiles of both longest first, each to the pair with the least work
// so far, and passes every pair its list: 100 K-block times for the two
// instead of 60 + 64 back to back. The LM head's backward GEMMs go the same
// way: dm (160 tiles of 512 K blocks) with dU (1280 tiles of 64).
//
// Roles per CTA (6 warps): warp 0 TMA producer, warp 1 MMA issuer (leader
// only), warps 2-5 epilogue (TMEM -> bf16 -> 128-byte row pieces). Loads in
// both CTAs count their bytes on the leader's stage barrier; the MMA commit
// releases a stage / publishes an accumulator in both CTAs at once; each
// epilogue warp returns its accumulator with an arrival on the leader's
// barrier. Every mbarrier wait is bounded.
#include <cuda.h>

#include <algorithm>
#include <functional>
#include <queue>
#include <utility>
#include <vector>

#include "launchers.h"
#include "tc_common.cuh"

namespace maglev {

cudaError_t make_tmap_bf16_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                              uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer);
cudaError_t make_tmap_bf16_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
                              uint32_t box_inner, uint32_t box_mid);

namespace {

using namespace tc;

constexpr int PM = 256;       // rows of a pair tile (128 per CTA)
constexpr int PN = 256;       // columns of a pair tile (B: 128 per CTA)
constexpr int EPI_BF16 = 0, EPI_CE = 1;
// Epilogue warps: 4 (one per TMEM lane quarter) for the bf16 store; 8 for the
// cross-entropy epilogue (two per lane quarter, each with 128 of the tile's 256
// columns: its per-element softcap and exponentials would otherwise pace the
// launch).
template <int EPI>
constexpr int pair_epi_warps() { return EPI == EPI_CE ? 8 : 4; }
template <int EPI>
constexpr int pair_threads() { return 64 + 32 * pair_epi_warps<EPI>(); }
constexpr int PAIR_MAX_PAIRS = 80;   // schedule table (a B200 holds 74 pairs)
constexpr int PAIR_MAX_ITEMS = 2048;  // tiles of a scheduled launch (the table is a kernel parameter)

// One GEMM of a launch: out [M, N] bf16 = A [M, K] x B [K, N], fp32 in TMEM.
// A is K-major (rows of K contiguous) or MN-major (a_mn: columns of M
// contiguous); B likewise with N (b_mn). The k / v halves of the projections
// live in two tensors: A moves to its second map at row a_switch_m or K index
// a_switch_k, B at column b_switch_n or K index b_switch_k, the output at row
// out_switch_m or column out_switch_n (0: no switch).
struct PairProblem {
  int M, N, K;
  int tiles_m, tiles_n, kblocks;
  int a_mn, b_mn;
  int a_switch_m, a_switch_k;
  int b_switch_n, b_switch_k;
  int out_switch_m, out_switch_n;
  int k_layers;  // > 0: A [k_layers][M][a_switch_k], B [k_layers][a_switch_k][N] (3-D maps), K = 2 L a_switch_k
  void* out0;
  void* out1;
  int64_t ldo;
};

struct PairMaps {
  CUtensorMap a0, a1, b0, b1;
};

struct PairParams {
  PairProblem pr[2];
  int tiles0;   // items [0, tiles0) are problem 0's tiles, [tiles0, n_items) problem 1's
  int n_items;
  int sched;    // 1: pair i runs order[first[i] .. first[i + 1]); 0: items i, i + pairs, ...
  int64_t spin_limit;
  int* err;
  // softcapped cross-entropy epilogue (one problem): out0 receives the capped
  // logits c = softcap * tanh(z / softcap) in fp32; per row and 128 columns the
  // (max, sum of exp(c - max)) pair goes to ce_part[row * ceil(N / 128) + i],
  // and the capped logit of the row's target to ce_tgt[row]
  const int64_t* ce_targets;
  float softcap;
  float2* ce_part;
  float* ce_tgt;
  uint16_t first[PAIR_MAX_PAIRS + 1];
  uint16_t order[PAIR_MAX_ITEMS];
};

template <int PK, int EPI = EPI_BF16>
struct PairCfg {
  // K block: 64 when both operands are K-major (one {64 K, 128 rows} box each,
  // six 32 KiB stages); 128 when one is MN-major, whose 16 KiB box is
  // {64 MN, 128 K} (three 64 KiB stages). A 16 KiB operand piece is
  // K-major [128 rows x 64 K] (pieces along K) or MN-major [128 K x 64 MN]
  // (pieces along MN).
  static_assert(PK == 64 || PK == 128, "K block of 64 or 128");
  static constexpr int A_BYTES = 128 * PK * 2;          // this CTA's 128 rows
  static constexpr int B_BYTES = (PN / 2) * PK * 2;     // this CTA's 128 columns
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = PK == 64 ? 6 : 3;
  static constexpr int PIECES = PK / 64;                // 16 KiB pieces per operand per stage
  static constexpr int TMEM_COLS = 512;                 // two 128 x 256 fp32 accumulators
  static constexpr int ACC_STRIDE = 256;
  static constexpr int OFF_BAR = STAGES * STAGE_BYTES;
  static constexpr int OFF_EPI = OFF_BAR + 256;         // per epilogue warp [32 rows x 128 B] output staging
  static constexpr size_t SMEM = 1024 + (size_t)OFF_EPI + pair_epi_warps<EPI>() * 4096;
};

// The i-th item (tile) of this pair, or -1 past its last.
__device__ __forceinline__ int pair_item(const PairParams& p, int pair, int npairs, int i) {
  if (p.sched) {
    const int k = (int)p.first[pair] + i;
    return k < (int)p.first[pair + 1] ? (int)p.order[k] : -1;
  }
  const int t = pair + i * npairs;
  return t < p.n_items ? t : -1;
}

struct PairTile {
  int prob, tm, tn;
};

__device__ __forceinline__ PairTile pair_tile(const PairParams& p, int item) {
  PairTile t;
  t.prob = item >= p.tiles0 ? 1 : 0;
  const int r = item - (t.prob ? p.tiles0 : 0);
  const int tiles_m = p.pr[t.prob].tiles_m;
  t.tm = r % tiles_m;
  t.tn = r / tiles_m;
  return t;
}

// cap * tanh(z / cap) = cap * (1 - 2 / (1 + e^(2z/cap))), with the hardware 2^x
// and the fast division intrinsic (both ends exact: 2 / inf = 0, 2 / 1 = 2)
__device__ __forceinline__ float pair_softcap(float z, float cap, float two_log2e_over_cap) {
  const float e = ex2_fast(z * two_log2e_over_cap);
  return cap * (1.0f - __fdividef(2.0f, 1.0f + e));
}

template <int PK, int EPI>
__global__ void __launch_bounds__(pair_threads<EPI>(), 1)
    tc_gemm_pair_kernel(const __grid_constant__ PairMaps mp0, const __grid_constant__ PairMaps mp1,
                        const __grid_constant__ PairParams p) {
  using C = PairCfg<PK, EPI>;
  constexpr int STAGES = C::STAGES;
  constexpr int EPI_WARPS = pair_epi_warps<EPI>();
  extern __shared__ uint8_t smem_raw[];
  // the same offset in both CTAs: the pair MMA reads both CTAs' operands at one address
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * C::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);  // [STAGES], used in the leader
  uint64_t* empty = full + STAGES;                                  // [STAGES]
  uint64_t* tfull = empty + STAGES;                                 // [2]
  uint64_t* tempty = tfull + 2;                                     // [2], used in the leader
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const Abort ab{abort_flag, p.err, p.spin_limit * 1000};

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * EPI_WARPS);  // one arrival per epilogue warp of both CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&mp0.a0);
    tma_prefetch_desc(&mp0.a1);
    tma_prefetch_desc(&mp0.b0);
    tma_prefetch_desc(&mp0.b1);
    if (p.tiles0 < p.n_items) {
      tma_prefetch_desc(&mp1.a0);
      tma_prefetch_desc(&mp1.a1);
      tma_prefetch_desc(&mp1.b0);
      tma_prefetch_desc(&mp1.b1);
    }
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any remote arrival or load
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int pair = (int)blockIdx.x >> 1, npairs = (int)gridDim.x >> 1;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int item = pair_item(p, pair, npairs, i);
        if (item < 0) break;
        const PairTile tl = pair_tile(p, item);
        const PairProblem& pr = p.pr[tl.prob];
        const PairMaps& mp = tl.prob ? mp1 : mp0;
        const int m0 = tl.tm * PM + 128 * (int)rank;  // this CTA's A rows
        const int n0 = tl.tn * PN + 128 * (int)rank;  // this CTA's B columns
        for (int kb = 0; kb < pr.kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, ab)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);  // both CTAs' bytes
          const uint32_t bar = mapa_cluster(smem_u32(&full[stage]), 0);
          uint8_t* dA = sA + stage * C::A_BYTES;
          uint8_t* dB = sB + stage * C::B_BYTES;
          const int k0 = kb * PK;
          bool done = false;
          if constexpr (PK == 128) {
            if (pr.k_layers > 0) {  // layer-strided K (A K-major, B MN-major): (k or v, layer l, k within the layer)
              const int LD = pr.k_layers * pr.a_switch_k;
              const int which = k0 >= LD ? 1 : 0;
              const int kr = k0 - which * LD;
              const int l = kr / pr.a_switch_k, kk = kr - l * pr.a_switch_k;
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                tma_load_3d_pair(dA + h * 16384, which ? &mp.a1 : &mp.a0, bar, kk + 64 * h, m0, l);
                tma_load_3d_pair(dB + h * 16384, which ? &mp.b1 : &mp.b0, bar, n0 + 64 * h, kk, l);
              }
              done = true;
            }
          }
          if (!done) {
            // operand A: this CTA's 128 rows; pieces along K (K-major) or M (MN-major).
            // The k / v switches fall on multiples of 128 (checked by the host).
            {
              const bool sw_m = pr.a_switch_m > 0 && m0 >= pr.a_switch_m;
              const bool sw_k = pr.a_switch_k > 0 && k0 >= pr.a_switch_k;
              const CUtensorMap* m = (sw_m || sw_k) ? &mp.a1 : &mp.a0;
              const int mm = sw_m ? m0 - pr.a_switch_m : m0;
              const int kk = sw_k ? k0 - pr.a_switch_k : k0;
#pragma unroll
              for (int h = 0; h < C::PIECES; ++h)
                tma_load_2d_pair(dA + h * 16384, m, bar, pr.a_mn ? mm + 64 * h : kk + 64 * h, pr.a_mn ? kk : mm);
            }
            // operand B: this CTA's 128 columns; pieces along K (K-major) or N (MN-major)
            {
              const bool sw_n = pr.b_switch_n > 0 && n0 >= pr.b_switch_n;
              const bool sw_k = pr.b_switch_k > 0 && k0 >= pr.b_switch_k;
              const CUtensorMap* m = (sw_n || sw_k) ? &mp.b1 : &mp.b0;
              const int nn = sw_n ? n0 - pr.b_switch_n : n0;
              const int kk = sw_k ? k0 - pr.b_switch_k : k0;
#pragma unroll
              for (int h = 0; h < C::PIECES; ++h)
                tma_load_2d_pair(dB + h * 16384, m, bar, pr.b_mn ? nn + 64 * h : kk + 64 * h, pr.b_mn ? kk : nn);
            }
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Every stage this CTA filled has been consumed (so its loads have landed)
      // before the CTA may exit: wait for the release of the last fill of each.
      for (int s = 0; s < STAGES; ++s) {
        mbar_drain(&empty[stage], phase ^ 1, DRAIN_LIMIT_NS);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
  } else if (warp == 1) {
    if (leader) {
      // ------------------------------------------------------------ MMA issuer (leader CTA)
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int item = pair_item(p, pair, npairs, i);
        if (item < 0) break;
        const PairProblem& pr = p.pr[pair_tile(p, item).prob];
        const bool a_mn = pr.a_mn != 0, b_mn = pr.b_mn != 0;
        const uint32_t idesc = idesc_bf16(PM, PN, a_mn, b_mn);
        if (!warp_wait(&tempty[acc], acc_phase ^ 1, ab)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * C::ACC_STRIDE);
        for (int kb = 0; kb < pr.kblocks; ++kb) {
          if (!warp_wait(&full[stage], phase, ab)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * C::B_BYTES);
          if (elect_one()) {
#pragma unroll
            for (int k16 = 0; k16 < PK / 16; ++k16) {
              // K-major: piece k16 / 4, 32 bytes per 16 K inside it; MN-major: 16 K rows
              // of 128 B per step, the two MN pieces 16 KiB apart
              const uint32_t koff = (uint32_t)(k16 >> 2) * 16384u + (uint32_t)(k16 & 3) * 32u;
              const uint64_t ad = a_mn ? sw128_desc(a_addr + (uint32_t)k16 * 2048u, 16384u, 1024u)
                                       : sw128_desc(a_addr + koff, 16u, 1024u);
              const uint64_t bd = b_mn ? sw128_desc(b_addr + (uint32_t)k16 * 2048u, 16384u, 1024u)
                                       : sw128_desc(b_addr + koff, 16u, 1024u);
              mma_ss_pair(d_tmem, ad, bd, idesc, (kb > 0 || k16 > 0) ? 1u : 0u);
            }
            mma_commit_pair_both(&empty[stage]);  // the stage is free in both CTAs
          }
          __syncwarp();
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        if (elect_one()) mma_commit_pair_both(&tfull[acc]);  // both CTAs' halves of the tile are ready
        __syncwarp();
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      // all issued MMAs finish before either CTA releases its TMEM
      if (elect_one()) {
        mma_commit_pair(drain);
        mbar_drain(drain, 0, DRAIN_LIMIT_NS);
      }
      __syncwarp();
    }
  } else if constexpr (EPI == EPI_CE) {
    // -------------------------------------------------------------- CE epilogue (both CTAs)
    // Thread = one of this CTA's 128 rows of the tile; warp w owns columns
    // [128 h, 128 h + 128), h = (w - 2) / 4. 32 columns at a time: TMEM ->
    // capped logits (running max / sum of exponentials of the row over the
    // warp's 128 columns, target logit) -> the warp's 4 KiB of fp32 staging ->
    // 128-byte row pieces; one (max, sum) partial per row and 128 columns.
    constexpr float LOG2E_F = 1.4426950408889634f;
    const float k2 = 2.0f * LOG2E_F / p.softcap;
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    uint8_t* stg = smem + C::OFF_EPI + (warp - 2) * 4096;
    const PairProblem& pr = p.pr[0];
    const int ce_tiles = (pr.N + 127) / 128;  // partials per row
    float* outc = static_cast<float*>(pr.out0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int i = 0;; ++i) {
      const int item = pair_item(p, pair, npairs, i);
      if (item < 0) break;
      const PairTile tl = pair_tile(p, item);
      const int m0 = tl.tm * PM + 128 * (int)rank, n0 = tl.tn * PN + 128 * half;
      if (!warp_wait(&tfull[acc], acc_phase, ab)) break;
      tc_fence_after();
      const int gm = m0 + row;
      const int64_t y = gm < pr.M ? p.ce_targets[gm] : -1;
      float mx = -INFINITY, sm = 0.f;
      const bool any = n0 < pr.N;  // the warp's columns start inside the row
#pragma unroll 1
      for (int c0 = 0; c0 < (any ? 128 : 0); c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * C::ACC_STRIDE + 128 * half + c0), r);
        tmem_wait_ld();
        float cmx = -INFINITY;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int col = n0 + c0 + e;
          const float c = pair_softcap(__uint_as_float(r[e]), p.softcap, k2);
          if (col == y) p.ce_tgt[gm] = c;
          const float cv = col < pr.N ? c : -INFINITY;
          cmx = fmaxf(cmx, cv);
          r[e] = __float_as_uint(cv);
        }
        const float nmx = fmaxf(mx, cmx);  // finite: column n0 < N is in the first chunk
        float se = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) se += ex2_fast((__uint_as_float(r[e]) - nmx) * LOG2E_F);
        sm = sm * ex2_fast((mx - nmx) * LOG2E_F) + se;
        mx = nmx;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint4*>(stg + lane * 128 + ((j ^ (lane & 7)) << 4)) =
              make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int rr = 4 * k + (lane >> 3), j = lane & 7;  // row of the warp's 32, 16-byte chunk
          const uint4 v = *reinterpret_cast<const uint4*>(stg + rr * 128 + ((j ^ (rr & 7)) << 4));
          const int col = n0 + c0 + 4 * j;
          const int grow = m0 + q * 32 + rr;
          if (grow < pr.M && col + 4 <= pr.N && MAGLEV_CHECK(p.err, grow >= 0 && col >= 0 && col + 4 <= pr.ldo))
            *reinterpret_cast<uint4*>(outc + (int64_t)grow * pr.ldo + col) = v;
        }
        __syncwarp();
      }
      if (gm < pr.M && any) p.ce_part[(int64_t)gm * ce_tiles + 2 * tl.tn + half] = make_float2(mx, sm);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_cluster(smem_u32(&tempty[acc]), 0));  // the leader may reuse it
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue (both CTAs)
    // This CTA's 128 rows of the tile, 64 columns at a time: TMEM -> bf16 ->
    // the warp's 4 KiB of staging (16-byte chunks swizzled by row) -> read back
    // so that each warp-wide store covers four whole 128-byte row pieces.
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    uint8_t* stg = smem + C::OFF_EPI + q * 4096;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int i = 0;; ++i) {
      const int item = pair_item(p, pair, npairs, i);
      if (item < 0) break;
      const PairTile tl = pair_tile(p, item);
      const PairProblem& pr = p.pr[tl.prob];
      const int m0 = tl.tm * PM + 128 * (int)rank, n0 = tl.tn * PN;
      if (!warp_wait(&tfull[acc], acc_phase, ab)) break;
      tc_fence_after();
      bf16* out = static_cast<bf16*>(pr.out0);
      int om0 = m0 + q * 32;  // first row of this warp in the output tensor
      if (pr.out_switch_m > 0 && m0 >= pr.out_switch_m) {
        out = static_cast<bf16*>(pr.out1);
        om0 -= pr.out_switch_m;
      }
#pragma unroll 1
      for (int c0 = 0; c0 < PN; c0 += 64) {
        uint32_t r[2][32];
        tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * C::ACC_STRIDE + c0), r[0]);
        tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * C::ACC_STRIDE + c0 + 32), r[1]);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint4 v;
          v.x = pack_bf16(__uint_as_float(r[j >> 2][8 * (j & 3) + 0]), __uint_as_float(r[j >> 2][8 * (j & 3) + 1]));
          v.y = pack_bf16(__uint_as_float(r[j >> 2][8 * (j & 3) + 2]), __uint_as_float(r[j >> 2][8 * (j & 3) + 3]));
          v.z = pack_bf16(__uint_as_float(r[j >> 2][8 * (j & 3) + 4]), __uint_as_float(r[j >> 2][8 * (j & 3) + 5]));
          v.w = pack_bf16(__uint_as_float(r[j >> 2][8 * (j & 3) + 6]), __uint_as_float(r[j >> 2][8 * (j & 3) + 7]));
          *reinterpret_cast<uint4*>(stg + lane * 128 + ((j ^ (lane & 7)) << 4)) = v;
        }
        __syncwarp();
        // 64 columns [col0, col0 + 64): this tensor, or the second one past out_switch_n
        const int col0 = n0 + c0;
        bf16* o = out;
        int ocol0 = col0, n_lim = pr.N;
        if (pr.out_switch_n > 0) {
          if (col0 >= pr.out_switch_n) {
            o = static_cast<bf16*>(pr.out1);
            ocol0 -= pr.out_switch_n;
          } else {
            n_lim = pr.out_switch_n;
          }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int rr = 4 * k + (lane >> 3), j = lane & 7;  // row of the warp's 32, 16-byte chunk
          const uint4 v = *reinterpret_cast<const uint4*>(stg + rr * 128 + ((j ^ (rr & 7)) << 4));
          if (m0 + q * 32 + rr < pr.M && col0 + 8 * j + 8 <= n_lim &&
              MAGLEV_CHECK(p.err, om0 + rr >= 0 && ocol0 >= 0 && ocol0 + 8 * j + 8 <= pr.ldo))
            *reinterpret_cast<uint4*>(o + (int64_t)(om0 + rr) * pr.ldo + ocol0 + 8 * j) = v;
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_cluster(smem_u32(&tempty[acc]), 0));  // the leader may reuse it
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }
  __syncthreads();
  cluster_sync_all();  // neither CTA releases TMEM / leaves while the pair still uses it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace

namespace {

// Largest number of two-CTA clusters of this kernel that can be resident at
// once (0 when clusters cannot be launched), cached per instantiation.
template <int PK, int EPI = EPI_BF16>
int max_pairs() {
  static int cached = -1;
  if (cached >= 0) return cached;
  using C = PairCfg<PK, EPI>;
  auto kern = tc_gemm_pair_kernel<PK, EPI>;
  int n = 0;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 74, 1, 1);
    cfg.blockDim = dim3(pair_threads<EPI>(), 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, (void*)kern, &cfg) != cudaSuccess) n = 0;
  }
  (void)cudaGetLastError();
  cached = n < PAIR_MAX_PAIRS ? n : PAIR_MAX_PAIRS;
  return cached;
}

// Longest processing time first: items in decreasing K-block count (ties in
// item order), each to the pair with the least work so far (ties to the lower
// pair); a pair runs its items in the order they were dealt.
void lpt_schedule(PairParams& p, int pairs) {
  std::vector<int> items(p.n_items);
  for (int i = 0; i < p.n_items; ++i) items[i] = i;
  auto cost = [&](int it) { return p.pr[it >= p.tiles0 ? 1 : 0].kblocks; };
  std::stable_sort(items.begin(), items.end(), [&](int x, int y) { return cost(x) > cost(y); });
  using Load = std::pair<int64_t, int>;  // (work so far, pair)
  std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
  for (int i = 0; i < pairs; ++i) heap.push({0, i});
  std::vector<std::vector<uint16_t>> lists(pairs);
  for (int it : items) {
    Load l = heap.top();
    heap.pop();
    lists[l.second].push_back((uint16_t)it);
    heap.push({l.first + cost(it), l.second});
  }
  int k = 0;
  for (int i = 0; i < pairs; ++i) {
    p.first[i] = (uint16_t)k;
    for (uint16_t it : lists[i]) p.order[k++] = it;
  }
  p.first[pairs] = (uint16_t)k;
  p.sched = 1;
}

template <int PK, int EPI = EPI_BF16>
cudaError_t run_pair(const PairMaps& m0, const PairMaps& m1, PairParams& p, bool schedule, cudaStream_t s) {
  using C = PairCfg<PK, EPI>;
  const int cap = max_pairs<PK, EPI>();
  if (cap < 1) return cudaErrorNotSupported;
  const int pairs = p.n_items < cap ? p.n_items : cap;
  if (schedule) {
    if (p.n_items > PAIR_MAX_ITEMS) return cudaErrorNotSupported;
    lpt_schedule(p, pairs);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(pair_threads<EPI>(), 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tc_gemm_pair_kernel<PK, EPI>, m0, m1, p);
}

PairProblem pair_problem(int M, int N, int K, bool a_mn, bool b_mn, int64_t ldo) {
  PairProblem q{};
  q.M = M;
  q.N = N;
  q.K = K;
  q.tiles_m = (M + PM - 1) / PM;
  q.tiles_n = (N + PN - 1) / PN;
  q.kblocks = (K + ((a_mn || b_mn) ? 128 : 64) - 1) / ((a_mn || b_mn) ? 128 : 64);
  q.a_mn = a_mn ? 1 : 0;
  q.b_mn = b_mn ? 1 : 0;
  q.ldo = ldo;
  return q;
}

PairParams pair_params(const PairProblem& q0, int64_t spin_limit, int* err) {
  PairParams p{};
  p.pr[0] = q0;
  p.pr[1] = q0;
  p.tiles0 = q0.tiles_m * q0.tiles_n;
  p.n_items = p.tiles0;
  p.spin_limit = spin_limit;
  p.err = err;
  return p;
}

// Problem and maps of dm [M, d] = dR_k [M, D] W_mk [D, d] + dR_v W_mv (K = 2D, B N-contiguous).
cudaError_t dm_problem(int64_t M, int D, int d, const void* dRk, const void* dRv, const void* w_mk,
                       const void* w_mv, void* dm, PairMaps& mp, PairProblem& q) {
  cudaError_t e;
  if ((e = make_tmap_bf16_2d(&mp.a0, dRk, D, M, (uint64_t)D * 2, 64, 128)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&mp.a1, dRv, D, M, (uint64_t)D * 2, 64, 128)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&mp.b0, w_mk, d, D, (uint64_t)d * 2, 64, 128)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&mp.b1, w_mv, d, D, (uint64_t)d * 2, 64, 128)) != cudaSuccess) return e;
  q = pair_problem((int)M, d, 2 * D, false, true, d);
  q.a_switch_k = D;
  q.b_switch_k = D;
  q.out0 = dm;
  q.out1 = dm;
  return cudaSuccess;
}

// Problem and maps of dW_mk | dW_mv [D, d] = dR^T [D, M] m_shift [M, d] (A and B both M-contiguous).
cudaError_t dw_problem(int64_t M, int D, int d, const void* dRk, const void* dRv, const void* m_shift, void* dwk,
                       void* dwv, PairMaps& mp, PairProblem& q) {
  cudaError_t e;
  if ((e = make_tmap_bf16_2d(&mp.a0, dRk, D, M, (uint64_t)D * 2, 64, 128)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&mp.a1, dRv, D, M, (uint64_t)D * 2, 64, 128)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&mp.b0, m_shift, d, M, (uint64_t)d * 2, 64, 128)) != cudaSuccess) return e;
  mp.b1 = mp.b0;
  q = pair_problem(2 * D, d, (int)M, true, true, d);
  q.a_switch_m = D;
  q.out_switch_m = D;
  q.out0 = dwk;
  q.out1 = dwv;
  return cudaSuccess;
}

}  // namespace

// The pair kernels move between the k and v operands only at multiples of 128
// (a CTA's rows / columns, a K block): D must be a multiple of 128; otherwise
// the caller uses the one-SM kernels.
bool pair_gemm_supported(int D) { return D % 128 == 0; }

// R_k | R_v [M, D] = m_shift [M, d] x W^T, W_mk / W_mv [D, d].
cudaError_t launch_proj_fwd_pair(int64_t M, int D, int d, const void* m_shift, const void* w_mk, const void* w_mv,
                                 void* Rk, void* Rv, int64_t spin_limit, int* err, cudaStream_t s) {
  PairMaps mp;
  cudaError_t e;
  if ((e = make_tmap_bf16_2d(&mp.a0, m_shift, d, M, (uint64_t)d * 2, 64, 128)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&mp.b0, w_mk, d, D, (uint64_t)d * 2, 64, 128)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&mp.b1, w_mv, d, D, (uint64_t)d * 2, 64, 128)) != cudaSuccess) return e;
  mp.a1 = mp.a0;
  PairProblem q = pair_problem((int)M, 2 * D, d, false, false, D);
  q.b_switch_n = D;
  q.out_switch_n = D;
  q.out0 = Rk;
  q.out1 = Rv;
  PairParams p = pair_params(q, spin_limit, err);
  return run_pair<64>(mp, mp, p, false, s);
}

// dm [M, d] = dR_k [M, D] W_mk [D, d] + dR_v W_mv (K = 2D, B operand N-contiguous).
cudaError_t launch_proj_bwd_dm_pair(int64_t M, int D, int d, const void* dRk, const void* dRv, const void* w_mk,
                                    const void* w_mv, void* dm, int64_t spin_limit, int* err, cudaStream_t s) {
  PairMaps mp;
  PairProblem q;
  cudaError_t e;
  if ((e = dm_problem(M, D, d, dRk, dRv, w_mk, w_mv, dm, mp, q)) != cudaSuccess) return e;
  PairParams p = pair_params(q, spin_limit, err);
  return run_pair<128>(mp, mp, p, false, s);
}

// dm [M, d] = sum over L layers of dR_k^l W_mk^l + dR_v^l W_mv^l (layer-strided, K = 2 L D).
cudaError_t launch_proj_bwd_dm_layers_pair(int64_t M, int D, int d, int L, const void* dRk, const void* dRv,
                                           const void* w_mk, const void* w_mv, void* dm, int64_t spin_limit,
                                           int* err, cudaStream_t s) {
  PairMaps mp;
  cudaError_t e;
  if ((e = make_tmap_bf16_3d(&mp.a0, dRk, D, M, L, 64, 128)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_3d(&mp.a1, dRv, D, M, L, 64, 128)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_3d(&mp.b0, w_mk, d, D, L, 64, 128)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_3d(&mp.b1, w_mv, d, D, L, 64, 128)) != cudaSuccess) return e;
  PairProblem q = pair_problem((int)M, d, 2 * L * D, false, true, d);
  q.a_switch_k = D;
  q.b_switch_k = D;
  q.k_layers = L;
  q.out0 = dm;
  q.out1 = dm;
  PairParams p = pair_params(q, spin_limit, err);
  return run_pair<128>(mp, mp, p, false, s);
}

// dW_mk | dW_mv [D, d] = dR^T [D, M] m_shift [M, d] (A and B both M-contiguous in memory).
cudaError_t launch_proj_bwd_dw_pair(int64_t M, int D, int d, const void* dRk, const void* dRv, const void* m_shift,
                                    void* dwk, void* dwv, int64_t spin_limit, int* err, cudaStream_t s) {
  PairMaps mp;
  PairProblem q;
  cudaError_t e;
  if ((e = dw_problem(M, D, d, dRk, dRv, m_shift, dwk, dwv, mp, q)) != cudaSuccess) return e;
  PairParams p = pair_params(q, spin_limit, err);
  return run_pair<128>(mp, mp, p, false, s);
}

// dm [N, d] = dz [N, V] U [V, d] (K = V) and dU [V, d] = dz^T [V, N] m [N, d]
// (K = N) in one launch, their tiles dealt longest first over the SM pairs.
// cudaErrorNotSupported when clusters cannot be launched or the two have more
// tiles than the schedule table holds; the caller then launches them one by one.
bool lm_bwd_grouped_available(int64_t N, int d, int V) {
  if (d % 8 != 0 || V % 8 != 0 || max_pairs<128>() < 1) return false;
  const int64_t tiles = ((N + PM - 1) / PM + ((int64_t)V + PM - 1) / PM) * (((int64_t)d + PN - 1) / PN);
  return tiles <= PAIR_MAX_ITEMS;
}

cudaError_t launch_lm_bwd_grouped_pair(int64_t N, int d, int V, const void* dz, const void* U, const void* m,
                                       void* dm, void* dU, int64_t spin_limit, int* err, cudaStream_t s) {
  PairMaps mm, mu;
  cudaError_t e;
  if ((e = make_tmap_bf16_2d(&mm.a0, dz, V, N, (uint64_t)V * 2, 64, 128)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&mm.b0, U, d, V, (uint64_t)d * 2, 64, 128)) != cudaSuccess) return e;
  mm.a1 = mm.a0;
  mm.b1 = mm.b0;
  mu.a0 = mm.a0;  // dz read MN-major: the same {64 V, 128 N} boxes
  if ((e = make_tmap_bf16_2d(&mu.b0, m, d, N, (uint64_t)d * 2, 64, 128)) != cudaSuccess) return e;
  mu.a1 = mu.a0;
  mu.b1 = mu.b0;
  PairProblem qm = pair_problem((int)N, d, V, false, true, d);
  qm.out0 = dm;
  qm.out1 = dm;
  PairProblem qu = pair_problem(V, d, (int)N, true, true, d);
  qu.out0 = dU;
  qu.out1 = dU;
  PairParams p = pair_params(qm, spin_limit, err);
  p.pr[1] = qu;
  p.n_items = p.tiles0 + qu.tiles_m * qu.tiles_n;
  return run_pair<128>(mm, mu, p, true, s);
}

// The LM head's logits z = m [N, d] U^T (U [V, d]) with the softcapped
// cross-entropy epilogue (see PairParams): capped logits c [N, V] fp32,
// part [N, ceil(V / 128)] and tgt [N].
cudaError_t launch_lm_logits_ce_pair(int64_t N, int d, int V, float softcap, const void* m, const void* U,
                                     const int64_t* targets, float* c, float2* part, float* tgt,
                                     int64_t spin_limit, int* err, cudaStream_t s) {
  if (V % 4 != 0) return cudaErrorNotSupported;
  PairMaps mp;
  cudaError_t e;
  if ((e = make_tmap_bf16_2d(&mp.a0, m, d, N, (uint64_t)d * 2, 64, 128)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&mp.b0, U, d, V, (uint64_t)d * 2, 64, 128)) != cudaSuccess) return e;
  mp.a1 = mp.a0;
  mp.b1 = mp.b0;
  PairProblem q = pair_problem((int)N, V, d, false, false, V);
  q.out0 = c;
  q.out1 = c;
  PairParams p = pair_params(q, spin_limit, err);
  p.ce_targets = targets;
  p.softcap = softcap;
  p.ce_part = part;
  p.ce_tgt = tgt;
  return run_pair<64, EPI_CE>(mp, mp, p, false, s);
}

// Whether launch_proj_bwd_grouped_pair can run dW and dm of these sizes.
bool proj_bwd_grouped_available(int64_t M, int D, int d) {
  if (!pair_gemm_supported(D) || max_pairs<128>() < 1) return false;
  const int64_t tiles = ((2 * (int64_t)D + PM - 1) / PM + (M + PM - 1) / PM) * (((int64_t)d + PN - 1) / PN);
  return tiles <= PAIR_MAX_ITEMS;
}

// dW and dm in one launch, their tiles dealt longest first over the SM pairs.
// cudaErrorNotSupported when clusters cannot be launched or the two have more
// than 512 tiles; the caller then launches them one by one.
cudaError_t launch_proj_bwd_grouped_pair(int64_t M, int D, int d, const void* dRk, const void* dRv, const void* w_mk,
                                         const void* w_mv, const void* m_shift, void* dm, void* dwk, void* dwv,
                                         int64_t spin_limit, int* err, cudaStream_t s) {
  PairMaps mw, mm;
  PairProblem qw, qm;
  cudaError_t e;
  if ((e = dw_problem(M, D, d, dRk, dRv, m_shift, dwk, dwv, mw, qw)) != cudaSuccess) return e;
  if ((e = dm_problem(M, D, d, dRk, dRv, w_mk, w_mv, dm, mm, qm)) != cudaSuccess) return e;
  PairParams p = pair_params(qw, spin_limit, err);
  p.pr[1] = qm;
  p.n_items = p.tiles0 + qm.tiles_m * qm.tiles_n;
  return run_pair<128>(mw, mm, p, true, s);
}

}  // namespace maglev
