// Persistent tcgen05 GEMM for the shared memory projection of Maglev's
// recurrent K/V injection ("Maglev: Sliding Recurrent Memory",
// paper.rainbus.top, 方法步骤详情: k_rec and v_rec come from the projections
// W_k^rec, W_v^rec shared by all layers) and its backward:
//   forward  R = m_shift [B*T, d] x [W_mk; W_mv]^T           -> R_k | R_v
//   backward dm = [dR_k | dR_v] x [W_mk; W_mv]                (K = 2D)
//            dW = [dR_k | dR_v]^T x m_shift                   (M = 2D)
//   per-layer projection (one W^rec per decoder layer, paper.rainbus.top,
//   未来方向: 逐层记忆投影): dm = sum over layers l of [dR_k^l | dR_v^l] x
//   [W_mk^l; W_mv^l], one GEMM with K = 2 L D over layer-strided operands
//   (3-D tensor maps), so the sum over layers accumulates in fp32 in TMEM.
//
// One CTA per SM, 6 warps: warp 0 issues TMA loads of 64-wide K blocks into a
// ring of 128B-swizzled shared-memory stages, warp 1 issues tcgen05.mma
// (128 x BN x 16, bf16 -> fp32) into one of two TMEM accumulators, warps 2-5
// drain the other accumulator (tcgen05.ld) and store bf16. Operands may be
// K-major or MN-major; a second tensor map per operand lets one launch span
// the two halves (k/v) without a concatenated copy. Every wait is bounded.
#include <cuda.h>

#include <mutex>

#include "launchers.h"
#include "tc_common.cuh"

namespace maglev {
namespace {

using namespace tc;

constexpr int BM = 128, BK = 64;
constexpr int NUM_THREADS = 192;

struct TcGemmParams {
  int M, N, K;
  int tiles_m, tiles_n;
  int a_switch_m, a_switch_k;  // rows / K index where operand A moves to map 1
  int b_switch_n, b_switch_k;
  int out_switch_m, out_switch_n;
  int k_layers;  // > 0: A is [k_layers][M][a_switch_k], B [k_layers][a_switch_k][N] (3-D maps), K = 2 L a_switch_k
  // softcapped cross-entropy epilogue (EPI_CE): out0 receives the capped
  // logits c = softcap * tanh(z / softcap) in fp32; per row and 128 columns the
  // (max, sum of exp(c - max)) pair goes to ce_part[row * ceil(N / 128) + i],
  // and the capped logit of the row's target to ce_tgt[row]
  const int64_t* targets;
  float softcap;
  float2* ce_part;
  float* ce_tgt;
  void* out0;
  void* out1;
  int64_t ldo;
  int64_t spin_limit;
  int* err;
};

template <int BN, bool A_MN, bool B_MN>
struct Cfg {
  static_assert(BN % 64 == 0 && BN <= 256, "N tiles are whole 64-column blocks");
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (200 * 1024) / STAGE_BYTES > 8 ? 8 : (200 * 1024) / STAGE_BYTES;
  static constexpr int TMEM_COLS = 2 * BN <= 256 ? 256 : 512;
  static constexpr int ACC_STRIDE = TMEM_COLS / 2;  // column of the second accumulator
  static constexpr int OFF_EPI = STAGES * STAGE_BYTES + 256;  // 4 warps x [32 rows x 128 B] output staging
  static constexpr size_t SMEM = 1024 + (size_t)OFF_EPI + 4 * 4096;
};

// Epilogues: bf16 store of the accumulator, or the softcapped cross-entropy
// statistics with an fp32 store of the capped logits.
constexpr int EPI_BF16 = 0, EPI_CE = 1;

// softcap * tanh(z / softcap), with tanh(x) = 1 - 2 / (1 + e^{2x}) (exact at
// +-inf: e^{2x} = inf gives 1, 0 gives -1; absolute error ~1e-7 near 0).
// cap * tanh(z / cap) = cap * (1 - 2 / (1 + e^(2z/cap))), with the hardware 2^x
// and the fast division intrinsic (both ends exact: 2 / inf = 0, 2 / 1 = 2)
__device__ __forceinline__ float softcap_of(float z, float cap, float two_log2e_over_cap) {
  const float e = ex2_fast(z * two_log2e_over_cap);
  return cap * (1.0f - __fdividef(2.0f, 1.0f + e));
}

template <int BN, bool A_MN, bool B_MN, int EPI = EPI_BF16>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                   const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
                   TcGemmParams p) {
  using C = Cfg<BN, A_MN, B_MN>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * C::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const Abort ab{abort_flag, p.err, p.spin_limit * 1000};

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmB1);
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_tiles = p.tiles_m * p.tiles_n;
  const int kblocks = (p.K + BK - 1) / BK;
  constexpr uint32_t IDESC = idesc_bf16(BM, BN, A_MN, B_MN);

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0;           // bit s: stage s was armed at least once
      uint32_t armed_parity = 0;    // bit s: parity of the last arming of stage s
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const int tm = t % p.tiles_m, tn = t / p.tiles_m;
        const int m0 = tm * BM, n0 = tn * BN;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, ab)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          const int k0 = kb * BK;
          if constexpr (!A_MN && B_MN) {
            if (p.k_layers > 0) {  // layer-strided K: (k or v, layer l, k within the layer)
              const int LD = p.k_layers * p.a_switch_k;
              const int which = k0 >= LD ? 1 : 0;
              const int kr = k0 - which * LD;
              const int l = kr / p.a_switch_k, kk = kr - l * p.a_switch_k;
              tma_load_3d(sA + stage * C::A_BYTES, which ? &tmA1 : &tmA0, &full[stage], kk, m0, l);
              uint8_t* dstb = sB + stage * C::B_BYTES;
#pragma unroll
              for (int j = 0; j < BN / 64; ++j)
                tma_load_3d(dstb + j * 8192, which ? &tmB1 : &tmB0, &full[stage], n0 + 64 * j, kk, l);
              if (++stage == STAGES) {
                stage = 0;
                phase ^= 1;
              }
              continue;
            }
          }
          // operand A
          {
            const bool second = (p.a_switch_m > 0 && m0 >= p.a_switch_m) || (p.a_switch_k > 0 && k0 >= p.a_switch_k);
            const CUtensorMap* m = second ? &tmA1 : &tmA0;
            const int mm = (p.a_switch_m > 0 && m0 >= p.a_switch_m) ? m0 - p.a_switch_m : m0;
            const int kk = (p.a_switch_k > 0 && k0 >= p.a_switch_k) ? k0 - p.a_switch_k : k0;
            uint8_t* dst = sA + stage * C::A_BYTES;
            if (A_MN) {
              tma_load_2d(dst, m, &full[stage], mm, kk);
              tma_load_2d(dst + 8192, m, &full[stage], mm + 64, kk);
            } else {
              tma_load_2d(dst, m, &full[stage], kk, mm);
            }
          }
          // operand B
          {
            const bool second = (p.b_switch_n > 0 && n0 >= p.b_switch_n) || (p.b_switch_k > 0 && k0 >= p.b_switch_k);
            const CUtensorMap* m = second ? &tmB1 : &tmB0;
            const int nn = (p.b_switch_n > 0 && n0 >= p.b_switch_n) ? n0 - p.b_switch_n : n0;
            const int kk = (p.b_switch_k > 0 && k0 >= p.b_switch_k) ? k0 - p.b_switch_k : k0;
            uint8_t* dst = sB + stage * C::B_BYTES;
            if (B_MN) {
#pragma unroll
              for (int j = 0; j < BN / 64; ++j) tma_load_2d(dst + j * 8192, m, &full[stage], nn + 64 * j, kk);
            } else {
              tma_load_2d(dst, m, &full[stage], kk, nn);
            }
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // every armed stage's last load must land before the CTA may exit
      for (int s = 0; s < STAGES; ++s)
        if (armed & (1u << s)) mbar_drain(&full[s], (armed_parity >> s) & 1u, DRAIN_LIMIT_NS);
    }
  } else if (warp == 1) {
    {
      // ------------------------------------------------------------ MMA issuer
      // Every lane runs the loop and the waits (warp-uniform descriptors and
      // counters); the elected lane issues each k-block's MMAs and commits.
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        if (!warp_wait(&tempty[acc], acc_phase ^ 1, ab)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * C::ACC_STRIDE);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!warp_wait(&full[stage], phase, ab)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * C::B_BYTES);
          if (elect_one()) {
#pragma unroll
            for (int k16 = 0; k16 < BK / 16; ++k16) {
              const uint64_t ad = A_MN ? mnmajor_desc(a_addr, k16) : kmajor_desc(a_addr, k16);
              const uint64_t bd = B_MN ? mnmajor_desc(b_addr, k16) : kmajor_desc(b_addr, k16);
              mma_ss(d_tmem, ad, bd, IDESC, (kb > 0 || k16 > 0) ? 1u : 0u);
            }
            mma_commit(&empty[stage]);
          }
          __syncwarp();
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        if (elect_one()) mma_commit(&tfull[acc]);
        __syncwarp();
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      // all issued MMAs must finish before TMEM is released
      if (elect_one()) {
        mma_commit(drain);
        mbar_drain(drain, 0, DRAIN_LIMIT_NS);
      }
      __syncwarp();
    }
  } else if constexpr (EPI == EPI_CE) {
    // -------------------------------------------------------------- CE epilogue
    // Thread = one row of the tile. 32 columns at a time: TMEM -> capped logits
    // (running max / sum of exponentials of the row over the tile, target
    // logit) -> the warp's 4 KiB of fp32 staging -> 128-byte row pieces.
    constexpr float LOG2E_F = 1.4426950408889634f;
    const float k2 = 2.0f * LOG2E_F / p.softcap;
    const int q = warp & 3;
    const int row = q * 32 + lane;
    uint8_t* stg = smem + C::OFF_EPI + q * 4096;
    float* outc = static_cast<float*>(p.out0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      const int tm = t % p.tiles_m, tn = t / p.tiles_m;
      const int m0 = tm * BM, n0 = tn * BN;
      if (!warp_wait(&tfull[acc], acc_phase, ab)) break;
      tc_fence_after();
      const int gm = m0 + row;
      const int64_t y = gm < p.M ? p.targets[gm] : -1;
      const int ce_tiles = (p.N + 127) / 128;  // partials per row
      float mx = -INFINITY, sm = 0.f;
#pragma unroll 1
      for (int c0 = 0; c0 < BN && n0 + c0 < p.N; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * C::ACC_STRIDE + c0), r);
        tmem_wait_ld();
        float cmx = -INFINITY;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int col = n0 + c0 + e;
          const float c = softcap_of(__uint_as_float(r[e]), p.softcap, k2);
          if (col == y) p.ce_tgt[gm] = c;
          const float cv = col < p.N ? c : -INFINITY;
          cmx = fmaxf(cmx, cv);
          r[e] = __float_as_uint(cv);
        }
        const float nmx = fmaxf(mx, cmx);  // finite: this chunk starts inside the row
        float se = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) se += ex2_fast((__uint_as_float(r[e]) - nmx) * LOG2E_F);
        sm = sm * ex2_fast((mx - nmx) * LOG2E_F) + se;
        mx = nmx;
        if (((c0 + 32) & 127) == 0 || n0 + c0 + 32 >= p.N) {  // the end of 128 columns (or of the row)
          if (gm < p.M) p.ce_part[(int64_t)gm * ce_tiles + (n0 + c0) / 128] = make_float2(mx, sm);
          mx = -INFINITY;
          sm = 0.f;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint4*>(stg + lane * 128 + ((j ^ (lane & 7)) << 4)) =
              make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rr = 4 * i + (lane >> 3), j = lane & 7;  // row of the warp's 32, 16-byte chunk
          const uint4 v = *reinterpret_cast<const uint4*>(stg + rr * 128 + ((j ^ (rr & 7)) << 4));
          const int col = n0 + c0 + 4 * j;
          const int grow = m0 + q * 32 + rr;
          if (grow < p.M && col + 4 <= p.N)
            *reinterpret_cast<uint4*>(outc + (int64_t)grow * p.ldo + col) = v;
        }
        __syncwarp();
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    // 64 columns at a time: TMEM -> bf16 -> the warp's 4 KiB of staging
    // (16-byte chunks swizzled by row) -> read back so that each warp-wide
    // store covers four whole 128-byte row pieces.
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;
    uint8_t* stg = smem + C::OFF_EPI + q * 4096;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      const int tm = t % p.tiles_m, tn = t / p.tiles_m;
      int m0 = tm * BM, n0 = tn * BN;
      if (!warp_wait(&tfull[acc], acc_phase, ab)) break;
      tc_fence_after();
      const int gm = m0 + row;
      bf16* out = static_cast<bf16*>(p.out0);
      int om = gm, on0 = n0;
      if (p.out_switch_m > 0 && m0 >= p.out_switch_m) {
        out = static_cast<bf16*>(p.out1);
        om -= p.out_switch_m;
      }
      if (p.out_switch_n > 0 && n0 >= p.out_switch_n) {
        out = static_cast<bf16*>(p.out1);
        on0 -= p.out_switch_n;
      }
      const int n_lim = (p.out_switch_n > 0 && n0 < p.out_switch_n) ? p.out_switch_n : p.N;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 64) {
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
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rr = 4 * i + (lane >> 3), j = lane & 7;  // row of the warp's 32, 16-byte chunk
          const uint4 v = *reinterpret_cast<const uint4*>(stg + rr * 128 + ((j ^ (rr & 7)) << 4));
          const int col = n0 + c0 + 8 * j;
          if (m0 + q * 32 + rr < p.M && col + 8 <= n_lim)
            *reinterpret_cast<uint4*>(out + (int64_t)(om - lane + rr) * p.ldo + on0 + c0 + 8 * j) = v;
        }
        __syncwarp();
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::once_flag g_encode_once;
EncodeTiledFn g_encode = nullptr;

}  // namespace

cudaError_t make_tmap_bf16_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                              uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer) {
  std::call_once(g_encode_once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  if (!g_encode) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// bf16 [outer][mid][inner] tensor, 128B swizzle, box {box_inner, box_mid, 1}.
cudaError_t make_tmap_bf16_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
                              uint32_t box_inner, uint32_t box_mid) {
  std::call_once(g_encode_once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  if (!g_encode) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {inner, mid, outer};
  const cuuint64_t strides[2] = {inner * 2, inner * mid * 2};
  const cuuint32_t box[3] = {box_inner, box_mid, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_tokens(CUtensorMap* m, const void* base, int B, int T, int H, int hd, uint32_t box_rows) {
  std::call_once(g_encode_once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  if (!g_encode) return cudaErrorNotSupported;
  const cuuint64_t dims[4] = {(cuuint64_t)hd, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)hd * 2, (cuuint64_t)H * hd * 2, (cuuint64_t)T * H * hd * 2};
  const cuuint32_t box[4] = {64, 1, box_rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// bf16 [rows, inner] row-major tensor without swizzle (the box lands row-major
// in shared memory), box {box_inner, box_rows}; inner * 2 bytes per row.
cudaError_t make_tmap_bf16_2d_plain(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                                    uint32_t box_inner, uint32_t box_rows) {
  std::call_once(g_encode_once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  if (!g_encode) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// fp32 [B,T,H,hd] token tensor, box {32 channels, 1 head, box_rows rows, 1},
// 128B swizzle: the target of the dQ reduce-add of the attention backward.
cudaError_t make_tmap_f32_tokens(CUtensorMap* m, void* base, int B, int T, int H, int hd, uint32_t box_rows) {
  std::call_once(g_encode_once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  if (!g_encode) return cudaErrorNotSupported;
  const cuuint64_t dims[4] = {(cuuint64_t)hd, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)hd * 4, (cuuint64_t)H * hd * 4, (cuuint64_t)T * H * hd * 4};
  const cuuint32_t box[4] = {32, 1, box_rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

namespace {

template <int BN, bool A_MN, bool B_MN, int EPI = EPI_BF16>
cudaError_t run_gemm(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b0, const CUtensorMap& b1,
                     TcGemmParams p, cudaStream_t s) {
  using C = Cfg<BN, A_MN, B_MN>;
  auto kern = tc_gemm_kernel<BN, A_MN, B_MN, EPI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  if (e != cudaSuccess) return e;
  const int tiles = p.tiles_m * p.tiles_n;
  const int grid = tiles < num_sms() ? tiles : num_sms();
  kern<<<grid, NUM_THREADS, C::SMEM, s>>>(a0, a1, b0, b1, p);
  return cudaGetLastError();
}

}  // namespace

// Two-SM (CTA pair) versions of the projection GEMMs (tc_gemm_pair.cu); they
// return cudaErrorNotSupported when clusters of two cannot be launched.
bool pair_gemm_supported(int D);
cudaError_t launch_proj_fwd_pair(int64_t M, int D, int d, const void* m_shift, const void* w_mk, const void* w_mv,
                                 void* Rk, void* Rv, int64_t spin_limit, int* err, cudaStream_t s);
cudaError_t launch_proj_bwd_dm_pair(int64_t M, int D, int d, const void* dRk, const void* dRv, const void* w_mk,
                                    const void* w_mv, void* dm, int64_t spin_limit, int* err, cudaStream_t s);
cudaError_t launch_proj_bwd_dm_layers_pair(int64_t M, int D, int d, int L, const void* dRk, const void* dRv,
                                           const void* w_mk, const void* w_mv, void* dm, int64_t spin_limit,
                                           int* err, cudaStream_t s);
cudaError_t launch_proj_bwd_dw_pair(int64_t M, int D, int d, const void* dRk, const void* dRv, const void* m_shift,
                                    void* dwk, void* dwv, int64_t spin_limit, int* err, cudaStream_t s);

// R_k | R_v [M, D] = m_shift [M, d] x W^T, W_mk / W_mv [D, d].
cudaError_t launch_proj_fwd_tc(int64_t M, int D, int d, const void* m_shift, const void* w_mk,
                               const void* w_mv, void* Rk, void* Rv, int64_t spin_limit, int* err,
                               cudaStream_t s) {
  if (pair_gemm_supported(D)) {
    const cudaError_t pe = launch_proj_fwd_pair(M, D, d, m_shift, w_mk, w_mv, Rk, Rv, spin_limit, err, s);
    if (pe != cudaErrorNotSupported) return pe;
  }
  constexpr int BN = 256;
  CUtensorMap a, b0, b1;
  cudaError_t e;
  if ((e = make_tmap_bf16_2d(&a, m_shift, d, M, (uint64_t)d * 2, 64, BM)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&b0, w_mk, d, D, (uint64_t)d * 2, 64, BN)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&b1, w_mv, d, D, (uint64_t)d * 2, 64, BN)) != cudaSuccess) return e;
  TcGemmParams p{};
  p.M = (int)M;
  p.N = 2 * D;
  p.K = d;
  p.tiles_m = (int)((M + BM - 1) / BM);
  p.tiles_n = (2 * D + BN - 1) / BN;
  p.b_switch_n = D;
  p.out_switch_n = D;
  p.out0 = Rk;
  p.out1 = Rv;
  p.ldo = D;
  p.spin_limit = spin_limit;
  p.err = err;
  return run_gemm<BN, false, false>(a, a, b0, b1, p, s);
}

// dm [M, d] = dR_k [M, D] W_mk [D, d] + dR_v W_mv (K = 2D, B operand N-contiguous).
cudaError_t launch_proj_bwd_dm_tc(int64_t M, int D, int d, const void* dRk, const void* dRv,
                                  const void* w_mk, const void* w_mv, void* dm, int64_t spin_limit,
                                  int* err, cudaStream_t s) {
  if (pair_gemm_supported(D)) {
    const cudaError_t pe = launch_proj_bwd_dm_pair(M, D, d, dRk, dRv, w_mk, w_mv, dm, spin_limit, err, s);
    if (pe != cudaErrorNotSupported) return pe;
  }
  constexpr int BN = 256;
  CUtensorMap a0, a1, b0, b1;
  cudaError_t e;
  if ((e = make_tmap_bf16_2d(&a0, dRk, D, M, (uint64_t)D * 2, 64, BM)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&a1, dRv, D, M, (uint64_t)D * 2, 64, BM)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&b0, w_mk, d, D, (uint64_t)d * 2, 64, 64)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&b1, w_mv, d, D, (uint64_t)d * 2, 64, 64)) != cudaSuccess) return e;
  TcGemmParams p{};
  p.M = (int)M;
  p.N = d;
  p.K = 2 * D;
  p.tiles_m = (int)((M + BM - 1) / BM);
  p.tiles_n = (d + BN - 1) / BN;
  p.a_switch_k = D;
  p.b_switch_k = D;
  p.out0 = dm;
  p.out1 = dm;
  p.ldo = d;
  p.spin_limit = spin_limit;
  p.err = err;
  return run_gemm<BN, false, true>(a0, a1, b0, b1, p, s);
}

// dm [M, d] = sum over L layers of dR_k^l [M, D] W_mk^l [D, d] + dR_v^l W_mv^l, with
// dR [L][M][D] and W [L][D][d] layer-strided (K = 2 L D, one fp32 accumulation).
cudaError_t launch_proj_bwd_dm_layers_tc(int64_t M, int D, int d, int L, const void* dRk, const void* dRv,
                                         const void* w_mk, const void* w_mv, void* dm, int64_t spin_limit,
                                         int* err, cudaStream_t s) {
  if (pair_gemm_supported(D)) {
    const cudaError_t pe =
        launch_proj_bwd_dm_layers_pair(M, D, d, L, dRk, dRv, w_mk, w_mv, dm, spin_limit, err, s);
    if (pe != cudaErrorNotSupported) return pe;
  }
  constexpr int BN = 256;
  CUtensorMap a0, a1, b0, b1;
  cudaError_t e;
  if ((e = make_tmap_bf16_3d(&a0, dRk, D, M, L, 64, BM)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_3d(&a1, dRv, D, M, L, 64, BM)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_3d(&b0, w_mk, d, D, L, 64, 64)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_3d(&b1, w_mv, d, D, L, 64, 64)) != cudaSuccess) return e;
  TcGemmParams p{};
  p.M = (int)M;
  p.N = d;
  p.K = 2 * L * D;
  p.tiles_m = (int)((M + BM - 1) / BM);
  p.tiles_n = (d + BN - 1) / BN;
  p.a_switch_k = D;
  p.b_switch_k = D;
  p.k_layers = L;
  p.out0 = dm;
  p.out1 = dm;
  p.ldo = d;
  p.spin_limit = spin_limit;
  p.err = err;
  return run_gemm<BN, false, true>(a0, a1, b0, b1, p, s);
}

// dW_mk | dW_mv [D, d] = dR^T [D, M] m_shift [M, d] (A and B both M-contiguous in memory).
// 128 x 192 tiles: at D = d = 1280 that is 20 x 7 = 140 tiles, one per SM in a
// single wave (128 x 256 would give 100 tiles and leave a third of the SMs idle);
// N = 192 still keeps the shared-memory operand traffic of an MMA under the
// per-cycle limit.
cudaError_t launch_proj_bwd_dw_tc(int64_t M, int D, int d, const void* dRk, const void* dRv,
                                  const void* m_shift, void* dwk, void* dwv, int64_t spin_limit,
                                  int* err, cudaStream_t s) {
  if (pair_gemm_supported(D)) {
    const cudaError_t pe = launch_proj_bwd_dw_pair(M, D, d, dRk, dRv, m_shift, dwk, dwv, spin_limit, err, s);
    if (pe != cudaErrorNotSupported) return pe;
  }
  constexpr int BN = 192;
  CUtensorMap a0, a1, b;
  cudaError_t e;
  if ((e = make_tmap_bf16_2d(&a0, dRk, D, M, (uint64_t)D * 2, 64, 64)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&a1, dRv, D, M, (uint64_t)D * 2, 64, 64)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&b, m_shift, d, M, (uint64_t)d * 2, 64, 64)) != cudaSuccess) return e;
  TcGemmParams p{};
  p.M = 2 * D;
  p.N = d;
  p.K = (int)M;
  p.tiles_m = (2 * D + BM - 1) / BM;
  p.tiles_n = (d + BN - 1) / BN;
  p.a_switch_m = D;
  p.out_switch_m = D;
  p.out0 = dwk;
  p.out1 = dwv;
  p.ldo = d;
  p.spin_limit = spin_limit;
  p.err = err;
  return run_gemm<BN, true, true>(a0, a1, b, b, p, s);
}

// ---------------------------------------------------------------- LM head
// c [N, V] fp32 = softcap * tanh(m [N, d] U [V, d]^T / softcap), with per-row,
// per-256-column (max, sum exp) pairs in part [N, ceil(V / 256)] and the
// target's capped logit in tgt [N]. Needs d % 8 == 0, V % 8 == 0.
cudaError_t launch_lm_logits_ce_tc(int64_t N, int d, int V, float softcap, const void* m, const void* U,
                                   const int64_t* targets, float* c, float2* part, float* tgt,
                                   int64_t spin_limit, int* err, cudaStream_t s) {
  {  // SM pairs first (tc_gemm_pair.cu); one SM per tile where clusters cannot run
    const cudaError_t pe = launch_lm_logits_ce_pair(N, d, V, softcap, m, U, targets, c, part, tgt, spin_limit, err, s);
    if (pe != cudaErrorNotSupported) return pe;
  }
  constexpr int BN = 256;
  CUtensorMap a, b;
  cudaError_t e;
  if ((e = make_tmap_bf16_2d(&a, m, d, N, (uint64_t)d * 2, 64, BM)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&b, U, d, V, (uint64_t)d * 2, 64, BN)) != cudaSuccess) return e;
  TcGemmParams p{};
  p.M = (int)N;
  p.N = V;
  p.K = d;
  p.tiles_m = (int)((N + BM - 1) / BM);
  p.tiles_n = (V + BN - 1) / BN;
  p.targets = targets;
  p.softcap = softcap;
  p.ce_part = part;
  p.ce_tgt = tgt;
  p.out0 = c;
  p.out1 = c;
  p.ldo = V;
  p.spin_limit = spin_limit;
  p.err = err;
  return run_gemm<BN, false, false, EPI_CE>(a, a, b, b, p, s);
}

int lm_ce_tiles(int V) { return (V + 127) / 128; }  // (max, sum) partials per row: one per 128 columns

// dm [N, d] = dz [N, V] U [V, d] (K = V).
cudaError_t launch_lm_dm_tc(int64_t N, int d, int V, const void* dz, const void* U, void* dm, int64_t spin_limit,
                            int* err, cudaStream_t s) {
  constexpr int BN = 256;
  CUtensorMap a, b;
  cudaError_t e;
  if ((e = make_tmap_bf16_2d(&a, dz, V, N, (uint64_t)V * 2, 64, BM)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&b, U, d, V, (uint64_t)d * 2, 64, 64)) != cudaSuccess) return e;
  TcGemmParams p{};
  p.M = (int)N;
  p.N = d;
  p.K = V;
  p.tiles_m = (int)((N + BM - 1) / BM);
  p.tiles_n = (d + BN - 1) / BN;
  p.out0 = dm;
  p.out1 = dm;
  p.ldo = d;
  p.spin_limit = spin_limit;
  p.err = err;
  return run_gemm<BN, false, true>(a, a, b, b, p, s);
}

// dU [V, d] = dz^T [V, N] m [N, d] (K = N).
cudaError_t launch_lm_dU_tc(int64_t N, int d, int V, const void* dz, const void* m, void* dU, int64_t spin_limit,
                            int* err, cudaStream_t s) {
  constexpr int BN = 256;
  CUtensorMap a, b;
  cudaError_t e;
  if ((e = make_tmap_bf16_2d(&a, dz, V, N, (uint64_t)V * 2, 64, 64)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2d(&b, m, d, N, (uint64_t)d * 2, 64, 64)) != cudaSuccess) return e;
  TcGemmParams p{};
  p.M = V;
  p.N = d;
  p.K = (int)N;
  p.tiles_m = (V + BM - 1) / BM;
  p.tiles_n = (d + BN - 1) / BN;
  p.out0 = dU;
  p.out1 = dU;
  p.ldo = d;
  p.spin_limit = spin_limit;
  p.err = err;
  return run_gemm<BN, true, true>(a, a, b, b, p, s);
}

}  // namespace maglev
