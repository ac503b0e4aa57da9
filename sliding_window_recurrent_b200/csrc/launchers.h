// Host-side launchers of libmaglev's kernels (internal C++ interface between
// the extern "C" boundary in api.cu and the kernel translation units).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace maglev {

// C[M,N] (+)= A1[M,K1] B1[K1,N] + A2[M,K2] B2[K2,N], fp32 accumulation, any
// element strides. A2/B2 may be null (K2 = 0). dtype: 0 = fp32, 1 = bf16 for
// all of A, B and C.
struct GemmArgs {
  int64_t M, N, K1, K2;
  const void *A1, *B1, *A2, *B2;
  int64_t sa1m, sa1k, sb1k, sb1n, sa2m, sa2k, sb2k, sb2n;
  void* C;
  int64_t scm, scn;
  int accumulate;
  int dtype;
};
cudaError_t launch_gemm_simt(const GemmArgs& g, cudaStream_t s);

struct SwaShape {
  int B, T, H, hd, W, pos0, inject, dtype;
  int vg;  // row of the value's first gate logit: 2 ([4, H] logits) or 0 (shared K/V gates, [2, H])
  double log2_base;
  float eps;
};

// q_rot = RoPE(q); k_bar, v_bar = gated mix (or RoPE(k), v when inject == 0).
cudaError_t launch_prep(const SwaShape& s, const void* q, const void* k, const void* v,
                        const void* Rk, const void* Rv, const float* gates, void* q_rot,
                        void* k_bar, void* v_bar, cudaStream_t st);
cudaError_t launch_attn_fwd_simt(const SwaShape& s, const void* q_rot, const void* k_bar,
                                 const void* v_bar, void* out, float* lse, cudaStream_t st);
// delta[b,h,i] = dout_i . out_i; zeroes dq_acc ([B,T,H,hd] fp32) when non-null.
cudaError_t launch_attn_delta(const SwaShape& s, const void* out, const void* dout, float* delta,
                              float* dq_acc, cudaStream_t st);
// dq = RoPE^T(dq_rot) written in dtype.
cudaError_t launch_attn_bwd_dq_simt(const SwaShape& s, const void* q_rot, const void* k_bar,
                                    const void* v_bar, const void* dout, const float* lse,
                                    const float* delta, void* dq, cudaStream_t st);
// dk_bar, dv_bar in the activation type.
cudaError_t launch_attn_bwd_dkdv_simt(const SwaShape& s, const void* q_rot, const void* k_bar,
                                      const void* v_bar, const void* dout, const float* lse,
                                      const float* delta, void* dk_bar, void* dv_bar,
                                      cudaStream_t st);
// How unmix stores dL/dR (values of maglev_dr_mode): DR_WRITE dR = g (dtype);
// DR_FIRST acc = g; DR_ADD acc += g; DR_LAST dR = acc + g (dtype), with the
// running sums acc in fp32.
constexpr int DR_WRITE = 0, DR_FIRST = 1, DR_ADD = 2, DR_LAST = 3;
// dk, dv, dR_k, dR_v (and dq from dq_acc when non-null) and per-row gate
// partials gpart[(g*H + h) * B*T + row] from dk_bar, dv_bar (activation type).
cudaError_t launch_unmix(const SwaShape& s, const void* dk_bar, const void* dv_bar,
                         const void* k, const void* v, const void* Rk, const void* Rv,
                         const float* gates, void* dk, void* dv, void* dRk, void* dRv,
                         float* accRk, float* accRv, int dr_mode, float* gpart,
                         const float* dq_acc, void* dq, cudaStream_t st);
// dgate [4, H] (or [2, H] when shared_kv) from the per-row partials.
cudaError_t launch_gate_reduce(int64_t rows, int H, int shared_kv, const float* gpart, const float* gates,
                               float* dgate, cudaStream_t st);

int loss_partial_blocks(int64_t n);
// dtype codes as in maglev_dtype
constexpr int DT_F32 = 0, DT_BF16 = 1;

// memory state m = RMSNorm(o) per row of d, with the shifted copy, and its backward
cudaError_t launch_memstate_fwd(const void* o, void* m, void* m_shift, float* rstd, int B, int T, int d,
                                float eps, int dtype, cudaStream_t st);
cudaError_t launch_memstate_bwd(const void* o, const float* rstd, const void* dm, const void* dm_shift,
                                const void* dout_in, void* dout, int B, int T, int d, int dtype, cudaStream_t st);

cudaError_t launch_consistency_loss(const void* m, const void* mt, int64_t rows, int d, int dtype,
                                    float scale_loss, float scale_grad, float* loss, void* dm,
                                    void* dmt, int accumulate, float* partials, cudaStream_t st);
// launch_consistency_loss of a layer's output (accumulating into dout) that also
// writes the attention backward's Delta [B,H,T] and zeroes dq_acc (nullable).
cudaError_t launch_consistency_loss_prep(const void* out, const void* mt, int64_t rows, int H, int hd, int seq,
                                         int dtype, float scale_loss, float scale_grad, float* loss, void* dout,
                                         float* delta, float* dq_acc, float* partials, cudaStream_t st);

struct DecShape {
  int B, H, hd, W, inject, dtype;
  int vg;  // as in SwaShape
  double log2_base;
  float eps;
};
cudaError_t launch_rmsnorm_rope_rows(const DecShape& s, const int64_t* pos, void* x,
                                     cudaStream_t st);
// Scratch of the split decode step: per work unit its partial softmax state.
size_t decode_workspace_bytes(const DecShape& s);
cudaError_t launch_decode_step(const DecShape& s, const int64_t* pos, const void* q, const void* k,
                               const void* v, const void* krec, const void* vrec,
                               const float* gates, void* k_ring, void* v_ring, void* out, void* workspace,
                               int64_t limit_us, int* err, cudaStream_t st);

// tcgen05 projection GEMMs (bf16 in/out, fp32 accumulation in TMEM).
// R_k | R_v [M, D] = m_shift [M, d] x [W_mk; W_mv]^T. Needs d % 8 == 0, D % 256 == 0.
cudaError_t launch_proj_fwd_tc(int64_t M, int D, int d, const void* m_shift, const void* w_mk,
                               const void* w_mv, void* Rk, void* Rv, int64_t spin_limit, int* err,
                               cudaStream_t s);
// dm [M, d] = dR_k W_mk + dR_v W_mv. Needs d % 8 == 0, D % 64 == 0.
cudaError_t launch_proj_bwd_dm_tc(int64_t M, int D, int d, const void* dRk, const void* dRv,
                                  const void* w_mk, const void* w_mv, void* dm, int64_t spin_limit,
                                  int* err, cudaStream_t s);
// dm [M, d] = sum over L layer-strided slabs of dR_k^l W_mk^l + dR_v^l W_mv^l
// (dR [L][M][D], W [L][D][d]). Needs d % 8 == 0, D % 64 == 0.
cudaError_t launch_proj_bwd_dm_layers_tc(int64_t M, int D, int d, int L, const void* dRk, const void* dRv,
                                         const void* w_mk, const void* w_mv, void* dm, int64_t spin_limit,
                                         int* err, cudaStream_t s);
// dW_mk | dW_mv [D, d] = dR^T m_shift. Needs d % 8 == 0, D % 128 == 0.
cudaError_t launch_proj_bwd_dw_tc(int64_t M, int D, int d, const void* dRk, const void* dRv,
                                  const void* m_shift, void* dwk, void* dwv, int64_t spin_limit,
                                  int* err, cudaStream_t s);
// dW and dm of the shared projection in one launch on SM pairs (tc_gemm_pair.cu),
// when proj_bwd_grouped_available says it can run.
bool proj_bwd_grouped_available(int64_t M, int D, int d);
// The LM head's dm and dU in one launch on SM pairs (tc_gemm_pair.cu), when
// lm_bwd_grouped_available says it can run.
bool lm_bwd_grouped_available(int64_t N, int d, int V);
// The LM head's logits GEMM with its softcapped CE epilogue on SM pairs;
// cudaErrorNotSupported when clusters cannot be launched (or V % 4 != 0).
cudaError_t launch_lm_logits_ce_pair(int64_t N, int d, int V, float softcap, const void* m, const void* U,
                                     const int64_t* targets, float* c, float2* part, float* tgt,
                                     int64_t spin_limit, int* err, cudaStream_t s);
cudaError_t launch_lm_bwd_grouped_pair(int64_t N, int d, int V, const void* dz, const void* U, const void* m,
                                       void* dm, void* dU, int64_t spin_limit, int* err, cudaStream_t s);
cudaError_t launch_proj_bwd_grouped_pair(int64_t M, int D, int d, const void* dRk, const void* dRv, const void* w_mk,
                                         const void* w_mv, const void* m_shift, void* dm, void* dwk, void* dwv,
                                         int64_t spin_limit, int* err, cudaStream_t s);
int num_sms();

// tcgen05 banded attention backward: dk_bar, dv_bar (bf16, rounded from the
// fp32 accumulators) and the rotated-frame dq reduce-added in fp32 into dq_acc
// (zeroed beforehand).
cudaError_t launch_attn_bwd_tc(const SwaShape& s, const void* q_rot, const void* k_bar, const void* v_bar,
                               const void* dout, const float* lse, const float* delta, float* dq_acc,
                               void* dk_bar, void* dv_bar, int64_t spin_limit, int* err, cudaStream_t st);

// tcgen05 banded attention forward on the saved bf16 q_rot / k_bar / v_bar.
cudaError_t launch_attn_fwd_tc(const SwaShape& s, const void* q_rot, const void* k_bar, const void* v_bar,
                               void* out, float* lse, int64_t spin_limit, int* err, cudaStream_t st);

// Copies k_bar, v_bar [B,T,H,hd] of the last min(T, W) positions into the
// rings [B,H,W,hd], position pos0 + t to slot (pos0 + t) mod W.
cudaError_t launch_ring_prefill(int B, int T, int H, int hd, int elt_bytes, int64_t W, int64_t pos0,
                                const void* k_bar, const void* v_bar, void* k_ring, void* v_ring,
                                cudaStream_t st);

// LM head with softcapped logits and cross-entropy (bf16 m [N,d], U [V,d]).
// Capped logits c [N,V] fp32 with per-row, per-256-column (max, sum exp) in
// part [N, lm_ce_tiles(V)] and the target's capped logit in tgt [N].
cudaError_t launch_lm_logits_ce_tc(int64_t N, int d, int V, float softcap, const void* m, const void* U,
                                   const int64_t* targets, float* c, float2* part, float* tgt,
                                   int64_t spin_limit, int* err, cudaStream_t s);
int lm_ce_tiles(int V);
// lse [N], ce [N] per row, loss = inv_count * sum ce; dz [N,V] bf16 when non-null.
cudaError_t launch_lm_ce_finish(int64_t N, int V, int tiles, float inv_count, float softcap, const float2* part,
                                const float* tgt, const int64_t* targets, const float* c, float* lse, float* ce,
                                float* loss, void* dz, cudaStream_t st);
// dm [N,d] = dz U; dU [V,d] = dz^T m (bf16, fp32 accumulation).
cudaError_t launch_lm_dm_tc(int64_t N, int d, int V, const void* dz, const void* U, void* dm, int64_t spin_limit,
                            int* err, cudaStream_t s);
cudaError_t launch_lm_dU_tc(int64_t N, int d, int V, const void* dz, const void* m, void* dU, int64_t spin_limit,
                            int* err, cudaStream_t s);

// One CTA: bulk copy of `bytes` from src into shared memory, tensor memory
// held, then a bounded wait on an mbarrier nothing completes (expires after
// limit_us, records DEV_TIMEOUT), drain, free, return.
cudaError_t launch_wait_selftest(const void* src, int bytes, int64_t limit_us, int* err, cudaStream_t st);

// Default bound of one in-kernel wait, in microseconds of GPU time (1 s).
constexpr int64_t DEFAULT_SPIN_LIMIT = 1000000;

// Sets the calling thread's message returned by maglev_last_error().
void set_last_error(const char* msg);

}  // namespace maglev
