/*
 * maglev.h -- C ABI of the B200 (sm_100a) implementation of Maglev's injected
 * sliding-window attention ("Maglev: Sliding Recurrent Memory", arXiv 2608.02870).
 *
 * Page citations: [rainbus] = paper.rainbus.top, sections 前置知识 (SWA, KV cache,
 * RoPE), 研究动机 (the interface p(x_{t+1}, m_t | x_{t-W+1:t}, M_{t-1})) and
 * 方法步骤详情 (every formula); [gist] = gist.science, section Inferentiemechanisme.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Ownership: every tensor argument is a caller-owned DEVICE pointer (any
 *    allocator). The library never allocates device memory and never frees
 *    the caller's. Scratch memory is passed in by the caller; its size comes
 *    from the matching *_bytes() query.
 *  - Layout: dense, row-major, innermost index last, 16-byte aligned base.
 *    Token-major activations: [B, T, H, hd] (equivalently [B, T, D], D = H*hd).
 *  - dtype: MAGLEV_BF16 (bf16 storage, fp32 accumulation; tensor-core path) or
 *    MAGLEV_F32 (fp32 storage and arithmetic on CUDA cores). Gate logits, LSE,
 *    gate gradients and the loss are always fp32.
 *  - Streams: `stream` is a cudaStream_t (NULL = legacy default stream). Every
 *    call only enqueues work; none synchronises the device.
 *  - Errors: arguments are validated on the host before any launch. A call
 *    returns MAGLEV_OK, or an error code with nothing enqueued (INVALID_ARG,
 *    UNSUPPORTED) or after a CUDA launch error (CUDA). maglev_last_error()
 *    returns the message of the calling thread's last failure. Kernels that
 *    wait on asynchronous copies or tensor-core work bound every wait by
 *    desc->spin_limit microseconds of GPU time (0 = 1 s); on expiry they
 *    record MAGLEV_ERR_TIMEOUT in a device status word, stop issuing work,
 *    drain what is in flight (bounded by 2 s), free their tensor memory and
 *    return; read the word with maglev_device_status().
 *  - Empty problems (B == 0 or T == 0, rows == 0) are valid and enqueue nothing.
 */
#ifndef MAGLEV_H
#define MAGLEV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MAGLEV_OK = 0,
  MAGLEV_ERR_INVALID_ARG = 1,
  MAGLEV_ERR_UNSUPPORTED = 2,
  MAGLEV_ERR_CUDA = 3,
  MAGLEV_ERR_TIMEOUT = 4,
  /* Only from a library built with -DMAGLEV_DEBUG (libmaglev_debug.so): an
   * in-kernel index check failed; the access was skipped. Reported through
   * maglev_device_status like MAGLEV_ERR_TIMEOUT. */
  MAGLEV_ERR_BOUNDS = 5
} maglev_status;

typedef enum { MAGLEV_F32 = 0, MAGLEV_BF16 = 1 } maglev_dtype;

/* Shapes and options of one injected sliding-window attention layer.
 * B batch, T sequence length, H heads, hd head dim (64 or 128), d_mem memory
 * width, window W >= 1 (keys j in [i-W+1, i]; W >= T is full causal attention),
 * rope_base (10000 in the d20 model), rms_eps (1e-6), inject (0: plain SWA --
 * memory arguments may be NULL), pos0 (absolute position of row 0), dtype,
 * spin_limit (bound on each in-kernel wait in microseconds, 0 = 1 s),
 * shared_kv_gates: 0 -- gate_logits is [4,H] (k_loc, k_rec, v_loc, v_rec);
 * 1 -- gate_logits is [2,H] (loc, rec), the value reusing the key's gates
 * ([rainbus] 方法步骤详情 gives the key's gates and mixes the value "likewise");
 * the gate gradient then has the same [2,H] shape. */
typedef struct {
  int B, T, H, hd, d_mem, window;
  float rope_base, rms_eps;
  int inject;
  int pos0;
  int dtype;
  int64_t spin_limit;
  int shared_kv_gates;
} maglev_swa_desc;

/* Shapes of one recurrent decode layer: B sequences, H heads, hd, d_mem,
 * window W = ring length; shared_kv_gates as in maglev_swa_desc. */
typedef struct {
  int B, H, hd, d_mem, window;
  float rope_base, rms_eps;
  int inject;
  int dtype;
  int64_t spin_limit;
  int shared_kv_gates;
} maglev_decode_desc;

/* Library version string (static storage). */
const char* maglev_version(void);

/* Tracing. maglev_launch_count() returns the number of kernels this library
 * has launched in the process so far (all threads, all devices).
 * maglev_profile_enable(1) brackets every later launch with CUDA events
 * recorded on the launch's own stream; maglev_profile_report() waits for the
 * recorded events and returns the length of the report text, one line
 * "name kernels milliseconds" per traced launch. With buf != NULL it also
 * copies the text into buf (NUL-terminated, truncated to n bytes) and clears
 * it; with buf == NULL it only returns the length. Tracing is off by default. */
long long maglev_launch_count(void);
void maglev_profile_enable(int on);
size_t maglev_profile_report(char* buf, size_t n);

/* Copies the calling thread's last error message into buf (NUL-terminated,
 * truncated to n bytes). Returns the full message length. */
size_t maglev_last_error(char* buf, size_t n);

/* Reads and clears the device status word of the current device after the
 * work queued on `stream` completes (this call synchronises that stream).
 * *code receives MAGLEV_OK or the first MAGLEV_ERR_TIMEOUT recorded. */
maglev_status maglev_device_status(void* stream, int* code);

/* Self-test of the bounded waits that every tensor-core kernel of this library
 * uses (no counterpart in the pages: part of this library's failure handling).
 * One CTA starts a bulk copy of `bytes` bytes from `src` into shared memory,
 * allocates tensor memory, then waits on an mbarrier that nothing completes;
 * after spin_limit microseconds of GPU time the wait gives up, raises the
 * CTA's abort flag and records MAGLEV_ERR_TIMEOUT in the device status word,
 * the copy is drained, the tensor memory freed, and the kernel returns. After
 * the work on `stream` completes, maglev_device_status reports the timeout.
 *   src: device buffer, 16-byte aligned; bytes: a multiple of 16 in [16, 4096].
 *   spin_limit: in [1, 1e7] microseconds. */
maglev_status maglev_wait_selftest(const void* src, int bytes, int64_t spin_limit, void* stream);

/* Bytes of the activations the forward saves for the backward ("saved"):
 * the rotated queries and the mixed keys/values, 3 x [B,T,H,hd] of dtype. */
size_t maglev_swa_saved_bytes(const maglev_swa_desc* desc);

/* Bytes of scratch memory maglev_inject_swa_bwd needs ("workspace"). */
size_t maglev_swa_bwd_workspace_bytes(const maglev_swa_desc* desc);

/* a1 -- memory projection ([rainbus] 方法步骤详情: k_rec, v_rec come from the
 * shared projections W_k^rec, W_v^rec applied to m'_{t-1}).
 *   m_shift [B,T,d_mem]: row t holds m'_{t-1}, row 0 holds m'_0 = 0.
 *   w_mk, w_mv [D, d_mem]: the shared projections (no layer index).
 *   R_k, R_v [B,T,D] (out): R_k = m_shift W_mk^T, R_v = m_shift W_mv^T (raw:
 *   no norm, no rotation). One call serves every layer of a step. */
maglev_status maglev_mem_project(const maglev_swa_desc* desc, const void* m_shift,
                                 const void* w_mk, const void* w_mv, void* R_k, void* R_v,
                                 void* stream);

/* a1-a5 -- forward of one injected sliding-window attention layer
 * ([rainbus] 方法步骤详情; 前置知识 for SWA and for rotating both keys before the
 * mix; [gist] Inferentiemechanisme: the memory rides in the existing K/V entry).
 *   q, k, v [B,T,H,hd]: local projections before RoPE.
 *   m_shift, w_mk, w_mv: if m_shift != NULL (and inject) the call first runs
 *     maglev_mem_project into R_k, R_v; if m_shift == NULL, R_k and R_v are
 *     inputs computed earlier (shared across layers). Unused when inject == 0.
 *   R_k, R_v [B,T,D]: raw projected memory (see a1), written or read as above.
 *   gate_logits [4,H] fp32: (k_loc, k_rec, v_loc, v_rec); g = 2*sigmoid(a),
 *     a = -inf allowed (g = 0); [2,H] (loc, rec) with shared_kv_gates.
 *   out [B,T,H,hd] (out): o_i = sum_j softmax_j(q~_i . k_bar_j / sqrt(hd)) v_bar_j
 *     over j in [i-W+1, i], with q~ = RoPE(q), k_bar = g_kl RoPE(k) +
 *     g_kr RoPE(RMSNorm_head(R_k)), v_bar = g_vl v + g_vr R_v.
 *   lse [B,H,T] fp32 (out): log-sum-exp of each row's scaled scores.
 *   saved (out): maglev_swa_saved_bytes(desc) bytes, read by the backward. */
maglev_status maglev_inject_swa_fwd(const maglev_swa_desc* desc, const void* q, const void* k,
                                    const void* v, const void* m_shift, const void* w_mk,
                                    const void* w_mv, void* R_k, void* R_v,
                                    const float* gate_logits, void* out, float* lse, void* saved,
                                    void* stream);

/* How maglev_inject_swa_bwd stores dL/dR of the shared projection. The layers
 * of a decoder share W^rec ([rainbus] 方法步骤详情: one projection for all
 * layers), so its gradient is the sum of every layer's dL/dR. The sum is kept
 * in fp32 running sums (dR_acc_k, dR_acc_v) and rounded to the activation type
 * once, by the last layer of the backward sweep:
 *   MAGLEV_DR_WRITE  dR (dtype) = this layer's dL/dR (a single layer)
 *   MAGLEV_DR_FIRST  dR_acc (fp32) = this layer's dL/dR (first layer of a sweep)
 *   MAGLEV_DR_ADD    dR_acc (fp32) += this layer's dL/dR
 *   MAGLEV_DR_LAST   dR (dtype) = dR_acc + this layer's dL/dR (last layer) */
typedef enum {
  MAGLEV_DR_WRITE = 0,
  MAGLEV_DR_FIRST = 1,
  MAGLEV_DR_ADD = 2,
  MAGLEV_DR_LAST = 3
} maglev_dr_mode;

/* Or'd into dR_mode of maglev_inject_swa_bwd: the backward workspace already
 * holds Delta and the zeroed dQ accumulator for this out and dout, written by
 * maglev_consistency_loss_prepare_bwd, so the backward skips its own first
 * pass over out and dout. */
#define MAGLEV_BWD_PREPARED 16

/* a6 -- backward of maglev_inject_swa_fwd (chain rule of the forward above).
 *   Inputs: the forward's k, v, R_k, R_v, gate_logits, out, lse, saved, and
 *   dout [B,T,H,hd] = dL/dout.
 *   dq, dk, dv [B,T,H,hd] (out, overwritten).
 *   dR_k, dR_v [B,T,D] of dtype (out): written in modes WRITE and LAST; may be
 *     NULL in modes FIRST and ADD, and when inject == 0.
 *   dR_acc_k, dR_acc_v [B,T,D] fp32: the running sums, written (FIRST), updated
 *     (ADD) or read (LAST); unused (may be NULL) in mode WRITE.
 *   dR_mode: a maglev_dr_mode value, with MAGLEV_BWD_PREPARED or'd in when
 *     maglev_consistency_loss_prepare_bwd has run on this out, dout and workspace.
 *   dgate_logits [4,H] fp32 ([2,H] with shared_kv_gates; out, overwritten);
 *     NULL when inject == 0.
 *   m_shift, w_mk, w_mv, dm_shift, dw_mk, dw_mv: if m_shift != NULL the call
 *     finishes with maglev_mem_project_bwd on dR_k, dR_v (modes WRITE and LAST).
 *   workspace: maglev_swa_bwd_workspace_bytes(desc) bytes of scratch.
 * Errors: INVALID_ARG for a bad dR_mode, for m_shift != NULL in modes FIRST or
 * ADD, and for a NULL pointer the mode needs. */
maglev_status maglev_inject_swa_bwd(const maglev_swa_desc* desc, const void* k, const void* v,
                                    const void* R_k, const void* R_v, const float* gate_logits,
                                    const void* out, const float* lse, const void* saved,
                                    const void* dout, void* dq, void* dk, void* dv, void* dR_k,
                                    void* dR_v, float* dR_acc_k, float* dR_acc_v, int dR_mode,
                                    float* dgate_logits, const void* m_shift, const void* w_mk,
                                    const void* w_mv, void* dm_shift, void* dw_mk, void* dw_mv,
                                    void* workspace, void* stream);

/* a6 -- backward of the shared memory projection.
 *   dm_shift [B,T,d_mem] = dR_k W_mk + dR_v W_mv (overwritten; NULL: not computed);
 *   dw_mk, dw_mv [D,d_mem] = dR^T m_shift summed over all B*T rows (overwritten;
 *     NULL as a pair: not computed).
 * With all three outputs, bf16, d_mem % 8 == 0 and H*hd % 128 == 0, both
 * products run in one launch on SM pairs. */
maglev_status maglev_mem_project_bwd(const maglev_swa_desc* desc, const void* m_shift,
                                     const void* w_mk, const void* w_mv, const void* dR_k,
                                     const void* dR_v, void* dm_shift, void* dw_mk, void* dw_mv,
                                     void* stream);

/* Backward of per-layer memory projections: one W^rec per decoder layer, the
 * variant [rainbus] 未来方向 lists (逐层记忆投影) beside the shared projection.
 * Layer l's forward is maglev_mem_project with that layer's weights into its
 * own R^l; its maglev_inject_swa_bwd writes dL/dR^l in mode MAGLEV_DR_WRITE.
 *   n_layers L >= 1.
 *   w_mk, w_mv [L, D, d_mem]: the layers' projections, layer-strided.
 *   dR_k, dR_v [L, B, T, D]: each layer's dL/dR^l, layer-strided.
 *   dm_shift [B,T,d_mem] (out, nullable) = sum over l of dR_k^l W_mk^l +
 *     dR_v^l W_mv^l, accumulated in fp32 over all layers and rounded once.
 *   dw_mk, dw_mv [L, D, d_mem] (out, nullable as a pair): dW^l = dR^l^T m_shift.
 * Errors: INVALID_ARG for n_layers < 1 or bad pointers; UNSUPPORTED for bf16
 * unless d_mem % 8 == 0 and H*hd % 128 == 0. */
maglev_status maglev_mem_project_bwd_layers(const maglev_swa_desc* desc, int n_layers,
                                            const void* m_shift, const void* w_mk, const void* w_mv,
                                            const void* dR_k, const void* dR_v, void* dm_shift,
                                            void* dw_mk, void* dw_mv, void* stream);

/* Memory state of a decoder stack ([rainbus] 方法步骤详情: m_t is the stack's
 * final state after RMSNorm; the injection reads the shifted memory m_{t-1},
 * with m_0 = 0). Reading: RMSNorm over the d channels of each row, no weight.
 *   o [B,T,d]: the last layer's output (dtype).
 *   m [B,T,d] (out): m[b,t] = o[b,t] / sqrt(mean_c o[b,t,c]^2 + eps).
 *   m_shift [B,T,d] (out, nullable): m_shift[b,0] = 0, m_shift[b,t] = m[b,t-1],
 *     the layout maglev_inject_swa_fwd reads.
 *   rstd [B*T] fp32 (out): 1/sqrt(mean(o^2) + eps), read by the backward.
 * Errors: MAGLEV_ERR_INVALID_ARG for negative sizes, d < 1, eps < 0, bad dtype or
 * a NULL pointer that is not marked nullable. */
maglev_status maglev_memory_state(int B, int T, int d, float eps, int dtype, const void* o,
                                  void* m, void* m_shift, float* rstd, void* stream);

/* Backward of maglev_memory_state. The incoming gradient of row (b,t) is
 * g = dm[b,t] + dm_shift[b,t+1] (a term is absent when its pointer is NULL or
 * t+1 = T); its image through RMSNorm is rstd * (g - m * mean_c(m * g)), with m
 * recomputed from o in fp32.
 *   d_o [B,T,d] (out) = dout_in + that image; dout_in (nullable) is the
 *   gradient o already receives from elsewhere and may alias d_o. */
maglev_status maglev_memory_state_bwd(int B, int T, int d, int dtype, const void* o,
                                      const float* rstd, const void* dm, const void* dm_shift,
                                      const void* dout_in, void* d_o, void* stream);

/* Bytes of scratch memory maglev_consistency_loss needs for `rows` x `d`. */
size_t maglev_consistency_workspace_bytes(int64_t rows, int d);

/* a7 -- consistency loss ([rainbus] 方法步骤详情):
 *   loss = lambda * inv_count * sum_t ||m_t - m'_t||^2 / sqrt(d)
 *   m, m_target [rows, d] of dtype; inv_count = 1/|I| (0 means 1/rows).
 *   loss: device fp32 scalar (out). The sum is reduced in a fixed order, so the
 *   result is bitwise reproducible.
 *   dm (nullable): dL/dm = 2 lambda inv_count (m - m') / sqrt(d); written, or
 *     added to when accumulate_dm != 0. dm_target (nullable): -dL/dm, written.
 *   workspace: maglev_consistency_workspace_bytes(rows, d) bytes. */
maglev_status maglev_consistency_loss(const void* m, const void* m_target, int64_t rows, int d,
                                      int dtype, float lambda, float inv_count, float* loss,
                                      void* dm, void* dm_target, int accumulate_dm,
                                      void* workspace, void* stream);

/* a7 fused with the first pass of a6, for a layer whose own output feeds the
 * consistency loss ([rainbus] 方法步骤详情: the loss on m; the backward of the
 * banded attention needs Delta_i = sum_c out_ic dout_ic per query row and head).
 * In one pass over out, m_target and dout it computes what
 * maglev_consistency_loss(m = out, dm = dout, accumulate_dm = 1) computes, the
 * same loss bit for bit and the same updated dout, and writes into the layer's
 * backward workspace Delta from the updated, stored dout and (bf16) the zeroed
 * fp32 dQ accumulator: what maglev_inject_swa_bwd's first pass writes. Call
 * maglev_inject_swa_bwd next on the same out, dout and workspace with
 * MAGLEV_BWD_PREPARED or'd into dR_mode.
 *   desc: the layer's descriptor (B, T, H, hd, dtype).
 *   out, m_target [B,T,H,hd] of dtype; dout [B,T,H,hd] (in/out).
 *   lambda, inv_count, loss: as in maglev_consistency_loss (d = H*hd).
 *   bwd_workspace: maglev_swa_bwd_workspace_bytes(desc) bytes;
 *   loss_workspace: maglev_consistency_workspace_bytes(B*T, H*hd) bytes.
 * Errors: as maglev_consistency_loss, and the descriptor checks of the layer
 * calls. */
maglev_status maglev_consistency_loss_prepare_bwd(const maglev_swa_desc* desc, const void* out,
                                                  const void* m_target, float lambda, float inv_count,
                                                  float* loss, void* dout, void* bwd_workspace,
                                                  void* loss_workspace, void* stream);

/* Scratch-free variant of maglev_consistency_loss, for callers that cannot
 * allocate device memory: e.g. a plugin or custom-op interface that hands over
 * its input and output tensors but no workspace, or a latency-critical loop in
 * which cudaMalloc (which may synchronise the device) is not allowed. The
 * paper has no counterpart: this is an interface convenience of this library,
 * not a step of the method.
 * Same arguments and results as maglev_consistency_loss, minus `workspace`:
 * the per-block partial sums live in a file-scope device array of 32768 floats
 * (128 KiB) that every device which loads the library keeps until exit.
 * Limit: rows * d <= 67,108,864 elements; larger inputs return
 * MAGLEV_ERR_UNSUPPORTED with a message. The first call on each device looks
 * up the array's device address (cudaGetSymbolAddress) with that device
 * current: make that first call before any stream capture (a first call
 * inside a capture returns MAGLEV_ERR_CUDA). Every later call whose stream is
 * not being captured looks the address up again, so a device reset (which
 * reloads the library's device code) leaves no stale address. All calls share
 * the array and each call overwrites the partials it reads, so nothing needs
 * clearing, but calls that overlap on the GPU race and must be serialised.
 * The call allocates no memory. */
maglev_status maglev_consistency_loss_noalloc(const void* m, const void* m_target, int64_t rows,
                                              int d, int dtype, float lambda, float inv_count,
                                              float* loss, void* dm, void* dm_target,
                                              int accumulate_dm, void* stream);

/* Bytes of scratch memory maglev_lm_head_ce needs: the capped logits (fp32)
 * and their gradient (bf16), N x V each, plus per-row statistics. */
size_t maglev_lm_head_workspace_bytes(int64_t N, int d, int V);

/* LM head with softcapped logits and cross-entropy ([rainbus] 方法步骤详情: the
 * memory state m_t feeds p(x_{t+1} | x_<=t) = softmax(15 tanh(U m_t / 15)); the
 * loss averages the per-token CE over the positions in I).
 *   m [N, d] bf16: the memory states (rows = tokens); U [V, d] bf16.
 *   targets [N] int64 (device): the next token of each row, in [0, V); a row
 *     with a target outside that range gets a NaN CE (and so a NaN loss).
 *   softcap: 15 in the pages' model. inv_count = 1/|I| (0 means 1/N).
 *   loss: device fp32 scalar (out) = inv_count * sum_t (LSE_t - c_t[y_t]),
 *     c = softcap * tanh(U m / softcap), reduced in a fixed order.
 *   lse [N] fp32 (out): LSE_t of each row's capped logits.
 *   dm [N, d], dU [V, d] bf16 (out, nullable): gradients of the loss.
 *   workspace: maglev_lm_head_workspace_bytes(N, d, V) bytes.
 *   spin_limit: bound on each in-kernel wait in microseconds (0 = 1 s).
 * Errors: UNSUPPORTED unless dtype is MAGLEV_BF16 and d, V are multiples of 8. */
maglev_status maglev_lm_head_ce(int64_t N, int d, int V, int dtype, float softcap, float inv_count,
                                const void* m, const void* U, const int64_t* targets, float* loss,
                                float* lse, void* dm, void* dU, void* workspace, int64_t spin_limit,
                                void* stream);

/* a8 -- decode-side memory projection, once per token step (W^rec is shared by
 * all layers and m_{p-1} is the same for all of them):
 *   pos [B] int64 (device): absolute position p of each sequence's new token.
 *   m_prev [B,d_mem]: m_{p-1}, the previous step's memory.
 *   krec_rot [B,D] (out) = RoPE_p(RMSNorm_head(W_mk m_{p-1})); vrec [B,D] (out)
 *   = W_mv m_{p-1}. */
maglev_status maglev_decode_mem_project(const maglev_decode_desc* desc, const int64_t* pos,
                                        const void* m_prev, const void* w_mk, const void* w_mv,
                                        void* krec_rot, void* vrec, void* stream);

/* Ring prefill from a prompt: the bridge from the training form to recurrent
 * decoding ([rainbus] 研究动机: at inference m_t = P(x_{t-W+1:t}, M_{t-1}) over a
 * fixed window; 前置知识: the cache is that of plain SWA; [gist]
 * Inferentiemechanisme: the memory rides in the existing K/V entries).
 * After maglev_inject_swa_fwd over a prompt of T tokens at positions
 * pos0..pos0+T-1 (same desc), copies the mixed entries k_bar, v_bar of its
 * last min(T, W) positions from the forward's `saved` buffer into the rings:
 * the entry of absolute position j goes to slot j mod W of ring [b, h], with
 * W = desc->window (the ring length). No other slot changes. The rings then
 * hold the window that maglev_decode_step continues from at position pos0 + T,
 * fed with m_{pos0+T-1}.
 *   saved: the forward's saved buffer (maglev_swa_saved_bytes(desc) bytes).
 *   k_ring, v_ring [B,H,W,hd] of desc->dtype (in/out).
 * Errors: INVALID_ARG for a bad desc or a NULL / misaligned pointer. */
maglev_status maglev_decode_prefill(const maglev_swa_desc* desc, const void* saved, void* k_ring,
                                    void* v_ring, void* stream);

/* a8 -- one recurrent decode step of one layer over its rolling W-entry K/V
 * ring ([rainbus] 研究动机: m_t = P(x_{t-W+1:t}, M_{t-1}); 前置知识: the cache is
 * that of plain SWA; [gist] Inferentiemechanisme).
 *   pos [B] int64 (device): absolute position p of the new token. A negative
 *     entry leaves that sequence's ring untouched and writes zeros to its out.
 *   q, k, v [B,H,hd]: local projections of the new token, before RoPE.
 *   krec_rot, vrec [B,H,hd]: from maglev_decode_mem_project (unused if inject == 0).
 *   gate_logits [4,H] fp32 ([2,H] with shared_kv_gates): this layer's gates.
 *   k_ring, v_ring [B,H,W,hd] (in/out): post-RoPE, post-mix entries; the entry
 *     of position j lives in slot j mod W. The call writes the new entry to slot
 *     p mod W (no other slot changes), then attends over the live slots
 *     (positions max(0, p-W+1)..p).
 *   out [B,H,hd] (out).
 *   workspace: maglev_decode_workspace_bytes(desc) bytes of scratch, zero-filled
 *     by the caller before its first use; every call that completes leaves it
 *     zero-filled again (after a call that recorded MAGLEV_ERR_TIMEOUT, fill it
 *     with zeros again). Calls that share a workspace must not overlap. */
maglev_status maglev_decode_step(const maglev_decode_desc* desc, const int64_t* pos,
                                 const void* q, const void* k, const void* v,
                                 const void* krec_rot, const void* vrec, const float* gate_logits,
                                 void* k_ring, void* v_ring, void* out, void* workspace,
                                 void* stream);

/* Bytes of scratch memory maglev_decode_step needs (its `workspace`): the bf16
 * path splits each (sequence, head) ring into two halves streamed by separate
 * CTAs and keeps each half's partial softmax state and a per-pair counter
 * there; 0 for the fp32 path (workspace may then be NULL). */
size_t maglev_decode_workspace_bytes(const maglev_decode_desc* desc);

#ifdef __cplusplus
}
#endif

#endif /* MAGLEV_H */
