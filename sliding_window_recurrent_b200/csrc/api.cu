// extern "C" boundary of libmaglev: argument validation, scratch layout and
// launch sequencing. Every step of the path runs in this library's kernels.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"
#include "launchers.h"
#include "maglev.h"

using namespace maglev;

namespace {

thread_local std::string g_last_error;

maglev_status fail(maglev_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

maglev_status cuda_fail(cudaError_t e, const char* where) {
  return fail(MAGLEV_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

// ---- tracing: launch counter and optional per-launch CUDA-event timing ----
std::atomic<long long> g_launches{0};
std::atomic<int> g_prof_on{0};
struct ProfRec {
  const char* name;
  int kernels;
  cudaEvent_t a, b;
};
std::mutex g_prof_mu;
std::vector<ProfRec> g_prof;
std::string g_prof_text;  // resolved records not yet handed out

struct ProfScope {
  const char* name;
  int kernels;
  cudaStream_t s;
  cudaEvent_t a = nullptr, b = nullptr;
  ProfScope(const char* n, int k, cudaStream_t st) : name(n), kernels(k), s(st) {
    if (g_prof_on.load(std::memory_order_relaxed)) {
      cudaEventCreate(&a);
      cudaEventCreate(&b);
      cudaEventRecord(a, s);
    }
  }
  ~ProfScope() {
    g_launches.fetch_add(kernels, std::memory_order_relaxed);
    if (a) {
      cudaEventRecord(b, s);
      std::lock_guard<std::mutex> lock(g_prof_mu);
      g_prof.push_back({name, kernels, a, b});
    }
  }
};

#define MAGLEV_CUDA(call, where)                        \
  do {                                                  \
    cudaError_t e_ = (call);                            \
    if (e_ != cudaSuccess) return cuda_fail(e_, where); \
  } while (0)

// Runs one launcher under a trace scope named `where` that launches `nk` kernels.
#define MAGLEV_LAUNCH(nk, stream, call, where)          \
  do {                                                  \
    ProfScope ps_(where, nk, stream);                   \
    cudaError_t e_ = (call);                            \
    if (e_ != cudaSuccess) return cuda_fail(e_, where); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define NEED_PTR(p)                                                                       \
  do {                                                                                    \
    if ((p) == nullptr) return fail(MAGLEV_ERR_INVALID_ARG, "%s must not be NULL", #p);   \
    if (!aligned16(p)) return fail(MAGLEV_ERR_INVALID_ARG, "%s must be 16-byte aligned", #p); \
  } while (0)

#define OPT_PTR(p)                                                                        \
  do {                                                                                    \
    if ((p) != nullptr && !aligned16(p))                                                  \
      return fail(MAGLEV_ERR_INVALID_ARG, "%s must be 16-byte aligned", #p);              \
  } while (0)

size_t elt(int dtype) { return dtype == MAGLEV_BF16 ? 2 : 4; }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

maglev_status check_swa(const maglev_swa_desc* d) {
  if (!d) return fail(MAGLEV_ERR_INVALID_ARG, "desc must not be NULL");
  if (d->B < 0 || d->T < 0) return fail(MAGLEV_ERR_INVALID_ARG, "B and T must be >= 0");
  if (d->H < 1) return fail(MAGLEV_ERR_INVALID_ARG, "H must be >= 1");
  if (d->hd != 64 && d->hd != 128)
    return fail(MAGLEV_ERR_UNSUPPORTED, "head dim %d unsupported (64 or 128)", d->hd);
  if (d->window < 1) return fail(MAGLEV_ERR_INVALID_ARG, "window must be >= 1");
  if (d->dtype != MAGLEV_F32 && d->dtype != MAGLEV_BF16)
    return fail(MAGLEV_ERR_INVALID_ARG, "dtype must be MAGLEV_F32 or MAGLEV_BF16");
  if (d->pos0 < 0) return fail(MAGLEV_ERR_INVALID_ARG, "pos0 must be >= 0");
  if (!(d->rope_base > 1.0f) || !std::isfinite(d->rope_base))
    return fail(MAGLEV_ERR_INVALID_ARG, "rope_base must be finite and > 1");
  if (!(d->rms_eps >= 0.0f) || !std::isfinite(d->rms_eps))
    return fail(MAGLEV_ERR_INVALID_ARG, "rms_eps must be finite and >= 0");
  if (d->inject && d->d_mem < 1) return fail(MAGLEV_ERR_INVALID_ARG, "d_mem must be >= 1");
  if ((int64_t)d->B * d->T > (int64_t)1 << 31)
    return fail(MAGLEV_ERR_UNSUPPORTED, "B*T too large");
  if ((int64_t)d->pos0 + d->T > (int64_t)1 << 30)
    return fail(MAGLEV_ERR_UNSUPPORTED, "positions beyond 2^30 are unsupported");
  return MAGLEV_OK;
}

SwaShape shape_of(const maglev_swa_desc* d) {
  SwaShape s;
  s.B = d->B;
  s.T = d->T;
  s.H = d->H;
  s.hd = d->hd;
  s.W = d->window < d->T ? d->window : (d->T > 0 ? d->T : 1);  // W >= T is full causal
  s.pos0 = d->pos0;
  s.inject = d->inject ? 1 : 0;
  s.dtype = d->dtype;
  s.vg = d->shared_kv_gates ? 0 : 2;
  s.log2_base = std::log2((double)d->rope_base);
  s.eps = d->rms_eps;
  return s;
}

// Offsets inside the caller's "saved" buffer: q_rot, k_bar, v_bar.
struct SavedLayout {
  size_t q, k, v, total;
};
SavedLayout saved_layout(const maglev_swa_desc* d) {
  const size_t n = align256((size_t)d->B * d->T * d->H * d->hd * elt(d->dtype));
  return {0, n, 2 * n, 3 * n};
}

// Offsets inside the backward's workspace.
struct BwdLayout {
  size_t dkb, dvb, delta, gpart, dq_acc, total;
};
BwdLayout bwd_layout(const maglev_swa_desc* d) {
  BwdLayout L;
  const size_t n = (size_t)d->B * d->T * d->H * d->hd;
  const size_t elt = d->dtype == MAGLEV_BF16 ? 2 : 4;  // dk_bar, dv_bar in the activation type
  L.dkb = 0;
  L.dvb = L.dkb + align256(n * elt);
  L.delta = L.dvb + align256(n * elt);
  L.gpart = L.delta + align256((size_t)d->B * d->H * d->T * 4);
  L.dq_acc = L.gpart + align256((size_t)d->B * d->T * 4 * d->H * 4);
  L.total = L.dq_acc + (d->dtype == MAGLEV_BF16 ? align256(n * 4) : 0);
  return L;
}

template <typename P>
P* at(void* base, size_t off) {
  return reinterpret_cast<P*>(static_cast<char*>(base) + off);
}
template <typename P>
const P* at(const void* base, size_t off) {
  return reinterpret_cast<const P*>(static_cast<const char*>(base) + off);
}

maglev_status status_word(int** out, cudaStream_t s);

int64_t spin_limit_of(int64_t v) { return v > 0 ? v : DEFAULT_SPIN_LIMIT; }

maglev_status run_mem_project(const maglev_swa_desc* d, const void* m, const void* wk,
                              const void* wv, void* Rk, void* Rv, cudaStream_t st) {
  const int64_t M = (int64_t)d->B * d->T, D = (int64_t)d->H * d->hd, K = d->d_mem;
  if (d->dtype == MAGLEV_BF16 && K % 8 == 0 && D % 256 == 0) {
    int* err = nullptr;
    maglev_status s = status_word(&err, st);
    if (s != MAGLEV_OK) return s;
    MAGLEV_LAUNCH(1, st, launch_proj_fwd_tc(M, (int)D, (int)K, m, wk, wv, Rk, Rv,
                                            spin_limit_of(d->spin_limit), err, st),
                  "mem_project_tc");
    return MAGLEV_OK;
  }
  for (int which = 0; which < 2; ++which) {
    GemmArgs g{};
    g.M = M;
    g.N = D;
    g.K1 = K;
    g.K2 = 0;
    g.A1 = m;
    g.sa1m = K;
    g.sa1k = 1;
    g.B1 = which ? wv : wk;  // B(k, n) = W[n, k]
    g.sb1k = 1;
    g.sb1n = K;
    g.C = which ? Rv : Rk;
    g.scm = D;
    g.scn = 1;
    g.accumulate = 0;
    g.dtype = d->dtype;
    MAGLEV_LAUNCH(1, st, launch_gemm_simt(g, st), "mem_project_gemm");
  }
  return MAGLEV_OK;
}

maglev_status run_mem_project_bwd(const maglev_swa_desc* d, const void* m, const void* wk,
                                  const void* wv, const void* dRk, const void* dRv, void* dm,
                                  void* dwk, void* dwv, cudaStream_t st) {
  const int64_t M = (int64_t)d->B * d->T, D = (int64_t)d->H * d->hd, K = d->d_mem;
  int* err = nullptr;
  maglev_status stw = status_word(&err, st);
  if (stw != MAGLEV_OK) return stw;
  const bool tc = d->dtype == MAGLEV_BF16 && K % 8 == 0;
  if (dm && dwk && dwv && tc && proj_bwd_grouped_available(M, (int)D, (int)K)) {
    MAGLEV_LAUNCH(1, st, launch_proj_bwd_grouped_pair(M, (int)D, (int)K, dRk, dRv, wk, wv, m, dm, dwk, dwv,
                                                      spin_limit_of(d->spin_limit), err, st),
                  "mem_project_bwd_tc");
    dm = nullptr;
    dwk = dwv = nullptr;
  }
  if (dm && tc && D % 64 == 0) {
    MAGLEV_LAUNCH(1, st, launch_proj_bwd_dm_tc(M, (int)D, (int)K, dRk, dRv, wk, wv, dm,
                                               spin_limit_of(d->spin_limit), err, st),
                  "mem_project_bwd_dm_tc");
    dm = nullptr;
  }
  if (dwk && dwv && tc && D % 128 == 0) {
    MAGLEV_LAUNCH(1, st, launch_proj_bwd_dw_tc(M, (int)D, (int)K, dRk, dRv, m, dwk, dwv,
                                               spin_limit_of(d->spin_limit), err, st),
                  "mem_project_bwd_dw_tc");
    dwk = dwv = nullptr;
  }
  if (dm) {  // dm[M, K] = dRk[M, D] W_mk[D, K] + dRv W_mv
    GemmArgs g{};
    g.M = M;
    g.N = K;
    g.K1 = D;
    g.K2 = D;
    g.A1 = dRk;
    g.sa1m = D;
    g.sa1k = 1;
    g.B1 = wk;
    g.sb1k = K;
    g.sb1n = 1;
    g.A2 = dRv;
    g.sa2m = D;
    g.sa2k = 1;
    g.B2 = wv;
    g.sb2k = K;
    g.sb2n = 1;
    g.C = dm;
    g.scm = K;
    g.scn = 1;
    g.dtype = d->dtype;
    MAGLEV_LAUNCH(1, st, launch_gemm_simt(g, st), "mem_project_bwd_dm_gemm");
  }
  for (int which = 0; which < 2; ++which) {  // dW[D, K] = dR^T[D, M] m[M, K]
    void* out = which ? dwv : dwk;
    if (!out) continue;
    GemmArgs g{};
    g.M = D;
    g.N = K;
    g.K1 = M;
    g.K2 = 0;
    g.A1 = which ? dRv : dRk;
    g.sa1m = 1;
    g.sa1k = D;
    g.B1 = m;
    g.sb1k = K;
    g.sb1n = 1;
    g.C = out;
    g.scm = K;
    g.scn = 1;
    g.dtype = d->dtype;
    MAGLEV_LAUNCH(1, st, launch_gemm_simt(g, st), "mem_project_bwd_dw_gemm");
  }
  return MAGLEV_OK;
}

// Device status word, one per device that loads the library.
__device__ int g_device_status_word;

std::mutex g_status_mu;
int* g_status_ptr[128];

// Device address of the status word on the current device: looked up on the
// first call and again on every call whose stream is not being captured (a
// device reset reloads the module, possibly at another address); calls made
// during stream capture use the address cached by an earlier call.
maglev_status status_word(int** out, cudaStream_t s) {
  int dev = 0;
  MAGLEV_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= 128) return fail(MAGLEV_ERR_UNSUPPORTED, "device index %d", dev);
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  const bool capturing = cudaStreamIsCapturing(s, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone;
  std::lock_guard<std::mutex> lock(g_status_mu);
  if (!capturing || !g_status_ptr[dev]) {
    if (capturing)
      return fail(MAGLEV_ERR_CUDA, "the first call of this library on a device must come before any stream capture");
    void* p = nullptr;
    MAGLEV_CUDA(cudaGetSymbolAddress(&p, g_device_status_word), "cudaGetSymbolAddress");
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  *out = g_status_ptr[dev];
  return MAGLEV_OK;
}

}  // namespace

namespace maglev {
void set_last_error(const char* msg) { g_last_error = msg; }
}  // namespace maglev

extern "C" {

const char* maglev_version(void) { return "maglev-b200 0.1.0 (sm_100a)"; }

long long maglev_launch_count(void) { return g_launches.load(); }

void maglev_profile_enable(int on) { g_prof_on.store(on ? 1 : 0); }

size_t maglev_profile_report(char* buf, size_t n) {
  std::vector<ProfRec> recs;
  std::lock_guard<std::mutex> lock(g_prof_mu);
  recs.swap(g_prof);
  for (const ProfRec& r : recs) {  // resolve finished records into the pending text
    float ms = -1.0f;
    if (cudaEventSynchronize(r.b) == cudaSuccess) cudaEventElapsedTime(&ms, r.a, r.b);
    char line[160];
    snprintf(line, sizeof(line), "%s %d %.6f\n", r.name, r.kernels, ms);
    g_prof_text += line;
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  const size_t len = g_prof_text.size();
  if (buf && n) {  // hand the text over and clear it
    size_t k = len < n - 1 ? len : n - 1;
    memcpy(buf, g_prof_text.data(), k);
    buf[k] = '\0';
    g_prof_text.clear();
  }
  return len;
}

size_t maglev_last_error(char* buf, size_t n) {
  if (buf && n) {
    size_t k = g_last_error.size() < n - 1 ? g_last_error.size() : n - 1;
    memcpy(buf, g_last_error.data(), k);
    buf[k] = '\0';
  }
  return g_last_error.size();
}

maglev_status maglev_device_status(void* stream, int* code) {
  if (!code) return fail(MAGLEV_ERR_INVALID_ARG, "code must not be NULL");
  int* w = nullptr;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  maglev_status st = status_word(&w, s);
  if (st != MAGLEV_OK) return st;
  int host = 0;
  MAGLEV_CUDA(cudaMemcpyAsync(&host, w, sizeof(int), cudaMemcpyDeviceToHost, s), "read status");
  MAGLEV_CUDA(cudaMemsetAsync(w, 0, sizeof(int), s), "clear status");
  MAGLEV_CUDA(cudaStreamSynchronize(s), "status sync");
  *code = host;
  return MAGLEV_OK;
}

size_t maglev_swa_saved_bytes(const maglev_swa_desc* d) {
  if (check_swa(d) != MAGLEV_OK) return 0;
  return saved_layout(d).total;
}

size_t maglev_swa_bwd_workspace_bytes(const maglev_swa_desc* d) {
  if (check_swa(d) != MAGLEV_OK) return 0;
  return bwd_layout(d).total;
}

size_t maglev_consistency_workspace_bytes(int64_t rows, int d) {
  if (rows < 0 || d < 1) return 0;
  return align256((size_t)loss_partial_blocks(rows * (int64_t)d) * sizeof(float));
}

maglev_status maglev_mem_project(const maglev_swa_desc* d, const void* m_shift, const void* w_mk,
                                 const void* w_mv, void* R_k, void* R_v, void* stream) {
  maglev_status st = check_swa(d);
  if (st != MAGLEV_OK) return st;
  if (d->d_mem < 1) return fail(MAGLEV_ERR_INVALID_ARG, "d_mem must be >= 1");
  NEED_PTR(m_shift);
  NEED_PTR(w_mk);
  NEED_PTR(w_mv);
  NEED_PTR(R_k);
  NEED_PTR(R_v);
  if (d->B == 0 || d->T == 0) return MAGLEV_OK;
  return run_mem_project(d, m_shift, w_mk, w_mv, R_k, R_v, static_cast<cudaStream_t>(stream));
}

maglev_status maglev_inject_swa_fwd(const maglev_swa_desc* d, const void* q, const void* k,
                                    const void* v, const void* m_shift, const void* w_mk,
                                    const void* w_mv, void* R_k, void* R_v,
                                    const float* gate_logits, void* out, float* lse, void* saved,
                                    void* stream) {
  maglev_status st = check_swa(d);
  if (st != MAGLEV_OK) return st;
  NEED_PTR(q);
  NEED_PTR(k);
  NEED_PTR(v);
  NEED_PTR(out);
  NEED_PTR(lse);
  NEED_PTR(saved);
  if (d->inject) {
    NEED_PTR(R_k);
    NEED_PTR(R_v);
    NEED_PTR(gate_logits);
    if (m_shift) {
      NEED_PTR(m_shift);
      NEED_PTR(w_mk);
      NEED_PTR(w_mv);
    }
  }
  if (d->B == 0 || d->T == 0) return MAGLEV_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const SwaShape sh = shape_of(d);
  const SavedLayout L = saved_layout(d);
  if (d->inject && m_shift) {
    st = run_mem_project(d, m_shift, w_mk, w_mv, R_k, R_v, s);
    if (st != MAGLEV_OK) return st;
  }
  MAGLEV_LAUNCH(1, s, launch_prep(sh, q, k, v, R_k, R_v, gate_logits, at<char>(saved, L.q),
                                   at<char>(saved, L.k), at<char>(saved, L.v), s),
                "inject_prep");
  if (d->dtype == MAGLEV_BF16) {
    int* err = nullptr;
    st = status_word(&err, s);
    if (st != MAGLEV_OK) return st;
    MAGLEV_LAUNCH(1, s, launch_attn_fwd_tc(sh, at<char>(saved, L.q), at<char>(saved, L.k),
                                            at<char>(saved, L.v), out, lse, spin_limit_of(d->spin_limit),
                                            err, s),
                  "attn_fwd_tc");
  } else {
    MAGLEV_LAUNCH(1, s, launch_attn_fwd_simt(sh, at<char>(saved, L.q), at<char>(saved, L.k),
                                              at<char>(saved, L.v), out, lse, s),
                  "attn_fwd");
  }
  return MAGLEV_OK;
}

maglev_status maglev_inject_swa_bwd(const maglev_swa_desc* d, const void* k, const void* v,
                                    const void* R_k, const void* R_v, const float* gate_logits,
                                    const void* out, const float* lse, const void* saved,
                                    const void* dout, void* dq, void* dk, void* dv, void* dR_k,
                                    void* dR_v, float* dR_acc_k, float* dR_acc_v, int dR_mode,
                                    float* dgate_logits, const void* m_shift, const void* w_mk,
                                    const void* w_mv, void* dm_shift, void* dw_mk, void* dw_mv,
                                    void* workspace, void* stream) {
  maglev_status st = check_swa(d);
  if (st != MAGLEV_OK) return st;
  NEED_PTR(k);
  NEED_PTR(v);
  NEED_PTR(out);
  NEED_PTR(lse);
  NEED_PTR(saved);
  NEED_PTR(dout);
  NEED_PTR(dq);
  NEED_PTR(dk);
  NEED_PTR(dv);
  NEED_PTR(workspace);
  // Delta and the zeroed dQ accumulator already in the workspace
  // (maglev_consistency_loss_prepare_bwd on this out and dout)
  const bool prepared = (dR_mode & MAGLEV_BWD_PREPARED) != 0;
  dR_mode &= ~MAGLEV_BWD_PREPARED;
  if (dR_mode < MAGLEV_DR_WRITE || dR_mode > MAGLEV_DR_LAST)
    return fail(MAGLEV_ERR_INVALID_ARG, "dR_mode %d is not a maglev_dr_mode", dR_mode);
  if (!d->inject) dR_mode = MAGLEV_DR_WRITE;
  const bool dr_out = dR_mode == MAGLEV_DR_WRITE || dR_mode == MAGLEV_DR_LAST;
  if (d->inject) {
    NEED_PTR(R_k);
    NEED_PTR(R_v);
    NEED_PTR(gate_logits);
    NEED_PTR(dgate_logits);
    if (dr_out) {
      NEED_PTR(dR_k);
      NEED_PTR(dR_v);
    }
    if (dR_mode != MAGLEV_DR_WRITE) {
      NEED_PTR(dR_acc_k);
      NEED_PTR(dR_acc_v);
    }
    if (m_shift && !dr_out)
      return fail(MAGLEV_ERR_INVALID_ARG,
                  "m_shift given in dR_mode %d: the projection backward needs the finished dR (WRITE or LAST)",
                  dR_mode);
    if (m_shift) {
      NEED_PTR(m_shift);
      NEED_PTR(w_mk);
      NEED_PTR(w_mv);
      OPT_PTR(dm_shift);
      OPT_PTR(dw_mk);
      OPT_PTR(dw_mv);
    }
  }
  if (d->B == 0 || d->T == 0) return MAGLEV_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const SwaShape sh = shape_of(d);
  const SavedLayout L = saved_layout(d);
  const BwdLayout Wk = bwd_layout(d);
  const void* qr = at<char>(saved, L.q);
  const void* kb = at<char>(saved, L.k);
  const void* vb = at<char>(saved, L.v);
  float* delta = at<float>(workspace, Wk.delta);
  void* dkb = at<char>(workspace, Wk.dkb);
  void* dvb = at<char>(workspace, Wk.dvb);
  float* gpart = at<float>(workspace, Wk.gpart);
  float* dq_acc = d->dtype == MAGLEV_BF16 ? at<float>(workspace, Wk.dq_acc) : nullptr;
  if (!prepared) MAGLEV_LAUNCH(1, s, launch_attn_delta(sh, out, dout, delta, dq_acc, s), "attn_delta");
  if (d->dtype == MAGLEV_BF16) {
    int* err = nullptr;
    st = status_word(&err, s);
    if (st != MAGLEV_OK) return st;
    MAGLEV_LAUNCH(1, s, launch_attn_bwd_tc(sh, qr, kb, vb, dout, lse, delta, dq_acc, dkb, dvb,
                                           spin_limit_of(d->spin_limit), err, s),
                  "attn_bwd_tc");
  } else {
    MAGLEV_LAUNCH(1, s, launch_attn_bwd_dq_simt(sh, qr, kb, vb, dout, lse, delta, dq, s), "attn_bwd_dq");
    MAGLEV_LAUNCH(1, s, launch_attn_bwd_dkdv_simt(sh, qr, kb, vb, dout, lse, delta, dkb, dvb, s),
                  "attn_bwd_dkdv");
  }
  MAGLEV_LAUNCH(1, s, launch_unmix(sh, dkb, dvb, k, v, R_k, R_v, gate_logits, dk, dv, dR_k, dR_v,
                                   dR_acc_k, dR_acc_v, dR_mode, gpart, dq_acc, dq, s),
                "unmix");
  if (d->inject) {
    MAGLEV_LAUNCH(1, s, launch_gate_reduce((int64_t)d->B * d->T, d->H, d->shared_kv_gates ? 1 : 0, gpart,
                                           gate_logits, dgate_logits, s),
                  "gate_reduce");
    if (m_shift) {
      st = run_mem_project_bwd(d, m_shift, w_mk, w_mv, dR_k, dR_v, dm_shift, dw_mk, dw_mv, s);
      if (st != MAGLEV_OK) return st;
    }
  }
  return MAGLEV_OK;
}

maglev_status maglev_mem_project_bwd(const maglev_swa_desc* d, const void* m_shift,
                                     const void* w_mk, const void* w_mv, const void* dR_k,
                                     const void* dR_v, void* dm_shift, void* dw_mk, void* dw_mv,
                                     void* stream) {
  maglev_status st = check_swa(d);
  if (st != MAGLEV_OK) return st;
  if (d->d_mem < 1) return fail(MAGLEV_ERR_INVALID_ARG, "d_mem must be >= 1");
  NEED_PTR(m_shift);
  NEED_PTR(w_mk);
  NEED_PTR(w_mv);
  NEED_PTR(dR_k);
  NEED_PTR(dR_v);
  OPT_PTR(dm_shift);
  OPT_PTR(dw_mk);
  OPT_PTR(dw_mv);
  if (d->B == 0 || d->T == 0) return MAGLEV_OK;
  return run_mem_project_bwd(d, m_shift, w_mk, w_mv, dR_k, dR_v, dm_shift, dw_mk, dw_mv,
                             static_cast<cudaStream_t>(stream));
}

maglev_status maglev_mem_project_bwd_layers(const maglev_swa_desc* d, int n_layers, const void* m_shift,
                                            const void* w_mk, const void* w_mv, const void* dR_k,
                                            const void* dR_v, void* dm_shift, void* dw_mk, void* dw_mv,
                                            void* stream) {
  maglev_status st = check_swa(d);
  if (st != MAGLEV_OK) return st;
  if (d->d_mem < 1) return fail(MAGLEV_ERR_INVALID_ARG, "d_mem must be >= 1");
  if (n_layers < 1) return fail(MAGLEV_ERR_INVALID_ARG, "n_layers must be >= 1");
  NEED_PTR(m_shift);
  NEED_PTR(w_mk);
  NEED_PTR(w_mv);
  NEED_PTR(dR_k);
  NEED_PTR(dR_v);
  OPT_PTR(dm_shift);
  OPT_PTR(dw_mk);
  OPT_PTR(dw_mv);
  if ((dw_mk == nullptr) != (dw_mv == nullptr))
    return fail(MAGLEV_ERR_INVALID_ARG, "dw_mk and dw_mv must both be given or both be NULL");
  const int64_t M = (int64_t)d->B * d->T, D = (int64_t)d->H * d->hd, K = d->d_mem;
  const bool tc = d->dtype == MAGLEV_BF16;
  if (tc && (K % 8 != 0 || D % 128 != 0))
    return fail(MAGLEV_ERR_UNSUPPORTED, "bf16 per-layer projection needs d_mem %% 8 == 0 and H*hd %% 128 == 0");
  if (M == 0) return MAGLEV_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t e = elt(d->dtype);
  const size_t w_layer = (size_t)D * K * e, r_layer = (size_t)M * D * e;
  int* err = nullptr;
  st = status_word(&err, s);
  if (st != MAGLEV_OK) return st;
  if (dm_shift) {
    if (tc) {
      MAGLEV_LAUNCH(1, s, launch_proj_bwd_dm_layers_tc(M, (int)D, (int)K, n_layers, dR_k, dR_v, w_mk, w_mv,
                                                       dm_shift, spin_limit_of(d->spin_limit), err, s),
                    "mem_project_bwd_dm_layers_tc");
    } else {  // fp32: accumulate the layers' products in the fp32 output
      for (int l = 0; l < n_layers; ++l) {
        GemmArgs g{};
        g.M = M;
        g.N = K;
        g.K1 = D;
        g.K2 = D;
        g.A1 = at<char>(dR_k, l * r_layer);
        g.sa1m = D;
        g.sa1k = 1;
        g.B1 = at<char>(w_mk, l * w_layer);
        g.sb1k = K;
        g.sb1n = 1;
        g.A2 = at<char>(dR_v, l * r_layer);
        g.sa2m = D;
        g.sa2k = 1;
        g.B2 = at<char>(w_mv, l * w_layer);
        g.sb2k = K;
        g.sb2n = 1;
        g.C = dm_shift;
        g.scm = K;
        g.scn = 1;
        g.accumulate = l > 0;
        g.dtype = d->dtype;
        MAGLEV_LAUNCH(1, s, launch_gemm_simt(g, s), "mem_project_bwd_dm_gemm");
      }
    }
  }
  if (dw_mk) {
    for (int l = 0; l < n_layers; ++l) {
      st = run_mem_project_bwd(d, m_shift, at<char>(w_mk, l * w_layer), at<char>(w_mv, l * w_layer),
                               at<char>(dR_k, l * r_layer), at<char>(dR_v, l * r_layer), nullptr,
                               at<char>(dw_mk, l * w_layer), at<char>(dw_mv, l * w_layer), s);
      if (st != MAGLEV_OK) return st;
    }
  }
  return MAGLEV_OK;
}

maglev_status maglev_consistency_loss(const void* m, const void* m_target, int64_t rows, int d,
                                      int dtype, float lambda, float inv_count, float* loss,
                                      void* dm, void* dm_target, int accumulate_dm,
                                      void* workspace, void* stream) {
  if (rows < 0) return fail(MAGLEV_ERR_INVALID_ARG, "rows must be >= 0");
  if (d < 1) return fail(MAGLEV_ERR_INVALID_ARG, "d must be >= 1");
  if (dtype != MAGLEV_F32 && dtype != MAGLEV_BF16)
    return fail(MAGLEV_ERR_INVALID_ARG, "dtype must be MAGLEV_F32 or MAGLEV_BF16");
  if (!std::isfinite(lambda) || !std::isfinite(inv_count) || inv_count < 0)
    return fail(MAGLEV_ERR_INVALID_ARG, "lambda and inv_count must be finite, inv_count >= 0");
  NEED_PTR(loss);
  OPT_PTR(dm);
  OPT_PTR(dm_target);
  if (rows == 0) return MAGLEV_OK;
  NEED_PTR(m);
  NEED_PTR(m_target);
  NEED_PTR(workspace);
  const double ic = inv_count == 0.0f ? 1.0 / (double)rows : (double)inv_count;
  const double sl = (double)lambda * ic / std::sqrt((double)d);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MAGLEV_LAUNCH(2, s, launch_consistency_loss(m, m_target, rows, d, dtype, (float)sl, (float)(2.0 * sl),
                                               loss, dm, dm_target, accumulate_dm ? 1 : 0,
                                               static_cast<float*>(workspace), s),
                "consistency_loss");
  return MAGLEV_OK;
}

maglev_status maglev_consistency_loss_prepare_bwd(const maglev_swa_desc* d, const void* out,
                                                  const void* m_target, float lambda, float inv_count,
                                                  float* loss, void* dout, void* bwd_workspace,
                                                  void* loss_workspace, void* stream) {
  maglev_status st = check_swa(d);
  if (st != MAGLEV_OK) return st;
  if (!std::isfinite(lambda) || !std::isfinite(inv_count) || inv_count < 0)
    return fail(MAGLEV_ERR_INVALID_ARG, "lambda and inv_count must be finite, inv_count >= 0");
  NEED_PTR(loss);
  if (d->B == 0 || d->T == 0) return MAGLEV_OK;
  NEED_PTR(out);
  NEED_PTR(m_target);
  NEED_PTR(dout);
  NEED_PTR(bwd_workspace);
  NEED_PTR(loss_workspace);
  const int64_t rows = (int64_t)d->B * d->T;
  const int D = d->H * d->hd;
  const double ic = inv_count == 0.0f ? 1.0 / (double)rows : (double)inv_count;
  const double sl = (double)lambda * ic / std::sqrt((double)D);
  const BwdLayout Wk = bwd_layout(d);
  float* delta = at<float>(bwd_workspace, Wk.delta);
  float* dq_acc = d->dtype == MAGLEV_BF16 ? at<float>(bwd_workspace, Wk.dq_acc) : nullptr;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MAGLEV_LAUNCH(2, s, launch_consistency_loss_prep(out, m_target, rows, d->H, d->hd, d->T, d->dtype, (float)sl,
                                                   (float)(2.0 * sl), loss, dout, delta, dq_acc,
                                                   static_cast<float*>(loss_workspace), s),
                "consistency_loss_prep");
  return MAGLEV_OK;
}

// Offsets inside the LM head's workspace.
struct LmLayout {
  size_t c, dz, part, tgt, ce, total;
};
LmLayout lm_layout(int64_t N, int V) {
  LmLayout L;
  L.c = 0;
  L.dz = align256((size_t)N * V * 4);
  L.part = L.dz + align256((size_t)N * V * 2);
  L.tgt = L.part + align256((size_t)N * lm_ce_tiles(V) * 8);
  L.ce = L.tgt + align256((size_t)N * 4);
  L.total = L.ce + align256((size_t)N * 4);
  return L;
}

size_t maglev_lm_head_workspace_bytes(int64_t N, int d, int V) {
  if (N < 0 || d < 1 || V < 1) return 0;
  return lm_layout(N, V).total;
}

maglev_status maglev_lm_head_ce(int64_t N, int d, int V, int dtype, float softcap, float inv_count,
                                const void* m, const void* U, const int64_t* targets, float* loss, float* lse,
                                void* dm, void* dU, void* workspace, int64_t spin_limit, void* stream) {
  if (N < 0 || d < 1 || V < 1) return fail(MAGLEV_ERR_INVALID_ARG, "need N >= 0, d >= 1, V >= 1");
  if (dtype != MAGLEV_BF16) return fail(MAGLEV_ERR_UNSUPPORTED, "the LM head runs in bf16 only");
  if (d % 8 != 0 || V % 8 != 0) return fail(MAGLEV_ERR_UNSUPPORTED, "d and V must be multiples of 8");
  if ((int64_t)V * N > ((int64_t)1 << 40)) return fail(MAGLEV_ERR_UNSUPPORTED, "N * V too large");
  if (!(softcap > 0.0f) || !std::isfinite(softcap)) return fail(MAGLEV_ERR_INVALID_ARG, "softcap must be > 0");
  if (!std::isfinite(inv_count) || inv_count < 0)
    return fail(MAGLEV_ERR_INVALID_ARG, "inv_count must be finite and >= 0");
  NEED_PTR(loss);
  OPT_PTR(dm);
  OPT_PTR(dU);
  if (N == 0) return MAGLEV_OK;
  NEED_PTR(m);
  NEED_PTR(U);
  NEED_PTR(targets);
  NEED_PTR(lse);
  NEED_PTR(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* err = nullptr;
  maglev_status st = status_word(&err, s);
  if (st != MAGLEV_OK) return st;
  const LmLayout L = lm_layout(N, V);
  const float ic = inv_count == 0.0f ? (float)(1.0 / (double)N) : inv_count;
  const int64_t lim = spin_limit_of(spin_limit);
  float* c = at<float>(workspace, L.c);
  void* dz = (dm || dU) ? at<char>(workspace, L.dz) : nullptr;
  float2* part = at<float2>(workspace, L.part);
  float* tgt = at<float>(workspace, L.tgt);
  float* ce = at<float>(workspace, L.ce);
  MAGLEV_LAUNCH(1, s, launch_lm_logits_ce_tc(N, d, V, softcap, m, U, targets, c, part, tgt, lim, err, s),
                "lm_logits_ce_tc");
  MAGLEV_LAUNCH(dz ? 3 : 2, s, launch_lm_ce_finish(N, V, lm_ce_tiles(V), ic, softcap, part, tgt, targets, c, lse,
                                                    ce, loss, dz, s),
                "lm_ce_finish");
  if (dm && dU && lm_bwd_grouped_available(N, d, V)) {  // both in one launch on SM pairs
    MAGLEV_LAUNCH(1, s, launch_lm_bwd_grouped_pair(N, d, V, dz, U, m, dm, dU, lim, err, s), "lm_bwd_tc");
  } else {
    if (dm) MAGLEV_LAUNCH(1, s, launch_lm_dm_tc(N, d, V, dz, U, dm, lim, err, s), "lm_dm_tc");
    if (dU) MAGLEV_LAUNCH(1, s, launch_lm_dU_tc(N, d, V, dz, m, dU, lim, err, s), "lm_dU_tc");
  }
  return MAGLEV_OK;
}

maglev_status maglev_memory_state(int B, int T, int d, float eps, int dtype, const void* o, void* m,
                                  void* m_shift, float* rstd, void* stream) {
  if (B < 0 || T < 0) return fail(MAGLEV_ERR_INVALID_ARG, "B and T must be >= 0");
  if (d < 1) return fail(MAGLEV_ERR_INVALID_ARG, "d must be >= 1");
  if (!(eps >= 0.0f) || !std::isfinite(eps)) return fail(MAGLEV_ERR_INVALID_ARG, "eps must be finite and >= 0");
  if (dtype != MAGLEV_F32 && dtype != MAGLEV_BF16)
    return fail(MAGLEV_ERR_INVALID_ARG, "dtype must be MAGLEV_F32 or MAGLEV_BF16");
  OPT_PTR(m_shift);
  if ((int64_t)B * T == 0) return MAGLEV_OK;
  NEED_PTR(o);
  NEED_PTR(m);
  NEED_PTR(rstd);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MAGLEV_LAUNCH(1, s, launch_memstate_fwd(o, m, m_shift, rstd, B, T, d, eps, dtype, s), "memory_state");
  return MAGLEV_OK;
}

maglev_status maglev_memory_state_bwd(int B, int T, int d, int dtype, const void* o, const float* rstd,
                                      const void* dm, const void* dm_shift, const void* dout_in, void* d_o,
                                      void* stream) {
  if (B < 0 || T < 0) return fail(MAGLEV_ERR_INVALID_ARG, "B and T must be >= 0");
  if (d < 1) return fail(MAGLEV_ERR_INVALID_ARG, "d must be >= 1");
  if (dtype != MAGLEV_F32 && dtype != MAGLEV_BF16)
    return fail(MAGLEV_ERR_INVALID_ARG, "dtype must be MAGLEV_F32 or MAGLEV_BF16");
  OPT_PTR(dm);
  OPT_PTR(dm_shift);
  OPT_PTR(dout_in);
  if ((int64_t)B * T == 0) return MAGLEV_OK;
  NEED_PTR(o);
  NEED_PTR(rstd);
  NEED_PTR(d_o);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MAGLEV_LAUNCH(1, s, launch_memstate_bwd(o, rstd, dm, dm_shift, dout_in, d_o, B, T, d, dtype, s),
                "memory_state_bwd");
  return MAGLEV_OK;
}

static maglev_status check_dec(const maglev_decode_desc* d) {
  if (!d) return fail(MAGLEV_ERR_INVALID_ARG, "desc must not be NULL");
  if (d->B < 0) return fail(MAGLEV_ERR_INVALID_ARG, "B must be >= 0");
  if (d->H < 1) return fail(MAGLEV_ERR_INVALID_ARG, "H must be >= 1");
  if (d->hd != 64 && d->hd != 128)
    return fail(MAGLEV_ERR_UNSUPPORTED, "head dim %d unsupported (64 or 128)", d->hd);
  if (d->window < 1 || d->window > 8192)
    return fail(MAGLEV_ERR_UNSUPPORTED, "window must be in [1, 8192]");
  if (d->dtype != MAGLEV_F32 && d->dtype != MAGLEV_BF16)
    return fail(MAGLEV_ERR_INVALID_ARG, "dtype must be MAGLEV_F32 or MAGLEV_BF16");
  if (!(d->rope_base > 1.0f) || !std::isfinite(d->rope_base))
    return fail(MAGLEV_ERR_INVALID_ARG, "rope_base must be finite and > 1");
  if (!(d->rms_eps >= 0.0f) || !std::isfinite(d->rms_eps))
    return fail(MAGLEV_ERR_INVALID_ARG, "rms_eps must be finite and >= 0");
  return MAGLEV_OK;
}

static DecShape dec_shape(const maglev_decode_desc* d) {
  DecShape s;
  s.B = d->B;
  s.H = d->H;
  s.hd = d->hd;
  s.W = d->window;
  s.inject = d->inject ? 1 : 0;
  s.dtype = d->dtype;
  s.vg = d->shared_kv_gates ? 0 : 2;
  s.log2_base = std::log2((double)d->rope_base);
  s.eps = d->rms_eps;
  return s;
}

maglev_status maglev_decode_mem_project(const maglev_decode_desc* d, const int64_t* pos,
                                        const void* m_prev, const void* w_mk, const void* w_mv,
                                        void* krec_rot, void* vrec, void* stream) {
  maglev_status st = check_dec(d);
  if (st != MAGLEV_OK) return st;
  if (d->d_mem < 1) return fail(MAGLEV_ERR_INVALID_ARG, "d_mem must be >= 1");
  NEED_PTR(pos);
  NEED_PTR(m_prev);
  NEED_PTR(w_mk);
  NEED_PTR(w_mv);
  NEED_PTR(krec_rot);
  NEED_PTR(vrec);
  if (d->B == 0) return MAGLEV_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t D = (int64_t)d->H * d->hd, K = d->d_mem;
  if (d->dtype == MAGLEV_BF16 && K % 8 == 0 && D % 256 == 0) {
    int* err = nullptr;
    st = status_word(&err, s);
    if (st != MAGLEV_OK) return st;
    MAGLEV_LAUNCH(1, s, launch_proj_fwd_tc(d->B, (int)D, (int)K, m_prev, w_mk, w_mv, krec_rot, vrec,
                                           spin_limit_of(d->spin_limit), err, s),
                  "decode_mem_project_tc");
    MAGLEV_LAUNCH(1, s, launch_rmsnorm_rope_rows(dec_shape(d), pos, krec_rot, s), "decode_krec_norm_rope");
    return MAGLEV_OK;
  }
  for (int which = 0; which < 2; ++which) {
    GemmArgs g{};
    g.M = d->B;
    g.N = D;
    g.K1 = K;
    g.A1 = m_prev;
    g.sa1m = K;
    g.sa1k = 1;
    g.B1 = which ? w_mv : w_mk;
    g.sb1k = 1;
    g.sb1n = K;
    g.C = which ? vrec : krec_rot;
    g.scm = D;
    g.scn = 1;
    g.dtype = d->dtype;
    MAGLEV_LAUNCH(1, s, launch_gemm_simt(g, s), "decode_mem_project_gemm");
  }
  MAGLEV_LAUNCH(1, s, launch_rmsnorm_rope_rows(dec_shape(d), pos, krec_rot, s), "decode_krec_norm_rope");
  return MAGLEV_OK;
}

maglev_status maglev_wait_selftest(const void* src, int bytes, int64_t spin_limit, void* stream) {
  NEED_PTR(src);
  if (bytes < 16 || bytes > 4096 || bytes % 16 != 0)
    return fail(MAGLEV_ERR_INVALID_ARG, "bytes must be a multiple of 16 in [16, 4096]");
  if (spin_limit < 1 || spin_limit > 10000000)
    return fail(MAGLEV_ERR_INVALID_ARG, "spin_limit must be in [1, 1e7] microseconds");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* err = nullptr;
  maglev_status st = status_word(&err, s);
  if (st != MAGLEV_OK) return st;
  MAGLEV_LAUNCH(1, s, launch_wait_selftest(src, bytes, spin_limit, err, s), "wait_selftest");
  return MAGLEV_OK;
}

maglev_status maglev_decode_prefill(const maglev_swa_desc* d, const void* saved, void* k_ring, void* v_ring,
                                    void* stream) {
  maglev_status st = check_swa(d);
  if (st != MAGLEV_OK) return st;
  NEED_PTR(saved);
  NEED_PTR(k_ring);
  NEED_PTR(v_ring);
  if (d->B == 0 || d->T == 0) return MAGLEV_OK;
  const SavedLayout L = saved_layout(d);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MAGLEV_LAUNCH(1, s, launch_ring_prefill(d->B, d->T, d->H, d->hd, (int)elt(d->dtype), d->window, d->pos0,
                                          at<char>(saved, L.k), at<char>(saved, L.v), k_ring, v_ring, s),
                "decode_prefill");
  return MAGLEV_OK;
}

size_t maglev_decode_workspace_bytes(const maglev_decode_desc* d) {
  if (check_dec(d) != MAGLEV_OK) return 0;
  return decode_workspace_bytes(dec_shape(d));
}

maglev_status maglev_decode_step(const maglev_decode_desc* d, const int64_t* pos, const void* q,
                                 const void* k, const void* v, const void* krec_rot,
                                 const void* vrec, const float* gate_logits, void* k_ring,
                                 void* v_ring, void* out, void* workspace, void* stream) {
  maglev_status st = check_dec(d);
  if (st != MAGLEV_OK) return st;
  if (decode_workspace_bytes(dec_shape(d)) > 0) NEED_PTR(workspace);
  NEED_PTR(pos);
  NEED_PTR(q);
  NEED_PTR(k);
  NEED_PTR(v);
  NEED_PTR(k_ring);
  NEED_PTR(v_ring);
  NEED_PTR(out);
  if (d->inject) {
    NEED_PTR(krec_rot);
    NEED_PTR(vrec);
    NEED_PTR(gate_logits);
  }
  if (d->B == 0) return MAGLEV_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* err = nullptr;
  st = status_word(&err, s);
  if (st != MAGLEV_OK) return st;
  MAGLEV_LAUNCH(1, s, launch_decode_step(dec_shape(d), pos, q, k, v, krec_rot, vrec, gate_logits, k_ring,
                                          v_ring, out, workspace, spin_limit_of(d->spin_limit), err, s),
                "decode_step");
  return MAGLEV_OK;
}

}  // extern "C"
