// Ring prefill from a prompt: after the training-form forward over a prompt,
// the mixed entries (k_bar, v_bar) of its last min(T, W) positions are copied
// into the rolling decode rings, the entry of absolute position j into slot
// j mod W, so that recurrent decoding continues at the position after the
// prompt ("Maglev: Sliding Recurrent Memory", paper.rainbus.top, 研究动机: at
// inference m_t = P(x_{t-W+1:t}, M_{t-1}) over a fixed window; 前置知识: the
// cache is that of plain SWA, the memory riding in the existing entries).
//
// A pure gather/scatter of 16-byte vectors: one thread per vector of one
// entry, consecutive threads walk an entry's channels, so both the reads of
// [B,T,H,hd] and the writes of [B,H,W,hd] are whole 16-byte pieces of
// contiguous rows.
#include "common.cuh"
#include "launchers.h"

namespace maglev {
namespace {

__global__ void __launch_bounds__(256) ring_prefill_kernel(int B, int T, int H, int vpe, int64_t W, int64_t pos0,
                                                           int t0, const uint4* __restrict__ kb,
                                                           const uint4* __restrict__ vb, uint4* __restrict__ kr,
                                                           uint4* __restrict__ vr) {
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int nt = T - t0;  // entries per (b, h)
  const int64_t n = (int64_t)B * nt * H * vpe;
  if (gid >= n) return;
  const int c = (int)(gid % vpe);
  const int64_t e = gid / vpe;  // entry (b, t - t0, h), h fastest: reads walk [B,T,H,hd] in order
  const int h = (int)(e % H);
  const int64_t bt = e / H;
  const int t = t0 + (int)(bt % nt);
  const int b = (int)(bt / nt);
  const int64_t src = (((int64_t)b * T + t) * H + h) * vpe + c;
  const int64_t slot = (pos0 + t) % W;
  const int64_t dst = (((int64_t)b * H + h) * W + slot) * vpe + c;
  kr[dst] = kb[src];
  vr[dst] = vb[src];
}

}  // namespace

cudaError_t launch_ring_prefill(int B, int T, int H, int hd, int elt_bytes, int64_t W, int64_t pos0,
                                const void* k_bar, const void* v_bar, void* k_ring, void* v_ring,
                                cudaStream_t st) {
  const int t0 = T > W ? (int)(T - W) : 0;
  const int vpe = hd * elt_bytes / 16;
  const int64_t n = (int64_t)B * (T - t0) * H * vpe;
  if (n == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((n + 255) / 256);
  ring_prefill_kernel<<<blocks, 256, 0, st>>>(B, T, H, vpe, W, pos0, t0, static_cast<const uint4*>(k_bar),
                                              static_cast<const uint4*>(v_bar), static_cast<uint4*>(k_ring),
                                              static_cast<uint4*>(v_ring));
  return cudaGetLastError();
}

}  // namespace maglev
