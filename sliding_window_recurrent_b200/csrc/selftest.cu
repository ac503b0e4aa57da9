// Self-test of the bounded-wait machinery that every tensor-core kernel of
// this library uses (tc_common.cuh): an mbarrier wait that outlives its limit
// raises the CTA's abort flag and records MAGLEV_ERR_TIMEOUT in the device
// status word, copies in flight are drained, tensor memory is freed, and the
// kernel returns. Nothing here faults, traps or spins without a bound: the
// kernel starts a bulk copy into shared memory, allocates tensor memory, and
// then waits on an mbarrier that nothing completes until the limit expires.
#include "launchers.h"
#include "tc_common.cuh"

namespace maglev {
namespace {

using namespace tc;

constexpr int SELFTEST_MAX_BYTES = 4096;

__global__ void __launch_bounds__(64) wait_selftest_kernel(const void* src, uint32_t bytes, int64_t limit_ns,
                                                           int* err) {
  __shared__ __align__(128) uint8_t buf[SELFTEST_MAX_BYTES];
  __shared__ __align__(8) uint64_t bars[2];  // [0] never completed, [1] the copy's completion
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&tmem_slot, 32);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  if (warp == 0 && lane == 0) {
    const Abort ab{&abort_flag, err, limit_ns};
    mbar_arrive_expect_tx(&bars[1], bytes);
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(buf)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(&bars[1]))
        : "memory");
    mbar_wait(&bars[0], 0, ab);                   // expires: nothing arrives on bars[0]
    mbar_drain(&bars[1], 0, DRAIN_LIMIT_NS);      // the copy lands before the CTA leaves
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 32);
  }
}

}  // namespace

cudaError_t launch_wait_selftest(const void* src, int bytes, int64_t limit_us, int* err, cudaStream_t st) {
  if (bytes < 16 || bytes > SELFTEST_MAX_BYTES || bytes % 16 != 0) return cudaErrorInvalidValue;
  wait_selftest_kernel<<<1, 64, 0, st>>>(src, (uint32_t)bytes, limit_us * 1000, err);
  return cudaGetLastError();
}

}  // namespace maglev
