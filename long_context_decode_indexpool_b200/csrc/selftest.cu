// Self-test of the failure path shared by every tcgen05 kernel of the
// library: bounded mbarrier waits that give up, the abort flag that stops
// the CTA's other roles, and the drain of a bulk copy already in flight
// before the CTA exits.  The pages have nothing to do with it; it exists so
// that a test can make a wait run out on purpose (barriers that nothing will
// ever complete) and check what the host reads back, without a fault, a trap
// or a hang: every wait here is bounded.
#include "spx_device.cuh"
#include "spx_internal.h"

namespace spx {

namespace {

constexpr int kCopyBytes = 1024;
__device__ __align__(16) uint8_t g_selftest_src[kCopyBytes];

// One CTA of two warps.  Lane 0 of warp 0 plays a producer: it starts a
// 1 KiB bulk copy into shared memory, then waits on a barrier that never
// completes (limit_ns), gives up, and drains the copy before it leaves.
// Lane 0 of warp 1 plays a consumer waiting on another barrier that never
// completes, with a limit 1000 times longer: it must give up as soon as the
// producer's abort flag is set.
//   res[0] producer's wait result (0: gave up)   res[1] consumer's (0: gave up)
//   res[2] the drained copy landed (1)            res[3], res[4] ns each waited
//   res[5] the copy's bytes equal the source (1)
__global__ void __launch_bounds__(64, 1) k_wait_selftest(uint64_t limit_ns, int64_t* res) {
  __shared__ __align__(16) uint8_t buf[kCopyBytes];
  __shared__ __align__(8) uint64_t bars[3];  // never (producer), never (consumer), copy
  __shared__ int abort_flag;
  __shared__ int copy_ok;
  const int tid = threadIdx.x;
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_init(&bars[2], 1);
    abort_flag = 0;
    copy_ok = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < kCopyBytes; i += 64) g_selftest_src[i] = static_cast<uint8_t>(i * 7 + 3);
  __threadfence();
  __syncthreads();
  volatile int* abort = &abort_flag;
  if (tid == 0) {
    mbar_arrive_expect_tx(&bars[2], kCopyBytes);
    asm volatile("fence.proxy.async.global;" ::: "memory");
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(buf)),
        "l"(g_selftest_src), "r"(kCopyBytes), "r"(smem_u32(&bars[2]))
        : "memory");
    const uint64_t t0 = globaltimer_ns();
    const bool ok = mbar_wait(&bars[0], 0, abort, limit_ns);
    res[3] = static_cast<int64_t>(globaltimer_ns() - t0);
    res[0] = ok ? 1 : 0;
    // drain: the copy issued above must land before the CTA exits
    volatile int no_abort = 0;
    copy_ok = mbar_wait(&bars[2], 0, &no_abort, limit_ns) ? 1 : 0;
    res[2] = copy_ok;
  } else if (tid == 32) {
    const uint64_t t0 = globaltimer_ns();
    const bool ok = mbar_wait(&bars[1], 0, abort, limit_ns * 1000ull);
    res[4] = static_cast<int64_t>(globaltimer_ns() - t0);
    res[1] = ok ? 1 : 0;
  }
  __syncthreads();
  if (tid == 0) {
    int same = copy_ok;
    for (int i = 0; i < kCopyBytes && same; ++i) same = buf[i] == static_cast<uint8_t>(i * 7 + 3);
    res[5] = same;
  }
}

}  // namespace

cudaError_t launch_wait_selftest(uint64_t limit_ns, int64_t* res, cudaStream_t stream) {
  k_wait_selftest<<<1, 64, 0, stream>>>(limit_ns, res);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace spx
