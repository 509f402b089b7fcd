// Self-test of the bounded device-side waits that every TMA / tcgen05 kernel
// of the library relies on.  One CTA plays two roles of such a kernel:
//
//  * the "waiting" role starts a bulk copy into shared memory (as a
//    producer has copies in flight), then waits on an mbarrier that nothing
//    ever completes, with the caller's time limit.  The wait runs out,
//    records MOE_ERR_TIMEOUT in the device status word and raises the CTA's
//    abort flag; the role then waits (bounded) for its own copy to land;
//  * the "other" role waits on the same barrier with a limit 100x longer,
//    sees the abort flag and stops early; it then drains the tensor core
//    (a commit that arrives once every tcgen05 op of the thread is done)
//    before the CTA releases its tensor memory.
//
// So a launch exercises the time limit, the status word, the abort flag
// seen by another role, the drain of an in-flight copy and of the tensor
// core, and the release of TMEM, and then returns: nothing in it can wait
// without a bound.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kCopyBytes = 1024;
__device__ __align__(128) uint8_t g_selftest_src[kCopyBytes];  // source of the in-flight copy

__global__ void __launch_bounds__(128, 1)
    k_selftest_wait(int* status, unsigned long long limit_ns, int32_t* result) {
  __shared__ __align__(8) uint64_t never_bar, copy_bar, drain_bar;
  __shared__ __align__(128) uint8_t buf[kCopyBytes];
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;
  __shared__ int gave_up[2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&never_bar, 1);
    mbar_init(&copy_bar, 1);
    mbar_init(&drain_bar, 1);
    abort_flag = 0;
    gave_up[0] = gave_up[1] = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == 0 && lane == 0) {
    mbar_arrive_expect_tx(&copy_bar, kCopyBytes);
    bulk_load(buf, g_selftest_src, kCopyBytes, &copy_bar);
    const bool ok = mbar_wait(&never_bar, 0, &abort_flag, status, limit_ns);
    gave_up[0] = ok ? 0 : 1;
    volatile int never = 0;
    mbar_wait(&copy_bar, 0, &never, nullptr, limit_ns);  // the copy lands before the CTA exits
  } else if (warp == 1 && lane == 0) {
    const bool ok = mbar_wait(&never_bar, 0, &abort_flag, status, 100ull * limit_ns);
    gave_up[1] = ok ? 0 : 1;
    umma_commit(&drain_bar);
    volatile int never = 0;
    mbar_wait(&drain_bar, 0, &never, nullptr, limit_ns);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base_sh, 32);
  }
  if (threadIdx.x == 0) {
    result[0] = gave_up[0];
    result[1] = gave_up[1];
  }
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" int moe_selftest_bounded_wait(int limit_us, int32_t* result, void* stream) {
  MOE_REQUIRE(limit_us >= 100 && limit_us <= 1000000, MOE_ERR_UNSUPPORTED,
              "moe_selftest_bounded_wait: limit_us=%d outside [100, 1000000]", limit_us);
  MOE_REQUIRE(result != nullptr, MOE_ERR_INVALID_ARG, "moe_selftest_bounded_wait: result is null");
  int* status = device_status_ptr();
  MOE_REQUIRE(status != nullptr, MOE_ERR_CUDA, "moe_selftest_bounded_wait: no device status word");
  k_selftest_wait<<<1, 128, 0, static_cast<cudaStream_t>(stream)>>>(status, (unsigned long long)limit_us * 1000ull,
                                                                     result);
  MOE_CHECK_CUDA(cudaGetLastError());
  return MOE_OK;
}
