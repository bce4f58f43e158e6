// selftest.cu -- a check of the bounded device wait that every kernel of the
// library relies on.
//
// Each mbarrier wait in the attention kernels gives up after a time limit,
// sets PA_ERRBIT_TIMEOUT in the call's error word and leaves its role, so that
// a pipeline whose producer never delivers ends the launch instead of hanging
// the GPU.  In correct operation no wait ever runs out, so nothing in a normal
// call exercises that exit.  pa_selftest_wait_timeout launches one warp whose
// lane 0 waits, through the same bounded-wait routine, on an mbarrier that
// nothing arrives at, with a caller-given short limit.  The wait must end by
// itself, report the timeout bit and leave the context usable.
#include "internal.h"
#include "ptx.cuh"

namespace pa {

namespace {

constexpr uint32_t kSelftestMaxLimitUs = 100000;  // 100 ms

__global__ void wait_timeout_kernel(uint64_t limit_ns, int32_t* err_word,
                                    unsigned long long* waited_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival expected; none ever comes
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x != 0) return;
  const uint64_t t0 = global_timer_ns();
  const bool completed = mbar_wait_bounded(&bar, 0, limit_ns);
  const uint64_t t1 = global_timer_ns();
  if (!completed && err_word) atomicOr(err_word, PA_ERRBIT_TIMEOUT);
  if (waited_ns) *waited_ns = static_cast<unsigned long long>(t1 - t0);
}

}  // namespace

}  // namespace pa

extern "C" pa_status pa_selftest_wait_timeout(uint32_t limit_us, int32_t* err_word,
                                              unsigned long long* waited_ns, void* stream) {
  if (limit_us == 0 || limit_us > pa::kSelftestMaxLimitUs || !err_word) return PA_ERR_INVALID_ARG;
  pa::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(limit_us) * 1000ull, err_word, waited_ns);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
