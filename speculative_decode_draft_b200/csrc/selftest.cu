// wmtp_selftest_wait (include/wmtp.h): runs the bounded mbarrier wait that
// every attention kernel uses, on a barrier that nothing completes, so a test
// can watch it give up on a live GPU.  Not on the attention path.

#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "ptx.cuh"
#include "wmtp.h"

static_assert(wmtp::ptx::kWaitLimitCycles == WMTP_WAIT_LIMIT_CYCLES,
              "the header's wait limit must match the kernels' bound");

namespace wmtp {
namespace {

// One thread: a shared-memory mbarrier expecting one arrival, then a wait for
// its first phase through ptx::mbar_wait, called exactly as the attention
// kernels call it.  With `arrive` set the thread completes the phase itself.
__global__ void __launch_bounds__(32) selftest_wait_kernel(int32_t arrive, int32_t* status,
                                                           long long* cycles) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = ptx::smem_addr(&bar);
  ptx::mbar_init(b, 1);
  if (arrive) ptx::mbar_arrive(b);
  const long long t0 = clock64();
  const bool done = ptx::mbar_wait(b, 0);
  const long long t1 = clock64();
  if (!done && status != nullptr) atomicOr(status, WMTP_DEV_TIMEOUT);
  if (cycles != nullptr) *cycles = t1 - t0;
}

}  // namespace
}  // namespace wmtp

extern "C" wmtp_status wmtp_selftest_wait(int32_t arrive, int32_t* status_word, int64_t* cycles_out,
                                          void* stream) {
  if (reinterpret_cast<uintptr_t>(cycles_out) % alignof(int64_t) != 0 ||
      reinterpret_cast<uintptr_t>(status_word) % alignof(int32_t) != 0)
    return WMTP_ERR_INVALID_ARG;
  // the launch's own return value decides, so an unrelated earlier error left
  // on this thread cannot be mistaken for a failure of this launch
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(32);
  cfg.stream = static_cast<cudaStream_t>(stream);
  long long* cyc = reinterpret_cast<long long*>(cycles_out);
  return cudaLaunchKernelEx(&cfg, wmtp::selftest_wait_kernel, arrive, status_word, cyc) == cudaSuccess
             ? WMTP_OK
             : WMTP_ERR_CUDA;
}
