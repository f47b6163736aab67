// vc_debug.cu -- test exports that exercise the library's failure handling
// on the device without faulting or hanging a GPU.
//
// Every on-chip wait of the hot-path kernels (bulk-copy and tensor-core
// completions on mbarriers) goes through mbar_wait_bounded: after a time
// limit it gives up, ORs VC_FLAG_WAIT_TIMEOUT into a flag word and returns
// false, and the kernel then skips the work that depended on the wait.  The
// kernel below runs that exact helper on an mbarrier no thread ever arrives
// on, with a short limit, so a test can watch the give-up path end a kernel
// normally and leave the context usable.
#include "vc_common.cuh"

namespace vc {
namespace {

__global__ void wait_timeout_kernel(uint32_t* flags, uint32_t* result, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) mbar_init(&bar, 1);  // one arrival completes phase 0; none ever comes
  fence_mbar_init();
  __syncthreads();
  const bool completed = mbar_wait_bounded(&bar, 0u, flags, limit_ns);
  if (threadIdx.x == 0) result[0] = completed ? 1u : 2u;  // 2: the wait gave up
}

}  // namespace
}  // namespace vc

extern "C" {

vc_status vc_debug_wait_timeout(uint32_t* flags, uint32_t* result, int64_t limit_ns, void* stream) {
  VC_REQUIRE(flags && result, "vc_debug_wait_timeout: null flags or result");
  VC_REQUIRE(limit_ns >= 1000 && limit_ns <= 100000000,
             "vc_debug_wait_timeout: limit must be 1 us .. 100 ms (got %lld ns)", static_cast<long long>(limit_ns));
  vc::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(flags, result,
                                                                          static_cast<uint64_t>(limit_ns));
  return vc::launch_status("vc_debug_wait_timeout");
}

}  // extern "C"
