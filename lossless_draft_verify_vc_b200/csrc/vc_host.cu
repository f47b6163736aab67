// vc_host.cu -- host-side plumbing of the C ABI: thread-local error text,
// device properties, workspace flag readback.
#include <mutex>

#include "vc_common.cuh"

namespace vc {

static thread_local char g_err[512] = "";

vc_status set_error(vc_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

void clear_error() { g_err[0] = '\0'; }

int sm_count() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lk(mu);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

}  // namespace vc

extern "C" {

const char* vc_last_error(void) { return vc::g_err; }

int vc_abi_version(void) { return VC_ABI_VERSION; }

vc_status vc_workspace_flags(void* ws, size_t ws_bytes, uint32_t* host_flags, void* stream) {
  VC_REQUIRE(ws != nullptr && ws_bytes >= sizeof(vc::WsHeader) && host_flags != nullptr,
             "vc_workspace_flags: null workspace / output or workspace too small");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(uint32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemsetAsync(ws, 0, sizeof(uint32_t), s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
    return vc::set_error(VC_ERR_CUDA, "vc_workspace_flags: %s", cudaGetErrorString(cudaGetLastError()));
  *host_flags = v;
  vc::clear_error();
  return VC_OK;
}

}  // extern "C"
