// vc_link.cu -- bandwidth-limited host -> device links.
//
// In remote prefix caching the compressed cache reaches the serving GPU over
// a slow network while the full cache comes over a fast local link; the
// pages' setup splits them as 1.2 GB/s remote against 40 GB/s local
// ("VeriCache: Turning Lossy KV Cache into Lossless LLM Inference",
// menfem.com, "Key Contributions" (two deployment pipelines) and
// "Methodology"; devshah.ca page "VeriCache: making lossy KV compression
// exact", section "Verifying Without Giving Back the Speedup").  One GPU machine
// has only its PCIe bus, so a link of a lower rate is emulated on it: the
// bytes really cross the bus, chunk by chunk, and a chunk is released no
// sooner than chunk_bytes / rate after the previous one started.  The wait
// is a one-thread kernel that sleeps on the device clock (bounded), so the
// pacing needs no host thread and the stream keeps CUDA ordering with the
// work that consumes the data.
#include "vc_link.h"

namespace vc {
namespace {

__global__ void link_stamp_kernel(uint64_t* clock) { clock[0] = global_timer_ns(); }

// Sleeps until clock[0] + wait_ns; gives up (flag) after max_wait_ns.
__global__ void link_pace_kernel(const uint64_t* clock, uint64_t wait_ns, uint64_t max_wait_ns, uint32_t* flags) {
  const uint64_t release = clock[0] + wait_ns;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    const uint64_t now = global_timer_ns();
    if (now >= release) return;
    if (now - t0 > max_wait_ns) {
      atomicOr(flags, VC_FLAG_WAIT_TIMEOUT);
      return;
    }
    const uint64_t left = release - now;
    __nanosleep(static_cast<unsigned>(left > 100000 ? 100000 : left));
  }
}

}  // namespace

vc_status PacedLink::init(cudaStream_t s, double gbps, size_t chunk_bytes) {
  stream = s;
  ns_per_byte = gbps > 0.0 ? 1.0 / gbps : 0.0;  // 1 GB/s = 1 byte per ns
  if (chunk_bytes) chunk = chunk_bytes;
  void* p = nullptr;
  if (cudaMalloc(&p, 64) != cudaSuccess) return set_error(VC_ERR_CUDA, "vc_link: could not allocate its clock");
  if (cudaMemsetAsync(p, 0, 64, stream) != cudaSuccess) {
    cudaFree(p);
    return set_error(VC_ERR_CUDA, "vc_link: could not clear its clock");
  }
  clock = static_cast<uint64_t*>(p);
  flags = reinterpret_cast<uint32_t*>(static_cast<char*>(p) + 32);
  return VC_OK;
}

PacedLink::~PacedLink() {
  if (clock) {
    cudaStreamSynchronize(stream);
    cudaFree(clock);
  }
}

vc_status PacedLink::copy(void* dst, const void* src, size_t bytes) {
  const char* s = static_cast<const char*>(src);
  char* d = static_cast<char*>(dst);
  if (ns_per_byte == 0.0) {
    if (cudaMemcpyAsync(d, s, bytes, cudaMemcpyHostToDevice, stream) != cudaSuccess)
      return set_error(VC_ERR_CUDA, "vc_link: copy failed: %s", cudaGetErrorString(cudaGetLastError()));
    return VC_OK;
  }
  for (size_t off = 0; off < bytes; off += chunk) {
    const size_t n = bytes - off < chunk ? bytes - off : chunk;
    link_stamp_kernel<<<1, 1, 0, stream>>>(clock);
    if (cudaMemcpyAsync(d + off, s + off, n, cudaMemcpyHostToDevice, stream) != cudaSuccess)
      return set_error(VC_ERR_CUDA, "vc_link: copy failed: %s", cudaGetErrorString(cudaGetLastError()));
    link_pace_kernel<<<1, 1, 0, stream>>>(clock, static_cast<uint64_t>(static_cast<double>(n) * ns_per_byte),
                                          static_cast<uint64_t>(max_wait_ns), flags);
  }
  if (cudaGetLastError() != cudaSuccess) return set_error(VC_ERR_CUDA, "vc_link: pacing launch failed");
  return VC_OK;
}

vc_status PacedLink::read_flags(uint32_t* host_flags) {
  uint32_t f = 0;
  if (cudaMemcpyAsync(&f, flags, 4, cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
      cudaMemsetAsync(flags, 0, 4, stream) != cudaSuccess || cudaStreamSynchronize(stream) != cudaSuccess)
    return set_error(VC_ERR_CUDA, "vc_link: could not read its flags");
  if (host_flags) *host_flags = f;
  return VC_OK;
}

}  // namespace vc

extern "C" {

vc_status vc_link_create(vc_link** out, void* stream, double gbps, size_t chunk_bytes) {
  VC_REQUIRE(out, "vc_link_create: null output");
  VC_REQUIRE(gbps >= 0.0 && gbps <= 1e4, "vc_link_create: rate must be in [0, 1e4] GB/s (0: unpaced)");
  VC_REQUIRE(chunk_bytes == 0 || (chunk_bytes >= 4096 && chunk_bytes <= (size_t(1) << 32)),
             "vc_link_create: chunk must be 0 (default 8 MiB) or 4 KiB .. 4 GiB");
  auto* l = new vc::PacedLink();
  vc_status st = l->init(static_cast<cudaStream_t>(stream), gbps, chunk_bytes);
  if (st != VC_OK) {
    delete l;
    return st;
  }
  *out = reinterpret_cast<vc_link*>(l);
  vc::clear_error();
  return VC_OK;
}

vc_status vc_link_copy(vc_link* link, void* dst, const void* src, size_t bytes) {
  VC_REQUIRE(link && dst && src, "vc_link_copy: null argument");
  vc_status st = reinterpret_cast<vc::PacedLink*>(link)->copy(dst, src, bytes);
  if (st == VC_OK) vc::clear_error();
  return st;
}

vc_status vc_link_flags(vc_link* link, uint32_t* host_flags) {
  VC_REQUIRE(link && host_flags, "vc_link_flags: null argument");
  vc_status st = reinterpret_cast<vc::PacedLink*>(link)->read_flags(host_flags);
  if (st == VC_OK) vc::clear_error();
  return st;
}

vc_status vc_link_destroy(vc_link* link) {
  if (!link) return VC_OK;
  delete reinterpret_cast<vc::PacedLink*>(link);
  vc::clear_error();
  return VC_OK;
}

}  // extern "C"
