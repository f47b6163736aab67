// vc_link.h -- a host -> device link of a given bandwidth, emulated on the
// GPU's own copy path (behind the vc_link_* entry points, the scheduler's
// remote link and the paced verification stream).
#pragma once

#include "vc_common.cuh"

namespace vc {

// Copies travel in chunks on one stream.  Before each chunk a one-thread
// kernel stamps the device clock; after it another one sleeps until the
// stamp plus chunk_bytes / rate has passed, so chunks leave the stream no
// faster than the rate (the real copy, at the bus speed, runs inside that
// window).  With rate 0 the copies are plain cudaMemcpyAsync calls.
struct PacedLink {
  cudaStream_t stream = nullptr;
  double ns_per_byte = 0.0;  // 0: unpaced
  size_t chunk = 8u << 20;
  uint64_t* clock = nullptr;  // device: [0] start stamp of the chunk in flight
  uint32_t* flags = nullptr;  // device: VC_FLAG_WAIT_TIMEOUT if a pace wait gave up
  double max_wait_ns = 60e9;  // bound of one pace wait

  vc_status init(cudaStream_t s, double gbps, size_t chunk_bytes);
  vc_status copy(void* dst, const void* src, size_t bytes);
  // reads (and clears) the flag word: a synchronous read on the stream
  vc_status read_flags(uint32_t* host_flags);
  ~PacedLink();
};

}  // namespace vc
