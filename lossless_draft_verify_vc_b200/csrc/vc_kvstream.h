// vc_kvstream.h -- the double-buffered host -> device layer stream behind the
// vc_kvstream_* entry points (also used by the scheduler).
#pragma once

#include <vector>

#include "vc_common.cuh"
#include "vc_link.h"

namespace vc {

struct KvStream {
  int n_layers = 0;
  std::vector<const void*> host_k, host_v;
  size_t bytes_per_layer = 0;
  void* dev_k[2] = {nullptr, nullptr};
  void* dev_v[2] = {nullptr, nullptr};
  int slot_layer[2] = {-1, -1};
  bool slot_used[2] = {false, false};
  bool slot_released[2] = {true, true};  // host-call order: the slot's layer was released
  cudaEvent_t copied[2] = {nullptr, nullptr};
  cudaEvent_t released[2] = {nullptr, nullptr};
  cudaStream_t copy_stream = nullptr;
  PacedLink* link = nullptr;  // optional: copies go through this link (on copy_stream) at its rate

  vc_status init(int n_layers, const void* const* hk, const void* const* hv, size_t bytes, void* const* dk,
                 void* const* dv, cudaStream_t cs);
  // t0 / t1 (optional, timing events) are recorded on the copy stream around the copies
  vc_status prefetch(int layer, cudaEvent_t t0, cudaEvent_t t1);
  vc_status acquire(int layer, cudaStream_t compute, const void** k, const void** v);
  vc_status release(int layer, cudaStream_t compute);
  ~KvStream();
};

}  // namespace vc
