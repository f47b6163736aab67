// vc_kvstream.cu -- per-layer host -> HBM streaming of the full KV cache for
// verification, double-buffered against compute.
//
// The full cache may stay in host memory and travel to the GPU only when a
// request verifies (devshah.ca page "VeriCache: making lossy KV compression
// exact", section "Verifying Without Giving Back the Speedup").  Layer l is
// copied into staging slot l % 2 on the copy stream while the compute stream
// verifies layer l - 1 from the other slot.  Ordering is carried entirely by
// CUDA events:
//   copied[s]   recorded on the copy stream after the copies into slot s,
//   released[s] recorded on the compute stream after the work that read s;
// the copy stream waits released[s] before overwriting slot s, the compute
// stream waits copied[s] before reading it.  No call blocks the host.
#include "vc_kvstream.h"

namespace vc {

vc_status KvStream::init(int n_layers_, const void* const* hk, const void* const* hv, size_t bytes,
                         void* const* dk, void* const* dv, cudaStream_t cs) {
  n_layers = n_layers_;
  host_k.assign(hk, hk + n_layers);
  host_v.assign(hv, hv + n_layers);
  bytes_per_layer = bytes;
  for (int s = 0; s < 2; ++s) {
    dev_k[s] = dk[s];
    dev_v[s] = dv[s];
    slot_layer[s] = -1;
    slot_used[s] = false;
    if (cudaEventCreateWithFlags(&copied[s], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&released[s], cudaEventDisableTiming) != cudaSuccess)
      return set_error(VC_ERR_CUDA, "vc_kvstream: event creation failed");
  }
  copy_stream = cs;
  return VC_OK;
}

KvStream::~KvStream() {
  for (int s = 0; s < 2; ++s) {
    if (copied[s]) cudaEventDestroy(copied[s]);
    if (released[s]) cudaEventDestroy(released[s]);
  }
}

vc_status KvStream::prefetch(int layer, cudaEvent_t t0, cudaEvent_t t1) {
  VC_REQUIRE(layer >= 0 && layer < n_layers, "vc_kvstream_prefetch: layer %d out of range", layer);
  const int s = layer & 1;
  VC_REQUIRE(slot_released[s], "vc_kvstream_prefetch: slot of layer %d still holds layer %d (release it first)",
             layer, slot_layer[s]);
  if (slot_used[s] && cudaStreamWaitEvent(copy_stream, released[s], 0) != cudaSuccess)
    return set_error(VC_ERR_CUDA, "vc_kvstream_prefetch: wait failed");
  if (t0) cudaEventRecord(t0, copy_stream);
  if (link) {
    vc_status st = link->copy(dev_k[s], host_k[layer], bytes_per_layer);
    if (st == VC_OK) st = link->copy(dev_v[s], host_v[layer], bytes_per_layer);
    if (st != VC_OK) return st;
  } else if (cudaMemcpyAsync(dev_k[s], host_k[layer], bytes_per_layer, cudaMemcpyHostToDevice, copy_stream) !=
                 cudaSuccess ||
             cudaMemcpyAsync(dev_v[s], host_v[layer], bytes_per_layer, cudaMemcpyHostToDevice, copy_stream) !=
                 cudaSuccess) {
    return set_error(VC_ERR_CUDA, "vc_kvstream_prefetch: copy failed: %s", cudaGetErrorString(cudaGetLastError()));
  }
  if (t1) cudaEventRecord(t1, copy_stream);
  if (cudaEventRecord(copied[s], copy_stream) != cudaSuccess)
    return set_error(VC_ERR_CUDA, "vc_kvstream_prefetch: event record failed");
  slot_layer[s] = layer;
  slot_used[s] = true;
  slot_released[s] = false;
  clear_error();
  return VC_OK;
}

vc_status KvStream::acquire(int layer, cudaStream_t compute, const void** k, const void** v) {
  VC_REQUIRE(layer >= 0 && layer < n_layers, "vc_kvstream_acquire: layer %d out of range", layer);
  const int s = layer & 1;
  VC_REQUIRE(slot_layer[s] == layer, "vc_kvstream_acquire: layer %d was not prefetched", layer);
  if (cudaStreamWaitEvent(compute, copied[s], 0) != cudaSuccess)
    return set_error(VC_ERR_CUDA, "vc_kvstream_acquire: wait failed");
  if (k) *k = dev_k[s];
  if (v) *v = dev_v[s];
  clear_error();
  return VC_OK;
}

vc_status KvStream::release(int layer, cudaStream_t compute) {
  VC_REQUIRE(layer >= 0 && layer < n_layers, "vc_kvstream_release: layer %d out of range", layer);
  const int s = layer & 1;
  VC_REQUIRE(slot_layer[s] == layer, "vc_kvstream_release: layer %d does not own its slot", layer);
  if (cudaEventRecord(released[s], compute) != cudaSuccess)
    return set_error(VC_ERR_CUDA, "vc_kvstream_release: event record failed");
  slot_released[s] = true;
  clear_error();
  return VC_OK;
}

}  // namespace vc

extern "C" {

vc_status vc_kvstream_create(vc_kvstream** out, int n_layers, const void* const* host_k, const void* const* host_v,
                             size_t bytes_per_layer, void* const* dev_k, void* const* dev_v, void* copy_stream) {
  VC_REQUIRE(out && host_k && host_v && dev_k && dev_v, "vc_kvstream_create: null argument");
  VC_REQUIRE(n_layers >= 1 && bytes_per_layer > 0, "vc_kvstream_create: need n_layers >= 1 and bytes > 0");
  for (int l = 0; l < n_layers; ++l)
    VC_REQUIRE(host_k[l] && host_v[l], "vc_kvstream_create: null host pointer for layer %d", l);
  for (int s = 0; s < 2; ++s)
    VC_REQUIRE(dev_k[s] && dev_v[s] && vc::aligned16(dev_k[s]) && vc::aligned16(dev_v[s]),
               "vc_kvstream_create: staging slots must be non-null and 16-byte aligned");
  auto* s = new vc::KvStream();
  vc_status st = s->init(n_layers, host_k, host_v, bytes_per_layer, dev_k, dev_v,
                         static_cast<cudaStream_t>(copy_stream));
  if (st != VC_OK) {
    delete s;
    return st;
  }
  *out = reinterpret_cast<vc_kvstream*>(s);
  vc::clear_error();
  return VC_OK;
}

vc_status vc_kvstream_prefetch(vc_kvstream* s, int layer) {
  VC_REQUIRE(s, "vc_kvstream_prefetch: null stream object");
  return reinterpret_cast<vc::KvStream*>(s)->prefetch(layer, nullptr, nullptr);
}

vc_status vc_kvstream_acquire(vc_kvstream* s, int layer, void* compute_stream, const void** k, const void** v) {
  VC_REQUIRE(s, "vc_kvstream_acquire: null stream object");
  return reinterpret_cast<vc::KvStream*>(s)->acquire(layer, static_cast<cudaStream_t>(compute_stream), k, v);
}

vc_status vc_kvstream_release(vc_kvstream* s, int layer, void* compute_stream) {
  VC_REQUIRE(s, "vc_kvstream_release: null stream object");
  return reinterpret_cast<vc::KvStream*>(s)->release(layer, static_cast<cudaStream_t>(compute_stream));
}

vc_status vc_kvstream_destroy(vc_kvstream* s) {
  if (!s) return VC_OK;
  auto* k = reinterpret_cast<vc::KvStream*>(s);
  cudaError_t e = cudaStreamSynchronize(k->copy_stream);
  delete k;
  if (e != cudaSuccess) return vc::set_error(VC_ERR_CUDA, "vc_kvstream_destroy: %s", cudaGetErrorString(e));
  vc::clear_error();
  return VC_OK;
}

}  // extern "C"
