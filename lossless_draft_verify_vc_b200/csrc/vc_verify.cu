// vc_verify.cu -- block verification attention (placeholder until the
// tcgen05 kernel lands in this file).
#include "vc_common.cuh"

extern "C" {

size_t vc_verify_attn_workspace_size(const vc_attn_shape* shape, int64_t T, int nq) {
  (void)shape;
  (void)T;
  (void)nq;
  return 0;
}

vc_status vc_verify_attn(const vc_attn_shape*, const void*, const void*, const void*, int64_t, int, float*, float*,
                         void*, size_t, void*) {
  return vc::set_error(VC_ERR_UNSUPPORTED, "vc_verify_attn: not built yet");
}

}  // extern "C"
