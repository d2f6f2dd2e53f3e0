// Launchers of the Speed3R pooled-query kernels and of the backward; they return
// LSRM_ERR_UNSUPPORTED until those kernels are built.
#include "lsrm_common.cuh"

namespace lsrm {
lsrm_status launch_route_pooled(const lsrm_nsa_desc&, const void*, const void*, int32_t*, uint32_t*, cudaStream_t) {
  return LSRM_ERR_UNSUPPORTED;
}
lsrm_status launch_pooled_cmp(const lsrm_nsa_desc&, const void*, const void*, const void*, float*, float*,
                              cudaStream_t) {
  return LSRM_ERR_UNSUPPORTED;
}
lsrm_status launch_pooled_broadcast(const lsrm_nsa_desc&, const int32_t*, const float*, const float*, float*, float*,
                                    cudaStream_t) {
  return LSRM_ERR_UNSUPPORTED;
}
lsrm_status launch_attn_pooled_fused(const lsrm_nsa_desc&, const int32_t*, const void*, const void*, const void*,
                                     const void*, const int32_t*, const float*, void*, float*, uint32_t*,
                                     cudaStream_t) {
  return LSRM_ERR_UNSUPPORTED;
}
lsrm_status launch_backward(const lsrm_nsa_desc&, const int32_t*, const void*, const void*, const void*, const void*,
                            const void*, const void*, const int32_t*, int, const float*, const void*, void*, void*,
                            void*, void*, unsigned char*, uint32_t*, cudaStream_t) {
  return LSRM_ERR_UNSUPPORTED;
}
}  // namespace lsrm
