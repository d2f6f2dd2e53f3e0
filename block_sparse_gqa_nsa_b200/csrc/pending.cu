// Launcher of the backward; it returns LSRM_ERR_UNSUPPORTED until that kernel is built.
#include "lsrm_common.cuh"

namespace lsrm {
lsrm_status launch_backward(const lsrm_nsa_desc&, const int32_t*, const void*, const void*, const void*, const void*,
                            const void*, const void*, const int32_t*, int, const float*, const void*, void*, void*,
                            void*, void*, unsigned char*, uint32_t*, cudaStream_t) {
  return LSRM_ERR_UNSUPPORTED;
}
}  // namespace lsrm
