// Geometric routing for callers that cannot allocate device memory.
//
// Some callers of this library may not allocate device memory at call time and have no
// workspace to hand over: a plugin inside a host framework whose memory pool owns the whole
// GPU, or a latency-critical loop whose policy forbids allocation after start-up.  For them
// lsrm_route_geometric_noalloc runs the same centroid and top-k kernels as
// lsrm_route_geometric, but keeps the per-block centroids in a fixed array that lives in
// the library's own device memory (a file-scope __device__ array, held by every GPU that
// loads the library until the process exits).
#include "lsrm_common.cuh"

namespace lsrm {

lsrm_status launch_route_geometric(const lsrm_nsa_desc& d, const int32_t* off, const int32_t* coords, int32_t* cen,
                                   int32_t* idx, uint32_t* status, cudaStream_t stream);

// at most this many blocks: 3 int32 centroids per block, 192 KiB per GPU
constexpr int kNoAllocMaxBlocks = 16384;
static __device__ __align__(256) int32_t g_noalloc_centroids[kNoAllocMaxBlocks * 3];

namespace {

// The host-side name of the array is not a device address.  Its address on the current device
// is looked up on every call (a host-side query that allocates nothing), so that no address
// outlives the context it belongs to: a pointer cached across a device reset or a recreated
// primary context would point into a dead module.
lsrm_status scratch_for_current_device(int32_t** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_centroids) != cudaSuccess || p == nullptr) return LSRM_ERR_CUDA;
  *out = static_cast<int32_t*>(p);
  return LSRM_OK;
}

}  // namespace
}  // namespace lsrm

extern "C" lsrm_status lsrm_route_geometric_noalloc(const lsrm_nsa_desc* desc, const int32_t* off,
                                                    const int32_t* coords, int32_t* idx, uint32_t* status_or_null,
                                                    void* stream) {
  using namespace lsrm;
  // the same descriptor checks as lsrm_route_geometric, then the size limit of the fixed scratch
  const lsrm_status ds = check_desc(desc);
  if (ds != LSRM_OK) return ds;
  if (off == nullptr || coords == nullptr || idx == nullptr) return LSRM_ERR_INVALID_ARG;
  if (desc->n_blocks > kNoAllocMaxBlocks) return LSRM_ERR_WORKSPACE;  // the fixed scratch is too small
  int32_t* cen = nullptr;
  const lsrm_status st = scratch_for_current_device(&cen);
  if (st != LSRM_OK) return st;
  return launch_route_geometric(*desc, off, coords, cen, idx, status_or_null, (cudaStream_t)stream);
}
