// cosa_plan_static: the KAP planning call for callers that cannot hand the
// library a workspace.  Some callers have no way to obtain device memory of
// their own: a serving engine that reserves the whole GPU at start-up and
// only passes kernels the tensors it owns, or a plug-in whose host framework
// keeps the allocator to itself.  This entry point gives them cosa_plan
// without a workspace argument: its scratch lives in a fixed-size array that
// is part of the library's device image.
//
// Costs and rules of that choice:
//  * every GPU on which the library loads this array holds
//    COSA_STATIC_SCRATCH_BYTES of device memory until the process exits;
//  * problems whose cosa_plan_workspace_bytes exceed that size are rejected
//    with COSA_EWORKSPACE before anything is launched;
//  * all calls share the one array and leave their contents in it, so two
//    calls whose work can overlap on the GPU (different streams, no ordering
//    between them) race on it; calls on one stream are safe;
//  * nothing in the array needs to start at zero: every byte a kernel reads
//    was written earlier in the same call;
//  * the first call on each device looks up the array's device address
//    (cudaGetSymbolAddress, with that device current); make that first call
//    before any stream capture.
// Nothing here allocates: no cudaMalloc, no cudaFree, no allocating library
// routine.
#include <mutex>

#include "cosa.h"

namespace {

static __device__ __align__(256) unsigned char g_plan_scratch[COSA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 256;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_plan_scratch on the current device (looked up once per
// device).  The array's name in host code is only a stand-in for the symbol.
cosa_status scratch_on_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return COSA_ECUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_plan_scratch) != cudaSuccess || !p) return COSA_ECUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return COSA_OK;
}

}  // namespace

extern "C" COSA_API cosa_status cosa_plan_static(const cosa_shape* shape, const void* q, const void* k,
                                                 const int32_t* page_table, double budget, int kmax,
                                                 int32_t* order, int32_t* count, int32_t* hrm_count,
                                                 float* block_score, uint8_t* hrm_flags, uint32_t* dev_status,
                                                 cudaStream_t stream) {
  const size_t need = cosa_plan_workspace_bytes(shape);
  if (need == 0)   // invalid shape: let cosa_plan report which check failed
    return cosa_plan(shape, q, k, page_table, budget, kmax, order, count, hrm_count, block_score, hrm_flags,
                     nullptr, 0, dev_status, stream);
  if (need > (size_t)COSA_STATIC_SCRATCH_BYTES) return COSA_EWORKSPACE;
  void* scratch = nullptr;
  const cosa_status st = scratch_on_current_device(&scratch);
  if (st != COSA_OK) return st;
  return cosa_plan(shape, q, k, page_table, budget, kmax, order, count, hrm_count, block_score, hrm_flags,
                   scratch, (size_t)COSA_STATIC_SCRATCH_BYTES, dev_status, stream);
}
