// egat_forward_noalloc: the fused forward pass with its scratch in a fixed,
// library-owned device array instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory when they call us: a plugin
// running inside a host framework that owns every device allocation and
// forbids others, or a long-running service that fixes its memory footprint at
// start-up and may not call cudaMalloc afterwards.  This entry point needs no
// allocation at call time: the scratch for h' lives in a file-scope
// __device__ array of kNoallocScratchBytes bytes that every GPU loading the
// library holds until the process exits.
//
// The array's name is only a host-side stand-in in host code, not a device
// address, so it is never handed to a kernel directly.  The first successful
// call on each device (with that device current) looks up the array's device
// address with cudaGetSymbolAddress, checks the result and caches it for that
// device; later calls on the device reuse the cached address.  A lookup that
// fails is not cached: the next call tries again.  That first call should
// come before any stream capture.  The cached address belongs to the device's
// context: after cudaDeviceReset (or anything else that destroys the primary
// context) it is stale, and this entry point must not be called again in that
// process.
//
// All calls share the one array and it keeps the previous call's contents.
// Nothing in it needs to start at zero: step 2 writes every element of h'
// before step 3 reads it.  Calls whose work overlaps on the GPU (for example
// on two streams) race on the array; callers serialise them.
#include <mutex>

#include "egat_device.cuh"
#include "egat_host.h"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(EGAT_NOALLOC_SCRATCH_BYTES);
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices];   // null until a lookup on that device succeeded

// Device address of the scratch array on the current device (looked up once
// per device; a failed lookup is retried by the next call).
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return EGAT_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();   // clear the sticky-free error so later calls start clean
      return EGAT_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return EGAT_OK;
}

}  // namespace

extern "C" {

int egat_forward_noalloc(const egat_shape* s, const void* d_h, const float* d_pos,
                         const void* d_q, const void* d_k, const int32_t* d_nbr_or_rowptr,
                         const int32_t* d_cnt_or_col, const int32_t* d_order, const float* d_w1,
                         const float* d_w2, float* d_out, void* stream) {
  size_t need = 0;
  const int rc = egat_forward_workspace_bytes(s, &need);
  if (rc != EGAT_OK) return rc;
  if (need > kNoallocScratchBytes) return EGAT_ERR_SCRATCH_LIMIT;
  if (s->n == 0) return EGAT_OK;
  void* scratch = nullptr;
  const int e = scratch_address(&scratch);
  if (e != EGAT_OK) return e;
  return egat_forward(s, d_h, d_pos, d_q, d_k, d_nbr_or_rowptr, d_cnt_or_col, d_order, d_w1,
                      d_w2, scratch, kNoallocScratchBytes, d_out, stream);
}

}  // extern "C"
