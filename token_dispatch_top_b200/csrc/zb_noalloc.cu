// zb_noalloc.cu -- zb_plan_noalloc: zb_plan for callers that cannot allocate
// device memory, with the plan's scratch workspace held in a fixed array that
// lives inside this library on every GPU that loads it.
//
// Some callers have no way to hand the library a scratch buffer: a plugin
// that a host framework enqueues from inside its own execution step, where the
// framework owns every device allocation and the plugin interface offers no
// workspace, or a serving loop that forbids cudaMalloc/cudaFree on its hot
// path because those calls can synchronise the whole device and stall every
// other stream.  Such callers still allocate the plan's outputs once, up
// front; only the per-call scratch comes from here.
#include <mutex>

#include "zb_internal.cuh"

namespace {

// The scratch array: one copy per device that loads the library, kept until
// the process exits.  Its name is a host-side stand-in for the device array:
// host code must never pass &zb_noalloc_scratch to a kernel; it asks the
// runtime for the device address instead (scratch_address below).
static __device__ __align__(256) unsigned char zb_noalloc_scratch[ZB_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_lock;
void* g_addr[kMaxDevices] = {};

// Device address of the scratch array on the calling thread's current device,
// looked up once per device (with that device current) and cached for the life
// of the process.  A device reset reloads the module, so the header tells
// callers not to use this entry point on a device after resetting it.
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ZB_ERR_CUDA;
  std::lock_guard<std::mutex> guard(g_lock);
  if (g_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, zb_noalloc_scratch) != cudaSuccess || p == nullptr)
      return ZB_ERR_CUDA;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return ZB_OK;
}

}  // namespace

extern "C" int zb_plan_noalloc(const zb_config* cfg, const int32_t* topk_ids,
                               const zb_plan_t* plan, void* stream) {
  if (zb_validate(cfg) != ZB_OK) return ZB_ERR_INVALID;
  if (zb_workspace_bytes(cfg) > size_t(ZB_NOALLOC_SCRATCH_BYTES)) return ZB_ERR_INVALID;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != ZB_OK) return rc;
  return zb_plan(cfg, topk_ids, plan, scratch, size_t(ZB_NOALLOC_SCRATCH_BYTES), stream);
}
