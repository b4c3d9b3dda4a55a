// Decode attention without a caller-provided workspace.
//
// kvq_decode_attention needs a device workspace for its split partials.  Some
// callers cannot provide one: a serving engine that has reserved nearly all of
// the device memory for its own pool and lets no one else call cudaMalloc, a
// plugin whose host gives it no allocator, or a latency-critical loop that must
// not pay for cudaMalloc/cudaFree and the device synchronization they imply.
// For them this entry point uses a fixed scratch array that lives in the
// library itself, so it allocates nothing at call time.
//
// The array below is a file-scope __device__ variable: every GPU on which this
// library's code is loaded holds kNoAllocScratchBytes of it until the process
// exits.  In host code its name is only a host-side stand-in, not a device
// address, so the real address is looked up once per device with
// cudaGetSymbolAddress while that device is current, and passed on as the
// workspace pointer.  That lookup happens inside the first call on each device
// (of the decode or of the status calls below).
//
// Its first word is the status word the decode kernels OR KVQ_STATUS_* bits
// into, exactly as in a caller's workspace: it starts at zero when the library
// is loaded, is never cleared by a decode, and is read and cleared by
// kvq_noalloc_read_status / kvq_noalloc_reset_status.
#include <atomic>
#include <mutex>

#include "../../include/kvq.h"
#include "kvq_internal.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = KVQ_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
std::atomic<void*> g_scratch_ptr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (looked up once per device;
// later calls read the cached address without taking the lock).
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (!p) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
    if (!p) {
      if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) {
        cudaGetLastError();
        return KVQ_ERR_CUDA;
      }
      g_scratch_ptr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return KVQ_OK;
}

}  // namespace

extern "C" int kvq_decode_attention_noalloc(kvq_cache* cache, const void* q, void* out,
                                            int num_splits, void* stream) {
  if (!cache || !q || !out || num_splits < 0) return KVQ_ERR_INVALID_ARG;
  // pick a split count whose partials fit in the scratch array
  size_t need = 0;
  int rc = kvq_decode_workspace_size(cache, num_splits, &need);
  if (rc) return rc;
  int splits = num_splits;
  if (need > kNoAllocScratchBytes) {
    if (num_splits > 0) return KVQ_ERR_WORKSPACE;     // the requested plan does not fit
    kvq_plan plan;
    rc = kvq_get_plan(cache, 0, &plan);
    if (rc) return rc;
    const int start = plan.splits_quant > 0 ? plan.splits_quant : plan.splits_fp16;
    splits = 0;
    for (int s = start - 1; s >= 1; --s) {
      rc = kvq_decode_workspace_size(cache, s, &need);
      if (rc) return rc;
      if (need <= kNoAllocScratchBytes) {
        splits = s;
        break;
      }
    }
    if (splits == 0) return KVQ_ERR_WORKSPACE;        // even one split per row is too large
  }
  void* scratch = nullptr;
  rc = scratch_for_current_device(&scratch);
  if (rc) return rc;
  return kvq_decode_attention(cache, q, out, scratch, kNoAllocScratchBytes, splits, stream);
}

extern "C" int kvq_noalloc_read_status(unsigned int* status, void* stream) {
  if (!status) return KVQ_ERR_INVALID_ARG;
  void* scratch = nullptr;
  const int rc = scratch_for_current_device(&scratch);
  if (rc) return rc;
  return kvq_read_status(scratch, status, stream);
}

extern "C" int kvq_noalloc_reset_status(void* stream) {
  void* scratch = nullptr;
  const int rc = scratch_for_current_device(&scratch);
  if (rc) return rc;
  return kvq_reset_status(scratch, stream);
}
