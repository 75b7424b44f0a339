// nsa_prefill_noalloc: the prefill entry point for callers that cannot
// allocate device memory.
//
// Some callers of this library cannot call cudaMalloc (or any allocator) at
// the point where they run attention: code that executes under a memory
// manager it does not own (a serving runtime or framework that hands out all
// device memory from its own pool and forbids side allocations), code that
// must not pay the device-wide synchronisation a cudaMalloc can cause, or
// code that simply has no handle on an allocator (a plugin called with bare
// tensor pointers).  nsa_prefill needs a caller-provided workspace; this
// variant instead uses one file-scope device array, so the caller passes only
// inputs and outputs.
//
// The array is a fixed kStaticWorkspaceBytes (32 MiB) per GPU: every GPU that
// loads the library holds it until the process exits.  Plans whose
// nsa_workspace_size(plan, NSA_MODE_PREFILL) exceeds it are rejected.
// The first call on each device looks up the array's device address with
// cudaGetSymbolAddress (with that device current) and caches it, so that first
// call should be made before any stream capture.
// Every call shares the array and it keeps the last call's contents; the
// launch sequence clears the one field that must start at zero (the status
// word) itself.  Calls that overlap on the GPU (on different streams, or
// from different host threads) race on the array and must not be issued.
// The cached address is tied to the device's primary context: after a
// device reset it is stale and the entry point must not be used again.
// Device-side faults land in the array's status word (offset 0), which
// nsa_noalloc_read_device_status reads and clears.
#include <cstdio>
#include <mutex>

#include "nsa_internal.cuh"

namespace {

constexpr size_t kStaticWorkspaceBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

std::mutex g_mutex;
void* g_device_ptr[kMaxDevices] = {};

// Device address of the array on the current device, looked up once per
// device (with that device current) and cached.
int static_workspace(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_device_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess || !p) {
      fprintf(stderr, "nsa_prefill_noalloc: cudaGetSymbolAddress failed: %s\n",
              cudaGetErrorString(e));
      return NSA_ERR_CUDA;
    }
    g_device_ptr[dev] = p;
  }
  *out = g_device_ptr[dev];
  return NSA_OK;
}

}  // namespace

extern "C" int nsa_prefill_noalloc(nsa_plan_t plan, const void* q, const void* k, const void* v,
                                   const float* gates, const float* w_k, const float* w_v,
                                   const int* cu_seqlens, int batch, int total_tokens, void* out,
                                   void* k_cmp, void* v_cmp, int* sel_idx, void* stream) {
  if (!plan) return NSA_ERR_INVALID_ARG;
  const size_t need = nsa_workspace_size(plan, NSA_MODE_PREFILL);
  if (need == 0 || need > kStaticWorkspaceBytes) {
    fprintf(stderr,
            "nsa_prefill_noalloc: the plan needs %zu workspace bytes, more than the %zu-byte "
            "static array; use nsa_prefill with a caller workspace\n",
            need, kStaticWorkspaceBytes);
    return NSA_ERR_WORKSPACE;
  }
  void* ws = nullptr;
  const int rc = static_workspace(&ws);
  if (rc != NSA_OK) return rc;
  return nsa_prefill(plan, q, k, v, gates, w_k, w_v, cu_seqlens, batch, total_tokens, out, k_cmp,
                     v_cmp, sel_idx, ws, kStaticWorkspaceBytes, stream);
}

extern "C" int nsa_noalloc_read_device_status(void* stream) {
  void* ws = nullptr;
  const int rc = static_workspace(&ws);
  if (rc != NSA_OK) return NSA_ERR_CUDA;
  return nsa_read_device_status(ws, stream);
}
