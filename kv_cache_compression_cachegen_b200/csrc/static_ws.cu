// static_ws.cu -- cg_encode_static: cg_encode for callers that cannot allocate
// device memory.
//
// The encoder needs scratch memory (quantised symbols, encoder constants,
// per-stream lengths and word slots).  cg_encode takes it from the caller.
// Some callers have no way to provide it: an inference server that reserved
// the whole device for its own pool, a plugin whose enqueue step must not call
// cudaMalloc, or a latency-critical path that cannot afford the implicit
// synchronisation of an allocation.  For them this file keeps one fixed block
// of scratch in device memory, reserved when the library's module is loaded
// and held by every GPU that loads the library until the process exits.
#include <cuda.h>  // CUcontext and CUresult types only; the driver calls are looked up at run time

#include <cstdint>
#include <mutex>

#include "cg_common.cuh"

namespace {

// 128 MiB: enough for, e.g., one 512-token chunk of an 8-head, 128-dim,
// 32-layer cache, or 7 chunks of a 2-head one.  cg_encode_static rejects
// larger requests with CG_ERR_CAPACITY.
constexpr uint64_t kStaticWorkspaceBytes = 128ull << 20;

static __device__ __align__(256) uint8_t g_static_workspace[kStaticWorkspaceBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;

// The block's device address belongs to the context the module was loaded
// into.  A device reset destroys that context; the next one loads the module
// again, possibly elsewhere.  So the cached address is kept together with the
// unique id of its context (cuCtxGetId) and looked up again when the current
// context of the device is another one.
struct Cached {
  unsigned long long ctx_id;
  void* ptr;
};
Cached g_cached[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

// Id of the calling thread's current context; false when there is none (or
// the driver does not offer the calls).  Called with g_mutex held.
bool current_context_id(unsigned long long* id) {
  if (g_ctx_get_current == nullptr || g_ctx_get_id == nullptr) {
    cudaDriverEntryPointQueryResult q1, q2;
    void* f1 = nullptr;
    void* f2 = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f1, 12000, cudaEnableDefault, &q1) !=
            cudaSuccess ||
        cudaGetDriverEntryPointByVersion("cuCtxGetId", &f2, 12000, cudaEnableDefault, &q2) !=
            cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess || q2 != cudaDriverEntryPointSuccess)
      return false;
    g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
    g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(f2);
  }
  CUcontext ctx = nullptr;
  if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return g_ctx_get_id(ctx, id) == CUDA_SUCCESS;
}

// The array's name is only a host-side handle; the kernels need its device
// address, looked up with the device current, once per device and context.
cudaError_t static_workspace(void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mutex);
  unsigned long long id = 0;
  if (current_context_id(&id) && g_cached[dev].ptr != nullptr && g_cached[dev].ctx_id == id) {
    *out = g_cached[dev].ptr;
    return cudaSuccess;
  }
  void* ptr = nullptr;
  err = cudaGetSymbolAddress(&ptr, g_static_workspace);  // also makes the context current
  if (err != cudaSuccess) return err;
  if (!current_context_id(&id)) return cudaErrorDeviceUninitialized;
  g_cached[dev] = Cached{id, ptr};
  *out = ptr;
  return cudaSuccess;
}

}  // namespace

extern "C" cg_status cg_encode_static(const cg_shape* shape, const uint16_t* kv_dev,
                                      int64_t total_tokens, int64_t token_start,
                                      int32_t num_chunks, int32_t chunk_tokens, cg_level level,
                                      const uint8_t* tables_dev, uint8_t* out_dev,
                                      uint64_t out_stride, uint64_t* out_sizes_dev,
                                      int32_t* status_dev, cudaStream_t stream) {
  uint64_t need = 0;
  cg_status st = cg_encode_workspace_bytes(shape, chunk_tokens, num_chunks, &need);
  if (st != CG_OK) return st;
  if (need > kStaticWorkspaceBytes) return CG_ERR_CAPACITY;
  void* ws = nullptr;
  if (static_workspace(&ws) != cudaSuccess) return CG_ERR_CUDA;
  // Every byte the encoder reads from its workspace is written earlier in the
  // same call, so nothing needs clearing between calls.
  return cg_encode(shape, kv_dev, total_tokens, token_start, num_chunks, chunk_tokens, level,
                   tables_dev, out_dev, out_stride, out_sizes_dev, status_dev, ws,
                   kStaticWorkspaceBytes, stream);
}
