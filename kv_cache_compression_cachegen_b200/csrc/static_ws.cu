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
// unique id of its context and looked up again when the current context of
// the device is another one.
struct Cached {
  unsigned long long ctx_id;
  void* ptr;
};
Cached g_cached[kMaxDevices] = {};

// The array's name is only a host-side handle; the kernels need its device
// address, looked up with the device current, once per device and context.
cudaError_t static_workspace(void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mutex);
  unsigned long long id = 0;
  if (cg::current_context_id(&id) && g_cached[dev].ptr != nullptr && g_cached[dev].ctx_id == id) {
    *out = g_cached[dev].ptr;
    return cudaSuccess;
  }
  void* ptr = nullptr;
  err = cudaGetSymbolAddress(&ptr, g_static_workspace);  // also makes the context current
  if (err != cudaSuccess) return err;
  if (!cg::current_context_id(&id)) return cudaErrorDeviceUninitialized;
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
