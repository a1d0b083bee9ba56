// context.cu -- per-device, per-context resources of the library: the id of
// the calling thread's current CUDA context, and the encoder's side stream.
//
// cg_encode splits a call of several chunks into two halves and runs the
// second half on a side stream, forked from the caller's stream with an event
// and joined back with another, so the call stays ordered on the caller's
// stream (and is captured as a fork/join when that stream is being captured
// into a graph).  The halves' kernels then overlap: one half's memory-bound
// compaction and quantiser loads run beside the other half's issue-bound rANS
// encoding.
#include <cuda.h>  // CUcontext and CUresult types only; the driver calls are looked up at run time

#include <functional>
#include <mutex>

#include "cg_common.cuh"

namespace cg {
namespace {

constexpr int kMaxDevices = 64;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

std::once_flag g_lookup_once;
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

void lookup_driver_calls() {
  cudaDriverEntryPointQueryResult q1, q2;
  void* f1 = nullptr;
  void* f2 = nullptr;
  if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f1, 12000, cudaEnableDefault, &q1) !=
          cudaSuccess ||
      cudaGetDriverEntryPointByVersion("cuCtxGetId", &f2, 12000, cudaEnableDefault, &q2) !=
          cudaSuccess ||
      q1 != cudaDriverEntryPointSuccess || q2 != cudaDriverEntryPointSuccess)
    return;
  g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
  g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(f2);
}

// A device reset destroys the context that owns the stream and the events;
// the next context gets new ones.
struct Side {
  unsigned long long ctx_id;
  cudaStream_t stream;
  cudaEvent_t fork, join;
};
Side g_side[kMaxDevices] = {};
std::mutex g_side_mutex;

}  // namespace

bool current_context_id(unsigned long long* id) {
  std::call_once(g_lookup_once, lookup_driver_calls);
  if (g_ctx_get_current == nullptr || g_ctx_get_id == nullptr) return false;
  CUcontext ctx = nullptr;
  if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return g_ctx_get_id(ctx, id) == CUDA_SUCCESS;
}

cudaError_t fork_join(cudaStream_t stream, const std::function<cudaError_t(cudaStream_t)>& first,
                      const std::function<cudaError_t(cudaStream_t)>& second, bool* forked) {
  *forked = false;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cudaSuccess;
  std::lock_guard<std::mutex> lock(g_side_mutex);
  unsigned long long id = 0;
  if (!current_context_id(&id)) return cudaSuccess;
  Side& s = g_side[dev];
  if (s.stream == nullptr || s.ctx_id != id) {
    // Creating the stream and events is not a stream operation, but it is
    // left out of a graph capture all the same: a capturing caller runs the
    // call on its own stream until an uncaptured call has created them.
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone)
      return cudaSuccess;
    Side n{id, nullptr, nullptr, nullptr};
    if (cudaStreamCreateWithFlags(&n.stream, cudaStreamNonBlocking) != cudaSuccess) {
      (void)cudaGetLastError();
      return cudaSuccess;
    }
    if (cudaEventCreateWithFlags(&n.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&n.join, cudaEventDisableTiming) != cudaSuccess) {
      (void)cudaGetLastError();
      if (n.fork) cudaEventDestroy(n.fork);
      cudaStreamDestroy(n.stream);
      return cudaSuccess;
    }
    s = n;  // a previous context's handles died with it
  }
  // A wait takes the event's most recent record at the time of the call, so
  // the events can be recorded again by the next call once these are queued.
  cudaError_t err = cudaEventRecord(s.fork, stream);
  if (err == cudaSuccess) err = cudaStreamWaitEvent(s.stream, s.fork, 0);
  if (err != cudaSuccess) return err;
  *forked = true;
  const cudaError_t e1 = first(stream);
  const cudaError_t e2 = second(s.stream);
  // The join is queued even when a launch failed, so the caller's stream never
  // runs ahead of work queued on the side stream.
  err = cudaEventRecord(s.join, s.stream);
  if (err == cudaSuccess) err = cudaStreamWaitEvent(stream, s.join, 0);
  if (e1 != cudaSuccess) return e1;
  if (e2 != cudaSuccess) return e2;
  return err;
}

}  // namespace cg
