// noalloc.cu -- LaCT entry point for callers that cannot allocate device
// memory: the workspace lives in a fixed, file-scope device array instead of
// a caller-provided buffer.
//
// Who needs it: code hosted inside another program that owns every device
// allocation (a plugin or extension handed only its input and output
// tensors, with no allocator hook), and code on latency-critical paths where
// cudaMalloc / cudaFree, which may synchronise the device, are not allowed.
// Such callers still pass q, k, v, lr, the state and the output.
//
// Limits and sharing:
//   * the scratch array holds kNoAllocScratchBytes (64 MiB); problems whose
//     lact_workspace_bytes_min() exceeds it are rejected with
//     TTT_ERR_WORKSPACE before anything is enqueued, and a problem whose
//     fastest form needs more runs the form that fits;
//   * every GPU on which the library's device code is loaded holds the array
//     until the process exits;
//   * all calls share the one array and it keeps the last call's contents:
//     the status block at its start is cleared on the stream at the start of
//     each call (the rest is fully rewritten before it is read), and calls
//     whose GPU work overlaps -- on different streams or host threads -- race
//     on it and must not be issued that way;
//   * the first call on each device looks up the array's device address
//     (cudaGetSymbolAddress, with that device current) and caches it; a
//     cudaDeviceReset of that device invalidates the cached address, so the
//     entry point must not be used after one;
//   * the stream must belong to the current device (checked: the address
//     is that device's copy of the array);
//   * a bounded in-kernel wait that runs out records its code in the
//     array's status block, which lact_noalloc_check_status() reads.
#include <mutex>

#include "../../include/ttt.h"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) uint8_t g_lact_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (nullptr on
// failure).  In host code `g_lact_scratch` names a host-side stand-in, so the
// address must come from the runtime, once per device.
void* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_lact_scratch) != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

// The stream's device must be the current one: the scratch address looked up
// for the current device names another GPU's copy of the array otherwise.
int check_stream_device(void* stream) {
  int cur = 0, sdev = 0;
  if (cudaGetDevice(&cur) != cudaSuccess) return TTT_ERR_CUDA;
  if (stream == nullptr) return TTT_OK;   // legacy default stream: the current device's
  if (cudaStreamGetDevice(reinterpret_cast<cudaStream_t>(stream), &sdev) != cudaSuccess) {
    cudaGetLastError();
    return TTT_ERR_ARG;
  }
  return sdev == cur ? TTT_OK : TTT_ERR_ARG;
}

}  // namespace

extern "C" int lact_chunk_fwd_noalloc(const lact_desc* desc, const void* q, const void* k,
                                      const void* v, const float* lr, void* state, void* out,
                                      void* stream) {
  size_t need = 0;
  int e = lact_workspace_bytes_min(desc, &need);
  if (e != TTT_OK) return e;
  if (need > kNoAllocScratchBytes) return TTT_ERR_WORKSPACE;
  e = check_stream_device(stream);
  if (e != TTT_OK) return e;
  void* scratch = scratch_on_current_device();
  if (scratch == nullptr) return TTT_ERR_CUDA;
  if (cudaMemsetAsync(scratch, 0, TTT_STATUS_BYTES, reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return TTT_ERR_CUDA;
  return lact_chunk_fwd(desc, q, k, v, lr, state, out, scratch, kNoAllocScratchBytes, stream);
}

extern "C" int lact_noalloc_check_status(void* stream) {
  const int e = check_stream_device(stream);
  if (e != TTT_OK) return e;
  void* scratch = scratch_on_current_device();
  if (scratch == nullptr) return TTT_ERR_CUDA;
  return ttt_check_device_status(scratch, stream);
}
