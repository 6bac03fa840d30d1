// bwd_noalloc.cu -- hstu_jagged_attn_bwd_noalloc: the backward for callers
// that cannot allocate device memory.
//
// hstu_jagged_attn_bwd needs a caller-provided fp32 workspace (the dQ
// accumulator).  Some callers cannot obtain one: code that runs inside another
// runtime's plugin or enqueue callback, where cudaMalloc is forbidden or would
// break the host program's memory plan, or a serving process that sizes all of
// its device memory at start-up and treats any later allocation as a failure.
// For them this entry point uses a fixed scratch array that lives in the
// library itself (a static __device__ array below), so the call allocates
// nothing; inputs and outputs are still the caller's buffers.
//
// Costs and rules of the static scratch:
//   * every GPU that loads the library holds HSTU_BWD_NOALLOC_MAX_ELEMS floats
//     (16 MiB) of device memory until the process exits;
//   * problems with T * num_heads * d_qk above that are rejected with
//     HSTU_ERR_WORKSPACE, nothing is launched;
//   * all calls on a device share the one array and it keeps the previous
//     call's contents; the backward clears the part it uses before use, but two
//     calls whose kernels overlap on the GPU (different streams, or several host
//     threads) race on it, so callers must order them (one stream, or events);
//   * the array is the current device's copy, so `stream` must belong to the
//     current device (HSTU_ERR_UNSUPPORTED otherwise);
//   * the array's device address is looked up (cudaGetSymbolAddress, with the
//     device current) on every call made outside a stream capture; a call
//     made during a capture reuses the address of the last uncaptured call on
//     that device, so make one call before any stream capture begins.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/hstu.h"

namespace {

// The host-side name of this array is only a stand-in for the symbol: its
// device address must be obtained with cudaGetSymbolAddress on each device.
static __device__ __align__(256) float g_bwd_dq_scratch[HSTU_BWD_NOALLOC_MAX_ELEMS];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  Outside a
// stream capture it is looked up on every call (cheap once the module is
// loaded), so a context that was torn down and created again (cudaDeviceReset)
// never leaves a stale address behind; during a capture, where the lookup
// could load the module, the address recorded by the last uncaptured call on
// this device is used.
int scratch_on_current_device(bool capturing, void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return HSTU_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return HSTU_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!capturing || g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_bwd_dq_scratch);
    if (e != cudaSuccess || p == nullptr) return HSTU_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return HSTU_OK;
}

}  // namespace

extern "C" int hstu_jagged_attn_bwd_noalloc(
    const void* q, const void* k, const void* v, const int64_t* seq_offsets, int64_t B,
    int64_t T, int64_t max_seq_len, const int64_t* timestamps, const float* w_pos, int64_t P,
    const float* w_ts, int64_t NB, int num_heads, int d_qk, int d_v, float scale,
    const void* dout, void* dq, void* dk, void* dv, float* dw_pos, float* dw_ts,
    int* dev_status, hstu_stream_t stream) {
  const int64_t need = hstu_jagged_attn_bwd_workspace_bytes(T, num_heads, d_qk);
  if (need < 0) return (int)need;
  const int64_t capacity = (int64_t)HSTU_BWD_NOALLOC_MAX_ELEMS * (int64_t)sizeof(float);
  if (need > capacity) return HSTU_ERR_WORKSPACE;
  // The scratch array used is the current device's copy, so the stream must
  // belong to the current device (kernels on another device's stream would
  // write that device's copy while the memset below clears this one).
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int dev = -1, sdev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaStreamGetDevice(s, &sdev) != cudaSuccess)
    return HSTU_ERR_CUDA;
  if (sdev != dev) return HSTU_ERR_UNSUPPORTED;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) return HSTU_ERR_CUDA;
  void* scratch = nullptr;
  const int st = scratch_on_current_device(cap != cudaStreamCaptureStatusNone, &scratch);
  if (st != HSTU_OK) return st;
  return hstu_jagged_attn_bwd(q, k, v, seq_offsets, B, T, max_seq_len, timestamps, w_pos, P,
                              w_ts, NB, num_heads, d_qk, d_v, scale, dout, dq, dk, dv, dw_pos,
                              dw_ts, scratch, capacity, dev_status, stream);
}
