// internal.h -- launchers shared between the libhstu translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace hstu {

// number of SMs of the current device (cached per device)
int num_sms();

// Per-device "done once" flags for launch attributes.  The dynamic shared
// memory opt-in (cudaFuncSetAttribute) belongs to the current device's
// context, so a kernel instance keeps one flag per device; setting it twice
// from racing host threads is harmless (the call is idempotent).
constexpr int kMaxDevices = 64;
struct DeviceFlags {
  std::atomic<bool> done[kMaxDevices];
};
// true when the flag of the current device is set; *slot receives the device
// index, or -1 when it is outside the table (then the caller sets the
// attribute on every launch)
bool device_flag_set(DeviceFlags& f, int* slot);
void device_flag_mark(DeviceFlags& f, int slot);

// count one kernel launch (read back through hstu_kernel_launches)
void count_launch();

// cuTensorMapEncodeTiled obtained through the runtime (no libcuda link)
CUresult encode_tiled(CUtensorMap* map, CUtensorMapDataType dtype, cuuint32_t rank, void* gaddr,
                      const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
                      const cuuint32_t* estrides, CUtensorMapSwizzle swizzle);

cudaError_t cp_reorder_launch(const void* src, void* dst, int64_t row_bytes,
                              const int64_t* offsets, int64_t B, int64_t T, int C,
                              int64_t* dst_offsets, int32_t* global_pos, int* status,
                              cudaStream_t stream);
cudaError_t cp_restore_launch(const void* src, void* dst, int64_t row_bytes,
                              const int64_t* offsets, int64_t B, int64_t T, int C, int* status,
                              cudaStream_t stream);
cudaError_t wait_timeout_launch(int64_t limit_ns, int* status, int* result, cudaStream_t stream);
cudaError_t bucket_launch(const int64_t* tq, const int64_t* tk, int64_t n, int64_t NB,
                          int32_t* out, cudaStream_t stream);

// Arguments of one attention call (forward or backward), already checked on
// the host.
struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  const int64_t* offsets;
  int64_t B;
  int64_t T;
  int64_t max_seq_len;
  const int64_t* ts;
  const float* w_pos;
  int64_t P;
  const float* w_ts;
  int64_t NB;
  int H;
  int D;
  float scale;
  int C;          // paired mode: number of virtual ranks (0 = plain jagged)
  int out_fp32;
  void* out;
  const int64_t* num_targets;  // forward, plain layout: candidates per sequence (or null)
  int cand_only;               // forward with num_targets: compute and write candidate rows only
  int64_t max_targets;         // cand_only: upper bound on num_targets[b] (0 = unknown)
  // backward only
  const void* dout;
  void* dq;
  void* dk;
  void* dv;
  float* dw_pos;
  float* dw_ts;
  float* dq_accum;  // fp32 [T, H, D] workspace
  int* status;
};

cudaError_t attn_fwd_launch(const AttnArgs& a, cudaStream_t stream);
// largest P the target-aware forward takes for head dimension D
int64_t attn_fwd_targets_max_P(int D);
cudaError_t attn_bwd_launch(const AttnArgs& a, cudaStream_t stream);

}  // namespace hstu
