// hstu_abi.cu -- the extern "C" entry points declared in include/hstu.h:
// host-side argument checks (no device synchronisation, the host never reads
// seq_offsets), then the launchers of the kernels in this directory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/hstu.h"
#include "internal.h"
#include "norm_gate.h"
#include "stochastic_length.h"

namespace hstu {

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

bool device_flag_set(DeviceFlags& f, int* slot) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *slot = -1;
    return false;
  }
  *slot = dev;
  return f.done[dev].load(std::memory_order_acquire);
}

void device_flag_mark(DeviceFlags& f, int slot) {
  if (slot >= 0 && slot < kMaxDevices) f.done[slot].store(true, std::memory_order_release);
}

namespace {
std::atomic<int64_t> g_launches{0};
}  // namespace

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;
}  // namespace

CUresult encode_tiled(CUtensorMap* map, CUtensorMapDataType dtype, cuuint32_t rank, void* gaddr,
                      const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
                      const cuuint32_t* estrides, CUtensorMapSwizzle swizzle) {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  if (g_encode == nullptr) return CUDA_ERROR_NOT_FOUND;
  return g_encode(map, dtype, rank, gaddr, dims, strides, box, estrides,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

}  // namespace hstu

namespace {

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

int check_attn_common(const void* q, const void* k, const void* v, const int64_t* offsets,
                      int64_t B, int64_t T, int64_t max_seq_len, const int64_t* ts,
                      const float* w_pos, int64_t P, const float* w_ts, int64_t NB, int H,
                      int d_qk, int d_v) {
  if (B < 0 || T < 0 || max_seq_len < 0 || T >= (int64_t)1 << 31) return HSTU_ERR_SHAPE;
  if (H < 1 || P < 1 || NB < 1) return HSTU_ERR_SHAPE;
  if (d_qk != d_v) return HSTU_ERR_UNSUPPORTED;
  if (d_qk != 32 && d_qk != 64 && d_qk != 128) return HSTU_ERR_UNSUPPORTED;
  if ((int64_t)H * d_qk * 2 >= ((int64_t)1 << 32)) return HSTU_ERR_SHAPE;
  if (offsets == nullptr) return HSTU_ERR_NULL;
  if (T == 0) return HSTU_OK;
  if (q == nullptr || k == nullptr || v == nullptr || ts == nullptr || w_pos == nullptr ||
      w_ts == nullptr)
    return HSTU_ERR_NULL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(ts, 8) ||
      !aligned(offsets, 8) || !aligned(w_pos, 4) || !aligned(w_ts, 4))
    return HSTU_ERR_ALIGN;
  return HSTU_OK;
}

// the CUDA error behind the last HSTU_ERR_CUDA returned on this host thread
thread_local cudaError_t t_last_cuda_error = cudaSuccess;

int from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return HSTU_OK;
  t_last_cuda_error = e;
  return HSTU_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* hstu_status_str(int status) {
  switch (status) {
    case HSTU_OK: return "HSTU_OK";
    case HSTU_ERR_NULL: return "HSTU_ERR_NULL: a required pointer is NULL";
    case HSTU_ERR_SHAPE: return "HSTU_ERR_SHAPE: bad or inconsistent size";
    case HSTU_ERR_ALIGN: return "HSTU_ERR_ALIGN: pointer not aligned as required";
    case HSTU_ERR_UNSUPPORTED: return "HSTU_ERR_UNSUPPORTED: unsupported head size or mode";
    case HSTU_ERR_OFFSETS: return "HSTU_ERR_OFFSETS: offsets decrease or offsets[B] != T";
    case HSTU_ERR_NOT_DIVISIBLE: return "HSTU_ERR_NOT_DIVISIBLE: length not a multiple of 2C";
    case HSTU_ERR_TIMEOUT: return "HSTU_ERR_TIMEOUT: a bounded wait inside a kernel gave up";
    case HSTU_ERR_CUDA: return "HSTU_ERR_CUDA: a CUDA call failed";
    case HSTU_ERR_WORKSPACE: return "HSTU_ERR_WORKSPACE: workspace missing or too small";
    default: return "unknown hstu status";
  }
}

const char* hstu_last_cuda_error(void) {
  return t_last_cuda_error == cudaSuccess ? "no CUDA error" : cudaGetErrorString(t_last_cuda_error);
}

int hstu_version(void) { return 100; }

int64_t hstu_kernel_launches(void) { return hstu::g_launches.load(std::memory_order_relaxed); }

int hstu_jagged_attn_fwd(const void* q, const void* k, const void* v,
                         const int64_t* seq_offsets, int64_t B, int64_t T, int64_t max_seq_len,
                         const int64_t* timestamps, const float* w_pos, int64_t P,
                         const float* w_ts, int64_t NB, int num_heads, int d_qk, int d_v,
                         float scale, int out_fp32, void* out, int* dev_status,
                         hstu_stream_t stream) {
  int st = check_attn_common(q, k, v, seq_offsets, B, T, max_seq_len, timestamps, w_pos, P, w_ts,
                             NB, num_heads, d_qk, d_v);
  if (st != HSTU_OK) return st;
  if (T == 0 || B == 0) return HSTU_OK;
  if (out == nullptr) return HSTU_ERR_NULL;
  if (!aligned(out, 16)) return HSTU_ERR_ALIGN;
  hstu::AttnArgs a = {};
  a.q = q; a.k = k; a.v = v;
  a.offsets = seq_offsets; a.B = B; a.T = T; a.max_seq_len = max_seq_len;
  a.ts = timestamps; a.w_pos = w_pos; a.P = P; a.w_ts = w_ts; a.NB = NB;
  a.H = num_heads; a.D = d_qk; a.scale = scale; a.C = 0; a.out_fp32 = out_fp32 ? 1 : 0;
  a.out = out; a.status = dev_status;
  return from_cuda(hstu::attn_fwd_launch(a, reinterpret_cast<cudaStream_t>(stream)));
}

int hstu_jagged_attn_fwd_targets(const void* q, const void* k, const void* v,
                                 const int64_t* seq_offsets, const int64_t* num_targets,
                                 int64_t B, int64_t T, int64_t max_seq_len,
                                 const int64_t* timestamps, const float* w_pos, int64_t P,
                                 const float* w_ts, int64_t NB, int num_heads, int d_qk,
                                 int d_v, float scale, int out_fp32, void* out,
                                 int* dev_status, hstu_stream_t stream) {
  int st = check_attn_common(q, k, v, seq_offsets, B, T, max_seq_len, timestamps, w_pos, P, w_ts,
                             NB, num_heads, d_qk, d_v);
  if (st != HSTU_OK) return st;
  if (T == 0 || B == 0) return HSTU_OK;
  if (out == nullptr || num_targets == nullptr) return HSTU_ERR_NULL;
  if (!aligned(out, 16) || !aligned(num_targets, 8)) return HSTU_ERR_ALIGN;
  if (P > hstu::attn_fwd_targets_max_P(d_qk)) return HSTU_ERR_UNSUPPORTED;
  hstu::AttnArgs a = {};
  a.q = q; a.k = k; a.v = v;
  a.offsets = seq_offsets; a.B = B; a.T = T; a.max_seq_len = max_seq_len;
  a.ts = timestamps; a.w_pos = w_pos; a.P = P; a.w_ts = w_ts; a.NB = NB;
  a.H = num_heads; a.D = d_qk; a.scale = scale; a.C = 0; a.out_fp32 = out_fp32 ? 1 : 0;
  a.out = out; a.status = dev_status; a.num_targets = num_targets;
  return from_cuda(hstu::attn_fwd_launch(a, reinterpret_cast<cudaStream_t>(stream)));
}

int hstu_jagged_attn_fwd_candidates(const void* q, const void* k, const void* v,
                                    const int64_t* seq_offsets, const int64_t* num_targets,
                                    int64_t B, int64_t T, int64_t max_seq_len,
                                    int64_t max_targets, const int64_t* timestamps,
                                    const float* w_pos, int64_t P, const float* w_ts, int64_t NB,
                                    int num_heads, int d_qk, int d_v, float scale, int out_fp32,
                                    void* out, int* dev_status, hstu_stream_t stream) {
  if (max_targets < 0) return HSTU_ERR_SHAPE;
  int st = check_attn_common(q, k, v, seq_offsets, B, T, max_seq_len, timestamps, w_pos, P, w_ts,
                             NB, num_heads, d_qk, d_v);
  if (st != HSTU_OK) return st;
  if (T == 0 || B == 0) return HSTU_OK;
  if (out == nullptr || num_targets == nullptr) return HSTU_ERR_NULL;
  if (!aligned(out, 16) || !aligned(num_targets, 8)) return HSTU_ERR_ALIGN;
  if (P > hstu::attn_fwd_targets_max_P(d_qk)) return HSTU_ERR_UNSUPPORTED;
  hstu::AttnArgs a = {};
  a.q = q; a.k = k; a.v = v;
  a.offsets = seq_offsets; a.B = B; a.T = T; a.max_seq_len = max_seq_len;
  a.ts = timestamps; a.w_pos = w_pos; a.P = P; a.w_ts = w_ts; a.NB = NB;
  a.H = num_heads; a.D = d_qk; a.scale = scale; a.C = 0; a.out_fp32 = out_fp32 ? 1 : 0;
  a.out = out; a.status = dev_status; a.num_targets = num_targets;
  a.cand_only = 1; a.max_targets = max_targets;
  return from_cuda(hstu::attn_fwd_launch(a, reinterpret_cast<cudaStream_t>(stream)));
}

int hstu_cp_paired_attn_fwd(const void* pq, const void* pk, const void* pv,
                            const int64_t* seq_offsets, int64_t B, int64_t T,
                            int64_t max_seq_len, int C, const int64_t* ptimestamps,
                            const float* w_pos, int64_t P, const float* w_ts, int64_t NB,
                            int num_heads, int d_qk, int d_v, float scale, int out_fp32,
                            void* out, int* dev_status, hstu_stream_t stream) {
  if (C < 1) return HSTU_ERR_SHAPE;
  int st = check_attn_common(pq, pk, pv, seq_offsets, B, T, max_seq_len, ptimestamps, w_pos, P,
                             w_ts, NB, num_heads, d_qk, d_v);
  if (st != HSTU_OK) return st;
  if (T == 0 || B == 0) return HSTU_OK;
  if (out == nullptr) return HSTU_ERR_NULL;
  if (!aligned(out, 16)) return HSTU_ERR_ALIGN;
  hstu::AttnArgs a = {};
  a.q = pq; a.k = pk; a.v = pv;
  a.offsets = seq_offsets; a.B = B; a.T = T; a.max_seq_len = max_seq_len;
  a.ts = ptimestamps; a.w_pos = w_pos; a.P = P; a.w_ts = w_ts; a.NB = NB;
  a.H = num_heads; a.D = d_qk; a.scale = scale; a.C = C; a.out_fp32 = out_fp32 ? 1 : 0;
  a.out = out; a.status = dev_status;
  return from_cuda(hstu::attn_fwd_launch(a, reinterpret_cast<cudaStream_t>(stream)));
}

int64_t hstu_jagged_attn_bwd_workspace_bytes(int64_t T, int num_heads, int d_qk) {
  if (T < 0 || num_heads < 1) return HSTU_ERR_SHAPE;
  if (d_qk != 32 && d_qk != 64 && d_qk != 128) return HSTU_ERR_UNSUPPORTED;
  const int64_t bytes = T * num_heads * d_qk * (int64_t)sizeof(float);
  return ((bytes + 255) / 256) * 256;
}

int hstu_jagged_attn_bwd(const void* q, const void* k, const void* v,
                         const int64_t* seq_offsets, int64_t B, int64_t T, int64_t max_seq_len,
                         const int64_t* timestamps, const float* w_pos, int64_t P,
                         const float* w_ts, int64_t NB, int num_heads, int d_qk, int d_v,
                         float scale, const void* dout, void* dq, void* dk, void* dv,
                         float* dw_pos, float* dw_ts, void* workspace, int64_t workspace_bytes,
                         int* dev_status, hstu_stream_t stream) {
  int st = check_attn_common(q, k, v, seq_offsets, B, T, max_seq_len, timestamps, w_pos, P, w_ts,
                             NB, num_heads, d_qk, d_v);
  if (st != HSTU_OK) return st;
  if (dw_pos == nullptr || dw_ts == nullptr) return HSTU_ERR_NULL;
  if (!aligned(dw_pos, 4) || !aligned(dw_ts, 4)) return HSTU_ERR_ALIGN;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // gradients of the bias tables are overwritten
  st = from_cuda(cudaMemsetAsync(dw_pos, 0, sizeof(float) * P, s));
  if (st != HSTU_OK) return st;
  st = from_cuda(cudaMemsetAsync(dw_ts, 0, sizeof(float) * NB, s));
  if (st != HSTU_OK) return st;
  if (T == 0 || B == 0) return HSTU_OK;
  if (dout == nullptr || dq == nullptr || dk == nullptr || dv == nullptr) return HSTU_ERR_NULL;
  if (!aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16))
    return HSTU_ERR_ALIGN;
  const int64_t need = hstu_jagged_attn_bwd_workspace_bytes(T, num_heads, d_qk);
  if (workspace == nullptr || workspace_bytes < need) return HSTU_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return HSTU_ERR_ALIGN;
  hstu::AttnArgs a = {};
  a.q = q; a.k = k; a.v = v;
  a.offsets = seq_offsets; a.B = B; a.T = T; a.max_seq_len = max_seq_len;
  a.ts = timestamps; a.w_pos = w_pos; a.P = P; a.w_ts = w_ts; a.NB = NB;
  a.H = num_heads; a.D = d_qk; a.scale = scale; a.C = 0;
  a.dout = dout; a.dq = dq; a.dk = dk; a.dv = dv; a.dw_pos = dw_pos; a.dw_ts = dw_ts;
  a.dq_accum = static_cast<float*>(workspace);
  a.status = dev_status;
  return from_cuda(hstu::attn_bwd_launch(a, s));
}

int hstu_cp_reorder(const void* src, void* dst, int64_t row_bytes, const int64_t* seq_offsets,
                    int64_t B, int64_t T, int C, int64_t* dst_offsets, int32_t* global_pos,
                    int* dev_status, hstu_stream_t stream) {
  if (C < 1 || B < 0 || T < 0 || row_bytes < 1 || T >= (int64_t)1 << 31) return HSTU_ERR_SHAPE;
  if (seq_offsets == nullptr) return HSTU_ERR_NULL;
  if (!aligned(seq_offsets, 8)) return HSTU_ERR_ALIGN;
  if (T > 0 && (src == nullptr || dst == nullptr)) return HSTU_ERR_NULL;
  if ((dst_offsets && !aligned(dst_offsets, 8)) || (global_pos && !aligned(global_pos, 4)))
    return HSTU_ERR_ALIGN;
  if (B == 0) return HSTU_OK;
  return from_cuda(hstu::cp_reorder_launch(src, dst, row_bytes, seq_offsets, B, T, C, dst_offsets,
                                           global_pos, dev_status,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

int hstu_cp_restore(const void* src, void* dst, int64_t row_bytes, const int64_t* seq_offsets,
                    int64_t B, int64_t T, int C, int* dev_status, hstu_stream_t stream) {
  if (C < 1 || B < 0 || T < 0 || row_bytes < 1 || T >= (int64_t)1 << 31) return HSTU_ERR_SHAPE;
  if (seq_offsets == nullptr) return HSTU_ERR_NULL;
  if (!aligned(seq_offsets, 8)) return HSTU_ERR_ALIGN;
  if (T > 0 && (src == nullptr || dst == nullptr)) return HSTU_ERR_NULL;
  if (B == 0) return HSTU_OK;
  return from_cuda(hstu::cp_restore_launch(src, dst, row_bytes, seq_offsets, B, T, C, dev_status,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

int hstu_bucket_indices(const int64_t* t_q, const int64_t* t_k, int64_t n, int64_t NB,
                        int32_t* buckets, hstu_stream_t stream) {
  if (n < 0 || NB < 1) return HSTU_ERR_SHAPE;
  if (n == 0) return HSTU_OK;
  if (t_q == nullptr || t_k == nullptr || buckets == nullptr) return HSTU_ERR_NULL;
  if (!aligned(t_q, 8) || !aligned(t_k, 8) || !aligned(buckets, 4)) return HSTU_ERR_ALIGN;
  return from_cuda(
      hstu::bucket_launch(t_q, t_k, n, NB, buckets, reinterpret_cast<cudaStream_t>(stream)));
}

namespace {
// checks shared by the two norm-gate entry points
int norm_gate_check(int64_t T, int64_t N, float eps) {
  if (T < 0 || N < 8 || N % 8 != 0) return HSTU_ERR_SHAPE;
  if (!(eps > 0.f) || !(eps < INFINITY)) return HSTU_ERR_SHAPE;
  if (N > 2048) return HSTU_ERR_UNSUPPORTED;
  if (T > (((int64_t)1 << 31) - 1) * 8) return HSTU_ERR_SHAPE;  // grid of T / 8 blocks
  return HSTU_OK;
}
// [a, a + n) and [b, b + n) share a byte
bool overlap(const void* a, const void* b, int64_t n) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + (uintptr_t)n && y < x + (uintptr_t)n;
}
}  // namespace

int hstu_norm_gate_fwd(const void* o, const void* u, void* y, int64_t T, int64_t N, float eps,
                       hstu_stream_t stream) {
  int st = norm_gate_check(T, N, eps);
  if (st != HSTU_OK) return st;
  if (T == 0) return HSTU_OK;
  if (o == nullptr || u == nullptr || y == nullptr) return HSTU_ERR_NULL;
  if (!aligned(o, 16) || !aligned(u, 16) || !aligned(y, 16)) return HSTU_ERR_ALIGN;
  const int64_t bytes = T * N * 2;
  if (overlap(y, o, bytes) || overlap(y, u, bytes)) return HSTU_ERR_SHAPE;
  return from_cuda(
      hstu::norm_gate_fwd_launch(o, u, y, T, N, eps, reinterpret_cast<cudaStream_t>(stream)));
}

int hstu_norm_gate_bwd(const void* o, const void* u, const void* dy, void* d_o, void* d_u,
                       int64_t T, int64_t N, float eps, hstu_stream_t stream) {
  int st = norm_gate_check(T, N, eps);
  if (st != HSTU_OK) return st;
  if (T == 0) return HSTU_OK;
  if (o == nullptr || u == nullptr || dy == nullptr || d_o == nullptr || d_u == nullptr)
    return HSTU_ERR_NULL;
  if (!aligned(o, 16) || !aligned(u, 16) || !aligned(dy, 16) || !aligned(d_o, 16) ||
      !aligned(d_u, 16))
    return HSTU_ERR_ALIGN;
  const int64_t bytes = T * N * 2;
  for (const void* out : {static_cast<const void*>(d_o), static_cast<const void*>(d_u)})
    if (overlap(out, o, bytes) || overlap(out, u, bytes) || overlap(out, dy, bytes))
      return HSTU_ERR_SHAPE;
  if (overlap(d_o, d_u, bytes)) return HSTU_ERR_SHAPE;
  return from_cuda(hstu::norm_gate_bwd_launch(o, u, dy, d_o, d_u, T, N, eps,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

int hstu_sl_select(const int64_t* seq_offsets, int64_t B, int64_t T, const uint32_t* u_tok,
                   const uint32_t* u_seq, int64_t L, int64_t* dst_offsets, int32_t* src_rows,
                   int* dev_status, hstu_stream_t stream) {
  if (B < 0 || T < 0 || T >= ((int64_t)1 << 31) || L < 1 || B >= ((int64_t)1 << 31))
    return HSTU_ERR_SHAPE;
  if (seq_offsets == nullptr || dst_offsets == nullptr) return HSTU_ERR_NULL;
  if (B > 0 && u_seq == nullptr) return HSTU_ERR_NULL;
  if (T > 0 && (u_tok == nullptr || src_rows == nullptr)) return HSTU_ERR_NULL;
  if (!aligned(seq_offsets, 8) || !aligned(dst_offsets, 8) || (u_tok && !aligned(u_tok, 4)) ||
      (u_seq && !aligned(u_seq, 4)) || (src_rows && !aligned(src_rows, 4)) ||
      (dev_status && !aligned(dev_status, 4)))
    return HSTU_ERR_ALIGN;
  return from_cuda(hstu::sl_select_launch(seq_offsets, B, T, u_tok, u_seq, L, dst_offsets,
                                          src_rows, dev_status,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

int hstu_gather_rows(const void* src, int64_t src_count, void* dst, int64_t row_bytes,
                     const int32_t* src_rows, const int64_t* n_rows, int64_t max_rows,
                     hstu_stream_t stream) {
  if (src_count < 0 || row_bytes < 1 || max_rows < 0 || max_rows >= ((int64_t)1 << 31))
    return HSTU_ERR_SHAPE;
  if (max_rows == 0) return HSTU_OK;
  if (src == nullptr || dst == nullptr || src_rows == nullptr || n_rows == nullptr)
    return HSTU_ERR_NULL;
  if (!aligned(src_rows, 4) || !aligned(n_rows, 8)) return HSTU_ERR_ALIGN;
  const uintptr_t s0 = reinterpret_cast<uintptr_t>(src), d0 = reinterpret_cast<uintptr_t>(dst);
  if (s0 < d0 + (uintptr_t)(max_rows * row_bytes) && d0 < s0 + (uintptr_t)(src_count * row_bytes))
    return HSTU_ERR_SHAPE;
  return from_cuda(hstu::gather_rows_launch(src, src_count, dst, row_bytes, src_rows, n_rows,
                                            max_rows, reinterpret_cast<cudaStream_t>(stream)));
}

int hstu_gather_rows_multi(int count, const void* const* srcs, void* const* dsts,
                           const int64_t* row_bytes, int64_t src_count, const int32_t* src_rows,
                           const int64_t* n_rows, int64_t max_rows, hstu_stream_t stream) {
  if (count < 1 || count > hstu::kMaxGatherTensors || src_count < 0 || max_rows < 0 ||
      max_rows >= ((int64_t)1 << 31))
    return HSTU_ERR_SHAPE;
  if (srcs == nullptr || dsts == nullptr || row_bytes == nullptr) return HSTU_ERR_NULL;
  if (max_rows == 0) return HSTU_OK;
  if (src_rows == nullptr || n_rows == nullptr) return HSTU_ERR_NULL;
  if (!aligned(src_rows, 4) || !aligned(n_rows, 8)) return HSTU_ERR_ALIGN;
  for (int t = 0; t < count; ++t) {
    if (row_bytes[t] < 1) return HSTU_ERR_SHAPE;
    if (srcs[t] == nullptr || dsts[t] == nullptr) return HSTU_ERR_NULL;
    const uintptr_t d0 = reinterpret_cast<uintptr_t>(dsts[t]);
    const uintptr_t dn = d0 + (uintptr_t)(max_rows * row_bytes[t]);
    for (int u = 0; u < count; ++u) {
      const uintptr_t s0 = reinterpret_cast<uintptr_t>(srcs[u]);
      if (s0 < dn && d0 < s0 + (uintptr_t)(src_count * row_bytes[u])) return HSTU_ERR_SHAPE;
    }
  }
  return from_cuda(hstu::gather_rows_multi_launch(count, srcs, dsts, row_bytes, src_count,
                                                  src_rows, n_rows, max_rows,
                                                  reinterpret_cast<cudaStream_t>(stream)));
}

int hstu_selftest_wait_timeout(int64_t limit_ns, int* dev_status, int* result,
                               hstu_stream_t stream) {
  if (limit_ns < 1000 || limit_ns > 1000000000) return HSTU_ERR_SHAPE;
  if (dev_status == nullptr || result == nullptr) return HSTU_ERR_NULL;
  if (!aligned(dev_status, 4) || !aligned(result, 4)) return HSTU_ERR_ALIGN;
  return from_cuda(hstu::wait_timeout_launch(limit_ns, dev_status, result,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
