// stochastic_length.cu -- Stochastic Length subsequence selection and the row
// gather that applies it ("Actions Speak Louder than Words", §3.2 and §4.2:
// subsequences of long histories raise sparsity; at alpha = 1.6 length-4096
// sequences become length 776 most of the time).
//
// Selection of sequence b (length n, target length L, the random draws are
// inputs): if n > L and u_seq[b] / 2^32 < 1 - (L / n)^2 (float64, in that
// order of operations), keep the L tokens with the smallest (u_tok, position)
// in position order; else keep all n.
//
//   sl_offsets_kernel : one block; the new lengths and their exclusive scan
//                       into dst_offsets[0 .. B].
//   sl_select_kernel  : one block per sequence; a cut sequence finds its L-th
//                       smallest key with a 4-pass, 8-bit radix select over
//                       u_tok, then writes the kept rows in order with block
//                       scans; a kept one writes o0 .. o1 - 1.
//   gather_rows_kernel: dst row r = src row src_rows[r], r < n_rows (read on
//                       the device), a group of lanes per row with the widest
//                       vector the row size and pointers allow.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"
#include "stochastic_length.h"

namespace hstu {

namespace {

constexpr int kSlThreads = 256;
constexpr int kScanThreads = 1024;

// a sequence the selection takes: offsets in range and non-decreasing
// (validate_offsets reports the others, and both kernels give them no rows)
__device__ __forceinline__ bool sl_valid(int64_t o0, int64_t o1, int64_t T) {
  return o0 >= 0 && o1 >= o0 && o1 <= T;
}

__device__ __forceinline__ bool sl_cut(int64_t n, int64_t L, uint32_t u) {
  if (n <= L) return false;
  const double frac = (double)L / (double)n;
  const double thresh = 1.0 - frac * frac;
  return (double)u / 4294967296.0 < thresh;
}

// exclusive block scan of one int per thread (blockDim.x = kSlThreads or
// kScanThreads, a multiple of 32); returns the block total in *total
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int w = lane < NT / 32 ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < NT / 32) s_warp[lane] = w;  // inclusive warp prefixes
  }
  __syncthreads();
  const int before = (wid > 0 ? s_warp[wid - 1] : 0) + x - v;
  *total = s_warp[NT / 32 - 1];
  __syncthreads();
  return before;
}

__global__ void __launch_bounds__(kScanThreads) sl_offsets_kernel(
    const int64_t* __restrict__ offsets, int64_t B, int64_t T,
    const uint32_t* __restrict__ u_seq, int64_t L, int64_t* __restrict__ dst_offsets,
    int* status) {
  __shared__ int s_warp[32];
  validate_offsets(offsets, B, T, 0, T, status);
  int64_t carry = 0;
  for (int64_t b0 = 0; b0 < B; b0 += kScanThreads) {
    const int64_t b = b0 + threadIdx.x;
    int len = 0;
    if (b < B) {
      const int64_t o0 = offsets[b], o1 = offsets[b + 1];
      if (sl_valid(o0, o1, T)) len = (int)(sl_cut(o1 - o0, L, u_seq[b]) ? L : o1 - o0);
    }
    int total;
    const int before = block_exclusive_scan<kScanThreads>(len, s_warp, &total);
    if (b < B) dst_offsets[b] = carry + before;
    carry += total;
  }
  if (threadIdx.x == 0) dst_offsets[B] = carry;
}

__global__ void __launch_bounds__(kSlThreads) sl_select_kernel(
    const int64_t* __restrict__ offsets, int64_t T,
    const uint32_t* __restrict__ u_tok, const uint32_t* __restrict__ u_seq, int64_t L,
    const int64_t* __restrict__ dst_offsets, int32_t* __restrict__ src_rows) {
  __shared__ int s_hist[256];
  __shared__ int s_warp[32];
  __shared__ uint32_t s_sel[2];  // chosen digit, elements below it
  const int b = blockIdx.x;
  const int64_t o0 = offsets[b], o1 = offsets[b + 1];
  const int64_t n = o1 - o0;
  if (!sl_valid(o0, o1, T) || n == 0) return;
  const int64_t dst0 = dst_offsets[b];
  if (!sl_cut(n, L, u_seq[b])) {
    for (int64_t i = threadIdx.x; i < n; i += kSlThreads) src_rows[dst0 + i] = (int32_t)(o0 + i);
    return;
  }
  // radix select: the k-th smallest u (k = L, 1-based) digit by digit
  uint32_t prefix = 0, mask = 0;
  int k = (int)L;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += kSlThreads) s_hist[i] = 0;
    __syncthreads();
    for (int64_t i = threadIdx.x; i < n; i += kSlThreads) {
      const uint32_t u = u_tok[o0 + i];
      if ((u & mask) == prefix) atomicAdd(&s_hist[(u >> shift) & 255u], 1);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // the digit whose cumulative count first reaches k (lanes own 8 bins each)
      int c[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = s_hist[threadIdx.x * 8 + j];
        sum += c[j];
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if ((int)threadIdx.x >= o) incl += y;
      }
      const int excl = incl - sum;
      if (excl < k && k <= incl) {
        int run = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (run < k && k <= run + c[j]) {
            s_sel[0] = threadIdx.x * 8 + j;
            s_sel[1] = (uint32_t)run;
          }
          run += c[j];
        }
      }
    }
    __syncthreads();
    prefix |= s_sel[0] << shift;
    mask |= 255u << shift;
    k -= (int)s_sel[1];
    __syncthreads();
  }
  // t = prefix: keep u < t, and the first k of the u == t in position order
  const uint32_t t = prefix;
  const int k_eq = k;
  int64_t kept_base = 0, eq_base = 0;
  for (int64_t c0 = 0; c0 < n; c0 += kSlThreads) {
    const int64_t i = c0 + threadIdx.x;
    const uint32_t u = i < n ? u_tok[o0 + i] : 0xffffffffu;
    const int is_eq = (i < n && u == t) ? 1 : 0;
    int eq_total;
    const int eq_before = block_exclusive_scan<kSlThreads>(is_eq, s_warp, &eq_total);
    const int keep = (i < n && (u < t || (is_eq && eq_base + eq_before < k_eq))) ? 1 : 0;
    int kept_total;
    const int kept_before = block_exclusive_scan<kSlThreads>(keep, s_warp, &kept_total);
    if (keep) src_rows[dst0 + kept_base + kept_before] = (int32_t)(o0 + i);
    kept_base += kept_total;
    eq_base += eq_total;
  }
}

template <typename V>
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint8_t* __restrict__ src,
                                                          int64_t src_count,
                                                          uint8_t* __restrict__ dst,
                                                          int64_t row_bytes,
                                                          const int32_t* __restrict__ src_rows,
                                                          const int64_t* __restrict__ n_rows_dev,
                                                          int64_t max_rows, int group) {
  int64_t n_rows = *n_rows_dev;
  n_rows = n_rows < 0 ? 0 : imin64(n_rows, max_rows);
  const int64_t vecs = row_bytes / (int64_t)sizeof(V);
  const int64_t groups_total = (int64_t)gridDim.x * (blockDim.x / group);
  const int g_in_block = threadIdx.x / group, gl = threadIdx.x % group;
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x / group) + g_in_block; r < n_rows;
       r += groups_total) {
    const int64_t sr = src_rows[r];
    if (sr < 0 || sr >= src_count) continue;  // never read outside src
    const V* s = reinterpret_cast<const V*>(src + sr * row_bytes);
    V* d = reinterpret_cast<V*>(dst + r * row_bytes);
    for (int64_t v = gl; v < vecs; v += group) d[v] = s[v];
  }
}

template <typename V>
cudaError_t launch_gather(const void* src, int64_t src_count, void* dst, int64_t row_bytes,
                          const int32_t* src_rows, const int64_t* n_rows, int64_t max_rows,
                          cudaStream_t stream) {
  const int64_t vecs = row_bytes / (int64_t)sizeof(V);
  int group = 32;
  while (group > 1 && group / 2 >= vecs) group >>= 1;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, gather_rows_kernel<V>, 256, 0) !=
          cudaSuccess ||
      occ < 1)
    occ = 1;
  int64_t blocks = (max_rows + (256 / group) - 1) / (256 / group);
  const int64_t cap = (int64_t)num_sms() * occ;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  count_launch();
  gather_rows_kernel<V><<<(unsigned)blocks, 256, 0, stream>>>(
      static_cast<const uint8_t*>(src), src_count, static_cast<uint8_t*>(dst), row_bytes,
      src_rows, n_rows, max_rows, group);
  return cudaGetLastError();
}

// Several tensors of the same rows in one launch: group g of lanes copies row
// r of tensor t for every (r, t) it owns, with tensor t's own vector width.
struct MultiRows {
  const uint8_t* src[kMaxGatherTensors];
  uint8_t* dst[kMaxGatherTensors];
  int64_t row_bytes[kMaxGatherTensors];
  int width[kMaxGatherTensors];  // bytes per access: 16, 8, 4, 2 or 1
  int count;
};

template <typename V>
__device__ __forceinline__ void copy_row(const uint8_t* s, uint8_t* d, int64_t bytes, int gl,
                                         int group) {
  const V* sv = reinterpret_cast<const V*>(s);
  V* dv = reinterpret_cast<V*>(d);
  for (int64_t v = gl; v < bytes / (int64_t)sizeof(V); v += group) dv[v] = sv[v];
}

__global__ void __launch_bounds__(256) gather_rows_multi_kernel(
    const MultiRows m, int64_t src_count, const int32_t* __restrict__ src_rows,
    const int64_t* __restrict__ n_rows_dev, int64_t max_rows) {
  constexpr int group = 16;
  int64_t n_rows = *n_rows_dev;
  n_rows = n_rows < 0 ? 0 : imin64(n_rows, max_rows);
  const int64_t groups_total = (int64_t)gridDim.x * (blockDim.x / group);
  const int gl = threadIdx.x % group;
  const int64_t units = n_rows * m.count;
  for (int64_t u = (int64_t)blockIdx.x * (blockDim.x / group) + threadIdx.x / group; u < units;
       u += groups_total) {
    const int64_t r = u / m.count;
    const int t = (int)(u - r * m.count);
    const int64_t sr = src_rows[r];
    if (sr < 0 || sr >= src_count) continue;  // never read outside src
    const int64_t rb = m.row_bytes[t];
    const uint8_t* sp = m.src[t] + sr * rb;
    uint8_t* dp = m.dst[t] + r * rb;
    switch (m.width[t]) {
      case 16: copy_row<uint4>(sp, dp, rb, gl, group); break;
      case 8: copy_row<uint2>(sp, dp, rb, gl, group); break;
      case 4: copy_row<uint32_t>(sp, dp, rb, gl, group); break;
      case 2: copy_row<uint16_t>(sp, dp, rb, gl, group); break;
      default: copy_row<uint8_t>(sp, dp, rb, gl, group); break;
    }
  }
}

}  // namespace

cudaError_t gather_rows_multi_launch(int count, const void* const* srcs, void* const* dsts,
                                     const int64_t* row_bytes, int64_t src_count,
                                     const int32_t* src_rows, const int64_t* n_rows,
                                     int64_t max_rows, cudaStream_t stream) {
  MultiRows m;
  m.count = count;
  for (int t = 0; t < count; ++t) {
    m.src[t] = static_cast<const uint8_t*>(srcs[t]);
    m.dst[t] = static_cast<uint8_t*>(dsts[t]);
    m.row_bytes[t] = row_bytes[t];
    const uintptr_t a = reinterpret_cast<uintptr_t>(srcs[t]) |
                        reinterpret_cast<uintptr_t>(dsts[t]) | static_cast<uintptr_t>(row_bytes[t]);
    m.width[t] = (a & 15) == 0 ? 16 : (a & 7) == 0 ? 8 : (a & 3) == 0 ? 4 : (a & 1) == 0 ? 2 : 1;
  }
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, gather_rows_multi_kernel, 256, 0) !=
          cudaSuccess ||
      occ < 1)
    occ = 1;
  int64_t blocks = (max_rows * count + 15) / 16;
  const int64_t cap = (int64_t)num_sms() * occ;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  count_launch();
  gather_rows_multi_kernel<<<(unsigned)blocks, 256, 0, stream>>>(m, src_count, src_rows, n_rows,
                                                                  max_rows);
  return cudaGetLastError();
}

cudaError_t sl_select_launch(const int64_t* offsets, int64_t B, int64_t T,
                             const uint32_t* u_tok, const uint32_t* u_seq, int64_t L,
                             int64_t* dst_offsets, int32_t* src_rows, int* status,
                             cudaStream_t stream) {
  count_launch();
  sl_offsets_kernel<<<1, kScanThreads, 0, stream>>>(offsets, B, T, u_seq, L, dst_offsets, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || B == 0) return e;
  count_launch();
  sl_select_kernel<<<(unsigned)B, kSlThreads, 0, stream>>>(offsets, T, u_tok, u_seq, L,
                                                          dst_offsets, src_rows);
  return cudaGetLastError();
}

cudaError_t gather_rows_launch(const void* src, int64_t src_count, void* dst, int64_t row_bytes,
                               const int32_t* src_rows, const int64_t* n_rows, int64_t max_rows,
                               cudaStream_t stream) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst) |
                      static_cast<uintptr_t>(row_bytes);
  if ((a & 15) == 0)
    return launch_gather<uint4>(src, src_count, dst, row_bytes, src_rows, n_rows, max_rows, stream);
  if ((a & 7) == 0)
    return launch_gather<uint2>(src, src_count, dst, row_bytes, src_rows, n_rows, max_rows, stream);
  if ((a & 3) == 0)
    return launch_gather<uint32_t>(src, src_count, dst, row_bytes, src_rows, n_rows, max_rows,
                                   stream);
  if ((a & 1) == 0)
    return launch_gather<uint16_t>(src, src_count, dst, row_bytes, src_rows, n_rows, max_rows,
                                   stream);
  return launch_gather<uint8_t>(src, src_count, dst, row_bytes, src_rows, n_rows, max_rows, stream);
}

}  // namespace hstu
