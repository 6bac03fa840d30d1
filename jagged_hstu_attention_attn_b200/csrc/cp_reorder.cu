// cp_reorder.cu -- load-balanced mini-chunk pairing as a single-GPU jagged
// permutation ("Scaling Generative Recommendations with Context Parallelism
// on Hierarchical Sequential Transducers", §2.3, figure "Load Balanced CP
// with 2*CP_size Mini-chunks": mini-chunks (r, 2C-1-r) go to rank r).
//
// Paired layout: rank-major, then sequence, then [chunk r rows, chunk 2C-1-r
// rows].  With m_b = L_b / 2C and TC = T / C rows per rank, original local
// row p of sequence b (chunk c = p / m_b, u = p % m_b) lands at
//     r = c < C ? c : 2C-1-c,  half = c >= C,
//     paired_row = r * TC + offsets[b] / C + half * m_b + u.
// Both directions iterate over SOURCE rows (original rows for the reorder,
// paired rows for the restore): every chunk is a contiguous run on both sides,
// so both sides are coalesced, and a source row below T is always a valid
// address, so its loads are issued before its destination is known.  The
// restore inverts the map: rank r = q / TC, q' = q - r TC, the sequence is the
// one with offsets[b] / C <= q' < offsets[b+1] / C, u2 = q' - offsets[b] / C,
// half = u2 >= m_b, chunk = half ? 2C-1-r : r.
// Each row is moved by a group of G lanes with the widest vector type the row
// size and the two base pointers allow (16 B for q/k/v rows).
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace hstu {

namespace {

constexpr int kCpThreads = 256;
constexpr int kCpSmemOffsets = 2048;  // offsets cached in smem when B + 1 <= this

// largest b with off[b] <= t (sequences with equal offsets are empty; the
// search lands on the last of them, which is the one holding t)
__device__ __forceinline__ int find_seq(const int64_t* off, int B, int64_t t) {
  int lo = 0, hi = B;  // invariant: off[lo] <= t, answer in [lo, hi)
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (off[mid] <= t) lo = mid; else hi = mid;
  }
  return lo;
}

template <typename V, bool RESTORE>
__global__ void __launch_bounds__(kCpThreads) cp_permute_kernel(
    const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, int64_t row_bytes,
    const int64_t* __restrict__ offsets, int B, int64_t T, int C, int group,
    int64_t* __restrict__ dst_offsets, int32_t* __restrict__ global_pos, int* status) {
  __shared__ int64_t s_off[kCpSmemOffsets];
  const bool cached = (B + 1) <= kCpSmemOffsets;
  if (cached) {
    for (int i = threadIdx.x; i <= B; i += blockDim.x) s_off[i] = offsets[i];
    __syncthreads();
  }
  const int64_t* off = cached ? s_off : offsets;
  const int64_t twoC = 2 * (int64_t)C;
  const int64_t TC = T / C;

  // block 0: global validation + the dst_offsets table (rank-major segments)
  if (blockIdx.x == 0) {
    if (threadIdx.x == 0 && (off[0] != 0 || off[B] != T)) report(status, HSTU_ERR_OFFSETS);
    for (int b = threadIdx.x; b < B; b += blockDim.x) {
      int64_t L = off[b + 1] - off[b];
      if (L < 0) report(status, HSTU_ERR_OFFSETS);
      else if (L % twoC != 0) report(status, HSTU_ERR_NOT_DIVISIBLE);
    }
    if (!RESTORE && dst_offsets != nullptr) {
      for (int64_t i = threadIdx.x; i < (int64_t)C * B; i += blockDim.x) {
        int64_t r = i / B, b = i % B;
        dst_offsets[i] = r * TC + off[b] / C;
      }
      if (threadIdx.x == 0) dst_offsets[(int64_t)C * B] = T;
    }
  }

  const int64_t nvec = row_bytes / (int64_t)sizeof(V);
  const int lane_in_group = threadIdx.x % group;
  const int64_t groups_per_block = blockDim.x / group;
  const int64_t gid0 = (int64_t)blockIdx.x * groups_per_block + threadIdx.x / group;
  const int64_t gstride = (int64_t)gridDim.x * groups_per_block;

  // Each group moves kRows consecutive source rows per trip: every load
  // first, then the destination of each row (while the loads are in flight),
  // then every store, so a lane has 2 * kRows vectors in flight.
  constexpr int kRows = 4;
  const bool small = T < 0x7fffffffLL;
  const bool fast = nvec == 2 * group;  // the common case: two vectors per lane per row
  int b = 0;
  for (int64_t t0 = gid0 * kRows; t0 < T; t0 += gstride * kRows) {
    V v[kRows][2];
    if (fast) {
#pragma unroll
      for (int j = 0; j < kRows; ++j)
        if (t0 + j < T) {
          const V* sp = reinterpret_cast<const V*>(src + (t0 + j) * row_bytes);
          v[j][0] = __ldg(sp + lane_in_group);
          v[j][1] = __ldg(sp + lane_in_group + group);
        }
    }
    int64_t drow[kRows];
    // RESTORE: rank of the first row, then stepped forward
    int64_t r = 0, rstart = 0;
    if (RESTORE && TC > 0) {
      r = small ? (int64_t)((uint32_t)t0 / (uint32_t)TC) : t0 / TC;
      rstart = r * TC;
    }
#pragma unroll
    for (int j = 0; j < kRows; ++j) {
      const int64_t t = t0 + j;
      drow[j] = -1;
      if (t >= T) continue;
      int64_t key;  // compared against the original offsets
      if (RESTORE) {
        if (TC <= 0) continue;  // T < C: the offsets are flagged above
        while (t >= rstart + TC) { ++r; rstart += TC; }
        if (r >= C) continue;   // T not a multiple of C (flagged above)
        key = (t - rstart) * C;
      } else {
        key = t;
      }
      if (j == 0 || key < off[b]) b = find_seq(off, B, key);
      while (b + 1 < B && off[b + 1] <= key) ++b;  // next non-empty sequence
      const int64_t o = off[b];
      const int64_t L = off[b + 1] - o;
      if (L <= 0 || L % twoC != 0 || off[b + 1] > T || o < 0) continue;  // flagged above
      const int64_t m = L / twoC;
      if (RESTORE) {
        const int64_t u2 = t - rstart - o / C;
        if (u2 < 0 || u2 >= 2 * m) continue;  // only with non-monotone offsets (flagged)
        const int64_t half = u2 >= m ? 1 : 0;
        const int64_t c = half ? twoC - 1 - r : r;
        drow[j] = o + c * m + (u2 - half * m);
      } else {
        const int64_t p = key - o;
        if (p < 0 || p >= L) continue;  // only with non-monotone offsets (flagged)
        int64_t c, u;
        if (L < 0x7fffffffLL) {
          const uint32_t pp = (uint32_t)p, mm = (uint32_t)m;
          const uint32_t cc = pp / mm;
          c = cc;
          u = pp - cc * mm;
        } else {
          c = p / m;
          u = p - c * m;
        }
        const int64_t rr = c < C ? c : twoC - 1 - c;
        const int64_t half = c >= C ? 1 : 0;
        drow[j] = rr * TC + o / C + half * m + u;
        if (global_pos != nullptr && lane_in_group == 0) global_pos[drow[j]] = (int32_t)p;
      }
    }
    if (fast) {
#pragma unroll
      for (int j = 0; j < kRows; ++j)
        if (drow[j] >= 0) {
          V* dp = reinterpret_cast<V*>(dst + drow[j] * row_bytes);
          dp[lane_in_group] = v[j][0];
          dp[lane_in_group + group] = v[j][1];
        }
    } else {
#pragma unroll
      for (int j = 0; j < kRows; ++j)
        if (drow[j] >= 0) {
          const V* sp = reinterpret_cast<const V*>(src + (t0 + j) * row_bytes);
          V* dp = reinterpret_cast<V*>(dst + drow[j] * row_bytes);
          for (int64_t i = lane_in_group; i < nvec; i += group) dp[i] = __ldg(sp + i);
        }
    }
  }
}

template <typename V, bool RESTORE>
cudaError_t launch_cp(const void* src, void* dst, int64_t row_bytes, const int64_t* offsets,
                      int64_t B, int64_t T, int C, int64_t* dst_offsets, int32_t* global_pos,
                      int* status, cudaStream_t stream) {
  int64_t nvec = row_bytes / (int64_t)sizeof(V);
  int group = 1;
  while (group < 32 && group * 2 <= nvec) group *= 2;
  int64_t groups_per_block = kCpThreads / group;
  int64_t blocks = (T + 4 * groups_per_block - 1) / (4 * groups_per_block);
  // one wave: as many blocks as fit on the SMs at once (the grid-stride loop
  // covers the rest), so no second, partly filled wave ends the launch
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, cp_permute_kernel<V, RESTORE>,
                                                    kCpThreads, 0) != cudaSuccess ||
      occ < 1)
    occ = 1;
  int64_t max_blocks = (int64_t)num_sms() * occ;
  if (blocks > max_blocks) blocks = max_blocks;
  if (blocks < 1) blocks = 1;
  count_launch();
  cp_permute_kernel<V, RESTORE><<<(unsigned)blocks, kCpThreads, 0, stream>>>(
      static_cast<const uint8_t*>(src), static_cast<uint8_t*>(dst), row_bytes, offsets, (int)B,
      T, C, group, dst_offsets, global_pos, status);
  return cudaGetLastError();
}

template <bool RESTORE>
cudaError_t dispatch_cp(const void* src, void* dst, int64_t row_bytes, const int64_t* offsets,
                        int64_t B, int64_t T, int C, int64_t* dst_offsets, int32_t* global_pos,
                        int* status, cudaStream_t stream) {
  uintptr_t a = reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst) |
                static_cast<uintptr_t>(row_bytes);
  if ((a & 15) == 0)
    return launch_cp<uint4, RESTORE>(src, dst, row_bytes, offsets, B, T, C, dst_offsets,
                                     global_pos, status, stream);
  if ((a & 7) == 0)
    return launch_cp<uint2, RESTORE>(src, dst, row_bytes, offsets, B, T, C, dst_offsets,
                                     global_pos, status, stream);
  if ((a & 3) == 0)
    return launch_cp<uint32_t, RESTORE>(src, dst, row_bytes, offsets, B, T, C, dst_offsets,
                                        global_pos, status, stream);
  if ((a & 1) == 0)
    return launch_cp<uint16_t, RESTORE>(src, dst, row_bytes, offsets, B, T, C, dst_offsets,
                                        global_pos, status, stream);
  return launch_cp<uint8_t, RESTORE>(src, dst, row_bytes, offsets, B, T, C, dst_offsets,
                                     global_pos, status, stream);
}

}  // namespace

cudaError_t cp_reorder_launch(const void* src, void* dst, int64_t row_bytes,
                              const int64_t* offsets, int64_t B, int64_t T, int C,
                              int64_t* dst_offsets, int32_t* global_pos, int* status,
                              cudaStream_t stream) {
  return dispatch_cp<false>(src, dst, row_bytes, offsets, B, T, C, dst_offsets, global_pos,
                            status, stream);
}

cudaError_t cp_restore_launch(const void* src, void* dst, int64_t row_bytes,
                              const int64_t* offsets, int64_t B, int64_t T, int C, int* status,
                              cudaStream_t stream) {
  return dispatch_cp<true>(src, dst, row_bytes, offsets, B, T, C, nullptr, nullptr, status,
                           stream);
}

// ---------------------------------------------------------------------------
// bucket debug kernel (parity of the integer bucket function)
// ---------------------------------------------------------------------------
namespace {
__global__ void bucket_kernel(const int64_t* __restrict__ tq, const int64_t* __restrict__ tk,
                              int64_t n, int nbm1, int32_t* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    out[i] = bucket_of(tq[i], tk[i], nbm1);
}
}  // namespace

cudaError_t bucket_launch(const int64_t* tq, const int64_t* tk, int64_t n, int64_t NB,
                          int32_t* out, cudaStream_t stream) {
  int64_t blocks = (n + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  if (blocks < 1) blocks = 1;
  int nbm1 = NB - 1 > 0x7fffffff ? 0x7fffffff : (int)(NB - 1);
  count_launch();
  bucket_kernel<<<(unsigned)blocks, 256, 0, stream>>>(tq, tk, n, nbm1, out);
  return cudaGetLastError();
}

}  // namespace hstu
