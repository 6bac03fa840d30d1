// norm_gate.cu -- the HSTU layer's step after attention, Y = Norm(A(X)V(X)) ⊙ U(X)
// ("Actions Speak Louder than Words", §3, Pointwise Transformation), and its
// backward.  Norm is a layer normalisation without a learned affine over the
// N = H·d features of each token (all heads' attention outputs together),
// with the biased variance and eps inside the square root:
//     y = (o - mean) rstd ⊙ u,  rstd = 1 / sqrt(var + eps).
// Backward, with x̂ = (o - mean) rstd and g = dy ⊙ u:
//     du = x̂ ⊙ dy,  do = rstd (g - mean(g) - x̂ mean(g ⊙ x̂)).
//
// Both directions are HBM-bound streams over [T, N] bf16 rows: one warp per
// row, each lane holding VPL 16-byte vectors (8 bf16) of it in registers, so a
// row is read from HBM once and the statistics (two-pass: mean, then the sum
// of squared deviations) come from registers.  All of a row's loads are issued
// before the first reduction.  Arithmetic in fp32; outputs rounded to bf16.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"
#include "norm_gate.h"

namespace hstu {

namespace {

constexpr int kNgThreads = 256;
constexpr int kNgWarps = kNgThreads / 32;

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  f[0] = bf16lo_to_f32(v.x); f[1] = bf16hi_to_f32(v.x);
  f[2] = bf16lo_to_f32(v.y); f[3] = bf16hi_to_f32(v.y);
  f[4] = bf16lo_to_f32(v.z); f[5] = bf16hi_to_f32(v.z);
  f[6] = bf16lo_to_f32(v.w); f[7] = bf16hi_to_f32(v.w);
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// read-only streaming load (the rows are read once)
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Row statistics from the lane's vectors: mean, then rstd from the sum of
// squared deviations.  Lanes without a vector j hold zeros there and are
// excluded from the deviations.
template <int VPL>
__device__ __forceinline__ void row_stats(const float (&x)[VPL][8], const bool (&has)[VPL],
                                          float inv_n, float eps, float& mean, float& rstd) {
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < VPL; ++j)
#pragma unroll
    for (int e = 0; e < 8; ++e) s += x[j][e];
  mean = warp_sum(s) * inv_n;
  float q = 0.f;
#pragma unroll
  for (int j = 0; j < VPL; ++j)
    if (has[j])
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float c = x[j][e] - mean;
        q = fmaf(c, c, q);
      }
  rstd = rsqrtf(warp_sum(q) * inv_n + eps);
}

template <int VPL>
__global__ void __launch_bounds__(kNgThreads) norm_gate_fwd_kernel(
    const uint4* __restrict__ o, const uint4* __restrict__ u, uint4* __restrict__ y, int64_t T,
    int nvec, float inv_n, float eps) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kNgWarps + (threadIdx.x >> 5);
  if (row >= T) return;
  const int64_t base = row * nvec;
  uint4 ov[VPL], uv[VPL];
  bool has[VPL];
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    const int c = lane + 32 * j;
    has[j] = c < nvec;
    ov[j] = has[j] ? ld_stream(o + base + c) : make_uint4(0, 0, 0, 0);
    uv[j] = has[j] ? ld_stream(u + base + c) : make_uint4(0, 0, 0, 0);
  }
  float x[VPL][8];
#pragma unroll
  for (int j = 0; j < VPL; ++j) unpack8(ov[j], x[j]);
  float mean, rstd;
  row_stats<VPL>(x, has, inv_n, eps, mean, rstd);
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    if (!has[j]) continue;
    float g[8], r[8];
    unpack8(uv[j], g);
#pragma unroll
    for (int e = 0; e < 8; ++e) r[e] = (x[j][e] - mean) * rstd * g[e];
    y[base + lane + 32 * j] = pack8(r);
  }
}

template <int VPL>
__global__ void __launch_bounds__(kNgThreads) norm_gate_bwd_kernel(
    const uint4* __restrict__ o, const uint4* __restrict__ u, const uint4* __restrict__ dy,
    uint4* __restrict__ d_o, uint4* __restrict__ d_u, int64_t T, int nvec, float inv_n,
    float eps) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kNgWarps + (threadIdx.x >> 5);
  if (row >= T) return;
  const int64_t base = row * nvec;
  uint4 ov[VPL], uv[VPL], dv[VPL];
  bool has[VPL];
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    const int c = lane + 32 * j;
    has[j] = c < nvec;
    ov[j] = has[j] ? ld_stream(o + base + c) : make_uint4(0, 0, 0, 0);
    uv[j] = has[j] ? ld_stream(u + base + c) : make_uint4(0, 0, 0, 0);
    dv[j] = has[j] ? ld_stream(dy + base + c) : make_uint4(0, 0, 0, 0);
  }
  float x[VPL][8];
#pragma unroll
  for (int j = 0; j < VPL; ++j) unpack8(ov[j], x[j]);
  float mean, rstd;
  row_stats<VPL>(x, has, inv_n, eps, mean, rstd);
  // x̂ replaces x; g = dy ⊙ u is formed again from the packed inputs below
  float sg = 0.f, sgx = 0.f;
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    float uu[8], dd[8], du[8];
    unpack8(uv[j], uu);
    unpack8(dv[j], dd);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      x[j][e] = has[j] ? (x[j][e] - mean) * rstd : 0.f;
      const float g = dd[e] * uu[e];
      sg += g;
      sgx = fmaf(g, x[j][e], sgx);
      du[e] = x[j][e] * dd[e];
    }
    if (has[j]) d_u[base + lane + 32 * j] = pack8(du);
  }
  const float mg = warp_sum(sg) * inv_n;
  const float mgx = warp_sum(sgx) * inv_n;
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    if (!has[j]) continue;
    float uu[8], dd[8], r[8];
    unpack8(uv[j], uu);
    unpack8(dv[j], dd);
#pragma unroll
    for (int e = 0; e < 8; ++e) r[e] = rstd * (dd[e] * uu[e] - mg - x[j][e] * mgx);
    d_o[base + lane + 32 * j] = pack8(r);
  }
}

int vectors_per_lane(int64_t N) {
  const int64_t nvec = N / 8;
  return nvec <= 32 ? 1 : nvec <= 64 ? 2 : nvec <= 128 ? 4 : 8;
}

unsigned ng_blocks(int64_t T) { return (unsigned)((T + kNgWarps - 1) / kNgWarps); }

}  // namespace

cudaError_t norm_gate_fwd_launch(const void* o, const void* u, void* y, int64_t T, int64_t N,
                                 float eps, cudaStream_t stream) {
  const int nvec = (int)(N / 8);
  const float inv_n = 1.0f / (float)N;
  const uint4* o4 = static_cast<const uint4*>(o);
  const uint4* u4 = static_cast<const uint4*>(u);
  uint4* y4 = static_cast<uint4*>(y);
  count_launch();
  switch (vectors_per_lane(N)) {
    case 1: norm_gate_fwd_kernel<1><<<ng_blocks(T), kNgThreads, 0, stream>>>(o4, u4, y4, T, nvec, inv_n, eps); break;
    case 2: norm_gate_fwd_kernel<2><<<ng_blocks(T), kNgThreads, 0, stream>>>(o4, u4, y4, T, nvec, inv_n, eps); break;
    case 4: norm_gate_fwd_kernel<4><<<ng_blocks(T), kNgThreads, 0, stream>>>(o4, u4, y4, T, nvec, inv_n, eps); break;
    default: norm_gate_fwd_kernel<8><<<ng_blocks(T), kNgThreads, 0, stream>>>(o4, u4, y4, T, nvec, inv_n, eps); break;
  }
  return cudaGetLastError();
}

cudaError_t norm_gate_bwd_launch(const void* o, const void* u, const void* dy, void* d_o,
                                 void* d_u, int64_t T, int64_t N, float eps,
                                 cudaStream_t stream) {
  const int nvec = (int)(N / 8);
  const float inv_n = 1.0f / (float)N;
  const uint4* o4 = static_cast<const uint4*>(o);
  const uint4* u4 = static_cast<const uint4*>(u);
  const uint4* dy4 = static_cast<const uint4*>(dy);
  uint4* do4 = static_cast<uint4*>(d_o);
  uint4* du4 = static_cast<uint4*>(d_u);
  count_launch();
  switch (vectors_per_lane(N)) {
    case 1: norm_gate_bwd_kernel<1><<<ng_blocks(T), kNgThreads, 0, stream>>>(o4, u4, dy4, do4, du4, T, nvec, inv_n, eps); break;
    case 2: norm_gate_bwd_kernel<2><<<ng_blocks(T), kNgThreads, 0, stream>>>(o4, u4, dy4, do4, du4, T, nvec, inv_n, eps); break;
    case 4: norm_gate_bwd_kernel<4><<<ng_blocks(T), kNgThreads, 0, stream>>>(o4, u4, dy4, do4, du4, T, nvec, inv_n, eps); break;
    default: norm_gate_bwd_kernel<8><<<ng_blocks(T), kNgThreads, 0, stream>>>(o4, u4, dy4, do4, du4, T, nvec, inv_n, eps); break;
  }
  return cudaGetLastError();
}

}  // namespace hstu
