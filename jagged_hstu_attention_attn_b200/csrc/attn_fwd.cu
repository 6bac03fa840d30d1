// attn_fwd.cu -- jagged HSTU pointwise attention, forward, for sm_100a.
//
//   O = Mask( SiLU( scale (Q K^T + Bias) ) ) V,
//   Bias[i,j] = w_pos[min(i-j, P-1)] + w_ts[bucket(t_i - t_j)]
// ("Scaling Generative Recommendations with Context Parallelism on
// Hierarchical Sequential Transducers", §2.1; pointwise aggregation without
// softmax: "Actions Speak Louder than Words", §3.1; relative attention bias:
// same paper, App. F.3).
//
// One CTA computes one (query tile of 128 rows, head) work item of one
// sequence and walks its key tiles j_tile <= i_tile (causal tile skipping on
// the jagged offsets, the "fully ragged" scheduling of the HSTU paper §3.2).
// Warp roles (224 threads):
//   warps 0-3 : epilogue.  Thread r owns query row r = TMEM lane r.  Reads the
//               fp32 S tile from TMEM, adds the gathered bias, applies scale,
//               SiLU (tanh.approx) and the causal / ragged mask, and writes P
//               back into TMEM as bf16 hi + lo parts (P = hi + lo to ~2^-17).
//   warp 4    : TMA producer for the Q tile and the K / V tile ring.
//   warp 5    : TMEM allocator and single-thread tcgen05.mma issuer:
//               S_n = Q K_n^T (SS form) into one of two TMEM S buffers, then
//               O += P_hi V_n + P_lo V_n (TS form, P read from TMEM).
//   warp 6    : per-tile metadata: key timestamps, the monotone flag used by
//               the uniform-bucket fast path, and the relative-position bias
//               window for the tile.
// There is no softmax, so there is no running max / sum and no rescaling of
// the O accumulator: O lives in TMEM for the whole CTA.
//
// TMEM columns (512 allocated): S0 [0,128) S1 [128,256) O [256,256+D)
// P_lo0 [384,448) P_lo1 [448,512); P_hi of buffer b overwrites the first 64
// columns of S_b once they have been read.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace hstu {
namespace {

constexpr int kBM = 128;          // queries per tile
constexpr int kBN = 128;          // keys per tile
constexpr int kThreads = 224;     // 7 warps
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kMetaWarp = 6;
constexpr int kMetaStages = 2;
constexpr int kWts = 65;          // int64 differences reach buckets 0..64 only
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;
constexpr uint32_t kColPlo = 384;

template <int D>
struct Cfg {
  static constexpr int BKD = D < 64 ? D : 64;        // elements per swizzle row
  static constexpr int NKB = D / BKD;                // swizzle blocks along d
  static constexpr int SWB = BKD * 2;                // swizzle row bytes (64 or 128)
  static constexpr uint32_t LAYOUT = SWB == 128 ? 2u : 4u;
  static constexpr int BLOCK_BYTES = 128 * SWB;      // 128 rows x one swizzle block
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int STAGES = D == 128 ? 2 : 3;
};

struct TileMeta {
  int64_t t_first;
  int64_t t_last;
  int64_t row0;
  int pos0;
  int valid;
  int mono;
  int pad;
};

template <int D>
struct __align__(1024) Smem {
  uint8_t q[Cfg<D>::TILE_BYTES];
  uint8_t k[Cfg<D>::STAGES][Cfg<D>::TILE_BYTES];
  uint8_t v[Cfg<D>::STAGES][Cfg<D>::TILE_BYTES];
  int64_t ts[kMetaStages][kBN];
  float wwin[kMetaStages][4][256];
  TileMeta meta[kMetaStages];
  float wts[68];
  uint64_t q_full;
  uint64_t k_full[Cfg<D>::STAGES];
  uint64_t k_empty[Cfg<D>::STAGES];
  uint64_t v_full[Cfg<D>::STAGES];
  uint64_t v_empty[Cfg<D>::STAGES];
  uint64_t meta_full[kMetaStages];
  uint64_t meta_empty[kMetaStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full;
  uint32_t tmem_base;
  int abort_flag;
};

struct FwdParams {
  const int64_t* offsets;
  const int64_t* ts;
  const float* w_pos;
  const float* w_ts;
  void* out;
  int* status;
  int64_t B;
  int64_t T;
  int64_t P;
  int64_t NB;
  int H;
  int C;        // 0: plain jagged; >= 1: paired layout with 2C mini-chunks
  int levels;   // query-tile levels in the grid
  float scale;
};

// One work item: a query tile of one sequence and head, plus what is needed
// to enumerate its key tiles.
struct Work {
  int64_t q_row0;  // buffer row of query 0
  int64_t seq_off; // offsets[b]
  int64_t m;       // plain: L_b; paired: mini-chunk length
  int64_t TC;      // paired: rows per rank
  int q_pos0;      // within-sequence position of query 0
  int q_count;     // valid query rows
  int nkv;         // key tiles to visit
  int tpc;         // paired: key tiles per mini-chunk
  int h;
  int valid;
};

struct KTile {
  int64_t row0;
  int pos0;
  int valid;
};

__device__ __forceinline__ Work decode_work(const FwdParams& p, int64_t id) {
  Work w;
  w.valid = 0;
  const int H = p.H;
  w.h = (int)(id % H);
  int64_t t = id / H;
  const int64_t B = p.B;
  int b = (int)(t % B);
  t /= B;
  const int64_t o0 = p.offsets[b], o1 = p.offsets[b + 1];
  const int64_t L = o1 - o0;
  if (o0 < 0 || L <= 0 || o1 > p.T) return w;
  w.seq_off = o0;
  if (p.C == 0) {
    const int lvl = (int)t;
    const int qt = p.levels - 1 - lvl;
    const int64_t ntiles = (L + kBM - 1) / kBM;
    if (qt >= ntiles) return w;
    w.m = L;
    w.TC = 0;
    w.q_pos0 = qt * kBM;
    w.q_row0 = o0 + w.q_pos0;
    w.q_count = (int)imin64((int64_t)kBM, L - w.q_pos0);
    w.nkv = qt + 1;
    w.tpc = 0;
  } else {
    const int C = p.C;
    const int twoC = 2 * C;
    const int cidx = (int)(t % twoC);
    const int lvl = (int)(t / twoC);
    if (L % twoC != 0) return w;
    const int64_t m = L / twoC;
    const int c = twoC - 1 - cidx;      // heavy chunks first
    const int tt = p.levels - 1 - lvl;  // tile inside the chunk
    const int tpc = (int)((m + kBM - 1) / kBM);
    if (tt >= tpc) return w;
    const int r = c < C ? c : twoC - 1 - c;
    const int half = c >= C ? 1 : 0;
    w.m = m;
    w.TC = p.T / C;
    w.tpc = tpc;
    w.q_pos0 = (int)(c * m + (int64_t)tt * kBM);
    w.q_row0 = r * w.TC + o0 / C + half * m + (int64_t)tt * kBM;
    w.q_count = (int)imin64((int64_t)kBM, m - (int64_t)tt * kBM);
    w.nkv = c * tpc + tt + 1;
  }
  w.valid = 1;
  return w;
}

__device__ __forceinline__ KTile key_tile(const FwdParams& p, const Work& w, int n) {
  KTile k;
  if (p.C == 0) {
    k.pos0 = n * kBN;
    k.row0 = w.seq_off + k.pos0;
    k.valid = (int)imin64((int64_t)kBN, w.m - k.pos0);
  } else {
    const int C = p.C;
    const int c = n / w.tpc, tt = n % w.tpc;
    const int r = c < C ? c : 2 * C - 1 - c;
    const int half = c >= C ? 1 : 0;
    k.pos0 = (int)(c * w.m + (int64_t)tt * kBN);
    k.row0 = r * w.TC + w.seq_off / C + half * w.m + (int64_t)tt * kBN;
    k.valid = (int)imin64((int64_t)kBN, w.m - (int64_t)tt * kBN);
  }
  return k;
}

// block 0 checks the whole offsets array once per launch
__device__ void validate_offsets(const FwdParams& p, int64_t max_len) {
  if (threadIdx.x == 0 && (p.offsets[0] != 0 || p.offsets[p.B] != p.T))
    report(p.status, HSTU_ERR_OFFSETS);
  for (int64_t b = threadIdx.x; b < p.B; b += blockDim.x) {
    const int64_t L = p.offsets[b + 1] - p.offsets[b];
    if (L < 0) report(p.status, HSTU_ERR_OFFSETS);
    if (p.C > 0 && L % (2 * p.C) != 0) report(p.status, HSTU_ERR_NOT_DIVISIBLE);
    if (L > max_len) report(p.status, HSTU_ERR_SHAPE);
  }
}

// SiLU(x) = x sigmoid(x) = h + h tanh(h) with h = x / 2
__device__ __forceinline__ float silu_from_half(float h) { return fmaf(h, tanh_approx(h), h); }

template <int D, bool OUT_F32>
__global__ void __launch_bounds__(kThreads, 1)
    hstu_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using CF = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  Smem<D>& s = *reinterpret_cast<Smem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (blockIdx.x == 0)
    validate_offsets(p, (int64_t)p.levels * kBM * (p.C > 0 ? 2 * p.C : 1));

  const Work w = decode_work(p, blockIdx.x);
  if (!w.valid) return;  // uniform over the CTA

  if (threadIdx.x == 0) {
    mbar_init(&s.q_full, 1);
    for (int i = 0; i < CF::STAGES; ++i) {
      mbar_init(&s.k_full[i], 1);
      mbar_init(&s.k_empty[i], 1);
      mbar_init(&s.v_full[i], 1);
      mbar_init(&s.v_empty[i], 1);
    }
    for (int i = 0; i < kMetaStages; ++i) {
      mbar_init(&s.meta_full[i], 32);
      mbar_init(&s.meta_empty[i], 128);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.p_full[i], 128);
    }
    mbar_init(&s.o_full, 1);
    s.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  for (int i = threadIdx.x; i < kWts; i += blockDim.x) s.wts[i] = i < p.NB ? p.w_ts[i] : 0.f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  volatile int* abort_flag = &s.abort_flag;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const int xh = w.h * D;
      mbar_arrive_expect_tx(&s.q_full, CF::TILE_BYTES);
      for (int kb = 0; kb < CF::NKB; ++kb)
        tma_load_2d(s.q + kb * CF::BLOCK_BYTES, &tm_q, &s.q_full, xh + kb * CF::BKD,
                    (int32_t)w.q_row0);
      for (int n = 0; n < w.nkv; ++n) {
        const int st = n % CF::STAGES;
        const uint32_t ph = (uint32_t)(n / CF::STAGES) & 1u;
        const KTile kt = key_tile(p, w, n);
        if (n >= CF::STAGES && !mbar_wait(&s.k_empty[st], ph ^ 1u, abort_flag, p.status)) break;
        mbar_arrive_expect_tx(&s.k_full[st], CF::TILE_BYTES);
        for (int kb = 0; kb < CF::NKB; ++kb)
          tma_load_2d(s.k[st] + kb * CF::BLOCK_BYTES, &tm_k, &s.k_full[st], xh + kb * CF::BKD,
                      (int32_t)kt.row0);
        if (n >= CF::STAGES && !mbar_wait(&s.v_empty[st], ph ^ 1u, abort_flag, p.status)) break;
        mbar_arrive_expect_tx(&s.v_full[st], CF::TILE_BYTES);
        for (int kb = 0; kb < CF::NKB; ++kb)
          tma_load_2d(s.v[st] + kb * CF::BLOCK_BYTES, &tm_v, &s.v_full[st], xh + kb * CF::BKD,
                      (int32_t)kt.row0);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(kBM, kBN, false, false);
      constexpr uint32_t idesc_o = idesc_bf16(kBM, D, false, true);
      const uint32_t q_base = smem_u32(s.q);
      bool ok = mbar_wait(&s.q_full, 0, abort_flag, p.status);
      tc_fence_after();
      auto issue_pv = [&](int n) -> bool {
        const int pb = n & 1;
        const int st = n % CF::STAGES;
        const uint32_t ph = (uint32_t)(n / CF::STAGES) & 1u;
        if (!mbar_wait(&s.p_full[pb], (uint32_t)(n >> 1) & 1u, abort_flag, p.status)) return false;
        if (!mbar_wait(&s.v_full[st], ph, abort_flag, p.status)) return false;
        tc_fence_after();
        const uint32_t v_base = smem_u32(s.v[st]);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t bd = smem_desc(v_base + kk * 16 * CF::SWB, CF::BLOCK_BYTES, 8 * CF::SWB,
                                        CF::LAYOUT);
          mma_bf16_ts(tmem + kColO, tmem + pb * 128 + kk * 8, bd, idesc_o,
                      (n > 0 || kk > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t bd = smem_desc(v_base + kk * 16 * CF::SWB, CF::BLOCK_BYTES, 8 * CF::SWB,
                                        CF::LAYOUT);
          mma_bf16_ts(tmem + kColO, tmem + kColPlo + pb * 64 + kk * 8, bd, idesc_o, 1u);
        }
        mma_commit(&s.v_empty[st]);
        return true;
      };
      for (int n = 0; ok && n < w.nkv; ++n) {
        const int st = n % CF::STAGES;
        const uint32_t ph = (uint32_t)(n / CF::STAGES) & 1u;
        const int sb = n & 1;
        if (!mbar_wait(&s.k_full[st], ph, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t k_base = smem_u32(s.k[st]);
#pragma unroll
        for (int kb = 0; kb < CF::NKB; ++kb) {
#pragma unroll
          for (int kk = 0; kk < CF::BKD / 16; ++kk) {
            const uint64_t ad = smem_desc(q_base + kb * CF::BLOCK_BYTES + kk * 32, 16,
                                          8 * CF::SWB, CF::LAYOUT);
            const uint64_t bd = smem_desc(k_base + kb * CF::BLOCK_BYTES + kk * 32, 16,
                                          8 * CF::SWB, CF::LAYOUT);
            mma_bf16_ss(tmem + sb * 128, ad, bd, idesc_s, (kb | kk) != 0 ? 1u : 0u);
          }
        }
        mma_commit(&s.k_empty[st]);
        mma_commit(&s.s_full[sb]);
        if (n > 0) ok = issue_pv(n - 1);
      }
      if (ok) ok = issue_pv(w.nkv - 1);
      mma_commit(&s.o_full);
    }
  } else if (warp == kMetaWarp) {
    // ------------------------------------------------------------ tile metadata
    bool ok = true;
    for (int n = 0; n < w.nkv; ++n) {
      const int ms = n % kMetaStages;
      if (n >= kMetaStages) {
        ok = mbar_wait(&s.meta_empty[ms], ((uint32_t)(n / kMetaStages) & 1u) ^ 1u, abort_flag,
                       p.status);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      const KTile kt = key_tile(p, w, n);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = lane + 32 * i;
        const int cc = c < kt.valid ? c : kt.valid - 1;
        s.ts[ms][c] = p.ts[kt.row0 + cc];
      }
      __syncwarp();
      bool mono = true;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = lane + 32 * i;
        if (c + 1 < kt.valid && s.ts[ms][c] > s.ts[ms][c + 1]) mono = false;
      }
      mono = __all_sync(0xffffffffu, mono);
      // relative-position window: wwin[sft][x] = w_pos[clamp(base + x + sft, 0, P - 1)],
      // base = (q_pos0 - k_pos0) - 127, so row r / column c reads index r - c + 127.
      const int64_t base = (int64_t)(w.q_pos0 - kt.pos0) - 127;
      for (int idx = lane; idx < 1024; idx += 32) {
        const int sft = idx >> 8, x = idx & 255;
        int64_t rel = base + x + sft;
        rel = rel < 0 ? 0 : (rel > p.P - 1 ? p.P - 1 : rel);
        s.wwin[ms][sft][x] = __ldg(p.w_pos + rel);
      }
      if (lane == 0) {
        TileMeta& m = s.meta[ms];
        m.t_first = s.ts[ms][0];
        m.t_last = s.ts[ms][kt.valid - 1];
        m.row0 = kt.row0;
        m.pos0 = kt.pos0;
        m.valid = kt.valid;
        m.mono = mono ? 1 : 0;
      }
      __syncwarp();
      mbar_arrive(&s.meta_full[ms]);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int r = threadIdx.x;  // 0..127 = TMEM lane
    const bool row_ok = r < w.q_count;
    const int64_t q_row = w.q_row0 + r;
    const int qpos = w.q_pos0 + r;
    const int64_t t_i = row_ok ? p.ts[q_row] : p.ts[w.q_row0];
    const float hs = 0.5f * p.scale;
    const int nbm1 = (int)(p.NB - 1 < 64 ? p.NB - 1 : 64);
    const float wpos_last = __ldg(p.w_pos + (p.P - 1));
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    bool ok = true;
    for (int n = 0; n < w.nkv; ++n) {
      const int sb = n & 1;
      const int ms = n % kMetaStages;
      ok = mbar_wait(&s.meta_full[ms], (uint32_t)(n / kMetaStages) & 1u, abort_flag, p.status);
      if (ok) ok = mbar_wait(&s.s_full[sb], (uint32_t)(n >> 1) & 1u, abort_flag, p.status);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const TileMeta tmeta = s.meta[ms];
      const int rel0 = qpos - tmeta.pos0;  // relative position at column 0
      const bool pos_const = (int64_t)rel0 - (kBN - 1) >= p.P - 1;
      bool ts_const = false;
      float wt_const = 0.f;
      if (tmeta.mono) {
        const int b1 = bucket_of(t_i, tmeta.t_first, nbm1);
        const int b2 = bucket_of(t_i, tmeta.t_last, nbm1);
        if (b1 == b2) {
          ts_const = true;
          wt_const = s.wts[b1];
        }
      }
      const bool need_mask = (tmeta.pos0 + kBN - 1 > w.q_pos0) || tmeta.valid < kBN;
      const float* win = &s.wwin[ms][0][0];
      const int64_t* tsk = s.ts[ms];
#pragma unroll 1
      for (int cc = 0; cc < kBN / 32; ++cc) {
        uint32_t sv[32];
        tmem_ld32(tmem + lane_base + sb * 128 + cc * 32, sv);
        tmem_wait_ld(sv);
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          float pr[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int c = cc * 32 + j + e;
            const float wp = pos_const ? wpos_last : win[r - c + 127];
            const float wt = ts_const ? wt_const : s.wts[bucket_of(t_i, tsk[c], nbm1)];
            const float h = fmaf(__uint_as_float(sv[j + e]), hs, (wp + wt) * hs);
            float pv = silu_from_half(h);
            if (need_mask && !(c < tmeta.valid && tmeta.pos0 + c <= qpos)) pv = 0.f;
            pr[e] = pv;
          }
          const uint32_t ph = pack_bf16x2(pr[0], pr[1]);
          hi[j >> 1] = ph;
          lo[j >> 1] = pack_bf16x2(pr[0] - bf16lo_to_f32(ph), pr[1] - bf16hi_to_f32(ph));
        }
        tmem_st16(tmem + lane_base + sb * 128 + cc * 16, hi);
        tmem_st16(tmem + lane_base + kColPlo + sb * 64 + cc * 16, lo);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&s.p_full[sb]);
      mbar_arrive(&s.meta_empty[ms]);
    }
    if (ok) ok = mbar_wait(&s.o_full, 0, abort_flag, p.status);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    if (ok) {
      const int64_t orow = (q_row * p.H + w.h) * (int64_t)D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t ov[32];
        tmem_ld32(tmem + lane_base + kColO + cc * 32, ov);
        tmem_wait_ld(ov);
        if (row_ok) {
          if (OUT_F32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow + cc * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(ov[4 * i]), __uint_as_float(ov[4 * i + 1]),
                                   __uint_as_float(ov[4 * i + 2]), __uint_as_float(ov[4 * i + 3]));
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + orow + cc * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint4 u;
              u.x = pack_bf16x2(__uint_as_float(ov[8 * i + 0]), __uint_as_float(ov[8 * i + 1]));
              u.y = pack_bf16x2(__uint_as_float(ov[8 * i + 2]), __uint_as_float(ov[8 * i + 3]));
              u.z = pack_bf16x2(__uint_as_float(ov[8 * i + 4]), __uint_as_float(ov[8 * i + 5]));
              u.w = pack_bf16x2(__uint_as_float(ov[8 * i + 6]), __uint_as_float(ov[8 * i + 7]));
              dst[i] = u;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
cudaError_t make_maps(const AttnArgs& a, CUtensorMap* mq, CUtensorMap* mk, CUtensorMap* mv) {
  using CF = Cfg<D>;
  const cuuint64_t dims[2] = {(cuuint64_t)a.H * D, (cuuint64_t)a.T};
  const cuuint64_t strides[1] = {(cuuint64_t)a.H * D * 2};
  const cuuint32_t box[2] = {(cuuint32_t)CF::BKD, 128u};
  const cuuint32_t es[2] = {1u, 1u};
  const CUtensorMapSwizzle sw =
      CF::SWB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  const void* ptrs[3] = {a.q, a.k, a.v};
  CUtensorMap* maps[3] = {mq, mk, mv};
  for (int i = 0; i < 3; ++i) {
    CUresult r = encode_tiled(maps[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                              const_cast<void*>(ptrs[i]), dims, strides, box, es, sw);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

template <int D, bool OUT_F32>
cudaError_t launch_fwd_t(const AttnArgs& a, cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  cudaError_t e = make_maps<D>(a, &mq, &mk, &mv);
  if (e != cudaSuccess) return e;
  FwdParams p;
  p.offsets = a.offsets;
  p.ts = a.ts;
  p.w_pos = a.w_pos;
  p.w_ts = a.w_ts;
  p.out = a.out;
  p.status = a.status;
  p.B = a.B;
  p.T = a.T;
  p.P = a.P;
  p.NB = a.NB;
  p.H = a.H;
  p.C = a.C;
  p.scale = a.scale;
  const int64_t bound = a.max_seq_len > 0 ? a.max_seq_len : a.T;
  int64_t groups;
  if (a.C == 0) {
    p.levels = (int)((bound + kBM - 1) / kBM);
    groups = a.B;
  } else {
    const int64_t mmax = (bound + 2 * a.C - 1) / (2 * a.C);
    p.levels = (int)((mmax + kBM - 1) / kBM);
    groups = a.B * 2 * a.C;
  }
  if (p.levels < 1) p.levels = 1;
  const int64_t blocks = (int64_t)p.levels * groups * a.H;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  // Each CTA allocates all 512 TMEM columns, so ask for enough shared memory
  // that a second CTA never becomes resident on the same SM.
  size_t smem = sizeof(Smem<D>) + 1024;
  if (smem < 120 * 1024) smem = 120 * 1024;
  static bool attr_set = false;  // per template instance
  if (!attr_set) {
    e = cudaFuncSetAttribute(hstu_fwd_kernel<D, OUT_F32>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  hstu_fwd_kernel<D, OUT_F32><<<(unsigned)blocks, kThreads, smem, stream>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t attn_fwd_launch(const AttnArgs& a, cudaStream_t stream) {
  switch (a.D) {
    case 32:
      return a.out_fp32 ? launch_fwd_t<32, true>(a, stream) : launch_fwd_t<32, false>(a, stream);
    case 64:
      return a.out_fp32 ? launch_fwd_t<64, true>(a, stream) : launch_fwd_t<64, false>(a, stream);
    case 128:
      return a.out_fp32 ? launch_fwd_t<128, true>(a, stream)
                        : launch_fwd_t<128, false>(a, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace hstu
