// attn_bwd.cu -- jagged HSTU pointwise attention, backward, for sm_100a.
//
// The pages give the forward only ("Scaling Generative Recommendations with
// Context Parallelism on Hierarchical Sequential Transducers", §2.1) and say
// that the efficient backward does not materialise h x N x N tensors ("Actions
// Speak Louder than Words", App. F.3).  This kernel is the exact derivative
// of the forward, for the loss sum(O * dO):
//   x_ij = scale (q_i.k_j + Bias_ij),  p_ij = SiLU(x_ij),   j <= i
//   g_ij = (dO_i . v_j) SiLU'(x_ij),   gs_ij = scale g_ij
//   dV_j = sum_i p_ij dO_i,  dK_j = sum_i gs_ij q_i,  dQ_i = sum_j gs_ij k_j,
//   dw_pos[min(i-j, P-1)] += gs_ij,   dw_ts[bucket(t_i - t_j)] += gs_ij.
// There is no softmax, hence no rowsum(dO * O) pre-pass.
//
// One CTA owns one (key tile of 128 rows, head) of one sequence and loops over
// the query tiles at or after it.  Per query tile:
//   MMA warp  : S^T = K Q^T and dP^T = V dO^T into TMEM (SS form);
//   epilogue  : 8 warps, thread (group g, lane r) owns key row r and query
//               columns [64 g, 64 g + 64): P^T = SiLU(x) written back into
//               TMEM (bf16, over the S^T columns already read) and dS^T = gs
//               written bf16 into 128B-swizzled shared memory; bias-gradient
//               partials accumulated on the fly (registers for the clamped
//               w_pos entry and for runs of one w_ts bucket, a 512-entry
//               shared ring for the near-diagonal w_pos entries);
//   MMA warp  : dV += P^T dO (A from TMEM), dK += dS^T Q (K-major A),
//               dQ = dS K (the same dS^T tile read through an MN-major
//               descriptor);
//   epilogue  : thread r now owns query row r of dQ and adds it to the fp32
//               workspace with vector reductions.
// dK / dV stay in TMEM for the whole CTA and are written once at the end.
// TMEM columns: S^T [0,128) (P^T of query group g packed into [64g, 64g+32)),
// dP^T [128,256), dK [256,256+D), dV [256+D,256+2D); dQ has its own columns
// [256+2D, 256+3D) for D <= 64 and reuses [128,128+D) once dP^T is read for
// D = 128.  The relative-position bias comes from four shifted, pre-scaled
// copies of the whole w_pos table in shared memory (P <= Cfg::PTAB) or from
// per-tile windows built by the metadata warp otherwise.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace hstu {
namespace {

constexpr int kBM = 128;           // keys per CTA tile
constexpr int kBN = 128;           // queries per inner tile
constexpr int kThreads = 352;      // 8 epilogue warps + producer + MMA + meta
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kMetaWarp = 10;
constexpr int kEpiThreads = 256;
constexpr int kMetaStages = 2;
constexpr int kWts = 65;
constexpr int kRing = 512;         // shared ring of near-diagonal w_pos gradients
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;
constexpr uint32_t kColDP = 128;
constexpr uint32_t kColDK = 256;

template <int D>
struct Cfg {
  static constexpr int BKD = D < 64 ? D : 64;
  static constexpr int NKB = D / BKD;
  static constexpr int SWB = BKD * 2;
  static constexpr uint32_t LAYOUT = SWB == 128 ? 2u : 4u;
  static constexpr int BLOCK_BYTES = 128 * SWB;
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int STAGES = D == 128 ? 1 : 2;
  static constexpr uint32_t COL_DV = kColDK + D;
  static constexpr bool ALIAS_DQ = D == 128;           // dQ reuses the dP^T columns
  static constexpr uint32_t COL_DQ = ALIAS_DQ ? kColDP : kColDK + 2 * D;
  static constexpr int PTAB = D == 128 ? 3328 : 4096;  // largest P kept whole in smem
  static constexpr int WT = PTAB + 264;
};

struct QMeta {
  int64_t t_first;
  int64_t t_last;
  int valid;
  int mono;
  int rel32;
  int pad;
};

template <int D>
struct __align__(1024) Smem {
  uint8_t k[Cfg<D>::TILE_BYTES];
  uint8_t v[Cfg<D>::TILE_BYTES];
  uint8_t q[Cfg<D>::STAGES][Cfg<D>::TILE_BYTES];
  uint8_t dout[Cfg<D>::STAGES][Cfg<D>::TILE_BYTES];
  uint8_t dst[128 * 128 * 2];    // dS^T [key][query], two 64-query swizzle blocks
  union {
    float wtab[4][Cfg<D>::WT];   // wtab[s][x] = hs * w_pos[clamp(x + s - 128)]
    float wwin[kMetaStages][4][256];
  };
  int64_t ts[kMetaStages][kBN];
  int32_t ts32[kMetaStages][kBN];
  QMeta meta[kMetaStages];
  float ring[kRing];              // w_pos gradient of rel at ring[rel % 512]
  float dwts[68 * 8];             // w_ts gradient partials, [bucket][lane % 8]
  float wts_s[68];
  float wts_tbl[36];
  uint64_t kv_full;
  uint64_t qdo_full[Cfg<D>::STAGES];
  uint64_t qdo_empty[Cfg<D>::STAGES];
  uint64_t meta_full[kMetaStages];
  uint64_t meta_empty[kMetaStages];
  uint64_t st_full;
  uint64_t ds_full;
  uint64_t dq_full;
  uint64_t dq_free;
  uint64_t kv_done;
  uint64_t epi_sync;              // the 256 epilogue threads meet here (bounded waits)
  uint32_t tmem_base;
  int abort_flag;
};

struct BwdParams {
  const int64_t* offsets;
  const int64_t* ts;
  const float* w_pos;
  const float* w_ts;
  void* dk;
  void* dv;
  float* dq_accum;
  float* dw_pos;
  float* dw_ts;
  int* status;
  int64_t B;
  int64_t T;
  int64_t P;
  int64_t NB;
  int H;
  int levels;
  int wtab;
  float scale;
};

struct BWork {
  int64_t seq_off;
  int64_t L;
  int kt;      // key tile index
  int kvalid;  // valid key rows
  int nq;      // query tiles kt .. ntiles-1
  int h;
  int valid;
};

__device__ __forceinline__ BWork decode_bwork(const BwdParams& p, int64_t id) {
  BWork w;
  w.valid = 0;
  w.h = (int)(id % p.H);
  int64_t t = id / p.H;
  const int b = (int)(t % p.B);
  const int kt = (int)(t / p.B);
  const int64_t o0 = p.offsets[b], o1 = p.offsets[b + 1];
  const int64_t L = o1 - o0;
  if (o0 < 0 || L <= 0 || o1 > p.T) return w;
  const int64_t ntiles = (L + kBM - 1) / kBM;
  if (kt >= ntiles) return w;
  w.seq_off = o0;
  w.L = L;
  w.kt = kt;
  w.kvalid = (int)imin64((int64_t)kBM, L - (int64_t)kt * kBM);
  w.nq = (int)(ntiles - kt);
  w.valid = 1;
  return w;
}

enum { kTsConst = 0, kTsRel32 = 1, kTsFull = 2 };
enum { kPosConst = 0, kPosNoClamp = 1, kPosMixed = 2 };

struct BRowCtx {
  const float* wrow;     // bias window so that column c reads wrow + c (float4 groups)
  const int32_t* ts32;   // query timestamps relative to t_first
  const int64_t* ts64;
  const float* tbl;      // scaled w_ts by bfind index (-1..31)
  const float* wts_s;
  float* s_dwts;
  uint32_t ring;         // shared address of the w_pos gradient ring
  int64_t t_j;
  float hs;              // scale / 2
  float wpc;
  float wtc;
  int tj_rel;
  int nbm1;
  int cmin;              // first unmasked column
  int cmax;              // last unmasked column
  int rel_c0;            // relative position of column 0: Delta0 - r
  int pm1;               // P - 1
  int bconst;            // bucket of the row when constant
};

struct BiasAcc {
  float pclamp;   // gradient of w_pos[P-1]
  float run;      // current run of one w_ts bucket
  int cur;        // bucket of the run (-1: none)
};

// No "memory" clobber: the ring is only read after the epilogue's mbarrier
// sync, which orders it; a clobber here would stop the compiler from
// scheduling the unrolled per-pair loop around every atomic.
__device__ __forceinline__ void red_shared_add(uint32_t addr, float v) {
  asm volatile("red.shared.add.f32 [%0], %1;" ::"r"(addr), "f"(v));
}

// Runs are flushed into one of 8 copies of the bucket table (chosen by lane),
// so lanes of a warp that close a run of the same bucket together rarely hit
// the same address.  s_dwts points at the copy of this lane.
__device__ __forceinline__ void flush_run(BiasAcc& acc, float* s_dwts) {
  if (acc.cur >= 0 && acc.run != 0.f) red_shared_add(smem_u32(&s_dwts[acc.cur * 8]), acc.run);
  acc.run = 0.f;
}

template <bool MASK, int POS_MODE, int TS_MODE>
__device__ __forceinline__ void bwd_chunk(const uint32_t (&sv)[32], const uint32_t (&dpv)[32],
                                          uint32_t (&pt)[16], uint32_t (&ds)[16], int cbase,
                                          const BRowCtx& rc, BiasAcc& acc) {
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    const int c0 = cbase + g * 4;
    float wp[4], wt[4];
    int bk[4];
    if (POS_MODE == kPosConst) {
      wp[0] = wp[1] = wp[2] = wp[3] = rc.wpc;
    } else {
      const float4 w4 = *reinterpret_cast<const float4*>(rc.wrow + c0);
      wp[0] = w4.x; wp[1] = w4.y; wp[2] = w4.z; wp[3] = w4.w;
    }
    if (TS_MODE == kTsConst) {
      wt[0] = wt[1] = wt[2] = wt[3] = rc.wtc;
      bk[0] = bk[1] = bk[2] = bk[3] = rc.bconst;
    } else if (TS_MODE == kTsRel32) {
      const int4 t4 = *reinterpret_cast<const int4*>(rc.ts32 + c0);
      const int tq[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int f = bfind_u32((uint32_t)max(tq[e] - rc.tj_rel, 0));
        wt[e] = rc.tbl[f];
        bk[e] = min(f + 1, rc.nbm1);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        bk[e] = bucket_of(rc.ts64[c0 + e], rc.t_j, rc.nbm1);
        wt[e] = rc.wts_s[bk[e]];
      }
    }
    float pv[4], gv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float h = fmaf(__uint_as_float(sv[g * 4 + e]), rc.hs, wp[e] + wt[e]);
      const float th = tanh_approx(h);
      const float pe = fmaf(h, th, h);                 // SiLU(x)
      const float ssig = fmaf(rc.hs, th, rc.hs);       // scale * sigmoid(x)
      const float d1 = fmaf(-h, th, h + 1.f);          // 1 + x (1 - sigmoid(x))
      float ge = __uint_as_float(dpv[g * 4 + e]) * ssig * d1;
      float pp = pe;
      bool valid = true;
      if (MASK) {
        valid = (c0 + e >= rc.cmin) && (c0 + e <= rc.cmax);
        if (!valid) { pp = 0.f; ge = 0.f; }
      }
      pv[e] = pp;
      gv[e] = ge;
      if (!MASK || valid) {
        if (POS_MODE == kPosConst) {
          acc.pclamp += ge;
        } else {
          const int rel = rc.rel_c0 + c0 + e;
          if (POS_MODE == kPosMixed && rel >= rc.pm1) acc.pclamp += ge;
          else red_shared_add(rc.ring + (uint32_t)((rel & (kRing - 1)) << 2), ge);
        }
        if (TS_MODE == kTsConst) {
          acc.run += ge;
        } else {
          if (bk[e] != acc.cur) {
            flush_run(acc, rc.s_dwts);
            acc.cur = bk[e];
          }
          acc.run += ge;
        }
      }
    }
    pt[g * 2] = pack_bf16x2(pv[0], pv[1]);
    pt[g * 2 + 1] = pack_bf16x2(pv[2], pv[3]);
    ds[g * 2] = pack_bf16x2(gv[0], gv[1]);
    ds[g * 2 + 1] = pack_bf16x2(gv[2], gv[3]);
  }
}

// variant = 3 * pos_mode + ts_mode (unmasked tiles) or ts_mode (masked tiles,
// which always take the mixed w_pos path)
__device__ __forceinline__ void bwd_chunk_dispatch(bool masked, int variant,
                                                   const uint32_t (&sv)[32],
                                                   const uint32_t (&dpv)[32], uint32_t (&pt)[16],
                                                   uint32_t (&ds)[16], int cbase,
                                                   const BRowCtx& rc, BiasAcc& acc) {
  if (masked) {
    switch (variant) {
      case kTsConst: bwd_chunk<true, kPosMixed, kTsConst>(sv, dpv, pt, ds, cbase, rc, acc); break;
      case kTsRel32: bwd_chunk<true, kPosMixed, kTsRel32>(sv, dpv, pt, ds, cbase, rc, acc); break;
      default: bwd_chunk<true, kPosMixed, kTsFull>(sv, dpv, pt, ds, cbase, rc, acc); break;
    }
    return;
  }
  switch (variant) {
    case 0: bwd_chunk<false, kPosConst, kTsConst>(sv, dpv, pt, ds, cbase, rc, acc); break;
    case 1: bwd_chunk<false, kPosConst, kTsRel32>(sv, dpv, pt, ds, cbase, rc, acc); break;
    case 2: bwd_chunk<false, kPosConst, kTsFull>(sv, dpv, pt, ds, cbase, rc, acc); break;
    case 3: bwd_chunk<false, kPosNoClamp, kTsConst>(sv, dpv, pt, ds, cbase, rc, acc); break;
    case 4: bwd_chunk<false, kPosNoClamp, kTsRel32>(sv, dpv, pt, ds, cbase, rc, acc); break;
    case 5: bwd_chunk<false, kPosNoClamp, kTsFull>(sv, dpv, pt, ds, cbase, rc, acc); break;
    case 6: bwd_chunk<false, kPosMixed, kTsConst>(sv, dpv, pt, ds, cbase, rc, acc); break;
    case 7: bwd_chunk<false, kPosMixed, kTsRel32>(sv, dpv, pt, ds, cbase, rc, acc); break;
    default: bwd_chunk<false, kPosMixed, kTsFull>(sv, dpv, pt, ds, cbase, rc, acc); break;
  }
}

// 16-byte store of 8 bf16 (4 packed words) into row r, 16-byte chunk `chunk`
// (0..15 over 128 columns) of a [128][128] bf16 tile in 128B-swizzled
// K-major layout (two 64-column blocks of 16 KB).
__device__ __forceinline__ void st_swizzled(uint8_t* tile, int r, int chunk, const uint32_t* w4) {
  const int blk = chunk >> 3;
  const int c = chunk & 7;
  uint8_t* dst = tile + blk * 16384 + r * 128 + ((c ^ (r & 7)) << 4);
  *reinterpret_cast<uint4*>(dst) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
}

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}

// Move the ring entries of relative positions [rel0, rel0 + n) to global
// memory and clear them (the 256 epilogue threads call this together).
__device__ __forceinline__ void flush_ring(float* ring, float* g_dwpos, int64_t rel0, int n,
                                           int tid) {
  if (tid < n) {
    const int64_t rel = rel0 + tid;
    if (rel >= 0) {
      float* slot = &ring[rel & (kRing - 1)];
      const float v = *slot;
      if (v != 0.f) {
        atomicAdd(g_dwpos + rel, v);
        *slot = 0.f;
      }
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    hstu_bwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_do, const BwdParams p) {
  using CF = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  Smem<D>& s = *reinterpret_cast<Smem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (blockIdx.x == 0)
    validate_offsets(p.offsets, p.B, p.T, 0, (int64_t)p.levels * kBM, p.status);

  const BWork w = decode_bwork(p, blockIdx.x);
  if (!w.valid) return;

  const float hs = 0.5f * p.scale;
  const int nbm1 = (int)(p.NB - 1 < 64 ? p.NB - 1 : 64);
  if (threadIdx.x == 0) {
    mbar_init(&s.kv_full, 1);
    for (int i = 0; i < CF::STAGES; ++i) {
      mbar_init(&s.qdo_full[i], 1);
      mbar_init(&s.qdo_empty[i], 1);
    }
    for (int i = 0; i < kMetaStages; ++i) {
      mbar_init(&s.meta_full[i], 32);
      mbar_init(&s.meta_empty[i], kEpiThreads);
    }
    mbar_init(&s.st_full, 1);
    mbar_init(&s.ds_full, kEpiThreads);
    mbar_init(&s.dq_full, 1);
    mbar_init(&s.dq_free, kEpiThreads);
    mbar_init(&s.kv_done, 1);
    mbar_init(&s.epi_sync, kEpiThreads);
    s.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (p.wtab) {
    // Wfull[x] = hs * w_pos[clamp(x - 128)], stored as wtab[s][x - s]
    const int64_t relmax = imin64(w.L - 1 - (int64_t)w.kt * kBM + (kBN - 1), p.P + 130);
    const int nx = (int)imin64(relmax + 136, (int64_t)CF::WT + 3);
    for (int x = threadIdx.x; x < nx; x += blockDim.x) {
      int64_t rel = (int64_t)x - 128;
      rel = rel < 0 ? 0 : (rel > p.P - 1 ? p.P - 1 : rel);
      const float val = __ldg(p.w_pos + rel) * hs;
#pragma unroll
      for (int sft = 0; sft < 4; ++sft) {
        const int xs = x - sft;
        if (xs >= 0 && xs < CF::WT) s.wtab[sft][xs] = val;
      }
    }
  }
  for (int i = threadIdx.x; i < kRing; i += blockDim.x) s.ring[i] = 0.f;
  for (int i = threadIdx.x; i < 68 * 8; i += blockDim.x) s.dwts[i] = 0.f;
  for (int i = threadIdx.x; i < 68; i += blockDim.x)
    s.wts_s[i] = (i < kWts && i < p.NB ? p.w_ts[i] : 0.f) * hs;
  for (int i = threadIdx.x; i < 34; i += blockDim.x) {
    const int b = i < nbm1 ? i : nbm1;
    s.wts_tbl[i] = (b < p.NB ? p.w_ts[b] : 0.f) * hs;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  volatile int* abort_flag = &s.abort_flag;
  const int64_t k_row0 = w.seq_off + (int64_t)w.kt * kBM;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    // The whole warp runs the loop (waits stay warp-uniform); one elected
    // lane issues each copy.
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
    }
    __syncwarp();
    const int xh = w.h * D;
    mbar_arrive_expect_tx_elect(&s.kv_full, 2 * CF::TILE_BYTES);
#pragma unroll
    for (int kb = 0; kb < CF::NKB; ++kb) {
      tma_load_2d_elect(s.k + kb * CF::BLOCK_BYTES, &tm_k, &s.kv_full, xh + kb * CF::BKD,
                        (int32_t)k_row0);
      tma_load_2d_elect(s.v + kb * CF::BLOCK_BYTES, &tm_v, &s.kv_full, xh + kb * CF::BKD,
                        (int32_t)k_row0);
    }
    for (int n = 0; n < w.nq; ++n) {
      const int st = n % CF::STAGES;
      const uint32_t ph = (uint32_t)(n / CF::STAGES) & 1u;
      const int64_t q_row0 = w.seq_off + (int64_t)(w.kt + n) * kBN;
      if (n >= CF::STAGES) {
        const bool ok = __all_sync(0xffffffffu,
                                   mbar_wait(&s.qdo_empty[st], ph ^ 1u, abort_flag, p.status));
        if (!ok) break;
      }
      mbar_arrive_expect_tx_elect(&s.qdo_full[st], 2 * CF::TILE_BYTES);
#pragma unroll
      for (int kb = 0; kb < CF::NKB; ++kb) {
        tma_load_2d_elect(s.q[st] + kb * CF::BLOCK_BYTES, &tm_q, &s.qdo_full[st],
                          xh + kb * CF::BKD, (int32_t)q_row0);
        tma_load_2d_elect(s.dout[st] + kb * CF::BLOCK_BYTES, &tm_do, &s.qdo_full[st],
                          xh + kb * CF::BKD, (int32_t)q_row0);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop and computes the (uniform) operands; one
    // elected lane issues every tcgen05.mma / commit.
    constexpr uint32_t idesc_s = idesc_bf16(kBM, kBN, false, false);   // S^T, dP^T
    constexpr uint32_t idesc_kv = idesc_bf16(kBM, D, false, true);     // dV, dK
    constexpr uint32_t idesc_q = idesc_bf16(kBN, D, true, true);       // dQ
    // Base descriptors are built once; each MMA adds a compile-time offset
    // (16-byte units) to the start-address field, a ring stage adds
    // st * TILE_BYTES / 16.
    const uint64_t kA = smem_desc(smem_u32(s.k), 16, 8 * CF::SWB, CF::LAYOUT);           // K, K-major
    const uint64_t vA = smem_desc(smem_u32(s.v), 16, 8 * CF::SWB, CF::LAYOUT);           // V, K-major
    const uint64_t kB = smem_desc(smem_u32(s.k), CF::BLOCK_BYTES, 8 * CF::SWB, CF::LAYOUT);  // K, MN
    const uint64_t qK0 = smem_desc(smem_u32(s.q[0]), 16, 8 * CF::SWB, CF::LAYOUT);
    const uint64_t qM0 = smem_desc(smem_u32(s.q[0]), CF::BLOCK_BYTES, 8 * CF::SWB, CF::LAYOUT);
    const uint64_t oK0 = smem_desc(smem_u32(s.dout[0]), 16, 8 * CF::SWB, CF::LAYOUT);
    const uint64_t oM0 = smem_desc(smem_u32(s.dout[0]), CF::BLOCK_BYTES, 8 * CF::SWB, CF::LAYOUT);
    const uint64_t dsK = smem_desc(smem_u32(s.dst), 16, 1024, 2u);       // dS^T, K-major
    const uint64_t dsM = smem_desc(smem_u32(s.dst), 16384, 1024, 2u);    // dS, MN-major
    bool ok = __all_sync(0xffffffffu, mbar_wait(&s.kv_full, 0, abort_flag, p.status));
    for (int n = 0; ok && n < w.nq; ++n) {
      const int st = n % CF::STAGES;
      const uint32_t ph = (uint32_t)(n / CF::STAGES) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(&s.qdo_full[st], ph, abort_flag, p.status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t stoff = (uint64_t)(st * (CF::TILE_BYTES >> 4));
      const uint64_t qK = qK0 + stoff, qM = qM0 + stoff, oK = oK0 + stoff, oM = oM0 + stoff;
      // S^T = K Q^T
#pragma unroll
      for (int kb = 0; kb < CF::NKB; ++kb)
#pragma unroll
        for (int kk = 0; kk < CF::BKD / 16; ++kk) {
          const uint64_t off = (uint64_t)((kb * CF::BLOCK_BYTES + kk * 32) >> 4);
          mma_bf16_ss_elect(tmem + kColS, kA + off, qK + off, idesc_s, (kb | kk) != 0 ? 1u : 0u);
        }
      // dP^T = V dO^T (with D = 128 into the columns dQ of the previous tile used)
      if (CF::ALIAS_DQ && n > 0 &&
          !__all_sync(0xffffffffu,
                      mbar_wait(&s.dq_free, (uint32_t)(n - 1) & 1u, abort_flag, p.status))) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int kb = 0; kb < CF::NKB; ++kb)
#pragma unroll
        for (int kk = 0; kk < CF::BKD / 16; ++kk) {
          const uint64_t off = (uint64_t)((kb * CF::BLOCK_BYTES + kk * 32) >> 4);
          mma_bf16_ss_elect(tmem + kColDP, vA + off, oK + off, idesc_s, (kb | kk) != 0 ? 1u : 0u);
        }
      mma_commit_elect(&s.st_full);
      if (!__all_sync(0xffffffffu, mbar_wait(&s.ds_full, (uint32_t)n & 1u, abort_flag, p.status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // dV += P^T dO (P^T from TMEM) ; dK += dS^T Q   (K = 128 queries in 8 steps)
#pragma unroll
      for (int kk = 0; kk < kBN / 16; ++kk) {
        const uint64_t b_off = (uint64_t)((kk * 16 * CF::SWB) >> 4);
        const uint32_t acc = (n > 0 || kk > 0) ? 1u : 0u;
        mma_bf16_ts_elect(tmem + CF::COL_DV, tmem + kColS + 64 * (kk >> 2) + 8 * (kk & 3),
                          oM + b_off, idesc_kv, acc);
        mma_bf16_ss_elect(tmem + kColDK,
                          dsK + (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4), qM + b_off,
                          idesc_kv, acc);
      }
      mma_commit_elect(&s.qdo_empty[st]);
      if (!CF::ALIAS_DQ && n > 0 &&
          !__all_sync(0xffffffffu,
                      mbar_wait(&s.dq_free, (uint32_t)(n - 1) & 1u, abort_flag, p.status))) {
        ok = false;
        break;
      }
      // dQ = dS K   (M = queries via the MN-major view of dS^T; K = 128 keys)
#pragma unroll
      for (int kk = 0; kk < kBM / 16; ++kk)
        mma_bf16_ss_elect(tmem + CF::COL_DQ, dsM + (uint64_t)((kk * 2048) >> 4),
                          kB + (uint64_t)((kk * 16 * CF::SWB) >> 4), idesc_q, kk > 0 ? 1u : 0u);
      mma_commit_elect(&s.dq_full);
    }
    mma_commit_elect(&s.kv_done);
  } else if (warp == kMetaWarp) {
    // ------------------------------------------------------------ query-tile metadata
    // The next tile's timestamps are requested before the current one is
    // processed, so the load latency overlaps one tile of work.
    bool ok = true;
    auto qvalid_of = [&](int n) {
      return (int)imin64((int64_t)kBN, w.L - (int64_t)(w.kt + n) * kBN);
    };
    auto load_ts = [&](int n, int64_t (&t4)[4]) {
      const int64_t q_row0 = w.seq_off + (int64_t)(w.kt + n) * kBN;
      const int qv = qvalid_of(n);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = lane + 32 * i;
        t4[i] = __ldg(p.ts + q_row0 + (c < qv ? c : qv - 1));
      }
    };
    int64_t tv[4];
    load_ts(0, tv);
    for (int n = 0; n < w.nq; ++n) {
      const int ms = n % kMetaStages;
      if (n >= kMetaStages) {
        ok = mbar_wait(&s.meta_empty[ms], ((uint32_t)(n / kMetaStages) & 1u) ^ 1u, abort_flag,
                       p.status);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      int64_t tn[4];
      if (n + 1 < w.nq) load_ts(n + 1, tn);
      const int qvalid = qvalid_of(n);
      if (!p.wtab) {
        // window: wwin[sft][x] = hs * w_pos[clamp(base + x + sft)], base = Delta0 - 127;
        // key row r / query column c reads index c - r + 127.
        const int64_t base = (int64_t)n * kBN - 127;
        for (int idx = lane; idx < 1024; idx += 32) {
          const int sft = idx >> 8, x = idx & 255;
          int64_t rel = base + x + sft;
          rel = rel < 0 ? 0 : (rel > p.P - 1 ? p.P - 1 : rel);
          s.wwin[ms][sft][x] = __ldg(p.w_pos + rel) * hs;
        }
      }
      const int64_t t_first = __shfl_sync(0xffffffffu, tv[0], 0);
      const int last = qvalid - 1;
      const int gsel = last >> 5;
      const int64_t tsel = gsel == 0 ? tv[0] : gsel == 1 ? tv[1] : gsel == 2 ? tv[2] : tv[3];
      const int64_t t_last = __shfl_sync(0xffffffffu, tsel, last & 31);
      bool mono = true, rel32 = true;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = lane + 32 * i;
        s.ts[ms][c] = tv[i];
        const int64_t d = tv[i] - t_first;
        rel32 = rel32 && (d > -(1ll << 30)) && (d < (1ll << 30));
        s.ts32[ms][c] = (int32_t)d;
        const int64_t nxt_same = __shfl_down_sync(0xffffffffu, tv[i], 1);
        const int64_t nxt_grp = __shfl_sync(0xffffffffu, tv[i < 3 ? i + 1 : 3], 0);
        const int64_t nxt = lane < 31 ? nxt_same : nxt_grp;
        if (c + 1 < qvalid && tv[i] > nxt) mono = false;
      }
      mono = __all_sync(0xffffffffu, mono);
      rel32 = __all_sync(0xffffffffu, rel32);
      if (lane == 0) {
        QMeta& m = s.meta[ms];
        m.t_first = t_first;
        m.t_last = t_last;
        m.valid = qvalid;
        m.mono = mono ? 1 : 0;
        m.rel32 = rel32 ? 1 : 0;
      }
      __syncwarp();
      mbar_arrive(&s.meta_full[ms]);
      if (n + 1 < w.nq) {
#pragma unroll
        for (int i = 0; i < 4; ++i) tv[i] = tn[i];
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int grp = warp >> 2;          // query columns [64 grp, 64 grp + 64)
    const int r = threadIdx.x & 127;    // key row = TMEM lane (S^T, dP^T, dK, dV) / query row (dQ)
    const int etid = threadIdx.x;       // 0..255
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const int64_t t_j = __ldg(p.ts + k_row0 + (r < w.kvalid ? r : w.kvalid - 1));
    BRowCtx rc;
    rc.t_j = t_j;
    rc.hs = hs;
    rc.wpc = __ldg(p.w_pos + (p.P - 1)) * hs;
    rc.nbm1 = nbm1;
    rc.tbl = s.wts_tbl + 1;
    rc.wts_s = s.wts_s;
    rc.s_dwts = s.dwts + (lane & 7);
    rc.ring = smem_u32(s.ring);
    rc.pm1 = (int)(p.P - 1 < 0x3fffffff ? p.P - 1 : 0x3fffffff);
    BiasAcc acc;
    acc.pclamp = 0.f;
    acc.run = 0.f;
    acc.cur = -1;
    bool ok = true;
    int n_done = 0;
    uint32_t sync_phase = 0;
    // all epilogue threads meet; bounded, so an aborted CTA cannot hang here
    auto epi_sync = [&]() -> bool {
      mbar_arrive(&s.epi_sync);
      const bool r_ok = mbar_wait(&s.epi_sync, sync_phase & 1u, abort_flag, p.status);
      ++sync_phase;
      return r_ok;
    };
    for (int n = 0; n < w.nq; ++n) {
      const int ms = n % kMetaStages;
      ok = mbar_wait(&s.meta_full[ms], (uint32_t)(n / kMetaStages) & 1u, abort_flag, p.status);
      if (ok) ok = mbar_wait(&s.st_full, (uint32_t)n & 1u, abort_flag, p.status);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const QMeta qm = s.meta[ms];
      const int delta0 = n * kBN;              // q_pos0 - k_pos0
      const int doff = delta0 - r;             // relative position of column 0
      rc.rel_c0 = doff;
      const int64_t rmin = (int64_t)doff + 64 * grp, rmax = rmin + 63;
      const bool all_const = __all_sync(0xffffffffu, rmin >= p.P - 1);
      const bool all_noclamp = __all_sync(0xffffffffu, rmax < p.P - 1);
      const int pos_mode = all_const ? kPosConst : all_noclamp ? kPosNoClamp : kPosMixed;
      bool lane_const = false, lane_fit = false;
      if (qm.mono) {
        const int b1 = bucket_of(qm.t_first, t_j, nbm1);
        const int b2 = bucket_of(qm.t_last, t_j, nbm1);
        if (b1 == b2) {
          lane_const = true;
          rc.bconst = b1;
          rc.wtc = s.wts_s[b1];
        }
      }
      if (qm.rel32) {
        const int64_t d = t_j - qm.t_first;
        if (d > -(1ll << 30) && d < (1ll << 30)) {
          lane_fit = true;
          rc.tj_rel = (int)d;
        }
      }
      const int ts_mode = __all_sync(0xffffffffu, lane_const) ? kTsConst
                          : __all_sync(0xffffffffu, lane_fit) ? kTsRel32 : kTsFull;
      if (ts_mode == kTsConst && acc.cur != rc.bconst) {
        flush_run(acc, rc.s_dwts);
        acc.cur = rc.bconst;
      }
      const bool masked = (n == 0) || qm.valid < kBN;
      const int variant = masked ? ts_mode : 3 * pos_mode + ts_mode;
      rc.cmin = r - delta0 > 0 ? r - delta0 : 0;
      rc.cmax = qm.valid - 1;
      if (p.wtab) {
        // lanes whose row is entirely clamped read entries that all hold w_pos[P-1]
        const int dc = doff < rc.pm1 ? doff : rc.pm1;
        const int sft = (dc + 128) & 3;
        rc.wrow = &s.wtab[sft][0] + (dc + 128 - sft);
      } else {
        const int sft = (3 - (r & 3)) & 3;
        rc.wrow = &s.wwin[ms][sft][0] + (127 - r - sft);
      }
      rc.ts32 = s.ts32[ms];
      rc.ts64 = s.ts[ms];
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int cbase = grp * 64 + cc * 32;
        uint32_t sv[32], dpv[32];
        tmem_ld32(tmem + lane_base + kColS + cbase, sv);
        tmem_ld32(tmem + lane_base + kColDP + cbase, dpv);
        tmem_wait_ld(sv);
        tmem_wait_ld(dpv);
        uint32_t pt[16], ds[16];
        bwd_chunk_dispatch(masked, variant, sv, dpv, pt, ds, cbase, rc, acc);
        __syncwarp();
        tmem_st16(tmem + lane_base + kColS + grp * 64 + cc * 16, pt);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) st_swizzled(s.dst, r, (cbase >> 3) + q4, &ds[q4 * 4]);
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&s.ds_full);
      mbar_arrive(&s.meta_empty[ms]);
      // relative positions below 128 n + 1 are final: move them to global memory
      ok = __all_sync(0xffffffffu, epi_sync());
      if (!ok) break;
      flush_ring(s.ring, p.dw_pos, (int64_t)delta0 - 127, 128, etid);
      n_done = n + 1;
      // dQ of this query tile: thread r owns query row r, columns of its group
      ok = mbar_wait(&s.dq_full, (uint32_t)n & 1u, abort_flag, p.status);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      {
        const int qt = w.kt + n;
        const bool q_ok = r < qm.valid;
        float* dst = p.dq_accum + ((w.seq_off + (int64_t)qt * kBN + r) * p.H + w.h) * D;
        constexpr int kHalf = D / 2;
        if (kHalf == 16) {
          uint32_t qv[16];
          tmem_ld16(tmem + lane_base + CF::COL_DQ + grp * 16, qv);
          tmem_wait_ld(qv);
          if (q_ok)
#pragma unroll
            for (int i = 0; i < 4; ++i)
              red_add_v4(dst + grp * 16 + 4 * i, __uint_as_float(qv[4 * i]),
                         __uint_as_float(qv[4 * i + 1]), __uint_as_float(qv[4 * i + 2]),
                         __uint_as_float(qv[4 * i + 3]));
        } else {
#pragma unroll 1
          for (int cc = 0; cc < kHalf / 32; ++cc) {
            const int col = grp * kHalf + cc * 32;
            uint32_t qv[32];
            tmem_ld32(tmem + lane_base + CF::COL_DQ + col, qv);
            tmem_wait_ld(qv);
            if (q_ok)
#pragma unroll
              for (int i = 0; i < 8; ++i)
                red_add_v4(dst + col + 4 * i, __uint_as_float(qv[4 * i]),
                           __uint_as_float(qv[4 * i + 1]), __uint_as_float(qv[4 * i + 2]),
                           __uint_as_float(qv[4 * i + 3]));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&s.dq_free);
    }
    flush_run(acc, rc.s_dwts);
    // w_pos[P-1] partial: warp sum, then one global atomic per warp
    float pc = acc.pclamp;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) pc += __shfl_xor_sync(0xffffffffu, pc, o);
    if (lane == 0 && pc != 0.f) atomicAdd(p.dw_pos + (p.P - 1), pc);
    // dK, dV: thread r owns key row r, its group's half of the columns
    if (ok) ok = mbar_wait(&s.kv_done, 0, abort_flag, p.status);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    if (ok) {
      const bool k_ok = r < w.kvalid;
      const int64_t orow = ((k_row0 + r) * p.H + w.h) * (int64_t)D;
      constexpr int kHalf = D / 2;
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        const uint32_t col0 = which == 0 ? kColDK : CF::COL_DV;
        uint16_t* out = static_cast<uint16_t*>(which == 0 ? p.dk : p.dv) + orow;
        if (kHalf == 16) {
          uint32_t v16[16];
          tmem_ld16(tmem + lane_base + col0 + grp * 16, v16);
          tmem_wait_ld(v16);
          if (k_ok) {
            uint4* d4 = reinterpret_cast<uint4*>(out + grp * 16);
#pragma unroll
            for (int i = 0; i < 2; ++i)
              d4[i] = make_uint4(
                  pack_bf16x2(__uint_as_float(v16[8 * i]), __uint_as_float(v16[8 * i + 1])),
                  pack_bf16x2(__uint_as_float(v16[8 * i + 2]), __uint_as_float(v16[8 * i + 3])),
                  pack_bf16x2(__uint_as_float(v16[8 * i + 4]), __uint_as_float(v16[8 * i + 5])),
                  pack_bf16x2(__uint_as_float(v16[8 * i + 6]), __uint_as_float(v16[8 * i + 7])));
          }
        } else {
#pragma unroll 1
          for (int cc = 0; cc < kHalf / 32; ++cc) {
            const int col = grp * kHalf + cc * 32;
            uint32_t v32[32];
            tmem_ld32(tmem + lane_base + col0 + col, v32);
            tmem_wait_ld(v32);
            if (k_ok) {
              uint4* d4 = reinterpret_cast<uint4*>(out + col);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                d4[i] = make_uint4(
                    pack_bf16x2(__uint_as_float(v32[8 * i]), __uint_as_float(v32[8 * i + 1])),
                    pack_bf16x2(__uint_as_float(v32[8 * i + 2]), __uint_as_float(v32[8 * i + 3])),
                    pack_bf16x2(__uint_as_float(v32[8 * i + 4]), __uint_as_float(v32[8 * i + 5])),
                    pack_bf16x2(__uint_as_float(v32[8 * i + 6]), __uint_as_float(v32[8 * i + 7])));
            }
          }
        }
      }
    }
    // the rest of the ring and the w_ts partials of this CTA -> global
    const bool synced = __all_sync(0xffffffffu, epi_sync());
    if (synced && n_done > 0)
      flush_ring(s.ring, p.dw_pos, (int64_t)(n_done - 1) * kBN + 1, 127, etid);
    for (int i = etid; synced && i < kWts && i < p.NB; i += kEpiThreads) {
      float v = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) v += s.dwts[i * 8 + c];
      if (v != 0.f) atomicAdd(p.dw_ts + i, v);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

__global__ void dq_convert_kernel(const float* __restrict__ acc, uint16_t* __restrict__ dq,
                                  int64_t n4) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(acc)[i];
    uint2 o;
    o.x = pack_bf16x2(v.x, v.y);
    o.y = pack_bf16x2(v.z, v.w);
    reinterpret_cast<uint2*>(dq)[i] = o;
  }
}

template <int D>
cudaError_t launch_bwd_t(const AttnArgs& a, cudaStream_t stream) {
  using CF = Cfg<D>;
  CUtensorMap mq, mk, mv, mdo;
  const cuuint64_t dims[2] = {(cuuint64_t)a.H * D, (cuuint64_t)a.T};
  const cuuint64_t strides[1] = {(cuuint64_t)a.H * D * 2};
  const cuuint32_t box[2] = {(cuuint32_t)CF::BKD, 128u};
  const cuuint32_t es[2] = {1u, 1u};
  const CUtensorMapSwizzle sw =
      CF::SWB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  const void* ptrs[4] = {a.q, a.k, a.v, a.dout};
  CUtensorMap* maps[4] = {&mq, &mk, &mv, &mdo};
  for (int i = 0; i < 4; ++i)
    if (encode_tiled(maps[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptrs[i]),
                     dims, strides, box, es, sw) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  BwdParams p;
  p.offsets = a.offsets;
  p.ts = a.ts;
  p.w_pos = a.w_pos;
  p.w_ts = a.w_ts;
  p.dk = a.dk;
  p.dv = a.dv;
  p.dq_accum = a.dq_accum;
  p.dw_pos = a.dw_pos;
  p.dw_ts = a.dw_ts;
  p.status = a.status;
  p.B = a.B;
  p.T = a.T;
  p.P = a.P;
  p.NB = a.NB;
  p.H = a.H;
  p.scale = a.scale;
  p.wtab = a.P <= CF::PTAB ? 1 : 0;
  const int64_t bound = a.max_seq_len > 0 ? a.max_seq_len : a.T;
  p.levels = (int)((bound + kBM - 1) / kBM);
  if (p.levels < 1) p.levels = 1;
  const int64_t blocks = (int64_t)p.levels * a.B * a.H;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const int64_t n = a.T * a.H * D;
  cudaError_t e = cudaMemsetAsync(a.dq_accum, 0, sizeof(float) * n, stream);
  if (e != cudaSuccess) return e;
  static_assert(sizeof(Smem<D>) + 1024 <= 232448, "shared memory budget (227 KB per CTA)");
  size_t smem = sizeof(Smem<D>) + 1024;
  if (smem < 120 * 1024) smem = 120 * 1024;  // one CTA per SM (all TMEM columns)
  static bool attr_set = false;
  if (!attr_set) {
    e = cudaFuncSetAttribute(hstu_bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  count_launch();
  hstu_bwd_kernel<D><<<(unsigned)blocks, kThreads, smem, stream>>>(mq, mk, mv, mdo, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t n4 = n / 4;
  int64_t grid = (n4 + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 16;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  count_launch();
  dq_convert_kernel<<<(unsigned)grid, 256, 0, stream>>>(a.dq_accum,
                                                        static_cast<uint16_t*>(a.dq), n4);
  return cudaGetLastError();
}

}  // namespace

cudaError_t attn_bwd_launch(const AttnArgs& a, cudaStream_t stream) {
  switch (a.D) {
    case 32: return launch_bwd_t<32>(a, stream);
    case 64: return launch_bwd_t<64>(a, stream);
    case 128: return launch_bwd_t<128>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hstu
