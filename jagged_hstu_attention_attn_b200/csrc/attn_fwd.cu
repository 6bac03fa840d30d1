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
// Warp roles (640 threads):
//   warps 0-15: epilogue, four warpgroups in two teams.  Team t (warpgroups
//               t and t + 2) handles the key tiles n = t (mod 2); tile n lives
//               in TMEM S buffer n mod 3, so while both teams work the tensor
//               core already fills the third buffer.  Warpgroup half h of a
//               team takes key columns [64 h, 64 h + 64).  Thread r owns
//               query row r = TMEM lane r.  It reads the fp32 S row from
//               TMEM, adds the gathered bias, applies scale, SiLU
//               (tanh.approx) and the causal / ragged mask, and writes P back
//               into TMEM as bf16 hi + lo parts (P = hi + lo to ~2^-17).
//   warp 16   : TMA producer for the Q tile and the K ring; warp 19 for the
//               V ring.
//   warp 17   : TMEM allocator and tcgen05.mma issuer (whole warp, one
//               elected lane): S_n = Q K_n^T (SS form) into buffer n % 3,
//               then O += P_hi V_n + P_lo V_n (TS form, P read from TMEM).
//   warp 18   : per-tile metadata: key timestamps (int64 and 32-bit relative),
//               flags for the bias fast paths, and the relative-position bias
//               window of the tile, pre-multiplied by scale / 2.
// There is no softmax, so there is no running max / sum and no rescaling of
// the O accumulator: O lives in TMEM for the whole CTA.
//
// Bias fast paths, chosen per (row, tile), all exact:
//   w_pos : constant w_pos[P-1] when the whole row of the tile is clamped,
//           else four shifted copies of the tile's window give float4 reads.
//   w_ts  : one bucket for the row when the tile's timestamps are monotone and
//           the buckets of its first and last key agree; else 32-bit relative
//           timestamps with bfind when they fit; else the 64-bit bucket.
//
// TMEM columns (512 allocated): S0 [0,128) S1 [128,256) S2 [256,384)
// O [384,384+D).  P of buffer b overwrites the S columns of b chunk by chunk
// once they have been read: for each 32-key chunk, 16 columns of P_hi then
// 16 of P_lo.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace hstu {
namespace {

constexpr int kBM = 128;          // queries per tile
constexpr int kBN = 128;          // keys per tile
constexpr int kEpiWarps = 16;      // four warpgroups: two teams of two
constexpr int kThreads = 640;      // 16 epilogue warps + Q/K producer + MMA + meta + V producer
constexpr int kProducerWarp = 16;  // Q and K tiles
constexpr int kMmaWarp = 17;
constexpr int kMetaWarp = 18;
constexpr int kVWarp = 19;         // V tiles
constexpr int kTeamThreads = 256;  // the epilogue threads of one tile
constexpr int kEpiThreads = 32 * kEpiWarps;
// Registers: 96 per thread (640 x 96 <= 65536) is enough for every role, so
// there is no per-warpgroup split (a 104 / 64 split spilled in the control
// warps).
constexpr int kLaunchRegs = 96;
constexpr int kMetaStages = 4;
constexpr int kWts = 65;          // int64 differences reach buckets 0..64 only
constexpr uint32_t kTmemCols = 512;
constexpr int kSBuf = 3;           // S / P buffers in TMEM
constexpr uint32_t kColO = 384;
// Row stride of the four shifted copies of a per-tile w_pos window: 264 = 8
// mod 32 puts copy s on banks shifted by 8 s, so the four rows of a lane quad
// (same base, copies 0..3) read distinct banks with 16-byte loads.
constexpr int kWinStride = 264;

template <int D>
struct Cfg {
  static constexpr int BKD = D < 64 ? D : 64;        // elements per swizzle row
  static constexpr int NKB = D / BKD;                // swizzle blocks along d
  static constexpr int SWB = BKD * 2;                // swizzle row bytes (64 or 128)
  static constexpr uint32_t LAYOUT = SWB == 128 ? 2u : 4u;
  static constexpr int BLOCK_BYTES = 128 * SWB;      // 128 rows x one swizzle block
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int STAGES = D == 128 ? 2 : 3;
  static constexpr int PTAB = D == 128 ? 3328 : 4096;  // largest P kept whole in smem
  static constexpr int WT = PTAB + 264;                 // entries per shifted copy
};

struct TileMeta {
  int64_t t_first;   // timestamp of the first key (also the 32-bit base)
  int64_t t_last;    // timestamp of the last valid key
  int64_t row0;
  int pos0;
  int valid;
  int mono;          // timestamps non-decreasing over the valid keys
  int rel32;         // every |t_j - t_first| < 2^30
};

template <int D>
struct __align__(1024) Smem {
  uint8_t q[Cfg<D>::TILE_BYTES];
  uint8_t k[Cfg<D>::STAGES][Cfg<D>::TILE_BYTES];
  uint8_t v[Cfg<D>::STAGES][Cfg<D>::TILE_BYTES];
  // relative-position bias, pre-multiplied by scale / 2, stored in reverse
  // (later columns of a row, i.e. smaller relative positions, at higher
  // addresses) so one 16-byte load gives four consecutive columns in order,
  // as four shifted copies (copy s starts s entries later) so that load is
  // aligned for every row: either the whole table (P <= Cfg::PTAB, built once
  // per CTA) or, for larger P, per-tile windows built by the metadata warp.
  union {
    float wtab[4][Cfg<D>::WT];
    float wwin[kMetaStages][4][kWinStride];
  };
  int64_t ts[kMetaStages][kBN];
  int32_t ts32[kMetaStages][kBN];
  TileMeta meta[kMetaStages];
  float wts_s[68];                   // w_ts * scale / 2 (buckets 0..64)
  float wts_tbl[36];                 // [1 + k] = wts_s[min(k, NB-1)], k = -1..32
  uint64_t q_full;
  uint64_t k_full[Cfg<D>::STAGES];
  uint64_t k_empty[Cfg<D>::STAGES];
  uint64_t v_full[Cfg<D>::STAGES];
  uint64_t v_empty[Cfg<D>::STAGES];
  uint64_t meta_full[kMetaStages];
  uint64_t meta_empty[kMetaStages];
  uint64_t s_full[kSBuf];
  uint64_t p_full[kSBuf];
  uint64_t o_full;
  uint32_t tmem_base;
  int abort_flag;
};

struct FwdParams {
  const int64_t* offsets;
  const int64_t* num_targets;  // candidates at the end of each sequence, or null
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
  int cand_only;  // with num_targets: only the query tiles holding candidates, only their rows written
  int64_t max_len;  // bound on every sequence length (max_seq_len, else T)
  int wtab;     // 1: whole w_pos table in shared memory; 0: per-tile windows
  int64_t group;  // (sequence, head) pairs per group of the grid order
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
  int qt;          // plain: index of the query tile (= its diagonal key tile)
  int lh;          // plain: history length L - num_targets (candidates from here on)
  int h;
  int valid;
};

struct KTile {
  int64_t row0;
  int pos0;
  int valid;
};

// Grid order: the (sequence, head) pairs are taken in groups of p.group;
// within a group the blocks run level by level, heaviest query tiles first,
// the group's pairs fastest.  A group's K and V fit in L2, so the blocks
// running at the same time share their key tiles there; with one group
// (everything fits anyway) this is plain longest-first order.
__device__ __forceinline__ Work decode_work(const FwdParams& p, int64_t id) {
  Work w;
  w.valid = 0;
  const int H = p.H;
  const int64_t B = p.B;
  const int64_t npairs = B * H;
  int64_t t;  // level slot
  int b;
  if (p.group >= npairs) {
    // one group: level by level over all pairs
    w.h = (int)(id % H);
    t = id / H;
    b = (int)(t % B);
    t /= B;
  } else {
    const int64_t nslots = p.C == 0 ? (int64_t)p.levels : (int64_t)p.levels * 2 * p.C;
    const int64_t g = id / (p.group * nslots);
    const int64_t rem = id - g * p.group * nslots;
    const int64_t gsize = imin64(p.group, npairs - g * p.group);
    t = rem / gsize;
    const int64_t pair = g * p.group + (rem - t * gsize);
    w.h = (int)(pair % H);
    b = (int)(pair / H);
  }
  const int64_t o0 = p.offsets[b], o1 = p.offsets[b + 1];
  const int64_t L = o1 - o0;
  if (o0 < 0 || L <= 0 || o1 > p.T) return w;
  w.seq_off = o0;
  if (p.C == 0) {
    const int lvl = (int)t;
    const int64_t ntiles = (L + kBM - 1) / kBM;
    // candidates-only: the levels count the sequence's tiles from its end
    const int qt = p.cand_only ? (int)(ntiles - 1) - lvl : p.levels - 1 - lvl;
    if (qt < 0 || qt >= ntiles) return w;
    // Target-aware mask: rows from L_h = L - num_targets on are candidates
    // that see the history and themselves only, so the key tiles past the
    // history other than the diagonal one are never needed.
    int64_t nt = 0;
    if (p.num_targets != nullptr) {
      nt = p.num_targets[b];
      if (nt < 0 || nt > L) {
        report(p.status, HSTU_ERR_SHAPE);
        return w;
      }
    }
    const int64_t lh = L - nt;
    // candidates-only: tiles without a candidate row have nothing to write
    if (p.cand_only && (nt == 0 || (int64_t)qt * kBM + kBM <= lh)) return w;
    const int64_t nhist = (lh + kBN - 1) / kBN;
    w.m = L;
    w.TC = 0;
    w.q_pos0 = qt * kBM;
    w.q_row0 = o0 + w.q_pos0;
    w.q_count = (int)imin64((int64_t)kBM, L - w.q_pos0);
    w.nkv = (int)imin64((int64_t)qt, nhist) + 1;
    w.tpc = 0;
    w.qt = qt;
    w.lh = (int)lh;
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
    w.qt = 0;
    w.lh = 0x7fffffff;  // no candidates
  }
  w.valid = 1;
  return w;
}

__device__ __forceinline__ KTile key_tile(const FwdParams& p, const Work& w, int n) {
  KTile k;
  if (p.C == 0) {
    // the last tile visited is the diagonal one (tile qt); the others are
    // tiles 0, 1, ... (all of them without candidates)
    k.pos0 = (n == w.nkv - 1 ? w.qt : n) * kBN;
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

// Entries of the reversed whole w_pos table this CTA builds (nx = 3 mod 4).
__device__ __forceinline__ int wtab_rows(const Work& w, const FwdParams& p) {
  const int64_t doffmax = imin64((int64_t)w.q_pos0 + (kBM - 1), p.P + 126);
  const int nx = (int)doffmax + 131;
  return nx + ((3 - nx) & 3);
}


// Per (row, tile) context of the epilogue.  Table addresses are 32-bit
// shared-memory addresses.
struct RowCtx {
  uint32_t wrow;         // w_pos entries of the row: a 16-byte load at wrow + 4 c gives columns c..c+3
  uint32_t ts32;         // 32-bit relative key timestamps of the tile
  uint32_t ts64;         // key timestamps of the tile (int64)
  uint32_t tbl;          // tbl[k] = scaled w_ts[min(k + 1, NB - 1)] for k = bfind = -1..31
  uint32_t wts_s;        // scaled w_ts
  int64_t t_i;
  float hs;              // scale / 2
  float wpc;             // scaled w_pos[P-1]
  float wtc;             // scaled w_ts of the row's single bucket
  int ti_rel;            // t_i - t_first when it fits
  int nbm1;
  int cmax;              // last unmasked column
  int cself;             // candidate rows: the column of the row's own key (else -1)
};

enum { kTsConst = 0, kTsRel32 = 1, kTsFull = 2 };

// 32 columns (one TMEM load) of one row: P = SiLU(scale (S + bias)), split
// into bf16 hi / lo pairs.  Packed fp32x2 arithmetic, two columns per
// instruction: h = S scale/2 + bias scale/2, P = h + h tanh(h) = SiLU(x).
template <bool MASK, bool POS_CONST, int TS_MODE>
__device__ __forceinline__ void compute_chunk(const uint32_t (&sv)[32], uint32_t (&hi)[16],
                                              uint32_t (&lo)[16], int cc, const RowCtx& rc) {
  const uint64_t HS2 = f2_make(rc.hs, rc.hs);
  const uint64_t WT2 = f2_make(rc.wtc, rc.wtc);
  const float hb = rc.wpc + rc.wtc;
  const uint64_t HB2 = f2_make(hb, hb);
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    const int c0 = cc * 32 + g * 4;
    uint64_t B01, B23;
    if (POS_CONST && TS_MODE == kTsConst) {
      B01 = B23 = HB2;
    } else {
      float wp[4], wt[4];
      if (POS_CONST) {
        wp[0] = wp[1] = wp[2] = wp[3] = rc.wpc;
      } else {
        const float4 w4 = lds_f32x4(rc.wrow + (uint32_t)(c0 * 4));
        wp[0] = w4.x; wp[1] = w4.y; wp[2] = w4.z; wp[3] = w4.w;
      }
      if (TS_MODE == kTsConst) {
        B01 = f2_add(f2_make(wp[0], wp[1]), WT2);
        B23 = f2_add(f2_make(wp[2], wp[3]), WT2);
      } else {
        if (TS_MODE == kTsRel32) {
          const int4 t4 = lds_s32x4(rc.ts32 + (uint32_t)(c0 * 4));
          wt[0] = lds_f32(rc.tbl + (uint32_t)(bfind_u32((uint32_t)max(rc.ti_rel - t4.x, 0)) * 4));
          wt[1] = lds_f32(rc.tbl + (uint32_t)(bfind_u32((uint32_t)max(rc.ti_rel - t4.y, 0)) * 4));
          wt[2] = lds_f32(rc.tbl + (uint32_t)(bfind_u32((uint32_t)max(rc.ti_rel - t4.z, 0)) * 4));
          wt[3] = lds_f32(rc.tbl + (uint32_t)(bfind_u32((uint32_t)max(rc.ti_rel - t4.w, 0)) * 4));
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            wt[e] = lds_f32(rc.wts_s +
                            (uint32_t)(bucket_of(rc.t_i, lds_s64(rc.ts64 + (uint32_t)((c0 + e) * 8)),
                                                 rc.nbm1) * 4));
        }
        B01 = f2_add(f2_make(wp[0], wp[1]), f2_make(wt[0], wt[1]));
        B23 = f2_add(f2_make(wp[2], wp[3]), f2_make(wt[2], wt[3]));
      }
    }
    const uint64_t H01 = f2_fma(f2_bits(sv[g * 4], sv[g * 4 + 1]), HS2, B01);
    const uint64_t H23 = f2_fma(f2_bits(sv[g * 4 + 2], sv[g * 4 + 3]), HS2, B23);
    float h[4];
    f2_split(H01, h[0], h[1]);
    f2_split(H23, h[2], h[3]);
    uint64_t P01 = f2_fma(H01, f2_make(tanh_approx(h[0]), tanh_approx(h[1])), H01);
    uint64_t P23 = f2_fma(H23, f2_make(tanh_approx(h[2]), tanh_approx(h[3])), H23);
    if (MASK) {
      float pv[4];
      f2_split(P01, pv[0], pv[1]);
      f2_split(P23, pv[2], pv[3]);
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (c0 + e > rc.cmax && c0 + e != rc.cself) pv[e] = 0.f;
      P01 = f2_make(pv[0], pv[1]);
      P23 = f2_make(pv[2], pv[3]);
    }
    // P_hi = bf16(P); P_lo = bf16(P - P_hi), P - P_hi exact in fp32
    const uint32_t h01 = f2_to_bf16x2(P01), h23 = f2_to_bf16x2(P23);
    hi[g * 2] = h01;
    hi[g * 2 + 1] = h23;
    lo[g * 2] = f2_to_bf16x2(f2_sub(P01, f2_bits(h01 << 16, h01 & 0xFFFF0000u)));
    lo[g * 2 + 1] = f2_to_bf16x2(f2_sub(P23, f2_bits(h23 << 16, h23 & 0xFFFF0000u)));
  }
}

template <bool MASK>
__device__ __forceinline__ void compute_chunk_dispatch(int variant, const uint32_t (&sv)[32],
                                                       uint32_t (&hi)[16], uint32_t (&lo)[16],
                                                       int cc, const RowCtx& rc) {
  switch (variant) {
    case 0: compute_chunk<MASK, true, kTsConst>(sv, hi, lo, cc, rc); break;
    case 1: compute_chunk<MASK, true, kTsRel32>(sv, hi, lo, cc, rc); break;
    case 2: compute_chunk<MASK, true, kTsFull>(sv, hi, lo, cc, rc); break;
    case 3: compute_chunk<MASK, false, kTsConst>(sv, hi, lo, cc, rc); break;
    case 4: compute_chunk<MASK, false, kTsRel32>(sv, hi, lo, cc, rc); break;
    default: compute_chunk<MASK, false, kTsFull>(sv, hi, lo, cc, rc); break;
  }
}

template <int D, bool OUT_F32>
__device__ __forceinline__ void store_out_cols(const FwdParams& p, int64_t orow, int col0,
                                               const uint32_t* ov, int ncols) {
  if (OUT_F32) {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow + col0);
    for (int i = 0; i < ncols / 4; ++i)
      dst[i] = make_float4(__uint_as_float(ov[4 * i]), __uint_as_float(ov[4 * i + 1]),
                           __uint_as_float(ov[4 * i + 2]), __uint_as_float(ov[4 * i + 3]));
  } else {
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + orow + col0);
    for (int i = 0; i < ncols / 8; ++i) {
      uint4 u;
      u.x = pack_bf16x2(__uint_as_float(ov[8 * i + 0]), __uint_as_float(ov[8 * i + 1]));
      u.y = pack_bf16x2(__uint_as_float(ov[8 * i + 2]), __uint_as_float(ov[8 * i + 3]));
      u.z = pack_bf16x2(__uint_as_float(ov[8 * i + 4]), __uint_as_float(ov[8 * i + 5]));
      u.w = pack_bf16x2(__uint_as_float(ov[8 * i + 6]), __uint_as_float(ov[8 * i + 7]));
      dst[i] = u;
    }
  }
}

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
    validate_offsets(p.offsets, p.B, p.T, p.C, p.max_len, p.status);

  const Work w = decode_work(p, blockIdx.x);
  if (!w.valid) return;  // uniform over the CTA

  const float hs = 0.5f * p.scale;
  const int nbm1 = (int)(p.NB - 1 < 64 ? p.NB - 1 : 64);
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
      mbar_init(&s.meta_empty[i], kTeamThreads);
    }
    for (int i = 0; i < kSBuf; ++i) {
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.p_full[i], kTeamThreads);
    }
    mbar_init(&s.o_full, 1);
    s.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  volatile int* abort_flag = &s.abort_flag;

  if (warp >= kEpiWarps) {
  if (warp == kProducerWarp || warp == kVWarp) {
    // ------------------------------------------------------------ TMA producers
    // Warp 16 loads Q and the K ring, warp 19 the V ring, so a V tile that is
    // still waiting for its P.V product never holds back the next K tile.
    // Each whole warp runs its loop (waits stay warp-uniform); one elected
    // lane issues each copy.
    const bool is_k = warp == kProducerWarp;
    if (lane == 0) {
      tma_prefetch_desc(is_k ? &tm_k : &tm_v);
      if (is_k) tma_prefetch_desc(&tm_q);
    }
    __syncwarp();
    const int xh = w.h * D;
    if (is_k) {
      mbar_arrive_expect_tx_elect(&s.q_full, CF::TILE_BYTES);
#pragma unroll
      for (int kb = 0; kb < CF::NKB; ++kb)
        tma_load_2d_elect(s.q + kb * CF::BLOCK_BYTES, &tm_q, &s.q_full, xh + kb * CF::BKD,
                          (int32_t)w.q_row0);
    }
    uint64_t* full = is_k ? s.k_full : s.v_full;
    uint64_t* empty = is_k ? s.k_empty : s.v_empty;
    uint8_t* ring = is_k ? &s.k[0][0] : &s.v[0][0];
    const CUtensorMap* map = is_k ? &tm_k : &tm_v;
    for (int n = 0; n < w.nkv; ++n) {
      const int st = n % CF::STAGES;
      const uint32_t ph = (uint32_t)(n / CF::STAGES) & 1u;
      const KTile kt = key_tile(p, w, n);
      if (n >= CF::STAGES) {
        const bool ok =
            __all_sync(0xffffffffu, mbar_wait(&empty[st], ph ^ 1u, abort_flag, p.status));
        if (!ok) break;
      }
      mbar_arrive_expect_tx_elect(&full[st], CF::TILE_BYTES);
#pragma unroll
      for (int kb = 0; kb < CF::NKB; ++kb)
        tma_load_2d_elect(ring + st * CF::TILE_BYTES + kb * CF::BLOCK_BYTES, map, &full[st],
                          xh + kb * CF::BKD, (int32_t)kt.row0);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop and computes the (uniform) operands; one
    // elected lane issues every tcgen05.mma / commit.
    constexpr uint32_t idesc_s = idesc_bf16(kBM, kBN, false, false);
    constexpr uint32_t idesc_o = idesc_bf16(kBM, D, false, true);
    // Base descriptors are built once; each MMA adds a compile-time offset
    // (in 16-byte units) to the start-address field, and a ring stage adds
    // st * TILE_BYTES / 16.
    const uint64_t q_desc = smem_desc(smem_u32(s.q), 16, 8 * CF::SWB, CF::LAYOUT);
    const uint64_t k_desc0 = smem_desc(smem_u32(s.k[0]), 16, 8 * CF::SWB, CF::LAYOUT);
    const uint64_t v_desc0 = smem_desc(smem_u32(s.v[0]), CF::BLOCK_BYTES, 8 * CF::SWB, CF::LAYOUT);
    bool ok = __all_sync(0xffffffffu, mbar_wait(&s.q_full, 0, abort_flag, p.status));
    tc_fence_after();
    // Every operand of an MMA is kept warp-uniform so it can live in uniform
    // registers: the ring stages, buffers and phases below are counters the
    // whole warp advances together (not derived from the per-thread work
    // decode), and the TMEM base is the constant 0 (this CTA allocated all
    // 512 columns, so its allocation starts at lane 0, column 0; a different
    // base is reported and the CTA winds down).  Operands in per-thread
    // registers cost several register-to-uniform moves per MMA, and the MMA
    // issue rate of this warp bounds the kernel.
    if (tmem != 0) {
      report(p.status, HSTU_ERR_UNSUPPORTED);
      *abort_flag = 1;
      ok = false;
    }
    constexpr uint32_t kT0 = 0;  // TMEM base
    uint32_t kst = 0, kph = 0;   // K ring: stage and phase of the next S
    uint32_t sbuf = 0;           // S buffer of the next S
    uint32_t vst = 0, vph = 0;   // V ring: stage and phase of the next P.V
    uint32_t pbuf = 0, pph = 0;  // P buffer and phase of the next P.V
    bool first_pv = true;
    // P of buffer b lives in the S columns of b: for each 32-key chunk c the
    // first 16 columns hold P_hi (bf16 pairs), the next 16 P_lo.
    auto issue_pv = [&]() -> bool {
      bool w_ok = mbar_wait(&s.p_full[pbuf], pph, abort_flag, p.status);
      if (w_ok) w_ok = mbar_wait(&s.v_full[vst], vph, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, w_ok)) return false;
      tc_fence_after();
      const uint64_t v_desc = v_desc0 + (uint64_t)(vst * (CF::TILE_BYTES >> 4));
      const uint32_t pbase = kT0 + pbuf * 128;
      // K step kk (16 keys): P_hi at chunk kk / 2, half kk % 2; P_lo 16 columns on
      const auto poff = [](int kk) { return (uint32_t)(32 * (kk >> 1) + 8 * (kk & 1)); };
      const auto voff = [](int kk) { return (uint64_t)((kk * 16 * CF::SWB) >> 4); };
      mma_ts_ksteps<idesc_o, kBN / 16>(kT0 + kColO, pbase, v_desc, poff, voff,
                                       first_pv ? 0u : 1u);
      mma_ts_ksteps<idesc_o, kBN / 16>(kT0 + kColO, pbase + 16, v_desc, poff, voff, 1u);
      mma_commit_elect(&s.v_empty[vst]);
      first_pv = false;
      if (++vst == (uint32_t)CF::STAGES) { vst = 0; vph ^= 1u; }
      if (++pbuf == (uint32_t)kSBuf) { pbuf = 0; pph ^= 1u; }
      return true;
    };
    // S_n goes into buffer n % 3 once P.V of tile n - 3 (same buffer) is issued;
    // the tensor pipe runs them in order.
    for (int n = 0; ok && n < w.nkv; ++n) {
      if (n >= kSBuf) {
        ok = issue_pv();
        if (!ok) break;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&s.k_full[kst], kph, abort_flag, p.status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t k_desc = k_desc0 + (uint64_t)(kst * (CF::TILE_BYTES >> 4));
      const uint32_t s_tmem = kT0 + sbuf * 128;
      // K step k = kb * (BKD / 16) + kk: feature block kb, 16 features kk
      const auto off = [](int k) {
        return (uint64_t)(((k / (CF::BKD / 16)) * CF::BLOCK_BYTES + (k % (CF::BKD / 16)) * 32) >>
                          4);
      };
      mma_ss_ksteps<idesc_s, D / 16>(s_tmem, q_desc, k_desc, off, off, 0u);
      mma_commit_elect(&s.k_empty[kst]);
      mma_commit_elect(&s.s_full[sbuf]);
      if (++kst == (uint32_t)CF::STAGES) { kst = 0; kph ^= 1u; }
      if (++sbuf == (uint32_t)kSBuf) sbuf = 0;
    }
    for (int m = w.nkv > kSBuf ? w.nkv - kSBuf : 0; ok && m < w.nkv; ++m) ok = issue_pv();
    mma_commit_elect(&s.o_full);

  } else if (warp == kMetaWarp) {
    // ------------------------------------------------------------ tile metadata
    // The next tile's timestamps are requested before the current tile is
    // processed, so the global-load latency overlaps one tile of work.
    bool ok = true;
    int64_t tv[4];
    KTile kt = key_tile(p, w, 0);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = lane + 32 * i;
      tv[i] = __ldg(p.ts + kt.row0 + (c < kt.valid ? c : kt.valid - 1));
    }
    for (int n = 0; n < w.nkv; ++n) {
      const int ms = n % kMetaStages;
      if (n >= kMetaStages) {
        ok = mbar_wait(&s.meta_empty[ms], ((uint32_t)(n / kMetaStages) & 1u) ^ 1u, abort_flag,
                       p.status);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      int64_t tn[4];
      KTile kn = kt;
      if (n + 1 < w.nkv) {
        kn = key_tile(p, w, n + 1);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c = lane + 32 * i;
          tn[i] = __ldg(p.ts + kn.row0 + (c < kn.valid ? c : kn.valid - 1));
        }
      }
      if (!p.wtab) {
        // per-tile window, reversed: V[y] = hs * w_pos[clamp(q_pos0 - k_pos0 + 127 - y)]
        // stored as wwin[sft][y - sft]; row r reads column c at V[127 - r + c]
        const int64_t base = (int64_t)(w.q_pos0 - kt.pos0) + 127;
        for (int idx = lane; idx < 1024; idx += 32) {
          const int sft = idx >> 8, x = idx & 255;
          int64_t rel = base - (x + sft);
          rel = rel < 0 ? 0 : (rel > p.P - 1 ? p.P - 1 : rel);
          s.wwin[ms][sft][x] = __ldg(p.w_pos + rel) * hs;
        }
      }
      const int64_t t_first = __shfl_sync(0xffffffffu, tv[0], 0);
      const int last = kt.valid - 1;
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
        // next key's timestamp: lane + 1 of the same group, or lane 0 of the next group
        const int64_t nxt_same = __shfl_down_sync(0xffffffffu, tv[i], 1);
        const int64_t nxt_grp = __shfl_sync(0xffffffffu, tv[i < 3 ? i + 1 : 3], 0);
        const int64_t nxt = lane < 31 ? nxt_same : nxt_grp;
        if (c + 1 < kt.valid && tv[i] > nxt) mono = false;
      }
      mono = __all_sync(0xffffffffu, mono);
      rel32 = __all_sync(0xffffffffu, rel32);
      if (lane == 0) {
        TileMeta& m = s.meta[ms];
        m.t_first = t_first;
        m.t_last = t_last;
        m.row0 = kt.row0;
        m.pos0 = kt.pos0;
        m.valid = kt.valid;
        m.mono = mono ? 1 : 0;
        m.rel32 = rel32 ? 1 : 0;
      }
      __syncwarp();
      mbar_arrive(&s.meta_full[ms]);
      if (n + 1 < w.nkv) {
#pragma unroll
        for (int i = 0; i < 4; ++i) tv[i] = tn[i];
        kt = kn;
      }
    }
  }
  } else {
    // ------------------------------------------------------------ epilogue
    // The epilogue's tables are built here, while the producers load the
    // first Q / K / V tiles and the tensor core computes the first S, and
    // the 512 epilogue threads meet at a named barrier before the first tile.
    //
    // Whole w_pos table: W[x] = hs * w_pos[clamp(x - 127, 0, P - 1)] for the x
    // this CTA can read, reversed as V[y] = W[nx - 1 - y] and stored as
    // wtab[s][y - s].  A row whose column 0 sits at relative position doff
    // (clamped to [0, P + 126]) reads column c at V[nx - 128 - doff + c].
    // nx = 3 (mod 4) makes the four rows of a lane quad share one 16-byte
    // aligned base (copies 3, 2, 1, 0), so with WT = 8 (mod 32) the 8 lanes of
    // one phase of a 16-byte shared load hit distinct banks.  All of a
    // thread's loads are issued before its stores.
    if (p.wtab) {
      const int nx = wtab_rows(w, p);
      constexpr int kIt = (CF::WT + kEpiThreads - 1) / kEpiThreads;
      float val[kIt];
#pragma unroll
      for (int it = 0; it < kIt; ++it) {
        const int y = (int)threadIdx.x + it * kEpiThreads;
        int64_t rel = (int64_t)(nx - 1 - y) - 127;
        rel = rel < 0 ? 0 : (rel > p.P - 1 ? p.P - 1 : rel);
        val[it] = y < nx ? __ldg(p.w_pos + rel) * hs : 0.f;
      }
#pragma unroll
      for (int it = 0; it < kIt; ++it) {
        const int y = (int)threadIdx.x + it * kEpiThreads;
        if (y < nx) {
#pragma unroll
          for (int sft = 0; sft < 4; ++sft) {
            const int ys = y - sft;
            if (ys >= 0 && ys < CF::WT) s.wtab[sft][ys] = val[it];
          }
        }
      }
    }
    for (int i = threadIdx.x; i < kWts; i += kEpiThreads)
      s.wts_s[i] = (i < p.NB ? p.w_ts[i] : 0.f) * hs;
    for (int i = threadIdx.x; i < 34; i += kEpiThreads) {
      const int k = i;  // bitlen = i, table index i (bfind + 1)
      const int b = k < nbm1 ? k : nbm1;
      s.wts_tbl[i] = (b < p.NB ? p.w_ts[b] : 0.f) * hs;
    }
    named_bar_sync(1, kEpiThreads);
    // Team t = (warp >> 2) & 1 takes the key tiles n = t (mod 2); within a
    // team, warpgroup half h = warp >> 3 takes key columns [64 h, 64 h + 64)
    // (two chunks of 32) and drains O columns [h D/2 + t D/4, + D/4).
    const int team = (warp >> 2) & 1;
    const int half = warp >> 3;
    const int r = threadIdx.x & 127;    // query row = TMEM lane
    const bool row_ok = r < w.q_count;
    const int64_t q_row = w.q_row0 + r;
    const int qpos = w.q_pos0 + r;
    const int64_t t_i = row_ok ? __ldg(p.ts + q_row) : __ldg(p.ts + w.q_row0);
    const float wpc = __ldg(p.w_pos + (p.P - 1)) * hs;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    RowCtx rc;
    rc.hs = hs;
    rc.wpc = wpc;
    rc.t_i = t_i;
    rc.nbm1 = nbm1;
    rc.wts_s = smem_u32(s.wts_s);
    rc.tbl = smem_u32(s.wts_tbl + 1);
    bool ok = true;
    for (int n = team; n < w.nkv; n += 2) {
      const int ms = n % kMetaStages;
      // the tile's metadata arrives before its S: the modes are worked out
      // while the tensor core is still computing S
      ok = __all_sync(0xffffffffu, mbar_wait(&s.meta_full[ms], (uint32_t)(n / kMetaStages) & 1u,
                                             abort_flag, p.status));
      if (!ok) break;
      const int sb = n % kSBuf;
      const TileMeta tmeta = s.meta[ms];
      // candidates (rows from L_h on) take position L_h for their bias, where a
      // separate pass over the history and the candidate puts them
      const bool cand = qpos >= w.lh;
      const int rel0 = (cand ? w.lh : qpos) - tmeta.pos0;  // relative position at column 0
      // Variants are chosen per warp (all lanes must agree), so no warp runs two.
      const bool pos_const =
          __all_sync(0xffffffffu, (int64_t)rel0 - (64 * half + 63) >= p.P - 1);
      bool lane_const = false, lane_fit = false;
      if (tmeta.mono) {
        const int b1 = bucket_of(t_i, tmeta.t_first, nbm1);
        const int b2 = bucket_of(t_i, tmeta.t_last, nbm1);
        if (b1 == b2) {
          lane_const = true;
          rc.wtc = s.wts_s[b1];
        }
      }
      if (tmeta.rel32) {
        const int64_t d = t_i - tmeta.t_first;
        if (d > -(1ll << 30) && d < (1ll << 30)) {
          lane_fit = true;
          rc.ti_rel = (int)d;
        }
      }
      const int ts_mode = __all_sync(0xffffffffu, lane_const) ? kTsConst
                          : __all_sync(0xffffffffu, lane_fit) ? kTsRel32 : kTsFull;
      const int variant = (pos_const ? 0 : 3) + ts_mode;
      const bool need_mask = (tmeta.pos0 + kBN - 1 > w.q_pos0) || tmeta.valid < kBN ||
                             (w.q_pos0 + w.q_count > w.lh && tmeta.pos0 + tmeta.valid > w.lh);
      rc.cmax = min(tmeta.valid - 1, cand ? rel0 - 1 : rel0);
      // only candidates keep their own column past cmax (in the paired layout a
      // row's own position can fall in a tile's columns beyond its chunk)
      rc.cself = cand ? qpos - tmeta.pos0 : -1;
      if (p.wtab) {
        // rows whose whole tile is clamped read entries that all hold w_pos[P-1]
        // A candidate's own column reads the entry of relative position
        // L_h - qpos <= 0 (base L_h - pos0 where the tile holds history keys,
        // else 0 with no history column), i.e. w_pos[0]: its bias to itself.
        const int doff = rel0 < 0 ? 0 : (rel0 < (int)(p.P + 126) ? rel0 : (int)(p.P + 126));
        const int y0 = wtab_rows(w, p) - 128 - doff;
        const int sft = y0 & 3;
        rc.wrow = smem_u32(&s.wtab[sft][0]) + (uint32_t)(4 * (y0 - sft));
      } else {
        const int y0 = 127 - r;
        const int sft = y0 & 3;
        rc.wrow = smem_u32(&s.wwin[ms][sft][0]) + (uint32_t)(4 * (y0 - sft));
      }
      rc.ts32 = smem_u32(s.ts32[ms]);
      rc.ts64 = smem_u32(s.ts[ms]);
      const uint32_t s_col = tmem + lane_base + sb * 128;
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&s.s_full[sb], (uint32_t)(n / kSBuf) & 1u, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      // The thread's two chunks of 32 keys, one TMEM load each (four warps
      // per SM sub-partition hide the load latency); P_hi / P_lo of a chunk
      // go into its own S columns, which have been read by then.
#pragma unroll 1
      for (int k = 0; k < 2; ++k) {
        const int cc = 2 * half + k;
        uint32_t ra[32];
        tmem_ld32(s_col + cc * 32, ra);
        tmem_wait_ld(ra);
        uint32_t hi[16], lo[16];
        if (need_mask) compute_chunk_dispatch<true>(variant, ra, hi, lo, cc, rc);
        else compute_chunk_dispatch<false>(variant, ra, hi, lo, cc, rc);
        __syncwarp();
        tmem_st16(s_col + cc * 32, hi);
        tmem_st16(s_col + cc * 32 + 16, lo);
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
      constexpr int kQuarter = D / 4;  // columns drained by each warpgroup
      const int c_begin = half * (D / 2) + team * kQuarter;
#pragma unroll 1
      for (int c = c_begin; c < c_begin + kQuarter; c += 8) {
        uint32_t ov[8];
        tmem_ld8(tmem + lane_base + kColO + c, ov);
        tmem_wait_ld(ov);
        if (row_ok && (!p.cand_only || qpos >= w.lh)) store_out_cols<D, OUT_F32>(p, orow, c, ov, 8);
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
  p.num_targets = a.C == 0 ? a.num_targets : nullptr;
  p.cand_only = (a.C == 0 && a.num_targets != nullptr && a.cand_only) ? 1 : 0;
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
  p.wtab = a.P <= Cfg<D>::PTAB ? 1 : 0;
  // the per-tile windows follow the rows' own positions: no candidates there
  if (a.num_targets != nullptr && !p.wtab) return cudaErrorNotSupported;
  const int64_t bound = a.max_seq_len > 0 ? a.max_seq_len : a.T;
  p.max_len = bound;
  int64_t groups;
  if (a.C == 0) {
    p.levels = (int)((bound + kBM - 1) / kBM);
    if (p.cand_only && a.max_targets > 0) {
      // the candidate rows of a sequence span at most ceil(max_targets / 128) + 1 tiles
      const int64_t lv = (a.max_targets + kBM - 1) / kBM + 1;
      if (lv < p.levels) p.levels = (int)lv;
    }
    groups = a.B;
  } else {
    const int64_t mmax = (bound + 2 * a.C - 1) / (2 * a.C);
    p.levels = (int)((mmax + kBM - 1) / kBM);
    groups = a.B * 2 * a.C;
  }
  if (p.levels < 1) p.levels = 1;
  // pairs per group of the grid order: all of them when the batch's K and V
  // fit in half of L2, else as many as have their K and V there
  {
    const int64_t npairs = a.B * a.H;
    const int64_t half_l2 = 64ll << 20;
    const int64_t pair_kv = (bound > 0 ? bound : 1) * D * 4;  // K and V rows, bf16
    p.group = npairs;
    if (a.T * a.H * D * 4 > half_l2) {
      const int64_t gp = half_l2 / pair_kv;
      p.group = gp < 1 ? 1 : (gp < npairs ? gp : npairs);
    }
    if (p.group < 1) p.group = 1;
  }
  const int64_t blocks = (int64_t)p.levels * groups * a.H;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  // Each CTA allocates all 512 TMEM columns, so ask for enough shared memory
  // that a second CTA never becomes resident on the same SM.
  static_assert(sizeof(Smem<D>) + 1024 <= 232448, "shared memory budget (227 KB per CTA)");
  size_t smem = sizeof(Smem<D>) + 1024;
  if (smem < 120 * 1024) smem = 120 * 1024;
  static DeviceFlags attr_done;  // per template instance and device
  int slot = -1;
  if (!device_flag_set(attr_done, &slot)) {
    // 640 threads need at most kLaunchRegs registers each
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, hstu_fwd_kernel<D, OUT_F32>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs > kLaunchRegs) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(hstu_fwd_kernel<D, OUT_F32>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    device_flag_mark(attr_done, slot);
  }
  count_launch();
  hstu_fwd_kernel<D, OUT_F32><<<(unsigned)blocks, kThreads, smem, stream>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

}  // namespace

int64_t attn_fwd_targets_max_P(int D) { return D == 128 ? Cfg<128>::PTAB : Cfg<64>::PTAB; }

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
