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
// One CTA owns one (key tile of 128 rows, head) of one sequence and walks the
// queries at or after it in steps of 64.  Step n uses TMEM buffer n % 2, so
// the tensor core computes step n + 1's products while the epilogue works on
// step n:
//   MMA warp   : S^T = K Q^T and dP^T = V dO^T (M = 128 keys, N = 64 queries);
//   epilogue   : 16 warps (four per TMEM lane quadrant), thread (group g,
//                lane r) owns key row r and query columns [16 g, 16 g + 16):
//                P^T = SiLU(x) (bf16) and dS^T = gs (bf16) written into
//                128B-swizzled shared-memory tiles (D <= 64; for D = 128 P^T
//                goes back into TMEM over the S^T columns already read, as
//                shared memory has no room for its tiles); bias-gradient partials
//                accumulated on the fly (registers for the clamped w_pos entry
//                and for runs of one w_ts bucket; warp-shuffle diagonal sums
//                for the other w_pos entries, added straight to global memory);
//   MMA warp   : dQ^T = K^T dS^T and dK += dS^T Q, then dV += P^T dO.
//                With P^T in shared memory the TMEM buffer of step n is free
//                once the epilogue has loaded it, so step n + 2's S^T / dP^T
//                are issued right then, ahead of step n's dQ / dK / dV, and
//                the epilogue never waits for them;
//   drain warps: 4 warps move dQ^T (TMEM lane = feature, column = query) to
//                a shared staging tile, and one TMA reduce-add per step adds it
//                to the fp32 workspace.
// dK / dV stay in TMEM for the whole CTA and are written once at the end.
// TMEM columns: buffer b: S^T [128 b, 128 b + 64) (for D = 128, P^T of group
// g packed into the first 8 of its own 16 columns, [128 b + 16 g, +8)), dP^T
// [128 b + 64, 128 b + 128); dK [256, 256 + D), dV [256 + D, 256 + 2 D); dQ^T
// of step n in the dP^T columns of buffer n % 2 (D = 128) or in
// [256 + 2 D + 64 (n % 2), +64) (D <= 64).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace hstu {
namespace {

constexpr int kBM = 128;           // keys per CTA tile (TMEM lanes)
constexpr int kBN = 64;            // queries per step
constexpr int kEpiWarps = 16;      // four warps per TMEM lane quadrant
constexpr int kTW = 16;            // query columns of one half step of an epilogue thread
constexpr int kDrainWarps = 4;     // one per TMEM lane quadrant
constexpr int kThreads = 768;      // 16 epilogue + 4 drain warps + producer, idle, meta, MMA
// Registers: launched at 80 per thread (the largest multiple of 8 with
// 768 x R <= 65536); the four epilogue warpgroups raise theirs to kEpiRegs,
// the drain warpgroup sets kDrainRegs and the control warpgroup lowers its
// own to kCtlRegs: 4 * 128 * 88 + 128 * 64 + 128 * 64 = 61440 = 768 * 80.
constexpr int kLaunchRegs = 80;
constexpr uint32_t kEpiRegs = 88;
constexpr uint32_t kDrainRegs = 64;
constexpr uint32_t kCtlRegs = 64;
static_assert(4 * 128 * kEpiRegs + 128 * kDrainRegs + 128 * kCtlRegs <= kThreads * kLaunchRegs,
              "register split");
constexpr int kDrainWarp0 = kEpiWarps;  // warps 16..19 (TMEM lane quadrants 0..3)
// Warp w runs on SM sub-partition w % 4, next to the epilogue and drain
// warps of TMEM lane quadrant w % 4.  The epilogue warps that share a
// sub-partition with the MMA warp fall behind the others (measured: ~2500
// cycles a step), so it goes where the drain warp is idle for D <= 64
// (quadrant 3: dQ^T has D feature rows) and the idle warp sits on quadrant 1.
constexpr int kProducerWarp = kEpiWarps + kDrainWarps;  // quadrant 0
constexpr int kMetaWarp = kProducerWarp + 2;            // quadrant 2
constexpr int kMmaWarp = kProducerWarp + 3;             // quadrant 3
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kWin = 192;          // w_pos window entries per shifted copy (64 + 127, padded)
// Row stride of the four shifted copies: 200 = 6 * 32 + 8 puts copy s on
// banks shifted by 8 s, so the 8 lanes of one phase of a 16-byte shared load
// (two rows of four consecutive key rows, one copy each) hit distinct banks;
// with a stride of 192 the four lanes of a quad collided 4 ways.
constexpr int kWinStride = 200;
constexpr int kWts = 65;
// Relative-position gradients are summed per CTA in a shared-memory ring of
// kRing floats indexed by rel mod kRing; a slot holding relative position rel
// is added to dw_pos[min(rel, P - 1)] when it is flushed, so blocks whose
// relative positions straddle the clamp need no per-pair test (blocks that
// are clamped throughout use a register accumulator instead).  Step n touches rel in
// [64 n - 127, 64 n + 63], so once every epilogue thread is done with step
// m, every rel below 64 m - 63 is final: the metadata warp flushes
// [64 m - 127, 64 m - 63) to global memory (and clears it) before it prepares
// step m + META (having waited for step m to be consumed), while the epilogue
// is at most at step m + META - 1 <= m + 3 and long before any step reuses
// those slots (rel + kRing is first touched by step m + 6), and the epilogue
// flushes the rest when the CTA ends.
constexpr int kRing = 512;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColDK = 256;
constexpr uint64_t kQuiesceNs = 200000000ull;  // 0.2 s

template <int D>
struct Cfg {
  static constexpr int BKD = D < 64 ? D : 64;     // features per swizzle block
  static constexpr int NKB = D / BKD;
  static constexpr int SWB = BKD * 2;             // bytes per row of a block
  static constexpr uint32_t LAYOUT = SWB == 128 ? 2u : 4u;
  static constexpr int KBLOCK = kBM * SWB;        // one block of a 128-row tile
  static constexpr int QBLOCK = kBN * SWB;        // one block of a 64-row tile
  static constexpr int KTILE = kBM * D * 2;
  static constexpr int QTILE = kBN * D * 2;
  // For D <= 64, P^T goes to shared memory (dV an SS product like dK), so
  // the S^T / dP^T buffer of step n is free as soon as the epilogue has read
  // it and step n + 2's products go in right then, ahead of step n's dQ / dK /
  // dV; four Q / dO stages keep step n + 2's tiles loaded by then.  For
  // D = 128 shared memory has no room: P^T is written over the S^T columns.
  static constexpr bool PT_SMEM = D <= 64;
  static constexpr int STAGES = PT_SMEM ? 4 : 3;
  // per-step metadata stages (timestamps, w_pos window): with four the
  // metadata warp runs up to three steps ahead of the epilogue, which
  // otherwise waited for it at the top of most steps; D = 128 has room for two
  static constexpr int META = D <= 64 ? 4 : 2;
  static constexpr uint32_t COL_DV = kColDK + D;
  // For D <= 64 there is room for dQ^T of its own (two 64-column buffers
  // after dV), so the next step's S^T / dP^T never wait for the drain; for
  // D = 128 dQ^T of step n goes into the dP^T columns of buffer n % 2.
  static constexpr bool DQ_OWN = kColDK + 2 * D + 2 * 64 <= 512;
  // dS^T tiles and dQ staging tiles: two of each where shared memory allows
  // (D <= 64), so the epilogue never waits for the MMAs of the previous step
  // to release the dS^T tile and the drain never waits for the previous TMA
  // reduction to finish reading its stage.
  static constexpr int DS_BUF = D <= 64 ? 2 : 1;
  static constexpr int DQ_BUF = D <= 64 ? 2 : 1;
  // drain warps with dQ^T rows (TMEM lane quadrants below D); the others skip
  // the per-step loop, whose waits would only take issue slots from the
  // epilogue warps of their sub-partition (measured on fixed 8192, d = 64:
  // -1.3 % for the backward)
  static constexpr int DRAIN_ACTIVE = (D + 31) / 32;
  // Epilogue teams.  TEAMS = 2 (possible with P^T in shared memory: two S^T /
  // dP^T buffers, two dS^T tiles) splits the 16 epilogue warps into two teams
  // of 8 (two per TMEM lane quadrant); team t takes the steps n = t (mod 2)
  // and every thread covers 32 of a step's 64 query columns in two halves of
  // kTW, which halves the per-step work (modes, waits, arrivals) per pair.
  // Measured on the fixed-8192 backward (d = 64) it was 1.5 % slower than
  // one team (the second half's TMEM load is exposed and the buffer is
  // released later), so all 16 warps share every step, 16 columns each.
  static constexpr int TEAMS = 1;
  static constexpr int HALVES = TEAMS;             // kTW-column halves per thread and step
  static constexpr int TEAM_THREADS = kEpiThreads / TEAMS;
  static __device__ __forceinline__ uint32_t col_dq(int buf) {
    return DQ_OWN ? kColDK + 2 * D + 64 * buf : 128 * buf + 64;
  }
};

// P^T tiles in shared memory, laid out like the dS^T tiles (D <= 64 only).
// The member sits last in Smem so that, where it is absent, no other
// member moves (the TMA source and destination offsets stay as they are).
template <bool ON>
struct PtTiles {
  alignas(1024) uint8_t b[2][kBM * kBN * 2];
};
template <>
struct PtTiles<false> {
  uint8_t b[1][16];
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
  uint8_t k[Cfg<D>::KTILE];
  // v directly follows k: for D < 128 the dQ^T product reads 128 rows of
  // K^T, and the rows past D land in v (their results are never used)
  uint8_t v[Cfg<D>::KTILE];
  uint8_t q[Cfg<D>::STAGES][Cfg<D>::QTILE];
  uint8_t dout[Cfg<D>::STAGES][Cfg<D>::QTILE];
  uint8_t dst[Cfg<D>::DS_BUF][kBM * kBN * 2];  // dS^T [key][query], one 64-query swizzle block
  float dq_stage[Cfg<D>::DQ_BUF][kBN * D];     // dQ of one step, [query][feature], TMA reduction
  float wwin[Cfg<D>::META][4][kWinStride];  // [s][x] = hs * w_pos[clamp(64 n - 127 + x + s)]
  int64_t ts[Cfg<D>::META][kBN];
  int32_t ts32[Cfg<D>::META][kBN];
  QMeta meta[Cfg<D>::META];
  float dwts[68 * 8];              // w_ts gradient partials, [bucket][lane % 8]
  float ring[kRing];               // w_pos gradient partials, [rel mod kRing]
  float wts_s[68];
  float wts_tbl[36];
  uint64_t kv_full;
  uint64_t qdo_full[Cfg<D>::STAGES];
  uint64_t qdo_empty[Cfg<D>::STAGES];
  uint64_t meta_full[Cfg<D>::META];
  uint64_t meta_empty[Cfg<D>::META];
  uint64_t st_full[2];
  uint64_t st_free[2];             // the epilogue has read S^T / dP^T of the buffer (D <= 64)
  uint64_t ds_full[2];
  uint64_t ds_free[Cfg<D>::DS_BUF];
  uint64_t dq_full[2];
  uint64_t dq_free[2];
  uint64_t stage_full[Cfg<D>::DQ_BUF];  // the drain warps wrote dq_stage
  uint64_t stage_free[Cfg<D>::DQ_BUF];  // the TMA unit has read dq_stage
  uint64_t kv_done;
  uint64_t epi_sync;               // the 256 epilogue threads meet here once, at the end
  uint32_t tmem_base;
  int abort_flag;
  PtTiles<Cfg<D>::PT_SMEM> pt;
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
  int64_t group;  // (sequence, head) pairs per group of the grid order
  float scale;
};

struct BWork {
  int64_t seq_off;
  int64_t L;
  int kt;      // key tile index
  int kvalid;  // valid key rows
  int nq;      // 64-query steps from the tile's first key to the end of the sequence
  int h;
  int valid;
};

// Grid order: (sequence, head) pairs in groups of p.group; within a group the
// blocks run key tile by key tile, the heaviest (first) tiles first, the
// group's pairs fastest, so the blocks in flight share the Q, dO rows and dQ
// accumulator rows of a few pairs in L2.  One group is the plain order.
__device__ __forceinline__ BWork decode_bwork(const BwdParams& p, int64_t id) {
  BWork w;
  w.valid = 0;
  const int64_t npairs = p.B * p.H;
  int kt, b;
  if (p.group >= npairs) {
    // one group: key tile by key tile over all pairs
    w.h = (int)(id % p.H);
    const int64_t t = id / p.H;
    b = (int)(t % p.B);
    kt = (int)(t / p.B);
  } else {
    const int64_t g = id / (p.group * p.levels);
    const int64_t rem = id - g * p.group * p.levels;
    const int64_t gsize = imin64(p.group, npairs - g * p.group);
    kt = (int)(rem / gsize);
    const int64_t pair = g * p.group + (rem - (int64_t)kt * gsize);
    w.h = (int)(pair % p.H);
    b = (int)(pair / p.H);
  }
  const int64_t o0 = p.offsets[b], o1 = p.offsets[b + 1];
  const int64_t L = o1 - o0;
  if (o0 < 0 || L <= 0 || o1 > p.T) return w;
  const int64_t ntiles = (L + kBM - 1) / kBM;
  if (kt >= ntiles) return w;
  w.seq_off = o0;
  w.L = L;
  w.kt = kt;
  w.kvalid = (int)imin64((int64_t)kBM, L - (int64_t)kt * kBM);
  w.nq = (int)((L - (int64_t)kt * kBM + kBN - 1) / kBN);
  w.valid = 1;
  return w;
}

__device__ __forceinline__ int qvalid_of(const BWork& w, int n) {
  return (int)imin64((int64_t)kBN, w.L - (int64_t)w.kt * kBM - (int64_t)n * kBN);
}

enum { kTsConst = 0, kTsRel32 = 1, kTsFull = 2 };

// No "memory" clobber on the reductions: their targets are only read after
// the epilogue's final mbarrier sync (shared) or by later kernels (global),
// and a clobber would stop the compiler from scheduling the unrolled per-pair
// loop around them.
__device__ __forceinline__ void red_shared_add(uint32_t addr, float v) {
  asm volatile("red.shared.add.f32 [%0], %1;" ::"r"(addr), "f"(v));
}
// the same, issued only where pred holds, as a predicated instruction (no branch)
__device__ __forceinline__ void red_shared_add_if(bool pred, uint32_t addr, float v) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %2, 0;\n\t"
      "@p red.shared.add.f32 [%0], %1;\n\t}\n" ::"r"(addr),
      "f"(v), "r"((int)pred));
}
__device__ __forceinline__ void red_global_add(float* addr, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(addr), "f"(v));
}

// Every gradient the epilogue forms is carried without the factor scale / 2:
// G = dP * 2 SiLU'(x), so that dS^T = (scale / 2) G.  dK, dQ, dw_pos and
// dw_ts are multiplied by scale / 2 once, where they leave the kernel.
//
// With h = x / 2 and t = tanh(h):  SiLU(x) = h (1 + t)  and
// 2 SiLU'(x) = (1 + t) + SiLU(x) (1 - t)  (from sigmoid(x) = (1 + t) / 2).
// One pair of columns in packed fp32x2 arithmetic: 9 instructions including
// the two tanh, plus the two bf16 packs.
__device__ __forceinline__ void silu_pair(uint32_t s0, uint32_t s1, uint32_t d0, uint32_t d1,
                                          uint64_t HS2, uint64_t B2, uint64_t ONE2,
                                          uint64_t& P2, uint64_t& G2) {
  const uint64_t H2 = f2_fma(f2_bits(s0, s1), HS2, B2);  // h = x / 2
  float h0, h1;
  f2_split(H2, h0, h1);
  const uint64_t TH2 = f2_make(tanh_approx(h0), tanh_approx(h1));
  const uint64_t E2 = f2_add(TH2, ONE2);  // 1 + t
  P2 = f2_mul(H2, E2);                    // SiLU(x)
  const uint64_t F2 = f2_sub(ONE2, TH2);  // 1 - t
  const uint64_t X2 = f2_fma(P2, F2, E2); // 2 SiLU'(x)
  G2 = f2_mul(f2_bits(d0, d1), X2);
}

// 16-byte store of 8 bf16 (4 packed words) into row r, 16-byte chunk `chunk`
// (0..7 over 64 columns) of a [128][64] bf16 tile in 128B-swizzled K-major
// layout.
__device__ __forceinline__ void st_swizzled(uint32_t tile, int r, int chunk, uint32_t w0,
                                            uint32_t w1, uint32_t w2, uint32_t w3) {
  const uint32_t dst = tile + (uint32_t)(r * 128 + ((chunk ^ (r & 7)) << 4));
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(w0), "r"(w1), "r"(w2),
               "r"(w3)
               : "memory");
}

// Per-thread view of one half step (thread = key row r, kTW query columns).
struct BStep {
  uint32_t ta;           // TMEM address of the thread's first S^T column (dP^T at +64)
  uint32_t dst;          // shared address of the dS^T tile
  uint32_t pdst;         // shared address of the P^T tile (P^T in shared memory)
  uint64_t* st_free;     // arrived on once the thread's S^T / dP^T are read (idem)
  uint64_t* ds_free;     // nullptr: the dS^T tile is free already
  uint32_t ds_parity;
  uint32_t ring;         // shared address of the w_pos gradient ring
  uint32_t wrow;         // shared address: hs * w_pos of the thread's column c at +4 c
  uint32_t ts32;         // shared address: query timestamps relative to t_first (int32)
  uint32_t tbl;          // shared address: scaled w_ts by bfind index + 1 (0..32)
  uint32_t ts64;         // shared address: query timestamps of the thread's columns (int64)
  uint32_t wts_s;        // shared address: scaled w_ts
  volatile int* abort_flag;
  int* status;
  int64_t t_j;
  float hs;
  float wpc;             // hs * w_pos[P - 1]
  float wtc;             // hs * w_ts of the thread's single bucket (constant mode)
  float keep;            // 0 on lanes 0 and 1 (they start new diagonals), 1 elsewhere
  int r;
  int chunk0;            // first 16-byte chunk of the thread's columns in a dS^T row
  int lane;
  int src2;              // lane - 2 (mod 32)
  int base_w;            // relative position of the warp's diagonal 0 (lane 0, column 0)
  int rel0;              // relative position of the thread's column 0
  int pm1;               // P - 1 (capped)
  int nbm1;
  int tj_rel;            // t_j - t_first when it fits in 31 bits
  int bconst;            // the thread's bucket in constant mode (the first one when split)
  int bsecond;           // split mode: the bucket of the columns from the split on
  int tthr;              // split mode: columns with ts32 < tthr are in bucket bconst
  float wtc2;            // split mode: hs * w_ts[bsecond]
  int cmin, cmax;        // unmasked columns
};

struct BiasAcc {
  float pclamp;   // G summed over pairs clamped at w_pos[P-1]
  float run;      // current run of one w_ts bucket
  int cur;        // bucket of the run (-1: none)
};

// The view of half hf of a thread's step: kTW columns further on.
__device__ __forceinline__ BStep half_of(const BStep& io, int hf) {
  BStep h = io;
  const int c = kTW * hf;
  h.ta += (uint32_t)c;
  h.wrow += (uint32_t)(4 * c);
  h.ts32 += (uint32_t)(4 * c);
  h.ts64 += (uint32_t)(8 * c);
  h.chunk0 += c >> 3;
  h.base_w += c;
  h.rel0 += c;
  h.cmin -= c;
  h.cmax -= c;
  return h;
}

// Runs are flushed into one of 8 copies of the bucket table (chosen by lane),
// so lanes of a warp that close a run of the same bucket together rarely hit
// the same address.  acc.cur may be a bit length above NB - 1 (the 32-bit path
// keys runs on the raw bit length), hence the clamp.
__device__ __forceinline__ void flush_run(BiasAcc& acc, float* s_dwts, int nbm1) {
  if (acc.cur >= 0 && acc.run != 0.f)
    red_shared_add(smem_u32(&s_dwts[min(acc.cur, nbm1) * 8]), acc.run);
  acc.run = 0.f;
}

__device__ __forceinline__ bool wait_ds_free(const BStep& io) {
  return io.ds_free == nullptr ||
         __all_sync(0xffffffffu, mbar_wait(io.ds_free, io.ds_parity, io.abort_flag, io.status));
}

// the thread has read its S^T / dP^T columns (P^T in shared memory only)
template <bool PTS>
__device__ __forceinline__ void release_st(const BStep& io) {
  if (PTS) {
    tc_fence_before();
    mbar_arrive(io.st_free);
  }
}

// Store P^T (8 packed words: over the thread's first 8 S^T columns, or two
// 16-byte chunks of its P^T row in shared memory) and dS^T (two 16-byte chunks
// of its dS^T row).  The first half step of a step waits until the tiles are
// free (wait_ds).
template <bool PTS>
__device__ __forceinline__ bool store_step(const BStep& io, const uint32_t (&pw)[kTW / 2],
                                           const uint32_t (&gw)[kTW / 2], bool wait_ds) {
  if (!PTS) {
    tmem_st4(io.ta, pw[0], pw[1], pw[2], pw[3]);
    tmem_st4(io.ta + 4, pw[4], pw[5], pw[6], pw[7]);
  }
  if (wait_ds && !wait_ds_free(io)) return false;
  if (PTS) {
    st_swizzled(io.pdst, io.r, io.chunk0, pw[0], pw[1], pw[2], pw[3]);
    st_swizzled(io.pdst, io.r, io.chunk0 + 1, pw[4], pw[5], pw[6], pw[7]);
  }
  st_swizzled(io.dst, io.r, io.chunk0, gw[0], gw[1], gw[2], gw[3]);
  st_swizzled(io.dst, io.r, io.chunk0 + 1, gw[4], gw[5], gw[6], gw[7]);
  return true;
}

// Unmasked step in one of the common configurations.  The relative
// positions of the warp's block are all clamped at P - 1 (WIN = false: one
// w_pos entry, whose gradient is the plain sum) or not (WIN = true: per-column
// window entries, which hold the clamped values where rel >= P - 1, and
// diagonal chains into the ring, whose flush clamps the destination).  The query
// timestamps of this row fall in one bucket (SPLIT = false) or, monotone, in
// two consecutive buckets bconst | bsecond, the second from the first column
// whose 32-bit relative timestamp reaches tthr on (SPLIT = true; rows with one
// bucket take tthr = INT_MAX).  Returns the sum of G over the thread's columns
// (gsum) and, when SPLIT, the part of it in bucket bconst (glo).
//
// The w_pos gradient of the warp's 32 x kTW block goes through two rotating
// chains, one per column parity e: before each column c of parity e (after the
// first) every lane takes lane l - 2's running sum, so lane l always adds into
// the sum of its own diagonal c - l.  Lanes 0 and 1 receive from lanes 30 and
// 31 the sums of diagonals c - 32 and c - 33 of that parity, which are
// complete by then (their next pair of the same parity would be on lane 32 or
// 33): they add them to the ring and start afresh.  After the last column of
// its parity, chain e holds diagonal kTW - 2 + e - l on lane l.  Each
// diagonal is the sum of the two chains' shares, which meet in the ring.
// up / lo parity chains (no shared-memory atomics per column): pairs with
// c >= lane go to the up chain, the others to the lo chain; both rotate by two
// lanes before each column of their parity.
struct Chains {
  float up[2], lo[2];
};

__device__ __forceinline__ void chain_col(Chains& ch, float g, int c, const BStep& io) {
  const int e = c & 1;
  if (c >= 2) {
    ch.up[e] = __shfl_sync(0xffffffffu, ch.up[e], io.src2);
    ch.lo[e] = __shfl_sync(0xffffffffu, ch.lo[e], io.src2);
  }
  if (c >= io.lane) ch.up[e] += g;
  else ch.lo[e] += g;
}

// one more rotation by one lane merges the parities: lane l < kTW then holds
// diagonal kTW - 1 - l (up) and -kTW - 1 - l (lo), lane l >= kTW diagonal
// kTW - 1 - l (lo)
__device__ __forceinline__ void chain_end(const Chains& ch, const BStep& io) {
  const float u = ch.up[1] + __shfl_sync(0xffffffffu, ch.up[0], (io.lane - 1) & 31);
  const float l = ch.lo[1] + __shfl_sync(0xffffffffu, ch.lo[0], (io.lane - 1) & 31);
  const bool low = io.lane < kTW;
  red_shared_add_if(low, io.ring + (uint32_t)(((io.base_w + kTW - 1 - io.lane) & (kRing - 1)) * 4), u);
  const int dl = low ? -kTW - 1 - io.lane : kTW - 1 - io.lane;
  red_shared_add_if(io.lane != kTW - 1,
                    io.ring + (uint32_t)(((io.base_w + dl) & (kRing - 1)) * 4), l);
}

// A half step: last_half releases the TMEM buffer once its columns are read,
// first_half waits for the shared-memory tiles before it stores.
template <bool WIN, bool SPLIT, bool PTS>
__device__ __forceinline__ bool step_fast(const BStep& io, float& gsum, float& glo,
                                          bool last_half, bool first_half) {
  uint32_t sv[kTW], dv[kTW];
  tmem_ld16(io.ta, sv);
  tmem_ld16(io.ta + 64, dv);
  tmem_wait_ld(sv);
  tmem_wait_ld(dv);
  if (last_half) release_st<PTS>(io);
  const uint64_t ONE2 = f2_make(1.f, 1.f);
  const uint64_t HS2 = f2_make(io.hs, io.hs);
  const uint64_t WT2 = f2_make(io.wtc, io.wtc);
  const uint64_t WP2 = f2_make(io.wpc, io.wpc);
  const float hb = io.wpc + io.wtc;
  const uint64_t HB2 = f2_make(hb, hb);
  uint32_t pw[kTW / 2], gw[kTW / 2];
  uint64_t GS2 = f2_make(0.f, 0.f);
  float lo_acc = 0.f;
  Chains ch = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
  for (int q = 0; q < kTW / 4; ++q) {
    uint64_t B01, B23;
    bool m[4];
    if (SPLIT) {
      const int4 t4 = lds_s32x4(io.ts32 + (uint32_t)(16 * q));
      m[0] = t4.x < io.tthr; m[1] = t4.y < io.tthr; m[2] = t4.z < io.tthr; m[3] = t4.w < io.tthr;
      const uint64_t T01 = f2_make(m[0] ? io.wtc : io.wtc2, m[1] ? io.wtc : io.wtc2);
      const uint64_t T23 = f2_make(m[2] ? io.wtc : io.wtc2, m[3] ? io.wtc : io.wtc2);
      if (WIN) {
        const float4 w4 = lds_f32x4(io.wrow + (uint32_t)(16 * q));
        B01 = f2_add(f2_make(w4.x, w4.y), T01);
        B23 = f2_add(f2_make(w4.z, w4.w), T23);
      } else {
        B01 = f2_add(WP2, T01);
        B23 = f2_add(WP2, T23);
      }
    } else if (WIN) {
      const float4 w4 = lds_f32x4(io.wrow + (uint32_t)(16 * q));
      B01 = f2_add(f2_make(w4.x, w4.y), WT2);
      B23 = f2_add(f2_make(w4.z, w4.w), WT2);
    } else {
      B01 = B23 = HB2;
    }
    uint64_t P2a, G2a, P2b, G2b;
    silu_pair(sv[4 * q], sv[4 * q + 1], dv[4 * q], dv[4 * q + 1], HS2, B01, ONE2, P2a, G2a);
    silu_pair(sv[4 * q + 2], sv[4 * q + 3], dv[4 * q + 2], dv[4 * q + 3], HS2, B23, ONE2, P2b, G2b);
    GS2 = f2_add(GS2, f2_add(G2a, G2b));
    pw[2 * q] = f2_to_bf16x2(P2a);
    pw[2 * q + 1] = f2_to_bf16x2(P2b);
    gw[2 * q] = f2_to_bf16x2(G2a);
    gw[2 * q + 1] = f2_to_bf16x2(G2b);
    if (SPLIT || WIN) {
      float g[4];
      f2_split(G2a, g[0], g[1]);
      f2_split(G2b, g[2], g[3]);
      if (SPLIT) {
#pragma unroll
        for (int e = 0; e < 4; ++e) lo_acc += m[e] ? g[e] : 0.f;
      }
      if (WIN) {
#pragma unroll
        for (int e = 0; e < 4; ++e) chain_col(ch, g[e], 4 * q + e, io);
      }
    }
  }
  if (WIN) chain_end(ch, io);
  float a, b;
  f2_split(GS2, a, b);
  gsum = a + b;
  glo = lo_acc;
  return store_step<PTS>(io, pw, gw, first_half);
}

// Any other step: masks, relative positions on both sides of P - 1 or below
// 0, per-column timestamp buckets (32-bit relative or 64-bit).  A rolled loop
// over groups of 4 columns with warp-uniform mode branches keeps the code
// small.  Masked pairs give P = G = 0, so their diagonals add nothing, and
// clamped pairs feed acc.pclamp instead of the chain: every ring entry the
// chain adds to outside [0, P - 1) receives exactly 0.
template <bool PTS>
__device__ __forceinline__ bool step_general(const BStep& io, bool masked, bool pos_clamped,
                                             int ts_mode, BiasAcc& acc, float* s_dwts,
                                             bool last_half, bool first_half) {
  const uint64_t ONE2 = f2_make(1.f, 1.f);
  const uint64_t HS2 = f2_make(io.hs, io.hs);
  Chains ch = {{0.f, 0.f}, {0.f, 0.f}};
  uint32_t sc[8], dc[8];
  tmem_ld8(io.ta, sc);
  tmem_ld8(io.ta + 64, dc);
#pragma unroll 1
  for (int k = 0; k < kTW / 8; ++k) {
    tmem_wait_ld(sc, dc);
    if (last_half && k == kTW / 8 - 1) release_st<PTS>(io);
    uint32_t pk[4], gk[4];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int c0 = 8 * k + 4 * q;
      float wp[4], wt[4];
      int bk[4];
      if (pos_clamped) {
        wp[0] = wp[1] = wp[2] = wp[3] = io.wpc;
      } else {
        const float4 w4 = lds_f32x4(io.wrow + (uint32_t)(c0 * 4));
        wp[0] = w4.x; wp[1] = w4.y; wp[2] = w4.z; wp[3] = w4.w;
      }
      if (ts_mode == kTsRel32) {
        const int4 t4 = lds_s32x4(io.ts32 + (uint32_t)(c0 * 4));
        const int tq[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          // bfind + 1 = bitlen < 32 here; with NB - 1 >= 31 it is the bucket
          // itself, otherwise the run key is mapped to its bucket when flushed
          const int f = bfind_u32((uint32_t)max(tq[e] - io.tj_rel, 0));
          wt[e] = lds_f32(io.tbl + (uint32_t)(f * 4));
          bk[e] = f + 1;
        }
      } else if (ts_mode == kTsConst) {
        wt[0] = wt[1] = wt[2] = wt[3] = io.wtc;
        bk[0] = bk[1] = bk[2] = bk[3] = io.bconst;
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          bk[e] = bucket_of(lds_s64(io.ts64 + (uint32_t)((c0 + e) * 8)), io.t_j, io.nbm1);
          wt[e] = lds_f32(io.wts_s + (uint32_t)(bk[e] * 4));
        }
      }
      uint64_t P2a, G2a, P2b, G2b;
      silu_pair(sc[4 * q], sc[4 * q + 1], dc[4 * q], dc[4 * q + 1], HS2,
                f2_make(wp[0] + wt[0], wp[1] + wt[1]), ONE2, P2a, G2a);
      silu_pair(sc[4 * q + 2], sc[4 * q + 3], dc[4 * q + 2], dc[4 * q + 3], HS2,
                f2_make(wp[2] + wt[2], wp[3] + wt[3]), ONE2, P2b, G2b);
      float pv[4], gv[4];
      f2_split(P2a, pv[0], pv[1]);
      f2_split(P2b, pv[2], pv[3]);
      f2_split(G2a, gv[0], gv[1]);
      f2_split(G2b, gv[2], gv[3]);
      if (masked) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (c0 + e < io.cmin || c0 + e > io.cmax) pv[e] = gv[e] = 0.f;
      }
      pk[2 * q] = pack_bf16x2(pv[0], pv[1]);
      pk[2 * q + 1] = pack_bf16x2(pv[2], pv[3]);
      gk[2 * q] = pack_bf16x2(gv[0], gv[1]);
      gk[2 * q + 1] = pack_bf16x2(gv[2], gv[3]);
      if (pos_clamped) {
        acc.pclamp += (gv[0] + gv[1]) + (gv[2] + gv[3]);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) chain_col(ch, gv[e], c0 + e, io);
      }
      // w_ts gradient: runs of one bucket (masked pairs add zero)
      if (ts_mode == kTsConst) {
        acc.run += (gv[0] + gv[1]) + (gv[2] + gv[3]);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          // a run ends where the bucket changes; lanes flush with a predicated
          // shared-memory add behind one warp-uniform test
          const bool ch = bk[e] != acc.cur;
          if (__any_sync(0xffffffffu, ch))
            red_shared_add_if(ch && acc.cur >= 0 && acc.run != 0.f,
                              smem_u32(&s_dwts[min(acc.cur, io.nbm1) * 8]), acc.run);
          acc.run = ch ? gv[e] : acc.run + gv[e];
          acc.cur = ch ? bk[e] : acc.cur;
        }
      }
    }
    if (k + 1 < kTW / 8) {
      tmem_ld8(io.ta + 8 * (k + 1), sc);
      tmem_ld8(io.ta + 64 + 8 * (k + 1), dc);
    }
    // P^T of columns 8k .. 8k + 7 (packed): over S^T columns 4k .. 4k + 3,
    // read in group k / 2, or chunk k of the thread's P^T row in shared memory
    if (!PTS) tmem_st4(io.ta + 4 * k, pk[0], pk[1], pk[2], pk[3]);
    if (first_half && k == 0 && !wait_ds_free(io)) return false;
    if (PTS) st_swizzled(io.pdst, io.r, io.chunk0 + k, pk[0], pk[1], pk[2], pk[3]);
    st_swizzled(io.dst, io.r, io.chunk0 + k, gk[0], gk[1], gk[2], gk[3]);
  }
  if (!pos_clamped) chain_end(ch, io);
  return true;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    hstu_bwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
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
    for (int i = 0; i < CF::META; ++i) {
      mbar_init(&s.meta_full[i], 32);
      mbar_init(&s.meta_empty[i], CF::TEAM_THREADS);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.st_full[i], 1);
      mbar_init(&s.st_free[i], CF::TEAM_THREADS);
      mbar_init(&s.ds_full[i], CF::TEAM_THREADS);
      mbar_init(&s.dq_full[i], 1);
      mbar_init(&s.dq_free[i], 32 * CF::DRAIN_ACTIVE);
    }
    for (int i = 0; i < CF::DS_BUF; ++i) mbar_init(&s.ds_free[i], 1);
    for (int i = 0; i < CF::DQ_BUF; ++i) {
      mbar_init(&s.stage_full[i], 32 * CF::DRAIN_ACTIVE);
      mbar_init(&s.stage_free[i], 1);
    }
    mbar_init(&s.kv_done, 1);
    mbar_init(&s.epi_sync, kEpiThreads);
    s.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  for (int i = threadIdx.x; i < 68 * 8; i += blockDim.x) s.dwts[i] = 0.f;
  for (int i = threadIdx.x; i < kRing; i += blockDim.x) s.ring[i] = 0.f;
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
  if (warp < kEpiWarps) {
    regs_inc<kEpiRegs>();   // the four epilogue warpgroups
    // ------------------------------------------------------------ epilogue
    // team: steps n = team (mod TEAMS); query columns [cbase, cbase + TW) of
    // each, in HALVES halves of kTW
    constexpr int TW = kTW * CF::HALVES;
    const int team = CF::TEAMS == 2 ? warp >> 3 : 0;
    const int cbase = (CF::TEAMS == 2 ? (warp >> 2) & 1 : warp >> 2) * TW;
    const int r = threadIdx.x & 127;    // key row = TMEM lane
    const int r0 = r & ~31;             // key row of lane 0 of this warp
    const int etid = threadIdx.x;       // 0 .. kEpiThreads - 1
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const int64_t t_j = __ldg(p.ts + k_row0 + (r < w.kvalid ? r : w.kvalid - 1));
    const int pm1 = (int)(p.P - 1 < 0x3fffffff ? p.P - 1 : 0x3fffffff);
    float* s_dwts = s.dwts + (lane & 7);
    BStep io;
    io.dst = smem_u32(s.dst[0]);
    io.pdst = smem_u32(s.pt.b[0]);
    io.st_free = nullptr;
    io.ring = smem_u32(s.ring);
    io.tbl = smem_u32(s.wts_tbl + 1);
    io.wts_s = smem_u32(s.wts_s);
    io.abort_flag = abort_flag;
    io.status = p.status;
    io.t_j = t_j;
    io.hs = hs;
    io.wpc = __ldg(p.w_pos + (p.P - 1)) * hs;
    io.keep = lane < 2 ? 0.f : 1.f;
    io.r = r;
    io.chunk0 = cbase >> 3;
    io.lane = lane;
    io.src2 = (lane - 2) & 31;
    io.pm1 = pm1;
    io.nbm1 = nbm1;
    io.wtc = 0.f;
    io.bconst = 0;
    io.tj_rel = 0;
    BiasAcc acc;
    acc.pclamp = 0.f;
    acc.run = 0.f;
    acc.cur = -1;
    bool ok = true;
    for (int n = team; n < w.nq; n += CF::TEAMS) {
      const int X = n & 1;
      const int ms = n % CF::META;
      // the step's metadata arrives well before its S^T / dP^T: the modes are
      // worked out while the tensor core is still computing them
      ok = __all_sync(0xffffffffu, mbar_wait(&s.meta_full[ms], (uint32_t)(n / CF::META) & 1u,
                                             abort_flag, p.status));
      if (!ok) break;
      const QMeta qm = s.meta[ms];
      const int delta0 = n * kBN;              // query position 0 of the step - key position 0
      io.base_w = delta0 + cbase - r0;         // warp-uniform
      io.rel0 = io.base_w - lane;
      // warp-uniform relative-position range of the warp's 32 x TW block
      const int wrel_min = io.base_w - 31;
      const bool masked = (n <= 1) || qm.valid < kBN;
      // the constant-bucket test covers this thread's own TW columns (their
      // first and last valid timestamp)
      // per row: the buckets of its first and last valid query column; with
      // monotone timestamps they bound every bucket in between
      bool lane_const = false, lane_split = false, lane_fit = false;
      if (qm.rel32) {
        const int64_t d = t_j - qm.t_first;
        if (d > -(1ll << 30) && d < (1ll << 30)) {
          lane_fit = true;
          io.tj_rel = (int)d;
        }
      }
      if (qm.mono) {
        const int c_first = cbase < qm.valid ? cbase : qm.valid - 1;
        const int c_last = cbase + TW - 1 < qm.valid ? cbase + TW - 1 : qm.valid - 1;
        const int b1 = bucket_of(s.ts[ms][c_first], t_j, nbm1);
        const int b2 = bucket_of(s.ts[ms][c_last], t_j, nbm1);
        io.bconst = b1;
        io.wtc = s.wts_s[b1];
        io.bsecond = b1;
        io.tthr = 0x7fffffff;
        io.wtc2 = io.wtc;
        if (b1 == b2) {
          lane_const = true;
        } else if (b2 == b1 + 1 && lane_fit) {
          // columns below t_j + 2^b1 (32-bit relative) are in bucket b1
          lane_split = true;
          io.bsecond = b2;
          io.tthr = io.tj_rel + (1 << b1);
          io.wtc2 = s.wts_s[b2];
        }
      }
      const int ts_mode = __all_sync(0xffffffffu, lane_const) ? kTsConst
                          : __all_sync(0xffffffffu, lane_fit) ? kTsRel32 : kTsFull;
      const bool split_ok = ts_mode != kTsConst && __all_sync(0xffffffffu, lane_const || lane_split);
      if ((ts_mode == kTsConst || (split_ok && !masked)) && acc.cur != io.bconst) {
        flush_run(acc, s_dwts, nbm1);
        acc.cur = io.bconst;
      }
      const bool pos_clamped = wrel_min >= pm1;
      io.cmin = r - delta0 - cbase > 0 ? r - delta0 - cbase : 0;
      io.cmax = qm.valid - 1 - cbase;
      {
        const int sft = (3 - (r & 3)) & 3;
        io.wrow = smem_u32(&s.wwin[ms][sft][0] + (127 - r - sft) + cbase);
      }
      io.ts32 = smem_u32(s.ts32[ms] + cbase);
      io.ts64 = smem_u32(s.ts[ms] + cbase);
      io.ta = tmem + lane_base + 128u * (uint32_t)X + cbase;
      // dS^T tile n % DS_BUF is free once the products of step n - DS_BUF have read it
      {
        const int db = n % CF::DS_BUF;
        io.dst = smem_u32(s.dst[db]);
        io.pdst = smem_u32(s.pt.b[CF::PT_SMEM ? db : 0]);
        io.st_free = &s.st_free[X];
        io.ds_free = n >= CF::DS_BUF ? &s.ds_free[db] : nullptr;
        io.ds_parity = (uint32_t)(n / CF::DS_BUF - 1) & 1u;
      }
      const bool all_masked = masked && __all_sync(0xffffffffu, io.cmin > TW - 1 || io.cmax < 0);
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&s.st_full[X], (uint32_t)(n >> 1) & 1u, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      constexpr bool PTS = CF::PT_SMEM;
      if (all_masked) {
        // the causal mask or the sequence end removes the whole warp's chunk:
        // only its zeros are written
        release_st<PTS>(io);
        static_assert(PTS || CF::HALVES == 1, "P^T in TMEM takes one half step per step");
        if (!PTS)
#pragma unroll
          for (int k = 0; k < kTW / 8; ++k) tmem_st4(io.ta + 4 * k, 0u, 0u, 0u, 0u);
        ok = wait_ds_free(io);
        if (ok)
#pragma unroll
          for (int k = 0; k < TW / 8; ++k) {
            st_swizzled(io.dst, r, io.chunk0 + k, 0u, 0u, 0u, 0u);
            if (PTS) st_swizzled(io.pdst, r, io.chunk0 + k, 0u, 0u, 0u, 0u);
          }
      } else if (!masked && (ts_mode == kTsConst || split_ok)) {
        float gsum = 0.f, glo = 0.f;
#pragma unroll 1
        for (int hf = 0; ok && hf < CF::HALVES; ++hf) {
          const BStep ioh = half_of(io, hf);
          const bool last = hf == CF::HALVES - 1, first = hf == 0;
          float gs, gl;
          if (ts_mode == kTsConst) {
            ok = pos_clamped ? step_fast<false, false, PTS>(ioh, gs, gl, last, first)
                             : step_fast<true, false, PTS>(ioh, gs, gl, last, first);
            gl = gs;
          } else {
            ok = pos_clamped ? step_fast<false, true, PTS>(ioh, gs, gl, last, first)
                             : step_fast<true, true, PTS>(ioh, gs, gl, last, first);
          }
          gsum += gs;
          glo += gl;
        }
        if (pos_clamped) acc.pclamp += gsum;
        // bucket bconst gets glo (its run goes on); a second bucket starts a new run
        acc.run += glo;
        if (io.bsecond != io.bconst) {
          flush_run(acc, s_dwts, nbm1);
          acc.cur = io.bsecond;
          acc.run = gsum - glo;
        }
      } else {
#pragma unroll 1
        for (int hf = 0; ok && hf < CF::HALVES; ++hf)
          ok = step_general<PTS>(half_of(io, hf), masked, pos_clamped, ts_mode, acc, s_dwts,
                                 hf == CF::HALVES - 1, hf == 0);
      }
      if (!ok) break;
      if (!PTS) tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&s.ds_full[X]);
      mbar_arrive(&s.meta_empty[ms]);
    }
    flush_run(acc, s_dwts, nbm1);
    // w_pos[P-1] partial: warp sum, then one global atomic per warp
    float pc = acc.pclamp;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) pc += __shfl_xor_sync(0xffffffffu, pc, o);
    if (lane == 0 && pc != 0.f) atomicAdd(p.dw_pos + (p.P - 1), pc * hs);
    // dK, dV: thread r owns key row r, its warp's quarter of the columns
    const int grp = warp >> 2;
    if (ok) ok = mbar_wait(&s.kv_done, 0, abort_flag, p.status);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    if (ok) {
      const bool k_ok = r < w.kvalid;
      const int64_t orow = ((k_row0 + r) * p.H + w.h) * (int64_t)D;
      constexpr int kQuarter = D / 4;
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        const uint32_t col0 = which == 0 ? kColDK : CF::COL_DV;
        // dK was accumulated from G: it takes the factor scale / 2 here
        const float f = which == 0 ? hs : 1.f;
        uint16_t* out = static_cast<uint16_t*>(which == 0 ? p.dk : p.dv) + orow;
#pragma unroll 1
        for (int c = grp * kQuarter; c < (grp + 1) * kQuarter; c += 8) {
          uint32_t v8[8];
          tmem_ld8(tmem + lane_base + col0 + c, v8);
          tmem_wait_ld(v8);
          if (k_ok)
            *reinterpret_cast<uint4*>(out + c) = make_uint4(
                pack_bf16x2(__uint_as_float(v8[0]) * f, __uint_as_float(v8[1]) * f),
                pack_bf16x2(__uint_as_float(v8[2]) * f, __uint_as_float(v8[3]) * f),
                pack_bf16x2(__uint_as_float(v8[4]) * f, __uint_as_float(v8[5]) * f),
                pack_bf16x2(__uint_as_float(v8[6]) * f, __uint_as_float(v8[7]) * f));
        }
      }
    }
    // the w_ts partials and the rest of the w_pos ring -> global, once all
    // epilogue threads are done
    mbar_arrive(&s.epi_sync);
    const bool synced =
        __all_sync(0xffffffffu, mbar_wait(&s.epi_sync, 0, abort_flag, p.status));
    for (int i = etid; synced && i < kWts && i < p.NB; i += kEpiThreads) {
      float v = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) v += s.dwts[i * 8 + c];
      if (v != 0.f) atomicAdd(p.dw_ts + i, v * hs);
    }
    // ring slots hold rel in [lo, lo + kRing): everything below lo was flushed
    // by the metadata warp (see there), which got to step nq - 1 - META
    const int ring_lo = (w.nq - CF::META) * kBN - 127;
    for (int i = etid; synced && i < kRing; i += kEpiThreads) {
      const int rel = ring_lo + ((i - ring_lo) & (kRing - 1));
      const float v = s.ring[i];
      if (rel >= 0 && v != 0.f) red_global_add(p.dw_pos + min(rel, pm1), v * hs);
    }
  } else if (warp < kDrainWarp0 + kDrainWarps) {
    regs_dec<kDrainRegs>();   // the drain warpgroup
    // ------------------------------------------------------------ dQ drain
    // Warp 16 + qd reads TMEM lanes 32 qd .. 32 qd + 31 (= features) of dQ^T,
    // writes them transposed into a staging tile [query][feature], and one
    // thread adds the whole [64][D] tile to the fp32 workspace with a TMA
    // reduction (rows past the sequence receive +0: the masked dS^T entries
    // are 0).  With two staging tiles (D <= 64) the reduction of step n is
    // still reading its tile while step n + 1 is written into the other.
    const int qd = warp & 3;
    const bool has = qd * 32 < D;
    const bool issuer = threadIdx.x == kDrainWarp0 * 32;
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    int pending = 0;  // TMA reductions issued by this thread
    for (int n = 0; has && n < w.nq; ++n) {
      const int X = n & 1;
      const int sb = n % CF::DQ_BUF;
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&s.dq_full[X], (uint32_t)(n >> 1) & 1u, abort_flag, p.status)))
        break;
      tc_fence_after();
      // the reduction issued DQ_BUF steps ago must have read this stage; then
      // the 64 columns move in pieces of 16
      if (n >= CF::DQ_BUF &&
          !__all_sync(0xffffffffu, mbar_wait(&s.stage_free[sb], (uint32_t)(n / CF::DQ_BUF - 1) & 1u,
                                             abort_flag, p.status)))
        break;
      if (has) {
        float* col = s.dq_stage[sb] + qd * 32 + lane;
#pragma unroll 1
        for (int c16 = 0; c16 < kBN; c16 += 16) {
          uint32_t v16[16];
          tmem_ld16(tmem + lane_base + CF::col_dq(X) + c16, v16);
          tmem_wait_ld(v16);
#pragma unroll
          for (int c = 0; c < 16; ++c) col[(c16 + c) * D] = __uint_as_float(v16[c]);
        }
      }
      tc_fence_before();
      mbar_arrive(&s.dq_free[X]);
      fence_proxy_async_smem();
      mbar_arrive(&s.stage_full[sb]);
      if (warp == kDrainWarp0) {
        bool ok = mbar_wait(&s.stage_full[sb], (uint32_t)(n / CF::DQ_BUF) & 1u, abort_flag,
                            p.status);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        if (issuer) {
          tma_reduce_add_2d(&tm_dq, s.dq_stage[sb], w.h * D, (int32_t)(k_row0 + (int64_t)n * kBN));
          bulk_commit_group();
          ++pending;
          if (CF::DQ_BUF == 1) {
            bulk_wait_group_read0();
            mbar_arrive(&s.stage_free[0]);
          } else if (n >= 1) {
            // the reduction of step n - 1 has read its stage
            bulk_wait_group_read1();
            mbar_arrive(&s.stage_free[(n - 1) % CF::DQ_BUF]);
          }
        }
        __syncwarp();
      }
    }
    // the reductions must be complete before the CTA exits
    if (issuer && pending > 0) bulk_wait_group0();
  } else {
    // the last warpgroup: producer, idle, metadata and MMA warps
    regs_dec<kCtlRegs>();
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
      mbar_arrive_expect_tx_elect(&s.kv_full, 2 * CF::KTILE);
  #pragma unroll
      for (int kb = 0; kb < CF::NKB; ++kb) {
        tma_load_2d_elect(s.k + kb * CF::KBLOCK, &tm_k, &s.kv_full, xh + kb * CF::BKD,
                          (int32_t)k_row0);
        tma_load_2d_elect(s.v + kb * CF::KBLOCK, &tm_v, &s.kv_full, xh + kb * CF::BKD,
                          (int32_t)k_row0);
      }
      int issued = 0;
      for (int n = 0; n < w.nq; ++n) {
        const int st = n % CF::STAGES;
        const uint32_t ph = (uint32_t)(n / CF::STAGES) & 1u;
        const int64_t q_row0 = k_row0 + (int64_t)n * kBN;
        if (n >= CF::STAGES) {
          const bool ok = __all_sync(0xffffffffu,
                                     mbar_wait(&s.qdo_empty[st], ph ^ 1u, abort_flag, p.status));
          if (!ok) break;
        }
        mbar_arrive_expect_tx_elect(&s.qdo_full[st], 2 * CF::QTILE);
  #pragma unroll
        for (int kb = 0; kb < CF::NKB; ++kb) {
          tma_load_2d_elect(s.q[st] + kb * CF::QBLOCK, &tm_q, &s.qdo_full[st], xh + kb * CF::BKD,
                            (int32_t)q_row0);
          tma_load_2d_elect(s.dout[st] + kb * CF::QBLOCK, &tm_do, &s.qdo_full[st],
                            xh + kb * CF::BKD, (int32_t)q_row0);
        }
        issued = n + 1;
      }
      // Before the CTA exits, the copies it issued must have landed (they are
      // all consumed already unless the CTA is aborting).
      mbar_wait_quiesce(&s.kv_full, 0, kQuiesceNs);
      for (int i = issued > CF::STAGES ? issued - CF::STAGES : 0; i < issued; ++i)
        mbar_wait_quiesce(&s.qdo_full[i % CF::STAGES], (uint32_t)(i / CF::STAGES) & 1u,
                          kQuiesceNs);
    } else if (warp == kMmaWarp) {
      // ------------------------------------------------------------ MMA issuer
      // The whole warp runs the loop and computes the (uniform) operands; one
      // elected lane issues every tcgen05.mma / commit.
      constexpr uint32_t idesc_s = idesc_bf16(kBM, kBN, false, false);   // S^T, dP^T
      constexpr uint32_t idesc_kv = idesc_bf16(kBM, D, false, true);     // dV, dK
      constexpr uint32_t idesc_q = idesc_bf16(kBM, kBN, true, true);     // dQ^T
      // Base descriptors are built once; each MMA adds a compile-time offset
      // (16-byte units) to the start-address field, a ring stage adds
      // st * QTILE / 16.
      const uint64_t kA = smem_desc(smem_u32(s.k), 16, 8 * CF::SWB, CF::LAYOUT);       // K, K-major
      const uint64_t vA = smem_desc(smem_u32(s.v), 16, 8 * CF::SWB, CF::LAYOUT);       // V, K-major
      const uint64_t kT = smem_desc(smem_u32(s.k), CF::KBLOCK, 8 * CF::SWB, CF::LAYOUT);  // K^T, MN
      const uint64_t qK0 = smem_desc(smem_u32(s.q[0]), 16, 8 * CF::SWB, CF::LAYOUT);
      const uint64_t qM0 = smem_desc(smem_u32(s.q[0]), CF::QBLOCK, 8 * CF::SWB, CF::LAYOUT);
      const uint64_t oK0 = smem_desc(smem_u32(s.dout[0]), 16, 8 * CF::SWB, CF::LAYOUT);
      const uint64_t oM0 = smem_desc(smem_u32(s.dout[0]), CF::QBLOCK, 8 * CF::SWB, CF::LAYOUT);
      const uint64_t dsK0 = smem_desc(smem_u32(s.dst[0]), 16, 1024, 2u);      // dS^T, K-major
      const uint64_t dsN0 = smem_desc(smem_u32(s.dst[0]), 16384, 1024, 2u);   // dS^T, MN-major
      const uint64_t ptK0 = smem_desc(smem_u32(s.pt.b[0]), 16, 1024, 2u);         // P^T, K-major
      // Every operand of an MMA is kept warp-uniform so it can live in uniform
      // registers: ring stages, buffers and phases are counters the whole warp
      // advances together (not derived from the per-thread work decode), and
      // the TMEM base is the constant 0 (this CTA allocated all 512 columns, so
      // its allocation starts at lane 0, column 0; a different base is reported
      // and the CTA winds down).  Operands in per-thread registers cost several
      // register-to-uniform moves per MMA, and this warp's issue rate bounds
      // the pipeline.
      constexpr uint32_t kT0 = 0;  // TMEM base
      bool ok = true;
      if (tmem != 0) {
        report(p.status, HSTU_ERR_UNSUPPORTED);
        *abort_flag = 1;
        ok = false;
      }
      // S^T and dP^T of step m: ring stage sst, TMEM buffer sx
      auto issue_sdp = [&](uint32_t sst, uint32_t sx) {
        const uint64_t stoff = (uint64_t)(sst * (CF::QTILE >> 4));
        const uint32_t col = 128u * sx;
        // K step k = kb * (BKD / 16) + kk: feature block kb, 16 features kk
        constexpr int KS = D / 16;
        const auto koff = [](int k) {
          return (uint64_t)(((k / (CF::BKD / 16)) * CF::KBLOCK + (k % (CF::BKD / 16)) * 32) >> 4);
        };
        const auto qoff = [](int k) {
          return (uint64_t)(((k / (CF::BKD / 16)) * CF::QBLOCK + (k % (CF::BKD / 16)) * 32) >> 4);
        };
        mma_ss_ksteps<idesc_s, KS>(kT0 + col, kA, qK0 + stoff, koff, qoff, 0u);
        mma_ss_ksteps<idesc_s, KS>(kT0 + col + 64, vA, oK0 + stoff, koff, qoff, 0u);
        mma_commit_elect(&s.st_full[sx]);
      };
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&s.kv_full, 0, abort_flag, p.status));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&s.qdo_full[0], 0, abort_flag, p.status));
      if (ok) {
        tc_fence_after();
        issue_sdp(0u, 0u);
      }
      constexpr bool PTS = CF::PT_SMEM;
      // P^T in shared memory: both TMEM buffers are filled up front, and step
      // m + 2's S^T / dP^T go in once the epilogue has loaded step m's.  The
      // tcgen05 operations issued from one SM sub-partition are taken in
      // order, so an epilogue warp of the MMA warp's sub-partition whose TMEM
      // load is issued behind queued MMAs waits for them: step n's dQ / dK /
      // dV wait until the epilogue has also loaded step n + 1 (st_free), which
      // keeps every TMEM load ahead of the MMAs that follow it.
      if (PTS && ok && w.nq > 1) {
        ok = __all_sync(0xffffffffu, mbar_wait(&s.qdo_full[1], 0, abort_flag, p.status));
        if (ok) {
          tc_fence_after();
          issue_sdp(1u, 1u);
        }
      }
      if (PTS && ok && w.nq > 2) {
        ok = mbar_wait(&s.st_free[0], 0, abort_flag, p.status);
        if (ok) ok = mbar_wait(&s.qdo_full[2], 0, abort_flag, p.status);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
          tc_fence_after();
          issue_sdp(2u, 0u);
        }
      }
      // uniform counters: step n's Q/dO stage (st), buffer X and its phase xph,
      // dS^T tile db; the stage of the next S^T / dP^T (step n + 1, or n + 3 with
      // P^T in shared memory) and the phase of its wait (nst, nph)
      uint32_t st = 0, X = 0, xph = 0, db = 0;
      constexpr int kAhead = PTS ? 3 : 1;
      uint32_t nst = (uint32_t)(kAhead % CF::STAGES), nph = kAhead >= CF::STAGES ? 1u : 0u;
      bool first = true;
      for (int n = 0; ok && n < w.nq; ++n) {
        if (!PTS && n + 1 < w.nq) {
          ok = mbar_wait(&s.qdo_full[nst], nph, abort_flag, p.status);
          // the dP^T columns of buffer (n + 1) % 2 hold dQ^T of step n - 1 until it
          // is drained (D = 128 only)
          if (ok && !CF::DQ_OWN && n >= 1)
            ok = mbar_wait(&s.dq_free[X ^ 1u], xph ^ (X ^ 1u), abort_flag, p.status);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          issue_sdp(nst, X ^ 1u);
          if (++nst == (uint32_t)CF::STAGES) { nst = 0; nph ^= 1u; }
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&s.ds_full[X], xph, abort_flag, p.status))) {
          ok = false;
          break;
        }
        // step n + 1's S^T / dP^T (buffer X ^ 1) loaded by every epilogue warp
        if (PTS && n + 1 < w.nq &&
            !__all_sync(0xffffffffu,
                        mbar_wait(&s.st_free[X ^ 1u], xph ^ X, abort_flag, p.status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t col = 128u * X;
        // dQ^T = K^T dS^T  (M = 128 feature rows, N = 64 queries, K = 128 keys);
        // with its own columns, dQ^T of step n - 2 must have been drained first
        if (CF::DQ_OWN && n >= 2 &&
            !__all_sync(0xffffffffu, mbar_wait(&s.dq_free[X], xph ^ 1u, abort_flag, p.status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t dsoff = (uint64_t)((db * kBM * kBN * 2) >> 4);
        mma_ss_ksteps<idesc_q, kBM / 16>(
            kT0 + CF::col_dq(X), kT, dsN0 + dsoff,
            [](int kk) { return (uint64_t)((kk * 16 * CF::SWB) >> 4); },
            [](int kk) { return (uint64_t)((kk * 2048) >> 4); }, 0u);
        mma_commit_elect(&s.dq_full[X]);
        // dK += dS^T Q, the other reader of the dS^T tile, goes first so the
        // epilogue can write the next tile sooner; then dV += P^T dO (P^T
        // from TMEM, or from its shared-memory tile, which the same commit
        // then releases with dS^T).  K = 64 queries in 4 steps each.
        const uint64_t stoff = (uint64_t)(st * (CF::QTILE >> 4));
        const auto mnoff = [](int kk) { return (uint64_t)((kk * 16 * CF::SWB) >> 4); };
        const auto kmoff = [](int kk) { return (uint64_t)((kk * 32) >> 4); };
        mma_ss_ksteps<idesc_kv, kBN / 16>(kT0 + kColDK, dsK0 + dsoff, qM0 + stoff, kmoff, mnoff,
                                          first ? 0u : 1u);
        if (PTS) {
          mma_ss_ksteps<idesc_kv, kBN / 16>(kT0 + CF::COL_DV, ptK0 + dsoff, oM0 + stoff, kmoff,
                                            mnoff, first ? 0u : 1u);
          mma_commit_elect(&s.ds_free[db]);
        } else {
          mma_commit_elect(&s.ds_free[db]);
          mma_ts_ksteps<idesc_kv, kBN / 16>(kT0 + CF::COL_DV, kT0 + col, oM0 + stoff,
                                            [](int kk) { return (uint32_t)(16 * kk); }, mnoff,
                                            first ? 0u : 1u);
        }
        mma_commit_elect(&s.qdo_empty[st]);
        // step n + 3 into buffer X ^ 1, whose step n + 1 the epilogue has loaded
        if (PTS && n + 3 < w.nq) {
          if (!__all_sync(0xffffffffu, mbar_wait(&s.qdo_full[nst], nph, abort_flag, p.status))) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_sdp(nst, X ^ 1u);
          if (++nst == (uint32_t)CF::STAGES) { nst = 0; nph ^= 1u; }
        }
        first = false;
        if (++st == (uint32_t)CF::STAGES) st = 0;
        if (++db == (uint32_t)CF::DS_BUF) db = 0;
        X ^= 1u;
        if (X == 0) xph ^= 1u;
      }
      mma_commit_elect(&s.kv_done);
      // nothing may still be writing TMEM when it is freed
      mbar_wait_quiesce(&s.kv_done, 0, kQuiesceNs);
    } else if (warp == kMetaWarp) {
      // ------------------------------------------------------------ per-step metadata
      // The next step's timestamps are requested before the current one is
      // processed, so the load latency overlaps one step of work.
      bool ok = true;
      auto load_ts = [&](int n, int64_t (&t2)[2]) {
        const int64_t q_row0 = k_row0 + (int64_t)n * kBN;
        const int qv = qvalid_of(w, n);
  #pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int c = lane + 32 * i;
          t2[i] = __ldg(p.ts + q_row0 + (c < qv ? c : qv - 1));
        }
      };
      int64_t tv[2];
      load_ts(0, tv);
      for (int n = 0; n < w.nq; ++n) {
        const int ms = n % CF::META;
        if (n >= CF::META) {
          ok = mbar_wait(&s.meta_empty[ms], ((uint32_t)(n / CF::META) & 1u) ^ 1u, abort_flag,
                         p.status);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
        }
        if (n >= CF::META) {
          // every epilogue thread is done with step m = n - META: flush the
          // w_pos gradient entries [64 m - 127, 64 m - 63), which no later
          // step touches (step m + 1 starts at 64 (m + 1) - 127)
          const int m = n - CF::META;
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int rel = m * kBN - 127 + lane + 32 * i;
            if (rel >= 0) {
              float* slot = &s.ring[rel & (kRing - 1)];
              const float v = *slot;
              if (v != 0.f) {
                red_global_add(p.dw_pos + imin64(rel, p.P - 1), v * hs);
                *slot = 0.f;
              }
            }
          }
        }
        int64_t tn[2];
        if (n + 1 < w.nq) load_ts(n + 1, tn);
        const int qvalid = qvalid_of(w, n);
        // w_pos window; only an unmasked step whose smallest relative position
        // is already clamped never reads it
        const int64_t base = (int64_t)n * kBN - 127;
        if (base < p.P - 1 || n <= 1 || qvalid < kBN) {
  #pragma unroll
          for (int sft = 0; sft < 4; ++sft)
  #pragma unroll
            for (int i = 0; i < kWin / 32; ++i) {
              const int x = lane + 32 * i;
              int64_t rel = base + x + sft;
              rel = rel < 0 ? 0 : (rel > p.P - 1 ? p.P - 1 : rel);
              s.wwin[ms][sft][x] = __ldg(p.w_pos + rel) * hs;
            }
        }
        const int64_t t_first = __shfl_sync(0xffffffffu, tv[0], 0);
        const int last = qvalid - 1;
        const int64_t tsel = last < 32 ? tv[0] : tv[1];
        const int64_t t_last = __shfl_sync(0xffffffffu, tsel, last & 31);
        bool mono = true, rel32 = true;
  #pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int c = lane + 32 * i;
          s.ts[ms][c] = tv[i];
          const int64_t d = tv[i] - t_first;
          rel32 = rel32 && (d > -(1ll << 30)) && (d < (1ll << 30));
          s.ts32[ms][c] = (int32_t)d;
          const int64_t nxt_same = __shfl_down_sync(0xffffffffu, tv[i], 1);
          const int64_t nxt_grp = __shfl_sync(0xffffffffu, tv[1], 0);
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
          tv[0] = tn[0];
          tv[1] = tn[1];
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

// dQ = (scale / 2) * the accumulated K^T G products, rounded to bf16
__global__ void dq_convert_kernel(const float* __restrict__ acc, uint16_t* __restrict__ dq,
                                  int64_t n4, float hs) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(acc)[i];
    uint2 o;
    o.x = pack_bf16x2(v.x * hs, v.y * hs);
    o.y = pack_bf16x2(v.z * hs, v.w * hs);
    reinterpret_cast<uint2*>(dq)[i] = o;
  }
}

template <int D>
cudaError_t launch_bwd_t(const AttnArgs& a, cudaStream_t stream) {
  using CF = Cfg<D>;
  static_assert(offsetof(Smem<D>, v) == offsetof(Smem<D>, k) + CF::KTILE,
                "v must follow k (dQ^T reads 128 rows of K^T)");
  static_assert((kBM / CF::BKD) * CF::KBLOCK <= 2 * CF::KTILE + 2 * CF::STAGES * CF::QTILE,
                "the 128 rows of K^T read by dQ^T stay inside the tiles");
  CUtensorMap mq, mk, mv, mdo, mdq;
  const cuuint64_t dims[2] = {(cuuint64_t)a.H * D, (cuuint64_t)a.T};
  const cuuint64_t strides[1] = {(cuuint64_t)a.H * D * 2};
  const cuuint32_t box_k[2] = {(cuuint32_t)CF::BKD, (cuuint32_t)kBM};
  const cuuint32_t box_q[2] = {(cuuint32_t)CF::BKD, (cuuint32_t)kBN};
  const cuuint32_t es[2] = {1u, 1u};
  const CUtensorMapSwizzle sw =
      CF::SWB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  const void* ptrs[4] = {a.q, a.k, a.v, a.dout};
  CUtensorMap* maps[4] = {&mq, &mk, &mv, &mdo};
  for (int i = 0; i < 4; ++i) {
    const cuuint32_t* box = (i == 1 || i == 2) ? box_k : box_q;
    if (encode_tiled(maps[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptrs[i]),
                     dims, strides, box, es, sw) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    // fp32 dQ workspace, written by TMA reductions of [64 queries][D] tiles
    const cuuint64_t qdims[2] = {(cuuint64_t)a.H * D, (cuuint64_t)a.T};
    const cuuint64_t qstrides[1] = {(cuuint64_t)a.H * D * 4};
    const cuuint32_t qbox[2] = {(cuuint32_t)D, (cuuint32_t)kBN};
    if (encode_tiled(&mdq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, a.dq_accum, qdims, qstrides, qbox,
                     es, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
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
  const int64_t bound = a.max_seq_len > 0 ? a.max_seq_len : a.T;
  p.levels = (int)((bound + kBM - 1) / kBM);
  if (p.levels < 1) p.levels = 1;
  // pairs per group of the grid order: all of them when every pair's Q, dO and
  // dQ accumulator rows (8 d bytes a row) fit in L2 together, else as many as
  // fit in 96 MB
  {
    const int64_t npairs = a.B * a.H;
    const int64_t pair_bytes = (bound > 0 ? bound : 1) * D * 8;
    p.group = npairs;
    if (a.T * a.H * D * 8 > (126ll << 20)) {
      const int64_t gp = (96ll << 20) / pair_bytes;
      p.group = gp < 1 ? 1 : (gp < npairs ? gp : npairs);
    }
  }
  const int64_t blocks = (int64_t)p.levels * a.B * a.H;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const int64_t n = a.T * a.H * D;
  cudaError_t e = cudaMemsetAsync(a.dq_accum, 0, sizeof(float) * n, stream);
  if (e != cudaSuccess) return e;
  static_assert(sizeof(Smem<D>) + 1024 <= 232448, "shared memory budget (227 KB per CTA)");
  size_t smem = sizeof(Smem<D>) + 1024;
  if (smem < 120 * 1024) smem = 120 * 1024;  // one CTA per SM (all TMEM columns)
  static DeviceFlags attr_done;  // per template instance and device
  int slot = -1;
  if (!device_flag_set(attr_done, &slot)) {
    // the register split assumes exactly kLaunchRegs per thread at launch
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, hstu_bwd_kernel<D>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(hstu_bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    device_flag_mark(attr_done, slot);
  }
  count_launch();
  hstu_bwd_kernel<D><<<(unsigned)blocks, kThreads, smem, stream>>>(mq, mk, mv, mdo, mdq, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t n4 = n / 4;
  int64_t grid = (n4 + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 16;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  count_launch();
  dq_convert_kernel<<<(unsigned)grid, 256, 0, stream>>>(a.dq_accum,
                                                        static_cast<uint16_t*>(a.dq), n4,
                                                        0.5f * a.scale);
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
