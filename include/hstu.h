/*
 * hstu.h -- C ABI of libhstu: jagged HSTU pointwise attention on NVIDIA B200
 * (sm_100a), with the load-balanced mini-chunk pairing used for context
 * parallelism.
 *
 * The operation (the HSTUAttention equation of "Scaling Generative
 * Recommendations with Context Parallelism on Hierarchical Sequential
 * Transducers", §2.1):
 *
 *     O = Mask( SiLU( scale * (Q K^T + Bias) ) ) V,   scale usually 1/sqrt(d_qk)
 *     Bias[i, j] = w_pos[min(i - j, P - 1)] + w_ts[bucket(t_i - t_j)]
 *     bucket(dt) = min(bitlen(max(dt, 0)), NB - 1),   bitlen(0) = 0,
 *                  bitlen(x) = floor(log2 x) + 1,  dt the exact difference
 *     Mask keeps j <= i (causal, diagonal included) and is applied after SiLU.
 *
 * The aggregation is pointwise: there is no softmax and no normalisation over
 * keys ("Actions Speak Louder than Words", §3.1).  The timestamp bias groups
 * timestamp differences into buckets that select entries of a learnable
 * table (CP paper §2.1); the relative-position term is the relative attention
 * bias of the HSTU paper, App. F.3.  The bucket function, the clamp of i - j
 * and the placement of scale are the plainest readings of those passages.
 *
 * Jagged layout (CP paper §2.2, "values + offsets"):
 *   q, k, v, out, dout, dq, dk, dv : [T, H, d] row-major, bf16 (out may be fp32),
 *                                    T = seq_offsets[B]; token t, head h, feature c
 *                                    at element (t * H + h) * d + c
 *   seq_offsets                    : int64 [B + 1], seq_offsets[0] = 0, non-decreasing
 *   timestamps                     : int64 [T], one per token, shared by all heads
 *   w_pos                          : fp32 [P]  (shared by all heads)
 *   w_ts                           : fp32 [NB] (shared by all heads)
 *
 * Conventions for every entry point:
 *   - All pointers are DEVICE pointers unless stated otherwise.  The caller
 *     owns and allocates every buffer, including workspaces; the library keeps
 *     no state between calls and allocates no memory.
 *   - Every call is asynchronous on `stream` (0 = legacy default stream) and
 *     never synchronises with the host; seq_offsets are read only on the device.
 *   - Host-checkable errors (null pointers, unsupported sizes, misalignment)
 *     return a negative hstu_status_t at once and launch nothing.
 *   - Data-dependent errors (offsets that decrease, offsets[B] != T, a length
 *     not divisible by 2C) are recorded on the device with atomicMin into
 *     *dev_status (an int the caller set to 0 beforehand; may be NULL) and
 *     the affected work is skipped.  Read it whenever convenient.
 *   - Limits: T < 2^31, num_heads >= 1, d_qk == d_v in {32, 64, 128},
 *     P >= 1, NB >= 1.  q, k, v, out, dout, dq, dk, dv must be 16-byte aligned.
 *   - A CUDA launch failure returns HSTU_ERR_CUDA.
 */
#ifndef HSTU_H_
#define HSTU_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* hstu_stream_t; /* same type as cudaStream_t */

typedef enum {
  HSTU_OK = 0,
  HSTU_ERR_NULL = -1,          /* a required pointer is NULL */
  HSTU_ERR_SHAPE = -2,         /* negative or inconsistent size argument */
  HSTU_ERR_ALIGN = -3,         /* a pointer is not aligned as required */
  HSTU_ERR_UNSUPPORTED = -4,   /* d not in {32, 64, 128}, d_qk != d_v, ... */
  HSTU_ERR_OFFSETS = -5,       /* (device) offsets decrease or offsets[B] != T */
  HSTU_ERR_NOT_DIVISIBLE = -6, /* (device) a sequence length is not a multiple of 2C */
  HSTU_ERR_TIMEOUT = -7,       /* (device) a bounded wait inside a kernel gave up */
  HSTU_ERR_CUDA = -8,          /* a CUDA call failed */
  HSTU_ERR_WORKSPACE = -9      /* workspace missing or too small */
} hstu_status_t;

/* Human-readable name of a status code (static string, never NULL). */
const char* hstu_status_str(int status);

/* Description of the CUDA error behind the last HSTU_ERR_CUDA that an entry
 * point returned on the calling host thread ("no CUDA error" if none); a
 * static string owned by the CUDA runtime, never NULL. */
const char* hstu_last_cuda_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int hstu_version(void);

/* Diagnostics: number of CUDA kernels this library has launched in this
 * process so far (all devices, all entry points).  Lets a caller count the
 * library's kernels inside a timed region. */
int64_t hstu_kernel_launches(void);

/*
 * Forward: out = HSTUAttention(q, k, v) over every sequence and head.
 *
 * max_seq_len : an upper bound on max_b (offsets[b+1] - offsets[b]) (the jagged
 *               tensor's max_lengths, CP paper §2.2), or 0 if unknown (then T
 *               is used as the bound).  Only sizes the launch; a wrong
 *               (too small) bound skips rows and sets HSTU_ERR_SHAPE in
 *               *dev_status.
 * scale       : multiplies (q.k + bias); pass 1/sqrt(d_qk) for the usual scale.
 * out_fp32    : 0 -> out is bf16 [T, H, d_v]; 1 -> out is fp32 [T, H, d_v].
 */
int hstu_jagged_attn_fwd(const void* q, const void* k, const void* v,
                         const int64_t* seq_offsets, int64_t B, int64_t T,
                         int64_t max_seq_len, const int64_t* timestamps,
                         const float* w_pos, int64_t P, const float* w_ts, int64_t NB,
                         int num_heads, int d_qk, int d_v, float scale, int out_fp32,
                         void* out, int* dev_status, hstu_stream_t stream);

/*
 * Target-aware forward for ranking (M-FALCON, "Actions Speak Louder than
 * Words", App. H): the last num_targets[b] rows of sequence b are candidates.
 * Candidates must not attend to one another, and one pass over the history
 * and a microbatch of candidates must give, for every candidate, what a
 * separate forward pass over the history followed by that candidate alone
 * gives.  So, with L_h = L_b - num_targets[b]:
 *   - a history row i < L_h is the plain causal row of hstu_jagged_attn_fwd;
 *   - a candidate row i >= L_h sits at position L_h: it attends every history
 *     key j < L_h with Bias = w_pos[min(L_h - j, P-1)] + w_ts[bucket(t_i - t_j)]
 *     and itself with Bias = w_pos[0] + w_ts[0]; no other key.
 * num_targets: device int64 [B], 8-byte aligned, each value in [0, L_b]
 * (num_targets[b] = L_b leaves no history: every row attends only itself;
 * all zero is the plain causal forward).  A value outside [0, L_b] sets
 * HSTU_ERR_SHAPE in dev_status and leaves that sequence's rows unwritten.
 * The key tiles between the history and a candidate block's own tile are
 * skipped, so a microbatch of m candidates costs about m * L_h pairs.
 * Returns HSTU_ERR_UNSUPPORTED when P exceeds the relative-position table the
 * kernel keeps in shared memory (4096 entries for d_qk <= 64, 3328 for 128).
 * Other arguments, layouts and errors as in hstu_jagged_attn_fwd.
 */
int hstu_jagged_attn_fwd_targets(const void* q, const void* k, const void* v,
                                 const int64_t* seq_offsets, const int64_t* num_targets,
                                 int64_t B, int64_t T, int64_t max_seq_len,
                                 const int64_t* timestamps, const float* w_pos, int64_t P,
                                 const float* w_ts, int64_t NB, int num_heads, int d_qk,
                                 int d_v, float scale, int out_fp32, void* out,
                                 int* dev_status, hstu_stream_t stream);

/*
 * Candidates-only target-aware forward (M-FALCON microbatch scoring, "Actions
 * Speak Louder than Words", App. H): the same operation and arguments as
 * hstu_jagged_attn_fwd_targets, but only the candidate rows are computed and
 * written; the history rows of out are left as they were.  Only the query
 * tiles that hold candidates run, and each visits the history key tiles and
 * its own tile, so a microbatch of m candidates over a history of L_h costs
 * about m * (L_h + 1) pairs.  The history K / V rows are read from the
 * caller's buffers: a caller scoring several microbatches keeps the history
 * rows of q, k, v, timestamps in place (its key/value cache) and writes each
 * microbatch's candidates into the rows after them.
 * max_targets: an upper bound on every num_targets[b] (sizes the launch; 0 =
 * unknown, then max_seq_len is used).  A num_targets[b] above it leaves
 * candidate rows unwritten: keep it an upper bound.
 */
int hstu_jagged_attn_fwd_candidates(const void* q, const void* k, const void* v,
                                    const int64_t* seq_offsets, const int64_t* num_targets,
                                    int64_t B, int64_t T, int64_t max_seq_len,
                                    int64_t max_targets, const int64_t* timestamps,
                                    const float* w_pos, int64_t P, const float* w_ts, int64_t NB,
                                    int num_heads, int d_qk, int d_v, float scale, int out_fp32,
                                    void* out, int* dev_status, hstu_stream_t stream);

/* Bytes of device workspace hstu_jagged_attn_bwd needs (fp32 dq accumulator),
 * or a negative status for bad sizes. */
int64_t hstu_jagged_attn_bwd_workspace_bytes(int64_t T, int num_heads, int d_qk);

/*
 * Backward of hstu_jagged_attn_fwd for the loss sum(out * dout).
 *
 * The pages do not write the backward out ("Actions Speak Louder than Words",
 * App. F.3 says only that it avoids materialising h x N x N tensors); this is
 * the exact derivative of the forward:
 *   g_ij = (dout_i . v_j) SiLU'(x_ij),  x_ij = scale (q_i.k_j + Bias_ij), j <= i
 *   dv_j = sum_i SiLU(x_ij) dout_i      dq_i = scale sum_j g_ij k_j
 *   dk_j = scale sum_i g_ij q_i
 *   dw_pos[r] = scale sum_{min(i-j,P-1)=r} g_ij   dw_ts[b] = scale sum_{bucket=b} g_ij
 * dq, dk, dv are bf16 [T, H, d] and are overwritten; dw_pos [P] and dw_ts [NB]
 * are fp32 and are OVERWRITTEN (not accumulated).  workspace must hold
 * hstu_jagged_attn_bwd_workspace_bytes(T, num_heads, d_qk) bytes, 256-byte
 * aligned; its contents on entry do not matter.  dq and the bias gradients
 * are accumulated with fp32 atomics, so their last bits may vary run to run.
 */
int hstu_jagged_attn_bwd(const void* q, const void* k, const void* v,
                         const int64_t* seq_offsets, int64_t B, int64_t T,
                         int64_t max_seq_len, const int64_t* timestamps,
                         const float* w_pos, int64_t P, const float* w_ts, int64_t NB,
                         int num_heads, int d_qk, int d_v, float scale, const void* dout,
                         void* dq, void* dk, void* dv, float* dw_pos, float* dw_ts,
                         void* workspace, int64_t workspace_bytes, int* dev_status,
                         hstu_stream_t stream);

/*
 * hstu_jagged_attn_bwd_noalloc -- the same backward as hstu_jagged_attn_bwd
 * for callers that cannot allocate device memory (code running inside another
 * runtime's plugin or enqueue callback where cudaMalloc is not allowed, or a
 * process that fixes its whole device-memory plan up front).  The pages have
 * no counterpart; this is a deployment convenience of this library.
 *
 * Instead of a caller workspace it uses a scratch array compiled into the
 * library (HSTU_BWD_NOALLOC_MAX_ELEMS floats = 16 MiB, held on every GPU that
 * loads the library until the process exits) and allocates nothing.  Other
 * arguments, outputs and errors as in hstu_jagged_attn_bwd, plus:
 *   - returns HSTU_ERR_WORKSPACE, launching nothing, when
 *     T * num_heads * d_qk > HSTU_BWD_NOALLOC_MAX_ELEMS;
 *   - all calls on a device share the scratch array (its contents persist
 *     between calls and are cleared where needed), so calls whose kernels
 *     could overlap on the GPU -- different streams, several host threads --
 *     race and must be ordered by the caller;
 *   - the scratch array used is the CURRENT device's copy: `stream` must
 *     belong to the current device, else HSTU_ERR_UNSUPPORTED (nothing
 *     launched);
 *   - the scratch array's device address is looked up (cudaGetSymbolAddress
 *     with the device current) on every call made outside a stream capture,
 *     so a device reset between calls is harmless; a call made while the
 *     stream is being captured reuses the address from the last uncaptured
 *     call on that device: make one call before any stream capture starts.
 */
#define HSTU_BWD_NOALLOC_MAX_ELEMS (4 * 1024 * 1024)
int hstu_jagged_attn_bwd_noalloc(const void* q, const void* k, const void* v,
                                 const int64_t* seq_offsets, int64_t B, int64_t T,
                                 int64_t max_seq_len, const int64_t* timestamps,
                                 const float* w_pos, int64_t P, const float* w_ts, int64_t NB,
                                 int num_heads, int d_qk, int d_v, float scale,
                                 const void* dout, void* dq, void* dk, void* dv, float* dw_pos,
                                 float* dw_ts, int* dev_status, hstu_stream_t stream);

/*
 * Load-balanced mini-chunk pairing (CP paper §2.3 and its figure "Load
 * Balanced CP with 2*CP_size Mini-chunks"): every sequence b is cut into 2C
 * mini-chunks of m_b = L_b / (2C) rows, and virtual rank r holds mini-chunks
 * r and 2C-1-r.  The paired layout is rank-major: for r = 0..C-1, for
 * b = 0..B-1, the rows of mini-chunk r followed by the rows of mini-chunk
 * 2C-1-r.  Each L_b must be a multiple of 2C (else HSTU_ERR_NOT_DIVISIBLE in
 * *dev_status and nothing is copied for that sequence).
 *
 * src, dst    : T rows of row_bytes bytes each (any row type: a [H, d] bf16
 *               slice of q/k/v/out, one int64 timestamp, ...); must not overlap.
 * dst_offsets : optional (NULL to skip) int64 [C * B + 1]: start row of each
 *               paired segment (r, b) in dst, at index r * B + b, and T last.
 * global_pos  : optional (NULL to skip) int32 [T]: for every dst row, its
 *               position inside its own sequence (0 .. L_b - 1).
 * The copy is byte-exact.
 */
int hstu_cp_reorder(const void* src, void* dst, int64_t row_bytes,
                    const int64_t* seq_offsets, int64_t B, int64_t T, int C,
                    int64_t* dst_offsets, int32_t* global_pos, int* dev_status,
                    hstu_stream_t stream);

/* Inverse of hstu_cp_reorder: src is in the paired layout, dst in the
 * original jagged layout.  Byte-exact. */
int hstu_cp_restore(const void* src, void* dst, int64_t row_bytes,
                    const int64_t* seq_offsets, int64_t B, int64_t T, int C,
                    int* dev_status, hstu_stream_t stream);

/*
 * Attention evaluated on paired buffers: pq, pk, pv [T, H, d] and
 * ptimestamps [T] are hstu_cp_reorder outputs, seq_offsets are the ORIGINAL
 * offsets.  A query at position i of sequence b attends every key of sequence
 * b at position j <= i, wherever that key sits in the paired buffer, and the
 * bias uses those within-sequence positions and the keys' own timestamps
 * (the correctness condition for cross-chunk pairs, CP paper §2.3).  out is
 * written in the paired layout; hstu_cp_restore brings it back, and the
 * result equals hstu_jagged_attn_fwd on the unpaired input up to rounding.
 * Other arguments as in hstu_jagged_attn_fwd.
 */
int hstu_cp_paired_attn_fwd(const void* pq, const void* pk, const void* pv,
                            const int64_t* seq_offsets, int64_t B, int64_t T,
                            int64_t max_seq_len, int C, const int64_t* ptimestamps,
                            const float* w_pos, int64_t P, const float* w_ts, int64_t NB,
                            int num_heads, int d_qk, int d_v, float scale, int out_fp32,
                            void* out, int* dev_status, hstu_stream_t stream);

/*
 * Debug / parity helper: buckets[i] = bucket(t_q[i] - t_k[i]) for i < n, as
 * the attention kernels compute it (int32 output).  Lets the integer bucket
 * function be compared bit for bit with the oracle.
 */
int hstu_bucket_indices(const int64_t* t_q, const int64_t* t_k, int64_t n, int64_t NB,
                        int32_t* buckets, hstu_stream_t stream);

/*
 * The HSTU layer's step after attention ("Actions Speak Louder than Words",
 * §3, Pointwise Transformation: Norm(A(X)V(X)) ⊙ U(X)).  For every token row
 * t of the [T, N] attention output o (N = num_heads * d_v, all heads of the
 * token together):
 *     y[t] = (o[t] - mean_t) * rsqrt(var_t + eps) ⊙ u[t]
 * with mean_t and the biased variance var_t over the row's N values: a layer
 * normalisation without a learned affine, gated by u (the gate the layer's
 * pointwise projection produced).
 *
 * o, u, y : bf16 [T, N] row-major, 16-byte aligned; y must not overlap o or u.
 * N       : a multiple of 8 with 8 <= N <= 2048 (else HSTU_ERR_SHAPE, or
 *           HSTU_ERR_UNSUPPORTED above 2048).
 * eps     : finite and > 0 (else HSTU_ERR_SHAPE).
 * T = 0 launches nothing.  Arithmetic in fp32, y rounded to bf16.
 */
int hstu_norm_gate_fwd(const void* o, const void* u, void* y, int64_t T, int64_t N, float eps,
                       hstu_stream_t stream);

/*
 * Backward of hstu_norm_gate_fwd: given dy (bf16 [T, N]) writes
 *     d_u = x̂ ⊙ dy,   d_o = rstd (g - mean(g) - x̂ mean(g ⊙ x̂)),
 * with x̂ = (o - mean) rstd and g = dy ⊙ u per row (the exact derivative; the
 * row statistics are recomputed from o).  d_o and d_u: bf16 [T, N], 16-byte
 * aligned, overlapping none of o, u, dy or each other.  Other arguments and
 * errors as in hstu_norm_gate_fwd.
 */
int hstu_norm_gate_bwd(const void* o, const void* u, const void* dy, void* d_o, void* d_u,
                       int64_t T, int64_t N, float eps, hstu_stream_t stream);

/*
 * Stochastic Length ("Actions Speak Louder than Words", §3.2 and §4.2):
 * subsequences of long histories, chosen at random, raise the sparsity the
 * attention exploits.  For each sequence b of the jagged batch (seq_offsets
 * [B + 1], T rows) of length n: if n > L and u_seq[b] / 2^32 < 1 - (L / n)^2
 * (evaluated in float64 in that order), the L tokens with the smallest
 * (u_tok[row], position) are kept, in their order; otherwise all n are kept.
 * L is the target length, floor(N^(alpha / 2)) for maximum length N and
 * parameter alpha (the caller computes it).  The random draws are inputs
 * (u_tok: uint32 [T], u_seq: uint32 [B]), so a selection is reproducible.
 *
 * dst_offsets : int64 [B + 1], written: offsets of the selected batch.
 * src_rows    : int32 [T], written: entries 0 .. dst_offsets[B] - 1 give the
 *               input row of each selected row, sequence by sequence.
 * T < 2^31, L >= 1.  Sequences with bad offsets (reported in *dev_status as
 * HSTU_ERR_OFFSETS) select nothing.  Two launches; nothing is read back.
 */
int hstu_sl_select(const int64_t* seq_offsets, int64_t B, int64_t T, const uint32_t* u_tok,
                   const uint32_t* u_seq, int64_t L, int64_t* dst_offsets, int32_t* src_rows,
                   int* dev_status, hstu_stream_t stream);

/*
 * Row gather that applies a selection: dst row r = src row src_rows[r] for
 * r < min(*n_rows, max_rows), where n_rows is a device int64 (for a
 * Stochastic Length selection, dst_offsets + B).  Rows are row_bytes bytes
 * (any row type: a [H, d] bf16 slice, one int64 timestamp, ...); src holds
 * src_count rows, and an index outside [0, src_count) leaves its dst row
 * unwritten.  dst (max_rows rows) must not overlap src.  Byte-exact.
 */
int hstu_gather_rows(const void* src, int64_t src_count, void* dst, int64_t row_bytes,
                     const int32_t* src_rows, const int64_t* n_rows, int64_t max_rows,
                     hstu_stream_t stream);

/*
 * hstu_gather_rows for count (1 .. 8) tensors of the same rows in one launch
 * (e.g. q, k, v and the timestamps of a Stochastic Length selection):
 * dsts[t] row r = srcs[t] row src_rows[r].  srcs, dsts and row_bytes are host
 * arrays of count entries; each tensor uses the widest access its row size and
 * pointers allow.  Otherwise as hstu_gather_rows (no dst may overlap a src).
 */
int hstu_gather_rows_multi(int count, const void* const* srcs, void* const* dsts,
                           const int64_t* row_bytes, int64_t src_count, const int32_t* src_rows,
                           const int64_t* n_rows, int64_t max_rows, hstu_stream_t stream);

/*
 * Self-test of the bounded waits (failure detection without a GPU fault).
 * Every wait inside the attention kernels gives up after a time limit,
 * records HSTU_ERR_TIMEOUT in *dev_status and lets the kernel wind down, so a
 * stuck pipeline ends with an error the host can read instead of a hang.
 * This launches one warp that waits, with limit_ns (1e3 .. 1e9 ns), on an
 * mbarrier nothing arrives on: afterwards *dev_status holds HSTU_ERR_TIMEOUT
 * (set with atomicMin, so the caller zeroes it first) and *result (device
 * int) holds 0 = the wait gave up, 1 = it completed (never expected).
 * Nothing else is in flight in that kernel, so the context stays usable.
 */
int hstu_selftest_wait_timeout(int64_t limit_ns, int* dev_status, int* result,
                               hstu_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HSTU_H_ */
