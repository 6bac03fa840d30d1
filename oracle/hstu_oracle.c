/*
 * hstu_oracle.c -- plain fp64 CPU oracle for jagged HSTU pointwise attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file; only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference arm use it.  It shares no code with the CUDA path.
 *
 * What it computes (sources are the two pages on the method):
 *
 *   HSTUAttention(Q,K,V) = Mask( SiLU( (Q K^T + Bias) / sqrt(d_k) ) ) V
 *     -- "Scaling Generative Recommendations with Context Parallelism on
 *        Hierarchical Sequential Transducers", §2.1 (Sequential Transducer
 *        Attention), the HSTUAttention equation.
 *   Pointwise aggregation, no softmax normalisation over keys
 *     -- "Actions Speak Louder than Words", §3.1 (pointwise aggregated attention).
 *   Bias[i,j] = w_pos[min(i-j, P-1)] + w_ts[bucket(t_i - t_j)]
 *     -- timestamp bias: CP paper §2.1 (timestamp differences -> grouping into
 *        bucket indices -> select from ts_weights); relative attention bias:
 *        HSTU paper App. F.3.  The bucket function is not written out on the
 *        pages; this oracle takes the plain log2 reading
 *            bucket(dt) = min(bitlen(max(dt, 0)), NB - 1),
 *        bitlen(0) = 0, bitlen(x) = floor(log2 x) + 1, with dt the exact
 *        integer difference of two int64 timestamps.
 *   Mask = causal (lower triangular, diagonal included), applied after SiLU
 *     -- CP paper §2.3 ("causal" / "lower-triangular" mask).
 *   Jagged layout: values [T, H, d] + offsets [B+1]
 *     -- CP paper §2.2 (Jagged Tensors).
 *   Load-balanced mini-chunk pairing: each sequence is cut into 2C
 *   mini-chunks and rank r holds chunks (r, 2C-1-r)
 *     -- CP paper §2.3 and its figure "Load Balanced CP with 2*CP_size
 *        Mini-chunks".
 *   The backward pass is not written out on the pages (HSTU paper App. F.3
 *   only says it avoids materialising h x N x N tensors); it is the exact
 *   derivative of the forward above.
 *
 * Every floating point value is double.  Sums over keys run in ascending key
 * position j; dot products run over the feature index c ascending.
 *
 * Parity pins (tests/test_oracle.py): a hand-worked 3-token example, dense
 * numpy evaluation of the special case of one sequence, closed forms, central
 * finite differences of the forward for the backward, the CP invariants
 * (paired == unsharded bit for bit, reorder o restore == identity, equal pair
 * counts per rank), and Python's int.bit_length for the bucket.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* threads                                                              */
/* ------------------------------------------------------------------ */
void oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int oracle_get_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* timestamp bucket                                                     */
/* ------------------------------------------------------------------ */
static int64_t bitlen_u64(uint64_t x) {
  int64_t n = 0;
  while (x != 0) {
    n += 1;
    x >>= 1;
  }
  return n;
}

/* bucket of the exact difference t_q - t_k of two int64 timestamps:
 * min(bitlen(max(t_q - t_k, 0)), NB - 1).  The difference is formed in
 * unsigned arithmetic only when it is positive, where it is exact. */
int64_t oracle_bucket_of(int64_t t_q, int64_t t_k, int64_t NB) {
  uint64_t delta = 0;
  if (t_q > t_k) delta = (uint64_t)t_q - (uint64_t)t_k;
  int64_t b = bitlen_u64(delta);
  return b < NB - 1 ? b : NB - 1;
}

/* oracle_bucket_of for n (t_q, t_k) pairs: out[i] = bucket of t_q[i] - t_k[i] */
void oracle_bucket_of_many(const int64_t* t_q, const int64_t* t_k, int64_t n, int64_t NB,
                           int64_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_bucket_of(t_q[i], t_k[i], NB);
}

/* bucket for a difference that is already an int64 value */
int64_t oracle_bucket(int64_t dt, int64_t NB) {
  uint64_t delta = dt > 0 ? (uint64_t)dt : 0;
  int64_t b = bitlen_u64(delta);
  return b < NB - 1 ? b : NB - 1;
}

/* relative position index: min(i - j, P - 1), for j <= i */
static int64_t rel_index(int64_t i, int64_t j, int64_t P) {
  int64_t r = i - j;
  return r < P - 1 ? r : P - 1;
}

/* ------------------------------------------------------------------ */
/* one (query, key) pair: the pre-activation x_ij                       */
/* ------------------------------------------------------------------ */
static double pair_x(const double* qi, const double* kj, int64_t d, double bias, double scale) {
  double s = 0.0;
  for (int64_t c = 0; c < d; ++c) s += qi[c] * kj[c];
  return scale * (s + bias);
}

static double silu(double x) { return x / (1.0 + exp(-x)); }

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* ------------------------------------------------------------------ */
/* forward                                                              */
/* ------------------------------------------------------------------ */
/* q, k, v, out: [T, H, d] row-major; offsets [B+1]; ts [T]. */
void oracle_fwd(const double* q, const double* k, const double* v, const int64_t* offsets,
                int64_t B, const int64_t* ts, const double* w_pos, int64_t P,
                const double* w_ts, int64_t NB, int64_t H, int64_t d, double scale,
                double* out) {
  int64_t T = offsets[B];
  memset(out, 0, sizeof(double) * (size_t)(T * H * d));
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int64_t b = 0; b < B; ++b) {
    for (int64_t h = 0; h < H; ++h) {
      int64_t o = offsets[b];
      int64_t L = offsets[b + 1] - o;
      for (int64_t i = 0; i < L; ++i) {
        const double* qi = q + ((o + i) * H + h) * d;
        double* oi = out + ((o + i) * H + h) * d;
        for (int64_t j = 0; j <= i; ++j) {
          const double* kj = k + ((o + j) * H + h) * d;
          const double* vj = v + ((o + j) * H + h) * d;
          double bias = w_pos[rel_index(i, j, P)] + w_ts[oracle_bucket_of(ts[o + i], ts[o + j], NB)];
          double p = silu(pair_x(qi, kj, d, bias, scale));
          for (int64_t c = 0; c < d; ++c) oi[c] += p * vj[c];
        }
      }
    }
  }
}

/* sequence that holds token t (offsets is monotone) */
static int64_t seq_of(const int64_t* offsets, int64_t B, int64_t t) {
  int64_t lo = 0, hi = B; /* offsets[lo] <= t < offsets[hi] */
  while (hi - lo > 1) {
    int64_t mid = (lo + hi) / 2;
    if (offsets[mid] <= t) lo = mid; else hi = mid;
  }
  while (lo < B && offsets[lo + 1] <= t) ++lo; /* skip empty sequences */
  return lo;
}

/* forward output of selected (token, head) rows: out_rows [n, d] */
void oracle_fwd_rows(const double* q, const double* k, const double* v, const int64_t* offsets,
                     int64_t B, const int64_t* ts, const double* w_pos, int64_t P,
                     const double* w_ts, int64_t NB, int64_t H, int64_t d, double scale,
                     const int64_t* tok, const int64_t* head, int64_t n, double* out_rows) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < n; ++r) {
    int64_t t = tok[r], h = head[r];
    int64_t b = seq_of(offsets, B, t);
    int64_t o = offsets[b];
    int64_t i = t - o;
    const double* qi = q + (t * H + h) * d;
    double* oi = out_rows + r * d;
    for (int64_t c = 0; c < d; ++c) oi[c] = 0.0;
    for (int64_t j = 0; j <= i; ++j) {
      const double* kj = k + ((o + j) * H + h) * d;
      const double* vj = v + ((o + j) * H + h) * d;
      double bias = w_pos[rel_index(i, j, P)] + w_ts[oracle_bucket_of(ts[t], ts[o + j], NB)];
      double p = silu(pair_x(qi, kj, d, bias, scale));
      for (int64_t c = 0; c < d; ++c) oi[c] += p * vj[c];
    }
  }
}

/* ------------------------------------------------------------------ */
/* backward: exact derivative of the forward                            */
/* ------------------------------------------------------------------ */
/*   x = scale (q_i.k_j + bias_ij),  p = SiLU(x),  O_i = sum_j p_ij v_j
 *   g_ij = (dO_i . v_j) SiLU'(x_ij),  SiLU'(x) = s (1 + x (1 - s)), s = sigmoid(x)
 *   dV_j += p_ij dO_i ; dQ_i += scale g_ij k_j ; dK_j += scale g_ij q_i
 *   dw_pos[min(i-j,P-1)] += scale g_ij ; dw_ts[bucket] += scale g_ij            */
void oracle_bwd(const double* q, const double* k, const double* v, const int64_t* offsets,
                int64_t B, const int64_t* ts, const double* w_pos, int64_t P,
                const double* w_ts, int64_t NB, int64_t H, int64_t d, double scale,
                const double* dout, double* dq, double* dk, double* dv, double* dw_pos,
                double* dw_ts) {
  int64_t T = offsets[B];
  size_t n = (size_t)(T * H * d);
  memset(dq, 0, sizeof(double) * n);
  memset(dk, 0, sizeof(double) * n);
  memset(dv, 0, sizeof(double) * n);
  /* per-(sequence, head) partial bias gradients, summed in a fixed order after */
  double* part_pos = (double*)calloc((size_t)(B * H * P) + 1, sizeof(double));
  double* part_ts = (double*)calloc((size_t)(B * H * NB) + 1, sizeof(double));
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int64_t b = 0; b < B; ++b) {
    for (int64_t h = 0; h < H; ++h) {
      int64_t o = offsets[b];
      int64_t L = offsets[b + 1] - o;
      double* pp = part_pos + (b * H + h) * P;
      double* pt = part_ts + (b * H + h) * NB;
      for (int64_t i = 0; i < L; ++i) {
        const double* qi = q + ((o + i) * H + h) * d;
        const double* doi = dout + ((o + i) * H + h) * d;
        double* dqi = dq + ((o + i) * H + h) * d;
        for (int64_t j = 0; j <= i; ++j) {
          const double* kj = k + ((o + j) * H + h) * d;
          const double* vj = v + ((o + j) * H + h) * d;
          double* dkj = dk + ((o + j) * H + h) * d;
          double* dvj = dv + ((o + j) * H + h) * d;
          int64_t rel = rel_index(i, j, P);
          int64_t bk = oracle_bucket_of(ts[o + i], ts[o + j], NB);
          double x = pair_x(qi, kj, d, w_pos[rel] + w_ts[bk], scale);
          double s = sigmoid(x);
          double p = x * s;
          double dsilu = s * (1.0 + x * (1.0 - s));
          double dp = 0.0;
          for (int64_t c = 0; c < d; ++c) dp += doi[c] * vj[c];
          double g = dp * dsilu;
          for (int64_t c = 0; c < d; ++c) {
            dqi[c] += scale * g * kj[c];
            dkj[c] += scale * g * qi[c];
            dvj[c] += p * doi[c];
          }
          pp[rel] += scale * g;
          pt[bk] += scale * g;
        }
      }
    }
  }
  for (int64_t r = 0; r < P; ++r) {
    double s = 0.0;
    for (int64_t bh = 0; bh < B * H; ++bh) s += part_pos[bh * P + r];
    dw_pos[r] = s;
  }
  for (int64_t r = 0; r < NB; ++r) {
    double s = 0.0;
    for (int64_t bh = 0; bh < B * H; ++bh) s += part_ts[bh * NB + r];
    dw_ts[r] = s;
  }
  free(part_pos);
  free(part_ts);
}

/* gradients of selected (token, head) rows: dq of the token as a query,
 * dk / dv of the token as a key.  Outputs are [n, d]. */
void oracle_bwd_rows(const double* q, const double* k, const double* v, const int64_t* offsets,
                     int64_t B, const int64_t* ts, const double* w_pos, int64_t P,
                     const double* w_ts, int64_t NB, int64_t H, int64_t d, double scale,
                     const double* dout, const int64_t* tok, const int64_t* head, int64_t n,
                     double* dq_rows, double* dk_rows, double* dv_rows) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < n; ++r) {
    int64_t t = tok[r], h = head[r];
    int64_t b = seq_of(offsets, B, t);
    int64_t o = offsets[b];
    int64_t L = offsets[b + 1] - o;
    int64_t me = t - o;
    double* dqr = dq_rows + r * d;
    double* dkr = dk_rows + r * d;
    double* dvr = dv_rows + r * d;
    for (int64_t c = 0; c < d; ++c) dqr[c] = dkr[c] = dvr[c] = 0.0;
    /* as a query: keys j <= me */
    {
      int64_t i = me;
      const double* qi = q + (t * H + h) * d;
      const double* doi = dout + (t * H + h) * d;
      for (int64_t j = 0; j <= i; ++j) {
        const double* kj = k + ((o + j) * H + h) * d;
        const double* vj = v + ((o + j) * H + h) * d;
        double bias = w_pos[rel_index(i, j, P)] + w_ts[oracle_bucket_of(ts[o + i], ts[o + j], NB)];
        double x = pair_x(qi, kj, d, bias, scale);
        double s = sigmoid(x);
        double dsilu = s * (1.0 + x * (1.0 - s));
        double dp = 0.0;
        for (int64_t c = 0; c < d; ++c) dp += doi[c] * vj[c];
        double g = dp * dsilu;
        for (int64_t c = 0; c < d; ++c) dqr[c] += scale * g * kj[c];
      }
    }
    /* as a key: queries i >= me */
    {
      int64_t j = me;
      const double* kj = k + (t * H + h) * d;
      const double* vj = v + (t * H + h) * d;
      for (int64_t i = j; i < L; ++i) {
        const double* qi = q + ((o + i) * H + h) * d;
        const double* doi = dout + ((o + i) * H + h) * d;
        double bias = w_pos[rel_index(i, j, P)] + w_ts[oracle_bucket_of(ts[o + i], ts[o + j], NB)];
        double x = pair_x(qi, kj, d, bias, scale);
        double s = sigmoid(x);
        double p = x * s;
        double dsilu = s * (1.0 + x * (1.0 - s));
        double dp = 0.0;
        for (int64_t c = 0; c < d; ++c) dp += doi[c] * vj[c];
        double g = dp * dsilu;
        for (int64_t c = 0; c < d; ++c) {
          dkr[c] += scale * g * qi[c];
          dvr[c] += p * doi[c];
        }
      }
    }
  }
}

/* ------------------------------------------------------------------ */
/* load-balanced mini-chunk pairing (CP paper §2.3, figure "lb")        */
/* ------------------------------------------------------------------ */
/* Layout of the paired buffer: for rank r = 0..C-1, for sequence b = 0..B-1,
 * the rows of mini-chunk r followed by the rows of mini-chunk 2C-1-r.
 * Mini-chunk c of sequence b holds its local rows [c m_b, (c+1) m_b),
 * m_b = L_b / (2C).  Returns 0, or -6 when some L_b is not divisible by 2C,
 * or -2 for C < 1 / bad offsets.  dst_offsets [C B + 1] and global_pos [T]
 * (local index of each paired row within its sequence) may be NULL. */
static int check_cp(const int64_t* offsets, int64_t B, int64_t C) {
  if (C < 1 || B < 0) return -2;
  if (offsets[0] != 0) return -5;
  for (int64_t b = 0; b < B; ++b) {
    int64_t L = offsets[b + 1] - offsets[b];
    if (L < 0) return -5;
    if (L % (2 * C) != 0) return -6;
  }
  return 0;
}

int oracle_cp_reorder(const uint8_t* src, uint8_t* dst, int64_t row_bytes, const int64_t* offsets,
                      int64_t B, int64_t C, int64_t* dst_offsets, int32_t* global_pos) {
  int st = check_cp(offsets, B, C);
  if (st != 0) return st;
  int64_t out = 0;
  for (int64_t r = 0; r < C; ++r) {
    for (int64_t b = 0; b < B; ++b) {
      int64_t L = offsets[b + 1] - offsets[b];
      int64_t m = L / (2 * C);
      if (dst_offsets) dst_offsets[r * B + b] = out;
      for (int half = 0; half < 2; ++half) {
        int64_t c = half == 0 ? r : 2 * C - 1 - r;
        for (int64_t u = 0; u < m; ++u) {
          int64_t local = c * m + u;
          memcpy(dst + out * row_bytes, src + (offsets[b] + local) * row_bytes, (size_t)row_bytes);
          if (global_pos) global_pos[out] = (int32_t)local;
          ++out;
        }
      }
    }
  }
  if (dst_offsets) dst_offsets[C * B] = out;
  return 0;
}

int oracle_cp_restore(const uint8_t* src, uint8_t* dst, int64_t row_bytes, const int64_t* offsets,
                      int64_t B, int64_t C) {
  int st = check_cp(offsets, B, C);
  if (st != 0) return st;
  int64_t in = 0;
  for (int64_t r = 0; r < C; ++r) {
    for (int64_t b = 0; b < B; ++b) {
      int64_t L = offsets[b + 1] - offsets[b];
      int64_t m = L / (2 * C);
      for (int half = 0; half < 2; ++half) {
        int64_t c = half == 0 ? r : 2 * C - 1 - r;
        for (int64_t u = 0; u < m; ++u) {
          int64_t local = c * m + u;
          memcpy(dst + (offsets[b] + local) * row_bytes, src + in * row_bytes, (size_t)row_bytes);
          ++in;
        }
      }
    }
  }
  return 0;
}

/* causal pairs each rank evaluates: for every paired query row at local
 * position i, the keys 0..i of its own sequence (i + 1 pairs).  counts [C]. */
int oracle_cp_rank_pairs(const int64_t* offsets, int64_t B, int64_t C, int64_t* counts) {
  int st = check_cp(offsets, B, C);
  if (st != 0) return st;
  for (int64_t r = 0; r < C; ++r) {
    int64_t n = 0;
    for (int64_t b = 0; b < B; ++b) {
      int64_t L = offsets[b + 1] - offsets[b];
      int64_t m = L / (2 * C);
      for (int half = 0; half < 2; ++half) {
        int64_t c = half == 0 ? r : 2 * C - 1 - r;
        for (int64_t u = 0; u < m; ++u) n += c * m + u + 1;
      }
    }
    counts[r] = n;
  }
  return 0;
}

/* Attention evaluated on the paired buffers.  pq, pk, pv [T, H, d] and
 * pts [T] are in the paired layout; offsets are the ORIGINAL sequence
 * offsets.  A query at local position i of sequence b attends every key of
 * the same sequence at local position j <= i, wherever that key sits in the
 * paired buffer; the bias uses the global (within-sequence) positions and the
 * timestamps the key and query carry.  Keys are visited in ascending j, so
 * the result equals oracle_fwd on the unpaired input bit for bit.  out is in
 * the paired layout. */
int oracle_paired_fwd(const double* pq, const double* pk, const double* pv, const int64_t* pts,
                      const int64_t* offsets, int64_t B, int64_t C, const double* w_pos,
                      int64_t P, const double* w_ts, int64_t NB, int64_t H, int64_t d,
                      double scale, double* out) {
  int st = check_cp(offsets, B, C);
  if (st != 0) return st;
  int64_t T = offsets[B];
  memset(out, 0, sizeof(double) * (size_t)(T * H * d));
  /* row_of[t]: paired row of original token t, by walking the paired layout */
  int64_t* row_of = (int64_t*)malloc(sizeof(int64_t) * (size_t)(T + 1));
  {
    int64_t pos = 0;
    for (int64_t r = 0; r < C; ++r)
      for (int64_t b = 0; b < B; ++b) {
        int64_t L = offsets[b + 1] - offsets[b];
        int64_t m = L / (2 * C);
        for (int half = 0; half < 2; ++half) {
          int64_t c = half == 0 ? r : 2 * C - 1 - r;
          for (int64_t u = 0; u < m; ++u) row_of[offsets[b] + c * m + u] = pos++;
        }
      }
  }
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int64_t b = 0; b < B; ++b) {
    for (int64_t h = 0; h < H; ++h) {
      int64_t o = offsets[b];
      int64_t L = offsets[b + 1] - o;
      for (int64_t i = 0; i < L; ++i) {
        int64_t qr = row_of[o + i];
        const double* qi = pq + (qr * H + h) * d;
        double* oi = out + (qr * H + h) * d;
        for (int64_t j = 0; j <= i; ++j) {
          int64_t kr = row_of[o + j];
          const double* kj = pk + (kr * H + h) * d;
          const double* vj = pv + (kr * H + h) * d;
          double bias = w_pos[rel_index(i, j, P)] + w_ts[oracle_bucket_of(pts[qr], pts[kr], NB)];
          double p = silu(pair_x(qi, kj, d, bias, scale));
          for (int64_t c = 0; c < d; ++c) oi[c] += p * vj[c];
        }
      }
    }
  }
  free(row_of);
  return 0;
}
