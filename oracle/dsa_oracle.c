/*
 * DSA CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, literal double-precision restatement of the three steps of
 * DeepSeek Sparse Attention (DSA): lightning-indexer scores, per-query top-k
 * selection, and MLA attention in its absorbed MQA form over the selected
 * tokens.  It shares no code with the CUDA library; only tests/, the smoke
 * check and the CPU-baseline leg of the benchmark may load it.
 *
 * Sources (page title, section):
 *  - "DeepSeek-V3.2" (transformers model doc), section "DeepSeek Sparse
 *    Attention (DSA)", item 1 "Lightning indexer": a module with few heads
 *    scores every pair of a query and a key at or before its position; item
 *    2 "Fine-grained token selection": every query retains its index_topk
 *    highest-scoring tokens and the main MLA attention sees only those (the
 *    transformers port expresses the restriction as an additive mask).
 *  - "DeepSeek-V3.2 / Exp" (visual-learn explainer), "Different questions
 *    select different tokens": cached entries are MLA's compressed vectors.
 *  - "DeepSeek-V3.2 - Experimental Exp Version" (altools), "Technical
 *    Principles": the indexer has few heads; MLA with MQA so that key
 *    entries are shared by all query heads.
 *  - "DeepSeek-V3.2-Exp" (token-ids page), released config excerpt
 *    (index_n_heads 64, index_head_dim 128, index_topk 2048, kv_lora_rank 512,
 *    qk_rope_head_dim 64) and "Position IDs" (causal mask: -inf strictly above
 *    the diagonal, so a query sees its own position).
 *
 * Readings where the pages are silent (all listed in the design notes):
 *  - indexer score I[t,s] = sum_j w[t,j] * max(0, q_I[t,j,:] . k_I[s,:]),
 *    defined for 0 <= s <= pos(t) (inclusive, matching the causal mask);
 *  - top-k order: higher score first, then lower sequence-local index; rows
 *    with fewer than k candidates keep all of them, padded with -1;
 *  - absorbed MQA attention: logits z_s = scale * q[t,h,:Dqk] . c[s,:Dqk],
 *    values are the first Dv columns of the same latent row c[s,:].
 *
 * Every function works on one query row at a time in double precision, with
 * no blocking, fusion or reordering beyond the definition.  OpenMP splits the
 * independent query rows across host cores.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* element kinds of an input array */
enum { ORACLE_BF16 = 0, ORACLE_E4M3 = 1, ORACLE_F64 = 2 };

/* bf16: the upper 16 bits of an IEEE-754 binary32 value (exact in double). */
double oracle_bf16_to_double(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* OCP FP8 E4M3 ("fn" variant): 1 sign bit, 4 exponent bits with bias 7,
 * 3 mantissa bits; exponent field 0 holds subnormals m * 2^-9; the pattern
 * S.1111.111 is NaN (there are no infinities); everything else is
 * (1 + m/8) * 2^(e-7). */
double oracle_e4m3_to_double(uint8_t byte) {
  int sign = (byte >> 7) & 1;
  int e = (byte >> 3) & 15;
  int m = byte & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9);
  else
    v = ldexp(1.0 + m / 8.0, e - 7);
  return sign ? -v : v;
}

static double load_elem(int kind, const void* base, int64_t i, const float* row_scale, int64_t row) {
  switch (kind) {
    case ORACLE_BF16: return oracle_bf16_to_double(((const uint16_t*)base)[i]);
    case ORACLE_E4M3: return oracle_e4m3_to_double(((const uint8_t*)base)[i]) * (double)row_scale[row];
    default: return ((const double*)base)[i];
  }
}

/* Which sequence holds global query row t, and its absolute position. */
static int locate_row(int B, const int32_t* cu_q, const int32_t* cu_k, int64_t t, int* b_out,
                      int64_t* pos_out, int64_t* kv_len_out) {
  for (int b = 0; b < B; ++b) {
    if (t >= cu_q[b] && t < cu_q[b + 1]) {
      int64_t q_len = cu_q[b + 1] - cu_q[b];
      int64_t kv_len = cu_k[b + 1] - cu_k[b];
      *b_out = b;
      *pos_out = kv_len - q_len + (t - cu_q[b]);
      *kv_len_out = kv_len;
      return 0;
    }
  }
  return -1;
}

static int check_varlen(int B, const int32_t* cu_q, const int32_t* cu_k) {
  if (B < 1 || cu_q[0] != 0 || cu_k[0] != 0) return -1;
  for (int b = 0; b < B; ++b) {
    int64_t q_len = cu_q[b + 1] - cu_q[b];
    int64_t kv_len = cu_k[b + 1] - cu_k[b];
    if (q_len < 0 || kv_len < q_len) return -1;
  }
  return 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/*
 * Step 1, lightning indexer.  For each requested query row t (global index
 * rows[r], or r itself when rows is NULL) and each key s of its sequence:
 *   scores[r, s] = sum_j w[t,j] * max(0, sum_d q_idx[t,j,d] * k_idx[s,d])  for s <= pos(t)
 *   scores[r, s] = -inf                                                     for s >  pos(t)
 * q_idx: [T, H_I, d_I]; w: [T, H_I] (double); k_idx: [sum kv, d_I] with, for
 * E4M3, one float32 scale per key row.
 */
static int indexer_scores(int B, const int32_t* cu_q, const int32_t* cu_k, int H_I, int d_I, int q_kind,
                          const void* q_idx, const float* q_scale, const double* w, int k_kind,
                          const void* k_idx, const float* k_scale, int64_t n_rows, const int32_t* rows,
                          double* scores, int64_t ld) {
  if (check_varlen(B, cu_q, cu_k)) return -1;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t r = 0; r < n_rows; ++r) {
    int64_t t = rows ? rows[r] : r;
    int b;
    int64_t pos, kv_len;
    if (locate_row(B, cu_q, cu_k, t, &b, &pos, &kv_len) || kv_len > ld) {
      bad = 1;
      continue;
    }
    double* out = scores + r * ld;
    for (int64_t s = 0; s < kv_len; ++s) {
      if (s > pos) {
        out[s] = -INFINITY;
        continue;
      }
      int64_t key_row = cu_k[b] + s;
      double total = 0.0;
      for (int j = 0; j < H_I; ++j) {
        double dot = 0.0;
        for (int d = 0; d < d_I; ++d) {
          double qv = load_elem(q_kind, q_idx, (t * H_I + j) * (int64_t)d_I + d, q_scale, t * H_I + j);
          double kv = load_elem(k_kind, k_idx, key_row * d_I + d, k_scale, key_row);
          dot += qv * kv;
        }
        double relu = dot > 0.0 ? dot : 0.0;
        total += w[t * H_I + j] * relu;
      }
      out[s] = total;
    }
  }
  return bad ? -1 : 0;
}

/* bf16 / float64 index queries (q_kind); keys as described above. */
int oracle_indexer_scores(int B, const int32_t* cu_q, const int32_t* cu_k, int H_I, int d_I,
                          int q_kind, const void* q_idx, const double* w, int k_kind,
                          const void* k_idx, const float* k_scale, int64_t n_rows,
                          const int32_t* rows, double* scores, int64_t ld) {
  if (q_kind == ORACLE_E4M3) return -1;   /* e4m3 queries need their scales: oracle_indexer_scores_fp8 */
  return indexer_scores(B, cu_q, cu_k, H_I, d_I, q_kind, q_idx, NULL, w, k_kind, k_idx, k_scale, n_rows, rows,
                        scores, ld);
}

typedef struct {
  double score;
  int32_t index;
} candidate;

/* Total order of the selection: higher score first, then lower index. */
static int candidate_cmp(const void* a, const void* b) {
  const candidate* x = (const candidate*)a;
  const candidate* y = (const candidate*)b;
  if (x->score > y->score) return -1;
  if (x->score < y->score) return 1;
  return (x->index > y->index) - (x->index < y->index);
}

/*
 * Step 2, fine-grained token selection.  Every requested row: sort the
 * candidates s = 0..pos(t) by (score desc, index asc) and keep the first
 * min(topk, pos(t)+1); idx[r, :] holds them in that order, then -1 padding.
 * scores rows follow the layout written by oracle_indexer_scores.
 */
int oracle_topk(int B, const int32_t* cu_q, const int32_t* cu_k, int64_t n_rows, const int32_t* rows,
                const double* scores, int64_t ld, int topk, int32_t* idx) {
  if (check_varlen(B, cu_q, cu_k) || topk < 1) return -1;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t r = 0; r < n_rows; ++r) {
    int64_t t = rows ? rows[r] : r;
    int b;
    int64_t pos, kv_len;
    if (locate_row(B, cu_q, cu_k, t, &b, &pos, &kv_len) || kv_len > ld) {
      bad = 1;
      continue;
    }
    int64_t n = pos + 1;
    candidate* c = (candidate*)malloc(sizeof(candidate) * (size_t)n);
    if (!c) {
      bad = 1;
      continue;
    }
    for (int64_t s = 0; s < n; ++s) {
      c[s].score = scores[r * ld + s];
      c[s].index = (int32_t)s;
    }
    qsort(c, (size_t)n, sizeof(candidate), candidate_cmp);
    int64_t keep = n < topk ? n : topk;
    for (int64_t i = 0; i < topk; ++i) idx[r * topk + i] = i < keep ? c[i].index : -1;
    free(c);
  }
  return bad ? -1 : 0;
}

/* An entry of idx takes part in attention for query position pos iff it is a
 * key of the sequence at or before pos; -1 (padding) and anything else is
 * ignored. */
static int selected_entry_valid(int32_t s, int64_t pos, int64_t kv_len) {
  return s >= 0 && s <= pos && s < kv_len;
}

/*
 * Step 3, MLA attention in absorbed MQA form over the selected tokens.
 * For each requested row t and head h, over the valid entries s of idx[r,:]:
 *   z_s = scale * sum_{d < Dqk} q[t,h,d] * c[s,d]
 *   out[r,h,:] = sum_s softmax(z)_s * c[s, :Dv],   lse[r,h] = log sum_s exp(z_s)
 * The softmax is evaluated as exp(z_s - max z) / sum exp(z - max z).  With no
 * valid entry, out = 0 and lse = -inf.
 * q: [T, H, Dqk]; latent: [sum kv, Dqk]; out: [n_rows, H, Dv]; lse: [n_rows, H].
 */
int oracle_sparse_mla(int B, const int32_t* cu_q, const int32_t* cu_k, int H, int d_qk, int d_v,
                      int q_kind, const void* q, int c_kind, const void* latent, int64_t n_rows,
                      const int32_t* rows, const int32_t* idx, int topk, double scale, double* out,
                      double* lse) {
  if (check_varlen(B, cu_q, cu_k) || d_v > d_qk || topk < 1) return -1;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t r = 0; r < n_rows; ++r) {
    int64_t t = rows ? rows[r] : r;
    int b;
    int64_t pos, kv_len;
    if (locate_row(B, cu_q, cu_k, t, &b, &pos, &kv_len)) {
      bad = 1;
      continue;
    }
    double* z = (double*)malloc(sizeof(double) * (size_t)topk);
    if (!z) {
      bad = 1;
      continue;
    }
    const int32_t* sel = idx + r * topk;
    for (int h = 0; h < H; ++h) {
      double zmax = -INFINITY;
      for (int i = 0; i < topk; ++i) {
        z[i] = -INFINITY;
        if (!selected_entry_valid(sel[i], pos, kv_len)) continue;
        int64_t row = cu_k[b] + sel[i];
        double dot = 0.0;
        for (int d = 0; d < d_qk; ++d)
          dot += load_elem(q_kind, q, (t * H + h) * (int64_t)d_qk + d, NULL, 0) *
                 load_elem(c_kind, latent, row * d_qk + d, NULL, 0);
        z[i] = scale * dot;
        if (z[i] > zmax) zmax = z[i];
      }
      double* o = out + (r * H + h) * (int64_t)d_v;
      for (int d = 0; d < d_v; ++d) o[d] = 0.0;
      if (zmax == -INFINITY) {
        lse[r * H + h] = -INFINITY;
        continue;
      }
      double denom = 0.0;
      for (int i = 0; i < topk; ++i)
        if (z[i] != -INFINITY) denom += exp(z[i] - zmax);
      for (int i = 0; i < topk; ++i) {
        if (z[i] == -INFINITY) continue;
        double p = exp(z[i] - zmax) / denom;
        int64_t row = cu_k[b] + sel[i];
        for (int d = 0; d < d_v; ++d) o[d] += p * load_elem(c_kind, latent, row * d_qk + d, NULL, 0);
      }
      lse[r * H + h] = zmax + log(denom);
    }
    free(z);
  }
  return bad ? -1 : 0;
}

/*
 * The additive-mask formulation named on the transformers page: dense MLA
 * attention over every key of the sequence, with mask 0 on the selected
 * positions and -inf elsewhere (the causal mask is -inf strictly above the
 * diagonal).  Mathematically identical to oracle_sparse_mla; kept as a
 * separate literal restatement so that each pins the other.
 */
int oracle_dense_mla_masked(int B, const int32_t* cu_q, const int32_t* cu_k, int H, int d_qk,
                            int d_v, int q_kind, const void* q, int c_kind, const void* latent,
                            int64_t n_rows, const int32_t* rows, const int32_t* idx, int topk,
                            double scale, double* out, double* lse) {
  if (check_varlen(B, cu_q, cu_k) || d_v > d_qk || topk < 1) return -1;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t r = 0; r < n_rows; ++r) {
    int64_t t = rows ? rows[r] : r;
    int b;
    int64_t pos, kv_len;
    if (locate_row(B, cu_q, cu_k, t, &b, &pos, &kv_len)) {
      bad = 1;
      continue;
    }
    double* mask = (double*)malloc(sizeof(double) * (size_t)kv_len);
    double* z = (double*)malloc(sizeof(double) * (size_t)kv_len);
    if (!mask || !z) {
      free(mask);
      free(z);
      bad = 1;
      continue;
    }
    for (int64_t s = 0; s < kv_len; ++s) mask[s] = -INFINITY;
    for (int i = 0; i < topk; ++i) {
      int32_t s = idx[r * topk + i];
      if (s >= 0 && s < kv_len) mask[s] = 0.0;
    }
    for (int64_t s = pos + 1; s < kv_len; ++s) mask[s] = -INFINITY; /* causal */
    for (int h = 0; h < H; ++h) {
      double zmax = -INFINITY;
      for (int64_t s = 0; s < kv_len; ++s) {
        int64_t row = cu_k[b] + s;
        double dot = 0.0;
        for (int d = 0; d < d_qk; ++d)
          dot += load_elem(q_kind, q, (t * H + h) * (int64_t)d_qk + d, NULL, 0) *
                 load_elem(c_kind, latent, row * d_qk + d, NULL, 0);
        z[s] = scale * dot + mask[s];
        if (z[s] > zmax) zmax = z[s];
      }
      double* o = out + (r * H + h) * (int64_t)d_v;
      for (int d = 0; d < d_v; ++d) o[d] = 0.0;
      if (zmax == -INFINITY) {
        lse[r * H + h] = -INFINITY;
        continue;
      }
      double denom = 0.0;
      for (int64_t s = 0; s < kv_len; ++s) denom += exp(z[s] - zmax);
      for (int64_t s = 0; s < kv_len; ++s) {
        double p = exp(z[s] - zmax) / denom;
        if (p == 0.0) continue;
        int64_t row = cu_k[b] + s;
        for (int d = 0; d < d_v; ++d) o[d] += p * load_elem(c_kind, latent, row * d_qk + d, NULL, 0);
      }
      lse[r * H + h] = zmax + log(denom);
    }
    free(mask);
    free(z);
  }
  return bad ? -1 : 0;
}

/* ===========================================================================
 * The FP8 indexer ("DeepSeek-V3.2", transformers model doc, section "DeepSeek
 * Sparse Attention (DSA)", item 1: DeepSeek's own indexer scores in e4m3
 * after a Hadamard rotation of both operands (rotate_activation);
 * "DeepSeek-V3.2-Exp" token-ids page, released config: scale_fmt "ue8m0").  Readings where the pages are silent:
 *  - the rotation is the Sylvester-Hadamard matrix of order d (d a power of
 *    two), H[i][j] = (-1)^popcount(i & j), orthonormal as H / sqrt(d); the
 *    FP8 path rotates both operands by H itself, so (Hq).(Hk) = d (q.k) and
 *    the score divides the factor d out (exact: d is a power of two);
 *  - quantization is per vector of d values (one index-head query, or one
 *    index key): a power-of-two scale s = 2^ceil(log2(amax / 448)) (an ue8m0
 *    exponent; s = 1 for a zero vector), values e4m3(x / s) rounded to
 *    nearest, ties to even;
 *  - the FP8 score is the indexer score of the dequantized values,
 *    sum_j w[t,j] * max(0, (s_q[t,j] qq[t,j,:]) . (s_k[s] kq[s,:])).
 * =========================================================================*/

/* y[v,:] = H x[v,:] / sqrt(d) (normalize != 0) or H x[v,:] (normalize == 0)
 * for n_vec vectors of length d (d a power of two). */
int oracle_hadamard(int64_t n_vec, int d, const double* x, double* y, int normalize) {
  if (d < 1 || (d & (d - 1))) return -1;
  const double norm = normalize ? 1.0 / sqrt((double)d) : 1.0;
#pragma omp parallel for schedule(static)
  for (int64_t v = 0; v < n_vec; ++v) {
    for (int i = 0; i < d; ++i) {
      double acc = 0.0;
      for (int j = 0; j < d; ++j) {
        const int sign = __builtin_popcount((unsigned)(i & j)) & 1;
        acc += sign ? -x[v * d + j] : x[v * d + j];
      }
      y[v * d + i] = acc * norm;
    }
  }
  return 0;
}

/* The e4m3 byte nearest to v (ties to the even mantissa), saturating at
 * +-448 (the largest finite magnitude); v must not be NaN.  Candidates are
 * the 127 finite non-negative codes, compared by distance in double. */
uint8_t oracle_double_to_e4m3(double v) {
  const int neg = signbit(v) ? 1 : 0;
  const double a = fabs(v);
  int best = 0;
  double best_err = INFINITY;
  for (int code = 0; code < 127; ++code) {   /* 0x00 .. 0x7E: every finite non-negative value */
    const double c = oracle_e4m3_to_double((uint8_t)code);
    const double err = fabs(c - a);
    /* on a tie the even mantissa (code & 1 == 0) wins */
    if (err < best_err || (err == best_err && (code & 1) == 0)) {
      best = code;
      best_err = err;
    }
  }
  return (uint8_t)(best | (neg << 7));
}

/* Per-vector e4m3 quantization with a power-of-two scale (see above). */
int oracle_quant_e4m3_pow2(int64_t n_vec, int d, const double* x, uint8_t* q, float* scale) {
  if (d < 1) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t v = 0; v < n_vec; ++v) {
    double amax = 0.0;
    for (int i = 0; i < d; ++i) amax = fmax(amax, fabs(x[v * d + i]));
    const double s = amax > 0.0 ? ldexp(1.0, (int)ceil(log2(amax / 448.0))) : 1.0;
    scale[v] = (float)s;
    for (int i = 0; i < d; ++i) q[v * d + i] = oracle_double_to_e4m3(x[v * d + i] / s);
  }
  return 0;
}

/* Indexer scores with e4m3 index queries (one float32 scale per query head
 * vector, q_scale[t * H_I + j]) and e4m3 index keys (one float32 scale per
 * key).  Same definition and layout as oracle_indexer_scores. */
int oracle_indexer_scores_fp8(int B, const int32_t* cu_q, const int32_t* cu_k, int H_I, int d_I,
                              const uint8_t* q_idx, const float* q_scale, const double* w,
                              const uint8_t* k_idx, const float* k_scale, int64_t n_rows,
                              const int32_t* rows, double* scores, int64_t ld) {
  return indexer_scores(B, cu_q, cu_k, H_I, d_I, ORACLE_E4M3, q_idx, q_scale, w, ORACLE_E4M3, k_idx, k_scale,
                        n_rows, rows, scores, ld);
}

/* ===========================================================================
 * Rotary position embedding of the RoPE part of queries and keys
 * ("DeepSeek-V3.2-Exp" token-ids page, "Position IDs": a per-position table
 * freqs_cis, sliced by position and handed to every layer; released config:
 * qk_rope_head_dim 64).  Reading: every consecutive pair (x[2i], x[2i+1]) is
 * a complex number multiplied by the table entry of its position and pair,
 * freqs[pos][i] = (cos, sin); the table itself is an input.
 * y[v, 2i]   = x[v, 2i] cos - x[v, 2i+1] sin
 * y[v, 2i+1] = x[v, 2i] sin + x[v, 2i+1] cos,   (cos, sin) = freqs[pos[v]][i]
 * x, y: [n_vec, d]; pos: [n_vec]; freqs: [max_pos, d/2, 2].
 * =========================================================================*/
int oracle_rope(int64_t n_vec, int d, const double* x, const int32_t* pos, const double* freqs,
                int64_t max_pos, double* y) {
  if (d < 2 || (d & 1)) return -1;
  int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
  for (int64_t v = 0; v < n_vec; ++v) {
    if (pos[v] < 0 || pos[v] >= max_pos) {
      bad = 1;
      continue;
    }
    for (int i = 0; i < d / 2; ++i) {
      const double c = freqs[((int64_t)pos[v] * (d / 2) + i) * 2 + 0];
      const double s = freqs[((int64_t)pos[v] * (d / 2) + i) * 2 + 1];
      const double re = x[v * d + 2 * i], im = x[v * d + 2 * i + 1];
      y[v * d + 2 * i] = re * c - im * s;
      y[v * d + 2 * i + 1] = re * s + im * c;
    }
  }
  return bad ? -1 : 0;
}

/* ===========================================================================
 * Up-projection of the absorbed attention output out of latent space
 * ("DeepSeek-V3.2-Exp" token-ids page, released config: kv_lora_rank 512,
 * v_head_dim 128, n_heads 128; "DeepSeek-V3.2" transformers doc: MLA with the
 * cached entries shared by all heads, so each head's output is formed in the
 * shared latent space).  Reading: per head h a matrix W_UV[h] of
 * [d_c = kv_lora_rank, d_v = v_head_dim],
 *   y[r, h, e] = sum_c o[r, h, c] * W_UV[h, c, e].
 * o: [n_rows, H, d_c] (double); w: [H, d_c, d_v] (bf16 or double); y: [n_rows, H, d_v].
 * =========================================================================*/
int oracle_up_proj(int64_t n_rows, int H, int d_c, int d_v, const double* o, int w_kind, const void* w,
                   double* y) {
  if (H < 1 || d_c < 1 || d_v < 1) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < n_rows; ++r) {
    for (int h = 0; h < H; ++h) {
      for (int e = 0; e < d_v; ++e) {
        double acc = 0.0;
        for (int c = 0; c < d_c; ++c)
          acc += o[(r * H + h) * (int64_t)d_c + c] * load_elem(w_kind, w, ((int64_t)h * d_c + c) * d_v + e, NULL, 0);
        y[(r * H + h) * (int64_t)d_v + e] = acc;
      }
    }
  }
  return 0;
}

/* ===========================================================================
 * Cache rows of a paged layout ("DeepSeek-V3.2" transformers doc, DSA:
 * besides the main cache, the indexer stores one key per token in a cache of
 * its own, held in a growing (DynamicIndexedLayer) or a preallocated
 * (StaticIndexedLayer) cache layer).  Reading: a preallocated pool of n_pages pages of page_size rows
 * each, shared by the index-key cache and the latent cache; entry s of
 * sequence b sits in page block_table[b * pages_per_seq + s / page_size], at
 * row s % page_size of that page.  With no block table the caches are packed:
 * entry s of sequence b is row cu_k[b] + s.
 * rows[cu_k[b] + s] receives the cache row of entry s of sequence b, or -1
 * when its page entry is missing (s / page_size >= pages_per_seq) or outside
 * [0, n_pages).
 * =========================================================================*/
int oracle_paged_rows(int B, const int32_t* cu_k, const int32_t* block_table, int page_size, int pages_per_seq,
                      int64_t n_pages, int64_t* rows) {
  if (B < 1 || cu_k[0] != 0) return -1;
  if (block_table && (page_size < 1 || pages_per_seq < 1 || n_pages < 1)) return -1;
  for (int b = 0; b < B; ++b) {
    if (cu_k[b + 1] < cu_k[b]) return -1;
    for (int64_t s = 0; s < cu_k[b + 1] - cu_k[b]; ++s) {
      int64_t r = cu_k[b] + s;
      if (block_table) {
        const int64_t j = s / page_size;
        const int64_t page = j < pages_per_seq ? block_table[(int64_t)b * pages_per_seq + j] : -1;
        r = (page >= 0 && page < n_pages) ? page * page_size + s % page_size : -1;
      }
      rows[cu_k[b] + s] = r;
    }
  }
  return 0;
}

/* e4m3 with one float32 scale per vector, scale = amax / 448 rounded to
 * float32 (448: the largest finite e4m3 magnitude; scale 1 for a zero
 * vector); byte i = the e4m3 value nearest (ties to even) to x_i / scale, the
 * quotient taken in float32 (x_i and scale are float32 values; the double
 * quotient of two float32 values rounded to float32 is the float32 quotient). */
int oracle_quant_e4m3_amax(int64_t n_vec, int d, const double* x, uint8_t* q, float* scale) {
  if (d < 1) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t v = 0; v < n_vec; ++v) {
    double amax = 0.0;
    for (int i = 0; i < d; ++i) amax = fmax(amax, fabs(x[v * d + i]));
    const float s = amax > 0.0 ? (float)(amax / 448.0) : 1.0f;
    scale[v] = s;
    for (int i = 0; i < d; ++i) {
      const float qf = (float)((double)(float)x[v * d + i] / (double)s);
      q[v * d + i] = oracle_double_to_e4m3((double)qf);
    }
  }
  return 0;
}
