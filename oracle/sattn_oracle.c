/*
 * sattn_oracle.c -- fp64 CPU oracle for structured-mask causal attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark do.  It shares no code, header, table or constant with
 * the CUDA path.
 *
 * It computes the plain definitions, slowly and literally:
 *   - decode every input exactly to double (own bf16 decoder);
 *   - materialise each query row's explicit 0/1 key mask;
 *   - compute each kept logit with the capped-distance rotary rule;
 *   - softmax in double, output O and the natural-log logsumexp.
 *
 * Sources (page title and section of the pages this follows):
 *   [LMI] "LM-Infinite" (NAACL 2024 summary), section "方法":
 *         Lambda-shaped mask A_i = {j<=i : j<n_start} U {j<=i : i-j<=L};
 *         distance cap d'_ij = min(d_ij, L); RoPE realisation: window keys
 *         use ordinary rotation, starting-span keys outside the window stay
 *         unrotated and the query is rotated to distance L; optional per-head
 *         top-k middle tokens chosen by largest attention logit.
 *   [SEP] "SepLLM" (CSDN article), sections 五.2 and 6.1: mask
 *         M_ij = 1 iff j in {initial a, separator before i, neighbouring n};
 *         masked positions are set to -inf before the softmax.
 *   [SHL] "SharedLLM" (papernotes summary), sections 关键设计 2 (context
 *         tree: halving splits, level rates alpha_w = 2 alpha_{w+1},
 *         equally spaced downsampling) and 4 (tree cross-attention with
 *         chunk-level rotary positions: queries n, chunk c's keys c).
 *   [SEG] "Training-Inference Consistent Segmented Execution for
 *         Long-Context LLMs", section "整体框架" and "关键设计": local heads
 *         attend a carried tail of the last M keys plus the segment
 *         causally; long heads additionally attend a prefix of R keys
 *         retrieved by top-k with the segment-end query from a read-only
 *         pool; prefix positions 0..P-1, current segment shifted right by P.
 *
 * Readings where the pages leave a step open (each is also listed in the
 * design notes of the repository):
 *   R1  the elementwise product with M in [SEP] 6.1 is read as an additive
 *       0/-inf mask, as [SEP] 五.2 states;
 *   R2  window membership is i-j <= w (w+1 keys including the query), as
 *       [LMI] writes it; SepLLM's n neighbours use the same rule;
 *   R3  "separator before i" is j < i; the mask is a union, so a key that is
 *       sink, window and separator at once counts once;
 *   R5  capped keys: when L > 0 and i-j > L the logit is <R(L)q_i, k_j>;
 *       otherwise <R(i)q_i, R(j)k_j>;
 *   R6  top-k: per query head, among j <= i that the structural mask left
 *       out, the k largest unscaled logits; ties go to the smaller j;
 *       fewer than k candidates -> all of them, padded with -1 / -inf;
 *   R7  rotary convention: rotate-half, inv_freq_c = theta^(-2c/d), angle
 *       pos*s*inv_freq_c; theta == 0 means no rotation; positions 0..T-1;
 *       s is the position-interpolation scale (the talk page, section on
 *       position interpolation: every position is squeezed by one constant
 *       factor so that extended positions stay in the pretraining range);
 *       s = 1 unless given; distances, the cap L included, scale alike;
 *   R8  GQA: query head h uses key/value head floor(h*Hkv/Hq);
 *   R9  segmented: local heads see tail+segment, long heads prefix+segment;
 *   R10 retrieval: block score = max over a block of the unrotated
 *       <q_{sS-1}, k_j>, top R/blk blocks (ties to the lower block), prefix
 *       in ascending block order; segment 0 has no tail and no prefix.
 *   R11 ALiBi ([LMI] 方法: for a model with ALiBi the distance bias is
 *       clipped at the same cap): the scaled logit gets -m_h * d'_ij with
 *       d'_ij = min(i-j, L) (i-j when L = 0); the pages name no slopes, so
 *       head h of H takes ALiBi's own geometric set m_h = 2^(-8(h+1)/H);
 *       distances are token distances (the rotary scale s does not apply);
 *       top-k ranks by z - sqrt(d) m_h d'_ij, the unscaled form of the
 *       biased logit, and reports z.
 *   R13 tree cross-attention ([SHL] "SharedLLM", sections 关键设计 2 and 4):
 *       each of the n context chunks (length l) is a binary tree; the
 *       language-modelling policy always expands the right child, so at
 *       levels w = 1..D the left child is kept and, at w = D, the right
 *       child too (depth D = 0 keeps the root); the split of a node of
 *       length m is b = floor(m/2) (the noise is 0 at test time); level w
 *       keeps a node of length m at rate alpha_w = alpha_D * 2^(D - w):
 *       m' = max(1, floor(m / alpha_w)) rows at offsets floor(k m / m'),
 *       k < m'; the kept rows of a chunk keep their text order; chunk c's
 *       keys take rotary position c and every query position n; the
 *       attention is a plain softmax over all kept rows of all chunks;
 *   R12 backward ([SEP] 6.2: training runs the forward and the backward
 *       pass through the masked product): the gradients of sum(dO . O)
 *       in exact arithmetic; the
 *       top-k selection and the mask are constants (no gradient flows
 *       through a choice); a capped pair contributes to k_j directly and to
 *       q_i through R(L)^T, an uncapped one through R(j)^T and R(i)^T.
 *   R14 segmented backward ([SEG] 整体框架 with R12): the same gradients
 *       over each row's segmented key list; the retrieved blocks, like the
 *       top-k sets, are constants, so a retrieved key's gradient goes back
 *       to its source position through its re-based rotary position, and a
 *       key used by several rows (or segments) sums their contributions.
 *
 * Parity pins: every function here is checked by the CPU tests against
 * closed forms, hand-written golden masks, library routines on degenerate
 * cases and brute force on tiny inputs.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_OK 0
#define OR_ERR_ARG -1
#define OR_ERR_MEM -2

typedef struct oracle_params {
  int32_t B, Hq, Hkv, T, d;
  int32_t dtype; /* 0: inputs are bf16 bit patterns (uint16); 1: float32 */
  int32_t n_start, window, L_pretrain, topk;
  double rope_theta;
  double rope_pos_scale; /* position interpolation scale s (R7); 0 means 1 */
  int32_t alibi;         /* 1: clipped ALiBi bias (R11) instead of a rotation */
} oracle_params;

/* rotary position of token position `pos` (R7) */
static double rot_pos(const oracle_params* p, double pos) {
  return pos * (p->rope_pos_scale > 0.0 ? p->rope_pos_scale : 1.0);
}

/* ALiBi slope of query head h (R11) */
static double alibi_slope(const oracle_params* p, int h) {
  return pow(2.0, -8.0 * (double)(h + 1) / (double)p->Hq);
}

/* clipped ALiBi distance d'_ij (R11) */
static double alibi_dist(int i, int j, int L) {
  int dist = i - j;
  if (L > 0 && dist > L) dist = L;
  return (double)dist;
}

/* ------------------------------------------------------------------ */
/* exact input decoding                                                */
/* ------------------------------------------------------------------ */

/* bf16 is the upper half of an IEEE-754 binary32: sign(1) exp(8) frac(7).
 * Decoded here from the fields, not by a type pun, so the test can pin it
 * against hand-computed values. */
double oracle_decode_bf16(uint16_t bits) {
  int sign = (bits >> 15) & 1;
  int expo = (bits >> 7) & 0xff;
  int frac = bits & 0x7f;
  double v;
  if (expo == 0xff) {
    v = frac ? NAN : INFINITY;
  } else if (expo == 0) {
    v = ldexp((double)frac, -126 - 7); /* subnormal: 0.frac * 2^-126 */
  } else {
    v = ldexp(1.0 + (double)frac / 128.0, expo - 127);
  }
  return sign ? -v : v;
}

static double load_elem(const void* base, int dtype, int64_t idx) {
  if (dtype == 0) return oracle_decode_bf16(((const uint16_t*)base)[idx]);
  return (double)((const float*)base)[idx];
}

/* ------------------------------------------------------------------ */
/* rotary position rotation (reading R7)                               */
/* ------------------------------------------------------------------ */

/* out = R(pos) x.  Rotate-half: pair (c, c+d/2) is rotated by the angle
 * pos * theta^(-2c/d).  theta == 0: identity. */
void oracle_rope(const double* x, int d, double pos, double theta, double* out) {
  int h = d / 2;
  if (theta == 0.0) {
    for (int c = 0; c < d; ++c) out[c] = x[c];
    return;
  }
  for (int c = 0; c < h; ++c) {
    double inv_freq = pow(theta, -2.0 * (double)c / (double)d);
    double a = pos * inv_freq;
    double cs = cos(a), sn = sin(a);
    out[c] = x[c] * cs - x[c + h] * sn;
    out[c + h] = x[c + h] * cs + x[c] * sn;
  }
}

static double dot(const double* a, const double* b, int d) {
  double s = 0.0;
  for (int c = 0; c < d; ++c) s += a[c] * b[c];
  return s;
}

/* ------------------------------------------------------------------ */
/* the structural mask row ([LMI] A_i, [SEP] M_ij; readings R2, R3)    */
/* ------------------------------------------------------------------ */

/* m[j] = 1 iff key j is in query i's structural key set:
 *   j <= i  and  ( j < n_start  or  i-j <= w  or  (is_sep[j] and j < i) ).
 * Returns the number of kept keys. */
int64_t oracle_mask_row(int T, int i, int n_start, int w, const uint8_t* is_sep, uint8_t* m) {
  int64_t cnt = 0;
  for (int j = 0; j < T; ++j) {
    int keep = 0;
    if (j <= i) {
      if (j < n_start) keep = 1;                   /* starting span */
      if (i - j <= w) keep = 1;                    /* recent window */
      if (is_sep && is_sep[j] && j < i) keep = 1;  /* separator before i */
    }
    m[j] = (uint8_t)keep;
    cnt += keep;
  }
  return cnt;
}

/* ------------------------------------------------------------------ */
/* the capped logit ([LMI] d'_ij = min(d_ij, L) and its RoPE form, R5)  */
/* ------------------------------------------------------------------ */

/* Unscaled logit z_ij given the pre-rotated query q_i = R(i)q, the query
 * rotated to the cap q_L = R(L)q, the rotated key R(j)k_j and the raw k_j. */
static double capped_logit(int i, int j, int L, int d, const double* q_i, const double* q_L,
                           const double* k_rot, const double* k_raw) {
  if (L > 0 && i - j > L) return dot(q_L, k_raw, d);
  return dot(q_i, k_rot, d);
}

/* Stand-alone form used by the tests: decode-free doubles in, logit out. */
double oracle_logit(const double* q, const double* k, int d, int i, int j, int L, double theta) {
  double* tmp = (double*)malloc(sizeof(double) * 3 * (size_t)d);
  double* qi = tmp;
  double* ql = tmp + d;
  double* kr = tmp + 2 * d;
  oracle_rope(q, d, (double)i, theta, qi);
  oracle_rope(q, d, (double)L, theta, ql);
  oracle_rope(k, d, (double)j, theta, kr);
  double z = capped_logit(i, j, L, d, qi, ql, kr, k);
  free(tmp);
  return z;
}

/* ------------------------------------------------------------------ */
/* top-k middle tokens ([LMI] optional top-k; reading R6)              */
/* ------------------------------------------------------------------ */

typedef struct {
  double z;    /* unscaled logit */
  double rank; /* ranking key: z, less the unscaled ALiBi bias (R11) */
  int32_t j;
} cand_t;

static int cand_cmp(const void* a, const void* b) {
  const cand_t* x = (const cand_t*)a;
  const cand_t* y = (const cand_t*)b;
  if (x->rank > y->rank) return -1;
  if (x->rank < y->rank) return 1;
  return (x->j < y->j) ? -1 : (x->j > y->j);
}

/* ------------------------------------------------------------------ */
/* one attention row                                                   */
/* ------------------------------------------------------------------ */

typedef struct {
  const oracle_params* p;
  const double* Kraw; /* [T, d] of this kv head */
  const double* Krot; /* [T, d], R(j) k_j */
  const double* Vd;   /* [T, d] */
  const uint8_t* sep; /* [T] or NULL */
} head_ctx;

/* The key set of row i: the structural mask, then the top-k middle keys
 * (taken from `forced` -- k entries, -1 = none -- or selected here).
 * q_i = R(i)q and q_L = R(L)q must be set.  Returns the number of keys. */
static int64_t row_key_set(const head_ctx* hc, const double* q_i, const double* q_L, int h, int i,
                           const int32_t* forced, int32_t* tk_idx, double* tk_z, uint8_t* m, cand_t* cands) {
  const oracle_params* p = hc->p;
  int T = p->T, d = p->d, L = p->L_pretrain;
  double slope = p->alibi ? alibi_slope(p, h) : 0.0;

  int64_t cnt = oracle_mask_row(T, i, p->n_start, p->window, hc->sep, m);

  if (p->topk > 0) {
    if (forced) {
      for (int r = 0; r < p->topk; ++r) {
        int j = forced[r];
        if (j >= 0 && j <= i && !m[j]) {
          m[j] = 1;
          ++cnt;
        }
      }
    } else {
      int n = 0;
      for (int j = 0; j <= i; ++j) {
        if (m[j]) continue;
        cands[n].z = capped_logit(i, j, L, d, q_i, q_L, hc->Krot + (size_t)j * d, hc->Kraw + (size_t)j * d);
        cands[n].rank = cands[n].z;
        if (p->alibi) cands[n].rank -= sqrt((double)d) * slope * alibi_dist(i, j, L);
        cands[n].j = j;
        ++n;
      }
      qsort(cands, (size_t)n, sizeof(cand_t), cand_cmp);
      for (int r = 0; r < p->topk; ++r) {
        if (r < n) {
          m[cands[r].j] = 1;
          ++cnt;
          if (tk_idx) tk_idx[r] = cands[r].j;
          if (tk_z) tk_z[r] = cands[r].z;
        } else {
          if (tk_idx) tk_idx[r] = -1;
          if (tk_z) tk_z[r] = -INFINITY;
        }
      }
    }
  }
  return cnt;
}

/* Scaled logit s_ij of a kept key: the capped rotary logit over sqrt(d),
 * less the clipped ALiBi bias (R5, R11). */
static double row_logit(const head_ctx* hc, const double* q_i, const double* q_L, double slope, int i, int j) {
  const oracle_params* p = hc->p;
  int d = p->d, L = p->L_pretrain;
  double s = capped_logit(i, j, L, d, q_i, q_L, hc->Krot + (size_t)j * d, hc->Kraw + (size_t)j * d) *
             (1.0 / sqrt((double)d));
  if (p->alibi) s -= slope * alibi_dist(i, j, L);
  return s;
}

/* Computes O_i and LSE_i for one row.  If forced != NULL the top-k set is
 * taken from it (k entries, -1 = none) instead of being selected. */
static int attn_row(const head_ctx* hc, const double* qraw, int h, int i, const int32_t* forced,
                    double* o_out, double* lse_out, int32_t* tk_idx, double* tk_z, int64_t* count,
                    uint8_t* m, double* zbuf, cand_t* cands, double* work) {
  const oracle_params* p = hc->p;
  int T = p->T, d = p->d, L = p->L_pretrain;
  double* q_i = work;
  double* q_L = work + d;
  oracle_rope(qraw, d, rot_pos(p, (double)i), p->rope_theta, q_i);
  oracle_rope(qraw, d, rot_pos(p, (double)(L > 0 ? L : 0)), p->rope_theta, q_L);
  double slope = p->alibi ? alibi_slope(p, h) : 0.0;
  int64_t cnt = row_key_set(hc, q_i, q_L, h, i, forced, tk_idx, tk_z, m, cands);
  if (count) *count = cnt;

  /* logits of kept keys, scaled by 1/sqrt(d); masked keys are -inf and
   * contribute exactly zero, so they are skipped */
  double mx = -INFINITY;
  for (int j = 0; j < T; ++j) {
    if (!m[j]) continue;
    double s = row_logit(hc, q_i, q_L, slope, i, j);
    zbuf[j] = s;
    if (s > mx) mx = s;
  }
  for (int c = 0; c < d; ++c) o_out[c] = 0.0;
  if (cnt == 0) {
    *lse_out = -INFINITY;
    return OR_OK;
  }
  double sum = 0.0;
  for (int j = 0; j < T; ++j)
    if (m[j]) sum += exp(zbuf[j] - mx);
  double lse = mx + log(sum);
  for (int j = 0; j < T; ++j) {
    if (!m[j]) continue;
    double pj = exp(zbuf[j] - lse);
    const double* vj = hc->Vd + (size_t)j * d;
    for (int c = 0; c < d; ++c) o_out[c] += pj * vj[c];
  }
  *lse_out = lse;
  return OR_OK;
}

/* ------------------------------------------------------------------ */
/* threading helper                                                    */
/* ------------------------------------------------------------------ */

typedef struct {
  void (*fn)(void*, int64_t);
  void* arg;
  int64_t n;
  int64_t next;
  pthread_mutex_t mu;
} pool_t;

static void* pool_worker(void* a) {
  pool_t* P = (pool_t*)a;
  for (;;) {
    pthread_mutex_lock(&P->mu);
    int64_t t = P->next++;
    pthread_mutex_unlock(&P->mu);
    if (t >= P->n) break;
    P->fn(P->arg, t);
  }
  return NULL;
}

static void run_parallel(void (*fn)(void*, int64_t), void* arg, int64_t n, int nthreads) {
  pool_t P;
  P.fn = fn;
  P.arg = arg;
  P.n = n;
  P.next = 0;
  pthread_mutex_init(&P.mu, NULL);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  pthread_t th[256];
  for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, pool_worker, &P);
  for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
  pthread_mutex_destroy(&P.mu);
}

/* decode the K / V of one kv head into doubles and rotate K */
static int load_head(const oracle_params* p, const void* K, const void* V, int b, int g,
                     double* Kraw, double* Krot, double* Vd) {
  int T = p->T, d = p->d;
  int64_t base = ((int64_t)b * p->Hkv + g) * (int64_t)T * d;
  for (int j = 0; j < T; ++j) {
    for (int c = 0; c < d; ++c) {
      Kraw[(size_t)j * d + c] = load_elem(K, p->dtype, base + (int64_t)j * d + c);
      Vd[(size_t)j * d + c] = load_elem(V, p->dtype, base + (int64_t)j * d + c);
    }
    oracle_rope(Kraw + (size_t)j * d, d, rot_pos(p, (double)j), p->rope_theta, Krot + (size_t)j * d);
  }
  return OR_OK;
}

/* ------------------------------------------------------------------ */
/* forward over a list of rows                                         */
/* ------------------------------------------------------------------ */

typedef struct {
  head_ctx hc;
  const void* Q;
  const int64_t* rows; /* (b, h, i) triples */
  const int64_t* sel;  /* indices into rows handled by this head */
  const int32_t* forced;
  double* O;
  double* lse;
  int32_t* tk_idx;
  double* tk_z;
  int64_t* counts;
} fwd_job;

static void fwd_one(void* a, int64_t t) {
  fwd_job* J = (fwd_job*)a;
  const oracle_params* p = J->hc.p;
  int T = p->T, d = p->d, k = p->topk;
  int64_t r = J->sel[t];
  int b = (int)J->rows[3 * r], h = (int)J->rows[3 * r + 1], i = (int)J->rows[3 * r + 2];
  uint8_t* m = (uint8_t*)malloc((size_t)T);
  double* zbuf = (double*)malloc(sizeof(double) * (size_t)T);
  cand_t* cands = (cand_t*)malloc(sizeof(cand_t) * (size_t)(T + 1));
  double* work = (double*)malloc(sizeof(double) * 3 * (size_t)d);
  double* qraw = work + 2 * d;
  int64_t qb = (((int64_t)b * p->Hq + h) * T + i) * d;
  for (int c = 0; c < d; ++c) qraw[c] = load_elem(J->Q, p->dtype, qb + c);
  attn_row(&J->hc, qraw, h, i, J->forced ? J->forced + r * k : NULL, J->O + r * d, J->lse + r,
           (J->tk_idx && k) ? J->tk_idx + r * k : NULL, (J->tk_z && k) ? J->tk_z + r * k : NULL,
           J->counts ? J->counts + r : NULL, m, zbuf, cands, work);
  free(m);
  free(zbuf);
  free(cands);
  free(work);
}

/* O[n, d], lse[n]; tk_idx/tk_z [n, k] (may be NULL); counts [n] (may be NULL);
 * forced [n, k] (may be NULL).  rows: n triples (b, h, i). */
int oracle_fwd_rows(const oracle_params* p, const void* Q, const void* K, const void* V,
                    const uint8_t* is_sep, int64_t n, const int64_t* rows, const int32_t* forced,
                    double* O, double* lse, int32_t* tk_idx, double* tk_z, int64_t* counts,
                    int nthreads) {
  if (!p || p->d <= 0 || (p->d & 1) || p->T <= 0 || p->Hq <= 0 || p->Hkv <= 0 ||
      p->Hq % p->Hkv)
    return OR_ERR_ARG;
  int T = p->T, d = p->d;
  double* Kraw = (double*)malloc(sizeof(double) * (size_t)T * d);
  double* Krot = (double*)malloc(sizeof(double) * (size_t)T * d);
  double* Vd = (double*)malloc(sizeof(double) * (size_t)T * d);
  int64_t* sel = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n + 1));
  if (!Kraw || !Krot || !Vd || !sel) return OR_ERR_MEM;
  for (int b = 0; b < p->B; ++b) {
    for (int g = 0; g < p->Hkv; ++g) {
      int64_t ns = 0;
      for (int64_t r = 0; r < n; ++r) {
        int rb = (int)rows[3 * r], rh = (int)rows[3 * r + 1];
        int rg = (int)(((int64_t)rh * p->Hkv) / p->Hq); /* reading R8 */
        if (rb == b && rg == g) sel[ns++] = r;
      }
      if (!ns) continue;
      load_head(p, K, V, b, g, Kraw, Krot, Vd);
      fwd_job J;
      J.hc.p = p;
      J.hc.Kraw = Kraw;
      J.hc.Krot = Krot;
      J.hc.Vd = Vd;
      J.hc.sep = is_sep ? is_sep + (size_t)b * T : NULL;
      J.Q = Q;
      J.rows = rows;
      J.sel = sel;
      J.forced = forced;
      J.O = O;
      J.lse = lse;
      J.tk_idx = tk_idx;
      J.tk_z = tk_z;
      J.counts = counts;
      run_parallel(fwd_one, &J, ns, nthreads);
    }
  }
  free(Kraw);
  free(Krot);
  free(Vd);
  free(sel);
  return OR_OK;
}

/* ------------------------------------------------------------------ */
/* backward: gradients of L = sum dO . O (R12)                          */
/* ------------------------------------------------------------------ */

/* One (batch, kv head): every row of every query head of the group.  The
 * key-side sums run over all rows, so a job owns its kv head's dK / dV. */
typedef struct {
  const oracle_params* p;
  const void *Q, *K, *V, *dO;
  const uint8_t* is_sep;
  const int32_t* forced; /* [B, Hq, T, k] or NULL */
  double *dQ, *dK, *dV;
} bwd_job;

/* Row i of query head h (kv head of hc): its dq_i (raw frame) into dq (when
 * dq != NULL) and, when gKrot / gKraw / gV are given, the row's terms of the
 * key-side sums (gKrot: d L / d (R(j) k_j) of uncapped pairs, gKraw:
 * d L / d k_j of capped pairs, gV: d L / d v_j).  With only_j >= 0 the
 * key-side sums are those of key only_j alone, held in d-entry accumulators,
 * and a row that does not keep only_j adds nothing.  work holds 7 d doubles;
 * m, P, dP, cands are per-thread row buffers of T (+1) entries. */
static void bwd_row(head_ctx* hc, const void* Q, const void* dO, const int32_t* forced, int b, int h, int i,
                    double* work, uint8_t* m, double* P, double* dP, cand_t* cands, double* gKrot,
                    double* gKraw, double* gV, double* dq, int only_j) {
  const oracle_params* p = hc->p;
  int T = p->T, d = p->d, L = p->L_pretrain, k = p->topk;
  const double* Kraw = hc->Kraw;
  const double* Krot = hc->Krot;
  const double* Vd = hc->Vd;
  double *qraw = work, *q_i = work + d, *q_L = work + 2 * d, *doi = work + 3 * d;
  double *gqr = work + 4 * d, *gqc = work + 5 * d, *tmp = work + 6 * d;
  double slope = p->alibi ? alibi_slope(p, h) : 0.0;
  double inv_sqrt_d = 1.0 / sqrt((double)d);
  int64_t qb = (((int64_t)b * p->Hq + h) * T + i) * d;
  for (int c = 0; c < d; ++c) {
    qraw[c] = load_elem(Q, p->dtype, qb + c);
    doi[c] = load_elem(dO, p->dtype, qb + c);
  }
  oracle_rope(qraw, d, rot_pos(p, (double)i), p->rope_theta, q_i);
  oracle_rope(qraw, d, rot_pos(p, (double)(L > 0 ? L : 0)), p->rope_theta, q_L);
  const int32_t* fr = forced ? forced + ((((int64_t)b * p->Hq + h) * T) + i) * k : NULL;
  int64_t cnt = row_key_set(hc, q_i, q_L, h, i, fr, NULL, NULL, m, cands);
  if (only_j >= 0 && (only_j > i || !m[only_j])) return;
  for (int c = 0; c < d; ++c) gqr[c] = gqc[c] = 0.0;
  if (cnt > 0) {
    /* forward quantities of the row: P_ij = exp(s_ij - LSE_i) */
    double mx = -INFINITY;
    for (int j = 0; j < T; ++j)
      if (m[j]) {
        P[j] = row_logit(hc, q_i, q_L, slope, i, j);
        if (P[j] > mx) mx = P[j];
      }
    double sum = 0.0;
    for (int j = 0; j < T; ++j)
      if (m[j]) sum += exp(P[j] - mx);
    double lse = mx + log(sum);
    /* dP_ij = dO_i . v_j and D_i = sum_j P_ij dP_ij (= dO_i . O_i) */
    double D = 0.0;
    for (int j = 0; j < T; ++j)
      if (m[j]) {
        P[j] = exp(P[j] - lse);
        dP[j] = dot(doi, Vd + (size_t)j * d, d);
        D += P[j] * dP[j];
      }
    for (int j = 0; j < T; ++j) {
      if (!m[j]) continue;
      /* dL/dz_ij: softmax Jacobian, then the 1/sqrt(d) scale */
      double dz = P[j] * (dP[j] - D) * inv_sqrt_d;
      /* slot of key j in the key-side accumulators (-1: not accumulated) */
      int64_t ks = only_j < 0 ? j : (j == only_j ? 0 : -1);
      if (gV && ks >= 0) {
        double* gv = gV + (size_t)ks * d;
        for (int c = 0; c < d; ++c) gv[c] += P[j] * doi[c];
      }
      if (L > 0 && i - j > L) {
        /* z = <R(L) q_i, k_j> */
        for (int c = 0; c < d; ++c) {
          gqc[c] += dz * Kraw[(size_t)j * d + c];
          if (gKraw && ks >= 0) gKraw[(size_t)ks * d + c] += dz * q_L[c];
        }
      } else {
        /* z = <R(i) q_i, R(j) k_j> */
        for (int c = 0; c < d; ++c) {
          gqr[c] += dz * Krot[(size_t)j * d + c];
          if (gKrot && ks >= 0) gKrot[(size_t)ks * d + c] += dz * q_i[c];
        }
      }
    }
  }
  if (!dq) return;
  /* back through the rotations: R(p)^T = R(-p) */
  oracle_rope(gqr, d, -rot_pos(p, (double)i), p->rope_theta, tmp);
  for (int c = 0; c < d; ++c) dq[c] = tmp[c];
  oracle_rope(gqc, d, -rot_pos(p, (double)(L > 0 ? L : 0)), p->rope_theta, tmp);
  for (int c = 0; c < d; ++c) dq[c] += tmp[c];
}

static void bwd_one(void* arg, int64_t t) {
  bwd_job* J = (bwd_job*)arg;
  const oracle_params* p = J->p;
  int T = p->T, d = p->d;
  int b = (int)(t / p->Hkv), g = (int)(t % p->Hkv);
  double* Kraw = (double*)malloc(sizeof(double) * (size_t)T * d);
  double* Krot = (double*)malloc(sizeof(double) * (size_t)T * d);
  double* Vd = (double*)malloc(sizeof(double) * (size_t)T * d);
  double* gKrot = (double*)calloc((size_t)T * d, sizeof(double)); /* d L / d (R(j) k_j), uncapped pairs */
  double* gKraw = (double*)calloc((size_t)T * d, sizeof(double)); /* d L / d k_j, capped pairs */
  double* gV = (double*)calloc((size_t)T * d, sizeof(double));
  uint8_t* m = (uint8_t*)malloc((size_t)T);
  double* P = (double*)malloc(sizeof(double) * (size_t)T);
  double* dP = (double*)malloc(sizeof(double) * (size_t)T);
  cand_t* cands = (cand_t*)malloc(sizeof(cand_t) * (size_t)(T + 1));
  double* work = (double*)malloc(sizeof(double) * 8 * (size_t)d);
  double* tmp = work + 7 * d;
  head_ctx hc;
  hc.p = p;
  hc.Kraw = Kraw;
  hc.Krot = Krot;
  hc.Vd = Vd;
  hc.sep = J->is_sep ? J->is_sep + (size_t)b * T : NULL;
  load_head(p, J->K, J->V, b, g, Kraw, Krot, Vd);
  int rep = p->Hq / p->Hkv;
  for (int h = g * rep; h < (g + 1) * rep; ++h)
    for (int i = 0; i < T; ++i)
      bwd_row(&hc, J->Q, J->dO, J->forced, b, h, i, work, m, P, dP, cands, gKrot, gKraw, gV,
              J->dQ + (((int64_t)b * p->Hq + h) * T + i) * d, -1);
  int64_t kb = ((int64_t)b * p->Hkv + g) * (int64_t)T * d;
  for (int j = 0; j < T; ++j) {
    oracle_rope(gKrot + (size_t)j * d, d, -rot_pos(p, (double)j), p->rope_theta, tmp);
    for (int c = 0; c < d; ++c) {
      J->dK[kb + (int64_t)j * d + c] = tmp[c] + gKraw[(size_t)j * d + c];
      J->dV[kb + (int64_t)j * d + c] = gV[(size_t)j * d + c];
    }
  }
  free(Kraw);
  free(Krot);
  free(Vd);
  free(gKrot);
  free(gKraw);
  free(gV);
  free(m);
  free(P);
  free(dP);
  free(cands);
  free(work);
}

/* dQ [B, Hq, T, d], dK / dV [B, Hkv, T, d] in double: the gradients of
 * sum(dO * O) with O the forward of the same parameters.  dO has the input
 * encoding (p->dtype).  forced [B, Hq, T, k]: the top-k sets (NULL: selected
 * here); the selection itself is a constant of the backward pass. */
int oracle_bwd(const oracle_params* p, const void* Q, const void* K, const void* V, const uint8_t* is_sep,
               const int32_t* forced, const void* dO, double* dQ, double* dK, double* dV, int nthreads) {
  if (!p || p->d <= 0 || (p->d & 1) || p->T <= 0 || p->Hq <= 0 || p->Hkv <= 0 || p->Hq % p->Hkv) return OR_ERR_ARG;
  bwd_job J;
  J.p = p;
  J.Q = Q;
  J.K = K;
  J.V = V;
  J.dO = dO;
  J.is_sep = is_sep;
  J.forced = forced;
  J.dQ = dQ;
  J.dK = dK;
  J.dV = dV;
  run_parallel(bwd_one, &J, (int64_t)p->B * p->Hkv, nthreads);
  return OR_OK;
}

/* dq of the sampled rows [(b, h, i)] alone (row i's dq depends on row i
 * only): the same row arithmetic as oracle_bwd, for sizes where the full
 * backward is too slow.  dq [n, d] in double. */
typedef struct {
  const oracle_params* p;
  const void *Q, *K, *V, *dO;
  const uint8_t* is_sep;
  const int32_t* forced;
  const int64_t* rows;
  double* dq;
} bwd_rows_job;

static void bwd_rows_one(void* arg, int64_t r) {
  bwd_rows_job* J = (bwd_rows_job*)arg;
  const oracle_params* p = J->p;
  int T = p->T, d = p->d;
  int b = (int)J->rows[3 * r], h = (int)J->rows[3 * r + 1], i = (int)J->rows[3 * r + 2];
  int g = h / (p->Hq / p->Hkv);
  double* Kraw = (double*)malloc(sizeof(double) * (size_t)T * d);
  double* Krot = (double*)malloc(sizeof(double) * (size_t)T * d);
  double* Vd = (double*)malloc(sizeof(double) * (size_t)T * d);
  uint8_t* m = (uint8_t*)malloc((size_t)T);
  double* P = (double*)malloc(sizeof(double) * (size_t)T);
  double* dP = (double*)malloc(sizeof(double) * (size_t)T);
  cand_t* cands = (cand_t*)malloc(sizeof(cand_t) * (size_t)(T + 1));
  double* work = (double*)malloc(sizeof(double) * 8 * (size_t)d);
  head_ctx hc;
  hc.p = p;
  hc.Kraw = Kraw;
  hc.Krot = Krot;
  hc.Vd = Vd;
  hc.sep = J->is_sep ? J->is_sep + (size_t)b * T : NULL;
  load_head(p, J->K, J->V, b, g, Kraw, Krot, Vd);
  bwd_row(&hc, J->Q, J->dO, J->forced, b, h, i, work, m, P, dP, cands, NULL, NULL, NULL, J->dq + r * d, -1);
  free(Kraw);
  free(Krot);
  free(Vd);
  free(m);
  free(P);
  free(dP);
  free(cands);
  free(work);
}

int oracle_bwd_dq_rows(const oracle_params* p, const void* Q, const void* K, const void* V, const uint8_t* is_sep,
                       const int32_t* forced, const void* dO, int64_t n, const int64_t* rows, double* dq,
                       int nthreads) {
  if (!p || p->d <= 0 || (p->d & 1) || p->T <= 0 || p->Hq <= 0 || p->Hkv <= 0 || p->Hq % p->Hkv || n < 0 ||
      (n > 0 && !rows))
    return OR_ERR_ARG;
  for (int64_t r = 0; r < n; ++r)
    if (rows[3 * r] < 0 || rows[3 * r] >= p->B || rows[3 * r + 1] < 0 || rows[3 * r + 1] >= p->Hq ||
        rows[3 * r + 2] < 0 || rows[3 * r + 2] >= p->T)
      return OR_ERR_ARG;
  bwd_rows_job J;
  J.p = p;
  J.Q = Q;
  J.K = K;
  J.V = V;
  J.dO = dO;
  J.is_sep = is_sep;
  J.forced = forced;
  J.rows = rows;
  J.dq = dq;
  run_parallel(bwd_rows_one, &J, n, nthreads);
  return OR_OK;
}

/* dK and dV of sampled keys [(b, g, j)] (kv head g) alone: key j's terms of
 * oracle_bwd's key-side sums, taken over every row of every query head of
 * the group in the same order (head ascending, then row ascending), so each
 * result equals oracle_bwd's dK / dV at that key bit for bit.  For sizes
 * where the full backward is too slow.  dk, dv [n, d] in double. */
typedef struct {
  const oracle_params* p;
  const void *Q, *K, *V, *dO;
  const uint8_t* is_sep;
  const int32_t* forced;
  const int64_t* keys;
  double *dk, *dv;
} bwd_keys_job;

static void bwd_keys_one(void* arg, int64_t r) {
  bwd_keys_job* J = (bwd_keys_job*)arg;
  const oracle_params* p = J->p;
  int T = p->T, d = p->d;
  int b = (int)J->keys[3 * r], g = (int)J->keys[3 * r + 1], j = (int)J->keys[3 * r + 2];
  double* Kraw = (double*)malloc(sizeof(double) * (size_t)T * d);
  double* Krot = (double*)malloc(sizeof(double) * (size_t)T * d);
  double* Vd = (double*)malloc(sizeof(double) * (size_t)T * d);
  uint8_t* m = (uint8_t*)malloc((size_t)T);
  double* P = (double*)malloc(sizeof(double) * (size_t)T);
  double* dP = (double*)malloc(sizeof(double) * (size_t)T);
  cand_t* cands = (cand_t*)malloc(sizeof(cand_t) * (size_t)(T + 1));
  double* work = (double*)malloc(sizeof(double) * 8 * (size_t)d);
  double* acc = (double*)calloc(3 * (size_t)d, sizeof(double));
  double *gkr = acc, *gkc = acc + d, *gv = acc + 2 * d;
  double* tmp = work + 7 * d;
  head_ctx hc;
  hc.p = p;
  hc.Kraw = Kraw;
  hc.Krot = Krot;
  hc.Vd = Vd;
  hc.sep = J->is_sep ? J->is_sep + (size_t)b * T : NULL;
  load_head(p, J->K, J->V, b, g, Kraw, Krot, Vd);
  int rep = p->Hq / p->Hkv;
  for (int h = g * rep; h < (g + 1) * rep; ++h)
    for (int i = j; i < T; ++i) /* a row i < j never keeps key j (causal) */
      bwd_row(&hc, J->Q, J->dO, J->forced, b, h, i, work, m, P, dP, cands, gkr, gkc, gv, NULL, j);
  oracle_rope(gkr, d, -rot_pos(p, (double)j), p->rope_theta, tmp);
  for (int c = 0; c < d; ++c) {
    J->dk[r * d + c] = tmp[c] + gkc[c];
    J->dv[r * d + c] = gv[c];
  }
  free(Kraw);
  free(Krot);
  free(Vd);
  free(m);
  free(P);
  free(dP);
  free(cands);
  free(work);
  free(acc);
}

int oracle_bwd_dkv_keys(const oracle_params* p, const void* Q, const void* K, const void* V, const uint8_t* is_sep,
                        const int32_t* forced, const void* dO, int64_t n, const int64_t* keys, double* dk, double* dv,
                        int nthreads) {
  if (!p || p->d <= 0 || (p->d & 1) || p->T <= 0 || p->Hq <= 0 || p->Hkv <= 0 || p->Hq % p->Hkv || n < 0 ||
      (n > 0 && !keys))
    return OR_ERR_ARG;
  for (int64_t r = 0; r < n; ++r)
    if (keys[3 * r] < 0 || keys[3 * r] >= p->B || keys[3 * r + 1] < 0 || keys[3 * r + 1] >= p->Hkv ||
        keys[3 * r + 2] < 0 || keys[3 * r + 2] >= p->T)
      return OR_ERR_ARG;
  bwd_keys_job J;
  J.p = p;
  J.Q = Q;
  J.K = K;
  J.V = V;
  J.dO = dO;
  J.is_sep = is_sep;
  J.forced = forced;
  J.keys = keys;
  J.dk = dk;
  J.dv = dv;
  run_parallel(bwd_keys_one, &J, n, nthreads);
  return OR_OK;
}

/* ------------------------------------------------------------------ */
/* SharedLLM tree cross-attention (R13)                                */
/* ------------------------------------------------------------------ */

/* Kept offsets of one chunk of length l, in text order; returns how many
 * (out may be NULL to count only). */
int oracle_tree_index(int l, int depth, int alpha_leaf, int32_t* out) {
  if (l < 1 || depth < 0 || alpha_leaf < 1 || depth > 30) return OR_ERR_ARG;
  int n = 0;
  int start = 0, len = l;
  for (int w = (depth == 0 ? 0 : 1); w <= depth; ++w) {
    /* the nodes kept at level w: [start, start + m) pieces */
    int piece_start[2], piece_len[2], pieces = 0;
    if (depth == 0) {
      piece_start[0] = 0;
      piece_len[0] = l;
      pieces = 1;
    } else {
      int b = len / 2;
      piece_start[pieces] = start;
      piece_len[pieces] = b;
      ++pieces;
      if (w == depth) {
        piece_start[pieces] = start + b;
        piece_len[pieces] = len - b;
        ++pieces;
      }
      start += b;
      len -= b;
    }
    double alpha = (double)alpha_leaf * pow(2.0, (double)(depth - w));
    for (int x = 0; x < pieces; ++x) {
      int m = piece_len[x];
      if (m <= 0) continue;
      int kept = (int)floor((double)m / alpha);
      if (kept < 1) kept = 1;
      for (int k = 0; k < kept; ++k) {
        if (out) out[n] = piece_start[x] + (int)(((int64_t)k * m) / kept);
        ++n;
      }
    }
  }
  return n;
}

typedef struct {
  const oracle_params* p;
  const void *Q, *K, *V;
  int n_chunks, chunk_len, n_kept;
  const int32_t* idx;
  double *O, *lse;
} tree_job;

static void tree_one(void* arg, int64_t r) {
  tree_job* J = (tree_job*)arg;
  const oracle_params* p = J->p;
  int d = p->d, T = p->T, b = (int)(r / ((int64_t)p->Hq * T)), h = (int)((r / T) % p->Hq), i = (int)(r % T);
  int g = (int)(((int64_t)h * p->Hkv) / p->Hq);
  int S = J->n_chunks * J->n_kept, Tc = J->n_chunks * J->chunk_len;
  double* q = (double*)malloc(sizeof(double) * 4 * (size_t)d);
  double *qr = q + d, *k = q + 2 * d, *kr = q + 3 * d;
  double* z = (double*)malloc(sizeof(double) * (size_t)S);
  for (int c = 0; c < d; ++c) q[c] = load_elem(J->Q, p->dtype, (((int64_t)b * p->Hq + h) * T + i) * d + c);
  oracle_rope(q, d, rot_pos(p, (double)J->n_chunks), p->rope_theta, qr);
  double mx = -INFINITY;
  for (int s = 0; s < S; ++s) {
    int c = s / J->n_kept, j = c * J->chunk_len + J->idx[s % J->n_kept];
    int64_t kb = (((int64_t)b * p->Hkv + g) * Tc + j) * d;
    for (int x = 0; x < d; ++x) k[x] = load_elem(J->K, p->dtype, kb + x);
    oracle_rope(k, d, rot_pos(p, (double)c), p->rope_theta, kr);
    z[s] = dot(qr, kr, d) * (1.0 / sqrt((double)d));
    if (z[s] > mx) mx = z[s];
  }
  double sum = 0.0;
  for (int s = 0; s < S; ++s) sum += exp(z[s] - mx);
  double l = mx + log(sum);
  double* o = J->O + r * d;
  for (int x = 0; x < d; ++x) o[x] = 0.0;
  for (int s = 0; s < S; ++s) {
    int c = s / J->n_kept, j = c * J->chunk_len + J->idx[s % J->n_kept];
    int64_t vb = (((int64_t)b * p->Hkv + g) * Tc + j) * d;
    double w = exp(z[s] - l);
    for (int x = 0; x < d; ++x) o[x] += w * load_elem(J->V, p->dtype, vb + x);
  }
  J->lse[r] = l;
  free(q);
  free(z);
}

/* O [B, Hq, T, d], lse [B, Hq, T] of the tree cross-attention: queries Q
 * [B, Hq, T, d] (p->T rows), context K, V [B, Hkv, n_chunks * chunk_len, d]. */
int oracle_tree_cross(const oracle_params* p, int n_chunks, int chunk_len, int depth, int alpha_leaf, const void* Q,
                      const void* K, const void* V, double* O, double* lse, int nthreads) {
  if (!p || n_chunks < 1 || p->d <= 0 || (p->d & 1) || p->Hq % p->Hkv) return OR_ERR_ARG;
  int n_kept = oracle_tree_index(chunk_len, depth, alpha_leaf, NULL);
  if (n_kept < 1) return OR_ERR_ARG;
  int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)n_kept);
  oracle_tree_index(chunk_len, depth, alpha_leaf, idx);
  tree_job J;
  J.p = p;
  J.Q = Q;
  J.K = K;
  J.V = V;
  J.n_chunks = n_chunks;
  J.chunk_len = chunk_len;
  J.n_kept = n_kept;
  J.idx = idx;
  J.O = O;
  J.lse = lse;
  run_parallel(tree_one, &J, (int64_t)p->B * p->Hq * p->T, nthreads);
  free(idx);
  return OR_OK;
}

/* ------------------------------------------------------------------ */
/* block map by brute force over the materialised structural mask       */
/* ------------------------------------------------------------------ */

/* cls [B, nQT, nKT] in {0 empty, 1 partial, 2 full} over in-range (i, j);
 * sep_pos [B, T] ascending positions of separators j >= n_start, then -1;
 * sep_count [B]; ranges [B, nQT, 2] = (#sep with j < t*BM - w,
 * #sep with j < last_row(t) - w), counted over separators j >= n_start. */
int oracle_blockmap(int B, int T, int n_start, int w, int BM, int BN, const uint8_t* is_sep,
                    uint8_t* cls, int32_t* sep_pos, int32_t* sep_count, int32_t* ranges) {
  if (B <= 0 || T <= 0 || BM <= 0 || BN <= 0 || n_start < 0 || w < 0) return OR_ERR_ARG;
  int nQT = (T + BM - 1) / BM, nKT = (T + BN - 1) / BN;
  uint8_t* m = (uint8_t*)malloc((size_t)T);
  int64_t* kept = (int64_t*)calloc((size_t)nKT, sizeof(int64_t));
  int64_t* total = (int64_t*)calloc((size_t)nKT, sizeof(int64_t));
  if (!m || !kept || !total) return OR_ERR_MEM;
  for (int b = 0; b < B; ++b) {
    const uint8_t* sep = is_sep ? is_sep + (size_t)b * T : NULL;
    for (int t = 0; t < nQT; ++t) {
      memset(kept, 0, sizeof(int64_t) * nKT);
      memset(total, 0, sizeof(int64_t) * nKT);
      for (int i = t * BM; i < (t + 1) * BM && i < T; ++i) {
        oracle_mask_row(T, i, n_start, w, sep, m);
        for (int j = 0; j < T; ++j) {
          kept[j / BN] += m[j];
          total[j / BN] += 1;
        }
      }
      for (int u = 0; u < nKT; ++u) {
        uint8_t c = kept[u] == 0 ? 0 : (kept[u] == total[u] ? 2 : 1);
        cls[((size_t)b * nQT + t) * nKT + u] = c;
      }
    }
    int32_t cnt = 0;
    for (int j = 0; j < T; ++j) {
      sep_pos[(size_t)b * T + j] = -1;
    }
    for (int j = n_start; j < T; ++j)
      if (sep && sep[j]) sep_pos[(size_t)b * T + cnt++] = j;
    sep_count[b] = cnt;
    for (int t = 0; t < nQT; ++t) {
      int first = t * BM;
      int last = (t + 1) * BM - 1;
      if (last > T - 1) last = T - 1;
      int32_t full = 0, any = 0;
      for (int j = n_start; j < T; ++j) {
        if (!(sep && sep[j])) continue;
        if (j < first - w) ++full;
        if (j < last - w) ++any;
      }
      ranges[((size_t)b * nQT + t) * 2 + 0] = full;
      ranges[((size_t)b * nQT + t) * 2 + 1] = any;
    }
  }
  free(m);
  free(kept);
  free(total);
  return OR_OK;
}

/* ------------------------------------------------------------------ */
/* segmented execution ([SEG]; readings R9, R10)                       */
/* ------------------------------------------------------------------ */

typedef struct {
  double s;
  int32_t blk;
} blk_t;

static int blk_cmp(const void* a, const void* b) {
  const blk_t* x = (const blk_t*)a;
  const blk_t* y = (const blk_t*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->blk < y->blk) ? -1 : (x->blk > y->blk);
}

static int int_cmp(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

/* Retrieval for segment s >= 1 of one (b, h): the prefix blocks, ascending.
 * Block score = max_{j in block} <q_{sS-1}, k_j>, both unrotated.  Writes
 * nb = R/blk entries (or fewer, then -1), returns the number selected.
 * scores (optional) receives the block scores in block order. */
static int retrieve_blocks(const double* qlast, const double* Kraw, int d, int pool, int blk,
                           int nb, int32_t* out, double* scores) {
  int nblocks = pool / blk;
  blk_t* bs = (blk_t*)malloc(sizeof(blk_t) * (size_t)(nblocks + 1));
  for (int u = 0; u < nblocks; ++u) {
    double best = -INFINITY;
    for (int j = u * blk; j < (u + 1) * blk; ++j) {
      double z = dot(qlast, Kraw + (size_t)j * d, d);
      if (z > best) best = z;
    }
    bs[u].s = best;
    bs[u].blk = u;
    if (scores) scores[u] = best;
  }
  qsort(bs, (size_t)nblocks, sizeof(blk_t), blk_cmp);
  int nsel = nblocks < nb ? nblocks : nb;
  for (int r = 0; r < nsel; ++r) out[r] = bs[r].blk;
  qsort(out, (size_t)nsel, sizeof(int32_t), int_cmp);
  for (int r = nsel; r < nb; ++r) out[r] = -1;
  free(bs);
  return nsel;
}

/* The key list of row i of (b, h) in segmented execution: global key
 * indices kj[] and their rotary positions kp[]; *P_out = prefix/tail length.
 * Local heads: tail [sS-M, sS) at positions 0..P-1, then the segment.
 * Long heads: the retrieved prefix at positions 0..P-1, then the segment.
 * The segment's keys sS..i sit at P + (j - sS); the query at P + (i - sS). */
static int segment_key_list(const void* Q, const oracle_params* p, const double* Kraw, int S, int M, int R,
                            int blk, const uint8_t* is_long, int b, int h, int i, int32_t* kj, int32_t* kp,
                            int* P_out, int32_t* blocks, double* qlast) {
  int T = p->T, d = p->d;
  int s = i / S, seg0 = s * S, nb = R / blk;
  int n = 0;
  if (is_long[h]) {
    if (s >= 1 && nb > 0) {
      int64_t qb = (((int64_t)b * p->Hq + h) * T + (seg0 - 1)) * d;
      for (int c = 0; c < d; ++c) qlast[c] = load_elem(Q, p->dtype, qb + c);
      int nsel = retrieve_blocks(qlast, Kraw, d, seg0, blk, nb, blocks, NULL);
      for (int u = 0; u < nsel; ++u)
        for (int x = 0; x < blk; ++x) {
          kj[n] = blocks[u] * blk + x;
          kp[n] = n;
          ++n;
        }
    }
  } else if (s >= 1) {
    int lo = seg0 - M;
    if (lo < 0) lo = 0;
    for (int j = lo; j < seg0; ++j) {
      kj[n] = j;
      kp[n] = n;
      ++n;
    }
  }
  int P = n;
  for (int j = seg0; j <= i; ++j) {
    kj[n] = j;
    kp[n] = P + (j - seg0);
    ++n;
  }
  *P_out = P;
  return n;
}

/* Exported for the tests: key list of one row (K decoded here). */
int oracle_segment_keys(const oracle_params* p, int S, int M, int R, int blk, const uint8_t* is_long,
                        const void* Q, const void* K, int b, int h, int i, int32_t* kj, int32_t* kp,
                        int32_t* P_out) {
  if (!p || S <= 0 || blk <= 0 || R % blk || i < 0 || i >= p->T) return OR_ERR_ARG;
  int T = p->T, d = p->d;
  int g = (int)(((int64_t)h * p->Hkv) / p->Hq);
  double* Kraw = (double*)malloc(sizeof(double) * (size_t)T * d);
  double* qlast = (double*)malloc(sizeof(double) * (size_t)d);
  int32_t* blocks = (int32_t*)malloc(sizeof(int32_t) * (size_t)(R / blk + 1));
  int64_t kb = ((int64_t)b * p->Hkv + g) * (int64_t)T * d;
  for (int64_t x = 0; x < (int64_t)T * d; ++x) Kraw[x] = load_elem(K, p->dtype, kb + x);
  int P = 0;
  int n = segment_key_list(Q, p, Kraw, S, M, R, blk, is_long, b, h, i, kj, kp, &P, blocks, qlast);
  *P_out = P;
  free(Kraw);
  free(qlast);
  free(blocks);
  return n;
}

typedef struct {
  const oracle_params* p;
  int S, M, R, blk;
  const uint8_t* is_long;
  const void* Q;
  const double* Kraw;
  const double* Vd;
  const int64_t* rows;
  const int64_t* sel;
  double* O;
  double* lse;
  int64_t* counts;
} seg_job;

static void seg_one(void* a, int64_t t) {
  seg_job* J = (seg_job*)a;
  const oracle_params* p = J->p;
  int T = p->T, d = p->d;
  int64_t r = J->sel[t];
  int b = (int)J->rows[3 * r], h = (int)J->rows[3 * r + 1], i = (int)J->rows[3 * r + 2];
  int s = i / J->S, tt = i - s * J->S;
  int nb = J->R / J->blk;
  /* key list: global index + rotary position */
  int cap = J->M + J->R + J->S + 1;
  int32_t* kj = (int32_t*)malloc(sizeof(int32_t) * (size_t)cap);
  int32_t* kp = (int32_t*)malloc(sizeof(int32_t) * (size_t)cap);
  int32_t* blocks = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nb + 1));
  double* q = (double*)malloc(sizeof(double) * 4 * (size_t)d);
  double* qrot = q + d;
  double* krot = q + 2 * d;
  double* qlast = q + 3 * d;
  int64_t qb = (((int64_t)b * p->Hq + h) * T) * d;
  for (int c = 0; c < d; ++c) q[c] = load_elem(J->Q, p->dtype, qb + (int64_t)i * d + c);
  int P = 0;
  int n = segment_key_list(J->Q, p, J->Kraw, J->S, J->M, J->R, J->blk, J->is_long, b, h, i, kj, kp, &P,
                           blocks, qlast);
  oracle_rope(q, d, rot_pos(p, (double)(P + tt)), p->rope_theta, qrot);
  double inv_sqrt_d = 1.0 / sqrt((double)d);
  double* sbuf = (double*)malloc(sizeof(double) * (size_t)(n + 1));
  double mx = -INFINITY;
  for (int x = 0; x < n; ++x) {
    oracle_rope(J->Kraw + (size_t)kj[x] * d, d, rot_pos(p, (double)kp[x]), p->rope_theta, krot);
    sbuf[x] = dot(qrot, krot, d) * inv_sqrt_d;
    if (sbuf[x] > mx) mx = sbuf[x];
  }
  double sum = 0.0;
  for (int x = 0; x < n; ++x) sum += exp(sbuf[x] - mx);
  double lse = mx + log(sum);
  double* o = J->O + r * d;
  for (int c = 0; c < d; ++c) o[c] = 0.0;
  for (int x = 0; x < n; ++x) {
    double pj = exp(sbuf[x] - lse);
    const double* vj = J->Vd + (size_t)kj[x] * d;
    for (int c = 0; c < d; ++c) o[c] += pj * vj[c];
  }
  J->lse[r] = lse;
  if (J->counts) J->counts[r] = n;
  free(sbuf);
  free(kj);
  free(kp);
  free(blocks);
  free(q);
}

int oracle_segment_rows(const oracle_params* p, int S, int M, int R, int blk, const uint8_t* is_long,
                        const void* Q, const void* K, const void* V, int64_t n, const int64_t* rows,
                        double* O, double* lse, int64_t* counts, int nthreads) {
  if (!p || S <= 0 || M < 0 || R < 0 || blk <= 0 || R % blk || p->T % S || p->Hq % p->Hkv)
    return OR_ERR_ARG;
  int T = p->T, d = p->d;
  double* Kraw = (double*)malloc(sizeof(double) * (size_t)T * d);
  double* Krot = (double*)malloc(sizeof(double) * (size_t)T * d);
  double* Vd = (double*)malloc(sizeof(double) * (size_t)T * d);
  int64_t* sel = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n + 1));
  if (!Kraw || !Krot || !Vd || !sel) return OR_ERR_MEM;
  for (int b = 0; b < p->B; ++b)
    for (int g = 0; g < p->Hkv; ++g) {
      int64_t ns = 0;
      for (int64_t r = 0; r < n; ++r) {
        int rb = (int)rows[3 * r], rh = (int)rows[3 * r + 1];
        if (rb == b && (int)(((int64_t)rh * p->Hkv) / p->Hq) == g) sel[ns++] = r;
      }
      if (!ns) continue;
      load_head(p, K, V, b, g, Kraw, Krot, Vd);
      seg_job J;
      J.p = p;
      J.S = S;
      J.M = M;
      J.R = R;
      J.blk = blk;
      J.is_long = is_long;
      J.Q = Q;
      J.Kraw = Kraw;
      J.Vd = Vd;
      J.rows = rows;
      J.sel = sel;
      J.O = O;
      J.lse = lse;
      J.counts = counts;
      run_parallel(seg_one, &J, ns, nthreads);
    }
  free(Kraw);
  free(Krot);
  free(Vd);
  free(sel);
  return OR_OK;
}

/* Backward of segmented execution: gradients of L = sum dO . O with each
 * row's key list (tail or retrieved prefix, then the segment causally) and
 * its rotary positions as in oracle_segment_rows; the retrieval selection,
 * like the top-k sets, is a constant of the backward pass.  Per kept key x
 * of row i (source position kj_x, rotary position kp_x, query position
 * P + t): z_x = <R(P + t) q_i, R(kp_x) k_{kj_x}> / sqrt(d), p = softmax(z),
 * dz_x = p_x (dO_i . v_{kj_x} - D_i), D_i = sum_x p_x dO_i . v_{kj_x};
 * dq_i = R(P+t)^T sum_x dz_x R(kp_x) k, dk_{kj_x} += R(kp_x)^T dz_x R(P+t) q_i,
 * dv_{kj_x} += p_x dO_i.  One job per (batch, kv head), rows in order. */
typedef struct {
  const oracle_params* p;
  int S, M, R, blk;
  const uint8_t* is_long;
  const void *Q, *K, *V, *dO;
  double *dQ, *dK, *dV;
} segbwd_job;

static void segbwd_one(void* a, int64_t t) {
  segbwd_job* J = (segbwd_job*)a;
  const oracle_params* p = J->p;
  int T = p->T, d = p->d;
  int b = (int)(t / p->Hkv), g = (int)(t % p->Hkv);
  int nb = J->R / J->blk;
  int cap = J->M + J->R + J->S + 1;
  double* Kraw = (double*)malloc(sizeof(double) * (size_t)T * d);
  double* Krot = (double*)malloc(sizeof(double) * (size_t)T * d);
  double* Vd = (double*)malloc(sizeof(double) * (size_t)T * d);
  double* gK = (double*)calloc((size_t)T * d, sizeof(double));
  double* gV = (double*)calloc((size_t)T * d, sizeof(double));
  int32_t* kj = (int32_t*)malloc(sizeof(int32_t) * (size_t)cap);
  int32_t* kp = (int32_t*)malloc(sizeof(int32_t) * (size_t)cap);
  int32_t* blocks = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nb + 1));
  double* kr = (double*)malloc(sizeof(double) * (size_t)cap * d); /* R(kp_x) k_{kj_x} */
  double* sbuf = (double*)malloc(sizeof(double) * (size_t)cap);
  double* dpb = (double*)malloc(sizeof(double) * (size_t)cap);
  double* w = (double*)malloc(sizeof(double) * 8 * (size_t)d);
  double *q = w, *qrot = w + d, *doi = w + 2 * d, *gq = w + 3 * d, *tmp = w + 4 * d, *qlast = w + 6 * d;
  load_head(p, J->K, J->V, b, g, Kraw, Krot, Vd);
  int rep = p->Hq / p->Hkv;
  double inv_sqrt_d = 1.0 / sqrt((double)d);
  for (int h = g * rep; h < (g + 1) * rep; ++h) {
    for (int i = 0; i < T; ++i) {
      int s = i / J->S, tt = i - s * J->S;
      int64_t qb = (((int64_t)b * p->Hq + h) * T + i) * d;
      for (int c = 0; c < d; ++c) {
        q[c] = load_elem(J->Q, p->dtype, qb + c);
        doi[c] = load_elem(J->dO, p->dtype, qb + c);
      }
      int P = 0;
      int n = segment_key_list(J->Q, p, Kraw, J->S, J->M, J->R, J->blk, J->is_long, b, h, i, kj, kp, &P, blocks,
                               qlast);
      oracle_rope(q, d, rot_pos(p, (double)(P + tt)), p->rope_theta, qrot);
      double mx = -INFINITY;
      for (int x = 0; x < n; ++x) {
        oracle_rope(Kraw + (size_t)kj[x] * d, d, rot_pos(p, (double)kp[x]), p->rope_theta, kr + (size_t)x * d);
        sbuf[x] = dot(qrot, kr + (size_t)x * d, d) * inv_sqrt_d;
        if (sbuf[x] > mx) mx = sbuf[x];
      }
      double sum = 0.0;
      for (int x = 0; x < n; ++x) sum += exp(sbuf[x] - mx);
      double lse = mx + log(sum);
      double D = 0.0;
      for (int x = 0; x < n; ++x) {
        sbuf[x] = exp(sbuf[x] - lse); /* now P_x */
        dpb[x] = dot(doi, Vd + (size_t)kj[x] * d, d);
        D += sbuf[x] * dpb[x];
      }
      for (int c = 0; c < d; ++c) gq[c] = 0.0;
      for (int x = 0; x < n; ++x) {
        double dz = sbuf[x] * (dpb[x] - D) * inv_sqrt_d;
        double* gv = gV + (size_t)kj[x] * d;
        for (int c = 0; c < d; ++c) {
          gv[c] += sbuf[x] * doi[c];
          gq[c] += dz * kr[(size_t)x * d + c];
        }
        /* d L / d k_{kj_x} = R(kp_x)^T dz R(P + t) q_i */
        for (int c = 0; c < d; ++c) tmp[c] = dz * qrot[c];
        oracle_rope(tmp, d, -rot_pos(p, (double)kp[x]), p->rope_theta, tmp + d);
        double* gk = gK + (size_t)kj[x] * d;
        for (int c = 0; c < d; ++c) gk[c] += tmp[d + c];
      }
      oracle_rope(gq, d, -rot_pos(p, (double)(P + tt)), p->rope_theta, tmp);
      for (int c = 0; c < d; ++c) J->dQ[qb + c] = tmp[c];
    }
  }
  int64_t kb = ((int64_t)b * p->Hkv + g) * (int64_t)T * d;
  for (int64_t x = 0; x < (int64_t)T * d; ++x) {
    J->dK[kb + x] = gK[x];
    J->dV[kb + x] = gV[x];
  }
  free(Kraw);
  free(Krot);
  free(Vd);
  free(gK);
  free(gV);
  free(kj);
  free(kp);
  free(blocks);
  free(kr);
  free(sbuf);
  free(dpb);
  free(w);
}

int oracle_segment_bwd(const oracle_params* p, int S, int M, int R, int blk, const uint8_t* is_long, const void* Q,
                       const void* K, const void* V, const void* dO, double* dQ, double* dK, double* dV,
                       int nthreads) {
  if (!p || !is_long || S <= 0 || M < 0 || R < 0 || blk <= 0 || R % blk || p->T % S || p->Hq % p->Hkv ||
      p->d <= 0 || (p->d & 1))
    return OR_ERR_ARG;
  segbwd_job J;
  J.p = p;
  J.S = S;
  J.M = M;
  J.R = R;
  J.blk = blk;
  J.is_long = is_long;
  J.Q = Q;
  J.K = K;
  J.V = V;
  J.dO = dO;
  J.dQ = dQ;
  J.dK = dK;
  J.dV = dV;
  run_parallel(segbwd_one, &J, (int64_t)p->B * p->Hkv, nthreads);
  return OR_OK;
}

/* Prefix blocks [B, Hq, N, R/blk] for every head flagged long (rows of
 * local heads and of segment 0 are -1); block scores of the retrieval for
 * the near-tie exemption go to scores_kth [B, Hq, N, 2] = (score of the
 * last selected block, score of the best unselected block). */
int oracle_segment_blocks(const oracle_params* p, int S, int R, int blk, const uint8_t* is_long,
                          const void* Q, const void* K, int32_t* prefix_blocks, double* scores_kth) {
  if (!p || S <= 0 || R < 0 || blk <= 0 || R % blk || p->T % S) return OR_ERR_ARG;
  int T = p->T, d = p->d, N = T / S, nb = R / blk;
  double* Kraw = (double*)malloc(sizeof(double) * (size_t)T * d);
  double* qlast = (double*)malloc(sizeof(double) * (size_t)d);
  double* scores = (double*)malloc(sizeof(double) * (size_t)(T / blk + 1));
  if (!Kraw || !qlast || !scores) return OR_ERR_MEM;
  for (int b = 0; b < p->B; ++b)
    for (int h = 0; h < p->Hq; ++h) {
      int g = (int)(((int64_t)h * p->Hkv) / p->Hq);
      int64_t kb = ((int64_t)b * p->Hkv + g) * (int64_t)T * d;
      for (int64_t x = 0; x < (int64_t)T * d; ++x) Kraw[x] = load_elem(K, p->dtype, kb + x);
      for (int s = 0; s < N; ++s) {
        int32_t* out = prefix_blocks + (((size_t)b * p->Hq + h) * N + s) * nb;
        double* sk = scores_kth ? scores_kth + (((size_t)b * p->Hq + h) * N + s) * 2 : NULL;
        for (int r = 0; r < nb; ++r) out[r] = -1;
        if (sk) sk[0] = sk[1] = -INFINITY;
        if (!is_long[h] || s == 0 || nb == 0) continue;
        int64_t qb = (((int64_t)b * p->Hq + h) * T + (s * S - 1)) * d;
        for (int c = 0; c < d; ++c) qlast[c] = load_elem(Q, p->dtype, qb + c);
        int nsel = retrieve_blocks(qlast, Kraw, d, s * S, blk, nb, out, scores);
        if (sk) {
          /* k-th best selected and best unselected */
          int nblocks = s * S / blk;
          double kth = INFINITY, best_out = -INFINITY;
          for (int u = 0; u < nblocks; ++u) {
            int chosen = 0;
            for (int r = 0; r < nsel; ++r) chosen |= (out[r] == u);
            if (chosen && scores[u] < kth) kth = scores[u];
            if (!chosen && scores[u] > best_out) best_out = scores[u];
          }
          sk[0] = kth;
          sk[1] = best_out;
        }
      }
    }
  free(Kraw);
  free(qlast);
  free(scores);
  return OR_OK;
}
