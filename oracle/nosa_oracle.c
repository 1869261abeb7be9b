/*
 * nosa_oracle.c -- plain, slow, fp64 CPU oracle of one NOSA decode step.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline / reference arm may load this library. It shares no
 * code with the CUDA library (no headers, helpers or tables).
 *
 * What it computes, per GQA group (b, g) and decode step t (sources are the
 * pages collected on NOSA, "Native and Offloadable Sparse Attention", the
 * Spanish technical summary at gist.science/es/paper/2510.13602, section
 * "Metodologia" 1 and 2, and the SparDA summary gist.science/de/paper/2606.04511,
 * section 2 "Kompakter Forecast-Indexer"):
 *
 *  append      the new key/value become token L-1 (L = context length after the
 *              append); the mean key of its sub-block is recomputed from the
 *              sub-block's present tokens.                    (NOSA 2, memory layout)
 *  score       two-stage pooling: sub-block score
 *                  u_i = (1/R) sum_r  sigma * (q_r . kbar_i)
 *              with kbar_i the mean key of sub-block i, then block score
 *                  s_j = max over the non-empty sub-blocks i of block j of u_i.
 *              No softmax (pre-exponential scores, NOSA 1 "ED-DMA"; SparDA's
 *              compact indexer drops it too). R rows = the group's G query heads,
 *              or one forecast row.               (NOSA 1 "Implementacion Basada en Bloques")
 *  select      query-agnostic set first: candidates C_e = S(t-1) & A(t-1); Gamma_e
 *              = top-min(k_e, |C_e|) of the eviction scores over C_e; candidates
 *              not chosen leave A for good (NOSA 1 "Seleccion Independiente de la
 *              Consulta": a block not selected at t is never selected at t' > t).
 *              Query-aware set: Gamma_q = top-min(k - |Gamma_e|, N - |Gamma_e|) of
 *              the block scores over all blocks outside Gamma_e ("Seleccion Sensible
 *              a la Consulta": may return to evicted blocks). S(t) = union,
 *              ascending. Order: higher score first, ties to the lower index.
 *              S(-1) = A(-1) = every prefill block.
 *              Since Gamma_e is a subset of S(t-1), |S(t) & S(t-1)| >= k_e, the
 *              locality bound gamma(t) >= k_e / k ("Garantia de Localidad").
 *  residency   (offload configurations; NOSA 2 "Layout de Memoria Optimizado":
 *              set difference for block swapping) misses = (S(t) + tail) minus the
 *              HBM-resident set; free slots first (ascending), then victims = the
 *              least recently used resident blocks outside S(t) + tail (ties to the
 *              lower index), taken in ascending block order; misses ascending are
 *              paired with that slot list in order; last_used = L for S(t) + tail.
 *  attend      exact softmax attention of every query head of the group over
 *              the tokens (< L) of the blocks of S(t), ascending:
 *                  o_h = sum_tau softmax_tau(sigma q_h . K_tau) V_tau
 *              computed max-subtracted in fp64.
 *
 * Inputs are bf16 bit patterns (uint16) widened exactly to double; eviction
 * scores are fp32 widened exactly. All accumulation is fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int32_t B, Hq, Hkv, d;
  int32_t bs, s;          /* block size, sub-block size (tokens) */
  int32_t k_q, k_e;
  int32_t n_rows;         /* scoring rows per group: G or 1 */
  int32_t max_blocks;     /* blocks per group the caches can hold */
  int32_t slots;          /* HBM slots per group (offload model) */
  int32_t offload;        /* 1: model HBM residency */
  int32_t score_mode;     /* scoring variant bits, see orc_block_scores (0: the NOSA pool) */
  int32_t kc_bf16;        /* 1: sub-block means stored as bf16 (see sub_mean) */
  double scale;           /* sigma = 1/sqrt(d) */
} orc_cfg;

typedef struct {
  uint16_t* K;            /* [B][Hkv][max_blocks*bs][d] bf16 */
  uint16_t* V;
  double* kbar;           /* [B][Hkv][max_sub][d] sub-block mean keys */
  int32_t* len;           /* [B][Hkv] tokens present */
  uint8_t* prev_sel;      /* [B][Hkv][max_blocks] S(t-1) */
  uint8_t* alive;         /* [B][Hkv][max_blocks] A(t-1) */
  int32_t* block_slot;    /* [B][Hkv][max_blocks] HBM slot or -1 */
  int32_t* slot_owner;    /* [B][Hkv][slots] block or -1 */
  int32_t* last_used;     /* [B][Hkv][max_blocks] */
} orc_state;

static double bf(uint16_t u) {
  uint32_t x = (uint32_t)u << 16;
  float f;
  memcpy(&f, &x, 4);
  return (double)f;
}

static int cdiv(int a, int b) { return (a + b - 1) / b; }

static int n_groups(const orc_cfg* c) { return c->B * c->Hkv; }
static int max_sub(const orc_cfg* c) { return c->max_blocks * (c->bs / c->s); }
static size_t tok_off(const orc_cfg* c, int gi, int tau) {
  return ((size_t)gi * c->max_blocks * c->bs + (size_t)tau) * c->d;
}

/* Mean key of sub-block i over its present tokens (fp64). */
/* bf16 bit pattern of a finite float, rounded to nearest, ties to even (the definition:
 * add half of the dropped part's unit, plus one when the kept part is odd, then truncate). */
static uint16_t bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* Mean key of sub-block i over its present tokens. fp64, or with kc_bf16 the value a bf16
 * store of the mean holds: the kernels sum the bf16 tokens in fp32 in token order, divide in
 * fp32 (correctly rounded) and round to bf16 (nearest, ties to even); the oracle takes that
 * quantisation the same way so that both sides hold the same codes. */
static void sub_mean(const orc_cfg* c, const orc_state* st, int gi, int i, double* out) {
  const int L = st->len[gi];
  const int t0 = i * c->s;
  const int t1 = (t0 + c->s < L) ? t0 + c->s : L;
  for (int x = 0; x < c->d; ++x) out[x] = 0.0;
  if (t1 <= t0) return;
  if (c->kc_bf16) {
    for (int x = 0; x < c->d; ++x) {
      float sum = 0.0f;
      for (int tau = t0; tau < t1; ++tau) sum += (float)bf(st->K[tok_off(c, gi, tau) + x]);
      out[x] = bf((uint16_t)bf16_rne(sum / (float)(t1 - t0)));
    }
    return;
  }
  for (int tau = t0; tau < t1; ++tau) {
    const uint16_t* k = st->K + tok_off(c, gi, tau);
    for (int x = 0; x < c->d; ++x) out[x] += bf(k[x]);
  }
  for (int x = 0; x < c->d; ++x) out[x] /= (double)(t1 - t0);
}

/* ------------------------------------------------------------------ top-m */

typedef struct { double key; int idx; } orc_item;

static int item_cmp(const void* a, const void* b) {
  const orc_item* x = (const orc_item*)a;
  const orc_item* y = (const orc_item*)b;
  if (x->key > y->key) return -1;
  if (x->key < y->key) return 1;
  return (x->idx < y->idx) ? -1 : (x->idx > y->idx);
}

/*
 * Top-m of key over the candidates (cand[i] != 0): higher key first, equal keys
 * to the lower index. chosen[i] = 1 for the m picked. *gap = key of the last
 * picked minus key of the first not picked (INFINITY when either is missing).
 * Returns the number picked, min(m, #candidates).
 */
int orc_topm(int n, const double* key, const uint8_t* cand, int m, uint8_t* chosen, double* gap) {
  orc_item* it = (orc_item*)malloc(sizeof(orc_item) * (size_t)(n > 0 ? n : 1));
  int nc = 0;
  for (int i = 0; i < n; ++i) {
    chosen[i] = 0;
    if (cand[i]) { it[nc].key = key[i]; it[nc].idx = i; ++nc; }
  }
  qsort(it, (size_t)nc, sizeof(orc_item), item_cmp);
  const int take = (m < nc) ? m : nc;
  for (int r = 0; r < take; ++r) chosen[it[r].idx] = 1;
  if (gap) *gap = (take >= 1 && take < nc) ? it[take - 1].key - it[take].key : INFINITY;
  free(it);
  return take;
}

/* ------------------------------------------------------------------ state */

int orc_init(const orc_cfg* c, orc_state* st, const int32_t* prefill_len, const uint8_t* resident) {
  const int NG = n_groups(c), nb = c->max_blocks, MS = max_sub(c);
  for (int gi = 0; gi < NG; ++gi) {
    const int b = gi / c->Hkv;
    const int T = prefill_len[b];
    if (T < 0 || T > nb * c->bs) return -1;
    st->len[gi] = T;
    const int n0 = cdiv(T, c->bs);
    for (int j = 0; j < nb; ++j) {
      st->prev_sel[(size_t)gi * nb + j] = (uint8_t)(j < n0);
      st->alive[(size_t)gi * nb + j] = 1;
      st->last_used[(size_t)gi * nb + j] = 0;
    }
    if (c->offload) {
      int used = 0;
      for (int z = 0; z < c->slots; ++z) st->slot_owner[(size_t)gi * c->slots + z] = -1;
      for (int j = 0; j < nb; ++j) {
        int32_t* bsl = st->block_slot + (size_t)gi * nb + j;
        *bsl = -1;
        if (resident && resident[(size_t)gi * nb + j]) {
          if (used >= c->slots) return -2;
          *bsl = used;
          st->slot_owner[(size_t)gi * c->slots + used] = j;
          ++used;
        }
      }
    }
  }
#pragma omp parallel for schedule(dynamic) collapse(2)
  for (int gi = 0; gi < NG; ++gi)
    for (int i = 0; i < MS; ++i) sub_mean(c, st, gi, i, st->kbar + ((size_t)gi * MS + i) * c->d);
  return 0;
}

void orc_append(const orc_cfg* c, orc_state* st, const uint16_t* k_new, const uint16_t* v_new) {
  const int NG = n_groups(c), MS = max_sub(c);
#pragma omp parallel for schedule(static)
  for (int gi = 0; gi < NG; ++gi) {
    const int pos = st->len[gi];
    memcpy(st->K + tok_off(c, gi, pos), k_new + (size_t)gi * c->d, sizeof(uint16_t) * c->d);
    memcpy(st->V + tok_off(c, gi, pos), v_new + (size_t)gi * c->d, sizeof(uint16_t) * c->d);
    st->len[gi] = pos + 1;
    const int i = pos / c->s;
    sub_mean(c, st, gi, i, st->kbar + ((size_t)gi * MS + i) * c->d);
  }
}

/* Block scores of the two-stage pool; blocks at or beyond N get -INFINITY.
 * gmask (NULL = all) restricts the call to the groups with gmask[gi] != 0.
 *
 * Scoring variants (score_mode bits; 0 is the pool described at the top):
 *   1  windows: the unit that starts at sub-block i pools the tokens [i*s, i*s + 2s) (its
 *      present ones) instead of [i*s, (i+1)*s): SparDA's inference window of kernel 32 and
 *      stride 16 at s = 16 (gist.science/de/paper/2606.04511, section 2,
 *      "Trainingsstrategie"). Its mean key is the count-weighted mean of the sub-block means
 *      of sub-blocks i and i+1, which is the mean over the window's tokens.
 *   2  softmax: for each scoring row r a softmax over all the group's units of
 *      sigma * (q_r . mean key), summed over the rows (the per-head scoring loop with
 *      softmax that SparDA's compact indexer removes, section 2 "Kompakter
 *      Forecast-Indexer"), instead of the mean of the raw logits.
 * Block score: the max over the units that start inside the block. */
void orc_block_scores(const orc_cfg* c, const orc_state* st, const uint16_t* rows, double* scores,
                      const uint8_t* gmask) {
  const int NG = n_groups(c), nb = c->max_blocks, MS = max_sub(c), spb = c->bs / c->s;
  const int R = c->n_rows;
  const int win = (c->score_mode & 1) != 0, soft = (c->score_mode & 2) != 0;
#pragma omp parallel for schedule(dynamic)
  for (int gi = 0; gi < NG; ++gi) {
    if (gmask && !gmask[gi]) continue;
    const int L = st->len[gi];
    const int M = cdiv(L, c->s);
    double* out = scores + (size_t)gi * nb;
    for (int j = 0; j < nb; ++j) out[j] = -INFINITY;
    if (M == 0) continue;
    double* z = (double*)malloc(sizeof(double) * (size_t)R * M);   /* logits [r][i] */
    double* kb = (double*)malloc(sizeof(double) * c->d);
    for (int i = 0; i < M; ++i) {
      const double* k0 = st->kbar + ((size_t)gi * MS + i) * c->d;
      const int n0 = (L - i * c->s < c->s) ? L - i * c->s : c->s;
      int n1 = 0;
      if (win && i + 1 < M) n1 = (L - (i + 1) * c->s < c->s) ? L - (i + 1) * c->s : c->s;
      for (int x = 0; x < c->d; ++x) kb[x] = k0[x];
      if (n1 > 0) {
        const double* k1 = st->kbar + ((size_t)gi * MS + i + 1) * c->d;
        for (int x = 0; x < c->d; ++x) kb[x] = (n0 * k0[x] + n1 * k1[x]) / (double)(n0 + n1);
      }
      for (int r = 0; r < R; ++r) {
        const uint16_t* q = rows + ((size_t)gi * R + r) * c->d;
        double dot = 0.0;
        for (int x = 0; x < c->d; ++x) dot += bf(q[x]) * kb[x];
        z[(size_t)r * M + i] = c->scale * dot;
      }
    }
    double* mx = (double*)malloc(sizeof(double) * 2 * R);  /* per row: max, sum of exp */
    double* den = mx + R;
    if (soft) {
      for (int r = 0; r < R; ++r) {
        const double* zr = z + (size_t)r * M;
        mx[r] = -INFINITY;
        den[r] = 0.0;
        for (int i = 0; i < M; ++i) if (zr[i] > mx[r]) mx[r] = zr[i];
        for (int i = 0; i < M; ++i) den[r] += exp(zr[i] - mx[r]);
      }
    }
    for (int i = 0; i < M; ++i) {
      double u = 0.0;
      if (soft) {
        for (int r = 0; r < R; ++r) u += exp(z[(size_t)r * M + i] - mx[r]) / den[r];
      } else {
        for (int r = 0; r < R; ++r) u += z[(size_t)r * M + i];
        u /= (double)R;
      }
      const int j = i / spb;
      if (u > out[j]) out[j] = u;
    }
    free(mx);
    free(kb);
    free(z);
  }
}

/*
 * Dual selection. sel[gi][0..k) = S(t) ascending, padded with -1; src = 1 for
 * Gamma_e, 2 for Gamma_q, 0 for padding. gap_q = margin of the query-aware cut.
 * commit != 0 updates prev_sel and alive; commit == 0 only previews. gmask as above.
 */
void orc_select(const orc_cfg* c, orc_state* st, const double* scores, const float* evict,
                int32_t* sel, int8_t* src, double* gap_q, int commit, const uint8_t* gmask) {
  const int NG = n_groups(c), nb = c->max_blocks, k = c->k_q + c->k_e;
#pragma omp parallel for schedule(dynamic)
  for (int gi = 0; gi < NG; ++gi) {
    if (gmask && !gmask[gi]) continue;
    const int L = st->len[gi];
    const int N = cdiv(L, c->bs);
    uint8_t* ps = st->prev_sel + (size_t)gi * nb;
    uint8_t* al = st->alive + (size_t)gi * nb;
    double* ekey = (double*)malloc(sizeof(double) * (size_t)nb);
    uint8_t* cand = (uint8_t*)malloc((size_t)nb);
    uint8_t* ge = (uint8_t*)malloc((size_t)nb);
    uint8_t* gq = (uint8_t*)malloc((size_t)nb);
    /* query-agnostic set over C_e = S(t-1) & A(t-1) */
    for (int j = 0; j < nb; ++j) {
      ekey[j] = (double)evict[(size_t)gi * nb + j];
      cand[j] = (uint8_t)(j < N && ps[j] && al[j]);
    }
    const int ne = orc_topm(nb, ekey, cand, c->k_e, ge, NULL);
    /* query-aware set over every block outside Gamma_e */
    for (int j = 0; j < nb; ++j) cand[j] = (uint8_t)(j < N && !ge[j]);
    const int mq = (k - ne < N - ne) ? k - ne : N - ne;
    double gap = INFINITY;
    orc_topm(nb, scores + (size_t)gi * nb, cand, mq, gq, &gap);
    if (gap_q) gap_q[gi] = gap;
    int w = 0;
    for (int j = 0; j < nb; ++j) {
      if (ge[j] || gq[j]) {
        sel[(size_t)gi * k + w] = j;
        if (src) src[(size_t)gi * k + w] = ge[j] ? 1 : 2;
        ++w;
      }
    }
    for (; w < k; ++w) {
      sel[(size_t)gi * k + w] = -1;
      if (src) src[(size_t)gi * k + w] = 0;
    }
    if (commit) {
      for (int j = 0; j < nb; ++j) {
        if (j < N && ps[j] && al[j] && !ge[j]) al[j] = 0; /* dropped from C_e: evicted */
      }
      for (int j = 0; j < nb; ++j) ps[j] = (uint8_t)(ge[j] || gq[j]);
    }
    free(ekey); free(cand); free(ge); free(gq);
  }
}

typedef struct { int32_t lu; int idx; } orc_lru;

static int lru_cmp(const void* a, const void* b) {
  const orc_lru* x = (const orc_lru*)a;
  const orc_lru* y = (const orc_lru*)b;
  if (x->lu != y->lu) return (x->lu < y->lu) ? -1 : 1;
  return (x->idx < y->idx) ? -1 : (x->idx > y->idx);
}

/* HBM residency model; returns 0, or -1 when no victim can be found. */
int orc_residency(const orc_cfg* c, orc_state* st, const int32_t* sel, int32_t* miss_count) {
  const int NG = n_groups(c), nb = c->max_blocks, k = c->k_q + c->k_e;
  int bad = 0;
  if (!c->offload) {
    for (int gi = 0; gi < NG; ++gi) miss_count[gi] = 0;
    return 0;
  }
#pragma omp parallel for schedule(dynamic) reduction(| : bad)
  for (int gi = 0; gi < NG; ++gi) {
    const int L = st->len[gi];
    const int tail = (L - 1) / c->bs;
    int32_t* bsl = st->block_slot + (size_t)gi * nb;
    int32_t* own = st->slot_owner + (size_t)gi * c->slots;
    int32_t* lu = st->last_used + (size_t)gi * nb;
    uint8_t* need = (uint8_t*)calloc((size_t)nb, 1);
    int* misses = (int*)malloc(sizeof(int) * (size_t)(k + 1));
    int* zl = (int*)malloc(sizeof(int) * (size_t)(k + 1));
    orc_lru* vc = (orc_lru*)malloc(sizeof(orc_lru) * (size_t)nb);
    int* vict = (int*)malloc(sizeof(int) * (size_t)(k + 1));
    for (int w = 0; w < k; ++w) {
      const int j = sel[(size_t)gi * k + w];
      if (j >= 0) need[j] = 1;
    }
    need[tail] = 1;
    int nm = 0;
    for (int j = 0; j < nb; ++j)
      if (need[j] && bsl[j] < 0) misses[nm++] = j;
    int nz = 0;
    for (int z = 0; z < c->slots && nz < nm; ++z)
      if (own[z] < 0) zl[nz++] = z;
    const int nv = nm - nz;
    if (nv > 0) {
      int nvc = 0;
      for (int j = 0; j < nb; ++j)
        if (bsl[j] >= 0 && !need[j]) { vc[nvc].lu = lu[j]; vc[nvc].idx = j; ++nvc; }
      if (nvc < nv) {
        bad |= 1;
      } else {
        qsort(vc, (size_t)nvc, sizeof(orc_lru), lru_cmp);
        uint8_t* isv = (uint8_t*)calloc((size_t)nb, 1);
        for (int r = 0; r < nv; ++r) isv[vc[r].idx] = 1;
        int w = 0;
        for (int j = 0; j < nb; ++j)
          if (isv[j]) vict[w++] = j;
        for (int r = 0; r < nv; ++r) {
          const int z = bsl[vict[r]];
          zl[nz++] = z;
          own[z] = -1;
          bsl[vict[r]] = -1;
        }
        free(isv);
      }
    }
    if (nz >= nm) {
      for (int r = 0; r < nm; ++r) {
        bsl[misses[r]] = zl[r];
        own[zl[r]] = misses[r];
      }
    }
    for (int j = 0; j < nb; ++j)
      if (need[j]) lu[j] = L;
    miss_count[gi] = nm;
    free(need); free(misses); free(zl); free(vc); free(vict);
  }
  return bad ? -1 : 0;
}

/* Exact softmax attention of the group's query heads over the selected tokens. */
void orc_attend(const orc_cfg* c, const orc_state* st, const uint16_t* q, const int32_t* sel,
                double* out) {
  const int NG = n_groups(c), G = c->Hq / c->Hkv, k = c->k_q + c->k_e, d = c->d;
#pragma omp parallel for schedule(dynamic) collapse(2)
  for (int gi = 0; gi < NG; ++gi) {
    for (int r = 0; r < G; ++r) {
      const int b = gi / c->Hkv, g = gi % c->Hkv;
      const int h = g * G + r;
      const int L = st->len[gi];
      const uint16_t* qh = q + ((size_t)b * c->Hq + h) * d;
      double* o = out + ((size_t)b * c->Hq + h) * d;
      double* z = (double*)malloc(sizeof(double) * (size_t)k * c->bs + 1);
      int* tk = (int*)malloc(sizeof(int) * (size_t)k * c->bs + 1);
      int nt = 0;
      double zmax = -INFINITY;
      for (int w = 0; w < k; ++w) {
        const int j = sel[(size_t)gi * k + w];
        if (j < 0) continue;
        for (int tau = j * c->bs; tau < (j + 1) * c->bs && tau < L; ++tau) {
          const uint16_t* kt = st->K + tok_off(c, gi, tau);
          double dot = 0.0;
          for (int x = 0; x < d; ++x) dot += bf(qh[x]) * bf(kt[x]);
          z[nt] = c->scale * dot;
          tk[nt] = tau;
          if (z[nt] > zmax) zmax = z[nt];
          ++nt;
        }
      }
      for (int x = 0; x < d; ++x) o[x] = 0.0;
      double den = 0.0;
      for (int n = 0; n < nt; ++n) {
        const double p = exp(z[n] - zmax);
        const uint16_t* vt = st->V + tok_off(c, gi, tk[n]);
        den += p;
        for (int x = 0; x < d; ++x) o[x] += p * bf(vt[x]);
      }
      for (int x = 0; x < d; ++x) o[x] = (nt > 0) ? o[x] / den : 0.0;
      free(z);
      free(tk);
    }
  }
}

/* S2O's monotone-gain early stop (gist.science/it/paper/2602.22575, "Regola di Arresto
 * Anticipato"), applied to the selected blocks of a step. The blocks of S(t) are visited in
 * decreasing block score (ties: lower index), the estimated importance, and every query
 * head of the group runs the online softmax over them block by block. After block b the
 * head's gain on b,
 *     dl = sum over the tokens tau < L of b of exp(z_tau - m)     (m: running max after b)
 * is compared with the accumulated mass l, which includes b: once dl < tau_stop * l the
 * head stops (b is kept). o_h = acc / l at that point; tau_stop <= 0 never stops.
 * used[b][h]: blocks the head visited. margin[gi]: the smallest |dl / l - tau_stop| / tau_stop
 * over every decision taken in the group (INFINITY if none). order_gap[gi]: the smallest
 * difference between the scores (their logs when score_mode has the softmax bit: those are
 * probabilities) of consecutive blocks of the order, over the pairs that decide which
 * blocks the heads visit (INFINITY if none). */
void orc_attend_stop(const orc_cfg* c, const orc_state* st, const uint16_t* q, const int32_t* sel,
                     const double* scores, double tau_stop, double* out, int32_t* used,
                     double* margin, double* order_gap) {
  const int NG = n_groups(c), G = c->Hq / c->Hkv, k = c->k_q + c->k_e, d = c->d;
  const int nb = c->max_blocks;
#pragma omp parallel for schedule(dynamic)
  for (int gi = 0; gi < NG; ++gi) {
    const int b = gi / c->Hkv, g = gi % c->Hkv;
    const int L = st->len[gi];
    orc_item* it = (orc_item*)malloc(sizeof(orc_item) * (size_t)(k + 1));
    int n = 0;
    for (int w = 0; w < k; ++w) {
      const int j = sel[(size_t)gi * k + w];
      if (j < 0) continue;
      it[n].key = scores[(size_t)gi * nb + j];
      it[n].idx = j;
      ++n;
    }
    qsort(it, n, sizeof(orc_item), item_cmp);
    double* acc = (double*)malloc(sizeof(double) * d);
    double* zb = (double*)malloc(sizeof(double) * c->bs);
    double mg = INFINITY;
    int maxu = 0;
    for (int r = 0; r < G; ++r) {
      const int h = g * G + r;
      const uint16_t* qh = q + ((size_t)b * c->Hq + h) * d;
      double m = -INFINITY, l = 0.0;
      for (int x = 0; x < d; ++x) acc[x] = 0.0;
      int u = 0;
      for (int p = 0; p < n; ++p) {
        const int j = it[p].idx;
        const int t0 = j * c->bs, t1 = ((j + 1) * c->bs < L) ? (j + 1) * c->bs : L;
        double bm = -INFINITY;
        for (int tau = t0; tau < t1; ++tau) {
          const uint16_t* kt = st->K + tok_off(c, gi, tau);
          double dot = 0.0;
          for (int x = 0; x < d; ++x) dot += bf(qh[x]) * bf(kt[x]);
          zb[tau - t0] = c->scale * dot;
          if (zb[tau - t0] > bm) bm = zb[tau - t0];
        }
        const double m2 = (bm > m) ? bm : m;
        const double rescale = (m == -INFINITY) ? 0.0 : exp(m - m2);
        for (int x = 0; x < d; ++x) acc[x] *= rescale;
        l *= rescale;
        double dl = 0.0;
        for (int tau = t0; tau < t1; ++tau) {
          const double e = exp(zb[tau - t0] - m2);
          const uint16_t* vt = st->V + tok_off(c, gi, tau);
          dl += e;
          for (int x = 0; x < d; ++x) acc[x] += e * bf(vt[x]);
        }
        l += dl;
        m = m2;
        ++u;
        if (tau_stop > 0.0) {
          const double ratio = dl / l;
          const double rel = fabs(ratio - tau_stop) / tau_stop;
          if (rel < mg) mg = rel;
          if (ratio < tau_stop) break;
        }
      }
      if (u > maxu) maxu = u;
      used[(size_t)b * c->Hq + h] = u;
      double* o = out + ((size_t)b * c->Hq + h) * d;
      for (int x = 0; x < d; ++x) o[x] = (l > 0.0) ? acc[x] / l : 0.0;
    }
    /* positions 0 .. maxu-1 are visited by some head: the pairs (p, p+1) with p < maxu
       (and p + 1 < n) decide which blocks those are */
    double og = INFINITY;
    if (tau_stop > 0.0)
      for (int p = 0; p < maxu && p + 1 < n; ++p) {
        const double gp = (c->score_mode & 2) ? log(it[p].key) - log(it[p + 1].key)
                                              : it[p].key - it[p + 1].key;
        if (gp < og) og = gp;
      }
    margin[gi] = mg;
    order_gap[gi] = og;
    free(zb);
    free(acc);
    free(it);
  }
}
