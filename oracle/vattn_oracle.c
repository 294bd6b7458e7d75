/*
 * Oracle for one verified-sparse-attention (vAttention) decode step.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg load this library. The product path (the CUDA
 * library and its Python binding) never calls it, and this file shares no code,
 * header or constant table with that path.
 *
 * Plain, slow, single-threaded C. Each step follows the pages in their order:
 *
 *   [VB] "vAttention: A New Approach to Sparse Attention with Guaranteed
 *        Accuracy" (edgentiq blog), section "How vAttention Works": attention
 *        splits into heavy hitters plus a long tail; a deterministic index set
 *        (attention sinks, a sliding window, predicted top-k) is combined with a
 *        uniform random sample of the remaining indices, whose size is chosen
 *        from the Central Limit Theorem so that the user's (eps, delta) accuracy
 *        holds; the paragraph after it says the guarantee is placed on the
 *        softmax denominator, calling that a relaxation of guaranteeing the
 *        attention output (the numerator as well) which makes the budget
 *        cheaper to compute. The unrelaxed form is the output guarantee here.
 *   [SQ] "SparQ Attention: Bandwidth-Efficient LLM Inference", abstract:
 *        approximate scores from selectively fetched parts of the cache.
 *   [LK] "Loki: Low-rank Keys for Efficient Sparse Attention", abstract: rank
 *        tokens by attention scores computed in a low-dimensional key space.
 *   [PH] Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1,
 *        2, 3", SC'11: the Philox4x32-10 counter-based generator.
 *   [CW] Cody and Waite, "Software Manual for the Elementary Functions" (1980):
 *        two-constant reduction of exp's argument by multiples of ln 2.
 *
 * Where the pages leave a step open, the reading taken is stated at that step.
 * Decisions that pick integers (ranking order, sample positions, budgets) are
 * taken in fp32 with an explicitly fixed operation order, so that a GPU
 * implementation of the same readings reproduces them bit for bit; the output
 * itself is computed in double.
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fPIC -shared (no fast-math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F32 0
#define ORC_BF16 1

#define ORC_EXACT 0
#define ORC_SPARQ 1
#define ORC_LOKI 2

#define ORC_GUARANTEE_DENOMINATOR 0
#define ORC_GUARANTEE_OUTPUT 1

typedef unsigned __int128 u128;

typedef struct {
  int batch, num_q_heads, num_kv_heads, head_dim, dtype;
  int page_size, pages_per_seq, max_ctx;
  int proxy, proxy_rank;
  int sinks, window;
  int topk_abs, topk_num, topk_den;
  int pilot_min, pilot_num, pilot_den;
  float eps, delta;
  uint64_t seed;
  int guarantee; /* ORC_GUARANTEE_DENOMINATOR or ORC_GUARANTEE_OUTPUT */
  int topp_num, topp_den; /* topp_den > 0: top-p selection with p = topp_num / topp_den */
  int batch_offset, head_offset; /* a shard's first sequence and KV head in the whole batch */
} orc_problem;

/* ------------------------------------------------------------------ */
/* Philox4x32-10 [PH]: ten rounds of two 32x32->64 multiplies, the high */
/* halves xored with the other two words and the round key; the key is  */
/* bumped by two Weyl constants between rounds.                         */
/* ------------------------------------------------------------------ */
void orc_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
  const uint32_t mult0 = 0xD2511F53u, mult1 = 0xCD9E8D57u;
  const uint32_t weyl0 = 0x9E3779B9u, weyl1 = 0xBB67AE85u;
  uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
  uint32_t k0 = key_in[0], k1 = key_in[1];
  for (int round = 0; round < 10; round++) {
    if (round > 0) {
      k0 += weyl0;
      k1 += weyl1;
    }
    uint64_t p0 = (uint64_t)mult0 * c0;
    uint64_t p1 = (uint64_t)mult1 * c2;
    uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
    uint32_t n1 = (uint32_t)p1;
    uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
    uint32_t n3 = (uint32_t)p0;
    c0 = n0; c1 = n1; c2 = n2; c3 = n3;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* Draw t of unit (b, h): counter (t/4, b, h, 0), key = the 64-bit seed split */
/* into (low word, high word); the draw is word t%4 of that block. b and h   */
/* name the sequence and KV head in the whole batch: a shard of a batch adds */
/* its offsets, so that the shards draw what the whole batch would.          */
uint32_t orc_draw_word(uint64_t seed, uint32_t b, uint32_t h, uint32_t t) {
  uint32_t ctr[4] = {t >> 2, b, h, 0u};
  uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  uint32_t out[4];
  orc_philox4x32_10(ctr, key, out);
  return out[t & 3u];
}

/* ------------------------------------------------------------------ */
/* exp for x <= 0 in fp32 with a fixed operation order.                 */
/* n = nearest integer to x*log2(e); r = x - n*C1 - n*C2 with the [CW]   */
/* split ln2 = C1 + C2 (C1 has 9 significant bits so n*C1 is exact);    */
/* e^r by its Taylor series to degree 7 in Horner form (|r| <= 0.35, so  */
/* the truncation error is below 1e-8 relative); result = p * 2^n.       */
/* Below -87 the result would leave the normal range: it returns 0.     */
/* ------------------------------------------------------------------ */
float orc_vexp(float x) {
  if (!(x >= -87.0f)) return 0.0f;
  const float log2e = 1.44269504088896341f;
  const float c1 = 0.693359375f;
  const float c2 = -2.12194440054690583e-4f;
  float n = rintf(x * log2e);
  float r = fmaf(-n, c1, x);
  r = fmaf(-n, c2, r);
  /* 1/k! for k = 7 .. 0 */
  float p = 1.98412698412698413e-4f;      /* 1/5040  */
  p = fmaf(p, r, 1.38888888888888889e-3f); /* 1/720   */
  p = fmaf(p, r, 8.33333333333333333e-3f); /* 1/120   */
  p = fmaf(p, r, 4.16666666666666667e-2f); /* 1/24    */
  p = fmaf(p, r, 1.66666666666666667e-1f); /* 1/6     */
  p = fmaf(p, r, 0.5f);
  p = fmaf(p, r, 1.0f);
  p = fmaf(p, r, 1.0f);
  int ni = (int)n;
  uint32_t bits = (uint32_t)(ni + 127) << 23;
  float scale;
  memcpy(&scale, &bits, 4);
  return p * scale;
}

void orc_vexp_array(const float* x, float* y, long n) {
  for (long i = 0; i < n; i++) y[i] = orc_vexp(x[i]);
}

/* ------------------------------------------------------------------ */
/* z_{1-delta/2}: 200 bisection steps on [0, 40] of the upper normal    */
/* tail 0.5*erfc(z/sqrt2) against delta/2 (the CLT quantile of [VB]).   */
/* ------------------------------------------------------------------ */
double orc_z(double delta) {
  double lo = 0.0, hi = 40.0, target = 0.5 * delta;
  for (int it = 0; it < 200; it++) {
    double mid = 0.5 * (lo + hi);
    if (0.5 * erfc(mid * 0.70710678118654752440) > target)
      lo = mid;
    else
      hi = mid;
  }
  return 0.5 * (lo + hi);
}

/* ------------------------------------------------------------------ */
/* Element access                                                       */
/* ------------------------------------------------------------------ */
static float elem(const void* base, size_t idx, int dtype) {
  if (dtype == ORC_F32) return ((const float*)base)[idx];
  uint32_t u = (uint32_t)((const uint16_t*)base)[idx] << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

static size_t elem_size(int dtype) { return dtype == ORC_F32 ? 4 : 2; }

/* Physical page holding position pos of sequence b. */
static size_t page_of(const orc_problem* pr, const int32_t* page_table, int b, int pos) {
  return (size_t)page_table[(size_t)b * pr->pages_per_seq + pos / pr->page_size];
}

/* Index of the first element of row pos, in a [pages][Hkv][page_size][width] cache. */
static size_t row_base(const orc_problem* pr, const int32_t* page_table, int b, int h, int pos,
                       int width) {
  size_t page = page_of(pr, page_table, b, pos);
  return ((page * pr->num_kv_heads + h) * pr->page_size + pos % pr->page_size) * (size_t)width;
}

/* ------------------------------------------------------------------ */
/* fp32 dot in the fixed order used for every score that decides an    */
/* integer: the n elements are cut into 16-byte chunks (4 fp32 or 8     */
/* bf16 values); each chunk is a fused multiply-add chain from 0 in     */
/* ascending element order; the chunk sums are then added pairwise,     */
/* halving the stride each time (chunk l += chunk l+L/2, ..., l += l+1).*/
/* ------------------------------------------------------------------ */
static float dot_chunked(const float* q, const void* base, size_t off, int n, int dtype) {
  int per = (int)(16 / elem_size(dtype));
  int nchunks = n / per;
  float part[64];
  for (int l = 0; l < nchunks; l++) {
    float acc = 0.0f;
    for (int i = l * per; i < (l + 1) * per; i++) acc = fmaf(q[i], elem(base, off + i, dtype), acc);
    part[l] = acc;
  }
  for (int stride = nchunks / 2; stride >= 1; stride /= 2)
    for (int l = 0; l < stride; l++) part[l] = part[l] + part[l + stride];
  return part[0];
}

float orc_dot_chunked(const float* q, const void* k, int n, int dtype) {
  return dot_chunked(q, k, 0, n, dtype);
}

/* Order-preserving map of an fp32 score onto uint32 (-0 counts as +0). */
uint32_t orc_ord(float f) {
  uint32_t u;
  if (f == 0.0f) f = 0.0f;
  memcpy(&u, &f, 4);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

static int cmp_u64_desc(const void* a, const void* b) {
  uint64_t x = *(const uint64_t*)a, y = *(const uint64_t*)b;
  return x < y ? 1 : (x > y ? -1 : 0);
}

static int cmp_i32_asc(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return x < y ? -1 : (x > y ? 1 : 0);
}

/* ------------------------------------------------------------------ */
/* One unit (sequence b, KV head h).                                    */
/* ------------------------------------------------------------------ */
typedef struct {
  const void *q, *k_cache, *v_cache, *k_t_cache, *k_proj_cache;
  const float* proj_basis;
  const int32_t *page_table, *seq_lens;
} orc_inputs;

typedef struct {
  double* out;
  int32_t *sel_idx, *sel_count, *budgets, *head_need;
  double *den_hat, *ref_max;
} orc_outputs;

static void decode_unit(const orc_problem* pr, const orc_inputs* in, const orc_outputs* ot, int b,
                        int h, double z) {
  const int d = pr->head_dim, Hq = pr->num_q_heads, Hkv = pr->num_kv_heads;
  const int G = Hq / Hkv;
  const int dt = pr->dtype;
  const int N = in->seq_lens[b];
  const size_t unit = (size_t)b * Hkv + h;
  int32_t* sel = ot->sel_idx + unit * (size_t)pr->max_ctx;

  /* queries of the group, as fp32 */
  float* qh = malloc(sizeof(float) * (size_t)G * d);
  for (int g = 0; g < G; g++)
    for (int i = 0; i < d; i++)
      qh[g * d + i] = elem(in->q, ((size_t)b * Hq + h * G + g) * d + i, dt);

  if (N <= 0) {
    for (int g = 0; g < G; g++) {
      for (int i = 0; i < d; i++) ot->out[((size_t)b * Hq + h * G + g) * d + i] = 0.0;
      ot->head_need[(size_t)b * Hq + h * G + g] = 0;
      if (ot->den_hat) ot->den_hat[(size_t)b * Hq + h * G + g] = 0.0;
      if (ot->ref_max) ot->ref_max[(size_t)b * Hq + h * G + g] = 0.0;
    }
    ot->sel_count[unit] = 0;
    ot->budgets[unit] = 0;
    free(qh);
    return;
  }

  /* Ranking query: mean of the group's queries, summed as a pairwise tree   */
  /* over adjacent heads, then scaled by 1/G (a power of two, so exact).     */
  /* Reading: the pages rank tokens per KV head; with grouped queries one    */
  /* index set is shared by the group, ranked by the group-mean query.       */
  float* qbar = malloc(sizeof(float) * d);
  {
    float* tmp = malloc(sizeof(float) * (size_t)G * d);
    memcpy(tmp, qh, sizeof(float) * (size_t)G * d);
    for (int stride = 1; stride < G; stride *= 2)
      for (int g = 0; g + stride < G; g += 2 * stride)
        for (int i = 0; i < d; i++) tmp[g * d + i] = tmp[g * d + i] + tmp[(g + stride) * d + i];
    for (int i = 0; i < d; i++) qbar[i] = tmp[i] * (1.0f / (float)G);
    free(tmp);
  }
  const float scale = (float)(1.0 / sqrt((double)d));

  /* Regions [VB]: sinks [0, s1), window [wst, N), middle M = [s1, wst). */
  const int s1 = pr->sinks < N ? pr->sinks : N;
  const int wst = (N - pr->window) > s1 ? (N - pr->window) : s1;
  const int mlen = wst - s1;
  long long kb = pr->topk_den ? ((long long)N * pr->topk_num) / pr->topk_den : pr->topk_abs;
  long long pb = pr->pilot_min;
  if (pr->pilot_den) {
    long long c = ((long long)N * pr->pilot_num + pr->pilot_den - 1) / pr->pilot_den;
    if (c > pb) pb = c;
  }
  const int p = (int)pb;

  /* Ranking scores over M. */
  float* rs = malloc(sizeof(float) * (size_t)(mlen > 0 ? mlen : 1));
  if (pr->proxy == ORC_EXACT) {
    for (int j = s1; j < wst; j++)
      rs[j - s1] = dot_chunked(qbar, in->k_cache, row_base(pr, in->page_table, b, h, j, d), d, dt);
  } else if (pr->proxy == ORC_SPARQ) {
    /* [SQ] reading: the r query components of largest magnitude (ties to  */
    /* the lower dimension), used in ascending dimension order; the score  */
    /* is one fused multiply-add chain over those dimensions.              */
    const int r = pr->proxy_rank;
    int* dims = malloc(sizeof(int) * r);
    char* taken = calloc((size_t)d, 1);
    for (int t = 0; t < r; t++) {
      int best = -1;
      for (int i = 0; i < d; i++)
        if (!taken[i] && (best < 0 || fabsf(qbar[i]) > fabsf(qbar[best]))) best = i;
      taken[best] = 1;
      dims[t] = best;
    }
    qsort(dims, (size_t)r, sizeof(int), cmp_i32_asc);
    for (int j = s1; j < wst; j++) {
      size_t page = page_of(pr, in->page_table, b, j);
      float acc = 0.0f;
      for (int t = 0; t < r; t++) {
        /* dim-major copy: [pages][Hkv][d][page_size] */
        size_t idx = ((page * Hkv + h) * d + dims[t]) * (size_t)pr->page_size + j % pr->page_size;
        acc = fmaf(qbar[dims[t]], elem(in->k_t_cache, idx, dt), acc);
      }
      rs[j - s1] = acc;
    }
    free(dims);
    free(taken);
  } else {
    /* [LK]: project the ranking query onto the stored low-rank basis       */
    /* (one fused chain over d per component), then score the stored       */
    /* projected keys with the chunked dot.                                 */
    const int rk = pr->proxy_rank;
    float* qt = malloc(sizeof(float) * rk);
    for (int c = 0; c < rk; c++) {
      float acc = 0.0f;
      for (int i = 0; i < d; i++) acc = fmaf(qbar[i], in->proj_basis[((size_t)h * d + i) * rk + c], acc);
      qt[c] = acc;
    }
    for (int j = s1; j < wst; j++)
      rs[j - s1] = dot_chunked(qt, in->k_proj_cache, row_base(pr, in->page_table, b, h, j, rk), rk, dt);
    free(qt);
  }

  /* Top-k over M: largest score first, equal scores to the lower position  */
  /* (reading: the pages give no tie rule). Key = ord(score) * 2^32 + (2^32-1-j). */
  uint64_t* keys = malloc(sizeof(uint64_t) * (size_t)(mlen > 0 ? mlen : 1));
  for (int j = s1; j < wst; j++)
    keys[j - s1] = ((uint64_t)orc_ord(rs[j - s1]) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)j);
  qsort(keys, (size_t)mlen, sizeof(uint64_t), cmp_u64_desc);
  int kk = (int)(kb < mlen ? kb : mlen);
  if (pr->topp_den > 0) {
    /* Top-p (reading: the pages name top-p selection as the mass-threshold   */
    /* variant of top-k and give no formula): the smallest number of the     */
    /* highest-ranked middle positions, in the key order above, whose share  */
    /* of the middle's softmax mass under the scaled ranking scores reaches  */
    /* p = topp_num / topp_den. Mass in 2^-32 fixed point, as the budget's:  */
    /* x_j = vexp(fl(r_j c) - max_M fl(r c)), xq_j = rint(x_j 2^32), so the  */
    /* cut is an exact integer comparison: prefix * den >= num * S.          */
    float mx = -INFINITY;
    for (int j = 0; j < mlen; j++) {
      float sc = rs[j] * scale;
      if (sc > mx) mx = sc;
    }
    uint64_t S = 0;
    for (int j = 0; j < mlen; j++) S += (uint64_t)llrintf(orc_vexp(rs[j] * scale - mx) * 4294967296.0f);
    const u128 target = (u128)S * (u128)(uint64_t)pr->topp_num;
    u128 prefix = 0;
    kk = 0;
    while (kk < mlen && prefix * (u128)(uint64_t)pr->topp_den < target) {
      const int j = (int)(0xFFFFFFFFu - (uint32_t)(keys[kk] & 0xFFFFFFFFu));
      prefix += (u128)(uint64_t)llrintf(orc_vexp(rs[j - s1] * scale - mx) * 4294967296.0f);
      kk++;
    }
  }
  int32_t* topk = malloc(sizeof(int32_t) * (size_t)(kk > 0 ? kk : 1));
  for (int i = 0; i < kk; i++) topk[i] = (int32_t)(0xFFFFFFFFu - (uint32_t)(keys[i] & 0xFFFFFFFFu));
  qsort(topk, (size_t)kk, sizeof(int32_t), cmp_i32_asc);
  free(keys);

  /* Deterministic set I_f, ascending; tail T = M minus top-k, ascending. */
  const int nI = s1 + kk + (N - wst);
  const int ntail = mlen - kk;
  int32_t* If = malloc(sizeof(int32_t) * (size_t)nI);
  {
    int w = 0;
    for (int j = 0; j < s1; j++) If[w++] = j;
    for (int i = 0; i < kk; i++) If[w++] = topk[i];
    for (int j = wst; j < N; j++) If[w++] = j;
  }
  int32_t* tail = malloc(sizeof(int32_t) * (size_t)(ntail > 0 ? ntail : 1));
  {
    int w = 0, ti = 0;
    for (int j = s1; j < wst; j++) {
      if (ti < kk && topk[ti] == j) {
        ti++;
        continue;
      }
      tail[w++] = j;
    }
  }

  /* Budget [VB]: pilot sample of p uniform tail draws (with replacement),   */
  /* per-head statistics of x = exp(s - m) in 2^-32 fixed point, then       */
  /* n_h = (z * N_tail * sigma / (eps * D))^2 with sigma^2 the unbiased      */
  /* pilot variance and D = sum over I_f + N_tail * pilot mean.             */
  int exhausted = 0, bsz = 0;
  int* need_h = malloc(sizeof(int) * G);
  if (ntail == 0) {
    for (int g = 0; g < G; g++) need_h[g] = 0;
  } else if (ntail <= p) {
    exhausted = 1;
    bsz = ntail;
    for (int g = 0; g < G; g++) need_h[g] = ntail;
  } else {
    int32_t* pil = malloc(sizeof(int32_t) * (size_t)p);
    for (int t = 0; t < p; t++) {
      uint32_t u = orc_draw_word(pr->seed, (uint32_t)(b + pr->batch_offset), (uint32_t)(h + pr->head_offset), (uint32_t)t);
      uint32_t rho = (uint32_t)(((uint64_t)u * (uint64_t)ntail) >> 32);
      pil[t] = tail[rho];
    }
    float* sf = malloc(sizeof(float) * (size_t)nI);
    float* sp = malloc(sizeof(float) * (size_t)p);
    float* xf = malloc(sizeof(float) * (size_t)nI);
    float* xp = malloc(sizeof(float) * (size_t)p);
    int nmax = 0;
    for (int g = 0; g < G; g++) {
      const float* qg = qh + (size_t)g * d;
      float m = -INFINITY;
      for (int i = 0; i < nI; i++) {
        sf[i] = dot_chunked(qg, in->k_cache, row_base(pr, in->page_table, b, h, If[i], d), d, dt) * scale;
        if (sf[i] > m) m = sf[i];
      }
      for (int t = 0; t < p; t++) {
        sp[t] = dot_chunked(qg, in->k_cache, row_base(pr, in->page_table, b, h, pil[t], d), d, dt) * scale;
        if (sp[t] > m) m = sp[t];
      }
      uint64_t Sf = 0, S1 = 0;
      u128 S2 = 0;
      for (int i = 0; i < nI; i++) {
        float x = orc_vexp(sf[i] - m);
        xf[i] = x;
        Sf += (uint64_t)llrintf(x * 4294967296.0f);
      }
      for (int t = 0; t < p; t++) {
        float x = orc_vexp(sp[t] - m);
        xp[t] = x;
        uint64_t xq = (uint64_t)llrintf(x * 4294967296.0f);
        S1 += xq;
        S2 += (u128)xq * xq;
      }
      u128 V = (u128)(uint64_t)p * S2 - (u128)S1 * S1;
      double Vd = (double)(uint64_t)(V >> 64) * 18446744073709551616.0 + (double)(uint64_t)V;
      double var = Vd / ((double)p * (double)(p - 1));
      double Dq = (double)Sf + ((double)ntail * (double)S1) / (double)p;
      double t = (z * (double)ntail) / ((double)pr->eps * Dq);
      double need = (t * t) * var;
      int nh = need >= (double)ntail ? ntail : (int)ceil(need);
      if (pr->guarantee == ORC_GUARANTEE_OUTPUT) {
        /* Output guarantee (reading: the pages state only that the         */
        /* denominator-only budget relaxes it). The same CLT condition is   */
        /* put on the numerator vector Nv = sum_j x_j v_j: estimated from   */
        /* b tail draws, its error has covariance N_tail^2 Sigma / b with   */
        /* Sigma the covariance of x v over the tail, so its expected       */
        /* squared length is N_tail^2 tr(Sigma) / b, and                    */
        /*   n >= (z * N_tail / (eps * |Nv|))^2 * tr(Sigma),                */
        /* tr(Sigma) = sum over dims of the unbiased pilot variance of x v, */
        /* Nv_hat = (sum over I_f of x v) + N_tail * (pilot mean), and      */
        /* |Nv|^2 its lower confidence bound below.                         */
        /* In double: each product x * v is exact (24 x 24 significant      */
        /* bits at most); sums run over I_f in list order and over the      */
        /* pilot in draw order, then over dims ascending. A negative        */
        /* variance (rounding) counts as 0.                                 */
        double tr = 0.0, nsq = 0.0;
        for (int e = 0; e < d; e++) {
          double A = 0.0, T1 = 0.0, T2 = 0.0;
          for (int i = 0; i < nI; i++)
            A = A + (double)xf[i] * (double)elem(in->v_cache, row_base(pr, in->page_table, b, h, If[i], d) + e, dt);
          for (int t = 0; t < p; t++) {
            double y = (double)xp[t] * (double)elem(in->v_cache, row_base(pr, in->page_table, b, h, pil[t], d) + e, dt);
            T1 = T1 + y;
            T2 = T2 + y * y;
          }
          double ve = ((double)p * T2 - T1 * T1) / ((double)p * (double)(p - 1));
          if (ve < 0.0) ve = 0.0;
          double Ne = A + ((double)ntail * T1) / (double)p;
          tr = tr + ve;
          nsq = nsq + Ne * Ne;
        }
        /* |Nv|^2 is sized from a one-sided lower confidence bound. The     */
        /* pilot mean's noise, with covariance C = N_tail^2 Sigma / p and   */
        /* energy R = tr(C), adds R to |Nv_hat|^2 in expectation, so         */
        /* nsq_u = |Nv_hat|^2 - R is unbiased. Its variance is              */
        /* 4 Nv' C Nv + 2 tr(C^2) <= 4 |Nv|^2 R + 2 R^2 (the largest         */
        /* eigenvalue of C is at most its trace), so                        */
        /*   L = nsq_u - z * sqrt(4 max(nsq_u, 0) R + 2 R^2)                */
        /* undershoots |Nv|^2 with probability about delta / 2 or less.     */
        /* When L is not positive the pilot cannot bound |Nv| away from 0   */
        /* and the whole tail is taken (unless every variance is 0).        */
        double R = (((double)ntail * (double)ntail) / (double)p) * tr;
        double nsq_u = nsq - R;
        double se2 = 4.0 * (nsq_u > 0.0 ? nsq_u : 0.0) * R + 2.0 * R * R;
        double L = nsq_u - z * sqrt(se2);
        double need_v;
        if (L > 0.0) {
          double tv = (z * (double)ntail) / ((double)pr->eps * sqrt(L));
          need_v = (tv * tv) * tr;
        } else {
          need_v = tr > 0.0 ? (double)ntail : 0.0;
        }
        int nv = need_v >= (double)ntail ? ntail : (int)ceil(need_v);
        if (nv > nh) nh = nv;
      }
      need_h[g] = nh;
      if (nh > nmax) nmax = nh;
    }
    bsz = nmax > p ? nmax : p;
    if (bsz >= ntail) {
      exhausted = 1;
      bsz = ntail;
    }
    free(pil);
    free(sf);
    free(sp);
    free(xf);
    free(xp);
  }

  /* Selected list: I_f, then the b draws in draw order (the pilot is the    */
  /* prefix of the sample; reading), or the whole tail when exhausted.      */
  const int nsel = nI + ((ntail == 0) ? 0 : bsz);
  const int ndet = exhausted ? nsel : nI; /* entries with weight 1 */
  for (int i = 0; i < nI; i++) sel[i] = If[i];
  if (exhausted) {
    for (int t = 0; t < ntail; t++) sel[nI + t] = tail[t];
  } else if (ntail > 0) {
    for (int t = 0; t < bsz; t++) {
      uint32_t u = orc_draw_word(pr->seed, (uint32_t)(b + pr->batch_offset), (uint32_t)(h + pr->head_offset), (uint32_t)t);
      uint32_t rho = (uint32_t)(((uint64_t)u * (uint64_t)ntail) >> 32);
      sel[nI + t] = tail[rho];
    }
  }
  ot->sel_count[unit] = nsel;
  ot->budgets[unit] = ntail == 0 ? 0 : bsz;

  /* Output, in double: softmax over the selected set with the sampled     */
  /* terms reweighted by N_tail / b (each draw counted once per occurrence). */
  const double rscale = 1.0 / sqrt((double)d);
  const double w = (exhausted || ntail == 0) ? 1.0 : (double)ntail / (double)bsz;
  double* sd = malloc(sizeof(double) * (size_t)nsel);
  double* Af = malloc(sizeof(double) * d);
  double* As = malloc(sizeof(double) * d);
  for (int g = 0; g < G; g++) {
    const float* qg = qh + (size_t)g * d;
    double M = -INFINITY;
    for (int i = 0; i < nsel; i++) {
      size_t kb0 = row_base(pr, in->page_table, b, h, sel[i], d);
      double acc = 0.0;
      for (int e = 0; e < d; e++) acc += (double)qg[e] * (double)elem(in->k_cache, kb0 + e, dt);
      sd[i] = acc * rscale;
      if (sd[i] > M) M = sd[i];
    }
    double Lf = 0.0, Ls = 0.0;
    for (int e = 0; e < d; e++) Af[e] = As[e] = 0.0;
    for (int i = 0; i < nsel; i++) {
      double ex = exp(sd[i] - M);
      size_t vb0 = row_base(pr, in->page_table, b, h, sel[i], d);
      if (i < ndet) {
        Lf += ex;
        for (int e = 0; e < d; e++) Af[e] += ex * (double)elem(in->v_cache, vb0 + e, dt);
      } else {
        Ls += ex;
        for (int e = 0; e < d; e++) As[e] += ex * (double)elem(in->v_cache, vb0 + e, dt);
      }
    }
    const size_t qi = (size_t)b * Hq + h * G + g;
    const double den = Lf + w * Ls;
    for (int e = 0; e < d; e++) ot->out[qi * d + e] = (Af[e] + w * As[e]) / den;
    ot->head_need[qi] = need_h[g];
    if (ot->den_hat) ot->den_hat[qi] = den;
    if (ot->ref_max) ot->ref_max[qi] = M;
  }

  free(sd); free(Af); free(As);
  free(need_h); free(If); free(tail); free(topk); free(rs); free(qbar); free(qh);
}

/* ------------------------------------------------------------------ */
/* Entry: decode the listed units (unit = b * num_kv_heads + h), or all */
/* units when units == NULL. Layouts are those of the CUDA library:     */
/* q [B][Hq][d]; k/v [pages][Hkv][page_size][d]; dim-major K            */
/* [pages][Hkv][d][page_size]; projected K [pages][Hkv][page_size][rank];*/
/* basis fp32 [Hkv][d][rank]; page_table [B][pages_per_seq]; out        */
/* [B][Hq][d] (double here); sel_idx [B][Hkv][max_ctx]; sel_count and   */
/* budgets [B][Hkv]; head_need [B][Hq]; den_hat and ref_max [B][Hq]     */
/* optional (the estimated denominator relative to exp(ref_max)).       */
/* ------------------------------------------------------------------ */
int orc_decode(const orc_problem* pr, const void* q, const void* k_cache, const void* v_cache,
               const void* k_t_cache, const void* k_proj_cache, const float* proj_basis,
               const int32_t* page_table, const int32_t* seq_lens, const int32_t* units,
               int n_units, double* out, int32_t* sel_idx, int32_t* sel_count, int32_t* budgets,
               int32_t* head_need, double* den_hat, double* ref_max) {
  if (pr->num_kv_heads <= 0 || pr->num_q_heads % pr->num_kv_heads) return -1;
  int G = pr->num_q_heads / pr->num_kv_heads;
  if (G & (G - 1)) return -1;
  if (!(pr->eps > 0.0f) || !(pr->delta > 0.0f && pr->delta < 1.0f)) return -1;
  if (pr->pilot_min < 2) return -1;
  if (pr->guarantee != ORC_GUARANTEE_DENOMINATOR && pr->guarantee != ORC_GUARANTEE_OUTPUT) return -1;
  if (pr->topp_den < 0 || pr->topp_num < 0 || (pr->topp_den > 0 && pr->topp_num > pr->topp_den)) return -1;
  if (pr->batch_offset < 0 || pr->head_offset < 0) return -1;
  if (pr->sinks < 0 || pr->window < 0 || pr->topk_abs < 0 || pr->topk_num < 0 || pr->topk_den < 0 ||
      pr->pilot_num < 0 || pr->pilot_den < 0)
    return -1;
  orc_inputs in = {q, k_cache, v_cache, k_t_cache, k_proj_cache, proj_basis, page_table, seq_lens};
  orc_outputs ot = {out, sel_idx, sel_count, budgets, head_need, den_hat, ref_max};
  double z = orc_z((double)pr->delta);
  int total = pr->batch * pr->num_kv_heads;
  int n = units ? n_units : total;
  for (int i = 0; i < n; i++) {
    int u = units ? units[i] : i;
    if (u < 0 || u >= total) return -2;
    decode_unit(pr, &in, &ot, u / pr->num_kv_heads, u % pr->num_kv_heads, z);
  }
  return 0;
}
