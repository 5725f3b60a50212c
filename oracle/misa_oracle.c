/*
 * MISA indexer oracle -- a plain, slow, obviously correct CPU implementation.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the CPU-baseline leg
 * of the benchmark may load this library.  The CUDA library never calls it and shares no code,
 * header, table or helper with it.
 *
 * Sources (all on "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference",
 * gist.science/paper/2605.07363, "Technical Summary"):
 *   - "Methodology: MISA", first stage ("Lightweight Block-Pooled Router"): the prefix is cut into
 *     M = ceil(L/B) blocks, each block is represented by the mean of its index keys, per-head
 *     affinities against those pooled keys are aggregated into one importance per head, and the
 *     top-h heads are kept.
 *   - "Methodology: MISA", second stage ("Sparse Token Scoring"): only the h routed heads score
 *     every prefix token and the top-k tokens by that reduced score are selected.
 *   - "Hierarchical Variant (MISA-dagger)": the routed pass keeps k' candidates, then the
 *     dense indexer with all H_I heads re-scores only those and keeps the top-k.
 *   - "Problem Statement": the dense DSA indexer scores every prefix token with all H_I heads.
 *   - "HISA: Efficient Hierarchical Indexing for Fine-Grained Sparse Attention" (arXiv 2603.28458),
 *     abstract: the token-axis block filter composed with MISA (orc_block_*).
 *   - paged key caches (orc_paged_gather, at the end of the file): a storage layout for serving,
 *     under which the definitions above apply to each sequence's logical cache.
 * The pages never write the score formulas; this oracle fixes them as
 *     token score  I_{t,s} = sum_{j in R_t} w_{t,j} * max(0, q_{t,j} . k_s)
 *     router score r_{t,j} = w_{t,j} * sum_{b < M_t} max(0, q_{t,j} . kbar_b)
 * with no scale factor, and the dense score F_{t,s} is I_{t,s} with R_t = all heads.
 *
 * Readings where the pages are silent (each one is also listed in the design notes):
 *   - query t sees the prefix s < n_t; its blocks are cut from that prefix, M_t = ceil(n_t/B),
 *     and a partial last block is the mean of its n_t - (M_t-1)B valid keys;
 *   - heads are summed in ascending head index, so h = H_I gives the dense score bit for bit;
 *   - every selection orders by value descending and breaks exact ties toward the lower index;
 *   - fewer valid items than requested: all of them are returned, remaining slots hold -1;
 *   - inputs arrive as float32 (bf16 values are exactly representable) and every sum, product
 *     and mean is taken in double.
 *
 * Parity status: every function here is pinned by the CPU tests (brute force on tiny inputs,
 * hand-computed fixtures, special cases that reduce to numpy routines, and invariants).
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
  double v;
  int32_t i;
} orc_item;

/* value descending, then index ascending */
static int orc_item_cmp(const void* pa, const void* pb) {
  const orc_item* a = (const orc_item*)pa;
  const orc_item* b = (const orc_item*)pb;
  if (a->v > b->v) return -1;
  if (a->v < b->v) return 1;
  if (a->i < b->i) return -1;
  if (a->i > b->i) return 1;
  return 0;
}

static double orc_relu(double x) { return x > 0.0 ? x : 0.0; }

static double orc_dot_ff(const float* a, const float* b, int d) {
  double s = 0.0;
  for (int i = 0; i < d; ++i) s += (double)a[i] * (double)b[i];
  return s;
}

static double orc_dot_fd(const float* a, const double* b, int d) {
  double s = 0.0;
  for (int i = 0; i < d; ++i) s += (double)a[i] * b[i];
  return s;
}

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/*
 * Select the kk best of n items: value v[i] descending, ties to the lower id.  ids == NULL
 * means id = position.  Items whose id is negative are skipped.  out[kk] receives the ids in
 * selection order, then -1 padding; out_v (optional) the matching values (0 for padding).
 * Returns the number of ids written (min(kk, number of valid items)).
 */
int64_t orc_topk(const double* v, const int32_t* ids, int64_t n, int64_t kk, int32_t* out,
                 double* out_v) {
  orc_item* it = (orc_item*)malloc(sizeof(orc_item) * (size_t)(n > 0 ? n : 1));
  int64_t m = 0;
  for (int64_t i = 0; i < n; ++i) {
    int32_t id = ids ? ids[i] : (int32_t)i;
    if (id < 0) continue;
    it[m].v = v[i];
    it[m].i = id;
    ++m;
  }
  qsort(it, (size_t)m, sizeof(orc_item), orc_item_cmp);
  int64_t take = m < kk ? m : kk;
  for (int64_t a = 0; a < kk; ++a) {
    out[a] = a < take ? it[a].i : -1;
    if (out_v) out_v[a] = a < take ? it[a].v : 0.0;
  }
  free(it);
  return take;
}

/* Mean of key rows [s0, s1) of a [*, d] cache (the block-pooled index key). */
void orc_block_mean(const float* k, int d, int64_t s0, int64_t s1, double* mean) {
  for (int i = 0; i < d; ++i) mean[i] = 0.0;
  for (int64_t s = s0; s < s1; ++s)
    for (int i = 0; i < d; ++i) mean[i] += (double)k[s * d + i];
  const double c = (double)(s1 - s0);
  for (int i = 0; i < d; ++i) mean[i] /= c;
}

/* Pool the first n keys into ceil(n/B) block means kbar[ceil(n/B), d]. */
void orc_pool_keys(const float* k, int64_t n, int d, int B, double* kbar) {
  const int64_t M = (n + B - 1) / B;
  for (int64_t b = 0; b < M; ++b) {
    int64_t s1 = (b + 1) * B < n ? (b + 1) * B : n;
    orc_block_mean(k, d, b * B, s1, kbar + b * d);
  }
}

/*
 * Router for one query: q[H_I,d], w[H_I], keys k[>= n, d].  Writes r[H_I] and the h routed
 * heads in descending r (ties to the lower head index).
 */
void orc_route(const float* q, const float* w, const float* k, int64_t n, int H_I, int d,
               int B, int h, double* r, int32_t* heads) {
  const int64_t M = (n + B - 1) / B;
  double* kbar = (double*)malloc(sizeof(double) * (size_t)(M > 0 ? M : 1) * (size_t)d);
  orc_pool_keys(k, n, d, B, kbar);
  for (int j = 0; j < H_I; ++j) {
    double acc = 0.0;
    for (int64_t b = 0; b < M; ++b) acc += orc_relu(orc_dot_fd(q + (int64_t)j * d, kbar + b * d, d));
    r[j] = (double)w[j] * acc;
  }
  orc_topk(r, NULL, H_I, h, heads, NULL);
  free(kbar);
}

static int orc_int_cmp(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

/*
 * Token scores of one query with the nh heads in heads[] (any order; summed in ascending head
 * index): I[s] = sum_j w[j] * max(0, q_j . k_s) for s in [0, n).
 */
void orc_token_scores(const float* q, const float* w, const int32_t* heads, int nh,
                      const float* k, int64_t n, int d, double* I) {
  int32_t* hs = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nh > 0 ? nh : 1));
  memcpy(hs, heads, sizeof(int32_t) * (size_t)nh);
  qsort(hs, (size_t)nh, sizeof(int32_t), orc_int_cmp);
  for (int64_t s = 0; s < n; ++s) {
    double acc = 0.0;
    for (int a = 0; a < nh; ++a) {
      const int j = hs[a];
      acc += (double)w[j] * orc_relu(orc_dot_ff(q + (int64_t)j * d, k + s * d, d));
    }
    I[s] = acc;
  }
  free(hs);
}

/* Dense (all-head) score of the tokens listed in ids[m] (ids < 0 or >= n give 0). */
static void orc_dense_at(const float* q, const float* w, int H_I, const float* k, int64_t n,
                         int d, const int32_t* ids, int64_t m, double* F) {
  for (int64_t a = 0; a < m; ++a) {
    const int32_t s = ids[a];
    double acc = 0.0;
    if (s >= 0 && s < n)
      for (int j = 0; j < H_I; ++j)
        acc += (double)w[j] * orc_relu(orc_dot_ff(q + (int64_t)j * d, k + (int64_t)s * d, d));
    F[a] = acc;
  }
}

/*
 * MISA-dagger fine stage for one query: re-score the candidates cand[kp] (entries < 0 or >= n
 * are empty) with all H_I heads and keep the top kk by that dense score.
 */
void orc_rerank(const float* q, const float* w, int H_I, const float* k, int64_t n, int d,
                const int32_t* cand, int64_t kp, int64_t kk, int32_t* out, double* out_v) {
  double* F = (double*)malloc(sizeof(double) * (size_t)(kp > 0 ? kp : 1));
  int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)(kp > 0 ? kp : 1));
  for (int64_t a = 0; a < kp; ++a) ids[a] = (cand[a] >= 0 && cand[a] < n) ? cand[a] : -1;
  orc_dense_at(q, w, H_I, k, n, d, ids, kp, F);
  orc_topk(F, ids, kp, kk, out, out_v);
  free(F);
  free(ids);
}

/*
 * Batched driver over T queries.  q[T,H_I,d], w[T,H_I], n[T]; query t reads the key cache at
 * k + t * k_seq_stride (elements; 0 = one shared cache).  mode:
 *   0 = MISA     : route (h heads), score with the routed heads, top kk
 *   1 = MISA-dag : route, score, top kp candidates, dense re-rank of the candidates, top kk
 *   2 = DSA      : dense score with all heads, top kk
 * Outputs (NULL to skip): r[T,H_I], heads[T,h], cand[T,kp], idx[T,kk], idx_v[T,kk].
 * With heads_in != NULL the router is skipped and heads_in[T,h] are used as the routed heads.
 */
void orc_indexer_batch(int mode, const float* q, const float* w, const float* k,
                       int64_t k_seq_stride, const int32_t* n, int T, int H_I, int d, int B,
                       int h, int64_t kk, int64_t kp, const int32_t* heads_in, double* r_out,
                       int32_t* heads_out, int32_t* cand_out, int32_t* idx, double* idx_v) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < T; ++t) {
    const float* qt = q + (int64_t)t * H_I * d;
    const float* wt = w + (int64_t)t * H_I;
    const float* kt = k + (int64_t)t * k_seq_stride;
    const int64_t nt = n[t] > 0 ? n[t] : 0;
    double* I = (double*)malloc(sizeof(double) * (size_t)(nt > 0 ? nt : 1));
    double* r = (double*)malloc(sizeof(double) * (size_t)H_I);
    int32_t* hd = (int32_t*)malloc(sizeof(int32_t) * (size_t)H_I);
    int32_t* ov = idx + (int64_t)t * kk;
    double* ovv = idx_v ? idx_v + (int64_t)t * kk : NULL;
    if (mode == 2) {
      for (int j = 0; j < H_I; ++j) hd[j] = j;
      orc_token_scores(qt, wt, hd, H_I, kt, nt, d, I);
      orc_topk(I, NULL, nt, kk, ov, ovv);
    } else {
      if (heads_in) {
        memcpy(hd, heads_in + (int64_t)t * h, sizeof(int32_t) * (size_t)h);
        for (int j = 0; j < H_I; ++j) r[j] = 0.0;
      } else {
        orc_route(qt, wt, kt, nt, H_I, d, B, h, r, hd);
      }
      if (r_out) memcpy(r_out + (int64_t)t * H_I, r, sizeof(double) * (size_t)H_I);
      if (heads_out) memcpy(heads_out + (int64_t)t * h, hd, sizeof(int32_t) * (size_t)h);
      orc_token_scores(qt, wt, hd, h, kt, nt, d, I);
      if (mode == 0) {
        orc_topk(I, NULL, nt, kk, ov, ovv);
      } else {
        int32_t* c = (int32_t*)malloc(sizeof(int32_t) * (size_t)(kp > 0 ? kp : 1));
        orc_topk(I, NULL, nt, kp, c, NULL);
        if (cand_out) memcpy(cand_out + (int64_t)t * kp, c, sizeof(int32_t) * (size_t)kp);
        orc_rerank(qt, wt, H_I, kt, nt, d, c, kp, kk, ov, ovv);
        free(c);
      }
    }
    free(I);
    free(r);
    free(hd);
  }
}

/*
 * Element-wise scores for parity checks: for each query t, I[t, s] for s < n_t with the heads
 * heads[t, nh] (heads == NULL: all H_I heads); entries s >= n_t are left untouched.
 * I is [T, ld] doubles.
 */
void orc_scores_batch(const float* q, const float* w, const float* k, int64_t k_seq_stride,
                      const int32_t* n, int T, int H_I, int d, const int32_t* heads, int nh,
                      double* I, int64_t ld) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < T; ++t) {
    int32_t* hd = (int32_t*)malloc(sizeof(int32_t) * (size_t)H_I);
    int m = heads ? nh : H_I;
    for (int a = 0; a < m; ++a) hd[a] = heads ? heads[(int64_t)t * nh + a] : a;
    const int64_t nt = n[t] > 0 ? n[t] : 0;
    orc_token_scores(q + (int64_t)t * H_I * d, w + (int64_t)t * H_I, hd, m,
                     k + (int64_t)t * k_seq_stride, nt, d, I + (int64_t)t * ld);
    free(hd);
  }
}

/* Dense scores of listed tokens for every query: ids[T, m] -> F[T, m]. */
void orc_dense_scores_at(const float* q, const float* w, const float* k, int64_t k_seq_stride,
                         const int32_t* n, int T, int H_I, int d, const int32_t* ids, int64_t m,
                         double* F) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < T; ++t) {
    const int64_t nt = n[t] > 0 ? n[t] : 0;
    orc_dense_at(q + (int64_t)t * H_I * d, w + (int64_t)t * H_I, H_I,
                 k + (int64_t)t * k_seq_stride, nt, d, ids + (int64_t)t * m, m, F + (int64_t)t * m);
  }
}

/* Router scores and heads for every query (r[T,H_I], heads[T,h]). */
void orc_route_batch(const float* q, const float* w, const float* k, int64_t k_seq_stride,
                     const int32_t* n, int T, int H_I, int d, int B, int h, double* r,
                     int32_t* heads) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < T; ++t) {
    const int64_t nt = n[t] > 0 ? n[t] : 0;
    orc_route(q + (int64_t)t * H_I * d, w + (int64_t)t * H_I, k + (int64_t)t * k_seq_stride, nt,
              H_I, d, B, h, r + (int64_t)t * H_I, heads + (int64_t)t * h);
  }
}

/* Pool n_seq caches: k[n_seq] at stride k_seq_stride, each of length L, into kbar[n_seq, M, d]. */
void orc_pool_batch(const float* k, int64_t k_seq_stride, int n_seq, int64_t L, int d, int B,
                    double* kbar) {
  const int64_t M = (L + B - 1) / B;
#pragma omp parallel for schedule(dynamic, 1)
  for (int s = 0; s < n_seq; ++s)
    orc_pool_keys(k + (int64_t)s * k_seq_stride, L, d, B, kbar + (int64_t)s * M * d);
}

/*
 * Token-axis block filter composed with MISA ("HISA: Efficient Hierarchical Indexing for
 * Fine-Grained Sparse Attention", abstract: a block-level coarse filter scores pooled block
 * representatives and discards regions, then the original indexer runs only inside the kept
 * candidate blocks, and the selected tokens keep the indexer's top-k form; "MISA: Mixture of
 * Indexer Sparse Attention ...", "Problem Statement" and "Significance and Claims": HISA saves on
 * the token axis, MISA on the head axis, and the two are complementary).
 * Readings where the pages are silent:
 *   - the pooled block representative is the same block mean the router uses (partial last
 *     block averaged over its valid keys), and a block is scored with the indexer's own formula
 *     and the query's routed heads: S[b] = sum_{j in R, ascending} w[j] * max(0, q_j . kbar_b);
 *     with h = H_I this is the dense indexer's block filter;
 *   - the m best blocks are kept (value descending, ties to the lower block);
 *   - the kept blocks' tokens of the prefix are scored with the routed heads, exactly as MISA
 *     scores them, and the top kk of those are selected (ties to the lower token).
 */
void orc_block_scores(const float* q, const float* w, const int32_t* heads, int nh,
                      const float* k, int64_t n, int d, int B, double* S) {
  const int64_t M = (n + B - 1) / B;
  double* kbar = (double*)malloc(sizeof(double) * (size_t)(M > 0 ? M : 1) * (size_t)d);
  int32_t* hs = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nh > 0 ? nh : 1));
  orc_pool_keys(k, n, d, B, kbar);
  memcpy(hs, heads, sizeof(int32_t) * (size_t)nh);
  qsort(hs, (size_t)nh, sizeof(int32_t), orc_int_cmp);
  for (int64_t b = 0; b < M; ++b) {
    double acc = 0.0;
    for (int a = 0; a < nh; ++a) {
      const int j = hs[a];
      acc += (double)w[j] * orc_relu(orc_dot_fd(q + (int64_t)j * d, kbar + b * d, d));
    }
    S[b] = acc;
  }
  free(kbar);
  free(hs);
}

/*
 * Block filter + refinement for one query with the heads heads[nh]: S[ceil(n/B)] block scores,
 * blocks[m] the kept blocks by descending S (-1 padded), out[kk] / out_v[kk] the selected tokens.
 */
void orc_block_filter(const float* q, const float* w, const int32_t* heads, int nh, const float* k,
                      int64_t n, int d, int B, int64_t m, int64_t kk, double* S, int32_t* blocks,
                      int32_t* out, double* out_v) {
  const int64_t M = (n + B - 1) / B;
  orc_block_scores(q, w, heads, nh, k, n, d, B, S);
  orc_topk(S, NULL, M, m, blocks, NULL);
  int64_t cnt = 0;
  for (int64_t a = 0; a < m; ++a) {
    if (blocks[a] < 0) continue;
    const int64_t s0 = (int64_t)blocks[a] * B;
    cnt += ((s0 + B < n) ? s0 + B : n) - s0;
  }
  double* I = (double*)malloc(sizeof(double) * (size_t)(cnt > 0 ? cnt : 1));
  int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)(cnt > 0 ? cnt : 1));
  int64_t c = 0;
  for (int64_t a = 0; a < m; ++a) {
    if (blocks[a] < 0) continue;
    const int64_t s0 = (int64_t)blocks[a] * B;
    const int64_t s1 = (s0 + B < n) ? s0 + B : n;
    orc_token_scores(q, w, heads, nh, k + s0 * d, s1 - s0, d, I + c);
    for (int64_t s = s0; s < s1; ++s) ids[c++] = (int32_t)s;
  }
  orc_topk(I, ids, cnt, kk, out, out_v);
  free(I);
  free(ids);
}

/*
 * Batched MISA + block filter over T queries (layouts as in orc_indexer_batch): route h heads
 * (or take heads_in[T,h]), then orc_block_filter keeping m blocks and kk tokens.  Outputs (NULL
 * to skip): r[T,H_I], heads[T,h], S[T,ldS] (entries past ceil(n_t/B) untouched), blocks[T,m],
 * idx[T,kk], idx_v[T,kk].
 */
void orc_block_filter_batch(const float* q, const float* w, const float* k, int64_t k_seq_stride,
                            const int32_t* n, int T, int H_I, int d, int B, int h, int64_t m,
                            int64_t kk, const int32_t* heads_in, double* r_out, int32_t* heads_out,
                            double* S_out, int64_t ldS, int32_t* blocks_out, int32_t* idx,
                            double* idx_v) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < T; ++t) {
    const float* qt = q + (int64_t)t * H_I * d;
    const float* wt = w + (int64_t)t * H_I;
    const float* kt = k + (int64_t)t * k_seq_stride;
    const int64_t nt = n[t] > 0 ? n[t] : 0;
    const int64_t Mt = (nt + B - 1) / B;
    double* r = (double*)malloc(sizeof(double) * (size_t)H_I);
    int32_t* hd = (int32_t*)malloc(sizeof(int32_t) * (size_t)H_I);
    double* S = (double*)malloc(sizeof(double) * (size_t)(Mt > 0 ? Mt : 1));
    int32_t* bl = (int32_t*)malloc(sizeof(int32_t) * (size_t)(m > 0 ? m : 1));
    if (heads_in) {
      memcpy(hd, heads_in + (int64_t)t * h, sizeof(int32_t) * (size_t)h);
      for (int j = 0; j < H_I; ++j) r[j] = 0.0;
    } else {
      orc_route(qt, wt, kt, nt, H_I, d, B, h, r, hd);
    }
    orc_block_filter(qt, wt, hd, h, kt, nt, d, B, m, kk, S, bl, idx + (int64_t)t * kk,
                     idx_v ? idx_v + (int64_t)t * kk : NULL);
    if (r_out) memcpy(r_out + (int64_t)t * H_I, r, sizeof(double) * (size_t)H_I);
    if (heads_out) memcpy(heads_out + (int64_t)t * h, hd, sizeof(int32_t) * (size_t)h);
    if (S_out) memcpy(S_out + (int64_t)t * ldS, S, sizeof(double) * (size_t)Mt);
    if (blocks_out) memcpy(blocks_out + (int64_t)t * m, bl, sizeof(int32_t) * (size_t)m);
    free(r);
    free(hd);
    free(S);
    free(bl);
  }
}

/*
 * Paged key caches (a serving layout; the pages call MISA a drop-in replacement for the DSA
 * indexer, "Key Contributions"): the keys of sequence t live in fixed-size pages of one shared
 * pool[num_pages, page_size, d], and its logical key s is row s % page_size of physical page
 * page_table[t][s / page_size].  The indexer's definitions apply unchanged to the logical cache.
 * This gathers the logical cache of every sequence: out[T, L, d] receives keys s < min(n_t, L)
 * and zeros past them; table entries of pages past the prefix are never read.  Returns the number
 * of page ids that were out of range (their keys are left zero).
 */
int64_t orc_paged_gather(const float* pool, int64_t num_pages, int page_size, int d,
                         const int32_t* page_table, int64_t max_pages, const int32_t* n, int T,
                         int64_t L, float* out) {
  int64_t bad = 0;
  for (int t = 0; t < T; ++t) {
    float* ot = out + (int64_t)t * L * d;
    memset(ot, 0, sizeof(float) * (size_t)L * (size_t)d);
    const int64_t nt = n[t] < 0 ? 0 : (n[t] > L ? L : n[t]);
    for (int64_t s = 0; s < nt; ++s) {
      const int64_t lp = s / page_size;
      const int32_t pg = lp < max_pages ? page_table[(int64_t)t * max_pages + lp] : -1;
      if (pg < 0 || pg >= num_pages) {
        ++bad;
        continue;
      }
      memcpy(ot + s * d, pool + ((int64_t)pg * page_size + s % page_size) * d, sizeof(float) * (size_t)d);
    }
  }
  return bad;
}
