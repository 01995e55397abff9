/*
 * vx_oracle.c -- plain, slow, fp64 CPU oracle for block top-k sparse decode over a
 * paged KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this
 * file: only the test suite, the package's smoke check and the benchmark's CPU-baseline
 * leg use it.  It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (source: "Vortex: Efficient and Programmable Sparse Attention
 * Serving for AI Agents", paper note, section 系统设计 1 "vFlow", the block top-k
 * attention example): a cache stage keeps one key centroid per KV block (page); an
 * indexer multiplies the query with the centroids, keeps the top-k blocks by score, and
 * exact softmax attention runs on the chosen blocks only.  The page-table layout
 * (batch size, pointer array, page index structure) follows section 系统设计 2
 * "vTensor".  The approximate top-k follows section 系统设计 3 (radix top-k with
 * stochastic early termination and remapping); the pages give no algorithm for it, so
 * the reading implemented here is stated at orc_topk_approx.
 *
 * Every floating-point quantity is computed in double precision from inputs widened
 * exactly from bf16.  Two steps are fixed in a lower precision on purpose, because the
 * method stores or decides in that precision: the stored centroid is rounded once to
 * bf16 (the cache's own element type), and the approximate top-k's 12-bit remap code is
 * decided in fp32 (the precision of the scores it quantises).
 *
 * Layouts (all row-major, bf16 passed as raw uint16 bit patterns):
 *   k_cache   [num_pool_pages][Hkv][P][Dqk]
 *   v_cache   [num_pool_pages][Hkv][P][Dv]   (unused when mla_shared_kv: V = K[..., :Dv])
 *   q         [B][Hq][Dqk]
 *   centroids [num_pool_pages][Hkv][Dqk]     (keyed by physical page)
 *   page table: page_ptr[B] = start of request b's row in page_indices; the row holds
 *               ceil(seq_lens[b] / P) physical page ids, logical page j first.
 *   scores    [B][Hkv][max_pages]; sel [B][Hkv][k] logical page ids, -1 past k_eff.
 *
 * Parity pins: every function here is checked against closed forms, brute force and
 * library routines in tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ bf16 <-> double */

/* A bf16 value is the upper half of an IEEE binary32; widening is exact. */
static double widen(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 (ties to even), directly from the double so that
 * no intermediate float rounding happens.  bf16 keeps 8 significant bits; its smallest
 * normal exponent is -126 and its subnormal spacing is 2^-133. */
static uint16_t narrow(double x) {
    if (isnan(x)) return 0x7fc0;
    if (x == 0.0) return signbit(x) ? 0x8000 : 0x0000;
    double ax = fabs(x);
    double r;
    int e;
    frexp(ax, &e);                 /* ax = f * 2^e, f in [0.5, 1) */
    if (e - 1 < -126) {            /* below the normal range: fixed spacing 2^-133 */
        r = ldexp(nearbyint(ldexp(ax, 133)), -133);
    } else {                       /* 8 significant bits: spacing 2^(e-8) */
        r = ldexp(nearbyint(ldexp(ax, 8 - e)), e - 8);
    }
    if (r >= ldexp(1.0, 128)) {    /* rounds past the largest finite bf16 */
        return signbit(x) ? 0xff80 : 0x7f80;
    }
    float f = (float)r;            /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint16_t h = (uint16_t)(u >> 16);
    return signbit(x) ? (uint16_t)(h | 0x8000) : h;
}

void orc_widen_bf16(const uint16_t *src, int64_t n, double *dst) {
    for (int64_t i = 0; i < n; ++i) dst[i] = widen(src[i]);
}

void orc_narrow_bf16(const double *src, int64_t n, uint16_t *dst) {
    for (int64_t i = 0; i < n; ++i) dst[i] = narrow(src[i]);
}

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads for the following calls on the calling host thread (n < 1: as many as the host has
 * processors); returns the previous count.  Used to time the baseline on one core. */
int orc_set_num_threads(int n) {
#ifdef _OPENMP
    int prev = omp_get_max_threads();
    omp_set_num_threads(n > 0 ? n : omp_get_num_procs());
    return prev;
#else
    (void)n;
    return 1;
#endif
}

/* --------------------------------------------------------------- page-table helpers */

static int32_t pages_of(int32_t seq_len, int32_t P) { return (seq_len + P - 1) / P; }

/* valid tokens in logical page j of a request holding seq_len tokens */
static int32_t valid_in_page(int32_t seq_len, int32_t P, int32_t j) {
    int32_t left = seq_len - j * P;
    return left < P ? left : P;
}

/* ----------------------------------------------------------- step 1: centroid cache */

/*
 * Cache stage: the key centroid of a page is the mean of the keys of its valid tokens,
 * per KV head (paper note, section 系统设计 1: the cache stage of block top-k keeps one
 * key centroid per block).  A partial last page averages only its valid tokens; slots past the
 * request's length never enter the sum.  cen_f64 (nullable) receives the exact mean,
 * cen_bf16 (nullable) the stored value: the mean rounded once to bf16.  Only pages that
 * some request references are written.
 */
int orc_centroids(const uint16_t *k_cache, int32_t Hkv, int32_t P, int32_t Dqk,
                  int32_t B, const int32_t *page_ptr, const int32_t *page_indices,
                  const int32_t *seq_lens, double *cen_f64, uint16_t *cen_bf16) {
    for (int32_t b = 0; b < B; ++b) {
        int32_t n = pages_of(seq_lens[b], P);
#pragma omp parallel for schedule(static)
        for (int32_t j = 0; j < n; ++j) {
            int64_t phys = page_indices[page_ptr[b] + j];
            int32_t m = valid_in_page(seq_lens[b], P, j);
            for (int32_t h = 0; h < Hkv; ++h) {
                for (int32_t d = 0; d < Dqk; ++d) {
                    double sum = 0.0;
                    for (int32_t t = 0; t < m; ++t)
                        sum += widen(k_cache[((phys * Hkv + h) * P + t) * Dqk + d]);
                    double mean = sum / (double)m;
                    int64_t o = (phys * Hkv + h) * Dqk + d;
                    if (cen_f64) cen_f64[o] = mean;
                    if (cen_bf16) cen_bf16[o] = narrow(mean);
                }
            }
        }
    }
    return 0;
}

/*
 * Append one decode token per request (continuous batching): seq_lens already counts
 * the new token, whose slot is position seq_lens[b]-1, i.e. slot (L-1) mod P of logical
 * page (L-1)/P.  The caller has installed that page in the page table.  The oracle only
 * writes the token; the page's centroid is then, by definition, the mean over its valid
 * keys and is obtained from orc_centroids.
 */
int orc_append(uint16_t *k_cache, uint16_t *v_cache, int32_t mla_shared_kv,
               int32_t Hkv, int32_t P, int32_t Dqk, int32_t Dv, int32_t B,
               const int32_t *page_ptr, const int32_t *page_indices, const int32_t *seq_lens,
               const uint16_t *k_new, const uint16_t *v_new) {
    for (int32_t b = 0; b < B; ++b) {
        int32_t pos = seq_lens[b] - 1;
        int64_t phys = page_indices[page_ptr[b] + pos / P];
        int32_t slot = pos % P;
        for (int32_t h = 0; h < Hkv; ++h) {
            for (int32_t d = 0; d < Dqk; ++d)
                k_cache[((phys * Hkv + h) * P + slot) * Dqk + d] = k_new[((int64_t)b * Hkv + h) * Dqk + d];
            if (!mla_shared_kv)
                for (int32_t d = 0; d < Dv; ++d)
                    v_cache[((phys * Hkv + h) * P + slot) * Dv + d] = v_new[((int64_t)b * Hkv + h) * Dv + d];
        }
    }
    return 0;
}

/*
 * Prefill write (cache stage, paper note section 系统设计 1: the cache is filled as tokens
 * arrive).  Positions [first_pos[b], seq_lens[b]) of request b arrive packed in request
 * order: k_new [N][Hkv][Dqk] and v_new [N][Hkv][Dv], request b's first row right after the
 * rows of the requests before it.  Each row goes to slot pos % P of page
 * page_indices[page_ptr[b] + pos / P].  A request whose length is not in [1, max_len] or
 * whose first_pos is outside [0, seq_lens[b]] contributes no rows.  The touched pages'
 * centroids are then plain page means (orc_centroids over the written cache).
 */
int orc_prefill_write(uint16_t *k_cache, uint16_t *v_cache, int32_t mla_shared_kv,
                      int32_t Hkv, int32_t P, int32_t Dqk, int32_t Dv, int32_t B, int32_t max_len,
                      const int32_t *page_ptr, const int32_t *page_indices, const int32_t *seq_lens,
                      const int32_t *first_pos, const uint16_t *k_new, const uint16_t *v_new) {
    int64_t row = 0; /* packed input row of the next new token */
    for (int32_t b = 0; b < B; ++b) {
        int32_t L = seq_lens[b], fp = first_pos[b];
        if (L < 1 || L > max_len || fp < 0 || fp > L) continue;
        for (int32_t pos = fp; pos < L; ++pos, ++row) {
            int64_t page = page_indices[page_ptr[b] + pos / P];
            int32_t in_page = pos % P;
            for (int32_t h = 0; h < Hkv; ++h) {
                for (int32_t d = 0; d < Dqk; ++d)
                    k_cache[((page * Hkv + h) * P + in_page) * Dqk + d] = k_new[(row * Hkv + h) * Dqk + d];
                if (!mla_shared_kv)
                    for (int32_t d = 0; d < Dv; ++d)
                        v_cache[((page * Hkv + h) * P + in_page) * Dv + d] = v_new[(row * Hkv + h) * Dv + d];
            }
        }
    }
    return 0;
}

/* ---------------------------------------------------------------- step 2: indexer */

/*
 * Page score: the query heads of a GQA group are each multiplied with the page's key
 * centroid and the products are summed over the group (paper note, section 系统设计 1: the
 * indexer scores blocks by a matrix product of query and centroids).  No softmax scale: it does not change the
 * ranking.  score_dims < Dqk scores on the first score_dims dimensions only (the
 * rope-unaware MLA variant of the MLA experiment section; the default is every
 * dimension, the rope-aware form).  The centroids [Npool][Hkv][Dqk] come either as
 * doubles (centroids) or as the stored bf16 values (centroids_bf16, used when centroids
 * is NULL).
 */
int orc_scores(const uint16_t *q, const double *centroids, const uint16_t *centroids_bf16,
               int32_t B, int32_t Hq, int32_t Hkv, int32_t Dqk, int32_t score_dims, int32_t P,
               const int32_t *page_ptr, const int32_t *page_indices, const int32_t *seq_lens,
               int32_t max_pages, double *scores) {
    int32_t G = Hq / Hkv;
    int32_t dims = score_dims > 0 ? score_dims : Dqk;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int32_t b = 0; b < B; ++b) {
        for (int32_t h = 0; h < Hkv; ++h) {
            int32_t n = pages_of(seq_lens[b], P);
            for (int32_t j = 0; j < n; ++j) {
                int64_t phys = page_indices[page_ptr[b] + j];
                int64_t c0 = (phys * Hkv + h) * Dqk;
                double s = 0.0;
                for (int32_t g = h * G; g < (h + 1) * G; ++g) {
                    const uint16_t *qg = q + ((int64_t)b * Hq + g) * Dqk;
                    double dot = 0.0;
                    for (int32_t d = 0; d < dims; ++d) {
                        double c = centroids ? centroids[c0 + d] : widen(centroids_bf16[c0 + d]);
                        dot += widen(qg[d]) * c;
                    }
                    s += dot;
                }
                scores[((int64_t)b * Hkv + h) * max_pages + j] = s;
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------ step 3: top-k pages */

typedef struct { double s; int32_t j; } scored_page;

/* Higher score first; equal scores: lower logical page index first.  +0 and -0
 * compare equal, so they tie and fall to the index rule. */
static int by_score_then_index(const void *a, const void *b) {
    const scored_page *x = (const scored_page *)a, *y = (const scored_page *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j > y->j) - (x->j < y->j);
}

static int by_index(const void *a, const void *b) {
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/*
 * Exact top-k (paper note, 系统设计 3, radix top-k; the definition of the result is the
 * k highest-scoring pages): the k_eff = min(k, n_b) pages with the largest score, ties
 * at the boundary going to the lower logical page index.  Obtained by a full sort on
 * (score descending, index ascending).  The chosen set is written in ascending page
 * order; slots past k_eff hold -1.
 */
int orc_topk_exact(const double *scores, int32_t B, int32_t Hkv, int32_t max_pages,
                   const int32_t *seq_lens, int32_t P, int32_t k, int32_t *sel) {
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int32_t b = 0; b < B; ++b) {
        for (int32_t h = 0; h < Hkv; ++h) {
            int32_t n = pages_of(seq_lens[b], P);
            int32_t keff = k < n ? k : n;
            const double *row = scores + ((int64_t)b * Hkv + h) * max_pages;
            scored_page *all = (scored_page *)malloc(sizeof(scored_page) * (size_t)(n > 0 ? n : 1));
            for (int32_t j = 0; j < n; ++j) { all[j].s = row[j]; all[j].j = j; }
            qsort(all, (size_t)n, sizeof(scored_page), by_score_then_index);
            int32_t *out = sel + ((int64_t)b * Hkv + h) * k;
            for (int32_t i = 0; i < k; ++i) out[i] = i < keff ? all[i].j : -1;
            qsort(out, (size_t)keff, sizeof(int32_t), by_index);
            free(all);
        }
    }
    return 0;
}

/*
 * SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
 * OOPSLA 2014; the 64-bit finaliser with the constants of Stafford's "Mix13").  The
 * i-th output (i = 0, 1, ...) of the generator seeded with `seed` is
 * mix(seed + (i + 1) * golden_gamma).
 */
uint64_t orc_splitmix64(uint64_t seed, uint64_t i) {
    uint64_t z = seed + (i + 1) * 0x9e3779b97f4a7c15ULL;
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
    return z ^ (z >> 31);
}

/*
 * Approximate top-k: stochastic early termination plus remapping (paper note, 系统设计 3;
 * the kernel-ablation section reports its recall@k > 0.97).  The pages name the two
 * ideas but give no algorithm; this is the reading implemented on both sides:
 *   1. remap: each score of the row becomes a bits-wide code
 *        code = min(2^bits - 1, floor((s - lo) * (2^bits / (hi - lo))))
 *      with lo, hi the row's minimum and maximum, every operation in fp32 round-to-
 *      nearest (the scores' own precision).  hi == lo, or a scale that is not finite,
 *      gives code 0 everywhere.
 *   2. one histogram of the codes; b* is the highest code such that at least k_eff
 *      scores have a code >= b*.
 *   3. every page with code > b* is selected.
 *   4. early termination: the remaining slots are filled from the pages whose code is
 *      exactly b*, without refining further, taken in cyclic page order starting at a
 *      pseudo-random offset o = SplitMix64(seed) draw number (b * Hkv + h), mod n_b.
 * The chosen set is written in ascending page order; slots past k_eff hold -1.
 */
int orc_topk_approx(const float *scores, int32_t B, int32_t Hkv, int32_t max_pages,
                    const int32_t *seq_lens, int32_t P, int32_t k, int32_t bits,
                    uint64_t seed, int32_t *sel) {
    int32_t nbins = 1 << bits;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int32_t b = 0; b < B; ++b) {
        for (int32_t h = 0; h < Hkv; ++h) {
            int32_t n = pages_of(seq_lens[b], P);
            int32_t keff = k < n ? k : n;
            const float *row = scores + ((int64_t)b * Hkv + h) * max_pages;
            int32_t *out = sel + ((int64_t)b * Hkv + h) * k;
            if (n <= 0) { for (int32_t i = 0; i < k; ++i) out[i] = -1; continue; }
            int32_t *code = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
            int64_t *count = (int64_t *)calloc((size_t)nbins, sizeof(int64_t));
            float lo = row[0], hi = row[0];
            for (int32_t j = 1; j < n; ++j) {
                if (row[j] < lo) lo = row[j];
                if (row[j] > hi) hi = row[j];
            }
            float range = hi - lo;              /* fp32, rounded */
            float scale = (float)nbins / range; /* fp32, rounded */
            int flat = !(hi > lo) || !isfinite(scale);
            for (int32_t j = 0; j < n; ++j) {
                int32_t c = 0;
                if (!flat) {
                    float diff = row[j] - lo;   /* fp32, rounded */
                    float t = diff * scale;     /* fp32, rounded; never fused */
                    double f = floor((double)t);
                    c = f >= (double)(nbins - 1) ? nbins - 1 : (int32_t)f;
                }
                code[j] = c;
                count[c] += 1;
            }
            /* b*: highest code whose top-down cumulative count reaches k_eff */
            int32_t bstar = 0;
            int64_t above = 0; /* scores with code > bstar */
            for (int32_t c = nbins - 1; c >= 0; --c) {
                if (above + count[c] >= keff) { bstar = c; break; }
                above += count[c];
            }
            int32_t need = keff - (int32_t)above; /* slots taken from bucket b* */
            int32_t filled = 0;
            for (int32_t j = 0; j < n; ++j)
                if (code[j] > bstar) out[filled++] = j;
            int32_t o = (int32_t)(orc_splitmix64(seed, (uint64_t)b * (uint64_t)Hkv + (uint64_t)h) % (uint64_t)n);
            for (int32_t i = 0; i < n && need > 0; ++i) {
                int32_t j = (o + i) % n;
                if (code[j] == bstar) { out[filled++] = j; --need; }
            }
            for (int32_t i = filled; i < k; ++i) out[i] = -1;
            qsort(out, (size_t)filled, sizeof(int32_t), by_index);
            free(code);
            free(count);
        }
    }
    return 0;
}

/* ------------------------------------------------------- step 4: sparse attention */

/*
 * Exact softmax attention over the selected pages (paper note, section 系统设计 1: softmax
 * attention, exact, restricted to the chosen blocks), gathered through the page table.  For query
 * head g of KV group h, the attended tokens are the valid tokens (position < seq_len)
 * of the pages listed in sel[b][h] (entries < 0 are skipped).  sel == NULL attends
 * every page of the request: dense decode attention.
 *   logit_t = sm_scale * q_g . K_t;   out_g = sum_t softmax(logit)_t V_t;
 *   lse_g = log(sum_t exp(logit_t))   (natural log).
 * With mla_shared_kv the value of a token is the first Dv dimensions of its key row.
 * A request whose attended set is empty gets out = 0 and lse = -inf.
 */
int orc_attend(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
               int32_t mla_shared_kv, int32_t B, int32_t Hq, int32_t Hkv, int32_t Dqk,
               int32_t Dv, int32_t P, const int32_t *page_ptr, const int32_t *page_indices,
               const int32_t *seq_lens, const int32_t *sel, int32_t k, double sm_scale,
               double *out, double *lse) {
    int32_t G = Hq / Hkv;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int32_t b = 0; b < B; ++b) {
        for (int32_t g = 0; g < Hq; ++g) {
            int32_t h = g / G;
            int32_t L = seq_lens[b];
            int32_t n = pages_of(L, P);
            int32_t npick = sel ? k : n;
            const uint16_t *qg = q + ((int64_t)b * Hq + g) * Dqk;
            /* collect (physical page, slot) of every attended token */
            int64_t cap = (int64_t)npick * P;
            double *logit = (double *)malloc(sizeof(double) * (size_t)(cap > 0 ? cap : 1));
            int64_t *row_k = (int64_t *)malloc(sizeof(int64_t) * (size_t)(cap > 0 ? cap : 1));
            int64_t *row_v = (int64_t *)malloc(sizeof(int64_t) * (size_t)(cap > 0 ? cap : 1));
            int64_t T = 0;
            for (int32_t i = 0; i < npick; ++i) {
                int32_t j = sel ? sel[((int64_t)b * Hkv + h) * k + i] : i;
                if (j < 0 || j >= n) continue;
                int64_t phys = page_indices[page_ptr[b] + j];
                int32_t m = valid_in_page(L, P, j);
                for (int32_t t = 0; t < m; ++t) {
                    row_k[T] = ((phys * Hkv + h) * P + t) * Dqk;
                    row_v[T] = mla_shared_kv ? row_k[T] : ((phys * Hkv + h) * P + t) * Dv;
                    double dot = 0.0;
                    for (int32_t d = 0; d < Dqk; ++d) dot += widen(qg[d]) * widen(k_cache[row_k[T] + d]);
                    logit[T] = sm_scale * dot;
                    ++T;
                }
            }
            double *o = out + ((int64_t)b * Hq + g) * Dv;
            for (int32_t d = 0; d < Dv; ++d) o[d] = 0.0;
            if (T == 0) {
                lse[(int64_t)b * Hq + g] = -INFINITY;
            } else {
                double mx = logit[0];
                for (int64_t t = 1; t < T; ++t) if (logit[t] > mx) mx = logit[t];
                double l = 0.0;
                for (int64_t t = 0; t < T; ++t) l += exp(logit[t] - mx);
                const uint16_t *vsrc = mla_shared_kv ? k_cache : v_cache;
                for (int64_t t = 0; t < T; ++t) {
                    double w = exp(logit[t] - mx) / l;
                    for (int32_t d = 0; d < Dv; ++d) o[d] += w * widen(vsrc[row_v[t] + d]);
                }
                lse[(int64_t)b * Hq + g] = mx + log(l);
            }
            free(logit);
            free(row_k);
            free(row_v);
        }
    }
    return 0;
}

/*
 * One whole decode step as the method runs it, for the CPU baseline: score every page
 * from the stored centroids, take the exact top-k, attend over the chosen pages.
 * centroids are the stored bf16 values.  Buffers: scores [B][Hkv][max_pages],
 * sel [B][Hkv][k], out [B][Hq][Dv], lse [B][Hq].
 */
int orc_decode_step(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                    const uint16_t *centroids_bf16, int32_t mla_shared_kv, int32_t B, int32_t Hq,
                    int32_t Hkv, int32_t Dqk, int32_t Dv, int32_t P, int64_t num_pool_pages,
                    const int32_t *page_ptr, const int32_t *page_indices, const int32_t *seq_lens,
                    int32_t max_pages, int32_t k, double sm_scale, double *scores, int32_t *sel,
                    double *out, double *lse) {
    (void)num_pool_pages;
    orc_scores(q, NULL, centroids_bf16, B, Hq, Hkv, Dqk, 0, P, page_ptr, page_indices, seq_lens,
               max_pages, scores);
    orc_topk_exact(scores, B, Hkv, max_pages, seq_lens, P, k, sel);
    orc_attend(q, k_cache, v_cache, mla_shared_kv, B, Hq, Hkv, Dqk, Dv, P, page_ptr, page_indices,
               seq_lens, sel, k, sm_scale, out, lse);
    return 0;
}
