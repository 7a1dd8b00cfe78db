/*
 * oracle.c -- plain, slow, fp64 CPU reference for the target model's
 * tree-verification step.  TEST INFRASTRUCTURE ONLY: the tests, the smoke
 * check and the benchmark's CPU-baseline leg call it; the library under test
 * never does.  It shares no code with the CUDA path.
 *
 * Sources (the web pages on tree-based speculative decoding):
 *  - "Tree-based speculative decoding" glossary (jisaku.com), section "Tree
 *    attention": M[i][j] = 1 iff node j is node i or one of its ancestors;
 *    every node attends to the prefix and to its own root-to-node path.
 *  - "Speculative decoding x tree attention" blog (radar-34b), section 3,
 *    figure "Tree Attention Verification Matrix" (5-node T0/A1/A2/B1/B2 mask).
 *  - same blog, section 2, table "Rejection Sampling Acceptance Condition"
 *    and its derivation: accept draft x when r < min(1, p(x)/q(x)), r ~ U(0,1);
 *    on rejection resample from max(0, p - q) / sum max(0, p - q).
 *  - glossary, section "SpecInfer": the tree is verified from the root,
 *    depth first; after a rejected child the next sibling is tried against the
 *    renormalised residual; if all children fail, sample the final residual.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - softmax scale 1/sqrt(D) is passed in by the caller; GQA maps query head h
 *    to KV head h / (Hq / Hkv).
 *  - node 0 is the root (the last committed token); it attends like any other
 *    node and is never tested by the sampler.
 *  - p[b][u] is the target distribution after node u's path, q[b][u] the draft
 *    distribution node u's children were drawn from; siblings are tried in
 *    ascending node index; q is not changed across siblings.
 *  - comparison is strict (r < alpha); q(x) = 0 accepts iff the current
 *    target mass at x is positive; a zero residual keeps the current
 *    distribution.
 *  - uniforms[b][c] (c >= 1) is node c's acceptance draw, uniforms[b][0] the
 *    single draw of the final (bonus) token; the draw is the first vocabulary
 *    index whose running sum exceeds u * total, else the last positive index.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_OK 0
#define OR_ERR_ARG 1
#define OR_ERR_TREE 3
#define OR_ERR_BLOCK 4

void or_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int or_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* A valid tree: node 0 is the root (parent -1), every other node's parent
 * comes before it. */
static int tree_ok(int32_t n, const int32_t *parent) {
    if (n < 1 || parent[0] != -1) return 0;
    for (int32_t i = 1; i < n; ++i)
        if (parent[i] < 0 || parent[i] >= i) return 0;
    return 1;
}

/* Dense tree mask from its definition: M[i][j] = 1 iff j == i or j lies on
 * the parent chain of i. */
int or_tree_mask(int32_t n, const int32_t *parent, uint8_t *mask) {
    if (!tree_ok(n, parent)) return OR_ERR_TREE;
    memset(mask, 0, (size_t)n * n);
    for (int32_t i = 0; i < n; ++i)
        for (int32_t j = i; j >= 0; j = parent[j]) mask[(size_t)i * n + j] = 1;
    return OR_OK;
}

static inline double load_elem(const void *base, int dtype, int64_t idx) {
    if (dtype == 1) return (double)((const float *)base)[idx];
    uint32_t bits = (uint32_t)((const uint16_t *)base)[idx] << 16; /* bfloat16 -> float, exact */
    float f;
    memcpy(&f, &bits, 4);
    return (double)f;
}

/*
 * Tree attention, one output row per (b, i, h):
 *   keys   = prefix positions t < L_b, then tree nodes j with M[i][j] = 1
 *            (node j's key/value sit at logical position L_b + j)
 *   s_t    = scale * <q[b][i][h], k[t][h / G]>
 *   out    = sum_t softmax(s)_t * v[t][h / G]
 * Logical position t of sequence b is slot t % bs of physical block
 * block_table[b][t / bs]; caches are [num_blocks][bs][Hkv][D].
 * rows: n_rows triples (b, i, h), or NULL for every row in (b, i, h) order.
 * out: n_rows x D doubles.  dtype: 0 = bfloat16 bits, 1 = float32.
 */
int or_tree_attention(int32_t B, int32_t N, int32_t Hq, int32_t Hkv, int32_t D, int32_t bs,
                      int32_t max_blocks, int32_t num_blocks, int32_t dtype, const void *q,
                      const void *k_cache, const void *v_cache, const int32_t *block_table,
                      const int32_t *prefix_lens, const int32_t *parent_idx, double scale,
                      int64_t n_rows, const int32_t *rows, double *out) {
    if (B < 1 || N < 1 || Hq < 1 || Hkv < 1 || D < 1 || bs < 1 || Hq % Hkv) return OR_ERR_ARG;
    const int32_t G = Hq / Hkv;
    if (!rows) n_rows = (int64_t)B * N * Hq;
    for (int32_t b = 0; b < B; ++b) {
        if (!tree_ok(N, parent_idx + (int64_t)b * N)) return OR_ERR_TREE;
        int64_t need = ((int64_t)prefix_lens[b] + N + bs - 1) / bs;
        if (prefix_lens[b] < 0 || need > max_blocks) return OR_ERR_ARG;
        for (int64_t j = 0; j < need; ++j) {
            int32_t blk = block_table[(int64_t)b * max_blocks + j];
            if (blk < 0 || blk >= num_blocks) return OR_ERR_BLOCK;
        }
    }
    int err = OR_OK;
#pragma omp parallel
    {
        uint8_t *mask = (uint8_t *)malloc((size_t)N * N);
        int64_t max_keys = 0;
        for (int32_t b = 0; b < B; ++b)
            if (prefix_lens[b] + N > max_keys) max_keys = prefix_lens[b] + N;
        int64_t *pos = (int64_t *)malloc(sizeof(int64_t) * max_keys);
        double *s = (double *)malloc(sizeof(double) * max_keys);
        double *acc = (double *)malloc(sizeof(double) * D);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < n_rows; ++r) {
            int32_t b, i, h;
            if (rows) { b = rows[3 * r]; i = rows[3 * r + 1]; h = rows[3 * r + 2]; }
            else { b = (int32_t)(r / ((int64_t)N * Hq)); i = (int32_t)((r / Hq) % N); h = (int32_t)(r % Hq); }
            double *o = out + r * D;
            if (b < 0 || b >= B || i < 0 || i >= N || h < 0 || h >= Hq) {
                for (int32_t d = 0; d < D; ++d) o[d] = NAN;
                err = OR_ERR_ARG;
                continue;
            }
            const int32_t kvh = h / G;
            const int64_t L = prefix_lens[b];
            or_tree_mask(N, parent_idx + (int64_t)b * N, mask);
            int64_t nk = 0;
            for (int64_t t = 0; t < L; ++t) pos[nk++] = t;
            for (int32_t j = 0; j < N; ++j)
                if (mask[(size_t)i * N + j]) pos[nk++] = L + j;
            const int64_t qoff = (((int64_t)b * N + i) * Hq + h) * D;
            double m = -INFINITY;
            for (int64_t t = 0; t < nk; ++t) {
                int64_t blk = block_table[(int64_t)b * max_blocks + pos[t] / bs];
                int64_t koff = ((blk * bs + pos[t] % bs) * Hkv + kvh) * D;
                double dot = 0.0;
                for (int32_t d = 0; d < D; ++d) dot += load_elem(q, dtype, qoff + d) * load_elem(k_cache, dtype, koff + d);
                s[t] = scale * dot;
                if (s[t] > m) m = s[t];
            }
            double z = 0.0;
            for (int32_t d = 0; d < D; ++d) acc[d] = 0.0;
            for (int64_t t = 0; t < nk; ++t) {
                double w = exp(s[t] - m);
                z += w;
                int64_t blk = block_table[(int64_t)b * max_blocks + pos[t] / bs];
                int64_t voff = ((blk * bs + pos[t] % bs) * Hkv + kvh) * D;
                for (int32_t d = 0; d < D; ++d) acc[d] += w * load_elem(v_cache, dtype, voff + d);
            }
            for (int32_t d = 0; d < D; ++d) o[d] = acc[d] / z;
        }
        free(mask); free(pos); free(s); free(acc);
    }
    return err;
}

/*
 * Lossless tree verification, literally: walk from the root; at node u try
 * its children in ascending index order, accepting child c (token x) when
 * uniforms[b][c] < P(x) / Q(x) with P the current target distribution
 * (initially p[b][u]) and Q = q[b][u].  A rejection replaces P by the
 * normalised residual max(0, P - Q) / sum(max(0, P - Q)).  On acceptance
 * descend into c with P = p[b][c].  When no child is accepted (or u is a
 * leaf) draw the bonus token from P with uniforms[b][0].
 *
 * Outputs per sequence: accepted_path[b][0..N) (accepted node indices,
 * root excluded, -1 padded), accepted_len[b], bonus_token[b].  Invalid
 * trees or tokens give accepted_len = -1, bonus = -1 and the return value
 * OR_ERR_TREE.
 * near[b] counts threshold events within eps: |r - alpha| < eps at a tested
 * child, or |u0 - C/total| < eps for either edge C of the drawn bucket.
 * rows[b] counts the vocabulary rows the walk had to read in full.
 */
int or_verify_sample(int32_t B, int32_t N, int64_t V, const float *p, const float *q,
                     const int32_t *tokens, const int32_t *parent_idx, const float *uniforms,
                     double eps, int32_t *accepted_path, int32_t *accepted_len, int32_t *bonus,
                     int32_t *near, int32_t *rows) {
    if (B < 1 || N < 1 || V < 1) return OR_ERR_ARG;
    int err = OR_OK;
#pragma omp parallel
    {
        double *P = (double *)malloc(sizeof(double) * V);
        double *R = (double *)malloc(sizeof(double) * V);
#pragma omp for schedule(dynamic, 1)
        for (int32_t b = 0; b < B; ++b) {
            const int32_t *par = parent_idx + (int64_t)b * N;
            const int32_t *tok = tokens + (int64_t)b * N;
            const float *ub = uniforms + (int64_t)b * N;
            int32_t *path = accepted_path + (int64_t)b * N;
            for (int32_t i = 0; i < N; ++i) path[i] = -1;
            near[b] = 0;
            rows[b] = 0;
            int valid = tree_ok(N, par);
            for (int32_t c = 1; valid && c < N; ++c)
                if (tok[c] < 0 || tok[c] >= V) valid = 0;
            if (!valid) {
                accepted_len[b] = -1;
                bonus[b] = -1;
                err = OR_ERR_TREE;
                continue;
            }
            int32_t u = 0, len = 0;
            const float *pu = p + ((int64_t)b * N) * V;
            for (int64_t x = 0; x < V; ++x) P[x] = (double)pu[x];
            for (;;) {
                const float *Q = q + ((int64_t)b * N + u) * V;
                int32_t accepted = -1;
                int row_read = 0;
                for (int32_t c = u + 1; c < N; ++c) {
                    if (par[c] != u) continue;
                    const int32_t x = tok[c];
                    const double r = (double)ub[c];
                    const double qx = (double)Q[x];
                    int accept;
                    if (qx > 0.0) {
                        const double alpha = P[x] / qx;
                        if (fabs(r - alpha) < eps) near[b]++;
                        accept = r < alpha;
                    } else {
                        accept = P[x] > 0.0;
                    }
                    if (accept) { accepted = c; break; }
                    double z = 0.0;
                    for (int64_t y = 0; y < V; ++y) {
                        R[y] = fmax(0.0, P[y] - (double)Q[y]);
                        z += R[y];
                    }
                    row_read = 1;
                    if (z > 0.0)
                        for (int64_t y = 0; y < V; ++y) P[y] = R[y] / z;
                }
                if (accepted >= 0) {
                    path[len++] = accepted;
                    u = accepted;
                    const float *pc = p + ((int64_t)b * N + u) * V;
                    for (int64_t x = 0; x < V; ++x) P[x] = (double)pc[x];
                    rows[b] += row_read;
                    continue;
                }
                /* final draw from P with uniforms[b][0] */
                double total = 0.0;
                for (int64_t x = 0; x < V; ++x) total += P[x];
                const double u0 = (double)ub[0];
                const double target = u0 * total;
                double run = 0.0, before = 0.0;
                int64_t k = -1, last_pos = -1;
                for (int64_t x = 0; x < V; ++x) {
                    if (P[x] > 0.0) last_pos = x;
                    before = run;
                    run += P[x];
                    if (run > target) { k = x; break; }
                }
                if (k < 0) { k = last_pos; before = total; run = total; }
                if (total > 0.0 && (fabs(u0 - before / total) < eps || fabs(u0 - run / total) < eps)) near[b]++;
                rows[b] += 1;
                accepted_len[b] = len;
                bonus[b] = (int32_t)k;
                break;
            }
        }
        free(P);
        free(R);
    }
    return err;
}

/*
 * or_commit_path -- the step after verification: the accepted path joins the
 * cached prefix and every other tree entry is released.
 *
 * Sources: blog "Speculative decoding x tree attention", section "KV cache
 * management and prefix sharing" (rejected tokens' KV must be freed or rolled
 * back at once; paged engines do it through block-table operations), and
 * glossary "Tree-based speculative decoding", section "KV cache management
 * challenges" (each tree node has a KV entry; after verification every entry
 * off the accepted path is pruned; page-based management avoids fragmentation).
 *
 * Readings (listed in the design notes): tree node j of sequence b sits at
 * logical position L_b + j; the root (node 0) stays at L_b; accepted node
 * path[k] (k = 0 .. len-1) moves to position L_b + 1 + k, for every KV head and
 * both K and V; the new prefix length is L_b + 1 + len.  Positions at or past
 * the new length are free (the caller's allocator may reclaim whole blocks past
 * it); nothing else in the cache changes.  A sequence with len < 0 (the walk
 * flagged its tree) keeps its length and cache.  A path that is not strictly
 * increasing inside [1, N), a length over N - 1, or a prefix / block id out of
 * range leaves the sequence untouched and returns an error code.
 *
 * Layout: cache [num_blocks][16][Hkv][D] elements of elem_size bytes; logical
 * position t of sequence b lives in block bt[b][t / 16], slot t % 16.
 * Rows are moved as bytes, so any element type works.
 */
int or_commit_path(int32_t B, int32_t N, int32_t Hkv, int32_t D, int32_t max_blocks, int32_t num_blocks,
                   int32_t elem_size, void *k_cache, void *v_cache, const int32_t *block_table,
                   const int32_t *prefix_lens, const int32_t *path, const int32_t *len, int32_t *new_prefix_lens) {
    const int64_t row = (int64_t)D * elem_size;  /* bytes of one (position, head) row */
    int err = OR_OK;
    for (int32_t b = 0; b < B; ++b) {
        const int32_t L = prefix_lens[b];
        const int32_t n = len[b];
        new_prefix_lens[b] = L;
        if (n < 0) continue;
        if (L < 0 || n > N - 1 || (int64_t)L + N > (int64_t)max_blocks * 16) { err = OR_ERR_ARG; continue; }
        const int32_t *pb = path + (int64_t)b * N;
        int ok = 1;
        for (int32_t k = 0; k < n; ++k) {
            const int32_t prev = k == 0 ? 0 : pb[k - 1];
            if (pb[k] <= prev || pb[k] >= N) ok = 0;
        }
        if (!ok) { err = OR_ERR_TREE; continue; }
        const int32_t *bt = block_table + (int64_t)b * max_blocks;
        for (int32_t t = L; t < L + N; ++t) {
            const int32_t id = bt[t / 16];
            if (id < 0 || id >= num_blocks) ok = 0;
        }
        if (!ok) { err = OR_ERR_BLOCK; continue; }
        /* read every source row first, then write: a destination may be another row's source */
        const int64_t per_pos = (int64_t)Hkv * row;
        unsigned char *tmp = (unsigned char *)malloc((size_t)(2 * (int64_t)n * per_pos + 1));
        for (int c = 0; c < 2; ++c) {
            unsigned char *cache = (unsigned char *)(c == 0 ? k_cache : v_cache);
            for (int32_t k = 0; k < n; ++k) {
                const int32_t t = L + pb[k];
                memcpy(tmp + ((int64_t)c * n + k) * per_pos,
                       cache + ((int64_t)bt[t / 16] * 16 + t % 16) * per_pos, (size_t)per_pos);
            }
        }
        for (int c = 0; c < 2; ++c) {
            unsigned char *cache = (unsigned char *)(c == 0 ? k_cache : v_cache);
            for (int32_t k = 0; k < n; ++k) {
                const int32_t t = L + 1 + k;
                memcpy(cache + ((int64_t)bt[t / 16] * 16 + t % 16) * per_pos,
                       tmp + ((int64_t)c * n + k) * per_pos, (size_t)per_pos);
            }
        }
        free(tmp);
        new_prefix_lens[b] = L + 1 + n;
    }
    return err;
}
