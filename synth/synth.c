/*
 * synth.c -- seeded synthetic inputs for the tree-verification step.
 *
 * This module generates inputs only.  It holds none of the arithmetic of the
 * method under test (no tree mask, no attention, no acceptance walk); both the
 * CUDA library's tests/benchmarks and the CPU oracle read what it produces.
 *
 * Random numbers come from Philox4x32-10, written from its published
 * definition (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as
 * 1, 2, 3", SC'11, section 3.2): a 10-round Feistel-like bijection of a 128-bit
 * counter under a 64-bit key, with multipliers 0xD2511F53 / 0xCD9E8D57 and the
 * key schedule constants 0x9E3779B9 / 0xBB67AE85 (golden-ratio and sqrt(3)-1
 * Weyl increments).
 *
 * Stream convention (stated once, used everywhere):
 *   key     = { low 32 bits of seed, stream id }
 *   counter = { low 32 bits of g, high 32 bits of g, 0, 0 }
 * where g is the index of a group of 4 outputs; element e of a stream is
 * output word e % 4 of group g = e / 4.  Every value is therefore a pure
 * function of (seed, stream, element index), independent of threading.
 *
 *   uniform(e)  = (word >> 8) * 2^-24                 in [0, 1)
 *   normal(e)   : Box-Muller on the group's 4 words:
 *                 u1 = ((w0 >> 8) + 1) * 2^-24 in (0,1], u2 = (w1 >> 8) * 2^-24
 *                 n0 = r cos(2 pi u2), n1 = r sin(2 pi u2), r = sqrt(-2 ln u1)
 *                 and likewise (w2, w3) -> n2, n3.  Computed in double.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>

#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

void sy_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int r = 0; r < 10; ++r) {
        if (r > 0) { k0 += PHILOX_W0; k1 += PHILOX_W1; }
        uint64_t p0 = (uint64_t)PHILOX_M0 * c0;
        uint64_t p1 = (uint64_t)PHILOX_M1 * c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

static inline void group_words(uint64_t seed, uint32_t stream, uint64_t g, uint32_t w[4]) {
    uint32_t ctr[4] = {(uint32_t)g, (uint32_t)(g >> 32), 0u, 0u};
    uint32_t key[2] = {(uint32_t)seed, stream};
    sy_philox4x32_10(ctr, key, w);
}

static inline void group_normals(uint64_t seed, uint32_t stream, uint64_t g, double n[4]) {
    uint32_t w[4];
    group_words(seed, stream, g, w);
    const double two_pi = 6.283185307179586476925286766559;
    for (int pair = 0; pair < 2; ++pair) {
        double u1 = ((double)(w[2 * pair] >> 8) + 1.0) * (1.0 / 16777216.0);
        double u2 = (double)(w[2 * pair + 1] >> 8) * (1.0 / 16777216.0);
        double r = sqrt(-2.0 * log(u1));
        n[2 * pair] = r * cos(two_pi * u2);
        n[2 * pair + 1] = r * sin(two_pi * u2);
    }
}

static inline double normal_at(uint64_t seed, uint32_t stream, uint64_t e) {
    double n[4];
    group_normals(seed, stream, e >> 2, n);
    return n[e & 3];
}

static inline float uniform_at(uint64_t seed, uint32_t stream, uint64_t e) {
    uint32_t w[4];
    group_words(seed, stream, e >> 2, w);
    return (float)((double)(w[e & 3] >> 8) * (1.0 / 16777216.0));
}

/* round-to-nearest-even float -> bfloat16 bits (inputs are finite) */
static inline uint16_t f32_to_bf16(float f) {
    uint32_t x;
    memcpy(&x, &f, 4);
    uint32_t lsb = (x >> 16) & 1u;
    x += 0x7FFFu + lsb;
    return (uint16_t)(x >> 16);
}

/* ---- flat streams ---------------------------------------------------- */

void sy_uniform_f32(float *out, int64_t n, uint64_t seed, uint32_t stream, int64_t offset) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = uniform_at(seed, stream, (uint64_t)(offset + i));
}

void sy_words_u32(uint32_t *out, int64_t n, uint64_t seed, uint32_t stream, int64_t offset) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        uint32_t w[4];
        uint64_t e = (uint64_t)(offset + i);
        group_words(seed, stream, e >> 2, w);
        out[i] = w[e & 3];
    }
}

void sy_normal_f32(float *out, int64_t n, uint64_t seed, uint32_t stream, int64_t offset, double stddev) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = (float)(stddev * normal_at(seed, stream, (uint64_t)(offset + i)));
}

void sy_normal_bf16(uint16_t *out, int64_t n, uint64_t seed, uint32_t stream, int64_t offset, double stddev) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = f32_to_bf16((float)(stddev * normal_at(seed, stream, (uint64_t)(offset + i))));
}

/*
 * Paged K or V cache.  Logical element (b, t, h, d) with t < seq_tokens[b]
 * takes normal value index ((b * t_stride + t) * hkv + h) * dim + d of the
 * stream, so the values do not depend on which physical block holds them.
 * Physical layout: cache[num_blocks][block_size][hkv][dim]; logical block j
 * of sequence b lives in physical block block_table[b * max_blocks + j].
 * dtype: 0 = bf16 (out is uint16), 1 = f32.
 */
void sy_paged_cache(void *out, int dtype, int32_t batch, int32_t max_blocks, int32_t block_size,
                    int32_t hkv, int32_t dim, const int32_t *block_table, const int32_t *seq_tokens,
                    int64_t t_stride, uint64_t seed, uint32_t stream, double stddev) {
    const int64_t row = (int64_t)hkv * dim;
    const int64_t blk_elems = (int64_t)block_size * row;
    for (int32_t b = 0; b < batch; ++b) {
        int32_t nblk = (seq_tokens[b] + block_size - 1) / block_size;
#pragma omp parallel for schedule(static)
        for (int32_t j = 0; j < nblk; ++j) {
            int64_t phys = block_table[(int64_t)b * max_blocks + j];
            for (int32_t s = 0; s < block_size; ++s) {
                int64_t t = (int64_t)j * block_size + s;
                int64_t dst = phys * blk_elems + (int64_t)s * row;
                for (int64_t k = 0; k < row; ++k) {
                    double v = 0.0;
                    if (t < seq_tokens[b])
                        v = stddev * normal_at(seed, stream, (uint64_t)((b * t_stride + t) * row + k));
                    if (dtype == 0) ((uint16_t *)out)[dst + k] = f32_to_bf16((float)v);
                    else ((float *)out)[dst + k] = (float)v;
                }
            }
        }
    }
}

/*
 * Target / draft distributions for `rows` tree nodes over a vocabulary of V.
 * Row r uses the logical row id row_ids[r] as its key, element x uses index
 * row_id * V + x of each stream.
 *   mode 0 (independent):  p = softmax(sp * n_a),  q = softmax(sp * n_b)
 *   mode 1 (correlated):   l = sp * n_a,  p = softmax(l),  q = softmax(l + sn * n_b)
 * Softmax is evaluated in double with the row maximum subtracted, then stored
 * as float.
 */
void sy_pq_rows(float *p, float *q, int64_t rows, const int64_t *row_ids, int64_t V, uint64_t seed,
                uint32_t stream_a, uint32_t stream_b, int mode, double sp, double sn) {
#pragma omp parallel
    {
        double *la = (double *)malloc(sizeof(double) * V);
        double *lb = (double *)malloc(sizeof(double) * V);
#pragma omp for schedule(dynamic)
        for (int64_t r = 0; r < rows; ++r) {
            uint64_t base = (uint64_t)row_ids[r] * (uint64_t)V;
            double ma = -INFINITY, mb = -INFINITY;
            for (int64_t x = 0; x < V; ++x) {
                double a = sp * normal_at(seed, stream_a, base + x);
                double nb = normal_at(seed, stream_b, base + x);
                double bb = (mode == 0) ? sp * nb : a + sn * nb;
                la[x] = a; lb[x] = bb;
                if (a > ma) ma = a;
                if (bb > mb) mb = bb;
            }
            double sa = 0.0, sb = 0.0;
            for (int64_t x = 0; x < V; ++x) {
                la[x] = exp(la[x] - ma); sa += la[x];
                lb[x] = exp(lb[x] - mb); sb += lb[x];
            }
            float *pr = p + r * V, *qr = q + r * V;
            for (int64_t x = 0; x < V; ++x) {
                pr[x] = (float)(la[x] / sa);
                qr[x] = (float)(lb[x] / sb);
            }
        }
        free(la);
        free(lb);
    }
}

/*
 * The same rows' logits, before any softmax: la = sp * n_a and lb = sp * n_b
 * (mode 0) or la + sn * n_b (mode 1), each rounded to float.  The inputs of a
 * verifier that takes the two models' logits.
 */
void sy_logit_rows(float *la, float *lb, int64_t rows, const int64_t *row_ids, int64_t V, uint64_t seed,
                   uint32_t stream_a, uint32_t stream_b, int mode, double sp, double sn) {
#pragma omp parallel for schedule(dynamic)
    for (int64_t r = 0; r < rows; ++r) {
        uint64_t base = (uint64_t)row_ids[r] * (uint64_t)V;
        for (int64_t x = 0; x < V; ++x) {
            double a = sp * normal_at(seed, stream_a, base + x);
            double nb = normal_at(seed, stream_b, base + x);
            la[r * V + x] = (float)a;
            lb[r * V + x] = (float)((mode == 0) ? sp * nb : a + sn * nb);
        }
    }
}

/*
 * Draw one index from the (not necessarily normalised) weights w[0..V) with
 * a uniform u in [0,1): the first index whose running double sum exceeds
 * u * total; the last positive index if rounding leaves none.  Used only to
 * pick synthetic draft tokens.
 */
int64_t sy_categorical(const float *w, int64_t V, double u) {
    double total = 0.0;
    for (int64_t x = 0; x < V; ++x) total += (double)w[x];
    double target = u * total, run = 0.0;
    int64_t last_pos = -1;
    for (int64_t x = 0; x < V; ++x) {
        if (w[x] > 0.0f) last_pos = x;
        run += (double)w[x];
        if (run > target && w[x] > 0.0f) return x;
    }
    return last_pos;
}
