/*
 * MicroAdam step: plain single-threaded CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may link, load or call
 * this file: only the tests, the package's smoke check and the CPU-baseline leg
 * of the benchmark do. It shares no code, header, table or constant generator
 * with the CUDA path.
 *
 * Built twice from this one source: plain (single-threaded) and with
 * -fopenmp, where the `omp` annotations spread independent blocks and
 * elements over threads. Every result is the same bit for bit in both: each
 * block's Top-k and each element's code are computed alone, min / max are
 * exact in any order, and every AdamStats sum adds its terms in the same
 * age order.
 *
 * Citations: [MicroAdam ¶n] is paragraph n of the web page "MicroAdam
 * (Sparse-Gradient Adaptive Optimization with Quantized Error Feedback)":
 *   ¶1 the per-step algorithm, ¶2 the state-memory formula, ¶3 Lemma 1 /
 *   Lemma 3, ¶5 the update sparsity.
 * Philox4x32-10 follows Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers:
 * As Easy as 1, 2, 3" (SC'11).
 *
 * Precision. The quantities that decide an integer result (a_t, the Top-k
 * order, delta/Delta and the 4-bit codes) are computed in fp32 with every
 * operation rounded to nearest and no contraction (build with
 * -ffp-contract=off), which is the precision the kernels decide them in.
 * The window statistics m_hat, v_hat and the update are computed in fp64;
 * parameters are stored in fp32 because that is their storage type.
 *
 * Readings of points the page leaves open (each also listed in the design
 * notes):
 *  - Q is uniform 4-bit stochastic rounding between the 16 levels
 *    delta + c*(Delta-delta)/15, c = 0..15 (Lemma 1's (Delta-delta)/(2^b-1)
 *    level spacing), done at 16-bit resolution: with s the position in level
 *    units and r a uniform 16-bit draw, c = min(15, floor((floor(2^16 s) + r)
 *    / 2^16)), which rounds up with probability frac(s) to within 2^-16.
 *  - Top-k ties break to the lower index; a row lists its entries in
 *    ascending index order; V is the signed value rounded to bf16 (RNE).
 *  - m_hat = (1-beta1)/(1-beta1^t) * sum_r beta1^r V_r and likewise v_hat
 *    with beta2 and V^2 (Adam's bias-corrected moments), r = age of the row.
 *  - update u = m_hat / (eps + sqrt(v_hat)); decoupled weight decay
 *    p <- p*(1 - lr*wd) is applied to every coordinate before the update.
 *  - bf16 parameters (no fp32 copy, the page's 7B fine-tune on one 40 GB
 *    GPU): every parameter the step changes is rounded once to bf16, to
 *    nearest with ties to even.
 *  - delta, Delta are global over the flat d-vector; blocks are cut over
 *    that vector, or, for a tensor list, over each tensor (segment) in turn;
 *    a ragged last block of length L keeps k = ceil(L*k_b/B_d) entries.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------------- */
/* Philox4x32-10 (Salmon et al., SC'11): 10 rounds of the 4x32 S-box with  */
/* multipliers M0, M1 and Weyl key increments W0, W1 between rounds.       */
/* ---------------------------------------------------------------------- */
#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

void mua_oracle_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2],
                              uint32_t out[4]) {
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += PHILOX_W0;
            k1 += PHILOX_W1;
        }
        uint64_t prod0 = (uint64_t)PHILOX_M0 * (uint64_t)c0;
        uint64_t prod1 = (uint64_t)PHILOX_M1 * (uint64_t)c2;
        uint32_t hi0 = (uint32_t)(prod0 >> 32), lo0 = (uint32_t)prod0;
        uint32_t hi1 = (uint32_t)(prod1 >> 32), lo1 = (uint32_t)prod1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* The 16-bit uniform draw used for element i at step t: Philox with key =
 * seed and counter = (i/8 low, i/8 high, t low, t high); element i takes the
 * (i mod 2)-th 16-bit half of output word (i/2) mod 4. */
uint32_t mua_oracle_draw16(uint64_t seed, int64_t t, int64_t i) {
    uint64_t j = (uint64_t)i >> 3;
    uint32_t ctr[4] = {(uint32_t)j, (uint32_t)(j >> 32), (uint32_t)(uint64_t)t,
                       (uint32_t)((uint64_t)t >> 32)};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    mua_oracle_philox4x32_10(ctr, key, out);
    uint32_t word = out[((uint64_t)i >> 1) & 3];
    return (i & 1) ? (word >> 16) : (word & 0xFFFFu);
}

/* ---------------------------------------------------------------------- */
/* bfloat16: the top 16 bits of an IEEE binary32.                          */
/* ---------------------------------------------------------------------- */
static float f32_from_bits(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t b; memcpy(&b, &f, 4); return b; }

float mua_oracle_bf16_to_f32(uint16_t h) { return f32_from_bits((uint32_t)h << 16); }

/* Round to nearest, ties to even, on the 16 discarded bits; NaN stays NaN. */
uint16_t mua_oracle_f32_to_bf16(float f) {
    uint32_t b = bits_from_f32(f);
    if ((b & 0x7F800000u) == 0x7F800000u && (b & 0x007FFFFFu) != 0)
        return (uint16_t)((b >> 16) | 0x0040u);
    uint32_t lsb = (b >> 16) & 1u;
    return (uint16_t)((b + 0x7FFFu + lsb) >> 16);
}

/* Round an fp64 value to bf16 (8 significant bits, the binary32 exponent
 * range) to nearest, ties to even, in one rounding: the value is scaled by a
 * power of two so that its bf16 unit in the last place becomes 1, rounded to
 * an integer with ties to even, and scaled back (all exact in fp64). Values
 * past the largest bf16 become +-inf; NaN stays NaN. */
uint16_t mua_oracle_f64_to_bf16(double x) {
    if (isnan(x)) return (uint16_t)0x7FC0u;
    if (x == 0.0) return (uint16_t)(signbit(x) ? 0x8000u : 0x0000u);
    int e;
    frexp(x, &e);                      /* |x| = f * 2^e, 0.5 <= f < 1 */
    int q = e - 1;                     /* floor(log2 |x|) */
    if (q < -126) q = -126;            /* subnormal bf16 share the spacing 2^-133 */
    const double ulp = ldexp(1.0, q - 7);
    double y = x / ulp;                /* exact: a power-of-two scaling */
    double r = floor(y);
    const double frac = y - r;         /* exact */
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
    r = copysign(r * ulp, x);          /* a value that rounds to zero keeps its sign */
    if (fabs(r) >= ldexp(1.0, 128)) return (uint16_t)(r > 0 ? 0x7F80u : 0xFF80u);
    return (uint16_t)(bits_from_f32((float)r) >> 16);   /* r is a bf16 value: exact */
}

/* ---------------------------------------------------------------------- */
/* The 4-bit codec Q / Q^{-1} [MicroAdam ¶1, ¶3 Lemma 1].                   */
/* Codes are packed two per byte, element 2q in the low nibble of byte q.   */
/* ---------------------------------------------------------------------- */
static unsigned get_code(const uint8_t* codes, int64_t i) {
    uint8_t byte = codes[i >> 1];
    return (i & 1) ? (unsigned)(byte >> 4) : (unsigned)(byte & 0xFu);
}

static void put_code(uint8_t* codes, int64_t i, unsigned c) {
    uint8_t byte = codes[i >> 1];
    if (i & 1) byte = (uint8_t)((byte & 0x0Fu) | (c << 4));
    else       byte = (uint8_t)((byte & 0xF0u) | c);
    codes[i >> 1] = byte;
}

/* Q^{-1}(e, delta, Delta)_i = delta + c_i * (Delta - delta)/15, in fp32. */
void mua_oracle_dequantize(const uint8_t* codes, int64_t n, float delta, float Delta,
                           float* out) {
    float unit = (Delta - delta) / 15.0f;
    for (int64_t i = 0; i < n; ++i) {
        float level = (float)get_code(codes, i) * unit;
        out[i] = delta + level;
    }
}

/* e = Q(x, delta, Delta): stochastic rounding of x onto the 16 levels at
 * 16-bit resolution. With s = (x - delta) * 15/(Delta - delta) in level units,
 * S = floor(2^16 s) and r a uniform 16-bit draw, c = min(15, floor((S + r) / 2^16)):
 * c = floor(s) + 1 with probability frac(S / 2^16), so E[c] = S / 2^16, within
 * 2^-16 of s. base is the global index of x[0] (it selects the draws). */
void mua_oracle_quantize(const float* x, int64_t n, int64_t base, float delta, float Delta,
                         int64_t t, uint64_t seed, uint8_t* codes) {
    float inv16 = (Delta == delta) ? 0.0f : (15.0f / (Delta - delta)) * 65536.0f;
    /* one byte (two elements) per iteration: no two iterations share a byte */
    #pragma omp parallel for schedule(static)
    for (int64_t i2 = 0; i2 < (n + 1) / 2; ++i2) {
        for (int64_t i = 2 * i2; i < 2 * i2 + 2 && i < n; ++i) {
            float s16 = (x[i] - delta) * inv16;
            uint32_t r = mua_oracle_draw16(seed, t, base + i);
            unsigned c = 15u;
            if (s16 >= 0.0f && s16 < 8388608.0f) {
                uint32_t S = (uint32_t)floorf(s16);
                uint32_t q = (S + r) >> 16;
                c = (q > 15u) ? 15u : q;
            }
            put_code(codes, i, c);
        }
    }
}

/* ---------------------------------------------------------------------- */
/* Per-block Top-k of |a| [MicroAdam ¶1].                                   */
/* ---------------------------------------------------------------------- */
typedef struct { uint32_t key; int32_t idx; } keyed_t;

/* Order: larger |a| first; among equal |a|, the lower index first. */
static int by_key_desc_idx_asc(const void* pa, const void* pb) {
    const keyed_t* a = (const keyed_t*)pa;
    const keyed_t* b = (const keyed_t*)pb;
    if (a->key != b->key) return (a->key > b->key) ? -1 : 1;
    return (a->idx < b->idx) ? -1 : (a->idx > b->idx);
}

static int by_idx_asc(const void* pa, const void* pb) {
    const keyed_t* a = (const keyed_t*)pa;
    const keyed_t* b = (const keyed_t*)pb;
    return (a->idx < b->idx) ? -1 : (a->idx > b->idx);
}

/* k for a block of length L: ceil(L * k_b / B_d). */
int64_t mua_oracle_block_k(int64_t L, int32_t Bd, int32_t kb) {
    return (L * (int64_t)kb + Bd - 1) / Bd;
}

/* ---------------------------------------------------------------------- */
/* One MicroAdam step [MicroAdam ¶1], stages in the page's order.           */
/*                                                                          */
/* p      [d]            fp32 parameters, updated in place                  */
/* g      [d]            bf16 gradient (raw bits)                           */
/* codes  [ceil(d/2)]    e_t in, e_{t+1} out                                */
/* scal   [2]            (delta_t, Delta_t) in, (delta_{t+1}, Delta_{t+1})  */
/* G_idx  [m][n_b][k_b]  int16 block-relative indices, -1 = empty slot      */
/* G_val  [m][n_b][k_b]  bf16 values (raw bits)                             */
/* mhat, vhat, mabs [d]  optional (NULL = skip): m_hat, v_hat and the       */
/*                       cancellation-free magnitude (1-b1)/(1-b1^t) *      */
/*                       sum_r b1^r |V_r|; zero where no window entry.      */
/* Returns 0, or -1 on bad arguments / allocation failure.                  */
/* ---------------------------------------------------------------------- */
/* Number of blocks when the d-vector is the concatenation of n_seg segments
 * (tensors) of the given lengths, each cut into its own blocks of B_d with a
 * ragged last block; one segment of length d is the plain flat cut. */
int64_t mua_oracle_num_blocks(const int64_t* seg, int32_t n_seg, int32_t Bd) {
    int64_t nb = 0;
    for (int32_t s = 0; s < n_seg; ++s) nb += (seg[s] + Bd - 1) / Bd;
    return nb;
}

/* One MicroAdam step [MicroAdam ¶1] over the concatenation of n_seg segments
 * of lengths seg[0..n_seg) (d = their sum), blocks cut per segment. The
 * parameters are fp32 (p32) or, when p16 is given instead, bf16 bits: then
 * each parameter the step changes is computed in fp64 from its bf16 value and
 * rounded once to bf16, nearest-even (there is no fp32 copy); p_exact, if
 * given, receives that fp64 value before the rounding (and f32(p) for the
 * parameters the step leaves alone). */
static int step_impl(const int64_t* seg, int32_t n_seg, int32_t Bd, int32_t kb, int32_t m,
                     float* p32, uint16_t* p16, double* p_exact, const uint16_t* g,
                     uint8_t* codes, float* scal, int16_t* G_idx, uint16_t* G_val, double lr,
                     double beta1, double beta2, double eps, double wd, int64_t t,
                     uint64_t seed, double* mhat, double* vhat, double* mabs) {
    if ((p32 == NULL) == (p16 == NULL)) return -1;
    if (n_seg < 1 || Bd < 1 || Bd > 32766 || kb < 1 || kb > Bd || m < 1 || t < 1) return -1;
    int64_t d = 0;
    for (int32_t s = 0; s < n_seg; ++s) {
        if (seg[s] < 1) return -1;
        d += seg[s];
    }
    const int64_t nb = mua_oracle_num_blocks(seg, n_seg, Bd);
    const float delta_t = scal[0], Delta_t = scal[1];

    float* a = (float*)malloc(sizeof(float) * (size_t)d);
    double* z1 = (double*)calloc((size_t)d, sizeof(double));
    double* z2 = (double*)calloc((size_t)d, sizeof(double));
    double* za = (double*)calloc((size_t)d, sizeof(double));
    uint8_t* touched = (uint8_t*)calloc((size_t)d, 1);
    int64_t* bstart = (int64_t*)malloc(sizeof(int64_t) * (size_t)nb);
    int64_t* blen = (int64_t*)malloc(sizeof(int64_t) * (size_t)nb);
    float* bmin = (float*)malloc(sizeof(float) * (size_t)nb);
    float* bmax = (float*)malloc(sizeof(float) * (size_t)nb);
    const int64_t rows = (t < m) ? t : m;
    double* wr1 = (double*)malloc(sizeof(double) * (size_t)rows);
    double* wr2 = (double*)malloc(sizeof(double) * (size_t)rows);
    int failed = 0;
    if (!a || !z1 || !z2 || !za || !touched || !bstart || !blen || !bmin || !bmax || !wr1 ||
        !wr2) {
        failed = 1;
        goto done;
    }
    /* The blocks, in order: segment by segment, B_d at a time. */
    {
        int64_t j = 0, off = 0;
        for (int32_t s = 0; s < n_seg; ++s) {
            for (int64_t b = 0; b < seg[s]; b += Bd, ++j) {
                bstart[j] = off + b;
                blen[j] = (seg[s] - b < Bd) ? (seg[s] - b) : Bd;
            }
            off += seg[s];
        }
    }

    /* (1) a_t = g_t + Q^{-1}(e_t, delta_t, Delta_t). */
    {
        float unit = (Delta_t - delta_t) / 15.0f;
        #pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < d; ++i) {
            float level = (float)get_code(codes, i) * unit;
            float deq = delta_t + level;
            a[i] = mua_oracle_bf16_to_f32(g[i]) + deq;
        }
    }

    /* (2) (I_t, V_t) = T_k(|a_t|) per block, written to row t mod m of G;
     * (3) the selected entries of a_t are set to zero; each block's residual
     * min and max are kept for (4). */
    const int64_t row = t % m;
    #pragma omp parallel
    {
        keyed_t* order = (keyed_t*)malloc(sizeof(keyed_t) * (size_t)Bd);
        #pragma omp for schedule(dynamic, 16)
        for (int64_t j = 0; j < nb; ++j) {
            if (!order) {
                failed = 1;
                continue;
            }
            const int64_t start = bstart[j];
            const int64_t L = blen[j];
            const int64_t k = mua_oracle_block_k(L, Bd, kb);
            for (int64_t q = 0; q < L; ++q) {
                order[q].key = bits_from_f32(a[start + q]) & 0x7FFFFFFFu;
                order[q].idx = (int32_t)q;
            }
            qsort(order, (size_t)L, sizeof(keyed_t), by_key_desc_idx_asc);
            qsort(order, (size_t)k, sizeof(keyed_t), by_idx_asc);
            int16_t* ri = G_idx + (row * nb + j) * kb;
            uint16_t* rv = G_val + (row * nb + j) * kb;
            for (int64_t s = 0; s < kb; ++s) {
                if (s < k) {
                    int64_t q = order[s].idx;
                    ri[s] = (int16_t)q;
                    rv[s] = mua_oracle_f32_to_bf16(a[start + q]);
                } else {
                    ri[s] = -1;
                    rv[s] = 0;
                }
            }
            for (int64_t s = 0; s < k; ++s) a[start + order[s].idx] = 0.0f;
            float lo = a[start], hi = a[start];
            for (int64_t q = 1; q < L; ++q) {
                if (a[start + q] < lo) lo = a[start + q];
                if (a[start + q] > hi) hi = a[start + q];
            }
            bmin[j] = lo;
            bmax[j] = hi;
        }
        free(order);
    }
    if (failed) goto done;

    /* (4) e_{t+1} = Q(a_t, delta_{t+1}, Delta_{t+1}) with the scalar min and
     * max of the residual over all d (exact in any order; a -0 result is
     * stored as +0). */
    float lo = bmin[0], hi = bmax[0];
    for (int64_t j = 1; j < nb; ++j) {
        if (bmin[j] < lo) lo = bmin[j];
        if (bmax[j] > hi) hi = bmax[j];
    }
    lo = lo + 0.0f;
    hi = hi + 0.0f;
    mua_oracle_quantize(a, d, 0, lo, hi, t, seed, codes);
    scal[0] = lo;
    scal[1] = hi;

    /* (5) m_hat = AdamStats(beta1, G), v_hat = AdamStats(beta2, G^2) by the
     * unrolled decay z[I] += beta^r V over the rows in the window, oldest
     * (largest age r) first at every index. */
    for (int64_t r = 0; r < rows; ++r) {
        const double w1 = pow(beta1, (double)r);
        const double w2 = pow(beta2, (double)r);
        wr1[r] = w1;
        wr2[r] = w2;
    }
    #pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < nb; ++j) {
        for (int64_t r = rows - 1; r >= 0; --r) {
            const int64_t rr = (t - r) % m;
            const int16_t* ri = G_idx + (rr * nb + j) * kb;
            const uint16_t* rv = G_val + (rr * nb + j) * kb;
            for (int64_t s = 0; s < kb; ++s) {
                if (ri[s] < 0) continue;
                const int64_t q = bstart[j] + ri[s];
                const double V = (double)mua_oracle_bf16_to_f32(rv[s]);
                z1[q] += wr1[r] * V;
                z2[q] += wr2[r] * (V * V);
                za[q] += wr1[r] * fabs(V);
                touched[q] = 1;
            }
        }
    }
    const double f1 = (1.0 - beta1) / (1.0 - pow(beta1, (double)t));
    const double f2 = (1.0 - beta2) / (1.0 - pow(beta2, (double)t));

    /* (6) p <- p*(1 - lr*wd) - lr * m_hat / (eps + sqrt(v_hat)). */
    const double decay = 1.0 - lr * wd;
    #pragma omp parallel for schedule(static)
    for (int64_t q = 0; q < d; ++q) {
        const double m_hat = f1 * z1[q];
        const double v_hat = f2 * z2[q];
        if (mhat) mhat[q] = m_hat;
        if (vhat) vhat[q] = v_hat;
        if (mabs) mabs[q] = f1 * za[q];
        double pq = p32 ? (double)p32[q] : (double)mua_oracle_bf16_to_f32(p16[q]);
        if (wd != 0.0) pq = pq * decay;
        if (touched[q]) pq = pq - lr * (m_hat / (eps + sqrt(v_hat)));
        if (p_exact) p_exact[q] = pq;
        if (wd != 0.0 || touched[q]) {
            if (p32) p32[q] = (float)pq;
            else p16[q] = mua_oracle_f64_to_bf16(pq);
        }
    }

done:
    free(a); free(z1); free(z2); free(za); free(touched);
    free(bstart); free(blen); free(bmin); free(bmax); free(wr1); free(wr2);
    return failed ? -1 : 0;
}

int mua_oracle_step_seg(const int64_t* seg, int32_t n_seg, int32_t Bd, int32_t kb, int32_t m,
                        float* p, const uint16_t* g, uint8_t* codes, float* scal,
                        int16_t* G_idx, uint16_t* G_val, double lr, double beta1,
                        double beta2, double eps, double wd, int64_t t, uint64_t seed,
                        double* mhat, double* vhat, double* mabs) {
    if (p == NULL) return -1;
    return step_impl(seg, n_seg, Bd, kb, m, p, NULL, NULL, g, codes, scal, G_idx, G_val, lr,
                     beta1, beta2, eps, wd, t, seed, mhat, vhat, mabs);
}

/* The same step with bf16 parameters (see step_impl). */
int mua_oracle_step_seg_bf16(const int64_t* seg, int32_t n_seg, int32_t Bd, int32_t kb,
                             int32_t m, uint16_t* p16, double* p_exact, const uint16_t* g,
                             uint8_t* codes, float* scal, int16_t* G_idx, uint16_t* G_val,
                             double lr, double beta1, double beta2, double eps, double wd,
                             int64_t t, uint64_t seed, double* mhat, double* vhat,
                             double* mabs) {
    if (p16 == NULL) return -1;
    return step_impl(seg, n_seg, Bd, kb, m, NULL, p16, p_exact, g, codes, scal, G_idx, G_val,
                     lr, beta1, beta2, eps, wd, t, seed, mhat, vhat, mabs);
}

/* The flat cut: one segment of length d. */
int mua_oracle_step(int64_t d, int32_t Bd, int32_t kb, int32_t m, float* p,
                    const uint16_t* g, uint8_t* codes, float* scal, int16_t* G_idx,
                    uint16_t* G_val, double lr, double beta1, double beta2, double eps,
                    double wd, int64_t t, uint64_t seed, double* mhat, double* vhat,
                    double* mabs) {
    if (d < 1) return -1;
    return mua_oracle_step_seg(&d, 1, Bd, kb, m, p, g, codes, scal, G_idx, G_val, lr, beta1,
                               beta2, eps, wd, t, seed, mhat, vhat, mabs);
}
