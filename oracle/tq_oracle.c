/*
 * tq_oracle.c -- plain, slow, fp64 CPU oracle for the TurboQuant KV-cache
 * codec and attention over the compressed cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check in
 * __graft_entry__.py and the cpu_baseline / reference arm of bench.py may
 * load or call this code.  The product library (libtq.so) never links,
 * loads or calls it, and this file shares no code, header, table or
 * constant generator with the CUDA path.
 *
 * Sources (docs.rs pages):
 *   [TQ]  turboquant-plus-rs 0.1.0 README: "Architecture" (the two-stage
 *         algorithm: PolarQuant at b-1 bits = random rotation + Lloyd
 *         scalar quantizer on the post-rotation Gaussian, then a 1-bit QJL
 *         sign sketch of the residual; V uses the MSE-only stage at b bits),
 *         "Modules" table (rotation: fast Walsh-Hadamard; codebook:
 *         closed form 1-2 bit, Lloyd for more; polar_quant: norm extraction
 *         and correction; qjl; utils: bit packing), "Key ideas".
 *   [BP]  bitpolar 0.3.3 src/kv_cache.rs: KvCacheConfig {head_dim, bits,
 *         projections, seed}; KvCacheCompressor::attention_scores (scores are
 *         pre-softmax and scaled by 1/sqrt(head_dim)); decode_values;
 *         MultiHeadKvCache::new (head h uses seed.wrapping_add(h)).
 *
 * Every step below follows those passages.  Where the pages are silent the
 * plainest reading is taken; those readings are:
 *   R1  PRNG: SplitMix64 (Steele, Lea, Flood 2014) seeded with seed+h.
 *       The first d draws give the signs of the rotation (top bit set ->
 *       -1); the next m*d values, taken in Box-Muller pairs, fill the QJL
 *       matrix S row-major [m][d]; every entry of S is rounded to binary16
 *       (round to nearest even) and that rounded value IS S.
 *   R2  Codebook: Lloyd-Max centroids of N(0,1), 2^B levels, ascending;
 *       closed form +-sqrt(2/pi) for B=1, Lloyd iteration otherwise; the
 *       result is made exactly antisymmetric.
 *   R3  Rotation Pi = H D / sqrt(d) (Sylvester Hadamard H, random signs D).
 *   R4  Quantizer input z = sqrt(d) * Pi x / ||x||; index = number of
 *       boundaries beta_k with z >= beta_k (ties go to the upper cell).
 *   R5  Norm correction: stored norm n_s = ||x|| / ||yhat||, yhat =
 *       C[idx]/sqrt(d), so the reconstruction has the input's norm.
 *   R6  QJL in the rotated frame: bit_i = [<S_i, r> >= 0] with
 *       r = ||x|| Pi x/||x|| - n_s yhat, gamma = ||r||; estimator
 *       sqrt(pi/2)/m * gamma * <S q_rot, 2 bit - 1>.
 *   R7  Zero or non-finite rows encode as: every index = 2^(B-1) (smallest
 *       positive centroid), n_s = 0, gamma = 0, all sign bits 1; non-finite
 *       rows are counted.
 *   R9  Haar rotation (the [TQ] Modules table's other rotation: "Haar-
 *       distributed rotation via QR"): Pi = Q, the orthogonal factor of the
 *       QR factorization of a d x d matrix G of iid N(0,1) entries, with the
 *       column signs chosen so that R has a positive diagonal, which makes Q
 *       Haar-distributed (Mezzadri 2007).  G is filled row-major by Box-Muller
 *       pairs (not rounded) from the head's SplitMix64 stream continued after
 *       the d sign draws and the draws of S.  The rest of the method is
 *       unchanged: z = sqrt(d) Q x / ||x||, reconstruction Q^T (...).
 *   R10 Outlier/normal channel splitting ([TQ] Modules, outlier: a
 *       fractional bit rate from coding outlier and normal channels at
 *       different widths): a head's d channels
 *       are split into two groups, outliers first (the caller orders the
 *       channels); each group is a codec of its own (its own rotation over the
 *       group's channels, its own bits), so the bits per value are the
 *       channel-weighted mean.  A key's score is the full inner product
 *       q.k_hat / sqrt(d) = (sum over groups g of q_g . k_hat_g) / sqrt(d); one
 *       softmax covers the token; the value is the concatenation of the groups'
 *       reconstructions.
 *   R8  Packed layout (the pages give none):
 *       K row: B_K index bit planes (plane p holds bit p of every index;
 *       coordinate j -> byte j/8, bit j%8), then the m-bit sign plane, then
 *       n_s (fp32), then gamma (fp32).
 *       V row: B_V-bit index fields, coordinate j at bit B_V*j of a
 *       little-endian bit stream, then n_s (fp32).
 *   R11 Binary16 key norms (turboquant-plus-rs "Compression formats": turbo4
 *       at 4.25 bits per value): with norm_f16 set, the K row ends in n_s
 *       and gamma each rounded to binary16 (ties to even), 2 bytes apiece,
 *       little-endian, instead of the two fp32 values; the index planes and
 *       sign bits are those of the fp32 format (computed from the unrounded
 *       norms), and every consumer reads the rounded norms.  A row whose
 *       rounded n_s or gamma is infinite (at or above 65520) is stored as the
 *       degenerate row of R7 and counted with the non-finite rows.  V rows
 *       keep their fp32 n_s: the row length stays a multiple of 4 bytes.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define TQO_MAXL 64

/* ---------------------------------------------------------------- PRNG -- */

/* SplitMix64 step, from its published definition (R1). */
uint64_t tqo_splitmix64_next(uint64_t *state) {
    *state += 0x9E3779B97F4A7C15ULL;
    uint64_t z = *state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Round a double to the nearest binary16 value (ties to even), returned as
 * a double.  Handles subnormals; overflow goes to +-inf. */
double tqo_round_fp16(double x) {
    if (x == 0.0 || !isfinite(x)) return x;
    double ax = fabs(x);
    int e;
    frexp(ax, &e);            /* ax in [2^(e-1), 2^e) */
    int ex = e - 1;           /* unbiased exponent */
    int q = (ex < -14) ? -24 : ex - 10;   /* exponent of one ulp */
    double r = nearbyint(ldexp(ax, -q)) ; /* default mode: ties to even */
    double res = ldexp(r, q);
    if (res > 65504.0) res = INFINITY;
    return copysign(res, x);
}

/* Per-head random tables (R1, [BP] MultiHeadKvCache::new: seed + h). */
void tqo_head_tables(int d, int m, uint64_t seed, int h, double *signs, double *S) {
    uint64_t st = seed + (uint64_t)(int64_t)h;    /* wrapping add */
    for (int j = 0; j < d; ++j) {
        uint64_t u = tqo_splitmix64_next(&st);
        signs[j] = (u >> 63) ? -1.0 : 1.0;
    }
    const double two_pi = 6.283185307179586476925286766559;
    int64_t n = (int64_t)m * d;
    for (int64_t i = 0; i < n; i += 2) {
        uint64_t ua = tqo_splitmix64_next(&st);
        uint64_t ub = tqo_splitmix64_next(&st);
        double u1 = (double)((ua >> 11) + 1) * 0x1.0p-53;   /* (0, 1] */
        double u2 = (double)(ub >> 11) * 0x1.0p-53;         /* [0, 1) */
        double rad = sqrt(-2.0 * log(u1));
        S[i] = tqo_round_fp16(rad * cos(two_pi * u2));
        if (i + 1 < n) S[i + 1] = tqo_round_fp16(rad * sin(two_pi * u2));
    }
}

/* Haar rotation of head h (R9): Householder QR of G, Q = H_0 H_1 ... H_(d-1),
 * then column k of Q multiplied by the sign of R[k][k]. */
/* The Gaussian matrix G [d][d] of head h (R9): Box-Muller pairs from the
 * stream continued after the d sign draws and the draws of S. */
void tqo_haar_gaussian(int d, int m, uint64_t seed, int h, double *G) {
    uint64_t st = seed + (uint64_t)(int64_t)h;    /* wrapping add */
    for (int j = 0; j < d; ++j) tqo_splitmix64_next(&st);          /* the rotation signs */
    int64_t ns = (int64_t)m * d;
    ns += ns & 1;                                                 /* S is drawn in pairs */
    for (int64_t i = 0; i < ns; ++i) tqo_splitmix64_next(&st);
    const double two_pi = 6.283185307179586476925286766559;
    for (int64_t i = 0; i < (int64_t)d * d; i += 2) {
        uint64_t ua = tqo_splitmix64_next(&st);
        uint64_t ub = tqo_splitmix64_next(&st);
        double u1 = (double)((ua >> 11) + 1) * 0x1.0p-53;
        double u2 = (double)(ub >> 11) * 0x1.0p-53;
        double rad = sqrt(-2.0 * log(u1));
        G[i] = rad * cos(two_pi * u2);
        if (i + 1 < (int64_t)d * d) G[i + 1] = rad * sin(two_pi * u2);
    }
}

void tqo_haar_matrix(int d, int m, uint64_t seed, int h, double *Q) {
    double *A = (double *)malloc(sizeof(double) * d * d);
    double *V = (double *)malloc(sizeof(double) * d * d);         /* reflector k in row k, entries k..d-1 */
    tqo_haar_gaussian(d, m, seed, h, A);
    for (int k = 0; k < d; ++k) {
        double nx = 0.0;
        for (int i = k; i < d; ++i) nx += A[i * d + k] * A[i * d + k];
        nx = sqrt(nx);
        double *v = V + (size_t)k * d;
        for (int i = 0; i < d; ++i) v[i] = 0.0;
        /* v = x - alpha e1, alpha = -sign(x0) |x| (no cancellation) */
        double alpha = A[k * d + k] >= 0.0 ? -nx : nx;
        for (int i = k; i < d; ++i) v[i] = A[i * d + k];
        v[k] -= alpha;
        double nv = 0.0;
        for (int i = k; i < d; ++i) nv += v[i] * v[i];
        nv = sqrt(nv);
        if (nv > 0.0)
            for (int i = k; i < d; ++i) v[i] /= nv;
        /* A[k:, k:] -= 2 v (v^T A[k:, k:]) */
        for (int j = k; j < d; ++j) {
            double dot = 0.0;
            for (int i = k; i < d; ++i) dot += v[i] * A[i * d + j];
            for (int i = k; i < d; ++i) A[i * d + j] -= 2.0 * v[i] * dot;
        }
    }
    /* Q = H_0 ... H_(d-1) I */
    for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j) Q[i * d + j] = (i == j) ? 1.0 : 0.0;
    for (int k = d - 1; k >= 0; --k) {
        const double *v = V + (size_t)k * d;
        for (int j = 0; j < d; ++j) {
            double dot = 0.0;
            for (int i = k; i < d; ++i) dot += v[i] * Q[i * d + j];
            for (int i = k; i < d; ++i) Q[i * d + j] -= 2.0 * v[i] * dot;
        }
    }
    /* positive diagonal of R: R[k][k] is A[k][k] after the reflections */
    for (int k = 0; k < d; ++k)
        if (A[k * d + k] < 0.0)
            for (int i = 0; i < d; ++i) Q[i * d + k] = -Q[i * d + k];
    free(A);
    free(V);
}

/* ------------------------------------------------------------ codebook -- */

static double std_pdf(double x) {
    if (isinf(x)) return 0.0;
    return exp(-0.5 * x * x) / sqrt(2.0 * M_PI);
}

/* Upper tail Q(x) = P(X > x) and CDF Phi(x), via erfc for accuracy. */
static double std_q(double x) { return 0.5 * erfc(x / sqrt(2.0)); }
static double std_cdf(double x) { return 0.5 * erfc(-x / sqrt(2.0)); }

/* Probability of the cell (a, b]. */
static double cell_mass(double a, double b) {
    if (a >= 0.0) return std_q(a) - std_q(b);
    if (b <= 0.0) return std_cdf(b) - std_cdf(a);
    return 1.0 - std_cdf(a) - std_q(b);
}

/* Lloyd-Max quantizer of N(0,1) with L = 2^B levels (R2).
 * c[L] ascending centroids, beta[L-1] boundaries (midpoints).
 * Returns L, or 0 if B is out of range. */
static int lloyd_max_compute(int B, double *c, double *beta) {
    int L = 1 << B;
    if (B == 1) {
        double v = sqrt(2.0 / M_PI);
        c[0] = -v; c[1] = v; beta[0] = 0.0;
        return L;
    }
    for (int k = 0; k < L; ++k) c[k] = -2.0 + 4.0 * k / (L - 1);
    for (int it = 0; it < 1000000; ++it) {
        for (int k = 0; k < L - 1; ++k) beta[k] = 0.5 * (c[k] + c[k + 1]);
        double maxd = 0.0;
        for (int k = 0; k < L; ++k) {
            double a = (k == 0) ? -INFINITY : beta[k - 1];
            double b = (k == L - 1) ? INFINITY : beta[k];
            double nc = (std_pdf(a) - std_pdf(b)) / cell_mass(a, b);
            double dd = fabs(nc - c[k]);
            if (dd > maxd) maxd = dd;
            c[k] = nc;
        }
        if (maxd < 1e-15) break;
    }
    for (int k = 0; k < L / 2; ++k) {          /* exact antisymmetry */
        double s = 0.5 * (c[L - 1 - k] - c[k]);
        c[k] = -s; c[L - 1 - k] = s;
    }
    for (int k = 0; k < L - 1; ++k) beta[k] = 0.5 * (c[k] + c[k + 1]);
    beta[L / 2 - 1] = 0.0;
    return L;
}

/* The iteration is deterministic, so each B is computed once per process. */
int tqo_lloyd_max(int B, double *c, double *beta) {
    static double cache_c[7][TQO_MAXL], cache_b[7][TQO_MAXL];
    static int done[7];
    if (B < 1 || B > 6) return 0;
    int L = 1 << B;
    if (!done[B]) {
        lloyd_max_compute(B, cache_c[B], cache_b[B]);
        done[B] = 1;
    }
    memcpy(c, cache_c[B], sizeof(double) * L);
    memcpy(beta, cache_b[B], sizeof(double) * (L - 1));
    return L;
}

/* -------------------------------------------------------------- rotation -- */

/* In-place unnormalized Walsh-Hadamard transform in Sylvester order:
 * v <- H v with H[i][j] = (-1)^popcount(i & j). */
void tqo_fwht(double *v, int d) {
    for (int len = 1; len < d; len <<= 1)
        for (int i = 0; i < d; i += 2 * len)
            for (int j = i; j < i + len; ++j) {
                double a = v[j], b = v[j + len];
                v[j] = a + b;
                v[j + len] = a - b;
            }
}

/* out = Pi x = H (D x) / sqrt(d)   (R3) */
void tqo_rotate(int d, const double *signs, const double *x, double *out) {
    for (int j = 0; j < d; ++j) out[j] = signs[j] * x[j];
    tqo_fwht(out, d);
    double s = 1.0 / sqrt((double)d);
    for (int j = 0; j < d; ++j) out[j] *= s;
}

/* out = Pi^T y = D H y / sqrt(d) */
void tqo_unrotate(int d, const double *signs, const double *y, double *out) {
    for (int j = 0; j < d; ++j) out[j] = y[j];
    tqo_fwht(out, d);
    double s = 1.0 / sqrt((double)d);
    for (int j = 0; j < d; ++j) out[j] *= s * signs[j];
}

/* out = Q x and out = Q^T y for a dense d x d rotation (R9), row-major Q. */
void tqo_rotate_dense(int d, const double *Q, const double *x, double *out) {
    for (int i = 0; i < d; ++i) {
        double a = 0.0;
        for (int j = 0; j < d; ++j) a += Q[(size_t)i * d + j] * x[j];
        out[i] = a;
    }
}

void tqo_unrotate_dense(int d, const double *Q, const double *y, double *out) {
    for (int j = 0; j < d; ++j) {
        double a = 0.0;
        for (int i = 0; i < d; ++i) a += Q[(size_t)i * d + j] * y[i];
        out[j] = a;
    }
}

/* --------------------------------------------------------------- config -- */

typedef struct {
    int d, bits, m;
    int BK, BV, LK, LV;
    int norm_correct;          /* 1: n_s = n/||yhat|| (R5); 0: n_s = n */
    double ck[TQO_MAXL], bk[TQO_MAXL], cv[TQO_MAXL], bv[TQO_MAXL];
    int rotation;              /* 0: Hadamard (R3), rot = d signs; 1: Haar (R9), rot = Q (d x d) */
    int norm_f16;              /* 1: K row norms as binary16 (R11); 0: fp32 (R8) */
} tqo_cfg;

/* Pi x and Pi^T y for the configured rotation; `rot` is the head's signs
 * (Hadamard) or its matrix Q (Haar). */
static void rot_apply(const tqo_cfg *c, const double *rot, const double *x, double *out) {
    if (c->rotation == 1) tqo_rotate_dense(c->d, rot, x, out);
    else tqo_rotate(c->d, rot, x, out);
}

static void rot_apply_t(const tqo_cfg *c, const double *rot, const double *y, double *out) {
    if (c->rotation == 1) tqo_unrotate_dense(c->d, rot, y, out);
    else tqo_unrotate(c->d, rot, y, out);
}

/* bits = total TurboQuant bits b: K uses b-1 PolarQuant bits + 1 QJL bit,
 * V uses b MSE bits ([TQ] Architecture, Key ideas). */
int tqo_cfg_init(tqo_cfg *cfg, int d, int bits, int m, int norm_correct) {
    memset(cfg, 0, sizeof(*cfg));
    if (d < 2 || (d & (d - 1)) || bits < 2 || bits > 6 || m < 1 || (m % 8)) return -1;
    cfg->d = d; cfg->bits = bits; cfg->m = m;
    cfg->BK = bits - 1; cfg->BV = bits;
    cfg->norm_correct = norm_correct;
    cfg->LK = tqo_lloyd_max(cfg->BK, cfg->ck, cfg->bk);
    cfg->LV = tqo_lloyd_max(cfg->BV, cfg->cv, cfg->bv);
    return 0;
}

int tqo_k_row_bytes(const tqo_cfg *c) { return c->BK * c->d / 8 + c->m / 8 + (c->norm_f16 ? 4 : 8); }
int tqo_v_row_bytes(const tqo_cfg *c) { return c->BV * c->d / 8 + 4; }

/* ---------------------------------------------------------------- encode -- */

static int quant_index(double z, const double *beta, int L) {
    int idx = 0;
    for (int k = 0; k < L - 1; ++k) if (z >= beta[k]) ++idx;
    return idx;
}

static void put_f32(uint8_t *dst, double v) {
    float f = (float)v;
    memcpy(dst, &f, 4);
}

static double get_f32(const uint8_t *src) {
    float f;
    memcpy(&f, src, 4);
    return (double)f;
}

/* Bits of a binary16 value h (a value tqo_round_fp16 returns: finite or
 * +-inf): sign, 5-bit biased exponent, 10-bit fraction. */
static uint16_t fp16_bits(double h) {
    const uint16_t sg = signbit(h) ? 0x8000u : 0u;
    const double a = fabs(h);
    if (isinf(a)) return (uint16_t)(sg | 0x7C00u);
    if (a < 0x1p-14) return (uint16_t)(sg | (uint16_t)(a * 0x1p24));     /* subnormal or zero */
    int e;
    frexp(a, &e);                                                       /* a in [2^(e-1), 2^e) */
    const int ex = e - 1;
    const uint16_t frac = (uint16_t)(ldexp(a, 10 - ex) - 1024.0);
    return (uint16_t)(sg | (uint16_t)((ex + 15) << 10) | frac);
}

static double fp16_value(uint16_t b) {
    const int ex = (b >> 10) & 31, frac = b & 1023;
    double v;
    if (ex == 0) v = ldexp((double)frac, -24);
    else if (ex == 31) v = frac ? NAN : INFINITY;
    else v = ldexp((double)(1024 + frac), ex - 25);
    return (b & 0x8000u) ? -v : v;
}

static void put_f16(uint8_t *dst, double h) {
    const uint16_t b = fp16_bits(h);
    dst[0] = (uint8_t)(b & 0xFFu);
    dst[1] = (uint8_t)(b >> 8);
}

static double get_f16(const uint8_t *src) { return fp16_value((uint16_t)(src[0] | (src[1] << 8))); }

/* Encode one row.  is_key selects TurboQuant (K) or MSE-only (V).
 * signs, S[m*d]: the head's tables (signs: the d rotation signs, or Q
 * (d x d) for the Haar rotation).  x[d]: the input, exactly converted.
 * row: packed output (row bytes of the K or V format), zeroed here.
 * Diagnostics (may be NULL): z_out[d] quantizer inputs (HUGE_VAL for a
 * degenerate row), pn_out[m] normalized projections p_i/gamma (HUGE_VAL if
 * gamma == 0 or degenerate), ns_out, gamma_out.
 * Returns 1 if the row had a non-finite value (R7), else 0. */
int tqo_encode_row(const tqo_cfg *cfg, int is_key, const double *signs, const double *S,
                   const double *x, uint8_t *row, double *z_out, double *pn_out,
                   double *ns_out, double *gamma_out) {
    const int d = cfg->d, m = cfg->m;
    const int B = is_key ? cfg->BK : cfg->BV;
    const int L = is_key ? cfg->LK : cfg->LV;
    const double *cb = is_key ? cfg->ck : cfg->cv;
    const double *bd = is_key ? cfg->bk : cfg->bv;
    const int nbytes = is_key ? tqo_k_row_bytes(cfg) : tqo_v_row_bytes(cfg);
    memset(row, 0, (size_t)nbytes);

    int *idx = (int *)malloc(sizeof(int) * d);
    double *y = (double *)malloc(sizeof(double) * d);
    double *r = (double *)malloc(sizeof(double) * d);
    unsigned char *bit = (unsigned char *)malloc((size_t)m);

    int nonfinite = 0;
    double mx = 0.0;
    for (int j = 0; j < d; ++j) {
        if (!isfinite(x[j])) nonfinite = 1;
        else if (fabs(x[j]) > mx) mx = fabs(x[j]);
    }
    /* a1: norm extraction ([TQ] polar_quant) */
    double n = 0.0;
    if (!nonfinite && mx > 0.0) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j) { double t = x[j] / mx; acc += t * t; }
        n = mx * sqrt(acc);
    }
    double ns = 0.0, gamma = 0.0;
    if (nonfinite || n == 0.0) {
        /* R7: degenerate row */
        for (int j = 0; j < d; ++j) idx[j] = L / 2;
        for (int i = 0; i < m; ++i) bit[i] = 1;
        if (z_out) for (int j = 0; j < d; ++j) z_out[j] = HUGE_VAL;
        if (pn_out) for (int i = 0; i < m; ++i) pn_out[i] = HUGE_VAL;
    } else {
        /* a2: rotate the unit vector: y = Pi x / n */
        rot_apply(cfg, signs, x, y);
        for (int j = 0; j < d; ++j) y[j] /= n;
        /* a3: scalar quantization of z = sqrt(d) y against the N(0,1) codebook */
        double sd = sqrt((double)d);
        double yh2 = 0.0;
        for (int j = 0; j < d; ++j) {
            double z = sd * y[j];
            if (z_out) z_out[j] = z;
            idx[j] = quant_index(z, bd, L);
            double yh = cb[idx[j]] / sd;
            yh2 += yh * yh;
        }
        /* a4: norm correction (R5) */
        ns = cfg->norm_correct ? n / sqrt(yh2) : n;
        if (is_key) {
            /* a5: residual in the rotated frame and its norm */
            double g2 = 0.0;
            for (int j = 0; j < d; ++j) {
                r[j] = n * y[j] - ns * (cb[idx[j]] / sd);
                g2 += r[j] * r[j];
            }
            gamma = sqrt(g2);
            /* a6: QJL signs of S r (R6) */
            for (int i = 0; i < m; ++i) {
                double p = 0.0;
                for (int j = 0; j < d; ++j) p += S[(int64_t)i * d + j] * r[j];
                bit[i] = (p >= 0.0) ? 1 : 0;
                if (pn_out) pn_out[i] = (gamma > 0.0) ? p / gamma : HUGE_VAL;
            }
        }
    }
    (void)B;
    /* R11: binary16 key norms; a norm that overflows makes the row degenerate */
    double ns16 = 0.0, gamma16 = 0.0;
    if (is_key && cfg->norm_f16) {
        ns16 = tqo_round_fp16(ns);
        gamma16 = tqo_round_fp16(gamma);
        if (isinf(ns16) || isinf(gamma16)) {
            nonfinite = 1;
            ns = gamma = ns16 = gamma16 = 0.0;
            for (int j = 0; j < d; ++j) idx[j] = L / 2;
            for (int i = 0; i < m; ++i) bit[i] = 1;
            if (z_out) for (int j = 0; j < d; ++j) z_out[j] = HUGE_VAL;
            if (pn_out) for (int i = 0; i < m; ++i) pn_out[i] = HUGE_VAL;
        }
    }
    /* a7: bit packing (R8) */
    if (is_key) {
        const int pb = d / 8;
        for (int p = 0; p < cfg->BK; ++p)
            for (int j = 0; j < d; ++j)
                if ((idx[j] >> p) & 1) row[p * pb + j / 8] |= (uint8_t)(1u << (j % 8));
        uint8_t *sg = row + cfg->BK * pb;
        for (int i = 0; i < m; ++i)
            if (bit[i]) sg[i / 8] |= (uint8_t)(1u << (i % 8));
        if (cfg->norm_f16) {
            put_f16(row + cfg->BK * pb + m / 8, ns16);
            put_f16(row + cfg->BK * pb + m / 8 + 2, gamma16);
        } else {
            put_f32(row + cfg->BK * pb + m / 8, ns);
            put_f32(row + cfg->BK * pb + m / 8 + 4, gamma);
        }
    } else {
        for (int j = 0; j < d; ++j)
            for (int k = 0; k < cfg->BV; ++k) {
                int q = cfg->BV * j + k;
                if ((idx[j] >> k) & 1) row[q / 8] |= (uint8_t)(1u << (q % 8));
            }
        put_f32(row + cfg->BV * d / 8, ns);
    }
    if (ns_out) *ns_out = ns;
    if (gamma_out) *gamma_out = gamma;
    free(idx); free(y); free(r); free(bit);
    return nonfinite;
}

/* Encode T rows of one head.  x: [T][d]; rows: [T][row bytes].  Optional
 * diagnostics z [T][d], pn [T][m], ns [T], gamma [T].  Returns the number
 * of non-finite rows. */
int tqo_encode_block(const tqo_cfg *cfg, int is_key, const double *signs, const double *S,
                     const double *x, int64_t T, uint8_t *rows, double *z, double *pn,
                     double *ns, double *gamma) {
    const int rb = is_key ? tqo_k_row_bytes(cfg) : tqo_v_row_bytes(cfg);
    int cnt = 0;
    for (int64_t t = 0; t < T; ++t)
        cnt += tqo_encode_row(cfg, is_key, signs, S, x + t * cfg->d, rows + t * rb,
                              z ? z + t * cfg->d : NULL, pn ? pn + t * cfg->m : NULL,
                              ns ? ns + t : NULL, gamma ? gamma + t : NULL);
    return cnt;
}

/* --------------------------------------------------------------- unpack -- */

void tqo_unpack_k(const tqo_cfg *cfg, const uint8_t *row, int *idx, int *bit, double *ns,
                  double *gamma) {
    const int d = cfg->d, m = cfg->m, pb = d / 8;
    for (int j = 0; j < d; ++j) {
        int v = 0;
        for (int p = 0; p < cfg->BK; ++p) v |= ((row[p * pb + j / 8] >> (j % 8)) & 1) << p;
        idx[j] = v;
    }
    const uint8_t *sg = row + cfg->BK * pb;
    for (int i = 0; i < m; ++i) bit[i] = (sg[i / 8] >> (i % 8)) & 1;
    if (cfg->norm_f16) {
        *ns = get_f16(row + cfg->BK * pb + m / 8);
        *gamma = get_f16(row + cfg->BK * pb + m / 8 + 2);
    } else {
        *ns = get_f32(row + cfg->BK * pb + m / 8);
        *gamma = get_f32(row + cfg->BK * pb + m / 8 + 4);
    }
}

void tqo_unpack_v(const tqo_cfg *cfg, const uint8_t *row, int *idx, double *ns) {
    const int d = cfg->d;
    for (int j = 0; j < d; ++j) {
        int v = 0;
        for (int k = 0; k < cfg->BV; ++k) {
            int q = cfg->BV * j + k;
            v |= ((row[q / 8] >> (q % 8)) & 1) << k;
        }
        idx[j] = v;
    }
    *ns = get_f32(row + cfg->BV * d / 8);
}

/* ------------------------------------------------------------ dequantize -- */

/* v_hat = n_s Pi^T (C[idx]/sqrt(d))    ([BP] decode_values) */
void tqo_dequant_v(const tqo_cfg *cfg, const double *signs, const uint8_t *row, double *out) {
    const int d = cfg->d;
    int *idx = (int *)malloc(sizeof(int) * d);
    double *w = (double *)malloc(sizeof(double) * d);
    double ns;
    tqo_unpack_v(cfg, row, idx, &ns);
    double sd = sqrt((double)d);
    for (int j = 0; j < d; ++j) w[j] = ns * cfg->cv[idx[j]] / sd;
    rot_apply_t(cfg, signs, w, out);
    free(idx); free(w);
}

/* k_hat = Pi^T (n_s C[idx]/sqrt(d) + sqrt(pi/2)/m * gamma * S^T (2 bit - 1))
 * ([TQ] Architecture: the QJL stage removes the inner-product bias). */
void tqo_dequant_k(const tqo_cfg *cfg, const double *signs, const double *S, const uint8_t *row,
                   double *out) {
    const int d = cfg->d, m = cfg->m;
    int *idx = (int *)malloc(sizeof(int) * d);
    int *bit = (int *)malloc(sizeof(int) * m);
    double *w = (double *)malloc(sizeof(double) * d);
    double ns, gamma;
    tqo_unpack_k(cfg, row, idx, bit, &ns, &gamma);
    double sd = sqrt((double)d);
    double cq = sqrt(M_PI / 2.0) / m;
    for (int j = 0; j < d; ++j) {
        double acc = 0.0;
        for (int i = 0; i < m; ++i) acc += S[(int64_t)i * d + j] * (2.0 * bit[i] - 1.0);
        w[j] = ns * cfg->ck[idx[j]] / sd + cq * gamma * acc;
    }
    rot_apply_t(cfg, signs, w, out);
    free(idx); free(bit); free(w);
}

/* ---------------------------------------------------------------- scores -- */

/* Score of one query against T packed keys of one head, evaluated from the
 * codes without decoding (section a9 of the method):
 *   s_t = [ n_s <q_rot, C[idx]>/sqrt(d) + sqrt(pi/2)/m gamma <S q_rot, 2b-1> ] / sqrt(d)
 * ([BP] attention_scores: pre-softmax, scaled by 1/sqrt(head_dim)). */
void tqo_scores_fused(const tqo_cfg *cfg, const double *signs, const double *S, const double *q,
                      const uint8_t *rows, int64_t T, double *scores) {
    const int d = cfg->d, m = cfg->m, rb = tqo_k_row_bytes(cfg);
    double *qr = (double *)malloc(sizeof(double) * d);
    double *sq = (double *)malloc(sizeof(double) * m);
    int *idx = (int *)malloc(sizeof(int) * d);
    int *bit = (int *)malloc(sizeof(int) * m);
    rot_apply(cfg, signs, q, qr);
    for (int i = 0; i < m; ++i) {
        double a = 0.0;
        for (int j = 0; j < d; ++j) a += S[(int64_t)i * d + j] * qr[j];
        sq[i] = a;
    }
    double sd = sqrt((double)d), cq = sqrt(M_PI / 2.0) / m;
    for (int64_t t = 0; t < T; ++t) {
        double ns, gamma;
        tqo_unpack_k(cfg, rows + t * rb, idx, bit, &ns, &gamma);
        double a = 0.0, b = 0.0;
        for (int j = 0; j < d; ++j) a += qr[j] * cfg->ck[idx[j]];
        for (int i = 0; i < m; ++i) b += sq[i] * (2.0 * bit[i] - 1.0);
        scores[t] = (ns * a / sd + cq * gamma * b) / sd;
    }
    free(qr); free(sq); free(idx); free(bit);
}

/* Same scores from the definition: <q, k_hat_t> / sqrt(d). */
void tqo_scores_dequant(const tqo_cfg *cfg, const double *signs, const double *S, const double *q,
                        const uint8_t *rows, int64_t T, double *scores) {
    const int d = cfg->d, rb = tqo_k_row_bytes(cfg);
    double *kh = (double *)malloc(sizeof(double) * d);
    for (int64_t t = 0; t < T; ++t) {
        tqo_dequant_k(cfg, signs, S, rows + t * rb, kh);
        double a = 0.0;
        for (int j = 0; j < d; ++j) a += q[j] * kh[j];
        scores[t] = a / sqrt((double)d);
    }
    free(kh);
}

/* --------------------------------------------------------- decode attention -- */

/* Attention of one query over a concatenation of segments of one head:
 * out = sum_t softmax(s)_t v_hat_t, with s_t = <q, k_hat_t>/sqrt(d), the
 * softmax taken over all tokens of all segments.  Each segment has its own
 * configuration and head tables.  Written directly from the definition:
 * every key and value is dequantized, scores are materialized, the softmax
 * is normalized by its maximum, and the weighted sum is formed. */
void tqo_attend(int nseg, const tqo_cfg *const *cfgs, const double *const *signs,
                const double *const *S, const uint8_t *const *krows, const uint8_t *const *vrows,
                const int64_t *T, const double *q, double *out) {
    int d = cfgs[0]->d;
    int64_t tot = 0;
    for (int s = 0; s < nseg; ++s) tot += T[s];
    for (int j = 0; j < d; ++j) out[j] = 0.0;
    if (tot == 0) return;
    double *sc = (double *)malloc(sizeof(double) * (size_t)tot);
    double *vh = (double *)malloc(sizeof(double) * d);
    int64_t o = 0;
    for (int s = 0; s < nseg; ++s) {
        tqo_scores_dequant(cfgs[s], signs[s], S[s], q, krows[s], T[s], sc + o);
        o += T[s];
    }
    double mx = -INFINITY;
    for (int64_t t = 0; t < tot; ++t) if (sc[t] > mx) mx = sc[t];
    double den = 0.0;
    for (int64_t t = 0; t < tot; ++t) { sc[t] = exp(sc[t] - mx); den += sc[t]; }
    o = 0;
    for (int s = 0; s < nseg; ++s) {
        int rb = tqo_v_row_bytes(cfgs[s]);
        for (int64_t t = 0; t < T[s]; ++t) {
            tqo_dequant_v(cfgs[s], signs[s], vrows[s] + t * rb, vh);
            double p = sc[o + t] / den;
            for (int j = 0; j < d; ++j) out[j] += p * vh[j];
        }
        o += T[s];
    }
    free(sc); free(vh);
}

/* Streaming form of the same softmax-weighted sum over pre-computed scores
 * and values: tokens are consumed in blocks of `blk`; each block keeps a
 * running maximum, a running denominator and a rescaled accumulator, and
 * the blocks are merged by their log-sum-exp.  Used only to check that the
 * streaming softmax equals the materialized one. */
void tqo_streaming_softmax_sum(int64_t T, int d, const double *scores, const double *vals,
                               int64_t blk, double *out) {
    double M = -INFINITY, l = 0.0;
    double *acc = (double *)calloc((size_t)d, sizeof(double));
    double *bacc = (double *)malloc(sizeof(double) * d);
    for (int64_t s = 0; s < T; s += blk) {
        int64_t e = s + blk < T ? s + blk : T;
        double bm = -INFINITY, bl = 0.0;
        for (int j = 0; j < d; ++j) bacc[j] = 0.0;
        for (int64_t t = s; t < e; ++t) {
            if (scores[t] > bm) {
                double f = exp(bm - scores[t]);
                bl *= f;
                for (int j = 0; j < d; ++j) bacc[j] *= f;
                bm = scores[t];
            }
            double p = exp(scores[t] - bm);
            bl += p;
            for (int j = 0; j < d; ++j) bacc[j] += p * vals[t * d + j];
        }
        double nm = bm > M ? bm : M;
        double fa = exp(M - nm), fb = exp(bm - nm);
        l = l * fa + bl * fb;
        for (int j = 0; j < d; ++j) acc[j] = acc[j] * fa + bacc[j] * fb;
        M = nm;
    }
    for (int j = 0; j < d; ++j) out[j] = l > 0.0 ? acc[j] / l : 0.0;
    free(acc); free(bacc);
}

/* Byte counts of the packed formats ([TQ] utils: memory footprint;
 * [BP] compression_ratio = original bytes / compressed bytes). */
int64_t tqo_packed_bytes(const tqo_cfg *cfg, int64_t n_rows) {
    return n_rows * (int64_t)(tqo_k_row_bytes(cfg) + tqo_v_row_bytes(cfg));
}

/* Decode attention of one query q[d_o + d_n] over T tokens of a split cache
 * (R10): group o (channels [0, d_o)) and group n (channels [d_o, d)) with
 * their own configs, rotation tables and packed rows.  Scores from each
 * group's dequantized keys (materialized), one softmax over the token's
 * total score, values concatenated. */
void tqo_attend_split(const tqo_cfg *co, const double *rot_o, const double *S_o, const uint8_t *krows_o,
                      const uint8_t *vrows_o, const tqo_cfg *cn, const double *rot_n, const double *S_n,
                      const uint8_t *krows_n, const uint8_t *vrows_n, int64_t T, const double *q, double *out) {
    const int d_o = co->d, d_n = cn->d, d = d_o + d_n;
    for (int j = 0; j < d; ++j) out[j] = 0.0;
    if (T == 0) return;
    double *sc = (double *)malloc(sizeof(double) * (size_t)T);
    double *kh = (double *)malloc(sizeof(double) * d);
    double *vh = (double *)malloc(sizeof(double) * d);
    const int rko = tqo_k_row_bytes(co), rkn = tqo_k_row_bytes(cn);
    const int rvo = tqo_v_row_bytes(co), rvn = tqo_v_row_bytes(cn);
    for (int64_t t = 0; t < T; ++t) {
        tqo_dequant_k(co, rot_o, S_o, krows_o + t * rko, kh);
        tqo_dequant_k(cn, rot_n, S_n, krows_n + t * rkn, kh + d_o);
        double a = 0.0;
        for (int j = 0; j < d; ++j) a += q[j] * kh[j];
        sc[t] = a / sqrt((double)d);
    }
    double mx = -INFINITY;
    for (int64_t t = 0; t < T; ++t) if (sc[t] > mx) mx = sc[t];
    double den = 0.0;
    for (int64_t t = 0; t < T; ++t) { sc[t] = exp(sc[t] - mx); den += sc[t]; }
    for (int64_t t = 0; t < T; ++t) {
        tqo_dequant_v(co, rot_o, vrows_o + t * rvo, vh);
        tqo_dequant_v(cn, rot_n, vrows_n + t * rvn, vh + d_o);
        const double p = sc[t] / den;
        for (int j = 0; j < d; ++j) out[j] += p * vh[j];
    }
    free(sc); free(kh); free(vh);
}
