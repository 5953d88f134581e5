// tq_tables.cpp -- host-side construction of a context's constant tables.
//
//  * Per-head random tables (bitpolar src/kv_cache.rs, MultiHeadKvCache::new:
//    head h uses seed.wrapping_add(h)).  The generator is SplitMix64 (Steele,
//    Lea, Flood 2014).  The first d outputs give the rotation's random signs
//    (top bit set -> -1); the following m*d values come in Box-Muller pairs
//    and fill the QJL matrix S row-major [m][d], each rounded to binary16
//    (nearest, ties to even) -- the rounded value is the matrix the codec
//    uses, which also makes it exact as a tensor-core operand.
//  * Haar rotations (turboquant-plus-rs README, Modules: rotation, which
//    names a Haar-random rotation built from a QR factorization): Q = the
//    orthogonal factor of the
//    QR factorization of a d x d Gaussian matrix G with R's diagonal
//    positive.  G's entries are Box-Muller pairs continuing head h's stream
//    after the sign and S draws.  The factorization here is Gram-Schmidt run
//    twice per column (its R diagonal is a norm, hence positive), in fp64.
//  * Lloyd-Max codebooks of N(0,1) (turboquant-plus-rs README, Modules:
//    codebook -- MSE-optimal centroids, given in closed form at 1 and 2 bits
//    and found by Lloyd iteration from 3 bits up): the iteration runs on the
//    positive half-line,
//    using the codebook's symmetry, to |change| < 1e-15.
//
// Compiled by the host C++ compiler (not nvcc) with contraction off so the
// double-precision Box-Muller values are the plain IEEE results.
#include <cmath>
#include <cstdint>
#include <cstring>

namespace {

struct SplitMix64 {
    uint64_t s;
    uint64_t next() {
        s += 0x9E3779B97F4A7C15ull;
        uint64_t z = s;
        z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
        z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
        return z ^ (z >> 31);
    }
};

uint16_t to_binary16_bits(double v) {
    _Float16 h = (_Float16)v;      // direct double -> binary16, round to nearest even
    uint16_t bits;
    std::memcpy(&bits, &h, 2);
    return bits;
}

double gauss_pdf(double x) { return std::exp(-0.5 * x * x) * 0.398942280401432677939946059934; }
double upper_tail(double x) { return 0.5 * std::erfc(x * 0.707106781186547524400844362105); }

}  // namespace

extern "C" __attribute__((visibility("hidden"))) void tq_host_head_tables(int d, int m, uint64_t seed, int h, uint32_t *sign_words,
                                    uint16_t *S_bits) {
    SplitMix64 g{seed + (uint64_t)(int64_t)h};
    for (int w = 0; w < d / 32; ++w) sign_words[w] = 0;
    for (int j = 0; j < d; ++j)
        if (g.next() >> 63) sign_words[j / 32] |= 1u << (j % 32);
    const int64_t total = (int64_t)m * d;
    for (int64_t i = 0; i < total; i += 2) {
        const uint64_t a = g.next(), b = g.next();
        const double u1 = (double)((a >> 11) + 1) * 0x1.0p-53;
        const double u2 = (double)(b >> 11) * 0x1.0p-53;
        const double rad = std::sqrt(-2.0 * std::log(u1));
        const double ang = 2.0 * M_PI * u2;
        S_bits[i] = to_binary16_bits(rad * std::cos(ang));
        if (i + 1 < total) S_bits[i + 1] = to_binary16_bits(rad * std::sin(ang));
    }
}

extern "C" __attribute__((visibility("hidden"))) void tq_host_haar(int d, int m, uint64_t seed, int h, double *Q) {
    SplitMix64 g{seed + (uint64_t)(int64_t)h};
    for (int j = 0; j < d; ++j) g.next();                    // rotation signs
    const int64_t sdraws = (int64_t)m * d + (((int64_t)m * d) & 1);
    for (int64_t i = 0; i < sdraws; ++i) g.next();            // S, drawn in pairs
    const int64_t n = (int64_t)d * d;
    double *G = new double[n];
    for (int64_t i = 0; i < n; i += 2) {
        const uint64_t a = g.next(), b = g.next();
        const double u1 = (double)((a >> 11) + 1) * 0x1.0p-53;
        const double u2 = (double)(b >> 11) * 0x1.0p-53;
        const double rad = std::sqrt(-2.0 * std::log(u1));
        const double ang = 2.0 * M_PI * u2;
        G[i] = rad * std::cos(ang);
        if (i + 1 < n) G[i + 1] = rad * std::sin(ang);
    }
    double *v = new double[d];
    for (int k = 0; k < d; ++k) {
        for (int i = 0; i < d; ++i) v[i] = G[(int64_t)i * d + k];
        for (int pass = 0; pass < 2; ++pass)
            for (int c = 0; c < k; ++c) {
                double r = 0.0;
                for (int i = 0; i < d; ++i) r += Q[(int64_t)i * d + c] * v[i];
                for (int i = 0; i < d; ++i) v[i] -= r * Q[(int64_t)i * d + c];
            }
        double nv = 0.0;
        for (int i = 0; i < d; ++i) nv += v[i] * v[i];
        nv = std::sqrt(nv);
        for (int i = 0; i < d; ++i) Q[(int64_t)i * d + k] = v[i] / nv;
    }
    delete[] v;
    delete[] G;
}

// Centroids c[L] (ascending) and boundaries beta[L-1] of the 2^B-level
// Lloyd-Max quantizer of N(0,1), rounded to float.  Returns L (0 on bad B).
extern "C" __attribute__((visibility("hidden"))) int tq_host_codebook(int B, float *c, float *beta) {
    if (B < 1 || B > 5) return 0;
    const int L = 1 << B, H = L / 2;
    double mag[16], edge[17];
    if (B == 1) {
        mag[0] = std::sqrt(2.0 / M_PI);
    } else {
        for (int k = 0; k < H; ++k) mag[k] = 2.0 * (2 * k + 1) / (L - 1);
        for (int it = 0; it < 1000000; ++it) {
            edge[0] = 0.0;
            for (int k = 1; k < H; ++k) edge[k] = 0.5 * (mag[k - 1] + mag[k]);
            double worst = 0.0;
            for (int k = 0; k < H; ++k) {
                const double a = edge[k];
                const bool last = (k == H - 1);
                const double pa = gauss_pdf(a), pb = last ? 0.0 : gauss_pdf(edge[k + 1]);
                const double qa = upper_tail(a), qb = last ? 0.0 : upper_tail(edge[k + 1]);
                const double nm = (pa - pb) / (qa - qb);
                worst = std::fmax(worst, std::fabs(nm - mag[k]));
                mag[k] = nm;
            }
            if (worst < 1e-15) break;
        }
    }
    for (int k = 0; k < H; ++k) {
        c[H + k] = (float)mag[k];
        c[H - 1 - k] = (float)-mag[k];
    }
    for (int k = 0; k < L - 1; ++k) {
        double lo = (k < H) ? -mag[H - 1 - k] : mag[k - H];
        double hi = (k + 1 < H) ? -mag[H - 2 - k] : mag[k + 1 - H];
        beta[k] = (float)(0.5 * (lo + hi));
    }
    beta[H - 1] = 0.0f;
    return L;
}
