// tq_encode.cu -- TurboQuant encode of keys and values (sm_100a).
//
// Method (turboquant-plus-rs 0.1.0 README, "Architecture"; "Modules":
// rotation, codebook, polar_quant with norm extraction and correction, qjl,
// utils/bit packing):
//   n = |x|;  u = H (D x)  (Sylvester Walsh-Hadamard, random signs D);
//   z = u / n;  idx_j = #{k : z_j >= beta_k}   (Lloyd-Max boundaries);
//   n_s = n / |C[idx]/sqrt(d)|                  (norm correction);
//   keys: r = (u - n_s C[idx]) / sqrt(d), gamma = |r|, bit_i = [<S_i, r> >= 0].
// Keys use b-1 index bits, values b bits (values are MSE-only).
//
// Kernel design: one thread per row, CTAs of 128 threads (one 128-row tile
// at a time, ENC_TILES tiles per CTA, all of one (batch, head)).  Keys and
// values are separate kernels.  A row is processed in 32-coordinate chunks,
// with the thread's TMEM lane as scratch (Blackwell tensor memory: 128 lanes
// x up to 512 32-bit columns per SM):
//   A. per chunk: 128-bit loads of the 32 inputs with the rotation's signs
//      applied to the packed words, the five butterfly stages inside the
//      chunk in registers, one tcgen05.st of the chunk to its TMEM columns;
//   B. the remaining butterfly stages (across chunks) on 8-column slices
//      read back from TMEM, accumulating |u|^2 (= d |x|^2);
//   C. per chunk: quantization of z = u / n by a binary search over the
//      positive boundaries (pre-scaled by n) done on pairs of coordinates in
//      packed fp32x2 arithmetic, each level's decision bit gathered from the
//      sign of |u| - boundary with a funnel shift; bit-plane (keys) or
//      bit-field (values) packing; sum C[idx]^2 from per-cell counts
//      (popcounts of the level words), sum |u| C[idx] (keys);
//   D. keys (the signed centroids kept in TMEM columns [d, 2d) by C): the
//      residual u - n_s C[idx], scaled to |e| ~ sqrt(d) and split
//      into binary16 hi + lo, written to shared memory in the 128-byte
//      swizzled K-major layout; one thread issues 2*(d/16) tcgen05.mma
//      (M = 128 rows, N = m projections, K = 16) against S (binary16, loaded
//      once per CTA by TMA), accumulating P = e S^T in fp32 in TMEM columns
//      [d, d + m); while it runs, the threads rotate the next tile into
//      columns [0, d).  Two passes make the projection accurate
//      to ~1e-7 relative, so sign bits agree with an fp64 evaluation away
//      from |p| ~ 1e-6.  Each thread then reads its row of P (tcgen05.ld)
//      and stores the m-bit sign plane.
// Small unrolled bodies and few live registers keep the instruction cache
// and the warp scheduler busy; DRAM traffic is the inputs read once plus the
// packed rows written once.  Rows whose rotated sum of squares d |x|^2
// overflows fp32 (|x| beyond ~1.5e18) are counted as non-finite; rows where
// it falls below the smallest normal float (|x| below ~1e-20) are encoded as
// zero rows (the exact search steps need normal-range boundaries).
#include <algorithm>
#include <cstdlib>
#include <type_traits>

#include "tq_internal.cuh"

namespace {

constexpr int ENC_ROWS = 128;    // threads per CTA = rows per tile = MMA M
constexpr int ENC_TILES = 4;     // tiles per CTA (S is loaded once per CTA)

struct EncodeParams {
    const void *x;          // keys or values
    int64_t sb, sh, st;     // input strides in elements
    uint8_t *out;           // packed rows of this side
    int64_t capacity, token_offset, T;
    int H;
    int row_bytes;
    int M;
    int64_t blocks_per_bh;
    const uint32_t *signs;  // [heads][d/32]
    unsigned long long *status;
    float mag[16];          // positive-half centroid magnitudes
    float pb[16];           // positive boundaries
    float cl[8];            // keys: centroid magnitude as a multilinear form in the search bits
    int norm_f16;           // keys: n_s and gamma as binary16 in one word
};

// ------------------------------------------------------------- row loading
// Chunk loaders: 32 consecutive elements, the rotation's random signs applied
// to the packed words (mask words hold the sign bit of every flipped element:
// bits 15/31 for 16-bit types, bit 31 for fp32).
template <typename Tin>
struct Chunk;

template <>
struct Chunk<float> {
    static constexpr int MASK_WORDS = 32;
    __device__ static void load(const float *src, const uint32_t *sm, float (&x)[32]) {
        const uint4 *p = reinterpret_cast<const uint4 *>(src);
        const uint4 *m = reinterpret_cast<const uint4 *>(sm);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint4 q = __ldg(p + i), f = m[i];
            x[4 * i] = __uint_as_float(q.x ^ f.x);
            x[4 * i + 1] = __uint_as_float(q.y ^ f.y);
            x[4 * i + 2] = __uint_as_float(q.z ^ f.z);
            x[4 * i + 3] = __uint_as_float(q.w ^ f.w);
        }
    }
};

template <>
struct Chunk<__half> {
    static constexpr int MASK_WORDS = 16;
    __device__ static void load(const __half *src, const uint32_t *sm, float (&x)[32]) {
        const uint4 *p = reinterpret_cast<const uint4 *>(src);
        const uint4 *m = reinterpret_cast<const uint4 *>(sm);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 q = __ldg(p + i), f = m[i];
            const uint32_t w[4] = {q.x ^ f.x, q.y ^ f.y, q.z ^ f.z, q.w ^ f.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 v = __half22float2(__halves2half2(__ushort_as_half((unsigned short)(w[e] & 0xFFFFu)),
                                                               __ushort_as_half((unsigned short)(w[e] >> 16))));
                x[8 * i + 2 * e] = v.x;
                x[8 * i + 2 * e + 1] = v.y;
            }
        }
    }
};

template <>
struct Chunk<__nv_bfloat16> {
    static constexpr int MASK_WORDS = 16;
    __device__ static void load(const __nv_bfloat16 *src, const uint32_t *sm, float (&x)[32]) {
        const uint4 *p = reinterpret_cast<const uint4 *>(src);
        const uint4 *m = reinterpret_cast<const uint4 *>(sm);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 q = __ldg(p + i), f = m[i];
            const uint32_t w[4] = {q.x ^ f.x, q.y ^ f.y, q.z ^ f.z, q.w ^ f.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                x[8 * i + 2 * e] = __uint_as_float(w[e] << 16);
                x[8 * i + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
            }
        }
    }
};

// The same conversion from 16-byte words already in registers (16-bit
// types: 4 words per chunk).
template <typename Tin>
__device__ __forceinline__ void chunk_from_words(const uint4 *q4, const uint32_t *sm, float (&x)[32]) {
    static_assert(sizeof(Tin) == 2, "16-bit inputs");
    const uint4 *m = reinterpret_cast<const uint4 *>(sm);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 q = q4[i], f = m[i];
        const uint32_t w[4] = {q.x ^ f.x, q.y ^ f.y, q.z ^ f.z, q.w ^ f.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if constexpr (std::is_same<Tin, __half>::value) {
                const float2 v = __half22float2(__halves2half2(__ushort_as_half((unsigned short)(w[e] & 0xFFFFu)),
                                                               __ushort_as_half((unsigned short)(w[e] >> 16))));
                x[8 * i + 2 * e] = v.x;
                x[8 * i + 2 * e + 1] = v.y;
            } else {
                x[8 * i + 2 * e] = __uint_as_float(w[e] << 16);
                x[8 * i + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
            }
        }
    }
}

// One 16-bit input row as 16-byte words, loaded ahead of its rotation so
// the load latency overlaps the previous tile's work.
template <int D>
struct RowWords {
    uint4 w[D / 8];
};
template <int D, typename Tin>
__device__ __forceinline__ void load_row_words(const Tin *row, bool valid, RowWords<D> &r) {
    const uint4 *p = reinterpret_cast<const uint4 *>(row);
#pragma unroll
    for (int i = 0; i < D / 8; ++i) r.w[i] = valid ? __ldg(p + i) : make_uint4(0u, 0u, 0u, 0u);
}

// Per-head input sign masks, in input-word order.
template <typename Tin, int D>
__device__ void build_sign_masks(const uint32_t *signs, uint32_t *sm) {
    constexpr int MW = Chunk<Tin>::MASK_WORDS * (D / 32);
    for (int w = threadIdx.x; w < MW; w += blockDim.x) {
        if constexpr (sizeof(Tin) == 4) {
            sm[w] = ((signs[w / 32] >> (w % 32)) & 1u) << 31;
        } else {
            const int j = 2 * w;
            sm[w] = (((signs[j / 32] >> (j % 32)) & 1u) << 15) | (((signs[(j + 1) / 32] >> ((j + 1) % 32)) & 1u) << 31);
        }
    }
}

// In-register Walsh-Hadamard butterflies over 32 values (strides 1..16).
// Strides 2..16 pair (x[j], x[j+1]) with (x[j+len], x[j+len+1]), so they run
// as packed fp32x2 adds / subtracts; stride 1 is done with scalar ops.
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    uint64_t r;
    asm("{\n\t.reg .b64 ra, rb;\n\t"
        "mov.b64 ra, {%1, %2};\n\t"
        "mov.b64 rb, {%3, %4};\n\t"
        "add.rn.f32x2 %0, ra, rb;\n\t}"
        : "=l"(r)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return make_float2(__uint_as_float((uint32_t)r), __uint_as_float((uint32_t)(r >> 32)));
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    uint64_t r;
    asm("{\n\t.reg .b64 ra, rb;\n\t"
        "mov.b64 ra, {%1, %2};\n\t"
        "mov.b64 rb, {%3, %4};\n\t"
        "sub.rn.f32x2 %0, ra, rb;\n\t}"
        : "=l"(r)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return make_float2(__uint_as_float((uint32_t)r), __uint_as_float((uint32_t)(r >> 32)));
}

__device__ __forceinline__ void fwht32(float (&x)[32]) {
    float2 P[16];   // P[k] = (x[2k], x[2k+1]) after the stride-1 stage
#pragma unroll
    for (int k = 0; k < 16; ++k) P[k] = make_float2(x[2 * k] + x[2 * k + 1], x[2 * k] - x[2 * k + 1]);
#pragma unroll
    for (int h = 1; h < 16; h <<= 1) {          // stride 2h in x, h in P
#pragma unroll
        for (int i = 0; i < 16; i += 2 * h) {
#pragma unroll
            for (int k = i; k < i + h; ++k) {
                const float2 a = P[k], b = P[k + h];
                P[k] = add2(a, b);
                P[k + h] = sub2(a, b);
            }
        }
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        x[2 * k] = P[k].x;
        x[2 * k + 1] = P[k].y;
    }
}

// Magnitude index of a = |u| among the HB cells of the positive half of the
// codebook: the number of positive boundaries nb[k] (pre-scaled by n) with
// a >= nb[k], found by a branchless binary search.  Used for 16 cells (5-bit
// values); fewer cells go through the packed search below.
template <int HB>
__device__ __forceinline__ uint32_t mag_index(float a, const float (&nb)[16]) {
    static_assert(HB == 16, "the compare-and-select search serves 16 cells");
    const bool t3 = a >= nb[7];
    const bool t2 = a >= (t3 ? nb[11] : nb[3]);
    const bool t1 = a >= (t3 ? (t2 ? nb[13] : nb[9]) : (t2 ? nb[5] : nb[1]));
    const float b0 = t3 ? (t2 ? (t1 ? nb[14] : nb[12]) : (t1 ? nb[10] : nb[8]))
                        : (t2 ? (t1 ? nb[6] : nb[4]) : (t1 ? nb[2] : nb[0]));
    const bool t0 = a >= b0;
    return (t3 ? 8u : 0u) | (t2 ? 4u : 0u) | (t1 ? 2u : 0u) | (t0 ? 1u : 0u);
}

// ------------------------------------------------------ packed quantization
// For up to 8 cells per half the binary search runs on pairs of coordinates
// in packed fp32x2 arithmetic (FMA pipe) instead of compares and selects:
// level L tests d_L = |u| - b_L >= 0, where b_L is the boundary chosen by the
// levels above; T_L = [d_L >= 0] in {0, 1} is saturate(d_L * 2^126 + 1) and
// selects the next boundary with one fused multiply-add.  The magnitude
// index is sum_L T_L 2^L; bit L of every coordinate of a 32-coordinate chunk
// is collected from the sign of d_L with one funnel shift.
__device__ __forceinline__ float2 dup2(float a) { return make_float2(a, a); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }

// [d >= 0] as 0.0 or 1.0, exact for d = 0 and |d| >= 2^-126; NaN gives 0.
__device__ __forceinline__ float step01(float d) {
    float r;
    asm("fma.rn.sat.f32 %0, %1, 0f7E800000, 0f3F800000;" : "=f"(r) : "f"(d));
    return r;
}
__device__ __forceinline__ float2 step2(float2 d) { return make_float2(step01(d.x), step01(d.y)); }

// Shift the sign bit of x into the bottom of w (coordinates are visited from
// 31 down to 0, so coordinate i ends at bit i).
__device__ __forceinline__ uint32_t push_sign(uint32_t w, float x) { return __funnelshift_l(__float_as_uint(x), w, 1); }

template <int HB>
struct Levels {
    static constexpr int L = HB == 1 ? 0 : HB == 2 ? 1 : HB == 4 ? 2 : 3;
};

// Row boundaries of the search (scaled by the row norm n), in the order the
// levels use them.
template <int HB>
__device__ __forceinline__ void row_bounds(float n, const float (&pb)[16], float (&rb)[8]) {
    float nb[8];
#pragma unroll
    for (int k = 0; k < HB - 1; ++k) nb[k] = n * pb[k];
    if constexpr (HB == 2) {
        rb[0] = nb[0];
    } else if constexpr (HB == 4) {
        rb[0] = nb[1];
        rb[1] = nb[2] - nb[0];
        rb[2] = nb[0];
    } else if constexpr (HB == 8) {
        rb[0] = nb[3];
        rb[1] = nb[5] - nb[1];
        rb[2] = nb[1];
        rb[3] = (nb[6] - nb[4]) - (nb[2] - nb[0]);
        rb[4] = nb[2] - nb[0];
        rb[5] = nb[4] - nb[0];
        rb[6] = nb[0];
    }
}

// The search for one pair of magnitudes A; T[L] and d[L] per level.
template <int HB>
__device__ __forceinline__ void search2(float2 A, const float (&rb)[8], float2 (&T)[3], float2 (&d)[3]) {
    if constexpr (HB == 2) {
        d[0] = sub2(A, dup2(rb[0]));
        T[0] = step2(d[0]);
    } else if constexpr (HB == 4) {
        d[1] = sub2(A, dup2(rb[0]));
        T[1] = step2(d[1]);
        d[0] = sub2(A, fma2(T[1], dup2(rb[1]), dup2(rb[2])));
        T[0] = step2(d[0]);
    } else if constexpr (HB == 8) {
        d[2] = sub2(A, dup2(rb[0]));
        T[2] = step2(d[2]);
        d[1] = sub2(A, fma2(T[2], dup2(rb[1]), dup2(rb[2])));
        T[1] = step2(d[1]);
        const float2 b0 = fma2(T[1], fma2(T[2], dup2(rb[3]), dup2(rb[4])), fma2(T[2], dup2(rb[5]), dup2(rb[6])));
        d[0] = sub2(A, b0);
        T[0] = step2(d[0]);
    }
}

// Number of coordinates of a chunk in each magnitude cell k = sum_L T_L 2^L,
// from the per-level sign words S[L] (bit set = T_L is 0); cell 0 is implied.
template <int HB>
__device__ __forceinline__ void count_cells(const uint32_t (&S)[3], int (&cnt)[8]) {
#pragma unroll
    for (int k = 1; k < HB; ++k) {
        uint32_t w = ~0u;
#pragma unroll
        for (int l = 0; l < Levels<HB>::L; ++l) w &= ((k >> l) & 1) ? ~S[l] : S[l];
        cnt[k] += __popc(w);
    }
}

// Packed-input words of the degenerate value row: every B-bit field = 2^(B-1).
template <int B>
__host__ __device__ constexpr uint32_t degenerate_field_word(int w) {
    uint32_t r = 0;
    for (int b = 0; b < 32; ++b) {
        const int bit = 32 * w + b;
        if (((1 << (B - 1)) >> (bit % B)) & 1) r |= 1u << b;
    }
    return r;
}

// Phases A and B: the row's rotation u = H (D x) into TMEM columns [0, D) of
// this thread's lane; returns |u|^2.  Rows past the end rotate zeros.
template <int D>
__device__ __forceinline__ float cross_chunk_stages(uint32_t tlane);

template <int D, typename Tin>
__device__ __forceinline__ float rotate_row_to_tmem(const Tin *row, bool valid, const uint32_t *s_mask,
                                                    uint32_t tlane) {
    constexpr int NC = D / 32;
#pragma unroll 1
    for (int c = 0; c < NC; ++c) {
        float v[32];
        if (valid) {
            Chunk<Tin>::load(row + 32 * c, s_mask + c * Chunk<Tin>::MASK_WORDS, v);
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.f;
        }
        fwht32(v);
        tqdev::tmem_st_32x32b_x32(tlane + 32 * c, v);
    }
    return cross_chunk_stages<D>(tlane);
}

// The same from a row already in registers (16-bit inputs; invalid rows were
// loaded as zeros).
template <int D, typename Tin>
__device__ __forceinline__ float rotate_words_to_tmem(const RowWords<D> &r, const uint32_t *s_mask,
                                                      uint32_t tlane) {
    constexpr int NC = D / 32;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        float v[32];
        chunk_from_words<Tin>(r.w + 4 * c, s_mask + c * Chunk<Tin>::MASK_WORDS, v);
        fwht32(v);
        tqdev::tmem_st_32x32b_x32(tlane + 32 * c, v);
    }
    return cross_chunk_stages<D>(tlane);
}

// Phase B: the butterfly stages across chunks, on 8-column slices; returns |u|^2.
template <int D>
__device__ __forceinline__ float cross_chunk_stages(uint32_t tlane) {
    constexpr int NC = D / 32;
    tqdev::tmem_wait_st();
    float2 n2p = make_float2(0.f, 0.f);
#pragma unroll 1
    for (int g = 0; g < 4; ++g) {
        float w[NC][8];
#pragma unroll
        for (int c = 0; c < NC; ++c) tqdev::tmem_ld_32x32b_x8_nowait(tlane + 32 * c + 8 * g, w[c]);
        tqdev::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
#pragma unroll
            for (int len = 1; len < NC; len <<= 1)
#pragma unroll
                for (int c = 0; c < NC; c += 2 * len)
#pragma unroll
                    for (int cc = c; cc < c + len; ++cc) {
                        const float2 a = make_float2(w[cc][i], w[cc][i + 1]);
                        const float2 b = make_float2(w[cc + len][i], w[cc + len][i + 1]);
                        const float2 s0 = add2(a, b), s1 = sub2(a, b);
                        w[cc][i] = s0.x;
                        w[cc][i + 1] = s0.y;
                        w[cc + len][i] = s1.x;
                        w[cc + len][i + 1] = s1.y;
                    }
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                const float2 wc = make_float2(w[c][i], w[c][i + 1]);
                n2p = fma2(wc, wc, n2p);
            }
        }
#pragma unroll
        for (int c = 0; c < NC; ++c) tqdev::tmem_st_32x32b_x8(tlane + 32 * c + 8 * g, w[c]);
    }
    tqdev::tmem_wait_st();
    return n2p.x + n2p.y;
}

__host__ __device__ constexpr uint32_t tmem_cols_for(int cols) {
    return cols <= 32 ? 32u : cols <= 64 ? 64u : cols <= 128 ? 128u : cols <= 256 ? 256u : 512u;
}

// ------------------------------------------------- dense (Haar) rotation
// The Haar rotation u = sqrt(d) Q x runs on the tensor cores: each thread
// writes its row, scaled by 2^e so that max_j |x_j| lies in [2^14, 2^15), as
// binary16 into the 128-byte-swizzled K-major operand layout (16-byte unit kk
// of row r at (kk / 8) * ATOM + r * 128 + ((kk % 8) ^ (r % 8)) * 16); the
// scaling is a power of two, so binary16 and bfloat16 rows are exact (up to
// binary16 subnormals below 2^-14 of the row maximum) and float32 rows are
// split into hi + lo.  The MMA against sqrt(d) Q (binary16 hi + lo) leaves
// 2^e u in TMEM; quantization is scale-free, and the stored norms are
// multiplied back by 2^-e.
struct DenseRow {
    float n2;          // d |2^e x|^2 = |2^e u|^2
    float inv_scale;   // 2^-e
    bool nonfinite;    // some x_j is Inf or NaN
    bool zero;         // zero operand: non-finite, all zero, or max |x_j| < 2^-100 (or past the end)
};

template <typename Tin>
__device__ __forceinline__ float2 word_to_float2(uint32_t w) {
    if constexpr (std::is_same<Tin, __half>::value)
        return __half22float2(*reinterpret_cast<const __half2 *>(&w));
    else
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

template <int D, typename Tin>
__device__ __forceinline__ DenseRow stage_dense_row(const RowWords<D> &raw, const Tin *rowp, bool valid, int r,
                                                    uint8_t *xHi, uint8_t *xLo) {
    constexpr int ATOM = ENC_ROWS * 128;
    constexpr bool H16 = sizeof(Tin) == 2;
    DenseRow out;
    float mx = 0.f;
    bool bad = false;
    if constexpr (H16) {
        uint32_t mb = 0u;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            const uint4 q = raw.w[i];
            mb = __vmaxu2(mb, q.x & 0x7FFF7FFFu);
            mb = __vmaxu2(mb, q.y & 0x7FFF7FFFu);
            mb = __vmaxu2(mb, q.z & 0x7FFF7FFFu);
            mb = __vmaxu2(mb, q.w & 0x7FFF7FFFu);
        }
        const uint32_t m16 = max(mb & 0xFFFFu, mb >> 16);
        if constexpr (std::is_same<Tin, __half>::value) {
            bad = m16 >= 0x7C00u;
            mx = __half2float(__ushort_as_half((unsigned short)m16));
        } else {
            bad = m16 >= 0x7F80u;
            mx = __uint_as_float(m16 << 16);
        }
    } else if (valid) {
        uint32_t mb = 0u;
        const uint4 *p4 = reinterpret_cast<const uint4 *>(rowp);
#pragma unroll 4
        for (int i = 0; i < D / 4; ++i) {
            const uint4 q = __ldg(p4 + i);
            mb = max(mb, max(max(q.x & 0x7FFFFFFFu, q.y & 0x7FFFFFFFu), max(q.z & 0x7FFFFFFFu, q.w & 0x7FFFFFFFu)));
        }
        bad = mb >= 0x7F800000u;
        mx = __uint_as_float(mb);
    }
    if (!valid) {
        bad = false;
        mx = 0.f;
    }
    out.nonfinite = bad;
    out.zero = bad || !(mx >= 0x1p-100f);
    const int ex = (int)((__float_as_uint(mx) >> 23) & 0xFFu) - 127;
    const int e = out.zero ? 0 : 14 - ex;               // in [-113, 114]
    const float sc = __uint_as_float((uint32_t)(e + 127) << 23);
    out.inv_scale = __uint_as_float((uint32_t)(127 - e) << 23);
    float2 acc = make_float2(0.f, 0.f);
#pragma unroll 4
    for (int kk = 0; kk < D / 8; ++kk) {
        float v[8];
        if constexpr (H16) {
            const uint4 q = raw.w[kk];
            const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
                const float2 f = word_to_float2<Tin>(w4[e2]);
                v[2 * e2] = f.x;
                v[2 * e2 + 1] = f.y;
            }
        } else {
            if (valid) {
                const float4 a = __ldg(reinterpret_cast<const float4 *>(rowp) + 2 * kk);
                const float4 b2 = __ldg(reinterpret_cast<const float4 *>(rowp) + 2 * kk + 1);
                v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
                v[4] = b2.x; v[5] = b2.y; v[6] = b2.z; v[7] = b2.w;
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = 0.f;
            }
        }
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
            const float2 a = out.zero ? make_float2(0.f, 0.f) : mul2(make_float2(v[2 * e2], v[2 * e2 + 1]), dup2(sc));
            acc = fma2(a, a, acc);
            const __half2 hh = __floats2half2_rn(a.x, a.y);
            hw[e2] = *reinterpret_cast<const uint32_t *>(&hh);
            if constexpr (!H16) {
                const float2 l = sub2(a, __half22float2(hh));
                const __half2 ll = __floats2half2_rn(l.x, l.y);
                lw[e2] = *reinterpret_cast<const uint32_t *>(&ll);
            }
        }
        const int off = (kk / 8) * ATOM + r * 128 + (((kk % 8) ^ (r & 7)) << 4);
        *reinterpret_cast<uint4 *>(xHi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        if constexpr (!H16) *reinterpret_cast<uint4 *>(xLo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    out.n2 = (acc.x + acc.y) * (float)D;
    return out;
}

// Issued by one thread: 2^e u = X (sqrt(d) Q)^T into TMEM columns [0, d):
// passes (X hi, Q hi), (X hi, Q lo) and, for float32 rows, (X lo, Q hi).
template <int D, typename Tin>
__device__ __forceinline__ void issue_dense_rotation(uint32_t tmem_base, const uint8_t *xHi, const uint8_t *xLo,
                                                     const uint8_t *sQ, uint64_t *bar) {
    constexpr int ATOM = ENC_ROWS * 128;
    constexpr int PASSES = sizeof(Tin) == 2 ? 2 : 3;
    const uint32_t idesc = tqdev::idesc_f16_f32(D);
#pragma unroll
    for (int pass = 0; pass < PASSES; ++pass) {
        const uint32_t abase = tqdev::smem_u32(pass == 2 ? xLo : xHi);
        const uint32_t bbase = tqdev::smem_u32(sQ + (pass == 1 ? (D / 64) * D * 128 : 0));
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t a_addr = abase + (ks / 4) * ATOM + (ks % 4) * 32;
            const uint32_t b_addr = bbase + (ks / 4) * (D * 128) + (ks % 4) * 32;
            tqdev::mma_f16_ss(tmem_base, tqdev::smem_desc_sw128(a_addr), tqdev::smem_desc_sw128(b_addr), idesc,
                              (pass | ks) != 0);
        }
    }
    tqdev::mma_commit(bar);
}

// TMA of head h's two binary16 pieces of sqrt(d) Q into sQ [2][d/64][d][128 B].
template <int D>
__device__ __forceinline__ void load_q_tiles(uint8_t *sQ, const CUtensorMap *tmapQ, int head, uint64_t *bar) {
    tqdev::mbar_expect_tx(bar, (uint32_t)(2 * D * D * 2));
#pragma unroll
    for (int piece = 0; piece < 2; ++piece)
#pragma unroll
        for (int a = 0; a < D / 64; ++a)
            tqdev::tma_load_2d(sQ + (piece * (D / 64) + a) * D * 128, tmapQ, a * 64, (head * 2 + piece) * D, bar);
}

// ------------------------------------------------------------------ values
// ROT: 0 = Walsh-Hadamard rotation in registers and TMEM; 1 = dense (Haar)
// rotation on the tensor cores.
template <int D, int BV, typename Tin, int ROT>
__global__ void __launch_bounds__(ENC_ROWS) tq_encode_v_kernel(const __grid_constant__ EncodeParams p,
                                                               const __grid_constant__ CUtensorMap tmapQ) {
    constexpr int HV = (1 << BV) / 2;
    constexpr int NC = D / 32;
    constexpr uint32_t FMASK = (1u << BV) - 1u;
    constexpr int ATOM = ENC_ROWS * 128;
    __shared__ __align__(16) uint32_t s_mask[Chunk<Tin>::MASK_WORDS * NC];
    __shared__ float s_mag2[16];
    __shared__ uint32_t s_tmem;
    // dense rotation only: [sQ: 2 x d/64 x d x 128 B][X: pieces x d/64 x ATOM], 1024-aligned
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t s_bars[2];    // [0] Q loaded, [1] rotation MMA done
    __shared__ int s_abort;
    uint8_t *sQ = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *xHi = sQ + 2 * (D / 64) * D * 128;
    uint8_t *xLo = xHi + (D / 64) * ATOM;
    const int tid = threadIdx.x, warp = tid / 32;
    const int64_t blk = blockIdx.x;
    const int64_t bh = blk / p.blocks_per_bh;
    const int head = (int)(bh % p.H);
    const int64_t b = bh / p.H;
    const int64_t tb0 = (blk % p.blocks_per_bh) * (int64_t)ENC_TILES * ENC_ROWS;
    build_sign_masks<Tin, D>(p.signs + (int64_t)head * (D / 32), s_mask);
    if (tid < 16) s_mag2[tid] = tid < HV ? p.mag[tid] * p.mag[tid] : 0.f;
    if constexpr (ROT == 1) {
        if (tid == 0) {
            tqdev::mbar_init(&s_bars[0], 1);
            tqdev::mbar_init(&s_bars[1], 1);
            s_abort = tqdev::status_aborted(p.status) ? 1 : 0;
            tqdev::fence_barrier_init();
        }
    }
    if (warp == 0) tqdev::tmem_alloc(&s_tmem, tmem_cols_for(D));
    tqdev::tc_fence_before();
    __syncthreads();
    tqdev::tc_fence_after();
    const uint32_t tlane = s_tmem + ((uint32_t)(warp * 32) << 16);
    const Tin *src = reinterpret_cast<const Tin *>(p.x) + b * p.sb + (int64_t)head * p.sh;
    bool q_pending = false;   // thread 0: Q tiles requested, not yet seen
    int rot_drain = -1;       // phase of a rotation MMA not seen complete
    if constexpr (ROT == 1) {
        if (tid == 0 && !s_abort) {
            load_q_tiles<D>(sQ, &tmapQ, head, &s_bars[0]);
            q_pending = true;
        }
    }
    // 16-bit inputs: each tile's rows are loaded into registers during the
    // previous tile's quantization (d <= 128: a d = 256 row is 128 registers)
    constexpr bool PF = sizeof(Tin) == 2 && D <= 128;
    RowWords<D> raw;
    if constexpr (PF) {
        if (tb0 < p.T) load_row_words<D, Tin>(src + (tb0 + tid) * p.st, tb0 + tid < p.T, raw);
    }
#pragma unroll 1
    for (int tile = 0; tile < ENC_TILES; ++tile) {
        const int64_t t0 = tb0 + tile * ENC_ROWS;
        if (t0 >= p.T) break;
        const int64_t t = t0 + tid;
        const bool valid = t < p.T;
        float n2, inv_scale = 1.f;
        bool nonfinite, degenerate;
        if constexpr (ROT == 1) {
            const DenseRow dr = stage_dense_row<D, Tin>(raw, src + t * p.st, valid, tid, xHi, xLo);
            if constexpr (PF) {
                if (tile + 1 < ENC_TILES && t0 + ENC_ROWS < p.T)
                    load_row_words<D, Tin>(src + (t + ENC_ROWS) * p.st, t + ENC_ROWS < p.T, raw);
            }
            tqdev::fence_proxy_async_smem();
            tqdev::tc_fence_before();
            __syncthreads();
            if (tid == 0 && !s_abort) {
                if (tile > 0 || tqdev::mbar_wait_bounded(&s_bars[0], 0)) {
                    q_pending = false;
                    tqdev::tc_fence_after();
                    issue_dense_rotation<D, Tin>(s_tmem, xHi, xLo, sQ, &s_bars[1]);
                } else {
                    atomicOr(reinterpret_cast<unsigned int *>(&p.status[1]), TQ_FLAG_WAIT_TIMEOUT);
                    s_abort = 1;
                    tqdev::mbar_arrive(&s_bars[1]);   // release the wait below
                }
            }
            const bool done = s_abort ? true : tqdev::mbar_wait_bounded(&s_bars[1], (uint32_t)(tile & 1));
            if (!done) rot_drain = tile & 1;
            if (__syncthreads_or(!done || s_abort)) {
                if (tid == 0 && !done) atomicOr(reinterpret_cast<unsigned int *>(&p.status[1]), TQ_FLAG_WAIT_TIMEOUT);
                break;
            }
            tqdev::tc_fence_after();
            n2 = dr.n2;
            inv_scale = dr.inv_scale;
            nonfinite = dr.nonfinite;
            degenerate = dr.zero;
        } else {
            if constexpr (PF) {
                n2 = rotate_words_to_tmem<D, Tin>(raw, s_mask, tlane);
                if (tile + 1 < ENC_TILES && t0 + ENC_ROWS < p.T)
                    load_row_words<D, Tin>(src + (t + ENC_ROWS) * p.st, t + ENC_ROWS < p.T, raw);
            } else {
                n2 = rotate_row_to_tmem<D, Tin>(src + t * p.st, valid, s_mask, tlane);
            }
            nonfinite = !(n2 <= 3.0e38f);
            degenerate = nonfinite || !(n2 >= 1.17549435e-38f);
        }
        if (valid && nonfinite) atomicAdd(&p.status[0], 1ull);
        uint32_t *dst = reinterpret_cast<uint32_t *>(p.out + (bh * p.capacity + p.token_offset + t) * p.row_bytes);
        const float n = sqrtf(n2 * (1.f / D));
        float c2 = 0.f;
        if constexpr (HV <= 8) {
            float rb[8];
            row_bounds<HV>(n, p.pb, rb);
            int cnt[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            // HV + magnitude index lands in the low bits of K = 2^23 + HV + sum T_L 2^L
            const float magic = 8388608.0f + (float)HV;
#pragma unroll 1
            for (int c = 0; c < NC; ++c) {
                float u[32];
                tqdev::tmem_ld_32x32b_x32_nowait(tlane + 32 * c, u);
                tqdev::tmem_wait_ld();
                uint32_t f[BV], S[3] = {0u, 0u, 0u};
#pragma unroll
                for (int w = 0; w < BV; ++w) f[w] = 0u;
#pragma unroll
                for (int j = 15; j >= 0; --j) {
                    const float2 A = make_float2(fabsf(u[2 * j]), fabsf(u[2 * j + 1]));
                    float2 T[3], dd[3];
                    search2<HV>(A, rb, T, dd);
                    float2 K = add2(T[0], dup2(magic));
                    if constexpr (HV >= 4) K = fma2(T[1], dup2(2.f), K);
                    if constexpr (HV >= 8) K = fma2(T[2], dup2(4.f), K);
#pragma unroll
                    for (int h = 1; h >= 0; --h) {
                        const int i = 2 * j + h;
                        const uint32_t kb = __float_as_uint(h ? K.y : K.x);
                        const uint32_t sg = (uint32_t)((int32_t)__float_as_uint(u[i]) >> 31);
                        const uint32_t idx = (kb ^ sg) & FMASK;   // negative: HV - 1 - cell
                        const int bit = BV * i;
                        f[bit / 32] |= idx << (bit % 32);
                        if ((bit % 32) + BV > 32) f[bit / 32 + 1] |= idx >> (32 - bit % 32);
#pragma unroll
                        for (int l = 0; l < Levels<HV>::L; ++l) S[l] = push_sign(S[l], h ? dd[l].y : dd[l].x);
                    }
                }
                count_cells<HV>(S, cnt);
                if (valid) {
#pragma unroll
                    for (int w = 0; w < BV; ++w)
                        dst[BV * c + w] = degenerate ? degenerate_field_word<BV>(BV * c + w) : f[w];
                }
            }
            int rest = D;
#pragma unroll
            for (int k = 1; k < HV; ++k) {
                rest -= cnt[k];
                c2 = fmaf((float)cnt[k], s_mag2[k], c2);
            }
            c2 = fmaf((float)rest, s_mag2[0], c2);
        } else {
            float nb[16];
#pragma unroll
            for (int k = 0; k < HV - 1; ++k) nb[k] = n * p.pb[k];
#pragma unroll 1
            for (int c = 0; c < NC; ++c) {
                float u[32];
                tqdev::tmem_ld_32x32b_x32_nowait(tlane + 32 * c, u);
                tqdev::tmem_wait_ld();
                uint32_t f[BV];
#pragma unroll
                for (int w = 0; w < BV; ++w) f[w] = 0u;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    uint32_t idx;
                    if (degenerate) {
                        idx = HV;
                    } else {
                        const uint32_t cell = mag_index<HV>(fabsf(u[i]), nb);
                        idx = u[i] < 0.f ? (uint32_t)(HV - 1) - cell : (uint32_t)HV + cell;
                        c2 += s_mag2[cell];
                    }
                    const int bit = BV * i;
                    f[bit / 32] |= idx << (bit % 32);
                    if ((bit % 32) + BV > 32) f[bit / 32 + 1] |= idx >> (32 - bit % 32);
                }
                if (valid) {
#pragma unroll
                    for (int w = 0; w < BV; ++w) dst[BV * c + w] = f[w];
                }
            }
        }
        if (valid) dst[BV * NC] = __float_as_uint(degenerate ? 0.f : n * sqrtf((float)D / c2) * inv_scale);
    }
    if (rot_drain >= 0) tqdev::mbar_wait_bounded(&s_bars[1], (uint32_t)rot_drain);
    if (q_pending) tqdev::mbar_wait_bounded(&s_bars[0], 0);
    tqdev::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tqdev::tc_fence_after();
        tqdev::tmem_dealloc(s_tmem, tmem_cols_for(D));
    }
}

// -------------------------------------------------------------------- keys
template <int D, int BK, typename Tin, int ROT>
__global__ void __launch_bounds__(ENC_ROWS) tq_encode_k_kernel(const __grid_constant__ EncodeParams p,
                                                               const __grid_constant__ CUtensorMap tmapS,
                                                               const __grid_constant__ CUtensorMap tmapQ) {
    constexpr int HK = (1 << BK) / 2;
    constexpr int NC = D / 32;                 // chunks = 32-bit words per bit plane
    constexpr int ATOM = ENC_ROWS * 128;       // bytes of one 128-row x 128-byte swizzle column
    constexpr int A_BYTES = (D / 64) * ATOM;   // one residual pass
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // misc region [0, MISC): sign masks (up to MISC / 2 bytes), squared
    // centroid magnitudes, barriers
    constexpr int MISC = D > 128 ? 2048 : 1024;
    uint32_t *s_mask = reinterpret_cast<uint32_t *>(smem);
    float *s_mag2 = reinterpret_cast<float *>(smem + MISC / 2);             // [16]
    // [0] S loaded, [1] QJL MMA done, [2] Q loaded, [3] rotation MMA done (dense rotation)
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + MISC / 2 + 256);
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bars + 4);
    int *s_abort = reinterpret_cast<int *>(s_tmem + 1);
    const int M = p.M;
    uint8_t *sS = smem + MISC;                                              // [D/64][M rows][128 B]
    uint8_t *sA = sS + (D / 64) * M * 128;                                   // [pass][D/64][128 rows][128 B]
    uint8_t *sQ = sA + 2 * A_BYTES;                                          // dense rotation: [2][D/64][D][128 B]
    const int tid = threadIdx.x, warp = tid / 32;
    const int64_t blk = blockIdx.x;
    const int64_t bh = blk / p.blocks_per_bh;
    const int head = (int)(bh % p.H);
    const int64_t b = bh / p.H;
    const int64_t tb0 = (blk % p.blocks_per_bh) * (int64_t)ENC_TILES * ENC_ROWS;
    // U [0, d); C [d, 2d); P [d, d + m) (written by the MMA while the next
    // tile's rotation fills U)
    const uint32_t tmem_cols = tmem_cols_for(D + (M > D ? M : D));
    build_sign_masks<Tin, D>(p.signs + (int64_t)head * (D / 32), s_mask);
    if (tid < 16) s_mag2[tid] = tid < HK ? p.mag[tid] * p.mag[tid] : 0.f;
    if (tid == 0) {
        for (int i = 0; i < 4; ++i) tqdev::mbar_init(&bars[i], 1);
        *s_abort = tqdev::status_aborted(p.status) ? 1 : 0;
        tqdev::fence_barrier_init();
    }
    if (warp == 0) tqdev::tmem_alloc(s_tmem, tmem_cols);
    tqdev::tc_fence_before();
    __syncthreads();
    tqdev::tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    const uint32_t tlane = tmem_base + ((uint32_t)(warp * 32) << 16);
    // Copies and MMAs that a timed-out wait left in flight; each gets one more
    // bounded wait before the CTA frees its TMEM and exits.
    bool s_pending = false, q_pending = false;   // thread 0: S / Q tiles requested, not yet seen
    int qjl_drain = -1, rot_drain = -1;          // phase of a QJL / rotation MMA not seen complete
    if (tid == 0 && !*s_abort) {
        tqdev::mbar_expect_tx(&bars[0], (uint32_t)(M * D * 2));
#pragma unroll
        for (int a = 0; a < D / 64; ++a) tqdev::tma_load_2d(sS + a * M * 128, &tmapS, a * 64, head * M, &bars[0]);
        s_pending = true;
        if constexpr (ROT == 1) {
            load_q_tiles<D>(sQ, &tmapQ, head, &bars[2]);
            q_pending = true;
        }
    }
    const Tin *src = reinterpret_cast<const Tin *>(p.x) + b * p.sb + (int64_t)head * p.sh;
    uint8_t *aHi = sA, *aLo = sA + A_BYTES;
    const uint32_t tP = tlane + (uint32_t)D;   // this lane's P columns
    int ntiles = 0;
    while (ntiles < ENC_TILES && tb0 + (int64_t)ntiles * ENC_ROWS < p.T) ++ntiles;
    // A, B of the first tile; later tiles' rotations overlap the previous MMA,
    // and (16-bit inputs, d <= 128) their rows are loaded into registers a tile ahead
    constexpr bool PF = sizeof(Tin) == 2 && D <= 128;
    RowWords<D> raw;
    float n2 = 0.f;
    if (ntiles > 0 && !*s_abort) {
        const int64_t t = tb0 + tid;
        if constexpr (PF) load_row_words<D, Tin>(src + t * p.st, t < p.T, raw);
        if constexpr (ROT == 0) {
            if constexpr (PF) n2 = rotate_words_to_tmem<D, Tin>(raw, s_mask, tlane);
            else n2 = rotate_row_to_tmem<D, Tin>(src + t * p.st, t < p.T, s_mask, tlane);
        }
    }
#pragma unroll 1
    for (int tile = 0; tile < ntiles; ++tile) {
        if (tile == 0 && *s_abort) break;   // uniform: set before the set-up barrier
        const int64_t t = tb0 + tile * ENC_ROWS + tid;
        const bool valid = t < p.T;
        float inv_scale = 1.f;
        bool dense_nonfinite = false, dense_zero = false;
        if constexpr (ROT == 1) {
            // A, B: the dense rotation of this tile on the tensor cores
            const DenseRow dr = stage_dense_row<D, Tin>(raw, src + t * p.st, valid, tid, aHi, aLo);
            tqdev::fence_proxy_async_smem();
            tqdev::tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                if (tile > 0 || tqdev::mbar_wait_bounded(&bars[2], 0)) {
                    q_pending = false;
                    tqdev::tc_fence_after();
                    issue_dense_rotation<D, Tin>(tmem_base, aHi, aLo, sQ, &bars[3]);
                } else {
                    atomicOr(reinterpret_cast<unsigned int *>(&p.status[1]), TQ_FLAG_WAIT_TIMEOUT);
                    *s_abort = 1;
                    tqdev::mbar_arrive(&bars[3]);   // release the wait below
                }
            }
            if constexpr (PF) {
                if (tile + 1 < ntiles) load_row_words<D, Tin>(src + (t + ENC_ROWS) * p.st, t + ENC_ROWS < p.T, raw);
            }
            const bool rdone = tqdev::mbar_wait_bounded(&bars[3], (uint32_t)(tile & 1));
            if (!rdone) rot_drain = tile & 1;
            if (__syncthreads_or(!rdone || *s_abort)) {
                if (tid == 0 && !rdone) atomicOr(reinterpret_cast<unsigned int *>(&p.status[1]), TQ_FLAG_WAIT_TIMEOUT);
                if (tid == 0) *s_abort = 1;
                break;
            }
            tqdev::tc_fence_after();
            n2 = dr.n2;
            inv_scale = dr.inv_scale;
            dense_nonfinite = dr.nonfinite;
            dense_zero = dr.zero;
        } else if constexpr (PF) {
            if (tile + 1 < ntiles) load_row_words<D, Tin>(src + (t + ENC_ROWS) * p.st, t + ENC_ROWS < p.T, raw);
        }
        uint32_t *dst = reinterpret_cast<uint32_t *>(p.out + (bh * p.capacity + p.token_offset + t) * p.row_bytes);
        const bool nonfinite = ROT == 1 ? dense_nonfinite : !(n2 <= 3.0e38f);
        const bool degenerate = ROT == 1 ? dense_zero : (nonfinite || !(n2 >= 1.17549435e-38f));
        if (valid && nonfinite) atomicAdd(&p.status[0], 1ull);
        const float n = sqrtf(n2 * (1.f / D));
        float rb[8];
        row_bounds<HK>(n, p.pb, rb);
        // C: index planes, the signed centroids (to TMEM columns [d, 2d)),
        // cell counts (for sum C[idx]^2) and sum |u| C[idx]
        int cnt[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        float2 ucp = make_float2(0.f, 0.f);
#pragma unroll 2
        for (int c = 0; c < NC; ++c) {
            float u[32];
            tqdev::tmem_ld_32x32b_x32_nowait(tlane + 32 * c, u);
            tqdev::tmem_wait_ld();
            uint32_t S[3] = {0u, 0u, 0u}, Sn = 0u;
#pragma unroll
            for (int j = 15; j >= 0; --j) {
                const float2 A = make_float2(fabsf(u[2 * j]), fabsf(u[2 * j + 1]));
                float2 T[3], dd[3];
                search2<HK>(A, rb, T, dd);
                float2 cm;
                if constexpr (HK == 1) {
                    cm = dup2(p.cl[0]);
                } else if constexpr (HK == 2) {
                    cm = fma2(T[0], dup2(p.cl[0]), dup2(p.cl[1]));
                } else if constexpr (HK == 4) {
                    const float2 lo = fma2(T[1], dup2(p.cl[0]), dup2(p.cl[1]));
                    const float2 df = fma2(T[1], dup2(p.cl[2]), dup2(p.cl[3]));
                    cm = fma2(T[0], df, lo);
                } else {
                    const float2 lo = fma2(T[1], fma2(T[2], dup2(p.cl[0]), dup2(p.cl[1])),
                                           fma2(T[2], dup2(p.cl[2]), dup2(p.cl[3])));
                    const float2 df = fma2(T[1], fma2(T[2], dup2(p.cl[4]), dup2(p.cl[5])),
                                           fma2(T[2], dup2(p.cl[6]), dup2(p.cl[7])));
                    cm = fma2(T[0], df, lo);
                }
                ucp = fma2(A, cm, ucp);
#pragma unroll
                for (int h = 1; h >= 0; --h) {
#pragma unroll
                    for (int l = 0; l < Levels<HK>::L; ++l) S[l] = push_sign(S[l], h ? dd[l].y : dd[l].x);
                    Sn = push_sign(Sn, u[2 * j + h]);
                }
                u[2 * j] = copysignf(cm.x, u[2 * j]);
                u[2 * j + 1] = copysignf(cm.y, u[2 * j + 1]);
            }
            tqdev::tmem_st_32x32b_x32(tlane + D + 32 * c, u);
            count_cells<HK>(S, cnt);
            if (valid) {
                // ascending index: top bit = non-negative, low bits = magnitude
                // index, complemented for negative values
#pragma unroll
                for (int q = 0; q < BK - 1; ++q)
                    dst[q * NC + c] = degenerate ? (((HK >> q) & 1) ? ~0u : 0u) : (~S[q] ^ Sn);
                dst[(BK - 1) * NC + c] = degenerate ? ~0u : ~Sn;
            }
        }
        tqdev::tmem_wait_st();
        float c2 = 0.f;
        {
            int rest = D;
#pragma unroll
            for (int k = 1; k < HK; ++k) {
                rest -= cnt[k];
                c2 = fmaf((float)cnt[k], s_mag2[k], c2);
            }
            c2 = fmaf((float)rest, s_mag2[0], c2);
        }
        const float uc = ucp.x + ucp.y;
        const float ns = degenerate ? 0.f : n * sqrtf((float)D / c2);
        // |e|^2 from the sums, only to scale the MMA operand (the stored gamma
        // comes from the direct sum below)
        float e2a = n2 - 2.f * ns * uc + ns * ns * c2;
        e2a = fmaxf(e2a, 1e-10f * n2);
        const float sc = degenerate ? 0.f : sqrtf((float)D / e2a);
        // D: residual u - n_s C[idx] as binary16 hi + lo, swizzled K-major operand
        float2 e2p = make_float2(0.f, 0.f);
#pragma unroll 2
        for (int c = 0; c < NC; ++c) {
            float u[32], cv[32];
            tqdev::tmem_ld_32x32b_x32_nowait(tlane + 32 * c, u);
            tqdev::tmem_ld_32x32b_x32_nowait(tlane + D + 32 * c, cv);
            tqdev::tmem_wait_ld();
#pragma unroll
            for (int j8 = 0; j8 < 4; ++j8) {
                uint32_t hw[4], lw[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = 8 * j8 + 2 * e;
                    const float2 E = fma2(dup2(-ns), make_float2(cv[i], cv[i + 1]), make_float2(u[i], u[i + 1]));
                    e2p = fma2(E, E, e2p);
                    const float2 a = mul2(E, dup2(sc));
                    const __half2 hh = __floats2half2_rn(a.x, a.y);
                    const float2 l = sub2(a, __half22float2(hh));
                    const __half2 ll = __floats2half2_rn(l.x, l.y);
                    hw[e] = *reinterpret_cast<const uint32_t *>(&hh);
                    lw[e] = *reinterpret_cast<const uint32_t *>(&ll);
                }
                const int kk = 4 * c + j8;          // 16-byte unit of the row
                const int off = (kk / 8) * ATOM + tid * 128 + (((kk % 8) ^ (tid & 7)) << 4);
                *reinterpret_cast<uint4 *>(aHi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4 *>(aLo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
        }
        const float e2 = e2p.x + e2p.y;
        bool zero_row = degenerate;
        {
            const int tail = BK * NC + M / 32;
            const float nsv = ns * inv_scale, gv = degenerate ? 0.f : sqrtf(e2 * (1.f / D)) * inv_scale;
            if (p.norm_f16) {
                uint32_t w;
                if (!tqdev::pack_norms_f16(nsv, gv, w)) {
                    // binary16 overflow: the zero row, counted with the non-finite rows
                    zero_row = true;
                    w = 0u;
                    if (valid) {
                        atomicAdd(&p.status[0], 1ull);
#pragma unroll 1
                        for (int c = 0; c < NC; ++c) {
#pragma unroll
                            for (int q = 0; q < BK - 1; ++q) dst[q * NC + c] = ((HK >> q) & 1) ? ~0u : 0u;
                            dst[(BK - 1) * NC + c] = ~0u;
                        }
                    }
                }
                if (valid) dst[tail] = w;
            } else if (valid) {
                dst[tail] = __float_as_uint(nsv);
                dst[tail + 1] = __float_as_uint(gv);
            }
        }
        // E: the QJL projection on the tensor cores (TMEM columns [d, d + m));
        // an abort flag set by any thread ends the loop here, for all threads
        tqdev::fence_proxy_async_smem();
        tqdev::tc_fence_before();
        if (__syncthreads_or(*s_abort)) break;
        if (tid == 0) {
            const bool ok = tile > 0 || tqdev::mbar_wait_bounded(&bars[0], 0);
            if (ok) s_pending = false;
            if (!ok) {
                atomicOr(reinterpret_cast<unsigned int *>(&p.status[1]), TQ_FLAG_WAIT_TIMEOUT);
                *s_abort = 1;
                tqdev::mbar_arrive(&bars[1]);   // release the epilogue wait below
            } else {
                tqdev::tc_fence_after();
                const uint32_t idesc = tqdev::idesc_f16_f32(M);
#pragma unroll
                for (int pass = 0; pass < 2; ++pass) {
                    const uint32_t abase = tqdev::smem_u32(pass ? aLo : aHi);
                    const uint32_t bbase = tqdev::smem_u32(sS);
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t a_addr = abase + (ks / 4) * ATOM + (ks % 4) * 32;
                        const uint32_t b_addr = bbase + (ks / 4) * (M * 128) + (ks % 4) * 32;
                        tqdev::mma_f16_ss(tmem_base + (uint32_t)D, tqdev::smem_desc_sw128(a_addr),
                                          tqdev::smem_desc_sw128(b_addr), idesc, (pass | ks) != 0);
                    }
                }
                tqdev::mma_commit(&bars[1]);
            }
        }
        // A, B of the next tile while the MMA runs (they touch only U)
        float n2_next = 0.f;
        if (ROT == 0 && tile + 1 < ntiles) {
            const int64_t tn = t + ENC_ROWS;
            if constexpr (PF) n2_next = rotate_words_to_tmem<D, Tin>(raw, s_mask, tlane);
            else n2_next = rotate_row_to_tmem<D, Tin>(src + tn * p.st, tn < p.T, s_mask, tlane);
        }
        // F: sign epilogue
        const bool done = tqdev::mbar_wait_bounded(&bars[1], (uint32_t)(tile & 1));
        if (!done || *s_abort) {
            // this thread skips the epilogue; the flag ends the loop for every
            // thread at the next pre-MMA barrier
            if (!done) {
                atomicOr(reinterpret_cast<unsigned int *>(&p.status[1]), TQ_FLAG_WAIT_TIMEOUT);
                qjl_drain = tile & 1;
            }
            *s_abort = 1;
            continue;
        }
        tqdev::tc_fence_after();
        uint32_t *sdst = dst + BK * NC;
#pragma unroll 2
        for (int c = 0; c < M / 32; ++c) {
            float pv[32];
            tqdev::tmem_ld_32x32b_x32_nowait(tP + (uint32_t)(c * 32), pv);
            tqdev::tmem_wait_ld();
            // bit i = [p_i >= 0]: collect the sign bits (p + 0 turns -0 into +0)
            uint32_t neg = 0u;
#pragma unroll
            for (int j = 15; j >= 0; --j) {
                const float2 q = add2(make_float2(pv[2 * j], pv[2 * j + 1]), dup2(0.f));
                neg = push_sign(neg, q.y);
                neg = push_sign(neg, q.x);
            }
            if (valid) sdst[c] = zero_row ? ~0u : ~neg;
        }
        n2 = n2_next;
    }
    if (qjl_drain >= 0) tqdev::mbar_wait_bounded(&bars[1], (uint32_t)qjl_drain);
    if (rot_drain >= 0) tqdev::mbar_wait_bounded(&bars[3], (uint32_t)rot_drain);
    if (s_pending) tqdev::mbar_wait_bounded(&bars[0], 0);
    if (q_pending) tqdev::mbar_wait_bounded(&bars[2], 0);
    tqdev::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tqdev::tc_fence_after();
        tqdev::tmem_dealloc(tmem_base, tmem_cols);
    }
}

// ===================================================== TMA-fed encoders
// For binary16 / bfloat16 rows and the Walsh-Hadamard rotation.  One
// persistent CTA per SM takes a contiguous range of 128-row tiles (each tile
// holds rows of one (batch, head)), so the head-dependent operands change
// only a few times per CTA.
//
// The last warp is the producer: one lane requests every tile's rows with
// 4-D TMA loads into a ring of shared-memory stages and issues the
// tensor-core work as soon as its inputs are ready (it polls the barriers,
// never blocking on one of them):
//   * the rotation U = X B^T with B[n][k] = H[n][k] D[k] (+-1, exact in the
//     16-bit input type), accumulated in fp32 in TMEM -- the Walsh-Hadamard
//     transform of the signed row as a dense product: exact products, fp32
//     sums (the rounding order differs from the butterflies, within float
//     rounding);
//   * keys: the QJL projection P = E S^T of the residual operand E written
//     by a compute group (binary16 hi + lo, two passes, fp32 in TMEM).
// The other warps form NG groups of four; group g takes tiles g, g + NG, ...
// of the CTA's range, one thread per row (the TMEM lane of warp w is 32 (w % 4)
// + lane): it reads the row's rotation from its group's TMEM columns in
// 32-coordinate chunks, takes |u|^2, quantizes chunk by chunk and stores the
// packed row.  Keys also stage the signed centroids in TMEM, write the
// residual operand (one shared buffer, taken in tile order), and store the
// sign plane once the QJL projection of their tile is done.  The groups run
// independently of each other, so while one waits for the tensor cores the
// others issue.
// B-bit index fields of 32 coordinates (coordinate j at bit B j of f[0..B),
// little-endian) from the B index planes (bit j of P[q] = bit q of index j),
// for B in {2, 3, 4}; spread[x] holds bit i of the byte x at bit B i.
template <int B>
__device__ __forceinline__ void fields_from_planes(const uint32_t (&P)[B], const uint32_t *spread, uint32_t (&f)[B]) {
    if constexpr (B == 2 || B == 4) {
        // a byte of the planes covers 8 coordinates = 8 B bits
        constexpr int PARTS = B == 2 ? 2 : 1;   // plane bytes per output word
#pragma unroll
        for (int w = 0; w < B; ++w) {
            uint32_t acc = 0u;
#pragma unroll
            for (int part = 0; part < PARTS; ++part) {
                const int byte = (B == 4) ? w : 2 * w + part;
                uint32_t g = 0u;
#pragma unroll
                for (int q = 0; q < B; ++q) g |= spread[(P[q] >> (8 * byte)) & 0xFFu] << q;
                acc |= (B == 4) ? g : g << (16 * part);
            }
            f[w] = acc;
        }
    } else if constexpr (B == 3) {
        // 8 coordinates = 24 bits; the four 24-bit groups straddle the words
        uint32_t g[4];
#pragma unroll
        for (int byte = 0; byte < 4; ++byte) {
            g[byte] = 0u;
#pragma unroll
            for (int q = 0; q < 3; ++q) g[byte] |= spread[(P[q] >> (8 * byte)) & 0xFFu] << q;
        }
        f[0] = g[0] | (g[1] << 24);
        f[1] = (g[1] >> 8) | (g[2] << 16);
        f[2] = (g[2] >> 16) | (g[3] << 8);
    }
}

struct PipeParams {
    uint8_t *out;           // packed rows of this side
    int64_t capacity, token_offset, T;
    int H;
    int row_bytes;
    int M;                  // keys: projections
    int64_t tiles_per_bh, n_tiles;
    uint32_t s_bytes;       // keys: bytes of head's S tile, (d/64) * m * 128
    unsigned long long *status;
    float mag[16];          // positive-half centroid magnitudes
    float pb[16];           // positive boundaries
    float cl[8];            // keys: centroid magnitude as a multilinear form in the search bits
    int norm_f16;
};

// NP: pieces of the rotation operand (1: the exact +-1 Walsh-Hadamard matrix;
// Haar values: sqrt(d) Q as binary16 hi + lo (2) or bfloat16 hi + mid + lo (3)).
template <int D, bool KEYS, int B, int NP = 1>
struct PipeLayout {
    // compute groups of 4 warps: keys hold U and C/P (2 x 128 TMEM columns)
    // per group; values hold U only (four groups fit 96 registers a thread)
    static constexpr int NG = KEYS ? 2 : 4;
    static constexpr int THREADS = 32 * (4 * NG + 1);    // + the producer warp
    static constexpr int XBOX = ENC_ROWS * 128;          // one 64-column box of a tile (16 KB)
    static constexpr int XSTAGE = (D / 64) * XBOX;       // one tile of 16-bit rows
    // stages of the row ring: keys at d = 128 have room for one next to the
    // two groups' residual buffers
    static constexpr int NS = KEYS ? (D == 128 ? 1 : 2) : (NP == 3 ? 3 : 4);
    static constexpr int OFF_HD = NS * XSTAGE;           // rotation operand [NP][d/64][d][128 B]
    static constexpr int OFF_A = OFF_HD + NP * D * D * 2;   // keys: residual operand hi, lo
    // keys: residual operand buffers, one per group with the Walsh-Hadamard
    // operand, one shared (taken in tile order) with the larger Haar operand
    static constexpr int NA = NP == 1 ? NG : 1;
    static constexpr int OFF_S = OFF_A + (KEYS ? NA * 2 * XSTAGE : 0);   // keys: S [d/64][m][128 B]
    static constexpr int FIXED = 1024 + OFF_S;           // dynamic bytes before S (with alignment slack)
};

// Non-blocking test of an mbarrier phase.
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t phase) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(tqdev::smem_u32(bar)), "r"(phase)
        : "memory");
    return ok != 0;
}

// Wait (bounded) by every lane of a warp; true if all of them saw the phase.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t phase) {
    const bool ok = tqdev::mbar_wait_bounded(bar, phase);
    return __all_sync(0xffffffffu, ok);
}

template <int D, int B, typename Tin, bool KEYS, int NP = 1>
__global__ void __launch_bounds__(PipeLayout<D, KEYS, B, NP>::THREADS, 1)
    tq_encode_pipe_kernel(const __grid_constant__ PipeParams p, const __grid_constant__ CUtensorMap tmapX,
                          const __grid_constant__ CUtensorMap tmapHD, const __grid_constant__ CUtensorMap tmapS) {
    using L = PipeLayout<D, KEYS, B, NP>;
    constexpr int NS = L::NS;
    constexpr int NG = L::NG;
    constexpr int HB = (1 << B) / 2;             // magnitude cells of the positive half
    constexpr int NC = D / 32;                   // 32-coordinate chunks per row (= words per key index plane)
    constexpr int PWARP = 4 * NG;                // the producer warp
    constexpr bool BF = std::is_same<Tin, __nv_bfloat16>::value;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sX = sm;
    uint8_t *sHD = sm + L::OFF_HD;
    uint8_t *sA = sm + L::OFF_A;
    uint8_t *sS = sm + L::OFF_S;
    __shared__ __align__(8) uint64_t bar_xfull[NS], bar_xfree[NS], bar_rot[NG], bar_ufree[NG], bar_qjl[NG];
    __shared__ __align__(8) uint64_t bar_afull[NG], bar_afree[NG], bar_hd, bar_s;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ float s_mag2[16];
    __shared__ uint32_t s_spread[KEYS ? 1 : 256];   // values: bit i of a byte -> bit B i

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if constexpr (!KEYS) {
        for (int i = tid; i < 256; i += blockDim.x) {
            uint32_t v = 0u;
            if (B <= 4)
                for (int bit = 0; bit < 8; ++bit) v |= ((uint32_t)(i >> bit) & 1u) << (B * bit);
            s_spread[i] = v;
        }
    }
    const int64_t tile_begin = (int64_t)blockIdx.x * p.n_tiles / gridDim.x;
    const int64_t tile_end = ((int64_t)blockIdx.x + 1) * p.n_tiles / gridDim.x;
    const int ntile = (int)(tile_end - tile_begin);
    const uint32_t tpb = (uint32_t)p.tiles_per_bh;
    const int M = KEYS ? p.M : 0;
    // TMEM: group g's rotation U at g * GSTRIDE, keys' signed centroids C and
    // then the projections P (C is consumed before the QJL MMA writes P) right after
    const uint32_t GSTRIDE = KEYS ? (uint32_t)(D + (M > D ? M : D)) : (uint32_t)D;
    const uint32_t tmem_cols = tmem_cols_for((int)(NG * GSTRIDE));

    if (tid == 0) {
        for (int i = 0; i < NS; ++i) {
            tqdev::mbar_init(&bar_xfull[i], 1);
            tqdev::mbar_init(&bar_xfree[i], 1);
        }
        for (int i = 0; i < NG; ++i) {
            tqdev::mbar_init(&bar_rot[i], 1);
            tqdev::mbar_init(&bar_ufree[i], 128);
            tqdev::mbar_init(&bar_qjl[i], 1);
        }
        for (int i = 0; i < NG; ++i) {
            tqdev::mbar_init(&bar_afull[i], 128);
            tqdev::mbar_init(&bar_afree[i], 1);
        }
        tqdev::mbar_init(&bar_hd, 1);
        tqdev::mbar_init(&bar_s, 1);
        s_abort = tqdev::status_aborted(p.status) ? 1 : 0;
        tqdev::fence_barrier_init();
    }
    if (tid < 16) s_mag2[tid] = tid < HB ? p.mag[tid] * p.mag[tid] : 0.f;
    if (warp == 0) tqdev::tmem_alloc(&s_tmem, tmem_cols);
    tqdev::tc_fence_before();
    __syncthreads();
    tqdev::tc_fence_after();
    const uint32_t tmem = s_tmem;
    const bool run = !s_abort && ntile > 0;

    if (warp == PWARP) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && run) {
            // tile indices fit in 32 bits (the launcher checks), so the
            // divisions are 32-bit ones
            auto head_of = [&](int li) { return (int)(((uint32_t)(tile_begin + li) / tpb) % (uint32_t)p.H); };
            auto issue_x = [&](int li) {
                const uint32_t tile = (uint32_t)(tile_begin + li), bh = tile / tpb;
                const int t0 = (int)((tile - bh * tpb) * ENC_ROWS);
                const int h = (int)(bh % p.H), b = (int)(bh / p.H);
                const int s = li % NS;
                tqdev::mbar_expect_tx(&bar_xfull[s], (uint32_t)L::XSTAGE);
#pragma unroll
                for (int a = 0; a < D / 64; ++a)
                    tqdev::tma_load_4d(sX + s * L::XSTAGE + a * L::XBOX, &tmapX, a * 64, t0, h, b, &bar_xfull[s]);
            };
            const uint32_t idesc_rot = BF ? tqdev::idesc_bf16_f32(D) : tqdev::idesc_f16_f32(D);
            const uint32_t idesc_qjl = tqdev::idesc_f16_f32(KEYS ? M : 16);
            int next_rot = 0, next_qjl = 0, next_x = 0, xfree_seen = 0;
            int hd_head = -1, s_head = -1;               // head of the operand loaded / being loaded
            bool hd_busy = false, s_busy = false;        // a load in flight
            uint32_t hd_ph = 0, s_ph = 0;
            bool ok = true;
            uint64_t last = 0;
            uint32_t idle = 0;
            for (; next_x < NS && next_x < ntile; ++next_x) issue_x(next_x);
            while (next_rot < ntile || (KEYS && next_qjl < ntile)) {
                bool progress = false;
                // ---- rotation of tile next_rot into its group's U
                if (next_rot < ntile) {
                    const int li = next_rot, g = li % NG, h = head_of(li);
                    if (h != hd_head && !hd_busy) {
                        // the previous rotation (old operand) must be complete
                        if (li == 0 || mbar_test(&bar_xfree[(li - 1) % NS], (uint32_t)(((li - 1) / NS) & 1))) {
                            tqdev::mbar_expect_tx(&bar_hd, (uint32_t)(NP * D * D * 2));
#pragma unroll
                            for (int piece = 0; piece < NP; ++piece)
#pragma unroll
                                for (int a = 0; a < D / 64; ++a)
                                    tqdev::tma_load_2d(sHD + (piece * (D / 64) + a) * D * 128, &tmapHD, a * 64,
                                                       (h * NP + piece) * D, &bar_hd);
                            hd_busy = true;
                            hd_head = h;
                            progress = true;
                        }
                    }
                    if (hd_busy && mbar_test(&bar_hd, hd_ph)) {
                        hd_ph ^= 1;
                        hd_busy = false;
                        progress = true;
                    }
                    if (h == hd_head && !hd_busy && mbar_test(&bar_xfull[li % NS], (uint32_t)((li / NS) & 1)) &&
                        (li < NG || mbar_test(&bar_ufree[g], (uint32_t)(((li - NG) / NG) & 1)))) {
                        tqdev::tc_fence_after();
                        const uint32_t abase = tqdev::smem_u32(sX + (li % NS) * L::XSTAGE);
                        const uint32_t bbase = tqdev::smem_u32(sHD);
#pragma unroll
                        for (int piece = 0; piece < NP; ++piece)
#pragma unroll
                            for (int ks = 0; ks < D / 16; ++ks) {
                                const uint32_t a_addr = abase + (ks / 4) * L::XBOX + (ks % 4) * 32;
                                const uint32_t b_addr = bbase + piece * (D / 64) * D * 128 + (ks / 4) * (D * 128) + (ks % 4) * 32;
                                tqdev::mma_f16_ss(tmem + (uint32_t)g * GSTRIDE, tqdev::smem_desc_sw128(a_addr),
                                                  tqdev::smem_desc_sw128(b_addr), idesc_rot, (piece | ks) != 0);
                            }
                        tqdev::mma_commit(&bar_rot[g]);
                        tqdev::mma_commit(&bar_xfree[li % NS]);
                        ++next_rot;
                        progress = true;
                    }
                }
                // ---- QJL projection of tile next_qjl (keys)
                if (KEYS && next_qjl < next_rot) {
                    const int j = next_qjl, h = head_of(j);
                    if (h != s_head && !s_busy) {
                        // the previous projection (old S) must be complete
                        if (j == 0 || mbar_test(&bar_afree[(j - 1) % L::NA], (uint32_t)(((j - 1) / L::NA) & 1))) {
                            tqdev::mbar_expect_tx(&bar_s, p.s_bytes);
#pragma unroll
                            for (int a = 0; a < D / 64; ++a)
                                tqdev::tma_load_2d(sS + a * M * 128, &tmapS, a * 64, h * M, &bar_s);
                            s_busy = true;
                            s_head = h;
                            progress = true;
                        }
                    }
                    if (s_busy && mbar_test(&bar_s, s_ph)) {
                        s_ph ^= 1;
                        s_busy = false;
                        progress = true;
                    }
                    if (h == s_head && !s_busy && mbar_test(&bar_afull[j % L::NA], (uint32_t)((j / L::NA) & 1))) {
                        tqdev::tc_fence_after();
                        const uint32_t col = (uint32_t)(j % NG) * GSTRIDE + (uint32_t)D;
#pragma unroll
                        for (int pass = 0; pass < 2; ++pass) {
                            const uint32_t abase = tqdev::smem_u32(sA + ((j % L::NA) * 2 + pass) * L::XSTAGE);
                            const uint32_t bbase = tqdev::smem_u32(sS);
#pragma unroll
                            for (int ks = 0; ks < D / 16; ++ks) {
                                const uint32_t a_addr = abase + (ks / 4) * L::XBOX + (ks % 4) * 32;
                                const uint32_t b_addr = bbase + (ks / 4) * (M * 128) + (ks % 4) * 32;
                                tqdev::mma_f16_ss(tmem + col, tqdev::smem_desc_sw128(a_addr),
                                                  tqdev::smem_desc_sw128(b_addr), idesc_qjl, (pass | ks) != 0);
                            }
                        }
                        tqdev::mma_commit(&bar_qjl[j % NG]);
                        tqdev::mma_commit(&bar_afree[j % L::NA]);
                        ++next_qjl;
                        progress = true;
                    }
                }
                // ---- refill the ring: tile next_x goes where tile next_x - NS was
                if (next_x < ntile && next_x - NS < next_rot &&
                    mbar_test(&bar_xfree[next_x % NS], (uint32_t)(((next_x - NS) / NS) & 1))) {
                    issue_x(next_x);
                    ++next_x;
                    xfree_seen = next_x - NS;
                    progress = true;
                }
                // poll shared-memory barriers only; the wall clock is read every
                // 256 idle rounds (the abort flag was read at the CTA's start)
                if (progress) {
                    idle = 0;
                } else if ((++idle & 255) == 0) {
                    const uint64_t now = tqdev::globaltimer_ns();
                    if (idle == 256) last = now;
                    else if (now - last > 200000000ull) {
                        ok = false;
                        break;
                    }
                }
            }
            if (!ok) atomicOr(reinterpret_cast<unsigned int *>(&p.status[1]), TQ_FLAG_WAIT_TIMEOUT);
            // Drain: every copy and MMA issued is seen complete (bounded) before
            // the CTA frees its TMEM and shared memory.
            for (int li = next_rot; li < next_x; ++li)                 // rows requested, never rotated
                tqdev::mbar_wait_bounded(&bar_xfull[li % NS], (uint32_t)((li / NS) & 1));
            for (int li = xfree_seen; li < next_rot; ++li)             // rotations not seen through xfree
                tqdev::mbar_wait_bounded(&bar_xfree[li % NS], (uint32_t)((li / NS) & 1));
            for (int j = next_qjl - L::NA < 0 ? 0 : next_qjl - L::NA; j < next_qjl; ++j)
                tqdev::mbar_wait_bounded(&bar_afree[j % L::NA], (uint32_t)((j / L::NA) & 1));
            if (hd_busy) tqdev::mbar_wait_bounded(&bar_hd, hd_ph);
            if (s_busy) tqdev::mbar_wait_bounded(&bar_s, s_ph);
        }
    } else if (run) {
        // ------------------------------------------------------------ compute
        const int g = warp >> 2;                                // group
        const int row = ((warp & 3) << 5) | lane;               // tile row = TMEM lane
        const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)g * GSTRIDE;
        const uint32_t tU = tl, tC = tl + (uint32_t)D;          // keys: C, then P, at tC
        bool failed = false;
        // keys: the sign plane of the group's previous tile is stored after this
        // tile's |u|^2 pass, so its QJL projection overlaps that pass
        uint32_t *prev_dst = nullptr;
        bool prev_valid = false, prev_zero = false;
        auto sign_epilogue = [&](int kprev) -> bool {
            if (!warp_wait(&bar_qjl[g], (uint32_t)(kprev & 1))) return false;
            tqdev::tc_fence_after();
            uint32_t *sdst = prev_dst + B * NC;
#pragma unroll 1
            for (int c = 0; c < M / 32; ++c) {
                uint32_t neg = 0u;
#pragma unroll
                for (int half = 1; half >= 0; --half) {
                    float pv[16];
                    tqdev::tmem_ld_32x32b_x16_nowait(tC + 32 * c + 16 * half, pv);
                    tqdev::tmem_wait_ld();
                    // bit i = [p_i >= 0] from the sign bit; an exact zero (of
                    // either sign) lies inside the decision band of p = 0
#pragma unroll
                    for (int j = 15; j >= 0; --j) neg = push_sign(neg, pv[j]);
                }
                if (prev_valid) sdst[c] = prev_zero ? ~0u : ~neg;
            }
            tqdev::tc_fence_before();
            return true;
        };
        int k = 0;
        for (int li = g; li < ntile && !failed; li += NG, ++k) {
            const uint32_t tile = (uint32_t)(tile_begin + li), bh32 = tile / tpb;
            const int64_t bh = bh32;
            const int64_t t = (int64_t)(tile - bh32 * tpb) * ENC_ROWS + row;
            const bool valid = t < p.T;
            uint32_t *dst = reinterpret_cast<uint32_t *>(p.out + (bh * p.capacity + p.token_offset + t) * p.row_bytes);
            if (!warp_wait(&bar_rot[g], (uint32_t)(k & 1))) {
                failed = true;
                break;
            }
            tqdev::tc_fence_after();
            // ---- |u|^2 over the row (the next chunk's load in flight meanwhile)
            float2 n2p = make_float2(0.f, 0.f);
            {
                float ua[32], ub[32];
                tqdev::tmem_ld_32x32b_x32(tU, ua);
#pragma unroll
                for (int c = 0; c < NC; ++c) {
                    float(&cur)[32] = (c & 1) ? ub : ua;
                    float(&nxt)[32] = (c & 1) ? ua : ub;
                    if (c + 1 < NC) tqdev::tmem_ld_32x32b_x32_nowait(tU + 32 * (c + 1), nxt);
#pragma unroll
                    for (int i = 0; i < 32; i += 2)
                        n2p = fma2(make_float2(cur[i], cur[i + 1]), make_float2(cur[i], cur[i + 1]), n2p);
                    if (c + 1 < NC) tqdev::tmem_wait_ld();
                }
            }
            if constexpr (KEYS) {
                if (k > 0 && !sign_epilogue(k - 1)) {
                    failed = true;
                    break;
                }
            }
            const float n2 = n2p.x + n2p.y;
            const bool nonfinite = !(n2 <= 3.0e38f);
            const bool degenerate = nonfinite || !(n2 >= 1.17549435e-38f);
            if (valid && nonfinite) atomicAdd(&p.status[0], 1ull);
            const float n = sqrtf(n2 * (1.f / D));
            float c2 = 0.f;
            if constexpr (!KEYS) {
                // ---- values: quantize chunk by chunk, B-bit fields
                constexpr uint32_t FMASK = (1u << B) - 1u;
                if constexpr (HB <= 8) {
                    // The search's level words give the cell bits of all 32
                    // coordinates (bit j of S[l] set: level l's test failed),
                    // so the B index planes are word operations; the fields
                    // are the planes' bits interleaved, byte by byte through
                    // the spread table (bit i of a byte to bit B i).
                    float rb[8];
                    row_bounds<HB>(n, p.pb, rb);
                    int cnt[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll 1
                    for (int c = 0; c < NC; ++c) {
                        float u[32];
                        tqdev::tmem_ld_32x32b_x32(tU + 32 * c, u);
                        uint32_t S[3] = {0u, 0u, 0u}, Sn = 0u;
#pragma unroll
                        for (int j = 15; j >= 0; --j) {
                            const float2 A = make_float2(fabsf(u[2 * j]), fabsf(u[2 * j + 1]));
                            float2 T[3], dd[3];
                            search2<HB>(A, rb, T, dd);
#pragma unroll
                            for (int hh = 1; hh >= 0; --hh) {
#pragma unroll
                                for (int l = 0; l < Levels<HB>::L; ++l) S[l] = push_sign(S[l], hh ? dd[l].y : dd[l].x);
                                Sn = push_sign(Sn, u[2 * j + hh]);
                            }
                        }
                        count_cells<HB>(S, cnt);
                        // index plane q: ascending index = top bit non-negative,
                        // low bits the cell, complemented for negative values
                        uint32_t P[B];
#pragma unroll
                        for (int q = 0; q < B - 1; ++q) P[q] = ~S[q] ^ Sn;
                        P[B - 1] = ~Sn;
                        uint32_t f[B];
                        fields_from_planes<B>(P, s_spread, f);
                        if (valid) {
#pragma unroll
                            for (int w = 0; w < B; ++w) dst[B * c + w] = degenerate ? degenerate_field_word<B>(B * c + w) : f[w];
                        }
                    }
                    int rest = D;
#pragma unroll
                    for (int kc = 1; kc < HB; ++kc) {
                        rest -= cnt[kc];
                        c2 = fmaf((float)cnt[kc], s_mag2[kc], c2);
                    }
                    c2 = fmaf((float)rest, s_mag2[0], c2);
                } else {
                    float nb[16];
#pragma unroll
                    for (int kc = 0; kc < HB - 1; ++kc) nb[kc] = n * p.pb[kc];
#pragma unroll 1
                    for (int c = 0; c < NC; ++c) {
                        float u[32];
                        tqdev::tmem_ld_32x32b_x32(tU + 32 * c, u);
                        uint32_t f[B];
#pragma unroll
                        for (int w = 0; w < B; ++w) f[w] = 0u;
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const uint32_t cell = mag_index<HB>(fabsf(u[i]), nb);
                            const uint32_t idx = u[i] < 0.f ? (uint32_t)(HB - 1) - cell : (uint32_t)HB + cell;
                            c2 += s_mag2[cell];
                            const int bit = B * i;
                            f[bit / 32] |= idx << (bit % 32);
                            if ((bit % 32) + B > 32) f[bit / 32 + 1] |= idx >> (32 - bit % 32);
                        }
                        if (valid) {
#pragma unroll
                            for (int w = 0; w < B; ++w) dst[B * c + w] = degenerate ? degenerate_field_word<B>(B * c + w) : f[w];
                        }
                    }
                }
                tqdev::tc_fence_before();
                tqdev::mbar_arrive(&bar_ufree[g]);                    // U read for the last time
                if (valid) dst[B * NC] = __float_as_uint(degenerate ? 0.f : n * sqrtf((float)D / c2));
            } else {
                // ---- keys: index planes, signed centroids to TMEM C, sum C^2, sum |u| C
                float rb[8];
                row_bounds<HB>(n, p.pb, rb);
                int cnt[8] = {0, 0, 0, 0, 0, 0, 0, 0};
                float2 ucp = make_float2(0.f, 0.f);
#pragma unroll 1
                for (int c = 0; c < NC; ++c) {
                    float u[32];
                    tqdev::tmem_ld_32x32b_x32(tU + 32 * c, u);
                    uint32_t S[3] = {0u, 0u, 0u}, Sn = 0u;
#pragma unroll
                    for (int j = 15; j >= 0; --j) {
                        const float2 A = make_float2(fabsf(u[2 * j]), fabsf(u[2 * j + 1]));
                        float2 T[3], dd[3];
                        search2<HB>(A, rb, T, dd);
                        float2 cm;
                        if constexpr (HB == 1) {
                            cm = dup2(p.cl[0]);
                        } else if constexpr (HB == 2) {
                            cm = fma2(T[0], dup2(p.cl[0]), dup2(p.cl[1]));
                        } else if constexpr (HB == 4) {
                            const float2 lo = fma2(T[1], dup2(p.cl[0]), dup2(p.cl[1]));
                            const float2 df = fma2(T[1], dup2(p.cl[2]), dup2(p.cl[3]));
                            cm = fma2(T[0], df, lo);
                        } else {
                            const float2 lo = fma2(T[1], fma2(T[2], dup2(p.cl[0]), dup2(p.cl[1])),
                                                   fma2(T[2], dup2(p.cl[2]), dup2(p.cl[3])));
                            const float2 df = fma2(T[1], fma2(T[2], dup2(p.cl[4]), dup2(p.cl[5])),
                                                   fma2(T[2], dup2(p.cl[6]), dup2(p.cl[7])));
                            cm = fma2(T[0], df, lo);
                        }
                        ucp = fma2(A, cm, ucp);
#pragma unroll
                        for (int hh = 1; hh >= 0; --hh) {
#pragma unroll
                            for (int l = 0; l < Levels<HB>::L; ++l) S[l] = push_sign(S[l], hh ? dd[l].y : dd[l].x);
                            Sn = push_sign(Sn, u[2 * j + hh]);
                        }
                        u[2 * j] = copysignf(cm.x, u[2 * j]);
                        u[2 * j + 1] = copysignf(cm.y, u[2 * j + 1]);
                    }
                    tqdev::tmem_st_32x32b_x32(tC + 32 * c, u);   // signed centroids
                    count_cells<HB>(S, cnt);
                    if (valid) {
#pragma unroll
                        for (int q = 0; q < B - 1; ++q)
                            dst[q * NC + c] = degenerate ? (((HB >> q) & 1) ? ~0u : 0u) : (~S[q] ^ Sn);
                        dst[(B - 1) * NC + c] = degenerate ? ~0u : ~Sn;
                    }
                }
                tqdev::tmem_wait_st();
                {
                    int rest = D;
#pragma unroll
                    for (int kc = 1; kc < HB; ++kc) {
                        rest -= cnt[kc];
                        c2 = fmaf((float)cnt[kc], s_mag2[kc], c2);
                    }
                    c2 = fmaf((float)rest, s_mag2[0], c2);
                }
                const float uc = ucp.x + ucp.y;
                const float ns = degenerate ? 0.f : n * sqrtf((float)D / c2);
                // |e|^2 from the sums, only to scale the MMA operand
                float e2a = n2 - 2.f * ns * uc + ns * ns * c2;
                e2a = fmaxf(e2a, 1e-10f * n2);
                const float sc = degenerate ? 0.f : sqrtf((float)D / e2a);
                // ---- residual operand: buffer li % NA, free once the projection
                // of the tile that used it before is done
                uint8_t *sAg = sA + (li % L::NA) * 2 * L::XSTAGE;
                if (li >= L::NA && !warp_wait(&bar_afree[li % L::NA], (uint32_t)(((li / L::NA) - 1) & 1))) {
                    failed = true;
                    break;
                }
                float2 e2p = make_float2(0.f, 0.f);
#pragma unroll 1
                for (int c = 0; c < NC; ++c) {
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        float uu[16], cv[16];
                        tqdev::tmem_ld_32x32b_x16_nowait(tU + 32 * c + 16 * half, uu);
                        tqdev::tmem_ld_32x32b_x16_nowait(tC + 32 * c + 16 * half, cv);
                        tqdev::tmem_wait_ld();
#pragma unroll
                        for (int jh = 0; jh < 2; ++jh) {
                            uint32_t hw[4], lw[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int i = 8 * jh + 2 * e;
                                const float2 E = fma2(dup2(-ns), make_float2(cv[i], cv[i + 1]), make_float2(uu[i], uu[i + 1]));
                                e2p = fma2(E, E, e2p);
                                const float2 a = mul2(E, dup2(sc));
                                const __half2 hh = __floats2half2_rn(a.x, a.y);
                                const float2 l = sub2(a, __half22float2(hh));
                                const __half2 ll = __floats2half2_rn(l.x, l.y);
                                hw[e] = *reinterpret_cast<const uint32_t *>(&hh);
                                lw[e] = *reinterpret_cast<const uint32_t *>(&ll);
                            }
                            const int kk = 4 * c + 2 * half + jh;             // 16-byte unit of the row
                            const int off = (kk / 8) * L::XBOX + row * 128 + (((kk % 8) ^ (row & 7)) << 4);
                            *reinterpret_cast<uint4 *>(sAg + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                            *reinterpret_cast<uint4 *>(sAg + L::XSTAGE + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                        }
                    }
                }
                tqdev::tc_fence_before();
                tqdev::mbar_arrive(&bar_ufree[g]);                    // U read for the last time
                tqdev::fence_proxy_async_smem();
                tqdev::mbar_arrive(&bar_afull[li % L::NA]);           // residual operand written
                const float e2 = e2p.x + e2p.y;
                bool zero_row = degenerate;
                const int tail = B * NC + M / 32;
                const float gv = degenerate ? 0.f : sqrtf(e2 * (1.f / D));
                if (p.norm_f16) {
                    uint32_t w;
                    if (!tqdev::pack_norms_f16(ns, gv, w)) {
                        // binary16 overflow: the zero row, counted with the non-finite rows
                        zero_row = true;
                        w = 0u;
                        if (valid) {
                            atomicAdd(&p.status[0], 1ull);
#pragma unroll 1
                            for (int c = 0; c < NC; ++c) {
#pragma unroll
                                for (int q = 0; q < B - 1; ++q) dst[q * NC + c] = ((HB >> q) & 1) ? ~0u : 0u;
                                dst[(B - 1) * NC + c] = ~0u;
                            }
                        }
                    }
                    if (valid) dst[tail] = w;
                } else if (valid) {
                    dst[tail] = __float_as_uint(ns);
                    dst[tail + 1] = __float_as_uint(gv);
                }
                prev_dst = dst;
                prev_valid = valid;
                prev_zero = zero_row;
            }
        }
        if constexpr (KEYS) {
            if (!failed && k > 0 && !sign_epilogue(k - 1)) failed = true;   // the group's last tile
        }
        if (failed && lane == 0) atomicOr(reinterpret_cast<unsigned int *>(&p.status[1]), TQ_FLAG_WAIT_TIMEOUT);
    }
    tqdev::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tqdev::tc_fence_after();
        tqdev::tmem_dealloc(tmem, tmem_cols);
    }
}

template <int D, typename Tin, bool KEYS, int NP = 1>
cudaError_t launch_pipe(int B, const PipeParams &p, const CUtensorMap &mx, const CUtensorMap &mhd,
                        const CUtensorMap &ms, int grid, cudaStream_t s) {
    using L = PipeLayout<D, KEYS, 2, NP>;   // the byte layout does not depend on B
    cudaError_t e = cudaSuccess;
    auto go = [&](auto kern, int threads) {
        size_t smem = (size_t)L::FIXED + (KEYS ? p.s_bytes : 0);
        // one CTA per SM: a second one could wait in tcgen05.alloc until the
        // first exits (the grid is one CTA per SM anyway)
        if (smem < 120 * 1024) smem = 120 * 1024;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return;
        }
        kern<<<grid, threads, smem, s>>>(p, mx, mhd, ms);
        e = cudaGetLastError();
    };
    switch (B) {
        case 1: if constexpr (KEYS) go(tq_encode_pipe_kernel<D, 1, Tin, KEYS, NP>, PipeLayout<D, KEYS, 1, NP>::THREADS); else return cudaErrorInvalidValue; break;
        case 2: go(tq_encode_pipe_kernel<D, 2, Tin, KEYS, NP>, PipeLayout<D, KEYS, 2, NP>::THREADS); break;
        case 3: go(tq_encode_pipe_kernel<D, 3, Tin, KEYS, NP>, PipeLayout<D, KEYS, 3, NP>::THREADS); break;
        case 4: go(tq_encode_pipe_kernel<D, 4, Tin, KEYS, NP>, PipeLayout<D, KEYS, 4, NP>::THREADS); break;
        case 5: if constexpr (!KEYS) go(tq_encode_pipe_kernel<D, 5, Tin, KEYS, NP>, PipeLayout<D, KEYS, 5, NP>::THREADS); else return cudaErrorInvalidValue; break;
        default: return cudaErrorInvalidValue;
    }
    return e;
}

template <int D, typename Tin, int ROT>
cudaError_t launch_k(int bits, const EncodeParams &p, const CUtensorMap &mapS, const CUtensorMap &mapQ, int64_t grid,
                     cudaStream_t s) {
    cudaError_t e = cudaSuccess;
    auto go = [&](auto kern) {
        size_t smem = (D > 128 ? 3072 : 2048) + (size_t)(D / 64) * p.M * 128 + 2 * (size_t)(D / 64) * ENC_ROWS * 128;
        if (ROT == 1) smem += 2 * (size_t)(D / 64) * D * 128;   // sqrt(d) Q, hi + lo
        // a CTA holding all 512 TMEM columns (d + m > 256) gets an SM to itself
        if (D + p.M > 256 && smem < 120 * 1024) smem = 120 * 1024;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) {
            cudaGetLastError();   // do not leave the failure as the thread's sticky last error
            return;
        }
        kern<<<(unsigned)grid, ENC_ROWS, smem, s>>>(p, mapS, mapQ);
        e = cudaGetLastError();
    };
    switch (bits) {
        case 2: go(tq_encode_k_kernel<D, 1, Tin, ROT>); break;
        case 3: go(tq_encode_k_kernel<D, 2, Tin, ROT>); break;
        case 4: go(tq_encode_k_kernel<D, 3, Tin, ROT>); break;
        case 5: go(tq_encode_k_kernel<D, 4, Tin, ROT>); break;
        default: return cudaErrorInvalidValue;
    }
    return e;
}

template <int D, typename Tin, int ROT>
cudaError_t launch_v(int bits, const EncodeParams &p, const CUtensorMap &mapQ, int64_t grid, cudaStream_t s) {
    cudaError_t e = cudaSuccess;
    auto go = [&](auto kern) {
        size_t smem = 0;
        if (ROT == 1)   // 1024-byte alignment slack, sqrt(d) Q (hi + lo), the row operand (hi [+ lo])
            smem = 1024 + 2 * (size_t)(D / 64) * D * 128 + (sizeof(Tin) == 2 ? 1 : 2) * (size_t)(D / 64) * ENC_ROWS * 128;
        if (smem > 48 * 1024) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) {
                cudaGetLastError();
                return;
            }
        }
        kern<<<(unsigned)grid, ENC_ROWS, smem, s>>>(p, mapQ);
        e = cudaGetLastError();
    };
    switch (bits) {
        case 2: go(tq_encode_v_kernel<D, 2, Tin, ROT>); break;
        case 3: go(tq_encode_v_kernel<D, 3, Tin, ROT>); break;
        case 4: go(tq_encode_v_kernel<D, 4, Tin, ROT>); break;
        case 5: go(tq_encode_v_kernel<D, 5, Tin, ROT>); break;
        default: return cudaErrorInvalidValue;
    }
    return e;
}

template <int D, typename Tin>
cudaError_t launch_dim(const tq_ctx *ctx, bool keys, const EncodeParams &p, int64_t grid, cudaStream_t s) {
    if (ctx->rotation == TQ_ROT_HAAR)
        return keys ? launch_k<D, Tin, 1>(ctx->bits, p, ctx->tmap_S, ctx->tmap_Q, grid, s)
                    : launch_v<D, Tin, 1>(ctx->bits, p, ctx->tmap_Q, grid, s);
    return keys ? launch_k<D, Tin, 0>(ctx->bits, p, ctx->tmap_S, ctx->tmap_Q, grid, s)
                : launch_v<D, Tin, 0>(ctx->bits, p, ctx->tmap_Q, grid, s);
}

template <typename Tin>
cudaError_t launch_side(const tq_ctx *ctx, bool keys, const EncodeParams &p, int64_t grid, cudaStream_t s) {
    if (ctx->d == 256) {
        // Walsh-Hadamard only: the Haar operands (2 x d x d binary16) do not
        // fit in shared memory at d = 256 (tq_create_ex rejects that pair)
        if (ctx->rotation != TQ_ROT_HADAMARD) return cudaErrorInvalidValue;
        return keys ? launch_k<256, Tin, 0>(ctx->bits, p, ctx->tmap_S, ctx->tmap_Q, grid, s)
                    : launch_v<256, Tin, 0>(ctx->bits, p, ctx->tmap_Q, grid, s);
    }
    if (ctx->d == 128) return launch_dim<128, Tin>(ctx, keys, p, grid, s);
    if (ctx->d == 64) return launch_dim<64, Tin>(ctx, keys, p, grid, s);
    return cudaErrorInvalidValue;
}

}  // namespace

// The key centroid magnitude C_k of cell k = sum_L T_L 2^L written as the
// multilinear form the key kernels evaluate in the search bits T_L
// (cb: the 2 HB centroids, ascending; cl: the form's 8 coefficients).
static void key_centroid_form(const float *cb, int HB, float *cl) {
    double m[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int i = 0; i < HB && i < 8; ++i) m[i] = cb[HB + i];
    double c[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (HB == 1) {
        c[0] = m[0];
    } else if (HB == 2) {
        c[0] = m[1] - m[0];
        c[1] = m[0];
    } else if (HB == 4) {
        c[0] = m[2] - m[0];
        c[1] = m[0];
        c[2] = (m[3] - m[2]) - (m[1] - m[0]);
        c[3] = m[1] - m[0];
    } else if (HB == 8) {
        const double d0 = m[1] - m[0], d2 = m[3] - m[2], d4 = m[5] - m[4], d6 = m[7] - m[6];
        c[0] = m[6] - m[4] - m[2] + m[0];
        c[1] = m[2] - m[0];
        c[2] = m[4] - m[0];
        c[3] = m[0];
        c[4] = d6 - d4 - d2 + d0;
        c[5] = d2 - d0;
        c[6] = d4 - d0;
        c[7] = d0;
    }
    for (int i = 0; i < 8; ++i) cl[i] = (float)c[i];
}

// Which encoder serves 16-bit Walsh-Hadamard rows: 0 = the TMA-fed
// persistent kernels where they apply (default), 1 = the per-thread
// Walsh-Hadamard kernels always.  Read once from TQ_ENCODE_PATH.
static int tq_encode_path() {
    static const int v = [] {
        const char *e = getenv("TQ_ENCODE_PATH");
        return (e && e[0] == '1') ? 1 : 0;
    }();
    return v;
}

bool tq_rows_map_4d(CUtensorMap *map, bool bf16, const void *base, int d, int64_t T, int H, int batch, int64_t sb,
                    int64_t sh, int64_t st);

// The TMA-fed encoder of one side, when it serves the call: 16-bit rows,
// the Walsh-Hadamard rotation, d in {64, 128}, and its shared memory and
// TMEM columns fit.  Returns false (nothing launched) otherwise.
static bool pipe_side(tq_ctx *ctx, bool keys, const void *x, tq_dtype dtype, int batch, int H, int64_t T, int64_t sb,
                      int64_t sh, int64_t st, const tq_codes *codes, int64_t token_offset, cudaStream_t stream,
                      int n_sms, cudaError_t *err) {
    if (dtype == TQ_F32 || (ctx->d != 64 && ctx->d != 128)) return false;
    // the Haar rotation: sqrt(d) Q in 2 (binary16 rows) or 3 (bfloat16 rows)
    // pieces; the key kernel then shares one residual buffer between its groups
    const bool haar = ctx->rotation == TQ_ROT_HAAR;
    if (haar) {
        if (!(dtype == TQ_BF16 ? (void *)ctx->d_Qbf : (void *)ctx->d_Qh)) return false;
    } else if (ctx->rotation != TQ_ROT_HADAMARD || !ctx->d_HD16 || !ctx->d_HDbf) {
        return false;
    }
    const int d = ctx->d, M = ctx->m;
    if (keys) {
        if (2 * (d + std::max(d, M)) > 512) return false;   // two groups' TMEM columns
        const int np = haar ? (dtype == TQ_BF16 ? 3 : 2) : 1;
        const size_t fixed = d == 128 ? (np == 1 ? PipeLayout<128, true, 2, 1>::FIXED
                                         : np == 2 ? PipeLayout<128, true, 2, 2>::FIXED : PipeLayout<128, true, 2, 3>::FIXED)
                                      : (np == 1 ? PipeLayout<64, true, 2, 1>::FIXED
                                         : np == 2 ? PipeLayout<64, true, 2, 2>::FIXED : PipeLayout<64, true, 2, 3>::FIXED);
        const size_t smem = fixed + (size_t)(d / 64) * M * 128;
        if (smem > 227 * 1024) return false;
    }
    if (T > 0x7FFFFFFF - ENC_ROWS) return false;
    CUtensorMap mx;
    if (!tq_rows_map_4d(&mx, dtype == TQ_BF16, x, d, T, H, batch, sb, sh, st)) return false;
    PipeParams p{};
    p.out = static_cast<uint8_t *>(keys ? codes->k : codes->v);
    p.capacity = codes->capacity;
    p.token_offset = token_offset;
    p.T = T;
    p.H = H;
    p.row_bytes = (int)tq_row_bytes(ctx, keys ? TQ_KEYS : TQ_VALUES);
    p.M = M;
    p.tiles_per_bh = (T + ENC_ROWS - 1) / ENC_ROWS;
    p.n_tiles = p.tiles_per_bh * (int64_t)batch * H;
    if (p.n_tiles > 0x7FFFFFFF) return false;   // the kernel's tile indices are 32-bit
    p.s_bytes = (uint32_t)((d / 64) * M * 128);
    p.status = ctx->d_status;
    p.norm_f16 = ctx->norm_f16;
    const int Bq = keys ? ctx->BK : ctx->BV;
    const float *cb = keys ? ctx->ck : ctx->cv;
    const float *bd = keys ? ctx->bk : ctx->bv;
    const int HBq = (1 << Bq) / 2;
    for (int i = 0; i < HBq; ++i) p.mag[i] = cb[HBq + i];
    for (int i = 0; i + 1 < HBq; ++i) p.pb[i] = bd[HBq + i];
    if (keys) key_centroid_form(cb, HBq, p.cl);
    const int grid = (int)std::min<int64_t>(p.n_tiles, n_sms > 0 ? n_sms : 148);
    const CUtensorMap &mhd = haar ? (dtype == TQ_BF16 ? ctx->tmap_Qbf : ctx->tmap_Q)
                                  : (dtype == TQ_BF16 ? ctx->tmap_HDbf : ctx->tmap_HD16);
    cudaError_t e;
    if (haar) {
        // sqrt(d) Q in 2 binary16 or 3 bfloat16 pieces
        const bool bf = dtype == TQ_BF16;
        if (d == 128)
            e = keys ? (bf ? launch_pipe<128, __nv_bfloat16, true, 3>(Bq, p, mx, mhd, ctx->tmap_S, grid, stream)
                           : launch_pipe<128, __half, true, 2>(Bq, p, mx, mhd, ctx->tmap_S, grid, stream))
                     : (bf ? launch_pipe<128, __nv_bfloat16, false, 3>(Bq, p, mx, mhd, ctx->tmap_S, grid, stream)
                           : launch_pipe<128, __half, false, 2>(Bq, p, mx, mhd, ctx->tmap_S, grid, stream));
        else
            e = keys ? (bf ? launch_pipe<64, __nv_bfloat16, true, 3>(Bq, p, mx, mhd, ctx->tmap_S, grid, stream)
                           : launch_pipe<64, __half, true, 2>(Bq, p, mx, mhd, ctx->tmap_S, grid, stream))
                     : (bf ? launch_pipe<64, __nv_bfloat16, false, 3>(Bq, p, mx, mhd, ctx->tmap_S, grid, stream)
                           : launch_pipe<64, __half, false, 2>(Bq, p, mx, mhd, ctx->tmap_S, grid, stream));
    } else if (d == 128) {
        e = dtype == TQ_BF16 ? (keys ? launch_pipe<128, __nv_bfloat16, true>(Bq, p, mx, mhd, ctx->tmap_S, grid, stream)
                                     : launch_pipe<128, __nv_bfloat16, false>(Bq, p, mx, mhd, ctx->tmap_S, grid, stream))
                             : (keys ? launch_pipe<128, __half, true>(Bq, p, mx, mhd, ctx->tmap_S, grid, stream)
                                     : launch_pipe<128, __half, false>(Bq, p, mx, mhd, ctx->tmap_S, grid, stream));
    } else {
        e = dtype == TQ_BF16 ? (keys ? launch_pipe<64, __nv_bfloat16, true>(Bq, p, mx, mhd, ctx->tmap_S, grid, stream)
                                     : launch_pipe<64, __nv_bfloat16, false>(Bq, p, mx, mhd, ctx->tmap_S, grid, stream))
                             : (keys ? launch_pipe<64, __half, true>(Bq, p, mx, mhd, ctx->tmap_S, grid, stream)
                                     : launch_pipe<64, __half, false>(Bq, p, mx, mhd, ctx->tmap_S, grid, stream));
    }
    *err = e;
    return true;
}

tq_status tq_launch_encode(tq_ctx *ctx, const void *k, const void *v, tq_dtype dtype, int batch, int H,
                           int64_t T, int64_t sb, int64_t sh, int64_t st, const tq_codes *codes,
                           int64_t token_offset, cudaStream_t stream, int n_sms) {
    if (tq_encode_path() != 1) {
        bool done_k = !k, done_v = !v;
        for (int side = 0; side < 2; ++side) {
            const bool keys = side == 0;
            const void *x = keys ? k : v;
            if (!x) continue;
            cudaError_t e = cudaSuccess;
            if (pipe_side(ctx, keys, x, dtype, batch, H, T, sb, sh, st, codes, token_offset, stream, n_sms, &e)) {
                tq_status s = tq_check_cuda(e);
                if (s != TQ_OK) return s;
                (keys ? done_k : done_v) = true;
            }
        }
        if (done_k && done_v) return TQ_OK;
        if (done_k) k = nullptr;
        if (done_v) v = nullptr;
    }
    const int64_t blocks_per_bh = (T + ENC_TILES * ENC_ROWS - 1) / (ENC_TILES * ENC_ROWS);
    const int64_t grid = blocks_per_bh * (int64_t)batch * H;
    if (grid == 0) return TQ_OK;
    if (grid > 0x7FFFFFFF) return TQ_ERR_LIMIT;
    for (int side = 0; side < 2; ++side) {
        const bool keys = side == 0;
        const void *x = keys ? k : v;
        if (!x) continue;
        EncodeParams p{};
        p.x = x;
        p.sb = sb;
        p.sh = sh;
        p.st = st;
        p.out = static_cast<uint8_t *>(keys ? codes->k : codes->v);
        p.capacity = codes->capacity;
        p.token_offset = token_offset;
        p.T = T;
        p.H = H;
        p.row_bytes = (int)tq_row_bytes(ctx, keys ? TQ_KEYS : TQ_VALUES);
        p.M = ctx->m;
        p.blocks_per_bh = blocks_per_bh;
        p.signs = ctx->d_signs;
        p.status = ctx->d_status;
        p.norm_f16 = ctx->norm_f16;
        const int B = keys ? ctx->BK : ctx->BV;
        const float *cb = keys ? ctx->ck : ctx->cv;
        const float *bd = keys ? ctx->bk : ctx->bv;
        const int HB = (1 << B) / 2;
        for (int i = 0; i < HB; ++i) p.mag[i] = cb[HB + i];
        for (int i = 0; i + 1 < HB; ++i) p.pb[i] = bd[HB + i];
        if (keys) key_centroid_form(cb, HB, p.cl);
        cudaError_t e;
        switch (dtype) {
            case TQ_F32: e = launch_side<float>(ctx, keys, p, grid, stream); break;
            case TQ_F16: e = launch_side<__half>(ctx, keys, p, grid, stream); break;
            case TQ_BF16: e = launch_side<__nv_bfloat16>(ctx, keys, p, grid, stream); break;
            default: return TQ_ERR_DIM_MISMATCH;
        }
        tq_status s = tq_check_cuda(e);
        if (s != TQ_OK) return s;
    }
    return TQ_OK;
}
