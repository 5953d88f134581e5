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
// Kernel design (CTAs of 128 threads, one thread per row; a CTA covers
// ENC_TILES x 128 consecutive tokens of one (batch, head); the first half
// of the grid encodes keys, the second half values, so each thread holds a
// single row and the hardware scheduler interleaves both kinds):
//   * A row lives in its thread's registers: 128-bit loads, norm, sign flip
//     and the full 7-stage butterfly without any shuffle, quantization
//     against the codebook boundaries scaled by n, bit-plane / field packing.
//   * The key residual, normalised to |e| = sqrt(d) and split into binary16
//     hi + lo parts, is written to shared memory in the 128-byte-swizzled
//     K-major layout; one thread per group issues 2*(d/16) tcgen05.mma
//     (M = 128 rows, N = m projections, K = 16) against S (binary16, loaded
//     once per head by TMA), accumulating P = e S^T in fp32 in TMEM.  The two
//     passes make the projection accurate to ~1e-7 relative, so sign bits
//     agree with an fp64 evaluation away from |p| ~ 1e-6.
//   * Epilogue: each thread reads its row of P from TMEM (tcgen05.ld
//     32x32b), turns signs into the m-bit plane and stores it.
#include <float.h>

#include "tq_internal.cuh"

namespace {

constexpr int ENC_GROUP = 128;   // threads per CTA = rows per tile = MMA M
constexpr int ENC_TILES = 4;     // tiles per CTA (S is loaded once per CTA)

struct EncodeParams {
    const void *k;
    const void *v;
    int64_t sb, sh, st;     // input strides in elements
    uint8_t *kc;
    uint8_t *vc;
    int64_t capacity, token_offset, T;
    int H;
    int krow, vrow;
    int M;
    int64_t blocks_per_bh, k_blocks;
    const uint32_t *signs;  // [heads][d/32]
    unsigned long long *status;
    TqBook book;
};

// Row loaders.  The rotation's random signs are applied while converting:
// `sm` holds, per 32-bit input word, a mask with the sign bit of every
// element that D flips (bits 15/31 for 16-bit types, bit 31 for fp32).
template <typename Tin>
struct Loader;

template <>
struct Loader<float> {
    template <int D>
    __device__ static void load(const float *src, const uint32_t *sm, float (&x)[D]) {
        const uint4 *p = reinterpret_cast<const uint4 *>(src);
        const uint4 *m = reinterpret_cast<const uint4 *>(sm);
#pragma unroll
        for (int i = 0; i < D / 4; ++i) {
            const uint4 q = __ldg(p + i), f = m[i];
            x[4 * i] = __uint_as_float(q.x ^ f.x);
            x[4 * i + 1] = __uint_as_float(q.y ^ f.y);
            x[4 * i + 2] = __uint_as_float(q.z ^ f.z);
            x[4 * i + 3] = __uint_as_float(q.w ^ f.w);
        }
    }
};

template <>
struct Loader<__half> {
    template <int D>
    __device__ static void load(const __half *src, const uint32_t *sm, float (&x)[D]) {
        const uint4 *p = reinterpret_cast<const uint4 *>(src);
        const uint4 *m = reinterpret_cast<const uint4 *>(sm);
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
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
struct Loader<__nv_bfloat16> {
    template <int D>
    __device__ static void load(const __nv_bfloat16 *src, const uint32_t *sm, float (&x)[D]) {
        const uint4 *p = reinterpret_cast<const uint4 *>(src);
        const uint4 *m = reinterpret_cast<const uint4 *>(sm);
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
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

template <typename Tin>
constexpr int mask_words(int D) { return sizeof(Tin) == 4 ? D : D / 2; }

// Per-head input sign masks: word w covers the elements stored in input
// word w.
template <typename Tin, int D>
__device__ void build_sign_masks(const uint32_t *signs, uint32_t *sm) {
    for (int w = threadIdx.x; w < mask_words<Tin>(D); w += blockDim.x) {
        if constexpr (sizeof(Tin) == 4) {
            sm[w] = ((signs[w / 32] >> (w % 32)) & 1u) << 31;
        } else {
            const int j = 2 * w;
            sm[w] = (((signs[j / 32] >> (j % 32)) & 1u) << 15) | (((signs[(j + 1) / 32] >> ((j + 1) % 32)) & 1u) << 31);
        }
    }
}

// Norm of a row held in registers.  Returns -1 for a row with a non-finite
// value, 0 for an all-zero row.  Rows whose sum of squares over- or
// underflows fp32 are rescaled by their largest magnitude.
template <int D>
__device__ __forceinline__ float row_norm(const float (&x)[D]) {
    float n2 = 0.f;
#pragma unroll
    for (int j = 0; j < D; ++j) n2 = fmaf(x[j], x[j], n2);
    if (n2 >= 1e-30f && n2 <= 1e30f) return sqrtf(n2);
    float mx = 0.f;
    bool bad = false;
#pragma unroll
    for (int j = 0; j < D; ++j) {
        bad |= !isfinite(x[j]);
        mx = fmaxf(mx, fabsf(x[j]));
    }
    if (bad) return -1.f;
    if (mx == 0.f) return 0.f;
    const float inv = 1.f / mx;
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < D; ++j) {
        const float t = x[j] * inv;
        acc = fmaf(t, t, acc);
    }
    return mx * sqrtf(acc);
}

// u <- H u in place (the signs were applied by the loader).
template <int D>
__device__ __forceinline__ void fwht_inplace(float (&x)[D]) {
#pragma unroll
    for (int len = 1; len < D; len <<= 1) {
#pragma unroll
        for (int i = 0; i < D; i += 2 * len) {
#pragma unroll
            for (int j = i; j < i + len; ++j) {
                const float a = x[j], b = x[j + len];
                x[j] = a + b;
                x[j + len] = a - b;
            }
        }
    }
}

// Magnitude index of a = |u| among the HB cells of the positive half of the
// codebook: the number of positive boundaries nb[k] (pre-scaled by n) with
// a >= nb[k], found by a branchless binary search (bit k of the result is
// decided at level k from the top).
template <int HB>
__device__ __forceinline__ uint32_t mag_index(float a, const float (&nb)[16]) {
    if constexpr (HB == 1) {
        return 0u;
    } else if constexpr (HB == 2) {
        return a >= nb[0] ? 1u : 0u;
    } else if constexpr (HB == 4) {
        const bool t1 = a >= nb[1];
        const bool t0 = a >= (t1 ? nb[2] : nb[0]);
        return (t1 ? 2u : 0u) | (t0 ? 1u : 0u);
    } else if constexpr (HB == 8) {
        const bool t2 = a >= nb[3];
        const bool t1 = a >= (t2 ? nb[5] : nb[1]);
        const float b0 = t2 ? (t1 ? nb[6] : nb[4]) : (t1 ? nb[2] : nb[0]);
        const bool t0 = a >= b0;
        return (t2 ? 4u : 0u) | (t1 ? 2u : 0u) | (t0 ? 1u : 0u);
    } else {
        const bool t3 = a >= nb[7];
        const bool t2 = a >= (t3 ? nb[11] : nb[3]);
        const bool t1 = a >= (t3 ? (t2 ? nb[13] : nb[9]) : (t2 ? nb[5] : nb[1]));
        const float b0 = t3 ? (t2 ? (t1 ? nb[14] : nb[12]) : (t1 ? nb[10] : nb[8]))
                            : (t2 ? (t1 ? nb[6] : nb[4]) : (t1 ? nb[2] : nb[0]));
        const bool t0 = a >= b0;
        return (t3 ? 8u : 0u) | (t2 ? 4u : 0u) | (t1 ? 2u : 0u) | (t0 ? 1u : 0u);
    }
}

template <int D, int BK, int BV, typename Tin>
__global__ void __launch_bounds__(ENC_GROUP, 1)
    tq_encode_kernel(const __grid_constant__ EncodeParams p, const __grid_constant__ CUtensorMap tmapS) {
    constexpr int HK = (1 << BK) / 2;
    constexpr int HV = (1 << BV) / 2;
    constexpr int NW = D / 32;                 // 32-bit words per bit plane
    constexpr int ATOM = ENC_GROUP * 128;      // bytes of one 128-row x 128-byte swizzle column
    constexpr int A_BYTES = (D / 64) * ATOM;   // one residual pass
    constexpr int MW = mask_words<Tin>(D);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // misc region [0, 1024): sign masks, centroid magnitudes, barriers
    uint32_t *s_mask = reinterpret_cast<uint32_t *>(smem);                 // [MW] (<= 512 B)
    float *s_mag = reinterpret_cast<float *>(smem + 512);                   // [16] magnitudes
    float *s_mag2 = s_mag + 16;                                             // [16] squared
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 768);              // [0] S loaded, [1] MMA done
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bars + 2);
    int *s_abort = reinterpret_cast<int *>(s_tmem + 1);
    const int tid = threadIdx.x, warp = tid / 32;
    // Blocks [0, k_blocks) encode keys, the rest encode values.
    const bool is_key = blockIdx.x < p.k_blocks;
    const int64_t blk = is_key ? blockIdx.x : blockIdx.x - p.k_blocks;
    const int64_t bh = blk / p.blocks_per_bh;
    const int head = (int)(bh % p.H);
    const int64_t b = bh / p.H;
    const int64_t tb0 = (blk % p.blocks_per_bh) * (int64_t)ENC_TILES * ENC_GROUP;
    build_sign_masks<Tin, D>(p.signs + (int64_t)head * NW, s_mask);
    if (tid < 16) {
        const float mg = is_key ? (tid < HK ? p.book.kmag[tid] : 0.f) : (tid < HV ? p.book.vmag[tid] : 0.f);
        s_mag[tid] = mg;
        s_mag2[tid] = mg * mg;
    }
    const Tin *src = reinterpret_cast<const Tin *>(is_key ? p.k : p.v) + b * p.sb + (int64_t)head * p.sh;

    if (!is_key) {
        __syncthreads();
        // ------------------------------------------------------- values
        constexpr int VW = BV * D / 32;
        for (int tile = 0; tile < ENC_TILES; ++tile) {
            const int64_t t = tb0 + tile * ENC_GROUP + tid;
            if (t >= p.T) break;
            float x[D];
            Loader<Tin>::template load<D>(src + t * p.st, s_mask, x);
            const float n = row_norm<D>(x);
            if (n < 0.f) atomicAdd(&p.status[0], 1ull);
            uint32_t f[VW];
#pragma unroll
            for (int w = 0; w < VW; ++w) f[w] = 0u;
            float ns = 0.f;
            if (n <= 0.f) {
#pragma unroll
                for (int j = 0; j < D; ++j) {
                    const int bit = BV * j;
                    f[bit / 32] |= (uint32_t)HV << (bit % 32);
                    if ((bit % 32) + BV > 32) f[bit / 32 + 1] |= (uint32_t)HV >> (32 - bit % 32);
                }
            } else {
                fwht_inplace<D>(x);
                float nb[16];
#pragma unroll
                for (int k2 = 0; k2 < HV - 1; ++k2) nb[k2] = n * p.book.vpb[k2];
                float c2 = 0.f;
#pragma unroll
                for (int j = 0; j < D; ++j) {
                    const uint32_t cnt = mag_index<HV>(fabsf(x[j]), nb);
                    const uint32_t idx = x[j] < 0.f ? (uint32_t)(HV - 1) - cnt : (uint32_t)HV + cnt;
                    c2 += s_mag2[cnt];
                    const int bit = BV * j;
                    f[bit / 32] |= idx << (bit % 32);
                    if ((bit % 32) + BV > 32) f[bit / 32 + 1] |= idx >> (32 - bit % 32);
                }
                ns = n * sqrtf((float)D / c2);
            }
            uint32_t *dst = reinterpret_cast<uint32_t *>(p.vc + (bh * p.capacity + p.token_offset + t) * p.vrow);
#pragma unroll
            for (int w = 0; w < VW; ++w) dst[w] = f[w];
            dst[VW] = __float_as_uint(ns);
        }
        return;
    }

    // ------------------------------------------------------------- keys
    const int M = p.M;
    uint8_t *sS = smem + 1024;                            // [D/64][M rows][128 B]
    uint8_t *sA = sS + (D / 64) * M * 128;                // [pass][D/64][128 rows][128 B]
    const uint32_t tmem_cols = M <= 128 ? 128u : 256u;
    if (tid == 0) {
        tqdev::mbar_init(&bars[0], 1);
        tqdev::mbar_init(&bars[1], 1);
        *s_abort = 0;
        tqdev::fence_barrier_init();
    }
    if (warp == 0) tqdev::tmem_alloc(s_tmem, tmem_cols);
    tqdev::tc_fence_before();
    __syncthreads();
    tqdev::tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    if (tid == 0) {
        tqdev::mbar_expect_tx(&bars[0], (uint32_t)(M * D * 2));
#pragma unroll
        for (int a = 0; a < D / 64; ++a) tqdev::tma_load_2d(sS + a * M * 128, &tmapS, a * 64, head * M, &bars[0]);
    }
    const float inv_sqrt_d = rsqrtf((float)D);
    uint8_t *aHi = sA, *aLo = sA + A_BYTES;
    if (tid == 0 && tqdev::status_aborted(p.status)) *s_abort = 1;
    __syncthreads();
    for (int tile = 0; tile < ENC_TILES && !*s_abort; ++tile) {
        const int64_t tt0 = tb0 + tile * ENC_GROUP;
        if (tt0 >= p.T) break;
        const int64_t t = tt0 + tid;
        const bool valid = t < p.T;
        uint8_t *rowp = p.kc + (bh * p.capacity + p.token_offset + t) * p.krow;
        {
            float x[D];
            float n = 0.f;
            if (valid) {
                Loader<Tin>::template load<D>(src + t * p.st, s_mask, x);
                n = row_norm<D>(x);
                if (n < 0.f) atomicAdd(&p.status[0], 1ull);
            }
            float ns = 0.f, gamma = 0.f;
            if (!valid || n <= 0.f) {
#pragma unroll
                for (int c = 0; c < D / 8; ++c) {
                    const int off = (c / 8) * ATOM + tid * 128 + (((c % 8) ^ (tid & 7)) << 4);
                    *reinterpret_cast<uint4 *>(aHi + off) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4 *>(aLo + off) = make_uint4(0, 0, 0, 0);
                }
                if (valid) {
                    uint32_t *dst = reinterpret_cast<uint32_t *>(rowp);
#pragma unroll
                    for (int q = 0; q < BK; ++q)
#pragma unroll
                        for (int w = 0; w < NW; ++w) dst[q * NW + w] = ((HK >> q) & 1) ? 0xFFFFFFFFu : 0u;
                }
            } else {
                fwht_inplace<D>(x);
                float nb[16];
#pragma unroll
                for (int k2 = 0; k2 < HK - 1; ++k2) nb[k2] = n * p.book.kpb[k2];
                // pass 1: magnitude and sign bits of every index, squared centroid norm
                float c2 = 0.f;
                uint32_t *dst = reinterpret_cast<uint32_t *>(rowp);
                uint32_t mb[BK > 1 ? BK - 1 : 1][NW];
#pragma unroll
                for (int w = 0; w < NW; ++w) {
                    uint32_t negw = 0u;
#pragma unroll
                    for (int q = 0; q < BK - 1; ++q) mb[q][w] = 0u;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float u = x[32 * w + i];
                        const uint32_t cnt = mag_index<HK>(fabsf(u), nb);
                        negw |= (__float_as_uint(u) >> 31) << i;
#pragma unroll
                        for (int q = 0; q < BK - 1; ++q) mb[q][w] |= ((cnt >> q) & 1u) << i;
                        c2 += s_mag2[cnt];
                    }
                    // ascending index: top bit = non-negative, low bits = magnitude
                    // index, complemented for negative values
#pragma unroll
                    for (int q = 0; q < BK - 1; ++q) dst[q * NW + w] = mb[q][w] ^ negw;
                    dst[(BK - 1) * NW + w] = ~negw;
                }
                ns = n * sqrtf((float)D / c2);
                // Hide the packed words' provenance so the compiler re-extracts
                // the bits instead of keeping 128 indices live across passes.
#pragma unroll
                for (int q = 0; q < BK - 1; ++q)
#pragma unroll
                    for (int w = 0; w < NW; ++w) asm volatile("" : "+r"(mb[q][w]));
                // pass 2: residual u - n_s C[idx], the magnitude index read back
                // from the packed bits
                float e2 = 0.f;
#pragma unroll
                for (int j = 0; j < D; ++j) {
                    const float u = x[j];
                    uint32_t cnt = 0u;
#pragma unroll
                    for (int q = 0; q < BK - 1; ++q) cnt |= ((mb[q][j / 32] >> (j % 32)) & 1u) << q;
                    const float c = copysignf(s_mag[cnt], u);
                    x[j] = fmaf(-ns, c, u);
                    e2 = fmaf(x[j], x[j], e2);
                }
                gamma = sqrtf(e2) * inv_sqrt_d;
                // pass 3: |e| = sqrt(d) scaled residual as binary16 hi + lo, swizzled K-major
                const float sc = e2 > 0.f ? sqrtf((float)D / e2) : 0.f;
#pragma unroll
                for (int c = 0; c < D / 8; ++c) {
                    uint32_t hw[4], lw[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float a0 = x[8 * c + 2 * e] * sc, a1 = x[8 * c + 2 * e + 1] * sc;
                        const __half2 hh = __floats2half2_rn(a0, a1);
                        const float2 hf = __half22float2(hh);
                        const __half2 ll = __floats2half2_rn(a0 - hf.x, a1 - hf.y);
                        hw[e] = (uint32_t)__half_as_ushort(__low2half(hh)) | ((uint32_t)__half_as_ushort(__high2half(hh)) << 16);
                        lw[e] = (uint32_t)__half_as_ushort(__low2half(ll)) | ((uint32_t)__half_as_ushort(__high2half(ll)) << 16);
                    }
                    const int off = (c / 8) * ATOM + tid * 128 + (((c % 8) ^ (tid & 7)) << 4);
                    *reinterpret_cast<uint4 *>(aHi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                    *reinterpret_cast<uint4 *>(aLo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                }
            }
            if (valid) {
                uint32_t *dst = reinterpret_cast<uint32_t *>(rowp);
                const int tail = BK * NW + M / 32;
                dst[tail] = __float_as_uint(ns);
                dst[tail + 1] = __float_as_uint(gamma);
            }
        }
        tqdev::fence_proxy_async_smem();
        tqdev::tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            bool ok = tile > 0 || tqdev::mbar_wait_bounded(&bars[0], 0);
            if (!ok) {
                atomicOr(reinterpret_cast<unsigned int *>(&p.status[1]), TQ_FLAG_WAIT_TIMEOUT);
                *s_abort = 1;
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
                        tqdev::mma_f16_ss(tmem_base, tqdev::smem_desc_sw128(a_addr), tqdev::smem_desc_sw128(b_addr),
                                          idesc, (pass | ks) != 0);
                    }
                }
                tqdev::mma_commit(&bars[1]);
            }
        }
        __syncthreads();
        if (*s_abort) break;
        // ---------------------------------------------- sign epilogue
        if (!tqdev::mbar_wait_bounded(&bars[1], (uint32_t)(tile & 1))) {
            if (tid == 0) atomicOr(reinterpret_cast<unsigned int *>(&p.status[1]), TQ_FLAG_WAIT_TIMEOUT);
            *s_abort = 1;   // benign race: every writer stores 1
        } else {
            tqdev::tc_fence_after();
            uint32_t *dst = reinterpret_cast<uint32_t *>(rowp) + BK * NW;
            const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
            for (int c = 0; c < M / 32; ++c) {
                float pv[32];
                tqdev::tmem_ld_32x32b_x32(tmem_base + lane_base + (uint32_t)(c * 32), pv);
                uint32_t word = 0u;
#pragma unroll
                for (int i = 0; i < 32; ++i) word |= (pv[i] >= 0.f ? 1u : 0u) << i;
                if (valid) dst[c] = word;
            }
        }
        tqdev::tc_fence_before();
        __syncthreads();
        tqdev::tc_fence_after();
        if (*s_abort) break;
    }
    __syncthreads();
    if (warp == 0) {
        tqdev::tc_fence_after();
        tqdev::tmem_dealloc(tmem_base, tmem_cols);
    }
}

template <int D, int BK, int BV, typename Tin>
cudaError_t launch_t(const EncodeParams &p, const CUtensorMap &map, int grid, cudaStream_t s) {
    const size_t smem = 2048 + (size_t)(D / 64) * p.M * 128 + 2 * (size_t)(D / 64) * ENC_GROUP * 128;
    auto kern = tq_encode_kernel<D, BK, BV, Tin>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) {
        cudaGetLastError();   // do not leave the failure as the thread's sticky last error
        return e;
    }
    kern<<<grid, ENC_GROUP, smem, s>>>(p, map);
    return cudaGetLastError();
}

template <int D, typename Tin>
cudaError_t launch_bits(int bits, const EncodeParams &p, const CUtensorMap &map, int grid, cudaStream_t s) {
    switch (bits) {
        case 2: return launch_t<D, 1, 2, Tin>(p, map, grid, s);
        case 3: return launch_t<D, 2, 3, Tin>(p, map, grid, s);
        case 4: return launch_t<D, 3, 4, Tin>(p, map, grid, s);
        case 5: return launch_t<D, 4, 5, Tin>(p, map, grid, s);
    }
    return cudaErrorInvalidValue;
}

template <typename Tin>
cudaError_t launch_dim(int d, int bits, const EncodeParams &p, const CUtensorMap &map, int grid, cudaStream_t s) {
    if (d == 128) return launch_bits<128, Tin>(bits, p, map, grid, s);
    if (d == 64) return launch_bits<64, Tin>(bits, p, map, grid, s);
    return cudaErrorInvalidValue;
}

}  // namespace

tq_status tq_launch_encode(tq_ctx *ctx, const void *k, const void *v, tq_dtype dtype, int batch, int H,
                           int64_t T, int64_t sb, int64_t sh, int64_t st, const tq_codes *codes,
                           int64_t token_offset, cudaStream_t stream, int n_sms) {
    EncodeParams p{};
    p.k = k;
    p.v = v;
    p.sb = sb; p.sh = sh; p.st = st;
    p.kc = static_cast<uint8_t *>(codes->k);
    p.vc = static_cast<uint8_t *>(codes->v);
    p.capacity = codes->capacity;
    p.token_offset = token_offset;
    p.T = T;
    p.H = H;
    p.krow = (int)tq_row_bytes(ctx, TQ_KEYS);
    p.vrow = (int)tq_row_bytes(ctx, TQ_VALUES);
    p.M = ctx->m;
    p.blocks_per_bh = (T + ENC_TILES * ENC_GROUP - 1) / (ENC_TILES * ENC_GROUP);
    const int64_t per_side = p.blocks_per_bh * (int64_t)batch * H;
    p.k_blocks = k ? per_side : 0;
    p.signs = ctx->d_signs;
    p.status = ctx->d_status;
    const int HK = (1 << ctx->BK) / 2, HV = (1 << ctx->BV) / 2;
    for (int i = 0; i < HK; ++i) p.book.kmag[i] = ctx->ck[HK + i];
    for (int i = 0; i + 1 < HK; ++i) p.book.kpb[i] = ctx->bk[HK + i];
    for (int i = 0; i < HV; ++i) p.book.vmag[i] = ctx->cv[HV + i];
    for (int i = 0; i + 1 < HV; ++i) p.book.vpb[i] = ctx->bv[HV + i];
    const int64_t total = p.k_blocks + (v ? per_side : 0);
    if (total == 0) return TQ_OK;
    if (total > 0x7FFFFFFF) return TQ_ERR_LIMIT;
    const int grid = (int)total;
    (void)n_sms;
    cudaError_t e;
    switch (dtype) {
        case TQ_F32: e = launch_dim<float>(ctx->d, ctx->bits, p, ctx->tmap_S, grid, stream); break;
        case TQ_F16: e = launch_dim<__half>(ctx->d, ctx->bits, p, ctx->tmap_S, grid, stream); break;
        case TQ_BF16: e = launch_dim<__nv_bfloat16>(ctx->d, ctx->bits, p, ctx->tmap_S, grid, stream); break;
        default: return TQ_ERR_DIM_MISMATCH;
    }
    return tq_check_cuda(e);
}
