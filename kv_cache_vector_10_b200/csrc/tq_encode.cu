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

template <typename Tin>
struct Loader;

template <>
struct Loader<float> {
    template <int D>
    __device__ static void load(const float *src, float (&x)[D]) {
        const float4 *p = reinterpret_cast<const float4 *>(src);
#pragma unroll
        for (int i = 0; i < D / 4; ++i) {
            float4 q = __ldg(p + i);
            x[4 * i] = q.x; x[4 * i + 1] = q.y; x[4 * i + 2] = q.z; x[4 * i + 3] = q.w;
        }
    }
};

template <>
struct Loader<__half> {
    template <int D>
    __device__ static void load(const __half *src, float (&x)[D]) {
        const uint4 *p = reinterpret_cast<const uint4 *>(src);
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            uint4 q = __ldg(p + i);
            uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                __half2 h2 = *reinterpret_cast<__half2 *>(&w[e]);
                float2 f = __half22float2(h2);
                x[8 * i + 2 * e] = f.x;
                x[8 * i + 2 * e + 1] = f.y;
            }
        }
    }
};

template <>
struct Loader<__nv_bfloat16> {
    template <int D>
    __device__ static void load(const __nv_bfloat16 *src, float (&x)[D]) {
        const uint4 *p = reinterpret_cast<const uint4 *>(src);
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            uint4 q = __ldg(p + i);
            uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                x[8 * i + 2 * e] = __uint_as_float(w[e] << 16);
                x[8 * i + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
            }
        }
    }
};

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

// u <- H (D x) in place: sign flip from bit masks, then the butterflies.
template <int D>
__device__ __forceinline__ void rotate_unnormalised(float (&x)[D], const uint32_t *sw) {
#pragma unroll
    for (int w = 0; w < D / 32; ++w) {
        const uint32_t m = sw[w];
#pragma unroll
        for (int i = 0; i < 32; ++i)
            x[32 * w + i] = __uint_as_float(__float_as_uint(x[32 * w + i]) ^ ((m << (31 - i)) & 0x80000000u));
    }
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

// Number of positive boundaries at or below |u| (boundaries pre-scaled by n)
// and the magnitude of the selected centroid.
template <int HB>
__device__ __forceinline__ int quant_mag(float a, const float (&nb)[16], const float *mag, float &cm) {
    int cnt = 0;
    cm = mag[0];
#pragma unroll
    for (int k = 0; k < HB - 1; ++k) {
        const bool t = a >= nb[k];
        cnt += t ? 1 : 0;
        cm = t ? mag[k + 1] : cm;
    }
    return cnt;
}

template <int D, int BK, int BV, typename Tin>
__global__ void __launch_bounds__(ENC_GROUP, 1)
    tq_encode_kernel(const __grid_constant__ EncodeParams p, const __grid_constant__ CUtensorMap tmapS) {
    constexpr int LK = 1 << BK, HK = LK / 2;
    constexpr int LV = 1 << BV, HV = LV / 2;
    constexpr int NW = D / 32;                 // 32-bit words per bit plane
    constexpr int ATOM = ENC_GROUP * 128;      // bytes of one 128-row x 128-byte swizzle column
    constexpr int A_BYTES = (D / 64) * ATOM;   // one residual pass
    (void)LK; (void)LV;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid / 32;
    // Blocks [0, k_blocks) encode keys, the rest encode values.
    const bool is_key = blockIdx.x < p.k_blocks;
    const int64_t blk = is_key ? blockIdx.x : blockIdx.x - p.k_blocks;
    const int64_t bh = blk / p.blocks_per_bh;
    const int head = (int)(bh % p.H);
    const int64_t b = bh / p.H;
    const int64_t tb0 = (blk % p.blocks_per_bh) * (int64_t)ENC_TILES * ENC_GROUP;
    uint32_t sw[NW];
#pragma unroll
    for (int w = 0; w < NW; ++w) sw[w] = __ldg(p.signs + (int64_t)head * NW + w);
    const Tin *src = reinterpret_cast<const Tin *>(is_key ? p.k : p.v) + b * p.sb + (int64_t)head * p.sh;

    if (!is_key) {
        // ------------------------------------------------------- values
        constexpr int VW = BV * D / 32;
        for (int tile = 0; tile < ENC_TILES; ++tile) {
            const int64_t t = tb0 + tile * ENC_GROUP + tid;
            if (t >= p.T) break;
            float x[D];
            Loader<Tin>::template load<D>(src + t * p.st, x);
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
                rotate_unnormalised<D>(x, sw);
                float nb[16];
#pragma unroll
                for (int k2 = 0; k2 < HV - 1; ++k2) nb[k2] = n * p.book.vpb[k2];
                float c2 = 0.f;
#pragma unroll
                for (int j = 0; j < D; ++j) {
                    float cm;
                    const int cnt = quant_mag<HV>(fabsf(x[j]), nb, p.book.vmag, cm);
                    const uint32_t idx = (uint32_t)(x[j] >= 0.f ? HV + cnt : HV - 1 - cnt);
                    c2 = fmaf(cm, cm, c2);
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
    uint8_t *sS = smem;                                   // [D/64][M rows][128 B]
    uint8_t *sA = smem + (D / 64) * M * 128;              // [pass][D/64][128 rows][128 B]
    uint64_t *bars = reinterpret_cast<uint64_t *>(sA + 2 * A_BYTES);  // [0] S loaded, [1] MMA done
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bars + 2);
    int *s_abort = reinterpret_cast<int *>(s_tmem + 1);
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
    for (int tile = 0; tile < ENC_TILES; ++tile) {
        const int64_t tt0 = tb0 + tile * ENC_GROUP;
        if (tt0 >= p.T) break;
        const int64_t t = tt0 + tid;
        const bool valid = t < p.T;
        uint8_t *rowp = p.kc + (bh * p.capacity + p.token_offset + t) * p.krow;
        {
            float x[D];
            float n = 0.f;
            if (valid) {
                Loader<Tin>::template load<D>(src + t * p.st, x);
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
                rotate_unnormalised<D>(x, sw);
                float nb[16];
#pragma unroll
                for (int k2 = 0; k2 < HK - 1; ++k2) nb[k2] = n * p.book.kpb[k2];
                // pass 1: squared norm of the selected centroids
                float c2 = 0.f;
#pragma unroll
                for (int j = 0; j < D; ++j) {
                    float cm;
                    quant_mag<HK>(fabsf(x[j]), nb, p.book.kmag, cm);
                    c2 = fmaf(cm, cm, c2);
                }
                ns = n * sqrtf((float)D / c2);
                // pass 2: index planes and the residual u - n_s C[idx]
                float e2 = 0.f;
#pragma unroll
                for (int w = 0; w < NW; ++w) {
                    uint32_t pl[BK];
#pragma unroll
                    for (int q = 0; q < BK; ++q) pl[q] = 0u;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int j = 32 * w + i;
                        float cm;
                        const int cnt = quant_mag<HK>(fabsf(x[j]), nb, p.book.kmag, cm);
                        const bool pos = x[j] >= 0.f;
                        const int idx = pos ? HK + cnt : HK - 1 - cnt;
#pragma unroll
                        for (int q = 0; q < BK; ++q) pl[q] |= (uint32_t)((idx >> q) & 1) << i;
                        x[j] = fmaf(-ns, pos ? cm : -cm, x[j]);
                        e2 = fmaf(x[j], x[j], e2);
                    }
                    uint32_t *dst = reinterpret_cast<uint32_t *>(rowp);
#pragma unroll
                    for (int q = 0; q < BK; ++q) dst[q * NW + w] = pl[q];
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
    const size_t smem = 1024 + (size_t)(D / 64) * p.M * 128 + 2 * (size_t)(D / 64) * ENC_GROUP * 128 + 64;
    auto kern = tq_encode_kernel<D, BK, BV, Tin>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
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
