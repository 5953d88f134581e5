// tq_aux.cu -- exact-path scores, dequantization, decode query preparation
// and the log-sum-exp combine of split-K partials (sm_100a).
//
//  * Scores (bitpolar src/kv_cache.rs, KvCacheCompressor::attention_scores;
//    pre-softmax, scaled by 1/sqrt(head_dim)), estimated from the codes:
//      s = [n_s <q_rot, C[idx]>/sqrt(d) + sqrt(pi/2)/m gamma <S q_rot, 2b-1>] / sqrt(d),
//    q_rot = Pi q (turboquant-plus-rs README, Architecture: TurboQuant
//    inner-product estimator; QJL removes the bias).
//  * Dequantization (bitpolar decode_values):
//      v_hat = n_s Pi^T C[idx]/sqrt(d),
//      k_hat = Pi^T (n_s C[idx]/sqrt(d) + sqrt(pi/2)/m gamma S^T (2b-1)).
//  * Decode query preparation: q_rot and S q_rot per (segment, sequence,
//    head), consumed by the split-K kernel's per-query lookup tables.
//  * Combine: partials (running max, sum, unnormalised output) of all
//    splits and segments of a (sequence, head) merged by log-sum-exp.
#include "tq_decode.cuh"

namespace {

constexpr int AUX_THREADS = 128;

// Block-wide: q_rot = H (D q) / sqrt(d) and sq = S q_rot, in shared memory.
// Warp 0 rotates (lane l holds coordinates l + 32k: the stages of stride
// >= 32 run in registers, the others across lanes by shuffles); then each
// thread computes whole projections sq_i = <S_i, q_rot>, with all 16-byte
// loads of its row of S in flight at once.
template <int D>
__device__ void prep_query(const float *sq_in, const uint32_t *signs, const __half *S, int M, float *s_qr,
                           float *s_sq, const float *Q) {
    const int tid = threadIdx.x;
    if (Q) {
        // Haar rotation: q_rot = Q q, one output per thread
        for (int i = tid; i < D; i += blockDim.x) {
            const float4 *row = reinterpret_cast<const float4 *>(Q + (int64_t)i * D);
            float a0 = 0.f, a1 = 0.f;
#pragma unroll 8
            for (int c = 0; c < D / 4; ++c) {
                const float4 w = __ldg(row + c);
                a0 = fmaf(w.x, sq_in[4 * c], a0);
                a1 = fmaf(w.y, sq_in[4 * c + 1], a1);
                a0 = fmaf(w.z, sq_in[4 * c + 2], a0);
                a1 = fmaf(w.w, sq_in[4 * c + 3], a1);
            }
            s_qr[i] = a0 + a1;
        }
    } else if (tid < 32) {
        constexpr int V = D / 32;
        const int lane = tid;
        float x[V];
#pragma unroll
        for (int k = 0; k < V; ++k) {
            const int j = lane + 32 * k;
            const float v = sq_in[j];
            x[k] = ((signs[j / 32] >> (j % 32)) & 1) ? -v : v;
        }
#pragma unroll
        for (int len = 1; len < V; len <<= 1)
#pragma unroll
            for (int k = 0; k < V; k += 2 * len)
#pragma unroll
                for (int kk = k; kk < k + len; ++kk) {
                    const float a = x[kk], b = x[kk + len];
                    x[kk] = a + b;
                    x[kk + len] = a - b;
                }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const bool upper = (lane & o) != 0;
#pragma unroll
            for (int k = 0; k < V; ++k) {
                const float y = __shfl_xor_sync(0xffffffffu, x[k], o);
                x[k] = upper ? y - x[k] : x[k] + y;
            }
        }
        const float sc = rsqrtf((float)D);
#pragma unroll
        for (int k = 0; k < V; ++k) s_qr[lane + 32 * k] = x[k] * sc;
    }
    __syncthreads();
    const float4 *q4 = reinterpret_cast<const float4 *>(s_qr);
    for (int i = tid; i < M; i += blockDim.x) {
        const uint4 *row = reinterpret_cast<const uint4 *>(S + (int64_t)i * D);
        uint4 w[D / 8];
#pragma unroll
        for (int c = 0; c < D / 8; ++c) w[c] = __ldg(row + c);
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
            const float4 qa = q4[2 * c], qb = q4[2 * c + 1];
            const float2 f0 = __half22float2(*reinterpret_cast<const __half2 *>(&w[c].x));
            const float2 f1 = __half22float2(*reinterpret_cast<const __half2 *>(&w[c].y));
            const float2 f2 = __half22float2(*reinterpret_cast<const __half2 *>(&w[c].z));
            const float2 f3 = __half22float2(*reinterpret_cast<const __half2 *>(&w[c].w));
            acc0 = fmaf(f0.x, qa.x, acc0);
            acc1 = fmaf(f0.y, qa.y, acc1);
            acc0 = fmaf(f1.x, qa.z, acc0);
            acc1 = fmaf(f1.y, qa.w, acc1);
            acc0 = fmaf(f2.x, qb.x, acc0);
            acc1 = fmaf(f2.y, qb.y, acc1);
            acc0 = fmaf(f3.x, qb.z, acc0);
            acc1 = fmaf(f3.y, qb.w, acc1);
        }
        s_sq[i] = acc0 + acc1;
    }
    __syncthreads();
}

struct ScoresParams {
    const uint8_t *kc;
    const float *q;
    float *scores;
    const uint32_t *signs;
    const __half *S;
    const float *Q;            // Haar rotation, or nullptr
    int64_t capacity, T;
    int Hq, Hkv, M, krow, bk;
    int kf16;                  // key norms as binary16
    int n_planes;              // sigma-planes: odd subsets of the index bits
    uint32_t plane_sets[8];    // index planes XOR-ed into sigma-plane s
    float alpha[8];            // Walsh coefficient of sigma-plane s
};

// One block of SCORE_THREADS per (token block, query head, sequence); every
// thread scores SCORE_TPT tokens, so the query preparation and the tables
// are amortized over SCORE_TPT * SCORE_THREADS tokens, and many resident
// warps cover the latency of each thread's row loads.
constexpr int SCORE_THREADS = 512;
constexpr int SCORE_TPT = 4;

// Scores from byte tables (the decode kernel's method, one thread per token):
// the codebook is antisymmetric, so C[idx_j] = sum_s alpha_s sigma_s,j with
// sigma_s,j = +-1 the parity of the index bits in the odd set s; for byte
// position g of a plane, T_g[x] = sum_{i<8} v[8g + i] (2 bit_i(x) - 1) with v =
// q_rot gives sum_j q_rot,j sigma_s,j as sum_g T_g[sigma-byte_g], and v = S q_rot
// gives <S q_rot, 2b - 1> from the sign plane's bytes.  Tables: [position][256]
// in dynamic shared memory, index positions (d/8) first, then sign positions
// (m/8).
template <int D>
__global__ void __launch_bounds__(SCORE_THREADS) tq_scores_kernel(const __grid_constant__ ScoresParams p) {
    __shared__ __align__(16) float s_qr[D];
    __shared__ float s_sq[256];
    extern __shared__ float s_tab[];
    constexpr int PK = D / 8, NW = D / 32;
    const int j = blockIdx.y, b = blockIdx.z;
    const int h = j / (p.Hq / p.Hkv);
    prep_query<D>(p.q + ((int64_t)b * p.Hq + j) * D, p.signs + (int64_t)h * (D / 32), p.S + (int64_t)h * p.M * D,
                  p.M, s_qr, s_sq, p.Q ? p.Q + (int64_t)h * D * D : nullptr);   // ends with a barrier
    const int PS = p.M / 8;
    for (int e = threadIdx.x; e < (PK + PS) * 256; e += blockDim.x) {
        const int g = e >> 8, x = e & 255;
        const float *v = g < PK ? s_qr + 8 * g : s_sq + 8 * (g - PK);
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) a += ((x >> i) & 1) ? v[i] : -v[i];
        s_tab[e] = a;
    }
    __syncthreads();
    const float *ts = s_tab + PK * 256;
    const float isd = rsqrtf((float)D);
    const float cq = 1.2533141373155003f / (float)p.M;   // sqrt(pi/2) / m
    const int bk = p.bk, np = p.n_planes;
    for (int k = 0; k < SCORE_TPT; ++k) {
        const int64_t t = ((int64_t)blockIdx.x * SCORE_TPT + k) * SCORE_THREADS + threadIdx.x;
        if (t >= p.T) break;
        const uint32_t *w = reinterpret_cast<const uint32_t *>(p.kc + (((int64_t)b * p.Hkv + h) * p.capacity + t) *
                                                                   p.krow);
        uint32_t pl[4][NW];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int wd = 0; wd < NW; ++wd) pl[q][wd] = q < bk ? w[q * NW + wd] : 0u;
        float a = 0.f;
#pragma unroll
        for (int g = 0; g < PK; ++g) {
            uint32_t by[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) by[q] = (pl[q][g / 4] >> (8 * (g % 4))) & 0xFFu;
            const float *tg = s_tab + g * 256;
#pragma unroll
            for (int sp = 0; sp < 8; ++sp) {
                if (sp < np) {
                    const uint32_t set = p.plane_sets[sp];
                    uint32_t x = 0u;
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        if ((set >> q) & 1u) x ^= by[q];
                    a = fmaf(p.alpha[sp], tg[x], a);
                }
            }
        }
        const uint32_t *sg = w + bk * NW;
        float bq = 0.f;
        for (int wd = 0; wd < p.M / 32; ++wd) {
            const uint32_t sw = sg[wd];
#pragma unroll
            for (int r = 0; r < 4; ++r) bq += ts[(4 * wd + r) * 256 + ((sw >> (8 * r)) & 0xFFu)];
        }
        const float2 nrm = tqdev::key_norms(sg + p.M / 32, p.kf16 != 0);
        p.scores[((int64_t)b * p.Hq + j) * p.T + t] = (nrm.x * a * isd + cq * nrm.y * bq) * isd;
    }
}

struct DequantParams {
    const uint8_t *kc;
    const uint8_t *vc;
    float *kh;
    float *vh;
    const uint32_t *signs;
    const __half *S;
    const float *Q;            // Haar rotation, or nullptr
    int64_t capacity, T;
    int H, M, krow, vrow, bk, bv;
    int kf16;                  // key norms as binary16
    float ck[16];
    float cv[32];
};

// Haar rotation: dst = Q^T w.
template <int D>
__device__ __forceinline__ void unrotate_dense_store(const float (&w)[D], const float *Q, float *dst) {
#pragma unroll 1
    for (int j = 0; j < D; ++j) {
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < D; ++i) a = fmaf(__ldg(Q + i * D + j), w[i], a);
        dst[j] = a;
    }
}

template <int D>
__device__ __forceinline__ void unrotate_store(float (&w)[D], const uint32_t *sg, float *dst) {
#pragma unroll
    for (int len = 1; len < D; len <<= 1)
#pragma unroll
        for (int i = 0; i < D; i += 2 * len)
#pragma unroll
            for (int j = i; j < i + len; ++j) {
                const float a = w[j], b = w[j + len];
                w[j] = a + b;
                w[j + len] = a - b;
            }
    const float sc = rsqrtf((float)D);
#pragma unroll
    for (int j = 0; j < D; j += 4) {
        float4 o;
        o.x = ((sg[j / 32] >> (j % 32)) & 1) ? -w[j] * sc : w[j] * sc;
        o.y = ((sg[(j + 1) / 32] >> ((j + 1) % 32)) & 1) ? -w[j + 1] * sc : w[j + 1] * sc;
        o.z = ((sg[(j + 2) / 32] >> ((j + 2) % 32)) & 1) ? -w[j + 2] * sc : w[j + 2] * sc;
        o.w = ((sg[(j + 3) / 32] >> ((j + 3) % 32)) & 1) ? -w[j + 3] * sc : w[j + 3] * sc;
        *reinterpret_cast<float4 *>(dst + j) = o;
    }
}

template <int D>
__global__ void __launch_bounds__(AUX_THREADS) tq_dequant_kernel(const __grid_constant__ DequantParams p) {
    extern __shared__ __align__(16) uint8_t dsm[];
    __half *sS = reinterpret_cast<__half *>(dsm);
    const int h = blockIdx.y, b = blockIdx.z;
    uint32_t sg[D / 32];
#pragma unroll
    for (int i = 0; i < D / 32; ++i) sg[i] = p.signs[(int64_t)h * (D / 32) + i];
    if (p.kh) {
        const __half *src = p.S + (int64_t)h * p.M * D;
        for (int i = threadIdx.x; i < p.M * D / 8; i += blockDim.x)
            reinterpret_cast<uint4 *>(sS)[i] = reinterpret_cast<const uint4 *>(src)[i];
        __syncthreads();
    }
    const int64_t t = (int64_t)blockIdx.x * AUX_THREADS + threadIdx.x;
    if (t >= p.T) return;
    const int64_t rowi = ((int64_t)b * p.H + h) * p.capacity + t;
    const int64_t outi = (((int64_t)b * p.H + h) * p.T + t) * D;
    const float isd = rsqrtf((float)D);
    if (p.vh) {
        const uint32_t *w = reinterpret_cast<const uint32_t *>(p.vc + rowi * p.vrow);
        float x[D];
        const float ns = __uint_as_float(w[p.bv * D / 32]);
#pragma unroll
        for (int j = 0; j < D; ++j) {
            const int bit = p.bv * j;
            uint32_t v = w[bit / 32] >> (bit % 32);
            if ((bit % 32) + p.bv > 32) v |= w[bit / 32 + 1] << (32 - bit % 32);
            x[j] = ns * p.cv[v & ((1u << p.bv) - 1)] * isd;
        }
        if (p.Q) unrotate_dense_store<D>(x, p.Q + (int64_t)h * D * D, p.vh + outi);
        else unrotate_store<D>(x, sg, p.vh + outi);
    }
    if (p.kh) {
        const uint32_t *w = reinterpret_cast<const uint32_t *>(p.kc + rowi * p.krow);
        const uint32_t *sgn = w + p.bk * (D / 32);
        const float2 nrm = tqdev::key_norms(sgn + p.M / 32, p.kf16 != 0);
        const float ns = nrm.x;
        const float cq = 1.2533141373155003f / (float)p.M * nrm.y;
        float x[D];
#pragma unroll
        for (int j = 0; j < D; ++j) {
            int idx = 0;
            for (int q = 0; q < p.bk; ++q) idx |= ((w[q * (D / 32) + j / 32] >> (j % 32)) & 1) << q;
            x[j] = ns * p.ck[idx] * isd;
        }
        for (int i = 0; i < p.M; ++i) {
            const float s = ((sgn[i / 32] >> (i % 32)) & 1) ? cq : -cq;
            const __half2 *srow = reinterpret_cast<const __half2 *>(sS + i * D);
#pragma unroll
            for (int j = 0; j < D / 2; ++j) {
                const float2 f = __half22float2(srow[j]);
                x[2 * j] = fmaf(s, f.x, x[2 * j]);
                x[2 * j + 1] = fmaf(s, f.y, x[2 * j + 1]);
            }
        }
        if (p.Q) unrotate_dense_store<D>(x, p.Q + (int64_t)h * D * D, p.kh + outi);
        else unrotate_store<D>(x, sg, p.kh + outi);
    }
}

// --------------------------------------------------------- decode helpers
template <typename T>
__device__ __forceinline__ float load_as_float(const void *p, int64_t i);
template <>
__device__ __forceinline__ float load_as_float<float>(const void *p, int64_t i) {
    return static_cast<const float *>(p)[i];
}
template <>
__device__ __forceinline__ float load_as_float<__half>(const void *p, int64_t i) {
    return __half2float(static_cast<const __half *>(p)[i]);
}
template <>
__device__ __forceinline__ float load_as_float<__nv_bfloat16>(const void *p, int64_t i) {
    return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
}

__device__ __forceinline__ float load_dt(const void *p, int64_t i, int dt) {
    if (dt == TQ_F32) return static_cast<const float *>(p)[i];
    if (dt == TQ_F16) return __half2float(static_cast<const __half *>(p)[i]);
    return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
}

// Threads of a query-preparation block: one per coordinate for the append
// step (at least AUX_THREADS).
__host__ __device__ constexpr int qprep_threads(int d) { return d > AUX_THREADS ? d : AUX_THREADS; }

// Sum over the block (NT threads); every thread gets the total.
template <int NT>
__device__ __forceinline__ float block_sum(float v, float *s_red) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = v;
    __syncthreads();
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) t += s_red[w];
    return t;
}

// Append step (bitpolar MultiHeadKvCache::push_token): encode one new key or
// value row of kv head h and store it as row t of the segment.  The same
// method as the bulk encoder (turboquant-plus-rs README, Architecture):
// u = H (D x); n = |x|; cell = #{positive boundaries <= |u| / n}; index
// 2^(B-1) + cell, mirrored for u < 0; n_s = n / |C[idx]/sqrt(d)|; keys add
// the QJL signs of S (u - n_s C[idx]) and gamma = |u - n_s C[idx]| / sqrt(d).
// One block of qprep_threads(D) threads, coordinate j on thread j.
template <int D>
__device__ void append_row(bool key, const void *src, int64_t src_off, int dt, const SegDesc &g, int h, int64_t t,
                           float *s_u, float *s_e, float *s_red, uint8_t *s_idx) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const TqBook &book = *g.book;
    const int B = key ? g.bk : g.bv;
    const int HB = 1 << (B - 1);
    const float *mag = key ? book.kmag : book.vmag;
    const float *pb = key ? book.kpb : book.vpb;
    float u = 0.f;
    if (g.Q) {
        // Haar rotation: u = sqrt(d) Q x
        if (tid < D) s_e[tid] = load_dt(src, src_off + tid, dt);
        __syncthreads();
        if (tid < D) {
            const float *row = g.Q + ((int64_t)h * D + tid) * D;
            float a = 0.f;
            for (int j = 0; j < D; ++j) a = fmaf(__ldg(row + j), s_e[j], a);
            u = a * sqrtf((float)D);
        }
        __syncthreads();
    } else {
        if (tid < D) {
            const float x = load_dt(src, src_off + tid, dt);
            s_u[tid] = ((g.signs[(int64_t)h * (D / 32) + tid / 32] >> (tid % 32)) & 1) ? -x : x;
        }
        __syncthreads();
        for (int len = 1; len < D; len <<= 1) {
            for (int i = tid; i < D / 2; i += blockDim.x) {
                const int j = (i / len) * 2 * len + (i % len);
                const float a = s_u[j], b = s_u[j + len];
                s_u[j] = a + b;
                s_u[j + len] = a - b;
            }
            __syncthreads();
        }
        u = tid < D ? s_u[tid] : 0.f;
    }
    const float n2 = block_sum<qprep_threads(D)>(u * u, s_red);
    const bool nonfinite = !(n2 <= 3.0e38f);
    const bool degenerate = nonfinite || !(n2 >= 1.17549435e-38f);
    if (tid == 0 && nonfinite) atomicAdd(&g.status[0], 1ull);
    const float n = sqrtf(n2 * (1.f / D));
    int cell = 0;
    for (int k = 0; k + 1 < HB; ++k) cell += fabsf(u) >= n * pb[k] ? 1 : 0;
    const float cm = mag[cell];
    const float c2 = block_sum<qprep_threads(D)>(tid < D ? cm * cm : 0.f, s_red);
    const float ns = degenerate ? 0.f : n * sqrtf((float)D / c2);
    const uint32_t idx = degenerate ? (uint32_t)HB : u < 0.f ? (uint32_t)(HB - 1 - cell) : (uint32_t)(HB + cell);
    const int64_t rowb = key ? g.krow : g.vrow;
    uint32_t *row = reinterpret_cast<uint32_t *>(const_cast<uint8_t *>(key ? g.kc : g.vc) +
                                                 ((int64_t)h * g.capacity + t) * rowb);
    if (key) {
        const float e = tid < D && !degenerate ? u - ns * (u < 0.f ? -cm : cm) : 0.f;
        if (tid < D) s_e[tid] = e;
        const float e2 = block_sum<qprep_threads(D)>(e * e, s_red);   // its barriers publish s_e
        const float gv = degenerate ? 0.f : sqrtf(e2 * (1.f / D));
        // binary16 norms: a row whose norms overflow is the zero row, counted
        // with the non-finite rows (ns and e2 are block-wide, so is this)
        bool zero_row = degenerate;
        uint32_t nw = 0u;
        if (g.kf16 && !tqdev::pack_norms_f16(ns, gv, nw)) {
            zero_row = true;
            nw = 0u;
            if (tid == 0) atomicAdd(&g.status[0], 1ull);
        }
        const uint32_t kidx = zero_row ? (uint32_t)HB : idx;
        // index bit planes: warp w holds coordinates [32w, 32w + 32)
#pragma unroll 1
        for (int q = 0; q < B; ++q) {
            const uint32_t w = __ballot_sync(0xffffffffu, (kidx >> q) & 1u);
            if (lane == 0 && tid < D) row[q * (D / 32) + warp] = w;
        }
        // QJL signs: projection i on thread i (and i + blockDim.x, ...)
        const int sw0 = B * (D / 32);
#pragma unroll 1
        for (int i0 = 0; i0 < g.m; i0 += blockDim.x) {
            const int i = i0 + tid;
            float p = 0.f;
            if (i < g.m) {
                const uint4 *Srow = reinterpret_cast<const uint4 *>(g.S + ((int64_t)h * g.m + i) * D);
#pragma unroll 4
                for (int c = 0; c < D / 8; ++c) {
                    const uint4 w = Srow[c];
                    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int e2i = 0; e2i < 4; ++e2i) {
                        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&ww[e2i]));
                        p = fmaf(f.x, s_e[8 * c + 2 * e2i], p);
                        p = fmaf(f.y, s_e[8 * c + 2 * e2i + 1], p);
                    }
                }
            }
            const uint32_t w = __ballot_sync(0xffffffffu, p >= 0.f);
            if (lane == 0 && i0 + 32 * warp < g.m) row[sw0 + (i0 + 32 * warp) / 32] = zero_row ? ~0u : w;
        }
        if (tid == 0) {
            const int tail = sw0 + g.m / 32;
            if (g.kf16) {
                row[tail] = nw;
            } else {
                row[tail] = __float_as_uint(ns);
                row[tail + 1] = __float_as_uint(gv);
            }
        }
    } else {
        if (tid < D) s_idx[tid] = (uint8_t)idx;
        __syncthreads();
        // B-bit fields, coordinate j at bit B j of the little-endian stream
        for (int w = tid; w < B * D / 32; w += blockDim.x) {
            uint32_t word = 0u;
            for (int b = 0; b < 32; ++b) {
                const int bit = 32 * w + b;
                word |= (uint32_t)((s_idx[bit / B] >> (bit % B)) & 1) << b;
            }
            row[w] = word;
        }
        if (tid == 0) row[B * D / 32] = __float_as_uint(ns);
    }
    __syncthreads();
}

// Query heads per pass of a query-preparation block.
constexpr int QP_GROUP = 4;

// Blocks [0, query blocks): one per (segment, seq_local, kv head), the
// prepared queries [q_rot | S q_rot] of the G query heads of the group, in
// passes of up to QP_GROUP heads.  Thread i's row of S (projection i) is
// requested before the first rotation and serves every head of the group.
// Blocks after those: one per (appending segment, kv head), the append
// step's new key and value rows.
template <int D, typename Tq>
__global__ void __launch_bounds__(qprep_threads(D)) tq_qprep_kernel(const __grid_constant__ DecodePlan P, const void *q) {
    tqdev::grid_dep_trigger();   // the decode CTAs may start their set-up now
    __shared__ __align__(16) float s_in[QP_GROUP][D];   // raw queries (Haar), append scratch
    __shared__ __align__(16) float s_qr[QP_GROUP][D];
    __shared__ float s_red[qprep_threads(D) / 32];
    __shared__ uint8_t s_idx[D];
    int s = 0;
    int64_t blk = blockIdx.x;
    for (; s < P.n_segs; ++s) {
        const int64_t n = (int64_t)P.seg[s].n_seqs * P.Hkv;
        if (blk < n) break;
        blk -= n;
    }
    if (s == P.n_segs) {
        // append block: blk counts (appending segment, kv head) pairs
        for (s = 0; s < P.n_segs; ++s) {
            if (!P.seg[s].append) continue;
            if (blk < P.Hkv) break;
            blk -= P.Hkv;
        }
        if (s == P.n_segs) return;
        const SegDesc &g = P.seg[s];
        const int h = (int)blk;
        const int64_t src = ((int64_t)g.first_seq * P.Hkv + h) * D;
        append_row<D>(true, P.k_new, src, P.kv_dtype, g, h, g.T - 1, s_in[0], s_qr[0], s_red, s_idx);
        append_row<D>(false, P.v_new, src, P.kv_dtype, g, h, g.T - 1, s_in[0], s_qr[0], s_red, s_idx);
        return;
    }
    const SegDesc &g = P.seg[s];
    const int seq_local = (int)(blk / P.Hkv), h = (int)(blk % P.Hkv);
    const int seq = g.first_seq + seq_local;
    const int M = g.m, G = P.G;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const __half *Sh = g.S + (int64_t)h * M * D;
    const float *Qh = g.Q ? g.Q + (int64_t)h * D * D : nullptr;
    // this thread's row of S, kept for every pass (head_dim <= 128)
    constexpr bool KEEP = D <= 128;
    uint4 wkeep[KEEP ? D / 8 : 1];
    if (KEEP && tid < M) {
        const uint4 *row = reinterpret_cast<const uint4 *>(Sh + (int64_t)tid * D);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) wkeep[c] = __ldg(row + c);
    }
    for (int g0 = 0; g0 < G; g0 += QP_GROUP) {
        const int ng = min(QP_GROUP, G - g0);
        const int64_t qrow0 = (int64_t)seq * P.Hq + h * G + g0;   // first query row of the pass
        if (Qh) {
            // Haar rotation: q_rot = Q q, one output coordinate per thread
            for (int e = tid; e < ng * D; e += blockDim.x) s_in[e / D][e % D] = load_as_float<Tq>(q, qrow0 * D + e);
            __syncthreads();
            for (int i = tid; i < D; i += blockDim.x) {
                const float4 *row = reinterpret_cast<const float4 *>(Qh + (int64_t)i * D);
                float a0[QP_GROUP], a1[QP_GROUP];
#pragma unroll
                for (int k = 0; k < QP_GROUP; ++k) a0[k] = a1[k] = 0.f;
#pragma unroll 4
                for (int c = 0; c < D / 4; ++c) {
                    const float4 w = __ldg(row + c);
#pragma unroll
                    for (int k = 0; k < QP_GROUP; ++k) {
                        if (k < ng) {
                            a0[k] = fmaf(w.x, s_in[k][4 * c], a0[k]);
                            a1[k] = fmaf(w.y, s_in[k][4 * c + 1], a1[k]);
                            a0[k] = fmaf(w.z, s_in[k][4 * c + 2], a0[k]);
                            a1[k] = fmaf(w.w, s_in[k][4 * c + 3], a1[k]);
                        }
                    }
                }
#pragma unroll
                for (int k = 0; k < QP_GROUP; ++k)
                    if (k < ng) s_qr[k][i] = a0[k] + a1[k];
            }
        } else if (warp < ng) {
            // Walsh-Hadamard: warp k rotates head g0 + k (lane l holds
            // coordinates l + 32 i: the stages of stride >= 32 in registers,
            // the others across lanes by shuffles)
            constexpr int V = D / 32;
            const uint32_t *sg = g.signs + (int64_t)h * (D / 32);
            float x[V];
#pragma unroll
            for (int k = 0; k < V; ++k) {
                const int j = lane + 32 * k;
                const float v = load_as_float<Tq>(q, (qrow0 + warp) * D + j);
                x[k] = ((sg[j / 32] >> (j % 32)) & 1) ? -v : v;
            }
#pragma unroll
            for (int len = 1; len < V; len <<= 1)
#pragma unroll
                for (int k = 0; k < V; k += 2 * len)
#pragma unroll
                    for (int kk = k; kk < k + len; ++kk) {
                        const float a = x[kk], b = x[kk + len];
                        x[kk] = a + b;
                        x[kk + len] = a - b;
                    }
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const bool upper = (lane & o) != 0;
#pragma unroll
                for (int k = 0; k < V; ++k) {
                    const float y = __shfl_xor_sync(0xffffffffu, x[k], o);
                    x[k] = upper ? y - x[k] : x[k] + y;
                }
            }
            const float sc = rsqrtf((float)D);
#pragma unroll
            for (int k = 0; k < V; ++k) s_qr[warp][lane + 32 * k] = x[k] * sc;
        }
        __syncthreads();
        float *dst0 = P.qprep + g.qprep_base + ((int64_t)seq_local * P.Hq + h * G + g0) * (D + M);
        // S q_rot: projection i of every head of the pass from one row of S
        for (int i = tid; i < M; i += blockDim.x) {
            uint4 w[D / 8];
            if (KEEP && i == tid) {
#pragma unroll
                for (int c = 0; c < D / 8; ++c) w[c] = wkeep[KEEP ? c : 0];
            } else {
                const uint4 *row = reinterpret_cast<const uint4 *>(Sh + (int64_t)i * D);
#pragma unroll
                for (int c = 0; c < D / 8; ++c) w[c] = __ldg(row + c);
            }
            float acc0[QP_GROUP], acc1[QP_GROUP];
#pragma unroll
            for (int k = 0; k < QP_GROUP; ++k) acc0[k] = acc1[k] = 0.f;
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
                const float2 f0 = __half22float2(*reinterpret_cast<const __half2 *>(&w[c].x));
                const float2 f1 = __half22float2(*reinterpret_cast<const __half2 *>(&w[c].y));
                const float2 f2 = __half22float2(*reinterpret_cast<const __half2 *>(&w[c].z));
                const float2 f3 = __half22float2(*reinterpret_cast<const __half2 *>(&w[c].w));
#pragma unroll
                for (int k = 0; k < QP_GROUP; ++k) {
                    if (k < ng) {
                        const float4 qa = reinterpret_cast<const float4 *>(s_qr[k])[2 * c];
                        const float4 qb = reinterpret_cast<const float4 *>(s_qr[k])[2 * c + 1];
                        acc0[k] = fmaf(f0.x, qa.x, acc0[k]);
                        acc1[k] = fmaf(f0.y, qa.y, acc1[k]);
                        acc0[k] = fmaf(f1.x, qa.z, acc0[k]);
                        acc1[k] = fmaf(f1.y, qa.w, acc1[k]);
                        acc0[k] = fmaf(f2.x, qb.x, acc0[k]);
                        acc1[k] = fmaf(f2.y, qb.y, acc1[k]);
                        acc0[k] = fmaf(f3.x, qb.z, acc0[k]);
                        acc1[k] = fmaf(f3.y, qb.w, acc1[k]);
                    }
                }
            }
#pragma unroll
            for (int k = 0; k < QP_GROUP; ++k)
                if (k < ng) dst0[(int64_t)k * (D + M) + D + i] = acc0[k] + acc1[k];
        }
        for (int e = tid; e < ng * D; e += blockDim.x) dst0[(int64_t)(e / D) * (D + M) + e % D] = s_qr[e / D][e % D];
        __syncthreads();
    }
}

template <typename To>
__device__ __forceinline__ void store_out(void *p, int64_t i, float v);
template <>
__device__ __forceinline__ void store_out<float>(void *p, int64_t i, float v) {
    static_cast<float *>(p)[i] = v;
}
template <>
__device__ __forceinline__ void store_out<__half>(void *p, int64_t i, float v) {
    static_cast<__half *>(p)[i] = __float2half_rn(v);
}
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(void *p, int64_t i, float v) {
    static_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(v);
}

// One block of d threads per (sequence, head).
template <int D, typename To>
__global__ void __launch_bounds__(D) tq_combine_kernel(const __grid_constant__ DecodePlan P, void *out) {
    tqdev::grid_dep_wait();   // the partials of the decode launches
    const int b = blockIdx.x / P.Hq, j = blockIdx.x % P.Hq;
    const int PF = tq_part_floats(D);
    // one pass with an online rescale; the (m, l, o_j) of CB splits are
    // loaded before any is used, so their latencies overlap
    constexpr int CB = 8;
    float mx = -INFINITY, l = 0.f, o = 0.f;
    for (int s = 0; s < P.n_segs; ++s) {
        const SegDesc &g = P.seg[s];
        if (b < g.first_seq || b >= g.first_seq + g.n_seqs || g.T == 0) continue;
        const float *base = P.part + (g.part_base + (int64_t)(b - g.first_seq) * P.Hq + j) * PF;
        const int64_t stride = (int64_t)g.n_seqs * P.Hq * PF;   // between splits
        for (int sp0 = 0; sp0 < g.n_splits; sp0 += CB) {
            float pm[CB], pl[CB], po[CB];
#pragma unroll
            for (int k = 0; k < CB; ++k) {
                const bool in = sp0 + k < g.n_splits;
                const float *pp = base + (int64_t)(sp0 + k) * stride;
                pm[k] = in ? pp[0] : -INFINITY;
                pl[k] = in ? pp[1] : 0.f;
                po[k] = in ? pp[4 + threadIdx.x] : 0.f;
            }
#pragma unroll
            for (int k = 0; k < CB; ++k) {
                if (pm[k] == -INFINITY) continue;
                if (pm[k] > mx) {
                    const float sc = __expf(mx - pm[k]);   // 0 while mx is -inf
                    l *= sc;
                    o *= sc;
                    mx = pm[k];
                }
                const float w = __expf(pm[k] - mx);
                l = fmaf(w, pl[k], l);
                o = fmaf(w, po[k], o);
            }
        }
    }
    store_out<To>(out, ((int64_t)b * P.Hq + j) * D + threadIdx.x, l > 0.f ? o / l : 0.f);
}

}  // namespace

// ------------------------------------------------------------------ launches
tq_status tq_launch_scores(tq_ctx *ctx, const tq_codes *codes, const float *q, int Hq, int64_t T, float *scores,
                           cudaStream_t stream) {
    ScoresParams p{};
    p.kc = static_cast<const uint8_t *>(codes->k);
    p.q = q;
    p.scores = scores;
    p.signs = ctx->d_signs;
    p.S = ctx->d_S;
    p.Q = ctx->rotation == TQ_ROT_HAAR ? ctx->d_Q32 : nullptr;
    p.capacity = codes->capacity;
    p.T = T;
    p.Hq = Hq;
    p.Hkv = codes->n_kv_heads;
    p.M = ctx->m;
    p.krow = (int)tq_row_bytes(ctx, TQ_KEYS);
    p.bk = ctx->BK;
    p.kf16 = ctx->norm_f16;
    tq_sigma_planes(ctx, &p.n_planes, p.plane_sets, p.alpha);
    const int64_t per_block = (int64_t)SCORE_THREADS * SCORE_TPT;
    dim3 grid((unsigned)((T + per_block - 1) / per_block), (unsigned)Hq, (unsigned)codes->batch);
    const size_t tab = (size_t)(ctx->d / 8 + ctx->m / 8) * 256 * sizeof(float);
    auto kern = ctx->d == 256 ? tq_scores_kernel<256> : ctx->d == 128 ? tq_scores_kernel<128> : tq_scores_kernel<64>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tab);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return tq_check_cuda(e);
    }
    kern<<<grid, SCORE_THREADS, tab, stream>>>(p);
    return tq_check_cuda(cudaGetLastError());
}

tq_status tq_launch_dequant(tq_ctx *ctx, const tq_codes *codes, int64_t T, float *k_hat, float *v_hat,
                            cudaStream_t stream) {
    DequantParams p{};
    p.kc = static_cast<const uint8_t *>(codes->k);
    p.vc = static_cast<const uint8_t *>(codes->v);
    p.kh = k_hat;
    p.vh = v_hat;
    p.signs = ctx->d_signs;
    p.S = ctx->d_S;
    p.Q = ctx->rotation == TQ_ROT_HAAR ? ctx->d_Q32 : nullptr;
    p.capacity = codes->capacity;
    p.T = T;
    p.H = codes->n_kv_heads;
    p.M = ctx->m;
    p.krow = (int)tq_row_bytes(ctx, TQ_KEYS);
    p.vrow = (int)tq_row_bytes(ctx, TQ_VALUES);
    p.bk = ctx->BK;
    p.bv = ctx->BV;
    p.kf16 = ctx->norm_f16;
    for (int i = 0; i < ctx->LK; ++i) p.ck[i] = ctx->ck[i];
    for (int i = 0; i < ctx->LV; ++i) p.cv[i] = ctx->cv[i];
    dim3 grid((unsigned)((T + AUX_THREADS - 1) / AUX_THREADS), (unsigned)codes->n_kv_heads, (unsigned)codes->batch);
    const size_t smem = k_hat ? (size_t)ctx->m * ctx->d * 2 : 0;
    cudaError_t e;
    if (ctx->d == 256) {
        e = cudaFuncSetAttribute(tq_dequant_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess) tq_dequant_kernel<256><<<grid, AUX_THREADS, smem, stream>>>(p);
    } else if (ctx->d == 128) {
        e = cudaFuncSetAttribute(tq_dequant_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess) tq_dequant_kernel<128><<<grid, AUX_THREADS, smem, stream>>>(p);
    } else {
        e = cudaFuncSetAttribute(tq_dequant_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess) tq_dequant_kernel<64><<<grid, AUX_THREADS, smem, stream>>>(p);
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        return tq_check_cuda(e);
    }
    return tq_check_cuda(cudaGetLastError());
}

cudaError_t tq_launch_qprep(const DecodePlan &P, const void *q, tq_dtype dt, cudaStream_t stream) {
    int64_t blocks = P.n_append_blocks;
    for (int s = 0; s < P.n_segs; ++s) blocks += (int64_t)P.seg[s].n_seqs * P.Hkv;
    if (blocks == 0) return cudaSuccess;
#define TQ_QPREP(DD, TT) tq_qprep_kernel<DD, TT><<<(unsigned)blocks, qprep_threads(DD), 0, stream>>>(P, q)
    if (P.d == 256) {
        if (dt == TQ_F32) TQ_QPREP(256, float);
        else if (dt == TQ_F16) TQ_QPREP(256, __half);
        else TQ_QPREP(256, __nv_bfloat16);
    } else if (P.d == 128) {
        if (dt == TQ_F32) TQ_QPREP(128, float);
        else if (dt == TQ_F16) TQ_QPREP(128, __half);
        else TQ_QPREP(128, __nv_bfloat16);
    } else {
        if (dt == TQ_F32) TQ_QPREP(64, float);
        else if (dt == TQ_F16) TQ_QPREP(64, __half);
        else TQ_QPREP(64, __nv_bfloat16);
    }
#undef TQ_QPREP
    return cudaGetLastError();
}

cudaError_t tq_launch_combine(const DecodePlan &P, void *out, tq_dtype dt, cudaStream_t stream) {
    const unsigned blocks = (unsigned)(P.batch * P.Hq);
#define TQ_COMB(DD, TT) \
    return tq_launch_dependent(tq_combine_kernel<DD, TT>, dim3((unsigned)blocks), dim3(DD), 0, stream, P, out)
    if (P.d == 256) {
        if (dt == TQ_F32) TQ_COMB(256, float);
        else if (dt == TQ_F16) TQ_COMB(256, __half);
        else TQ_COMB(256, __nv_bfloat16);
    } else if (P.d == 128) {
        if (dt == TQ_F32) TQ_COMB(128, float);
        else if (dt == TQ_F16) TQ_COMB(128, __half);
        else TQ_COMB(128, __nv_bfloat16);
    } else {
        if (dt == TQ_F32) TQ_COMB(64, float);
        else if (dt == TQ_F16) TQ_COMB(64, __half);
        else TQ_COMB(64, __nv_bfloat16);
    }
#undef TQ_COMB
    return cudaGetLastError();
}
