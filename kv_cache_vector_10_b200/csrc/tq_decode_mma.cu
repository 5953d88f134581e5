// tq_decode_mma.cu -- decode attention on the tensor cores, for segments
// whose staged code tiles serve many queries (a prefix shared by many
// sequences, wide query-head groups).
//
// The estimate is the one the lookup-table decode computes (turboquant-plus-rs
// README, Architecture: PolarQuant indices plus the QJL sign correction), with
// the queries of a kv head as the 128 rows of every MMA:
//
//   S_mse[q, t] = sum_j q_rot[q, j] C[idx_tj]              K = d
//   S_qjl[q, t] = sum_i (S q_rot)[q, i] (2 b_ti - 1)        K = m
//   score       = n_t / d * S_mse + gamma_t sqrt(pi/2) / (m sqrt d) * S_qjl
//   O[q, j]    += sum_t P[q, t] Cv[vidx_tj]                  K = tokens
//   P           = exp(score - m_run) * |v_t|_s
//
// One CTA per (segment, kv head, token split, block of 128 queries), three
// roles:
//   * warps 0-7, two threads per query (= TMEM lane), each taking 32 tokens
//     of a tile: stage the queries (coalesced, through shared memory) and
//     write the query operands (q_rot and S q_rot as bfloat16 hi + lo) into
//     TMEM, then per 64-token tile read the scores, keep the online softmax,
//     write P (bfloat16 hi + lo) into shared memory; at the end rotate the
//     output back (Walsh-Hadamard, TMEM as scratch) and write it through
//     shared memory, coalesced;
//   * warps 8-14: expand each staged tile into MMA operands: the key
//     centroids C[idx] as bfloat16 hi + lo and the QJL signs as exact +-1
//     (K-major, one 128-byte swizzled row per token), the value centroids as
//     bfloat16 hi + lo (token rows of the MN-major B operand), and the
//     per-token norms;
//   * warp 15: bulk copies of the packed key and value rows (two stages)
//     and the MMAs, issued by one thread: 3 passes for the centroid products
//     (hi*hi, hi*lo, lo*hi), 2 for the signs, 3 for the value sum.
// The running maximum is raised only when a tile's maximum exceeds it by
// more than kRescale (then the thread rescales its TMEM output row); both the
// output and the sum of weights use the same maximum, so the result is the
// same softmax.
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>

#include "tq_decode.cuh"

namespace {

constexpr int MMA_NT = 64;          // tokens per tile
constexpr int MMA_Q = 128;          // queries per CTA (MMA rows)
constexpr int SM_WARPS = 8;         // softmax warps: two per TMEM lane quadrant
constexpr int EX_WARPS = 7;         // operand expansion warps (16 warps in all: 128 registers each)
constexpr int MMA_THREADS = 32 * (SM_WARPS + EX_WARPS + 1);   // + the producer warp
constexpr float kRescale = 8.f;

template <int D, int MP>
struct MmaLayout {
    static constexpr int KX = MMA_NT * 128;              // one 64-wide K block of a [64 x 64] bf16 operand
    static constexpr int C_BYTES = (D / 64) * KX;        // a centroid expansion (hi or lo)
    static constexpr int S_BYTES = (MP / 64) * KX;       // the sign expansion
    static constexpr int KEXP = 2 * C_BYTES + S_BYTES;   // one key buffer: C hi, C lo, signs
    static constexpr int VEXP = 2 * C_BYTES;             // one value buffer: hi, lo
    static constexpr int PB = MMA_Q * 128;               // P hi (or lo): 128 rows x 64 tokens
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + 2 * KEXP;
    static constexpr int OFF_P = OFF_V + 2 * VEXP;
    static constexpr int OFF_SC = OFF_P + 2 * PB;        // per-token scalars [2][3][64] floats
    static constexpr int OFF_X = OFF_SC + 2 * 3 * MMA_NT * 4;   // softmax exchange: maxima, sums, (m, l)
    static constexpr int OFF_TAB = OFF_X + 4096;
    // TMEM columns
    static constexpr int COL_QHI = 0, COL_QLO = D / 2, COL_SHI = D, COL_SLO = D + MP / 2;
    static constexpr int COL_MSE = D + MP, COL_QJL = COL_MSE + MMA_NT, COL_O = COL_QJL + MMA_NT;
    static constexpr int COLS = COL_O + D;
    static_assert(COLS <= 512, "TMEM columns");
};

// D[tmem] (+)= A[tmem] * B[smem desc]^T, kind::f16, one CTA.
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Descriptor of an MN-major operand in 128-byte swizzled atoms: rows of 64
// consecutive MN elements, one row per K index, 8-row groups `sbo` bytes
// apart, 64-element MN blocks `lbo` bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128_mn(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t desc = 0;
    desc |= (uint64_t)((saddr >> 4) & 0x3FFF);
    desc |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    desc |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    desc |= (uint64_t)1 << 46;
    desc |= (uint64_t)2 << 61;
    return desc;
}

// bfloat16 hi + lo of a pair: hi = round(x), lo = round(x - hi); low half = first.
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t &hi, uint32_t &lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = *reinterpret_cast<const uint32_t *>(&l);
}

// Byte offset of 16-byte chunk `c` of row `r` in a 128-byte swizzled operand
// whose rows are grouped by 64 columns into blocks `block` bytes apart.
__device__ __forceinline__ uint32_t sw128_off(int r, int c, int block) {
    return (uint32_t)((c >> 3) * block + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Sylvester Walsh-Hadamard butterflies over 32 values.
__device__ __forceinline__ void wht32(float (&x)[32]) {
#pragma unroll
    for (int len = 1; len < 32; len <<= 1) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (i & len) continue;
            const float a = x[i], b = x[i + len];
            x[i] = a + b;
            x[i + len] = a - b;
        }
    }
}

// 16-byte asynchronous copy global -> shared; src_bytes = 0 fills zeros.
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(tqdev::smem_u32(smem)), "l"(gmem),
                 "r"(src_bytes)
                 : "memory");
}

// One output element in the caller's type.
__device__ __forceinline__ void store_out_elem(void *p, int64_t i, float v, int dt) {
    if (dt == TQ_F32) static_cast<float *>(p)[i] = v;
    else if (dt == TQ_F16) static_cast<__half *>(p)[i] = __float2half_rn(v);
    else static_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(v);
}

}  // namespace

namespace {

// Bounded wait by every lane of a warp; true if all of them saw the phase.
__device__ __forceinline__ bool bar_wait_warp(uint64_t *bar, uint32_t phase) {
    const bool ok = tqdev::mbar_wait_bounded(bar, phase);
    return __all_sync(0xffffffffu, ok);
}

struct MmaBars {
    uint64_t codes_full[2], codes_free[2];   // staged packed rows
    uint64_t kexp_full[2], kexp_free[2];     // key operands (C hi, C lo, signs)
    uint64_t vexp_full[2], vexp_free[2];     // value operands
    uint64_t scal_full[2], scal_free[2];     // per-token norms
    uint64_t s_full, s_free;                 // scores in TMEM
    uint64_t p_full, p_free;                 // P in shared memory (p_free: the value MMAs of a tile done)
    uint64_t a_ready, done;                  // query operands in TMEM (staging area free); every MMA complete
    uint64_t pair[4];                        // the two softmax warps of a TMEM lane quadrant
};

// Value pair table: two B_V-bit codes per entry (one code per entry at B_V = 5).
template <int BV>
__host__ __device__ constexpr int vpair_entries_mma() { return BV == 5 ? 32 : 1 << (2 * BV); }

template <int D, int BK, int BV, int MP>
__global__ void __launch_bounds__(MMA_THREADS, 1) tq_decode_mma_kernel(const __grid_constant__ DecodePlan P) {
    using L = MmaLayout<D, MP>;
    constexpr int NT = MMA_NT;
    constexpr int NKP = 1 << (2 * BK);   // key pair table: two coordinates' index bits, plane-interleaved
    constexpr int NVP = vpair_entries_mma<BV>();
    constexpr int EX0 = 32 * SM_WARPS;   // first expansion thread
    constexpr int PWARP = SM_WARPS + EX_WARPS;
    constexpr float LOG2E = 1.4426950408889634f;
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(MP == 64 || MP == 128, "projections");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint2 *kpt = reinterpret_cast<uint2 *>(sm + L::OFF_TAB);
    uint2 *vpt = kpt + NKP;
    float *scal = reinterpret_cast<float *>(sm + L::OFF_SC);   // [buffer][a1, a2, |v|][NT]
    float *xch = reinterpret_cast<float *>(sm + L::OFF_X);     // [parity][half][128] tile maxima
    float *lx = xch + 512;                                      // [half][128] partial sums
    float *mlr = lx + 256;                                      // [128][2] (m, l) per query row
    uint8_t *codes = reinterpret_cast<uint8_t *>(vpt + NVP);
    __shared__ MmaBars bars;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;

    // An append step's new rows are written by the query-preparation kernel.
    if (P.n_append_blocks) tqdev::grid_dep_wait();
    tqdev::grid_dep_trigger();
    int s = 0;
    const int64_t item = blockIdx.x;
    for (; s < P.n_segs; ++s) {
        const SegDesc &g0 = P.seg[s];
        const int64_t n = (int64_t)P.Hkv * g0.n_splits * g0.n_qchunks;
        if (g0.bk == BK && item >= g0.item_base && item < g0.item_base + n) break;
    }
    if (s >= P.n_segs) return;
    const SegDesc &g = P.seg[s];
    const int64_t local = item - g.item_base;
    const int qchunk = (int)(local % g.n_qchunks);
    const int split = (int)((local / g.n_qchunks) % g.n_splits);
    const int h = (int)(local / ((int64_t)g.n_qchunks * g.n_splits));
    const int krow = g.krow, vrow = g.vrow;
    const int64_t t_begin = (int64_t)split * g.split_len;
    const int64_t t_end = std::min<int64_t>(g.T, t_begin + g.split_len);
    const int nt = t_end > t_begin ? (int)((t_end - t_begin + NT - 1) / NT) : 0;
    const int nq = g.n_seqs * P.G;
    const int stage_bytes = NT * (krow + vrow);
    const uint8_t *kbase = g.kc + (int64_t)h * g.capacity * krow;
    const uint8_t *vbase = g.vc + (int64_t)h * g.capacity * vrow;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            tqdev::mbar_init(&bars.codes_full[i], 1);
            tqdev::mbar_init(&bars.codes_free[i], EX_WARPS);
            tqdev::mbar_init(&bars.kexp_full[i], EX_WARPS);
            tqdev::mbar_init(&bars.kexp_free[i], 1);
            tqdev::mbar_init(&bars.vexp_full[i], EX_WARPS);
            tqdev::mbar_init(&bars.vexp_free[i], 1);
            tqdev::mbar_init(&bars.scal_full[i], EX_WARPS);
            tqdev::mbar_init(&bars.scal_free[i], SM_WARPS);
        }
        tqdev::mbar_init(&bars.s_full, 1);
        tqdev::mbar_init(&bars.s_free, SM_WARPS);
        tqdev::mbar_init(&bars.p_full, SM_WARPS);
        tqdev::mbar_init(&bars.p_free, 1);
        tqdev::mbar_init(&bars.a_ready, SM_WARPS);
        tqdev::mbar_init(&bars.done, 1);
        for (int i = 0; i < 4; ++i) tqdev::mbar_init(&bars.pair[i], 2);
        s_abort = tqdev::status_aborted(g.status) ? 1 : 0;
        tqdev::fence_barrier_init();
    }
    if (tid >= EX0 && tid < EX0 + 32 * EX_WARPS) {
        // pair tables: bfloat16 hi + lo of two centroids per entry
        for (int i = tid - EX0; i < NKP; i += 32 * EX_WARPS) {
            int i0 = 0, i1 = 0;
#pragma unroll
            for (int p = 0; p < BK; ++p) {
                i0 |= ((i >> (2 * p)) & 1) << p;
                i1 |= ((i >> (2 * p + 1)) & 1) << p;
            }
            uint32_t hi, lo;
            split_bf16x2(g.ktab[i0], g.ktab[i1], hi, lo);
            kpt[i] = make_uint2(hi, lo);
        }
        for (int i = tid - EX0; i < NVP; i += 32 * EX_WARPS) {
            uint32_t hi, lo;
            if (BV == 5) split_bf16x2(g.vtab[i], 0.f, hi, lo);    // one code: hi, lo in the low halves
            else split_bf16x2(g.vtab[i & ((1 << BV) - 1)], g.vtab[i >> BV], hi, lo);
            vpt[i] = make_uint2(hi, lo);
        }
    }
    if (warp == 0) tqdev::tmem_alloc(&s_tmem, 512);
    tqdev::tc_fence_before();
    __syncthreads();
    tqdev::tc_fence_after();
    const uint32_t tmem = s_tmem;
    const bool run = !s_abort && nt > 0;
    bool failed = false;

    if (warp == PWARP) {
        // ------------------------------------------------------------ producer
        // One thread, in a fixed order: the scores of tile i + 1 (as soon as
        // the softmax has read tile i's), then the value sum of tile i.
        if (lane == 0 && run) {
            auto issue_codes = [&](int i) {
                const int st = i & 1;
                const int64_t tb = t_begin + (int64_t)i * NT;
                // the capacity and every tile start are multiples of 16 rows,
                // so the sizes are multiples of 16 bytes
                const int64_t ntok = std::min<int64_t>(NT, g.capacity - tb);
                uint8_t *dk = codes + st * stage_bytes;
                tqdev::mbar_expect_tx(&bars.codes_full[st], (uint32_t)(ntok * (krow + vrow)));
                tqdev::bulk_load(dk, kbase + tb * krow, (uint32_t)(ntok * krow), &bars.codes_full[st]);
                tqdev::bulk_load(dk + NT * krow, vbase + tb * vrow, (uint32_t)(ntok * vrow), &bars.codes_full[st]);
            };
            const uint32_t idesc_s = tqdev::idesc_bf16_f32(NT);
            const uint32_t idesc_v = tqdev::idesc_bf16_f32(D) | (1u << 16);   // B (values) MN-major
            const uint32_t kb0 = tqdev::smem_u32(sm + L::OFF_K), vb0 = tqdev::smem_u32(sm + L::OFF_V);
            const uint32_t pb = tqdev::smem_u32(sm + L::OFF_P);
            auto issue_scores = [&](int i) {
                tqdev::tc_fence_after();
                const uint32_t kb = kb0 + (uint32_t)((i & 1) * L::KEXP);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = (uint32_t)((ks >> 2) * L::KX + (ks & 3) * 32);
                    const uint64_t bh = tqdev::smem_desc_sw128(kb + off);
                    const uint64_t bl = tqdev::smem_desc_sw128(kb + L::C_BYTES + off);
                    mma_f16_ts(tmem + L::COL_MSE, tmem + L::COL_QHI + 8 * ks, bh, idesc_s, ks != 0);
                    mma_f16_ts(tmem + L::COL_MSE, tmem + L::COL_QHI + 8 * ks, bl, idesc_s, 1u);
                    mma_f16_ts(tmem + L::COL_MSE, tmem + L::COL_QLO + 8 * ks, bh, idesc_s, 1u);
                }
#pragma unroll
                for (int ks = 0; ks < MP / 16; ++ks) {
                    const uint32_t off = (uint32_t)(2 * L::C_BYTES + (ks >> 2) * L::KX + (ks & 3) * 32);
                    const uint64_t bs = tqdev::smem_desc_sw128(kb + off);
                    mma_f16_ts(tmem + L::COL_QJL, tmem + L::COL_SHI + 8 * ks, bs, idesc_s, ks != 0);
                    mma_f16_ts(tmem + L::COL_QJL, tmem + L::COL_SLO + 8 * ks, bs, idesc_s, 1u);
                }
                tqdev::mma_commit(&bars.s_full);
                tqdev::mma_commit(&bars.kexp_free[i & 1]);
            };
            auto issue_values = [&](int i) {
                tqdev::tc_fence_after();
                const uint32_t vb = vb0 + (uint32_t)((i & 1) * L::VEXP);
#pragma unroll
                for (int ks = 0; ks < NT / 16; ++ks) {
                    const uint64_t ah = tqdev::smem_desc_sw128(pb + 32 * ks);
                    const uint64_t al = tqdev::smem_desc_sw128(pb + L::PB + 32 * ks);
                    const uint64_t bh = smem_desc_sw128_mn(vb + 2048 * ks, L::KX, 1024);
                    const uint64_t bl = smem_desc_sw128_mn(vb + L::C_BYTES + 2048 * ks, L::KX, 1024);
                    tqdev::mma_f16_ss(tmem + L::COL_O, ah, bh, idesc_v, (i | ks) != 0);
                    tqdev::mma_f16_ss(tmem + L::COL_O, ah, bl, idesc_v, 1u);
                    tqdev::mma_f16_ss(tmem + L::COL_O, al, bh, idesc_v, 1u);
                }
                tqdev::mma_commit(&bars.p_free);
                tqdev::mma_commit(&bars.vexp_free[i & 1]);
            };
            int nc = 0;
            for (; nc < 2 && nc < nt; ++nc) issue_codes(nc);
            bool ok = tqdev::mbar_wait_bounded(&bars.a_ready, 0u) && tqdev::mbar_wait_bounded(&bars.kexp_full[0], 0u);
            if (ok) issue_scores(0);
            for (int i = 0; ok && i < nt; ++i) {
                if (i + 1 < nt) {
                    ok = tqdev::mbar_wait_bounded(&bars.kexp_full[(i + 1) & 1], (uint32_t)(((i + 1) >> 1) & 1)) &&
                         tqdev::mbar_wait_bounded(&bars.s_free, (uint32_t)(i & 1));
                    if (!ok) break;
                    issue_scores(i + 1);
                }
                // the expansion of tile i is complete: its stage may be refilled
                ok = tqdev::mbar_wait_bounded(&bars.vexp_full[i & 1], (uint32_t)((i >> 1) & 1)) &&
                     tqdev::mbar_wait_bounded(&bars.codes_free[i & 1], (uint32_t)((i >> 1) & 1));
                if (!ok) break;
                if (nc < nt) issue_codes(nc++);
                ok = tqdev::mbar_wait_bounded(&bars.p_full, (uint32_t)(i & 1));
                if (!ok) break;
                issue_values(i);
            }
            failed = !ok;
            // drain: every issued copy lands and every issued MMA completes
            // before the CTA's shared memory and TMEM are released
            for (int i = std::max(0, nc - 2); i < nc; ++i)
                tqdev::mbar_wait_bounded(&bars.codes_full[i & 1], (uint32_t)((i >> 1) & 1));
            tqdev::mma_commit(&bars.done);
            if (!tqdev::mbar_wait_bounded(&bars.done, 0u)) failed = true;
        }
    } else if (warp >= SM_WARPS) {
        // ----------------------------------------------------------- expansion
        constexpr int NE = 32 * EX_WARPS;
        const int e = tid - EX0;
        // scores arrive in log2 units: a1 = n_s / d, a2 = gamma sqrt(pi/2) / (m sqrt d), times log2(e)
        const float cqs = 1.2533141373155003f / (float)MP * rsqrtf((float)D) * LOG2E;
        // the query staging area (the operand buffers) is free once the queries are in TMEM
        if (run && !bar_wait_warp(&bars.a_ready, 0u)) failed = true;
        for (int i = 0; run && !failed && i < nt; ++i) {
            const int b = i & 1;
            const uint32_t use = (uint32_t)(i >> 1);
            if (!bar_wait_warp(&bars.codes_full[b], use & 1)) {
                failed = true;
                break;
            }
            const uint8_t *ck = codes + b * stage_bytes;   // key rows of the tile
            const uint8_t *cv = ck + NT * krow;            // value rows
            uint8_t *kx = sm + L::OFF_K + b * L::KEXP;
            uint8_t *vx = sm + L::OFF_V + b * L::VEXP;
            float *sc = scal + b * 3 * NT;
            const int64_t t0 = t_begin + (int64_t)i * NT;
            if (i >= 2 && !bar_wait_warp(&bars.kexp_free[b], (use - 1) & 1)) {
                failed = true;
                break;
            }
            // key centroids: token t, 32 coordinates (one word of each index plane)
#pragma unroll 1
            for (int j = e; j < NT * (D / 32); j += NE) {
                const int t = j % NT, w = j / NT;
                const uint8_t *kr = ck + t * krow;
                uint32_t pl[BK];
#pragma unroll
                for (int p = 0; p < BK; ++p) pl[p] = *reinterpret_cast<const uint32_t *>(kr + p * (D / 8) + 4 * w);
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    uint32_t x = 0u;
#pragma unroll
                    for (int p = 0; p < BK; ++p) x |= ((pl[p] >> (2 * k)) & 3u) << (2 * p);
                    const uint2 v = kpt[x];
                    hi[k] = v.x;
                    lo[k] = v.y;
                }
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const uint32_t off = sw128_off(t, 4 * w + c4, L::KX);
                    *reinterpret_cast<uint4 *>(kx + off) = make_uint4(hi[4 * c4], hi[4 * c4 + 1], hi[4 * c4 + 2], hi[4 * c4 + 3]);
                    *reinterpret_cast<uint4 *>(kx + L::C_BYTES + off) =
                        make_uint4(lo[4 * c4], lo[4 * c4 + 1], lo[4 * c4 + 2], lo[4 * c4 + 3]);
                }
            }
            // QJL signs: bit 1 -> +1 (0x3F80), bit 0 -> -1 (0xBF80)
#pragma unroll 1
            for (int j = e; j < NT * (MP / 32); j += NE) {
                const int t = j % NT, w = j / NT;
                const uint32_t sg = *reinterpret_cast<const uint32_t *>(ck + t * krow + BK * (D / 8) + 4 * w);
                uint32_t v[16];
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    v[k] = 0xBF80BF80u ^ (((sg >> (2 * k)) & 1u) << 15) ^ (((sg >> (2 * k + 1)) & 1u) << 31);
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4)
                    *reinterpret_cast<uint4 *>(kx + 2 * L::C_BYTES + sw128_off(t, 4 * w + c4, L::KX)) =
                        make_uint4(v[4 * c4], v[4 * c4 + 1], v[4 * c4 + 2], v[4 * c4 + 3]);
            }
            tqdev::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) tqdev::mbar_arrive(&bars.kexp_full[b]);
            // per-token scalars (tokens past the split's end weigh nothing)
            if (i >= 2 && !bar_wait_warp(&bars.scal_free[b], (use - 1) & 1)) {
                failed = true;
                break;
            }
            if (e < NT) {
                float a1 = 0.f, a2 = 0.f, vn = 0.f;
                if (t0 + e < t_end) {
                    const float2 nrm =
                        tqdev::key_norms(reinterpret_cast<const uint32_t *>(ck + e * krow + BK * (D / 8) + MP / 8), g.kf16 != 0);
                    a1 = nrm.x * (LOG2E / (float)D);
                    a2 = nrm.y * cqs;
                    vn = *reinterpret_cast<const float *>(cv + e * vrow + BV * D / 8);
                }
                sc[e] = a1;
                sc[NT + e] = a2;
                sc[2 * NT + e] = vn;
            }
            __syncwarp();
            if (lane == 0) tqdev::mbar_arrive(&bars.scal_full[b]);
            // value centroids: token t, 32 coordinates (B_V words of fields)
            if (i >= 2 && !bar_wait_warp(&bars.vexp_free[b], (use - 1) & 1)) {
                failed = true;
                break;
            }
#pragma unroll 1
            for (int j = e; j < NT * (D / 32); j += NE) {
                const int t = j % NT, w = j / NT;
                const uint32_t *vr = reinterpret_cast<const uint32_t *>(cv + t * vrow);
                uint32_t W[BV];
#pragma unroll
                for (int q = 0; q < BV; ++q) W[q] = vr[BV * w + q];
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    constexpr uint32_t MASK = (1u << (2 * BV)) - 1u;
                    const int o = 2 * BV * k, wi = o >> 5, sh = o & 31;
                    uint32_t x;
                    if (sh + 2 * BV <= 32) x = W[wi] >> sh;
                    else x = __funnelshift_r(W[wi], W[wi + 1 < BV ? wi + 1 : wi], sh);
                    x &= MASK;
                    if constexpr (BV == 5) {
                        // one code per entry: hi and lo in the low halves
                        const uint2 v0 = vpt[x & 31u], v1 = vpt[x >> 5];
                        hi[k] = __byte_perm(v0.x, v1.x, 0x5410);
                        lo[k] = __byte_perm(v0.y, v1.y, 0x5410);
                    } else {
                        const uint2 v = vpt[x];
                        hi[k] = v.x;
                        lo[k] = v.y;
                    }
                }
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const uint32_t off = sw128_off(t, 4 * w + c4, L::KX);
                    *reinterpret_cast<uint4 *>(vx + off) = make_uint4(hi[4 * c4], hi[4 * c4 + 1], hi[4 * c4 + 2], hi[4 * c4 + 3]);
                    *reinterpret_cast<uint4 *>(vx + L::C_BYTES + off) =
                        make_uint4(lo[4 * c4], lo[4 * c4 + 1], lo[4 * c4 + 2], lo[4 * c4 + 3]);
                }
            }
            tqdev::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tqdev::mbar_arrive(&bars.vexp_full[b]);
                tqdev::mbar_arrive(&bars.codes_free[b]);
            }
        }
    } else {
        // ------------------------------------------------------------ softmax
        // Two threads per query row (= TMEM lane): `half` 0 takes tokens
        // 0-31 of each tile, half 1 tokens 32-63; both keep the same running
        // maximum (exchanged through shared memory each tile) and their own
        // partial sum of weights.
        const int quad = warp & 3, half = warp >> 2;
        const int r = quad * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);   // this quadrant's lanes
        const int qi = qchunk * MMA_Q + r;
        const bool qvalid = qi < nq;
        const int seq_local = qvalid ? qi / P.G : 0, jh = h * P.G + (qvalid ? qi % P.G : 0);
        uint64_t *pair = &bars.pair[quad];
        uint32_t pair_phase = 0;
        auto pair_sync = [&]() -> bool {   // both warps of the quadrant have arrived
            __syncwarp();
            if (lane == 0) tqdev::mbar_arrive(pair);
            const bool ok = bar_wait_warp(pair, pair_phase);
            pair_phase ^= 1u;
            return ok;
        };
        float m2 = -INFINITY, l_part = 0.f;   // running maximum in log2 units
        if (run) {
            tqdev::grid_dep_wait();   // the prepared queries
            // ---- the CTA's 128 query rows [q_rot | S q_rot] (fp32), staged
            // coalesced in the operand buffers: row rr, 16-byte chunk k at
            // chunk k ^ (rr % 8)
            constexpr int QCH = (D + MP) / 4;
            uint8_t *stg = sm + L::OFF_K;
            const float *qp0 = P.qprep + g.qprep_base;
#pragma unroll 1
            for (int rr = warp; rr < MMA_Q; rr += SM_WARPS) {
                const int q2 = qchunk * MMA_Q + rr;
                const bool ok = q2 < nq;
                const float4 *src = reinterpret_cast<const float4 *>(
                    ok ? qp0 + ((int64_t)(q2 / P.G) * P.Hq + h * P.G + q2 % P.G) * (D + MP) : qp0);
                for (int k = lane; k < QCH; k += 32)
                    cp_async16(stg + rr * QCH * 16 + ((k ^ (rr & 7)) << 4), src + (ok ? k : 0), ok ? 16u : 0u);
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
            asm volatile("cp.async.wait_group 0;" ::: "memory");
            tqdev::named_sync(1, 32 * SM_WARPS);
            // ---- bfloat16 hi + lo into TMEM (column c: elements 2c, 2c + 1):
            // half 0 writes q_rot, half 1 writes S q_rot
            {
                const int n = half == 0 ? D : MP;
                const int k0 = half == 0 ? 0 : D / 4;
                const uint32_t col_hi = half == 0 ? L::COL_QHI : L::COL_SHI;
                const uint32_t col_lo = half == 0 ? L::COL_QLO : L::COL_SLO;
#pragma unroll 1
                for (int cg = 0; cg < n / 64; ++cg) {
                    float hi[32], lo[32];
#pragma unroll
                    for (int c4 = 0; c4 < 16; ++c4) {
                        const int k = k0 + 16 * cg + c4;
                        const float4 x = *reinterpret_cast<const float4 *>(stg + r * QCH * 16 + ((k ^ (r & 7)) << 4));
                        uint32_t h0, l0, h1, l1;
                        split_bf16x2(x.x, x.y, h0, l0);
                        split_bf16x2(x.z, x.w, h1, l1);
                        hi[2 * c4] = __uint_as_float(h0);
                        hi[2 * c4 + 1] = __uint_as_float(h1);
                        lo[2 * c4] = __uint_as_float(l0);
                        lo[2 * c4 + 1] = __uint_as_float(l1);
                    }
                    tqdev::tmem_st_32x32b_x32(tl + col_hi + 32 * cg, hi);
                    tqdev::tmem_st_32x32b_x32(tl + col_lo + 32 * cg, lo);
                }
            }
            tqdev::tmem_wait_st();
            tqdev::tc_fence_before();
            __syncwarp();
            if (lane == 0) tqdev::mbar_arrive(&bars.a_ready);

            uint8_t *prow = sm + L::OFF_P;
            const int tb0 = 32 * half;   // this thread's first token of a tile
            for (int i = 0; i < nt; ++i) {
                const int b = i & 1;
                const int64_t t0 = t_begin + (int64_t)i * NT;
                const int nval = (int)std::min<int64_t>(NT, t_end - t0) - tb0;   // valid tokens of this half
                if (!bar_wait_warp(&bars.s_full, (uint32_t)(i & 1)) ||
                    !bar_wait_warp(&bars.scal_full[b], (uint32_t)((i >> 1) & 1))) {
                    failed = true;
                    break;
                }
                tqdev::tc_fence_after();
                const float4 *sc4 = reinterpret_cast<const float4 *>(scal + b * 3 * NT + tb0);
                float sv[32];
                {
                    float a[32], c[32];
                    tqdev::tmem_ld_32x32b_x32_nowait(tl + L::COL_MSE + tb0, a);
                    tqdev::tmem_ld_32x32b_x32_nowait(tl + L::COL_QJL + tb0, c);
                    tqdev::tmem_wait_ld();
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4) {
                        const float4 x1 = sc4[q4], x2 = sc4[NT / 4 + q4];
                        const float a1[4] = {x1.x, x1.y, x1.z, x1.w}, a2[4] = {x2.x, x2.y, x2.z, x2.w};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int t = 4 * q4 + u;
                            sv[t] = t < nval ? fmaf(a1[u], a[t], a2[u] * c[t]) : -INFINITY;
                        }
                    }
                }
                tqdev::tc_fence_before();
                __syncwarp();
                if (lane == 0) tqdev::mbar_arrive(&bars.s_free);   // the next tile's scores may be written
                float mx[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) mx[u] = fmaxf(fmaxf(sv[4 * u], sv[4 * u + 1]), fmaxf(sv[4 * u + 2], sv[4 * u + 3]));
                float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
                xch[((i & 1) * 2 + half) * 128 + r] = mt;
                if (!pair_sync()) {
                    failed = true;
                    break;
                }
                mt = fmaxf(mt, xch[((i & 1) * 2 + (half ^ 1)) * 128 + r]);
                float corr = 1.f;
                bool resc = false;
                if (mt > m2 + kRescale) {
                    corr = m2 == -INFINITY ? 0.f : exp2f(m2 - mt);
                    m2 = mt;
                    resc = true;
                }
                uint32_t ph[16], pq[16];
                float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) {
                    const float4 vn = sc4[NT / 2 + q4];
                    const float vv[4] = {vn.x, vn.y, vn.z, vn.w};
                    float p[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int t = 4 * q4 + u;
                        p[u] = t < nval ? exp2f(sv[t] - m2) : 0.f;
                        ls[u] += p[u];
                    }
                    split_bf16x2(p[0] * vv[0], p[1] * vv[1], ph[2 * q4], pq[2 * q4]);
                    split_bf16x2(p[2] * vv[2], p[3] * vv[3], ph[2 * q4 + 1], pq[2 * q4 + 1]);
                }
                l_part = fmaf(l_part, corr, (ls[0] + ls[1]) + (ls[2] + ls[3]));
                __syncwarp();
                if (lane == 0) tqdev::mbar_arrive(&bars.scal_free[b]);
                if (i > 0) {
                    // the previous tile's value MMAs have read P and written O
                    if (!bar_wait_warp(&bars.p_free, (uint32_t)((i - 1) & 1))) {
                        failed = true;
                        break;
                    }
                    tqdev::tc_fence_after();
                    if (__any_sync(0xffffffffu, resc)) {
                        // each half rescales its half of the output columns
#pragma unroll 1
                        for (int c = half * (D / 64); c < (half + 1) * (D / 64); ++c) {
                            float o[32];
                            tqdev::tmem_ld_32x32b_x32(tl + L::COL_O + 32 * c, o);
#pragma unroll
                            for (int k = 0; k < 32; ++k) o[k] *= corr;
                            tqdev::tmem_st_32x32b_x32(tl + L::COL_O + 32 * c, o);
                        }
                        tqdev::tmem_wait_st();
                    }
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t off = sw128_off(r, 4 * half + c, 0);
                    *reinterpret_cast<uint4 *>(prow + off) = make_uint4(ph[4 * c], ph[4 * c + 1], ph[4 * c + 2], ph[4 * c + 3]);
                    *reinterpret_cast<uint4 *>(prow + L::PB + off) =
                        make_uint4(pq[4 * c], pq[4 * c + 1], pq[4 * c + 2], pq[4 * c + 3]);
                }
                tqdev::fence_proxy_async_smem();
                tqdev::tc_fence_before();
                __syncwarp();
                if (lane == 0) tqdev::mbar_arrive(&bars.p_full);
            }
            if (!failed && !bar_wait_warp(&bars.p_free, (uint32_t)((nt - 1) & 1))) failed = true;
        }
        // ---- the row's sum of weights, then rotate back: out = D H O / d with
        // H_d = H_2 x H_{d/2}: each half transforms its d/2 columns in
        // registers, and the halves' last stage meets in shared memory
        constexpr int HC = D / 2;   // output columns per half
        lx[half * 128 + r] = l_part;
        const bool paired = pair_sync();
        const float l_run = lx[r] + lx[128 + r];
        const bool have = run && !failed && paired;
        float o[HC];
        if (have) {
            tqdev::tc_fence_after();
#pragma unroll
            for (int c = 0; c < HC / 32; ++c) {
                float t32[32];
                tqdev::tmem_ld_32x32b_x32(tl + L::COL_O + HC * half + 32 * c, t32);
                wht32(t32);
#pragma unroll
                for (int k = 0; k < 32; ++k) o[32 * c + k] = t32[k];
            }
#pragma unroll
            for (int len = 32; len < HC; len <<= 1)
#pragma unroll
                for (int k = 0; k < HC; ++k) {
                    if (k & len) continue;
                    const float x0 = o[k], x1 = o[k + len];
                    o[k] = x0 + x1;
                    o[k + len] = x0 - x1;
                }
        } else {
#pragma unroll
            for (int k = 0; k < HC; ++k) o[k] = 0.f;
        }
        // exchange buffers [half][row][HC] and the output staging [row][d],
        // both with 16-byte chunk c of row r at chunk c ^ (r % 8)
        float *xo = reinterpret_cast<float *>(sm + L::OFF_K);
        float *ost = xo + 2 * 128 * HC;
        {
            float *mine = xo + (half * 128 + r) * HC;
#pragma unroll
            for (int c = 0; c < HC / 4; ++c)
                *reinterpret_cast<float4 *>(mine + ((c ^ (r & 7)) << 2)) =
                    make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
        }
        const bool both = pair_sync() && have;
        const float *other = xo + ((half ^ 1) * 128 + r) * HC;
        const float sc = both ? 1.f / (float)D : 0.f;
        uint32_t sgn[HC / 32];   // sign words of this half's output columns
#pragma unroll
        for (int c = 0; c < HC / 32; ++c) sgn[c] = __ldg(g.signs + (int64_t)h * (D / 32) + (HC / 32) * half + c);
        // half 0: a + b (output columns [0, d/2)); half 1: a - b, a being half 0's
        const float sa = half == 0 ? 1.f : -1.f;
#pragma unroll
        for (int c = 0; c < HC / 4; ++c) {
            const float4 p4 = *reinterpret_cast<const float4 *>(other + ((c ^ (r & 7)) << 2));
            o[4 * c] = (p4.x + sa * o[4 * c]) * sc;
            o[4 * c + 1] = (p4.y + sa * o[4 * c + 1]) * sc;
            o[4 * c + 2] = (p4.z + sa * o[4 * c + 2]) * sc;
            o[4 * c + 3] = (p4.w + sa * o[4 * c + 3]) * sc;
        }
#pragma unroll
        for (int k = 0; k < HC; ++k)
            if ((sgn[k >> 5] >> (k & 31)) & 1u) o[k] = -o[k];
        if (P.direct) {
            if (qvalid) {
                const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
                const int64_t obase = ((int64_t)(g.first_seq + seq_local) * P.Hq + jh) * D + HC * half;
#pragma unroll
                for (int k = 0; k < HC; ++k) store_out_elem(P.out, obase + k, o[k] * inv_l, P.out_dtype);
            }
        } else {
#pragma unroll
            for (int c = 0; c < HC / 4; ++c) {
                const int k = (HC * half) / 4 + c;   // 16-byte chunk of the output row
                *reinterpret_cast<float4 *>(ost + r * D + ((k ^ (r & 7)) << 2)) =
                    make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
            }
        }
        if (half == 0) {
            mlr[2 * r] = both ? m2 * 0.6931471805599453f : -INFINITY;   // back to natural units
            mlr[2 * r + 1] = both ? l_run : 0.f;
        }
        if (!P.direct) {
            // coalesced partials: one warp per row, [m, l, 0, 0 | o]
            tqdev::named_sync(1, 32 * SM_WARPS);
            constexpr int OCH = D / 4;   // 16-byte chunks of a row's output
            const int rows = min(MMA_Q, nq - qchunk * MMA_Q);
            int sl = (qchunk * MMA_Q + warp) / P.G, gq = (qchunk * MMA_Q + warp) % P.G;
#pragma unroll 1
            for (int rr = warp; rr < rows; rr += SM_WARPS) {
                float *dst = P.part + (g.part_base + ((int64_t)split * g.n_seqs + sl) * P.Hq + h * P.G + gq) * tq_part_floats(D);
                if (lane < OCH) {
                    const float4 x = *reinterpret_cast<const float4 *>(ost + rr * D + ((lane ^ (rr & 7)) << 2));
                    reinterpret_cast<float4 *>(dst + 4)[lane] = x;
                }
                if (lane == 0) reinterpret_cast<float4 *>(dst)[0] = make_float4(mlr[2 * rr], mlr[2 * rr + 1], 0.f, 0.f);
                // next row of this warp: query index + SM_WARPS
                gq += SM_WARPS;
                while (gq >= P.G) {
                    gq -= P.G;
                    ++sl;
                }
            }
        }
    }
    if (failed) atomicOr(reinterpret_cast<unsigned int *>(g.status + 1), TQ_FLAG_WAIT_TIMEOUT);
    tqdev::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tqdev::tc_fence_after();
        tqdev::tmem_dealloc(tmem, 512);
    }
}

}  // namespace

// ------------------------------------------------------------------ host side
namespace {

constexpr size_t kMaxDynSmemMma = 232448;   // 227 KB per block on sm_100

size_t mma_smem_bytes(int d, int m, int bk, int bv, int krow, int vrow) {
    const size_t kx = (size_t)MMA_NT * 128;
    const size_t cb = (size_t)(d / 64) * kx, sb = (size_t)(m / 64) * kx;
    const size_t fixed = 2 * (2 * cb + sb) + 2 * (2 * cb) + 2 * (size_t)MMA_Q * 128 + 2 * 3 * MMA_NT * 4 + 4096;
    const size_t tabs = ((size_t)1 << (2 * bk)) * 8 + (size_t)(bv == 5 ? 32 : 1 << (2 * bv)) * 8;
    return 1024 + fixed + tabs + 2 * (size_t)MMA_NT * (size_t)(krow + vrow);
}

template <int D, int BK, int BV, int MP>
cudaError_t launch_mma_t(const DecodePlan &P, int64_t items, int krow, int vrow, cudaStream_t stream) {
    static_assert(MmaLayout<D, MP>::OFF_TAB + 16 <= (int)kMaxDynSmemMma, "layout");
    const size_t smem = mma_smem_bytes(D, MP, BK, BV, krow, vrow);
    if (smem > kMaxDynSmemMma) return cudaErrorInvalidValue;
    auto kern = tq_decode_mma_kernel<D, BK, BV, MP>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return e;
    }
    e = tq_launch_dependent(kern, dim3((unsigned)items), dim3(MMA_THREADS), smem, stream, P);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int D, int MP>
cudaError_t launch_mma_bits(int bk, const DecodePlan &P, int64_t items, int krow, int vrow, cudaStream_t st) {
    switch (bk) {
        case 1: return launch_mma_t<D, 1, 2, MP>(P, items, krow, vrow, st);
        case 2: return launch_mma_t<D, 2, 3, MP>(P, items, krow, vrow, st);
        case 3: return launch_mma_t<D, 3, 4, MP>(P, items, krow, vrow, st);
        case 4: return launch_mma_t<D, 4, 5, MP>(P, items, krow, vrow, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

bool tq_decode_mma_fits(int d, int m, int bk, int bv, int krow, int vrow) {
    if (!(d == 64 || d == 128) || !(m == 64 || m == 128) || bk < 1 || bk > 4 || bv != bk + 1) return false;
    return mma_smem_bytes(d, m, bk, bv, krow, vrow) <= kMaxDynSmemMma;
}

cudaError_t tq_launch_decode_mma(const DecodePlan &P, int64_t items, int d, int m, int bk, int krow, int vrow,
                                 cudaStream_t stream) {
    if (d == 128) {
        if (m == 128) return launch_mma_bits<128, 128>(bk, P, items, krow, vrow, stream);
        if (m == 64) return launch_mma_bits<128, 64>(bk, P, items, krow, vrow, stream);
    } else if (d == 64) {
        if (m == 128) return launch_mma_bits<64, 128>(bk, P, items, krow, vrow, stream);
        if (m == 64) return launch_mma_bits<64, 64>(bk, P, items, krow, vrow, stream);
    }
    return cudaErrorInvalidValue;
}
