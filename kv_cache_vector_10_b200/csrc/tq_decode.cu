// tq_decode.cu -- split-K decode attention over the packed cache (sm_100a).
//
// For each (segment, kv-head, token split, query chunk) one CTA of 8 warps:
//   * builds per-query lookup tables in shared memory.  Key scores need
//     <q_rot, C[idx]> and <S q_rot, 2b-1> (turboquant-plus-rs README,
//     Architecture: TurboQuant inner-product estimate).  The codebook is
//     antisymmetric, so C[idx] is a sum over odd subsets A of the index bits
//     of alpha_A * sigma_A with sigma_A = +-1 the parity of the bits in A
//     (Walsh expansion).  Each sigma-plane, like the QJL sign plane, is a
//     +-1 pattern, so its inner product with a vector is a sum of 16 byte
//     lookups into a table LUT[g][byte] = sum_{i<8} v[8g+i] (2 bit_i - 1).
//   * streams 32-token chunks of packed key and value rows into shared
//     memory with bulk async copies (two buffers per warp);
//   * scores two tokens per warp step (16 lanes per token, one byte group
//     per lane), reduces the 16 partial sums by a transposing butterfly,
//     keeps an online softmax per query, and accumulates the value sum in
//     the rotated frame with the same layout (8 coordinates of one token per
//     lane per step; two codes per lookup in a replicated pair table; packed
//     fp32x2 multiply-adds);
//   * merges its warps, rotates the partial output back (Pi^T) and writes
//     (max, sum, output) for the combine kernel.
// Every query of a kv-head group (GQA) and every sequence of a shared
// segment reads the same staged tile.
#include <algorithm>
#include <climits>
#include <cstdlib>
#include <cstring>
#include <cmath>
#include <vector>

#include "tq_decode.cuh"

cudaError_t tq_launch_qprep(const DecodePlan &P, const void *q, tq_dtype dt, cudaStream_t stream);
cudaError_t tq_launch_combine(const DecodePlan &P, void *out, tq_dtype dt, cudaStream_t stream);

namespace {

template <int QC>
struct Vec;
template <>
struct Vec<1> {
    using T = float;
    __device__ static float get(const float &v, int) { return v; }
    __device__ static float make(const float (&a)[1]) { return a[0]; }
};
template <>
struct Vec<2> {
    using T = float2;
    __device__ static float get(const float2 &v, int i) { return i == 0 ? v.x : v.y; }
    __device__ static float2 make(const float (&a)[2]) { return make_float2(a[0], a[1]); }
};
template <>
struct Vec<4> {
    using T = float4;
    __device__ static float get(const float4 &v, int i) { return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w; }
    __device__ static float4 make(const float (&a)[4]) { return make_float4(a[0], a[1], a[2], a[3]); }
};

// Odd subsets of BK index bits: XOR masks of the sigma-planes.
__host__ __device__ constexpr int n_sigma_planes(int bk) { return bk == 1 ? 1 : bk == 2 ? 2 : bk == 3 ? 4 : 8; }
__host__ __device__ constexpr uint32_t sigma_set(int bk, int s) {
    // singletons first, then triples
    return s < bk ? (1u << s)
                  : (bk == 3 ? 7u : (s == 4 ? 7u : s == 5 ? 11u : s == 6 ? 13u : 14u));
}

// Table slot of (round, byte, half, slot): QC == 1 keeps one copy per half
// warp so 32 lanes read 32 distinct banks; wider entries are read in
// half/quarter-warp phases and need no copy.
template <int QC>
__device__ __forceinline__ int lut_slot(int round, int byte, int half, int slot) {
    if constexpr (QC == 1) return ((round * 256 + byte) * 2 + half) * 16 + slot;
    else return (round * 256 + byte) * 16 + slot;
}
template <int QC>
__host__ __device__ constexpr int lut_entries(int rounds) {
    return rounds * 256 * 16 * (QC == 1 ? 2 : 1);
}

// Stage one chunk of packed key and value rows (tokens [tb, tb + 32),
// clipped to the buffer capacity) into shared memory with two bulk copies
// completing on `bar`.
__device__ __forceinline__ void issue_chunk(uint8_t *dk, uint64_t *bar, const uint8_t *kbase, const uint8_t *vbase,
                                            int64_t tb, int64_t capacity, int krow, int vrow) {
    const int64_t ntok = min((int64_t)TQ_DEC_CHUNK, capacity - tb);
    uint8_t *dv = dk + TQ_DEC_CHUNK * krow;
    tqdev::mbar_expect_tx(bar, (uint32_t)(ntok * (krow + vrow)));
    tqdev::bulk_load(dk, kbase + tb * krow, (uint32_t)(ntok * krow), bar);
    tqdev::bulk_load(dv, vbase + tb * vrow, (uint32_t)(ntok * vrow), bar);
}

// Value pair table: entry e = two consecutive B_V-bit codes (low code in the
// low bits) -> the two centroids.  VCOPIES copies, indexed by the lane's slot,
// keep every half-warp access conflict-free.
template <int BV>
__host__ __device__ constexpr int vpair_copies() { return BV <= 4 ? 16 : 1; }
template <int BV>
__host__ __device__ constexpr int vpair_entries() { return 1 << (2 * BV); }

// One output element in the caller's type.
__device__ __forceinline__ void store_out_dt(void *p, int64_t i, float v, int dt) {
    if (dt == TQ_F32) static_cast<float *>(p)[i] = v;
    else if (dt == TQ_F16) static_cast<__half *>(p)[i] = __float2half_rn(v);
    else static_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(v);
}

// MT = number of QJL projections when known at compile time (128), else 0;
// KF = key norms as binary16 (1) or fp32 (0) when MT > 0 (else read from the
// segment); NBUF = staging buffers per warp (2, or 1 where two do not fit in
// shared memory: head_dim 256 at the larger bit widths).
template <int D, int BK, int BV, int QC, int MT, int KF, int NBUF>
__global__ void __launch_bounds__(TQ_DEC_WARPS * 32, 1) tq_decode_kernel(const __grid_constant__ DecodePlan P) {
    using VT = typename Vec<QC>::T;
    constexpr int NGK = D / 8;                    // byte groups of an index plane = value slots
    constexpr int RK = (NGK + 15) / 16;
    constexpr int NP = n_sigma_planes(BK);
    constexpr int VPB = 2 * BV;                   // bits of a value pair
    constexpr int VCOP = vpair_copies<BV>();
    static_assert(D == 64 || D == 128 || D == 256, "head_dim");
    static_assert(NBUF == 1 || NBUF == 2, "staging depth");
    constexpr int VR = D > 128 ? D / 128 : 1;      // value rounds: 128 coordinates per warp-half each
    extern __shared__ __align__(128) uint8_t smem_raw[];

    // An append step's new rows are written by the query-preparation kernel:
    // wait for it before any row is read.  Otherwise only the prepared
    // queries depend on it (wait below, after the first tiles are requested).
    if (P.n_append_blocks) tqdev::grid_dep_wait();
    tqdev::grid_dep_trigger();
    // ---- locate the work item
    int s = 0;
    int64_t item = blockIdx.x;
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
    const int M = MT > 0 ? MT : g.m;
    const int NGS = M / 8, RS = (NGS + 15) / 16;
    const int krow = MT > 0 ? BK * D / 8 + MT / 8 + (KF ? 4 : 8) : g.krow;
    const int vrow = MT > 0 ? BV * D / 8 + 4 : g.vrow;
    const int64_t t_begin = (int64_t)split * g.split_len;
    const int64_t t_end = std::min<int64_t>(g.T, t_begin + g.split_len);
    const int nq = g.n_seqs * P.G;

    // ---- shared memory carve-up
    VT *lutq = reinterpret_cast<VT *>(smem_raw);
    VT *luts = lutq + lut_entries<QC>(RK);
    float2 *vlut = reinterpret_cast<float2 *>(luts + lut_entries<QC>(RS));
    uint64_t *bars = reinterpret_cast<uint64_t *>(vlut + vpair_entries<BV>() * VCOP);
    // several queries per CTA: the value pass reads each token's softmax
    // weights (all queries in one entry) from a per-warp array
    VT *wbuf = reinterpret_cast<VT *>(bars + NBUF * TQ_DEC_WARPS);
    uint8_t *stage = reinterpret_cast<uint8_t *>(wbuf + (QC > 1 ? TQ_DEC_WARPS * TQ_DEC_CHUNK : 0));
    const int chunk_bytes = TQ_DEC_CHUNK * (krow + vrow);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int half = lane >> 4, slot = lane & 15;             // value pass: 16 lanes per token
    // score pass: lanes per token; 8 for 4 queries per CTA (16-byte table
    // entries: a quarter-warp of one token reads 8 distinct bank groups)
    constexpr int LPT = QC == 4 ? 8 : 16;
    constexpr int TPS = 32 / LPT;                              // tokens per score step
    const int sl = lane % LPT, tg = lane / LPT;

    for (int i = tid; i < vpair_entries<BV>() * VCOP; i += blockDim.x) {
        const int e = i / VCOP;
        vlut[i] = make_float2(g.vtab[e & ((1 << BV) - 1)], g.vtab[e >> BV]);
    }
    // The abort flag is read once per CTA, before any copy is requested: a CTA
    // of an aborted context requests nothing and waits for nothing.
    __shared__ int s_abort;
    if (tid == 0) {
        for (int i = 0; i < NBUF * TQ_DEC_WARPS; ++i) tqdev::mbar_init(&bars[i], 1);
        tqdev::fence_barrier_init();
        s_abort = tqdev::status_aborted(g.status) ? 1 : 0;
    }
    __syncthreads();
    const bool pre_aborted = s_abort != 0;

    const int64_t n_chunks = t_end > t_begin ? (t_end - t_begin + TQ_DEC_CHUNK - 1) / TQ_DEC_CHUNK : 0;
    const uint8_t *kbase = g.kc + (int64_t)h * g.capacity * krow;
    const uint8_t *vbase = g.vc + (int64_t)h * g.capacity * vrow;
    if (lane == 0 && !pre_aborted) {
#pragma unroll
        for (int b = 0; b < NBUF; ++b)
            if (warp + b * TQ_DEC_WARPS < n_chunks)
                issue_chunk(stage + (warp * NBUF + b) * chunk_bytes, &bars[warp * NBUF + b], kbase, vbase,
                            t_begin + (warp + b * TQ_DEC_WARPS) * TQ_DEC_CHUNK, g.capacity, krow, vrow);
    }

    // ---- per-query lookup tables (from the query-preparation kernel's output)
    tqdev::grid_dep_wait();
    const float *qp_base = P.qprep + g.qprep_base;
    for (int li = tid; li < 256; li += blockDim.x) {
        const int gslot = li % 16, lo = li / 16;     // fixed low nibble per build lane
        for (int kind = 0; kind < 2; ++kind) {
            const int NG = kind == 0 ? NGK : NGS, R = kind == 0 ? RK : RS;
            VT *lut = kind == 0 ? lutq : luts;
            for (int r = 0; r < R; ++r) {
                const int gg = r * 16 + gslot;
                float lo_v[QC], hi_v[QC], hv[QC][4];
#pragma unroll
                for (int qq = 0; qq < QC; ++qq) {
                    const int qi = qchunk * QC + qq;
                    const float *v = qi < nq ? qp_base + ((int64_t)(qi / P.G) * P.Hq + h * P.G + qi % P.G) * (D + M)
                                             : nullptr;
                    float vals[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) vals[i] = (v && gg < NG) ? v[(kind == 0 ? 0 : D) + 8 * gg + i] : 0.f;
                    float a = 0.f, b = 0.f;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        a += ((lo >> i) & 1) ? vals[i] : -vals[i];
                        b -= vals[4 + i];
                        hv[qq][i] = 2.f * vals[4 + i];
                    }
                    lo_v[qq] = a;
                    hi_v[qq] = b;
                }
                int gray = 0;
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    if (k > 0) {
                        const int f = __ffs(k) - 1;
                        const bool up = !((gray >> f) & 1);
                        gray ^= 1 << f;
#pragma unroll
                        for (int qq = 0; qq < QC; ++qq) hi_v[qq] += up ? hv[qq][f] : -hv[qq][f];
                    }
                    const int byte = lo | (gray << 4);
                    float ev[QC];
#pragma unroll
                    for (int qq = 0; qq < QC; ++qq) ev[qq] = lo_v[qq] + hi_v[qq];
                    const VT e = Vec<QC>::make(ev);
                    lut[lut_slot<QC>(r, byte, 0, gslot)] = e;
                    if constexpr (QC == 1) lut[lut_slot<QC>(r, byte, 1, gslot)] = e;
                }
            }
        }
    }
    __syncthreads();

    // ---- main loop
    float alpha[NP];
#pragma unroll
    for (int sp = 0; sp < NP; ++sp) alpha[sp] = g.alpha[sp];
    const float inv_d = 1.f / (float)D;
    const float cqs = 1.2533141373155003f / (float)M * rsqrtf((float)D);   // sqrt(pi/2)/m/sqrt(d)
    const int off_sign = BK * (D / 8);
    const int off_ns = off_sign + M / 8;
    const bool kf16 = MT > 0 ? KF != 0 : g.kf16 != 0;
    const int voff_ns = BV * D / 8;
    // value bits of this lane's 8 coordinates of round r (coordinates
    // 128 r + 8 slot .. + 7): [8*BV*(16 r + slot), + 8*BV)
    const bool vslot = slot < NGK;
    const int vcopy = VCOP > 1 ? slot : 0;

    float m_run[QC], l_lane[QC];
    float2 o[QC][4 * VR];   // coordinates 128 r + 8*slot + 2p, +1 at [4 r + p] (tokens of parity `half`)
#pragma unroll
    for (int qq = 0; qq < QC; ++qq) {
        m_run[qq] = -INFINITY;
        l_lane[qq] = 0.f;
#pragma unroll
        for (int c = 0; c < 4 * VR; ++c) o[qq][c] = make_float2(0.f, 0.f);
    }
    bool aborted = pre_aborted;
    for (int64_t k = 0; !aborted; ++k) {
        const int64_t ci = warp + k * TQ_DEC_WARPS;
        if (ci >= n_chunks) break;
        const int buf = (int)(k % NBUF);
        if (!tqdev::mbar_wait_bounded(&bars[warp * NBUF + buf], (uint32_t)((k / NBUF) & 1))) {
            aborted = true;
            // Each of this warp's buffers may still have a copy in flight (the
            // one just waited for, and with two buffers the next chunk's in the
            // other): give each one more bounded wait before `stage` is reused.
            tqdev::mbar_wait_bounded(&bars[warp * NBUF + buf], (uint32_t)((k / NBUF) & 1));
            if (NBUF == 2 && ci + TQ_DEC_WARPS < n_chunks)
                tqdev::mbar_wait_bounded(&bars[warp * NBUF + (buf ^ 1)], (uint32_t)(((k + 1) / NBUF) & 1));
            break;
        }
        const uint8_t *sK = stage + (warp * NBUF + buf) * chunk_bytes;
        const uint8_t *sV = sK + TQ_DEC_CHUNK * krow;
        const int64_t t0 = t_begin + ci * TQ_DEC_CHUNK;

        // scores: LPT lanes per token (16, or 8 for 4 queries per CTA),
        // TPS tokens per step; lane (tg, sl) scores token TPS * st + tg, byte
        // groups sl + LPT * i of each 16-group round
        float part[QC][LPT];
#pragma unroll
        for (int st = 0; st < LPT; ++st) {
            const uint8_t *kr = sK + (TPS * st + tg) * krow;
            // query pairs accumulate in packed fp32x2 (one pair when QC == 1)
            float2 am[(QC + 1) / 2], as[(QC + 1) / 2];
#pragma unroll
            for (int qp = 0; qp < (QC + 1) / 2; ++qp) am[qp] = as[qp] = make_float2(0.f, 0.f);
#pragma unroll
            for (int r = 0; r < RK; ++r) {
#pragma unroll
                for (int gi = 0; gi < 16 / LPT; ++gi) {
                    const int gs = sl + LPT * gi, gg = r * 16 + gs;
                    if (gg < NGK) {
                        uint32_t pb[BK];
#pragma unroll
                        for (int pl = 0; pl < BK; ++pl) pb[pl] = kr[pl * (D / 8) + gg];
#pragma unroll
                        for (int sp = 0; sp < NP; ++sp) {
                            uint32_t x = 0;
#pragma unroll
                            for (int pl = 0; pl < BK; ++pl)
                                if ((sigma_set(BK, sp) >> pl) & 1) x ^= pb[pl];
                            const VT e = lutq[lut_slot<QC>(r, (int)x, tg, gs)];
                            if constexpr (QC == 1) {
                                am[0].x = fmaf(alpha[sp], Vec<QC>::get(e, 0), am[0].x);
                            } else {
#pragma unroll
                                for (int qp = 0; qp < QC / 2; ++qp)
                                    am[qp] = __ffma2_rn(make_float2(alpha[sp], alpha[sp]),
                                                        make_float2(Vec<QC>::get(e, 2 * qp), Vec<QC>::get(e, 2 * qp + 1)), am[qp]);
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < RS; ++r) {
#pragma unroll
                for (int gi = 0; gi < 16 / LPT; ++gi) {
                    const int gs = sl + LPT * gi, gg = r * 16 + gs;
                    if (gg < NGS) {
                        const VT e = luts[lut_slot<QC>(r, kr[off_sign + gg], tg, gs)];
                        if constexpr (QC == 1) {
                            as[0].x += Vec<QC>::get(e, 0);
                        } else {
#pragma unroll
                            for (int qp = 0; qp < QC / 2; ++qp)
                                as[qp] = __fadd2_rn(make_float2(Vec<QC>::get(e, 2 * qp), Vec<QC>::get(e, 2 * qp + 1)), as[qp]);
                        }
                    }
                }
            }
            const float2 nrm = tqdev::key_norms(reinterpret_cast<const uint32_t *>(kr + off_ns), kf16);
            const float a1 = nrm.x * inv_d, a2 = nrm.y * cqs;
            if constexpr (QC == 1) {
                part[0][st] = fmaf(a1, am[0].x, a2 * as[0].x);
            } else {
#pragma unroll
                for (int qp = 0; qp < QC / 2; ++qp) {
                    const float2 v = __ffma2_rn(make_float2(a1, a1), am[qp], __fmul2_rn(make_float2(a2, a2), as[qp]));
                    part[2 * qp][st] = v.x;
                    part[2 * qp + 1][st] = v.y;
                }
            }
        }
        // transposing butterfly over the LPT lanes of each token group
#pragma unroll
        for (int qq = 0; qq < QC; ++qq) {
#pragma unroll
            for (int w = LPT / 2; w >= 1; w >>= 1) {
                const bool up = (sl & w) != 0;
#pragma unroll
                for (int i = 0; i < w; ++i) {
                    const float send = up ? part[qq][i] : part[qq][i + w];
                    const float keep = up ? part[qq][i + w] : part[qq][i];
                    part[qq][i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
                }
            }
        }
        // this lane now holds the score of token TPS * sl + tg
        const int tok = TPS * sl + tg;
        const bool valid = t0 + tok < t_end;
        const float nsv = *reinterpret_cast<const float *>(sV + tok * vrow + voff_ns);
        float w_tok[QC];
#pragma unroll
        for (int qq = 0; qq < QC; ++qq) {
            const float sc = valid ? part[qq][0] : -INFINITY;
            float cm = sc;
#pragma unroll
            for (int w = 16; w >= 1; w >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, w));
            const float mn = fmaxf(m_run[qq], cm);
            const float corr = (mn == -INFINITY) ? 1.f : __expf(m_run[qq] - mn);
            const float pr = valid ? __expf(sc - mn) : 0.f;
            l_lane[qq] = fmaf(l_lane[qq], corr, pr);
            const float2 c2 = make_float2(corr, corr);
#pragma unroll
            for (int c = 0; c < 4 * VR; ++c) o[qq][c] = __fmul2_rn(o[qq][c], c2);
            m_run[qq] = mn;
            w_tok[qq] = valid ? pr * nsv : 0.f;
        }
        if constexpr (QC > 1) {
            wbuf[warp * TQ_DEC_CHUNK + tok] = Vec<QC>::make(w_tok);
            __syncwarp();
        }
        // values: step st again covers tokens 2*st + half; lane slot g owns
        // coordinates 8g..8g+7 (four value pairs)
#pragma unroll 4
        for (int st = 0; st < 16; ++st) {
            const uint32_t *vr = reinterpret_cast<const uint32_t *>(sV + (2 * st + half) * vrow);
            float2 wq[QC];
            if constexpr (QC > 1) {
                const VT w4 = wbuf[warp * TQ_DEC_CHUNK + 2 * st + half];
#pragma unroll
                for (int qq = 0; qq < QC; ++qq) wq[qq] = make_float2(Vec<QC>::get(w4, qq), Vec<QC>::get(w4, qq));
            } else {
                const int tv = 2 * st + half;   // held by lane (tv % TPS) * LPT + tv / TPS
                const float wv = __shfl_sync(0xffffffffu, w_tok[0], (tv % TPS) * LPT + tv / TPS);
                wq[0] = make_float2(wv, wv);
            }
            if (vslot) {
#pragma unroll
                for (int r = 0; r < VR; ++r) {
                    const int vbit = 8 * BV * (16 * r + slot);
                    const int vw0 = vbit / 32, vsh = vbit % 32;
                    uint32_t raw;
                    if constexpr (BV == 4) raw = vr[vw0];
                    else raw = __funnelshift_r(vr[vw0], vr[vw0 + 1], vsh);
                    uint32_t raw_hi = 0;
                    if constexpr (BV == 5) raw_hi = __funnelshift_r(vr[vw0 + 1], vr[vw0 + 2], vsh);
#pragma unroll
                    for (int pp = 0; pp < 4; ++pp) {
                        uint32_t e;
                        if constexpr (BV == 5) {
                            const int sh = VPB * pp;
                            e = (sh >= 32 ? raw_hi >> (sh - 32) : (sh + VPB > 32 ? (raw >> sh) | (raw_hi << (32 - sh)) : raw >> sh)) &
                                ((1u << VPB) - 1);
                        } else {
                            e = (raw >> (VPB * pp)) & ((1u << VPB) - 1);
                        }
                        const float2 cv = vlut[e * VCOP + vcopy];
#pragma unroll
                        for (int qq = 0; qq < QC; ++qq) o[qq][4 * r + pp] = __ffma2_rn(wq[qq], cv, o[qq][4 * r + pp]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0 && ci + NBUF * TQ_DEC_WARPS < n_chunks) {
            tqdev::fence_proxy_async_smem();
            issue_chunk(stage + (warp * NBUF + buf) * chunk_bytes, &bars[warp * NBUF + buf], kbase, vbase,
                        t_begin + (ci + NBUF * TQ_DEC_WARPS) * TQ_DEC_CHUNK, g.capacity, krow, vrow);
        }
    }
    if (aborted && lane == 0) atomicOr(reinterpret_cast<unsigned int *>(g.status + 1), TQ_FLAG_WAIT_TIMEOUT);

    // ---- merge token parities, then warps; rotate back; write partials
    __syncthreads();
    float *scr = reinterpret_cast<float *>(stage);              // [warp][QC][D + 2]
#pragma unroll
    for (int qq = 0; qq < QC; ++qq) {
        float lt = l_lane[qq];
#pragma unroll
        for (int w = 16; w >= 1; w >>= 1) lt += __shfl_xor_sync(0xffffffffu, lt, w);
        float *row = scr + (warp * QC + qq) * (D + 2);
        if (lane == 0) {
            row[0] = aborted ? -INFINITY : m_run[qq];
            row[1] = aborted ? 0.f : lt;
        }
#pragma unroll
        for (int c = 0; c < 4 * VR; ++c) {
            float2 v = o[qq][c];
            v.x += __shfl_xor_sync(0xffffffffu, v.x, 16);
            v.y += __shfl_xor_sync(0xffffffffu, v.y, 16);
            if (half == 0 && vslot) {
                const int j = 128 * (c / 4) + 8 * slot + 2 * (c % 4);
                row[2 + j] = aborted ? 0.f : v.x;
                row[2 + j + 1] = aborted ? 0.f : v.y;
            }
        }
    }
    __syncthreads();
    float *acc = scr + TQ_DEC_WARPS * QC * (D + 2);             // [QC][D]
    float *ml = acc + QC * D;                                    // [QC][2]
    for (int i = tid; i < QC * D; i += blockDim.x) {
        const int qq = i / D, j = i % D;
        float mx = -INFINITY;
        for (int w = 0; w < TQ_DEC_WARPS; ++w) mx = fmaxf(mx, scr[(w * QC + qq) * (D + 2)]);
        float a = 0.f, l = 0.f;
        if (mx != -INFINITY)
            for (int w = 0; w < TQ_DEC_WARPS; ++w) {
                const float *row = scr + (w * QC + qq) * (D + 2);
                if (row[0] == -INFINITY) continue;
                const float f = __expf(row[0] - mx);
                a = fmaf(f, row[2 + j], a);
                l = fmaf(f, row[1], l);
            }
        acc[qq * D + j] = a;
        if (j == 0) {
            ml[2 * qq] = mx;
            ml[2 * qq + 1] = l;
        }
    }
    __syncthreads();
    if (g.Q) {
        // Haar rotation: out = Q^T acc / sqrt(d)
        const float *Qh = g.Q + (int64_t)h * D * D;
        const float isd = rsqrtf((float)D);
        for (int i = tid; i < QC * D; i += blockDim.x) {
            const int qq = i / D, j = i % D;
            const int qi = qchunk * QC + qq;
            if (qi >= nq) continue;
            const int seq_local = qi / P.G, jh = h * P.G + qi % P.G;
            float v = 0.f;
            for (int r = 0; r < D; ++r) v = fmaf(Qh[r * D + j], acc[qq * D + r], v);
            v *= isd;
            if (P.direct) {
                const float l = ml[2 * qq + 1];
                store_out_dt(P.out, ((int64_t)(g.first_seq + seq_local) * P.Hq + jh) * D + j, l > 0.f ? v / l : 0.f,
                             P.out_dtype);
                continue;
            }
            float *dst = P.part + (g.part_base + ((int64_t)split * g.n_seqs + seq_local) * P.Hq + jh) * tq_part_floats(D);
            dst[4 + j] = v;
            if (j == 0) {
                dst[0] = ml[2 * qq];
                dst[1] = ml[2 * qq + 1];
                dst[2] = 0.f;
                dst[3] = 0.f;
            }
        }
        return;
    }
    // Pi^T with the 1/sqrt(d) of the value scale: out = D H acc / d
    for (int len = 1; len < D; len <<= 1) {
        for (int i = tid; i < QC * D / 2; i += blockDim.x) {
            const int qq = i / (D / 2), ii = i % (D / 2);
            const int j = (ii / len) * 2 * len + (ii % len);
            float *a = acc + qq * D;
            const float x = a[j], y = a[j + len];
            a[j] = x + y;
            a[j + len] = x - y;
        }
        __syncthreads();
    }
    const uint32_t *sg = g.signs + (int64_t)h * (D / 32);
    for (int i = tid; i < QC * D; i += blockDim.x) {
        const int qq = i / D, j = i % D;
        const int qi = qchunk * QC + qq;
        if (qi >= nq) continue;
        const int seq_local = qi / P.G, jh = h * P.G + qi % P.G;
        float v = acc[qq * D + j] * inv_d;
        if ((sg[j / 32] >> (j % 32)) & 1) v = -v;
        if (P.direct) {
            const float l = ml[2 * qq + 1];
            store_out_dt(P.out, ((int64_t)(g.first_seq + seq_local) * P.Hq + jh) * D + j, l > 0.f ? v / l : 0.f,
                         P.out_dtype);
            continue;
        }
        float *dst = P.part + (g.part_base + ((int64_t)split * g.n_seqs + seq_local) * P.Hq + jh) * tq_part_floats(D);
        dst[4 + j] = v;
        if (j == 0) {
            dst[0] = ml[2 * qq];
            dst[1] = ml[2 * qq + 1];
            dst[2] = 0.f;
            dst[3] = 0.f;
        }
    }
}

// ------------------------------------------------------------------ planning
struct SegPlan {
    int qc;                    // queries per CTA (TQ_MMA_QUERIES: the tensor-core decode)
    int n_qchunks, n_splits, split_len;
    int64_t part_floats, qprep_floats;
};

// Queries per kv head (sequences x query heads of a group) from which a
// segment is decoded on the tensor cores, where its format fits them.
// TQ_DECODE_PATH=lut keeps every segment on the lookup-table decode and
// TQ_DECODE_PATH=mma sends every segment that fits to the tensor cores.
int mma_min_queries() {
    const char *e = getenv("TQ_DECODE_PATH");
    if (e && strcmp(e, "lut") == 0) return 1 << 30;
    if (e && strcmp(e, "mma") == 0) return 1;
    return 16;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Shared memory of one decode CTA with nbuf staging buffers per warp (must
// match tq_decode_kernel's carve-up).
size_t decode_smem_bytes(int d, int bv, int qc, int krow, int vrow, int M, int nbuf) {
    const int RK = (d / 8 + 15) / 16, RS = (M / 8 + 15) / 16;
    const size_t vt = qc == 1 ? 4 : qc == 2 ? 8 : 16;
    const size_t lut = (size_t)(RK + RS) * 256 * 16 * (qc == 1 ? 2 : 1) * vt;
    const size_t vpair = (size_t)(1 << (2 * bv)) * (bv <= 4 ? 16 : 1) * 8;
    const size_t stage = (size_t)TQ_DEC_WARPS * nbuf * TQ_DEC_CHUNK * (krow + vrow);
    const size_t merge = ((size_t)TQ_DEC_WARPS * qc * (d + 2) + qc * d + 2 * qc) * 4;
    const size_t wbuf = qc > 1 ? (size_t)TQ_DEC_WARPS * TQ_DEC_CHUNK * vt : 0;
    return lut + vpair + (size_t)nbuf * TQ_DEC_WARPS * 8 + wbuf + std::max(stage, merge);
}

constexpr size_t kMaxDynSmem = 232448;   // 227 KB per block on sm_100

// Staging buffers per warp: two where they fit, else one (0: none fits).
int decode_nbuf(int d, int bv, int qc, int krow, int vrow, int M) {
    if (decode_smem_bytes(d, bv, qc, krow, vrow, M, 2) <= kMaxDynSmem) return 2;
    if (decode_smem_bytes(d, bv, qc, krow, vrow, M, 1) <= kMaxDynSmem) return 1;
    return 0;
}

void plan_segments(const tq_segment *segs, int n_segs, int Hq, int Hkv, int n_sms, std::vector<SegPlan> &out) {
    const int G = Hq / Hkv;
    const int qmin = mma_min_queries();
    out.resize(n_segs);
    for (int s = 0; s < n_segs; ++s) {
        const int nq = segs[s].n_seqs * G;
        SegPlan &p = out[s];
        const tq_ctx *c = segs[s].ctx;
        const int krow = (int)tq_row_bytes(c, TQ_KEYS), vrow = (int)tq_row_bytes(c, TQ_VALUES);
        if (nq >= qmin && c->rotation != TQ_ROT_HAAR && tq_decode_mma_fits(c->d, c->m, c->BK, c->BV, krow, vrow)) {
            p.qc = TQ_MMA_QUERIES;
        } else {
            p.qc = nq >= 4 ? 4 : nq >= 2 ? 2 : 1;
            while (p.qc > 1 && decode_nbuf(c->d, c->BV, p.qc, krow, vrow, c->m) == 0) p.qc /= 2;
        }
        p.n_qchunks = (nq + p.qc - 1) / p.qc;
    }
    // Split lengths, one per decode kind, each chosen to minimise the
    // estimated time = waves x (tokens per CTA + fixed per-CTA cost), so the
    // last wave is not mostly empty.  One decode CTA per SM is resident.
    auto choose = [&](bool mma, int64_t unit, int64_t fixed) {
        int64_t Tmax = 0;
        for (int s = 0; s < n_segs; ++s)
            if ((out[s].qc == TQ_MMA_QUERIES) == mma) Tmax = std::max<int64_t>(Tmax, segs[s].n_tokens);
        int64_t bestL = unit;
        double best = 1e300;
        for (int64_t L = unit;; L += unit) {
            int64_t items = 0;
            for (int s = 0; s < n_segs; ++s)
                if ((out[s].qc == TQ_MMA_QUERIES) == mma)
                    items += (int64_t)Hkv * out[s].n_qchunks * std::max<int64_t>(1, (segs[s].n_tokens + L - 1) / L);
            const int64_t waves = (items + n_sms - 1) / std::max(n_sms, 1);
            const double t = (double)waves * (double)(std::min(L, std::max<int64_t>(Tmax, 1)) + fixed);
            if (t < best - 1e-9) {
                best = t;
                bestL = L;
            }
            if (L >= Tmax) break;
        }
        return bestL;
    };
    // lookup-table decode: per-CTA set-up (tables, merge) ~ 256 tokens;
    // tensor-core decode: 64-token tiles, set-up and output ~ 3 tiles
    const int64_t L_lut = choose(false, TQ_DEC_SPLIT_UNIT, 256);
    const int64_t L_mma = choose(true, 64, 192);
    const int d = segs[0].ctx->d;
    for (int s = 0; s < n_segs; ++s) {
        SegPlan &p = out[s];
        const int64_t T = segs[s].n_tokens;
        const int64_t L = p.qc == TQ_MMA_QUERIES ? L_mma : L_lut;
        const int64_t ns = std::max<int64_t>(1, (T + L - 1) / L);
        p.n_splits = (int)ns;
        p.split_len = (int)L;
        p.part_floats = (int64_t)ns * segs[s].n_seqs * Hq * tq_part_floats(d);
        p.qprep_floats = (int64_t)segs[s].n_seqs * Hq * (d + segs[s].ctx->m);
    }
}

template <int D, int BK, int BV, int QC>
cudaError_t launch_decode_t(const DecodePlan &P, int64_t items, int krow, int vrow, int M, cudaStream_t stream) {
    const int nbuf = decode_nbuf(D, BV, QC, krow, vrow, M);
    if (nbuf == 0) return cudaErrorInvalidValue;
    const size_t smem = decode_smem_bytes(D, BV, QC, krow, vrow, M, nbuf);
    // the launch's segments share one key-row length, hence one norm format
    const bool kf16 = krow == BK * D / 8 + M / 8 + 4;
    auto kern = nbuf == 2 ? (M != 128 ? tq_decode_kernel<D, BK, BV, QC, 0, 0, 2>
                             : kf16   ? tq_decode_kernel<D, BK, BV, QC, 128, 1, 2>
                                      : tq_decode_kernel<D, BK, BV, QC, 128, 0, 2>)
                          : (M != 128 ? tq_decode_kernel<D, BK, BV, QC, 0, 0, 1>
                             : kf16   ? tq_decode_kernel<D, BK, BV, QC, 128, 1, 1>
                                      : tq_decode_kernel<D, BK, BV, QC, 128, 0, 1>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) {
        cudaGetLastError();   // do not leave the failure as the thread's sticky last error
        return e;
    }
    // starts while the query preparation (or the previous decode launch) runs
    e = tq_launch_dependent(kern, dim3((unsigned)items), dim3(TQ_DEC_WARPS * 32), smem, stream, P);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int D, int QC>
cudaError_t launch_decode_bits(int bits, const DecodePlan &P, int64_t items, int krow, int vrow, int M,
                               cudaStream_t st) {
    switch (bits) {
        case 2: return launch_decode_t<D, 1, 2, QC>(P, items, krow, vrow, M, st);
        case 3: return launch_decode_t<D, 2, 3, QC>(P, items, krow, vrow, M, st);
        case 4: return launch_decode_t<D, 3, 4, QC>(P, items, krow, vrow, M, st);
        case 5: return launch_decode_t<D, 4, 5, QC>(P, items, krow, vrow, M, st);
    }
    return cudaErrorInvalidValue;
}

template <int D>
cudaError_t launch_decode_dim(int bits, int qc, const DecodePlan &P, int64_t items, int krow, int vrow, int M,
                              cudaStream_t st) {
    if (qc == 1) return launch_decode_bits<D, 1>(bits, P, items, krow, vrow, M, st);
    if (qc == 2) return launch_decode_bits<D, 2>(bits, P, items, krow, vrow, M, st);
    return launch_decode_bits<D, 4>(bits, P, items, krow, vrow, M, st);
}

// Walsh coefficients of an antisymmetric codebook over its index bits:
// alpha_A = 2^-B sum_idx c[idx] prod_{p in A} (2 bit_p(idx) - 1).
void sigma_alphas(const tq_ctx *ctx, float *alpha) {
    const int B = ctx->BK, L = 1 << B;
    const int NP = n_sigma_planes(B);
    for (int sp = 0; sp < NP; ++sp) {
        const uint32_t set = sigma_set(B, sp);
        double a = 0.0;
        for (int idx = 0; idx < L; ++idx) {
            double prod = 1.0;
            for (int p = 0; p < B; ++p)
                if ((set >> p) & 1) prod *= ((idx >> p) & 1) ? 1.0 : -1.0;
            a += (double)ctx->ck[idx] * prod;
        }
        alpha[sp] = (float)(a / L);
    }
}

}  // namespace

void tq_sigma_planes(const tq_ctx *ctx, int *n_planes, uint32_t *sets, float *alpha) {
    *n_planes = n_sigma_planes(ctx->BK);
    for (int i = 0; i < *n_planes; ++i) sets[i] = sigma_set(ctx->BK, i);
    sigma_alphas(ctx, alpha);
}

namespace {
// Direct output: every sequence is covered by exactly one (segment, split)
// holding tokens, so the decode kernel can write out = o / l itself.
bool direct_output(const tq_segment *segs, int n_segs, int batch, const std::vector<SegPlan> &pl) {
    std::vector<int> cover((size_t)batch, 0);
    for (int s = 0; s < n_segs; ++s) {
        if (pl[s].n_splits != 1 || segs[s].n_tokens <= 0) return false;
        for (int b = segs[s].first_seq; b < segs[s].first_seq + segs[s].n_seqs; ++b)
            if (b >= 0 && b < batch) ++cover[(size_t)b];
    }
    for (int b = 0; b < batch; ++b)
        if (cover[(size_t)b] != 1) return false;
    return true;
}
}  // namespace

int tq_decode_launches(const tq_segment *segs, int n_segs, int batch, int Hq, int Hkv, int n_sms) {
    std::vector<SegPlan> pl;
    plan_segments(segs, n_segs, Hq, Hkv, n_sms, pl);
    // one decode launch per (bits, queries per CTA, m, key-row length) group
    std::vector<int> done(n_segs, 0);
    int groups = 0;
    for (int s0 = 0; s0 < n_segs; ++s0) {
        if (done[s0]) continue;
        const tq_ctx *c0 = segs[s0].ctx;
        for (int s = 0; s < n_segs; ++s) {
            const tq_ctx *c = segs[s].ctx;
            if (!done[s] && c->BK == c0->BK && pl[s].qc == pl[s0].qc && c->m == c0->m &&
                tq_row_bytes(c, TQ_KEYS) == tq_row_bytes(c0, TQ_KEYS))
                done[s] = 1;
        }
        ++groups;
    }
    return 1 + groups + (direct_output(segs, n_segs, batch, pl) ? 0 : 1);
}

size_t tq_decode_ws(const tq_segment *segs, int n_segs, int batch, int Hq, int Hkv, int n_sms) {
    (void)batch;
    std::vector<SegPlan> pl;
    plan_segments(segs, n_segs, Hq, Hkv, n_sms, pl);
    size_t q = 0, p = 0;
    for (auto &x : pl) {
        q += x.qprep_floats;
        p += x.part_floats;
    }
    return align256(q * 4) + align256(p * 4);
}

tq_status tq_launch_decode(const tq_segment *segs, int n_segs, const void *q, tq_dtype q_dtype, int batch, int Hq,
                           int Hkv, void *out, tq_dtype out_dtype, void *ws, size_t ws_bytes, cudaStream_t stream,
                           int n_sms, const TqAppend *app) {
    (void)ws_bytes;
    std::vector<SegPlan> pl;
    plan_segments(segs, n_segs, Hq, Hkv, n_sms, pl);
    // large (it is the kernels' parameter block); one per host thread, so
    // calls from different threads do not share it
    thread_local DecodePlan P;
    P = DecodePlan{};
    P.n_segs = n_segs;
    P.Hq = Hq;
    P.Hkv = Hkv;
    P.G = Hq / Hkv;
    P.d = segs[0].ctx->d;
    P.batch = batch;
    P.out = out;
    P.out_dtype = (int)out_dtype;
    P.direct = direct_output(segs, n_segs, batch, pl) ? 1 : 0;
    size_t qtot = 0;
    for (auto &x : pl) qtot += x.qprep_floats;
    P.qprep = static_cast<float *>(ws);
    P.part = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + align256(qtot * 4));
    int64_t qoff = 0, poff = 0;
    for (int s = 0; s < n_segs; ++s) {
        const tq_segment &sg = segs[s];
        const tq_ctx *c = sg.ctx;
        SegDesc &d = P.seg[s];
        const int64_t krow = tq_row_bytes(c, TQ_KEYS), vrow = tq_row_bytes(c, TQ_VALUES);
        d.kc = static_cast<const uint8_t *>(sg.codes.k) + (int64_t)sg.codes_batch * Hkv * sg.codes.capacity * krow;
        d.vc = static_cast<const uint8_t *>(sg.codes.v) + (int64_t)sg.codes_batch * Hkv * sg.codes.capacity * vrow;
        d.signs = c->d_signs;
        d.S = c->d_S;
        d.status = c->d_status;
        d.book = c->d_book;
        d.Q = c->rotation == TQ_ROT_HAAR ? c->d_Q32 : nullptr;
        d.append = app && app->flags[s] ? 1 : 0;
        if (d.append) P.n_append_blocks += Hkv;
        d.capacity = sg.codes.capacity;
        d.T = sg.n_tokens;
        d.part_base = poff / tq_part_floats(P.d);
        d.qprep_base = qoff;
        d.first_seq = sg.first_seq;
        d.n_seqs = sg.n_seqs;
        d.krow = (int)krow;
        d.kf16 = c->norm_f16;
        d.vrow = (int)vrow;
        d.m = c->m;
        d.bk = c->BK;
        d.bv = c->BV;
        d.n_splits = pl[s].n_splits;
        d.split_len = pl[s].split_len;
        d.n_qchunks = pl[s].n_qchunks;
        d.n_planes = n_sigma_planes(c->BK);
        for (int i = 0; i < d.n_planes; ++i) d.plane_sets[i] = sigma_set(c->BK, i);
        sigma_alphas(c, d.alpha);
        for (int i = 0; i < 32; ++i) d.vtab[i] = i < c->LV ? c->cv[i] : 0.f;
        for (int i = 0; i < 16; ++i) d.ktab[i] = i < (1 << c->BK) ? c->ck[i] : 0.f;
        qoff += pl[s].qprep_floats;
        poff += pl[s].part_floats;
    }
    if (app) {
        P.k_new = app->k_new;
        P.v_new = app->v_new;
        P.kv_dtype = (int)app->dtype;
    }
    cudaError_t e = tq_launch_qprep(P, q, q_dtype, stream);
    if (e != cudaSuccess) return tq_check_cuda(e);
    // one launch per (bits, queries per CTA, row format) group: the CTA's
    // shared memory is sized by the group's row lengths.  Lookup-table groups
    // go first: a tensor-core launch after them fills the SMs they leave
    // idle and those that finish first.
    std::vector<int> done(n_segs, 0);
    for (int pass = 0; pass < 2; ++pass)
    for (int s0 = 0; s0 < n_segs; ++s0) {
        if (done[s0] || (pl[s0].qc == TQ_MMA_QUERIES) != (pass == 1)) continue;
        const int bk = P.seg[s0].bk, qc = pl[s0].qc, m = P.seg[s0].m, kr = P.seg[s0].krow;
        auto same = [&](int s) {
            return P.seg[s].bk == bk && pl[s].qc == qc && P.seg[s].m == m && P.seg[s].krow == kr;
        };
        int64_t items = 0;
        for (int s = 0; s < n_segs; ++s) {
            SegDesc &d = P.seg[s];
            if (!done[s] && same(s)) {
                d.item_base = items;
                items += (int64_t)Hkv * d.n_splits * d.n_qchunks;
            } else if (!done[s]) {
                d.item_base = -(int64_t)1 << 62;   // not in this launch
            }
        }
        DecodePlan Pg = P;
        for (int s = 0; s < n_segs; ++s)
            if (done[s]) Pg.seg[s].item_base = -(int64_t)1 << 62;
        for (int s = 0; s < n_segs; ++s)
            if (!done[s] && same(s)) done[s] = 1;
        if (items == 0) continue;
        if (qc == TQ_MMA_QUERIES) {
            e = tq_launch_decode_mma(Pg, items, P.d, m, bk, P.seg[s0].krow, P.seg[s0].vrow, stream);
            if (e != cudaSuccess) return tq_check_cuda(e);
            continue;
        }
        e = P.d == 256   ? launch_decode_dim<256>(bk + 1, qc, Pg, items, P.seg[s0].krow, P.seg[s0].vrow, m, stream)
            : P.d == 128 ? launch_decode_dim<128>(bk + 1, qc, Pg, items, P.seg[s0].krow, P.seg[s0].vrow, m, stream)
                         : launch_decode_dim<64>(bk + 1, qc, Pg, items, P.seg[s0].krow, P.seg[s0].vrow, m, stream);
        if (e != cudaSuccess) return tq_check_cuda(e);
    }
    if (P.direct) return TQ_OK;   // the decode kernel wrote the output
    e = tq_launch_combine(P, out, out_dtype, stream);
    return tq_check_cuda(e);
}
