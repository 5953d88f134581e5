// tq_split.cu -- decode attention over an outlier/normal channel-split cache
// (turboquant-plus-rs README, Modules: outlier -- fractional bits per value
// obtained by coding outlier and normal channels at different widths).
//
// A head's channels are split into an outlier group (channels [0, d_o)) and
// a normal group (channels [d_o, d_o + d_n)); each group is a codec of its
// own, with its own rotation and bit width.  A key's score is the inner
// product over both groups, q.k_hat / sqrt(d_o + d_n) = (sqrt(d_o) s_o +
// sqrt(d_n) s_n) / sqrt(d_o + d_n) with s_g the group's own score (scaled by
// 1/sqrt(d_g)); one softmax covers the token; the output is the concatenation
// of the groups' value reconstructions.
//
// Kernels: the query's groups as fp32 rows; each group's scores with the
// exact scoring kernel (tq_scores_kernel); then one block per (sequence,
// query head, chunk of tokens) combines the scores, takes the chunk's softmax
// terms and accumulates each group's values in its rotated frame from the
// packed codes (512-token tiles of probabilities and of both groups' value
// rows staged in shared memory, the next tile's rows copied with cp.async
// while the current one is accumulated); a last kernel merges the
// chunks by their maxima and sums (log-sum-exp) and rotates each group back.
#include <cmath>

#include "tq_internal.cuh"

tq_status tq_launch_scores(tq_ctx *ctx, const tq_codes *codes, const float *q, int Hq, int64_t T, float *scores,
                           cudaStream_t stream);
tq_status tq_check_cuda(cudaError_t e);

namespace {

constexpr int SPLIT_TILE = 512;    // tokens per pass: per-token weights and both groups' value rows in smem

struct SplitGroup {
    const uint8_t *vc;        // packed value rows [batch][H_kv][capacity][vrow]
    const uint32_t *signs;    // Walsh-Hadamard signs [H_kv][d/32]
    const float *Q;           // Haar rotation [H_kv][d][d], or nullptr
    const float *scores;      // [batch][H_q][T]
    int d, bv, vrow;
    float cv[32];             // value centroids by code
};

struct SplitParams {
    SplitGroup g[2];
    const void *q;            // [batch][H_q][d_o + d_n] in q_dtype
    float *qo, *qn;           // fp32 group rows of q
    void *out;                // [batch][H_q][d_o + d_n] in out_dtype
    int64_t capacity, T;
    int batch, Hq, Hkv;
    int q_dtype, out_dtype;
};

__device__ __forceinline__ float load_any(const void *p, int64_t i, int dt) {
    if (dt == TQ_F32) return static_cast<const float *>(p)[i];
    if (dt == TQ_F16) return __half2float(static_cast<const __half *>(p)[i]);
    return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
}

__device__ __forceinline__ void store_any(void *p, int64_t i, float v, int dt) {
    if (dt == TQ_F32) static_cast<float *>(p)[i] = v;
    else if (dt == TQ_F16) static_cast<__half *>(p)[i] = __float2half_rn(v);
    else static_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(v);
}

// q [batch][H_q][d_o + d_n] -> fp32 rows qo [batch][H_q][d_o], qn [batch][H_q][d_n].
__global__ void tq_split_q_kernel(const __grid_constant__ SplitParams P) {
    const int dt = P.g[0].d + P.g[1].d;
    const int64_t row = blockIdx.x;
    for (int j = threadIdx.x; j < dt; j += blockDim.x) {
        const float v = load_any(P.q, row * dt + j, P.q_dtype);
        if (j < P.g[0].d) P.qo[row * P.g[0].d + j] = v;
        else P.qn[row * P.g[1].d + (j - P.g[0].d)] = v;
    }
}

constexpr int SPLIT_SLICES = 8;      // token slices per coordinate pair in a block
constexpr int SPLIT_TARGET_BLOCKS = 1184;   // 8 blocks per SM of 148

// Tokens per chunk: a multiple of SPLIT_TILE, chosen so that (rows x chunks)
// fills the GPU; every chunk holds at least one token.
int64_t split_chunk_len(int rows, int64_t T) {
    if (rows <= 0 || T <= 0) return SPLIT_TILE;
    const int64_t tiles = (T + SPLIT_TILE - 1) / SPLIT_TILE;
    int64_t want = (SPLIT_TARGET_BLOCKS + rows - 1) / rows;
    want = want > tiles ? tiles : (want < 1 ? 1 : want);
    const int64_t per = (tiles + want - 1) / want;
    return per * SPLIT_TILE;
}

// Both groups' value rows of a tile, [group 0 rows][group 1 rows], copied
// with 4-byte cp.async by all threads (one commit group per tile).
__device__ __forceinline__ void split_stage_tile(const SplitParams &P, int b, int h, int64_t base, int n, uint8_t *dst,
                                                 int ltid, int nthr) {
#pragma unroll
    for (int gg = 0; gg < 2; ++gg) {
        const uint32_t *src = reinterpret_cast<const uint32_t *>(
            P.g[gg].vc + (((int64_t)b * P.Hkv + h) * P.capacity + base) * P.g[gg].vrow);
        const uint32_t d = tqdev::smem_u32(dst + (gg ? SPLIT_TILE * P.g[0].vrow : 0));
        const int words = n * (P.g[gg].vrow / 4);
        for (int i = ltid; i < words; i += nthr)
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d + 4u * (uint32_t)i), "l"(src + i)
                         : "memory");
    }
}

// Partial attention of one chunk of tokens for one (sequence, query head):
// grid (rows, chunks), SPLIT_SLICES * (d_o + d_n) / 2 threads; thread
// (slice, q) accumulates coordinates 2q and 2q + 1 of the concatenated output
// (group 0 first; d_o is even, so both are in one group), in that group's
// rotated frame, over the chunk's tokens i = slice (mod SPLIT_SLICES).
// Writes the chunk's max combined score m, sum of exp(s - m) and the
// unnormalised accumulator sum_i exp(s_i - m) n_s,i c[idx_i,t].
__global__ void __launch_bounds__(1024) tq_split_attend_kernel(const __grid_constant__ SplitParams P,
                                                               int64_t chunk_len, float *part) {
    // value rows of two tiles (double-buffered): [buf][SPLIT_TILE x (vrow_0 + vrow_1) bytes]
    extern __shared__ __align__(16) uint8_t s_rows[];
    __shared__ float s_w[2][SPLIT_TILE];     // exp(s_i - m) n_s,i of this tile, per group
    __shared__ float s_red[32];
    __shared__ float s_acc[SPLIT_SLICES][256];
    __shared__ float s_cv[2][32];
    const int nthr = blockDim.x, ltid = threadIdx.x;
    const int d0 = P.g[0].d, d1 = P.g[1].d, dt = d0 + d1, np = dt / 2;
    const int slice = ltid / np, q = ltid % np;
    const int row = blockIdx.x, b = row / P.Hq, j = row % P.Hq;
    const int h = j / (P.Hq / P.Hkv);
    const int64_t t0 = (int64_t)blockIdx.y * chunk_len;
    const int64_t t1 = min(P.T, t0 + chunk_len);
    const float w0 = sqrtf((float)d0) * rsqrtf((float)dt), w1 = sqrtf((float)d1) * rsqrtf((float)dt);
    const float *s0 = P.g[0].scores + (int64_t)row * P.T;
    const float *s1 = P.g[1].scores + (int64_t)row * P.T;
    if (ltid < 64) s_cv[ltid / 32][ltid % 32] = P.g[ltid / 32].cv[ltid % 32];
    float mx = -INFINITY;
    for (int64_t t = t0 + ltid; t < t1; t += nthr) mx = fmaxf(mx, w0 * s0[t] + w1 * s1[t]);
    for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((ltid & 31) == 0) s_red[ltid >> 5] = mx;
    __syncthreads();
    mx = -INFINITY;
    for (int w = 0; w < nthr / 32; ++w) mx = fmaxf(mx, s_red[w]);
    const int c0 = 2 * q;
    const int g = c0 < d0 ? 0 : 1;
    const int jj = g == 0 ? c0 : c0 - d0;
    const SplitGroup &G = P.g[g];
    const int bit = G.bv * jj, wi = bit / 32, sh = bit % 32;
    const bool straddle = sh + 2 * G.bv > 32;
    const uint32_t fm = (1u << G.bv) - 1u;
    const int vw = G.vrow / 4;
    float acc0 = 0.f, acc1 = 0.f, lsum = 0.f;
    // tile k's rows land while tile k - 1 is accumulated
    const int buf_bytes = SPLIT_TILE * (P.g[0].vrow + P.g[1].vrow);
    const int goff = g ? SPLIT_TILE * P.g[0].vrow : 0;
    split_stage_tile(P, b, h, t0, (int)min((int64_t)SPLIT_TILE, t1 - t0), s_rows, ltid, nthr);
    asm volatile("cp.async.commit_group;" ::: "memory");
    int k = 0;
    for (int64_t base = t0; base < t1; base += SPLIT_TILE, ++k) {
        const int n = (int)min((int64_t)SPLIT_TILE, t1 - base);
        const int buf = k & 1;
        // the other buffer was last read in iteration k - 1, which ended with a barrier
        if (base + SPLIT_TILE < t1)
            split_stage_tile(P, b, h, base + SPLIT_TILE, (int)min((int64_t)SPLIT_TILE, t1 - base - SPLIT_TILE),
                             s_rows + (buf ^ 1) * buf_bytes, ltid, nthr);
        asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_group 1;" ::: "memory");   // this tile's copies (not the next's)
        __syncthreads();
        // per-token weights of both groups: exp(s_i - m) n_s,i
        for (int e = ltid; e < 2 * n; e += nthr) {
            const int gg = e >= n ? 1 : 0, i = e - gg * n;
            const float p = __expf(w0 * s0[base + i] + w1 * s1[base + i] - mx);
            if (gg == 0) lsum += p;
            const uint32_t *r = reinterpret_cast<const uint32_t *>(s_rows + buf * buf_bytes +
                                                                   (gg ? SPLIT_TILE * P.g[0].vrow : 0)) +
                                i * (P.g[gg].vrow / 4);
            s_w[gg][i] = p * __uint_as_float(r[P.g[gg].bv * P.g[gg].d / 32]);
        }
        __syncthreads();
        const uint32_t *sv = reinterpret_cast<const uint32_t *>(s_rows + buf * buf_bytes + goff);
        const float *sw = s_w[g];
#pragma unroll 4
        for (int i = slice; i < n; i += SPLIT_SLICES) {
            const uint32_t *vr = sv + i * vw;
            uint32_t raw = vr[wi] >> sh;
            if (straddle) raw |= vr[wi + 1] << (32 - sh);
            const float w = sw[i];
            acc0 = fmaf(w, s_cv[g][raw & fm], acc0);
            acc1 = fmaf(w, s_cv[g][(raw >> G.bv) & fm], acc1);
        }
        __syncthreads();
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    for (int o = 16; o >= 1; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
    if ((ltid & 31) == 0) s_red[ltid >> 5] = lsum;
    s_acc[slice][c0] = acc0;
    s_acc[slice][c0 + 1] = acc1;
    __syncthreads();
    float *dst = part + ((int64_t)blockIdx.y * gridDim.x + row) * (dt + 2);
    for (int c = ltid; c < dt; c += nthr) {
        float a2 = 0.f;
#pragma unroll
        for (int sl = 0; sl < SPLIT_SLICES; ++sl) a2 += s_acc[sl][c];
        dst[2 + c] = a2;
    }
    if (ltid == 0) {
        float l = 0.f;
        for (int w = 0; w < nthr / 32; ++w) l += s_red[w];
        dst[0] = mx;
        dst[1] = l;
    }
}

// Combines the chunks of one (sequence, query head) by their maxima and sums
// and rotates each group back: v = Pi^T (acc / sqrt(d_g)); d_o + d_n threads.
__global__ void __launch_bounds__(256) tq_split_combine_kernel(const __grid_constant__ SplitParams P, int chunks,
                                                               const float *part) {
    __shared__ float s_a[256];
    const int d0 = P.g[0].d, d1 = P.g[1].d, dt = d0 + d1;
    const int tid = threadIdx.x, row = blockIdx.x, rows = gridDim.x;
    const int h = (row % P.Hq) / (P.Hq / P.Hkv);
    float M = -INFINITY;
    for (int c = 0; c < chunks; ++c) M = fmaxf(M, part[((int64_t)c * rows + row) * (dt + 2)]);
    float L = 0.f, a = 0.f;
    for (int c = 0; c < chunks; ++c) {
        const float *pc = part + ((int64_t)c * rows + row) * (dt + 2);
        const float e = __expf(pc[0] - M);
        L = fmaf(pc[1], e, L);
        a = fmaf(pc[2 + tid], e, a);
    }
    s_a[tid] = a / L;
    __syncthreads();
    const int g = tid < d0 ? 0 : 1;
    const int jj = g == 0 ? tid : tid - d0;
    const SplitGroup &G = P.g[g];
    const float isd = rsqrtf((float)G.d);
    const float *av = s_a + (g == 0 ? 0 : d0);
    float v = 0.f;
    if (G.Q) {
        const float *Qh = G.Q + (int64_t)h * G.d * G.d;
        for (int r = 0; r < G.d; ++r) v = fmaf(Qh[r * G.d + jj], av[r], v);
        v *= isd;
    } else {
        // (H a)_jj = sum_r (-1)^popcount(r & jj) a_r; Pi^T = D H / sqrt(d)
        for (int r = 0; r < G.d; ++r) v += (__popc(r & jj) & 1) ? -av[r] : av[r];
        v *= isd * isd;
        if ((G.signs[(int64_t)h * (G.d / 32) + jj / 32] >> (jj % 32)) & 1) v = -v;
    }
    store_any(P.out, (int64_t)row * dt + tid, v, P.out_dtype);
}

}  // namespace

size_t tq_split_ws(int batch, int Hq, int d_o, int d_n, int64_t T) {
    const int rows = batch * Hq;
    const int64_t L = split_chunk_len(rows, T), chunks = (T + L - 1) / L;
    const size_t q = (size_t)rows * (d_o + d_n) * 4;
    const size_t s = 2 * (size_t)rows * (size_t)T * 4;
    const size_t pt = (size_t)chunks * rows * (d_o + d_n + 2) * 4;
    return ((q + 255) & ~size_t(255)) + ((s + 255) & ~size_t(255)) + ((pt + 255) & ~size_t(255));
}

tq_status tq_launch_split(tq_ctx *co, const tq_codes *ko, tq_ctx *cn, const tq_codes *kn, int64_t T, const void *q,
                          tq_dtype q_dtype, int batch, int Hq, void *out, tq_dtype out_dtype, void *ws,
                          cudaStream_t stream) {
    SplitParams P{};
    const int d0 = co->d, d1 = cn->d;
    P.qo = static_cast<float *>(ws);
    P.qn = P.qo + (size_t)batch * Hq * d0;
    float *sc = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) +
                                          (((size_t)batch * Hq * (d0 + d1) * 4 + 255) & ~size_t(255)));
    const tq_ctx *cx[2] = {co, cn};
    const tq_codes *cd[2] = {ko, kn};
    for (int g = 0; g < 2; ++g) {
        SplitGroup &G = P.g[g];
        G.vc = static_cast<const uint8_t *>(cd[g]->v);
        G.signs = cx[g]->d_signs;
        G.Q = cx[g]->rotation == TQ_ROT_HAAR ? cx[g]->d_Q32 : nullptr;
        G.scores = sc + (size_t)g * batch * Hq * T;
        G.d = cx[g]->d;
        G.bv = cx[g]->BV;
        G.vrow = (int)tq_row_bytes(cx[g], TQ_VALUES);
        for (int i = 0; i < 32; ++i) G.cv[i] = i < cx[g]->LV ? cx[g]->cv[i] : 0.f;
    }
    P.q = q;
    P.out = out;
    P.capacity = ko->capacity;
    P.T = T;
    P.batch = batch;
    P.Hq = Hq;
    P.Hkv = ko->n_kv_heads;
    P.q_dtype = (int)q_dtype;
    P.out_dtype = (int)out_dtype;
    const unsigned rows = (unsigned)(batch * Hq);
    tq_split_q_kernel<<<rows, 128, 0, stream>>>(P);
    tq_status st = tq_check_cuda(cudaGetLastError());
    if (st != TQ_OK) return st;
    if ((st = tq_launch_scores(co, ko, P.qo, Hq, T, const_cast<float *>(P.g[0].scores), stream)) != TQ_OK) return st;
    if ((st = tq_launch_scores(cn, kn, P.qn, Hq, T, const_cast<float *>(P.g[1].scores), stream)) != TQ_OK) return st;
    const int64_t L = split_chunk_len((int)rows, T), chunks = (T + L - 1) / L;
    float *part = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(sc) +
                                            ((2 * (size_t)rows * (size_t)T * 4 + 255) & ~size_t(255)));
    const size_t rows_smem = 2 * (size_t)SPLIT_TILE * (P.g[0].vrow + P.g[1].vrow);
    if ((st = tq_check_cuda(cudaFuncSetAttribute(tq_split_attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)rows_smem))) != TQ_OK)
        return st;
    tq_split_attend_kernel<<<dim3(rows, (unsigned)chunks), SPLIT_SLICES * (d0 + d1) / 2, rows_smem, stream>>>(P, L,
                                                                                                        part);
    if ((st = tq_check_cuda(cudaGetLastError())) != TQ_OK) return st;
    tq_split_combine_kernel<<<rows, d0 + d1, 0, stream>>>(P, (int)chunks, part);
    return tq_check_cuda(cudaGetLastError());
}
