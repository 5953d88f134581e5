// tq_api.cu -- the C ABI of libtq: argument validation, context lifetime,
// table upload and kernel dispatch.  No computation on the data path
// happens on the host; every step runs in the kernels of tq_encode.cu,
// tq_decode.cu and tq_aux.cu.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <vector>

#include "tq_decode.cuh"

extern "C" void tq_host_head_tables(int d, int m, uint64_t seed, int h, uint32_t *sign_words,
                                    uint16_t *S_bits);
extern "C" int tq_host_codebook(int B, float *c, float *beta);
extern "C" void tq_host_haar(int d, int m, uint64_t seed, int h, double *Q);

tq_status tq_launch_encode(tq_ctx *ctx, const void *k, const void *v, tq_dtype dtype, int batch, int H,
                           int64_t T, int64_t sb, int64_t sh, int64_t st, const tq_codes *codes,
                           int64_t token_offset, cudaStream_t stream, int n_sms);
tq_status tq_launch_scores(tq_ctx *ctx, const tq_codes *codes, const float *q, int Hq, int64_t T,
                           float *scores, cudaStream_t stream);
tq_status tq_launch_dequant(tq_ctx *ctx, const tq_codes *codes, int64_t T, float *k_hat, float *v_hat,
                            cudaStream_t stream);
size_t tq_decode_ws(const tq_segment *segs, int n_segs, int batch, int Hq, int Hkv, int n_sms);
int tq_decode_launches(const tq_segment *segs, int n_segs, int batch, int Hq, int Hkv, int n_sms);
size_t tq_split_ws(int batch, int Hq, int d_o, int d_n, int64_t T);
tq_status tq_launch_split(tq_ctx *co, const tq_codes *ko, tq_ctx *cn, const tq_codes *kn, int64_t T, const void *q,
                          tq_dtype q_dtype, int batch, int Hq, void *out, tq_dtype out_dtype, void *ws,
                          cudaStream_t stream);
tq_status tq_launch_decode(const tq_segment *segs, int n_segs, const void *q, tq_dtype q_dtype, int batch,
                           int Hq, int Hkv, void *out, tq_dtype out_dtype, void *ws, size_t ws_bytes,
                           cudaStream_t stream, int n_sms, const TqAppend *app = nullptr);

static thread_local char g_cuda_msg[256] = "no error";

tq_status tq_check_cuda(cudaError_t e) {
    if (e == cudaSuccess) return TQ_OK;
    snprintf(g_cuda_msg, sizeof(g_cuda_msg), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
    return TQ_ERR_CUDA;
}

static int device_sms(int dev) {
    static std::atomic<int> cached[64];   // zero-initialized; concurrent fills store the same value
    if (dev < 0 || dev >= 64) return 148;
    int v = cached[dev].load(std::memory_order_relaxed);
    if (!v) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        v = n > 0 ? n : 148;
        cached[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

tq_status tq_check_device(const tq_ctx *ctx) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ERR_CUDA;
    if (ctx && dev != ctx->device) return TQ_ERR_DEVICE;
    return TQ_OK;
}

typedef CUresult (*PFN_encodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                    const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                    CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                    CUtensorMapFloatOOBfill);

static PFN_encodeTiled get_encode_tiled() {
    // looked up once, thread-safely (function-local static initialization)
    static const PFN_encodeTiled fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_encodeTiled>(p);
        return static_cast<PFN_encodeTiled>(nullptr);
    }();
    return fn;
}

// 4-D TMA map over caller rows of a 16-bit type, element (b, h, t, j) at
// base + b sb + h sh + t st + j (strides in elements): dims {d, T, H, batch},
// box 64 x 128 tokens x 1 x 1, 128-byte swizzle, zero fill past T.  False if
// the driver rejects the layout (the caller then uses another kernel).
bool tq_rows_map_4d(CUtensorMap *map, bool bf16, const void *base, int d, int64_t T, int H, int batch, int64_t sb,
                    int64_t sh, int64_t st) {
    PFN_encodeTiled enc = get_encode_tiled();
    if (!enc || T <= 0 || T > 0xFFFFFFFFll) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)T, (cuuint64_t)H, (cuuint64_t)batch};
    cuuint64_t strides[3] = {(cuuint64_t)st * 2, (cuuint64_t)sh * 2, (cuuint64_t)sb * 2};
    for (int i = 0; i < 3; ++i)
        if (strides[i] == 0 || strides[i] % 16 || strides[i] >= (1ull << 40)) return false;
    cuuint32_t box[4] = {64, 128, 1, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4,
                     const_cast<void *>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

extern "C" {

const char *tq_status_string(tq_status s) {
    switch (s) {
        case TQ_OK: return "TQ_OK";
        case TQ_ERR_NULL: return "TQ_ERR_NULL";
        case TQ_ERR_ZERO_DIM: return "TQ_ERR_ZERO_DIM";
        case TQ_ERR_DIM: return "TQ_ERR_DIM";
        case TQ_ERR_BITS: return "TQ_ERR_BITS";
        case TQ_ERR_ZERO_PROJ: return "TQ_ERR_ZERO_PROJ";
        case TQ_ERR_PROJ: return "TQ_ERR_PROJ";
        case TQ_ERR_EMPTY: return "TQ_ERR_EMPTY";
        case TQ_ERR_DIM_MISMATCH: return "TQ_ERR_DIM_MISMATCH";
        case TQ_ERR_WORKSPACE: return "TQ_ERR_WORKSPACE";
        case TQ_ERR_ALIGN: return "TQ_ERR_ALIGN";
        case TQ_ERR_CUDA: return "TQ_ERR_CUDA";
        case TQ_ERR_DEVICE: return "TQ_ERR_DEVICE";
        case TQ_ERR_LIMIT: return "TQ_ERR_LIMIT";
    }
    return "TQ_ERR_UNKNOWN";
}

const char *tq_last_cuda_error(void) { return g_cuda_msg; }

tq_status tq_create(int head_dim, int bits, int projections, uint64_t seed, tq_ctx **out) {
    return tq_create_ex(head_dim, bits, projections, seed, TQ_ROT_HADAMARD, out);
}

tq_status tq_create_ex(int head_dim, int bits, int projections, uint64_t seed, tq_rotation rotation,
                       tq_ctx **out) {
    return tq_create_format(head_dim, bits, projections, seed, rotation, TQ_NORMS_F32, out);
}

tq_status tq_create_format(int head_dim, int bits, int projections, uint64_t seed, tq_rotation rotation,
                           tq_norm_format key_norms, tq_ctx **out) {
    if (!out) return TQ_ERR_NULL;
    if ((rotation != TQ_ROT_HADAMARD && rotation != TQ_ROT_HAAR) ||
        (key_norms != TQ_NORMS_F32 && key_norms != TQ_NORMS_F16)) {
        *out = nullptr;
        return TQ_ERR_DIM;
    }
    *out = nullptr;
    if (head_dim == 0) return TQ_ERR_ZERO_DIM;
    if (head_dim != 64 && head_dim != 128 && head_dim != 256) return TQ_ERR_DIM;
    // d = 256: the Haar operands (2 x d x d binary16) do not fit in shared memory
    if (head_dim == 256 && rotation == TQ_ROT_HAAR) return TQ_ERR_DIM;
    if (bits < 2 || bits > 5) return TQ_ERR_BITS;
    if (projections == 0) return TQ_ERR_ZERO_PROJ;
    if (projections < 32 || projections > 256 || projections % 32) return TQ_ERR_PROJ;
    // d = 256: the key encoder's S tile and residual operand take
    // (d/64) (128 m + 32 K) bytes of shared memory, within 227 KB for m <= 192
    if (head_dim == 256 && projections > 192) return TQ_ERR_PROJ;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ERR_CUDA;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return TQ_ERR_CUDA;
    if (prop.major != 10 || prop.minor != 0) return TQ_ERR_DEVICE;
    tq_ctx *c = new tq_ctx();
    std::memset(c, 0, sizeof(*c));
    c->d = head_dim;
    c->bits = bits;
    c->m = projections;
    c->BK = bits - 1;
    c->BV = bits;
    c->seed = seed;
    c->device = dev;
    c->rotation = (int)rotation;
    c->norm_f16 = key_norms == TQ_NORMS_F16 ? 1 : 0;
    c->LK = tq_host_codebook(c->BK, c->ck, c->bk);
    c->LV = tq_host_codebook(c->BV, c->cv, c->bv);
    TqBook book;
    std::memset(&book, 0, sizeof(book));
    for (int i = 0; i < c->LK / 2; ++i) book.kmag[i] = c->ck[c->LK / 2 + i];
    for (int i = 0; i + 1 < c->LK / 2; ++i) book.kpb[i] = c->bk[c->LK / 2 + i];
    for (int i = 0; i < c->LV / 2; ++i) book.vmag[i] = c->cv[c->LV / 2 + i];
    for (int i = 0; i + 1 < c->LV / 2; ++i) book.vpb[i] = c->bv[c->LV / 2 + i];
    tq_status st = tq_check_cuda(cudaMalloc(&c->d_status, 2 * sizeof(unsigned long long)));
    if (st == TQ_OK) st = tq_check_cuda(cudaMemset(c->d_status, 0, 2 * sizeof(unsigned long long)));
    if (st == TQ_OK) st = tq_check_cuda(cudaMalloc(&c->d_book, sizeof(TqBook)));
    if (st == TQ_OK) st = tq_check_cuda(cudaMemcpy(c->d_book, &book, sizeof(TqBook), cudaMemcpyHostToDevice));
    if (st != TQ_OK) {
        tq_destroy(c);
        return st;
    }
    *out = c;
    return TQ_OK;
}

void tq_destroy(tq_ctx *ctx) {
    if (!ctx) return;
    cudaDeviceSynchronize();
    cudaFree(ctx->d_signs);
    cudaFree(ctx->d_S);
    cudaFree(ctx->d_status);
    cudaFree(ctx->d_book);
    cudaFree(ctx->d_Q32);
    cudaFree(ctx->d_Qh);
    cudaFree(ctx->d_Qbf);
    cudaFree(ctx->d_HD16);
    cudaFree(ctx->d_HDbf);
    delete ctx;
}

// 2-D TMA map over [rows][d] 16-bit entries: box 64 x box_rows, 128-byte swizzle.
static tq_status encode_rows_map(CUtensorMap *map, CUtensorMapDataType dt, void *base, int d, int64_t rows,
                                 int box_rows) {
    PFN_encodeTiled enc = get_encode_tiled();
    if (!enc) return TQ_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = enc(map, dt, 2, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(g_cuda_msg, sizeof(g_cuda_msg), "cuTensorMapEncodeTiled failed: %d", (int)r);
        return TQ_ERR_CUDA;
    }
    return TQ_OK;
}

tq_status tq_ensure_heads(tq_ctx *ctx, int n_heads) {
    if (!ctx) return TQ_ERR_NULL;
    if (n_heads <= 0) return TQ_ERR_EMPTY;
    if (n_heads > TQ_MAX_HEADS) return TQ_ERR_LIMIT;
    if (n_heads <= ctx->heads_built) return TQ_OK;
    tq_status st = tq_check_device(ctx);
    if (st != TQ_OK) return st;
    const int d = ctx->d, m = ctx->m;
    std::vector<uint32_t> signs((size_t)n_heads * (d / 32));
    std::vector<uint16_t> S((size_t)n_heads * m * d);
    for (int h = 0; h < n_heads; ++h)
        tq_host_head_tables(d, m, ctx->seed, h, &signs[(size_t)h * (d / 32)], &S[(size_t)h * m * d]);
    uint32_t *nsig = nullptr;
    __half *nS = nullptr;
    st = tq_check_cuda(cudaMalloc(&nsig, signs.size() * 4));
    if (st == TQ_OK) st = tq_check_cuda(cudaMalloc(&nS, S.size() * 2));
    if (st == TQ_OK) st = tq_check_cuda(cudaMemcpy(nsig, signs.data(), signs.size() * 4, cudaMemcpyHostToDevice));
    if (st == TQ_OK) st = tq_check_cuda(cudaMemcpy(nS, S.data(), S.size() * 2, cudaMemcpyHostToDevice));
    CUtensorMap map;
    if (st == TQ_OK) {
        PFN_encodeTiled enc = get_encode_tiled();
        if (!enc) st = TQ_ERR_CUDA;
        else {
            cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)n_heads * m};
            cuuint64_t strides[1] = {(cuuint64_t)d * 2};
            cuuint32_t box[2] = {64, (cuuint32_t)m};
            cuuint32_t es[2] = {1, 1};
            CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, nS, dims, strides, box, es,
                             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
            if (r != CUDA_SUCCESS) {
                snprintf(g_cuda_msg, sizeof(g_cuda_msg), "cuTensorMapEncodeTiled failed: %d", (int)r);
                st = TQ_ERR_CUDA;
            }
        }
    }
    float *nQ32 = nullptr;
    __half *nQh = nullptr;
    uint16_t *nQbf = nullptr;
    CUtensorMap qmap, qbfmap;
    std::memset(&qmap, 0, sizeof(qmap));
    std::memset(&qbfmap, 0, sizeof(qbfmap));
    if (st == TQ_OK && ctx->rotation == TQ_ROT_HAAR) {
        const size_t dd = (size_t)d * d;
        std::vector<double> Q(dd);
        std::vector<float> q32((size_t)n_heads * dd);
        std::vector<__half> qh((size_t)n_heads * 2 * dd);
        const double sd = std::sqrt((double)d);
        for (int h = 0; h < n_heads; ++h) {
            tq_host_haar(d, m, ctx->seed, h, Q.data());
            for (size_t i = 0; i < dd; ++i) {
                q32[(size_t)h * dd + i] = (float)Q[i];
                const double v = sd * Q[i];
                const __half hi = __double2half(v);
                qh[(size_t)h * 2 * dd + i] = hi;
                qh[(size_t)h * 2 * dd + dd + i] = __double2half(v - (double)__half2float(hi));
            }
        }
        st = tq_check_cuda(cudaMalloc(&nQ32, q32.size() * 4));
        if (st == TQ_OK) st = tq_check_cuda(cudaMalloc(&nQh, qh.size() * 2));
        if (st == TQ_OK) st = tq_check_cuda(cudaMemcpy(nQ32, q32.data(), q32.size() * 4, cudaMemcpyHostToDevice));
        if (st == TQ_OK) st = tq_check_cuda(cudaMemcpy(nQh, qh.data(), qh.size() * 2, cudaMemcpyHostToDevice));
        // bfloat16 hi + mid + lo of sqrt(d) Q for the TMA-fed value encoder
        // (bfloat16 rows need a bfloat16 operand; three pieces keep 24 bits)
        if (st == TQ_OK && d <= 128) {
            auto bf16_bits = [](double v) -> uint16_t {
                const float f = (float)v;
                uint32_t u;
                std::memcpy(&u, &f, 4);
                u += 0x7FFFu + ((u >> 16) & 1u);   // round to nearest even
                return (uint16_t)(u >> 16);
            };
            auto bf16_val = [](uint16_t b) -> double {
                const uint32_t u = (uint32_t)b << 16;
                float f;
                std::memcpy(&f, &u, 4);
                return (double)f;
            };
            std::vector<uint16_t> qb((size_t)n_heads * 3 * dd);
            for (int h = 0; h < n_heads; ++h) {
                tq_host_haar(d, m, ctx->seed, h, Q.data());
                for (size_t i = 0; i < dd; ++i) {
                    double r = sd * Q[i];
                    for (int piece = 0; piece < 3; ++piece) {
                        const uint16_t b = bf16_bits(r);
                        qb[((size_t)h * 3 + piece) * dd + i] = b;
                        r -= bf16_val(b);
                    }
                }
            }
            st = tq_check_cuda(cudaMalloc(&nQbf, qb.size() * 2));
            if (st == TQ_OK) st = tq_check_cuda(cudaMemcpy(nQbf, qb.data(), qb.size() * 2, cudaMemcpyHostToDevice));
            if (st == TQ_OK) st = encode_rows_map(&qbfmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, nQbf, d, (int64_t)n_heads * 3 * d, d);
        }
        if (st == TQ_OK) {
            PFN_encodeTiled enc = get_encode_tiled();
            cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)n_heads * 2 * d};
            cuuint64_t strides[1] = {(cuuint64_t)d * 2};
            cuuint32_t box[2] = {64, (cuuint32_t)d};
            cuuint32_t es[2] = {1, 1};
            CUresult r = enc ? enc(&qmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, nQh, dims, strides, box, es,
                                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                   CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE)
                             : CUDA_ERROR_NOT_FOUND;
            if (r != CUDA_SUCCESS) {
                snprintf(g_cuda_msg, sizeof(g_cuda_msg), "cuTensorMapEncodeTiled failed: %d", (int)r);
                st = TQ_ERR_CUDA;
            }
        }
    }
    // The Walsh-Hadamard rotation with the head's signs as a +-1 matrix,
    // B[n][k] = (-1)^popcount(n & k) D[k], in both 16-bit types.
    uint16_t *nHD16 = nullptr, *nHDbf = nullptr;
    CUtensorMap hdmap16, hdmapbf;
    std::memset(&hdmap16, 0, sizeof(hdmap16));
    std::memset(&hdmapbf, 0, sizeof(hdmapbf));
    if (st == TQ_OK && ctx->rotation == TQ_ROT_HADAMARD && d <= 128) {   // the TMA-fed encoders' d
        const size_t dd = (size_t)d * d;
        std::vector<uint16_t> h16((size_t)n_heads * dd), hbf((size_t)n_heads * dd);
        for (int h = 0; h < n_heads; ++h)
            for (int n = 0; n < d; ++n)
                for (int k = 0; k < d; ++k) {
                    const bool neg = (__builtin_popcount((unsigned)(n & k)) & 1) ^ ((signs[(size_t)h * (d / 32) + k / 32] >> (k % 32)) & 1);
                    h16[(size_t)h * dd + (size_t)n * d + k] = neg ? 0xBC00u : 0x3C00u;   // binary16 -1 / +1
                    hbf[(size_t)h * dd + (size_t)n * d + k] = neg ? 0xBF80u : 0x3F80u;   // bfloat16 -1 / +1
                }
        st = tq_check_cuda(cudaMalloc(&nHD16, h16.size() * 2));
        if (st == TQ_OK) st = tq_check_cuda(cudaMalloc(&nHDbf, hbf.size() * 2));
        if (st == TQ_OK) st = tq_check_cuda(cudaMemcpy(nHD16, h16.data(), h16.size() * 2, cudaMemcpyHostToDevice));
        if (st == TQ_OK) st = tq_check_cuda(cudaMemcpy(nHDbf, hbf.data(), hbf.size() * 2, cudaMemcpyHostToDevice));
        if (st == TQ_OK) st = encode_rows_map(&hdmap16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, nHD16, d, (int64_t)n_heads * d, d);
        if (st == TQ_OK) st = encode_rows_map(&hdmapbf, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, nHDbf, d, (int64_t)n_heads * d, d);
    }
    if (st != TQ_OK) {
        cudaFree(nsig);
        cudaFree(nS);
        cudaFree(nQ32);
        cudaFree(nQh);
        cudaFree(nQbf);
        cudaFree(nHD16);
        cudaFree(nHDbf);
        return st;
    }
    cudaDeviceSynchronize();   // no kernel may still read the old tables
    cudaFree(ctx->d_signs);
    cudaFree(ctx->d_S);
    cudaFree(ctx->d_Q32);
    cudaFree(ctx->d_Qh);
    cudaFree(ctx->d_Qbf);
    cudaFree(ctx->d_HD16);
    cudaFree(ctx->d_HDbf);
    ctx->d_signs = nsig;
    ctx->d_S = nS;
    ctx->tmap_S = map;
    ctx->d_Q32 = nQ32;
    ctx->d_Qh = nQh;
    ctx->tmap_Q = qmap;
    ctx->d_Qbf = nQbf;
    ctx->tmap_Qbf = qbfmap;
    ctx->d_HD16 = nHD16;
    ctx->d_HDbf = nHDbf;
    ctx->tmap_HD16 = hdmap16;
    ctx->tmap_HDbf = hdmapbf;
    ctx->heads_built = n_heads;
    return TQ_OK;
}

int64_t tq_row_bytes(const tq_ctx *ctx, tq_which which) {
    if (!ctx) return 0;
    const int64_t kb = (int64_t)ctx->BK * ctx->d / 8 + ctx->m / 8 + (ctx->norm_f16 ? 4 : 8);
    const int64_t vb = (int64_t)ctx->BV * ctx->d / 8 + 4;
    return which == TQ_KEYS ? kb : which == TQ_VALUES ? vb : kb + vb;
}

size_t tq_packed_bytes(const tq_ctx *ctx, int batch, int n_kv_heads, int64_t capacity, tq_which which) {
    if (!ctx || batch < 0 || n_kv_heads < 0 || capacity < 0) return 0;
    return (size_t)batch * n_kv_heads * capacity * tq_row_bytes(ctx, which);
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

static tq_status check_codes(const tq_ctx *ctx, const tq_codes *codes, bool need_k, bool need_v) {
    if (!codes) return TQ_ERR_NULL;
    if ((need_k && !codes->k) || (need_v && !codes->v)) return TQ_ERR_NULL;
    if (codes->batch <= 0 || codes->n_kv_heads <= 0) return TQ_ERR_EMPTY;
    if (codes->capacity < 0 || codes->capacity % 16) return TQ_ERR_DIM_MISMATCH;
    if ((need_k && !aligned16(codes->k)) || (need_v && !aligned16(codes->v))) return TQ_ERR_ALIGN;
    (void)ctx;
    return TQ_OK;
}

tq_status tq_encode_kv(tq_ctx *ctx, const void *k, const void *v, tq_dtype dtype, int batch, int n_kv_heads,
                       int64_t n_tokens, int64_t stride_b, int64_t stride_h, int64_t stride_t,
                       const tq_codes *codes, int64_t token_offset, void *stream) {
    if (!ctx || !codes) return TQ_ERR_NULL;
    if (batch <= 0 || n_kv_heads <= 0) return TQ_ERR_EMPTY;
    if (n_tokens == 0 && token_offset >= 0 && token_offset <= codes->capacity) return TQ_OK;   // nothing to encode
    if (!k && !v) return TQ_ERR_NULL;
    if (dtype != TQ_F32 && dtype != TQ_F16 && dtype != TQ_BF16) return TQ_ERR_DIM_MISMATCH;
    tq_status st = check_codes(ctx, codes, k != nullptr, v != nullptr);
    if (st != TQ_OK) return st;
    if (codes->batch != batch || codes->n_kv_heads != n_kv_heads) return TQ_ERR_DIM_MISMATCH;
    if (n_tokens < 0 || token_offset < 0 || token_offset + n_tokens > codes->capacity) return TQ_ERR_DIM_MISMATCH;
    const int64_t es = dtype == TQ_F32 ? 4 : 2;
    if (stride_t < ctx->d || stride_b < 0 || stride_h < 0) return TQ_ERR_DIM_MISMATCH;
    if ((stride_b * es) % 16 || (stride_h * es) % 16 || (stride_t * es) % 16) return TQ_ERR_ALIGN;
    if ((k && !aligned16(k)) || (v && !aligned16(v))) return TQ_ERR_ALIGN;
    if ((st = tq_check_device(ctx)) != TQ_OK) return st;
    if ((st = tq_ensure_heads(ctx, n_kv_heads)) != TQ_OK) return st;
    if (n_tokens == 0) return TQ_OK;
    return tq_launch_encode(ctx, k, v, dtype, batch, n_kv_heads, n_tokens, stride_b, stride_h, stride_t, codes,
                            token_offset, static_cast<cudaStream_t>(stream), device_sms(ctx->device));
}

tq_status tq_attention_scores(tq_ctx *ctx, const tq_codes *codes, const float *q, int n_q_heads, int64_t n_tokens,
                              float *scores, void *stream) {
    if (!ctx || !q || !scores) return TQ_ERR_NULL;
    tq_status st = check_codes(ctx, codes, true, false);
    if (st != TQ_OK) return st;
    if (n_q_heads <= 0) return TQ_ERR_EMPTY;
    if (n_q_heads % codes->n_kv_heads) return TQ_ERR_DIM_MISMATCH;
    if (n_tokens < 0 || n_tokens > codes->capacity) return TQ_ERR_DIM_MISMATCH;
    if ((st = tq_check_device(ctx)) != TQ_OK) return st;
    if ((st = tq_ensure_heads(ctx, codes->n_kv_heads)) != TQ_OK) return st;
    if (n_tokens == 0) return TQ_OK;
    return tq_launch_scores(ctx, codes, q, n_q_heads, n_tokens, scores, static_cast<cudaStream_t>(stream));
}

tq_status tq_dequantize(tq_ctx *ctx, const tq_codes *codes, int64_t n_tokens, float *k_hat, float *v_hat,
                        void *stream) {
    if (!ctx) return TQ_ERR_NULL;
    if (!k_hat && !v_hat) return TQ_ERR_NULL;
    tq_status st = check_codes(ctx, codes, k_hat != nullptr, v_hat != nullptr);
    if (st != TQ_OK) return st;
    if (n_tokens < 0 || n_tokens > codes->capacity) return TQ_ERR_DIM_MISMATCH;
    if ((st = tq_check_device(ctx)) != TQ_OK) return st;
    if ((st = tq_ensure_heads(ctx, codes->n_kv_heads)) != TQ_OK) return st;
    if (n_tokens == 0) return TQ_OK;
    return tq_launch_dequant(ctx, codes, n_tokens, k_hat, v_hat, static_cast<cudaStream_t>(stream));
}

static tq_status check_segments(const tq_segment *segs, int n_segs, int batch, int Hq, int Hkv) {
    if (!segs) return TQ_ERR_NULL;
    if (n_segs <= 0 || batch <= 0 || Hq <= 0 || Hkv <= 0) return TQ_ERR_EMPTY;
    if (n_segs > TQ_MAX_SEGMENTS) return TQ_ERR_LIMIT;
    if (Hq % Hkv) return TQ_ERR_DIM_MISMATCH;
    std::vector<int> covered(batch, 0);
    const int d = segs[0].ctx ? segs[0].ctx->d : 0;
    for (int s = 0; s < n_segs; ++s) {
        const tq_segment &g = segs[s];
        if (!g.ctx) return TQ_ERR_NULL;
        if (g.ctx->d != d) return TQ_ERR_DIM_MISMATCH;
        tq_status st = check_codes(g.ctx, &g.codes, true, true);
        if (st != TQ_OK) return st;
        if (g.codes.n_kv_heads != Hkv) return TQ_ERR_DIM_MISMATCH;
        if (g.codes_batch < 0 || g.codes_batch >= g.codes.batch) return TQ_ERR_DIM_MISMATCH;
        if (g.n_tokens < 0 || g.n_tokens > g.codes.capacity) return TQ_ERR_DIM_MISMATCH;
        if (g.n_seqs <= 0 || g.first_seq < 0 || g.first_seq + g.n_seqs > batch) return TQ_ERR_DIM_MISMATCH;
        for (int b = g.first_seq; b < g.first_seq + g.n_seqs; ++b) covered[b] = 1;
    }
    for (int b = 0; b < batch; ++b)
        if (!covered[b]) return TQ_ERR_DIM_MISMATCH;
    return TQ_OK;
}

size_t tq_decode_workspace_bytes(const tq_segment *segs, int n_segs, int batch, int n_q_heads, int n_kv_heads) {
    if (check_segments(segs, n_segs, batch, n_q_heads, n_kv_heads) != TQ_OK) return 0;
    int dev = 0;
    cudaGetDevice(&dev);
    return tq_decode_ws(segs, n_segs, batch, n_q_heads, n_kv_heads, device_sms(dev));
}

int tq_decode_launch_count(const tq_segment *segs, int n_segs, int batch, int n_q_heads, int n_kv_heads) {
    if (check_segments(segs, n_segs, batch, n_q_heads, n_kv_heads) != TQ_OK) return -1;
    int dev = 0;
    cudaGetDevice(&dev);
    return tq_decode_launches(segs, n_segs, batch, n_q_heads, n_kv_heads, device_sms(dev));
}

tq_status tq_decode_attention(const tq_segment *segs, int n_segs, const void *q, tq_dtype q_dtype, int batch,
                              int n_q_heads, int n_kv_heads, void *out, tq_dtype out_dtype, void *workspace,
                              size_t ws_bytes, void *stream) {
    if (!q || !out) return TQ_ERR_NULL;
    tq_status st = check_segments(segs, n_segs, batch, n_q_heads, n_kv_heads);
    if (st != TQ_OK) return st;
    if ((q_dtype != TQ_F32 && q_dtype != TQ_F16 && q_dtype != TQ_BF16) ||
        (out_dtype != TQ_F32 && out_dtype != TQ_F16 && out_dtype != TQ_BF16))
        return TQ_ERR_DIM_MISMATCH;
    for (int s = 0; s < n_segs; ++s) {
        tq_ctx *c = const_cast<tq_ctx *>(segs[s].ctx);
        if ((st = tq_check_device(c)) != TQ_OK) return st;
        if ((st = tq_ensure_heads(c, n_kv_heads)) != TQ_OK) return st;
    }
    int dev = 0;
    cudaGetDevice(&dev);
    const size_t need = tq_decode_ws(segs, n_segs, batch, n_q_heads, n_kv_heads, device_sms(dev));
    if (!workspace || ws_bytes < need) return TQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return TQ_ERR_ALIGN;
    return tq_launch_decode(segs, n_segs, q, q_dtype, batch, n_q_heads, n_kv_heads, out, out_dtype, workspace,
                            ws_bytes, static_cast<cudaStream_t>(stream), device_sms(dev));
}

}  // extern "C"

// Segments as an append step sees them: the private tail of every sequence b
// (the one segment with n_seqs == 1 and first_seq == b) grows by one token,
// which the step writes.
static tq_status append_segments(const tq_segment *segs, int n_segs, int batch, std::vector<tq_segment> &grown,
                                 std::vector<uint8_t> &flags) {
    grown.assign(segs, segs + n_segs);
    flags.assign(n_segs, 0);
    std::vector<int> tail(batch, -1);
    for (int s = 0; s < n_segs; ++s) {
        if (segs[s].n_seqs != 1) continue;
        const int b = segs[s].first_seq;
        if (tail[b] >= 0) return TQ_ERR_DIM_MISMATCH;   // two private tails
        tail[b] = s;
    }
    for (int b = 0; b < batch; ++b) {
        if (tail[b] < 0) return TQ_ERR_DIM_MISMATCH;   // nowhere to append
        tq_segment &g = grown[tail[b]];
        if (g.n_tokens + 1 > g.codes.capacity) return TQ_ERR_DIM_MISMATCH;
        g.n_tokens += 1;
        flags[tail[b]] = 1;
    }
    return TQ_OK;
}

extern "C" {

size_t tq_decode_append_workspace_bytes(const tq_segment *segs, int n_segs, int batch, int n_q_heads,
                                        int n_kv_heads) {
    if (check_segments(segs, n_segs, batch, n_q_heads, n_kv_heads) != TQ_OK) return 0;
    std::vector<tq_segment> grown;
    std::vector<uint8_t> flags;
    if (append_segments(segs, n_segs, batch, grown, flags) != TQ_OK) return 0;
    int dev = 0;
    cudaGetDevice(&dev);
    return tq_decode_ws(grown.data(), n_segs, batch, n_q_heads, n_kv_heads, device_sms(dev));
}

tq_status tq_decode_append(const tq_segment *segs, int n_segs, const void *k_new, const void *v_new,
                           tq_dtype kv_dtype, const void *q, tq_dtype q_dtype, int batch, int n_q_heads,
                           int n_kv_heads, void *out, tq_dtype out_dtype, void *workspace, size_t ws_bytes,
                           void *stream) {
    if (!q || !out || !k_new || !v_new) return TQ_ERR_NULL;
    tq_status st = check_segments(segs, n_segs, batch, n_q_heads, n_kv_heads);
    if (st != TQ_OK) return st;
    if ((q_dtype != TQ_F32 && q_dtype != TQ_F16 && q_dtype != TQ_BF16) ||
        (out_dtype != TQ_F32 && out_dtype != TQ_F16 && out_dtype != TQ_BF16) ||
        (kv_dtype != TQ_F32 && kv_dtype != TQ_F16 && kv_dtype != TQ_BF16))
        return TQ_ERR_DIM_MISMATCH;
    const uintptr_t es = kv_dtype == TQ_F32 ? 4 : 2;
    if ((reinterpret_cast<uintptr_t>(k_new) | reinterpret_cast<uintptr_t>(v_new)) % es) return TQ_ERR_ALIGN;
    std::vector<tq_segment> grown;
    std::vector<uint8_t> flags;
    if ((st = append_segments(segs, n_segs, batch, grown, flags)) != TQ_OK) return st;
    for (int s = 0; s < n_segs; ++s) {
        tq_ctx *c = const_cast<tq_ctx *>(segs[s].ctx);
        if ((st = tq_check_device(c)) != TQ_OK) return st;
        if ((st = tq_ensure_heads(c, n_kv_heads)) != TQ_OK) return st;
    }
    int dev = 0;
    cudaGetDevice(&dev);
    const size_t need = tq_decode_ws(grown.data(), n_segs, batch, n_q_heads, n_kv_heads, device_sms(dev));
    if (!workspace || ws_bytes < need) return TQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return TQ_ERR_ALIGN;
    const TqAppend app{k_new, v_new, kv_dtype, flags.data()};
    return tq_launch_decode(grown.data(), n_segs, q, q_dtype, batch, n_q_heads, n_kv_heads, out, out_dtype,
                            workspace, ws_bytes, static_cast<cudaStream_t>(stream), device_sms(dev), &app);
}

size_t tq_decode_split_workspace_bytes(const tq_ctx *ctx_o, const tq_ctx *ctx_n, int batch, int n_q_heads,
                                       int64_t n_tokens) {
    if (!ctx_o || !ctx_n || batch <= 0 || n_q_heads <= 0 || n_tokens < 0) return 0;
    return tq_split_ws(batch, n_q_heads, ctx_o->d, ctx_n->d, n_tokens);
}

tq_status tq_decode_attention_split(tq_ctx *ctx_o, const tq_codes *codes_o, tq_ctx *ctx_n, const tq_codes *codes_n,
                                    int64_t n_tokens, const void *q, tq_dtype q_dtype, int batch, int n_q_heads,
                                    void *out, tq_dtype out_dtype, void *workspace, size_t ws_bytes, void *stream) {
    if (!ctx_o || !ctx_n || !q || !out) return TQ_ERR_NULL;
    tq_status st = check_codes(ctx_o, codes_o, true, true);
    if (st == TQ_OK) st = check_codes(ctx_n, codes_n, true, true);
    if (st != TQ_OK) return st;
    if (batch <= 0 || n_q_heads <= 0 || n_tokens <= 0) return TQ_ERR_EMPTY;
    if (codes_o->batch != batch || codes_n->batch != batch || codes_o->n_kv_heads != codes_n->n_kv_heads ||
        codes_o->capacity != codes_n->capacity || n_q_heads % codes_o->n_kv_heads ||
        n_tokens > codes_o->capacity)
        return TQ_ERR_DIM_MISMATCH;
    if ((q_dtype != TQ_F32 && q_dtype != TQ_F16 && q_dtype != TQ_BF16) ||
        (out_dtype != TQ_F32 && out_dtype != TQ_F16 && out_dtype != TQ_BF16))
        return TQ_ERR_DIM_MISMATCH;
    if ((st = tq_check_device(ctx_o)) != TQ_OK || (st = tq_check_device(ctx_n)) != TQ_OK) return st;
    if ((st = tq_ensure_heads(ctx_o, codes_o->n_kv_heads)) != TQ_OK) return st;
    if ((st = tq_ensure_heads(ctx_n, codes_n->n_kv_heads)) != TQ_OK) return st;
    const size_t need = tq_split_ws(batch, n_q_heads, ctx_o->d, ctx_n->d, n_tokens);
    if (!workspace || ws_bytes < need) return TQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return TQ_ERR_ALIGN;
    return tq_launch_split(ctx_o, codes_o, ctx_n, codes_n, n_tokens, q, q_dtype, batch, n_q_heads, out, out_dtype,
                           workspace, static_cast<cudaStream_t>(stream));
}

tq_status tq_get_status(tq_ctx *ctx, void *stream, uint64_t *nonfinite_rows, uint32_t *error_flags) {
    if (!ctx) return TQ_ERR_NULL;
    unsigned long long h[2] = {0, 0};
    tq_status st = tq_check_cuda(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    if (st == TQ_OK) st = tq_check_cuda(cudaMemcpy(h, ctx->d_status, sizeof(h), cudaMemcpyDeviceToHost));
    if (st != TQ_OK) return st;
    if (nonfinite_rows) *nonfinite_rows = h[0];
    if (error_flags) *error_flags = (uint32_t)h[1];
    return TQ_OK;
}

tq_status tq_reset_status(tq_ctx *ctx, void *stream) {
    if (!ctx) return TQ_ERR_NULL;
    return tq_check_cuda(
        cudaMemsetAsync(ctx->d_status, 0, 2 * sizeof(unsigned long long), static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

// ------------------------------------------------ allocation-free decode support
// Used only by tq_decode_attention_static (tq_static.cu): the same argument
// checks as tq_decode_attention, except that head tables are never built
// here (building allocates); a context without tables for n_kv_heads heads
// is rejected with TQ_ERR_LIMIT.
int tq_device_sms(int dev) { return device_sms(dev); }

tq_status tq_validate_decode(const tq_segment *segs, int n_segs, const void *q, tq_dtype q_dtype, int batch, int Hq,
                             int Hkv, const void *out, tq_dtype out_dtype, bool build_tables) {
    if (!q || !out) return TQ_ERR_NULL;
    tq_status st = check_segments(segs, n_segs, batch, Hq, Hkv);
    if (st != TQ_OK) return st;
    if ((q_dtype != TQ_F32 && q_dtype != TQ_F16 && q_dtype != TQ_BF16) ||
        (out_dtype != TQ_F32 && out_dtype != TQ_F16 && out_dtype != TQ_BF16))
        return TQ_ERR_DIM_MISMATCH;
    for (int s = 0; s < n_segs; ++s) {
        tq_ctx *c = const_cast<tq_ctx *>(segs[s].ctx);
        if ((st = tq_check_device(c)) != TQ_OK) return st;
        if (build_tables) {
            if ((st = tq_ensure_heads(c, Hkv)) != TQ_OK) return st;
        } else if (c->heads_built < Hkv) {
            return TQ_ERR_LIMIT;
        }
    }
    return TQ_OK;
}
