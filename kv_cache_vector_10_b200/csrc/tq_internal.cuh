// tq_internal.cuh -- definitions shared by the libtq translation units:
// the context, kernel parameter blocks, and thin wrappers over the sm_100a
// PTX used by the kernels (mbarrier, TMA, tcgen05).  Every wait on an
// mbarrier is bounded: when the bound is hit the caller records an error
// flag in the context's status word and abandons the tile.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/tq.h"

#define TQ_MAX_LEVELS 32

// Status word layout (device, 2 x u64): [0] non-finite rows, [1] error flags.
#define TQ_FLAG_WAIT_TIMEOUT 1u

struct tq_ctx {
    int d, bits, m, BK, BV, LK, LV;
    uint64_t seed;
    int device;
    int heads_built;
    uint32_t *d_signs;              // [heads][d/32]; bit j set -> sign -1
    __half *d_S;                    // [heads][m][d] binary16 QJL matrix
    unsigned long long *d_status;   // [2]
    CUtensorMap tmap_S;             // 2-D view of d_S: inner d, outer heads*m
    // Lloyd-Max codebooks of N(0,1): centroids ascending and boundaries.
    float ck[TQ_MAX_LEVELS], bk[TQ_MAX_LEVELS], cv[TQ_MAX_LEVELS], bv[TQ_MAX_LEVELS];
    struct TqBook *d_book;          // device copy of the positive halves (TqBook)
    int rotation;                   // tq_rotation
    int norm_f16;                   // 1: key rows end in n_s, gamma as binary16 (tq_norm_format)
    // Haar rotation tables (rotation == TQ_ROT_HAAR): Q [heads][d][d] fp32,
    // and sqrt(d) Q as binary16 hi + lo [heads][2][d][d] with its TMA map
    // (inner d, outer heads*2*d rows, box 64 x d, 128-byte swizzle).
    float *d_Q32;
    __half *d_Qh;
    CUtensorMap tmap_Q;
    // and sqrt(d) Q as bfloat16 hi + mid + lo [heads][3][d][d] (d <= 128) for
    // the TMA-fed value encoder's bfloat16 rows, same map geometry.
    uint16_t *d_Qbf;
    CUtensorMap tmap_Qbf;
    // Walsh-Hadamard rotation as a tensor-core operand: B[h][n][k] = H[n][k] D_h[k]
    // (+-1, exact in both 16-bit types), binary16 and bfloat16 copies
    // [heads][d][d], with TMA maps (inner d, outer heads*d rows, box 64 x d,
    // 128-byte swizzle).  Built for TQ_ROT_HADAMARD contexts.
    uint16_t *d_HD16, *d_HDbf;
    CUtensorMap tmap_HD16, tmap_HDbf;
};

// Positive halves of the codebooks: magnitudes of the centroids and the
// positive boundaries.  For L levels, mag[k] = c[L/2 + k] (k < L/2) and
// pb[k] = beta[L/2 + k] (k < L/2 - 1).
struct TqBook {
    float kmag[16];
    float kpb[16];
    float vmag[16];
    float vpb[16];
};

namespace tqdev {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t phase) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(phase)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait on an mbarrier phase: gives up after timeout_ns of wall time
// (default 200 ms) and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t phase,
                                                  uint64_t timeout_ns = 200000000ull) {
    if (mbar_try_wait(bar, phase)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, phase)) {
        if (globaltimer_ns() - t0 > timeout_ns) return false;
    }
    return true;
}

// True once any kernel of this context recorded a timed-out wait; later
// CTAs then skip their work instead of waiting again.
__device__ __forceinline__ bool status_aborted(const unsigned long long *status) {
    return (*reinterpret_cast<const volatile unsigned long long *>(status + 1) & TQ_FLAG_WAIT_TIMEOUT) != 0;
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------- TMA
// 2-D tiled bulk tensor load into shared memory, completion on an mbarrier
// (no multicast).
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// 4-D tiled bulk tensor load (no multicast), completion on an mbarrier.
__device__ __forceinline__ void tma_load_4d(void *smem_dst, const CUtensorMap *map, int x, int y, int z, int w,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
        : "memory");
}

// Named barrier `id` over `nthreads` threads (a multiple of 32).
__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// 1-D bulk copy global -> shared (16-byte aligned addresses, size % 16 == 0).
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gsrc, uint32_t bytes,
                                          uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(smem_dst)),
        "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t *smem_dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(smem_dst)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16, one CTA.
__device__ __forceinline__ void mma_f16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on an mbarrier once all previously issued tcgen05.mma of this thread complete.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// Each thread of the warp reads 32 consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Loads without the completion wait (pair with tmem_wait_ld).
__device__ __forceinline__ void tmem_ld_32x32b_x32_nowait(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld_32x32b_x8_nowait(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7])
                 : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// Each thread of the warp reads 16 consecutive 32-bit columns of its lane (no wait).
__device__ __forceinline__ void tmem_ld_32x32b_x16_nowait(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Each thread of the warp writes 32 (or 8) consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

__device__ __forceinline__ void tmem_st_32x32b_x8(uint32_t taddr, const float (&v)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
                 "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
                 "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
                 "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
                 : "memory");
}

// Shared-memory matrix descriptor for a K-major operand stored in 128-byte
// swizzled atoms (8 rows x 128 bytes, 16-byte chunk c of row r stored at
// chunk c ^ (r % 8)); consecutive 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
    uint64_t desc = 0;
    desc |= (uint64_t)((saddr >> 4) & 0x3FFF);          // start address
    desc |= (uint64_t)1 << 16;                          // leading byte offset (unused, 16 B)
    desc |= (uint64_t)(1024 >> 4) << 32;                // stride byte offset: 8 rows
    desc |= (uint64_t)1 << 46;                          // descriptor version (sm_100)
    desc |= (uint64_t)2 << 61;                          // 128-byte swizzle
    return desc;
}

// Instruction descriptor: kind::f16, A and B binary16, K-major, fp32
// accumulator, M = 128, N = n.
// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start before the previous kernel in the stream ends;
// grid_dep_wait blocks until that kernel has completed and its memory is
// visible (it returns at once for a kernel launched without the attribute),
// and grid_dep_trigger lets the next such kernel start launching.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Key-row norms.  Binary16 format: n_s and gamma rounded to binary16 (ties
// to even) in one 32-bit word, n_s in the low half; pack returns false if
// either rounds to infinity (the row is then stored as a zero row).
__device__ __forceinline__ bool pack_norms_f16(float ns, float g, uint32_t &w) {
    const __half hn = __float2half_rn(ns), hg = __float2half_rn(g);
    w = (uint32_t)__half_as_ushort(hn) | ((uint32_t)__half_as_ushort(hg) << 16);
    return !(__hisinf(hn) || __hisinf(hg));
}
// (n_s, gamma) from a key row's tail words.
__device__ __forceinline__ float2 key_norms(const uint32_t *tail, bool f16) {
    if (f16) {
        const uint32_t w = tail[0];
        return make_float2(__half2float(__ushort_as_half((unsigned short)(w & 0xFFFFu))),
                           __half2float(__ushort_as_half((unsigned short)(w >> 16))));
    }
    return make_float2(__uint_as_float(tail[0]), __uint_as_float(tail[1]));
}

__host__ __device__ constexpr uint32_t idesc_f16_f32(int n) {
    return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
// The same with A and B in bfloat16.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int n) {
    return idesc_f16_f32(n) | (1u << 7) | (1u << 10);
}

}  // namespace tqdev

// ------------------------------------------------------------ host helpers
// Launch with programmatic stream serialization: the kernel may begin while
// the previous kernel in the stream is still running; it must call
// tqdev::grid_dep_wait() before it reads anything that kernel writes.
template <typename... KArgs, typename... Args>
cudaError_t tq_launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

tq_status tq_check_cuda(cudaError_t e);
tq_status tq_check_device(const tq_ctx *ctx);
// Sigma-plane decomposition of the key codebook (odd subsets of the B_K index
// bits and their Walsh coefficients), as the decode kernel uses it.
void tq_sigma_planes(const tq_ctx *ctx, int *n_planes, uint32_t *sets, float *alpha);
