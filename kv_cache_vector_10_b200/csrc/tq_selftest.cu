// tq_selftest.cu -- failure-detection self-test of the bounded waits.
//
// Every wait of the library's kernels on an mbarrier (TMA tiles, MMA
// completion) is bounded by wall time (%globaltimer); when a wait runs out
// the kernel records TQ_FLAG_WAIT_TIMEOUT in the context's status word,
// abandons the tile, and later kernels of the context skip their work until
// the host clears the word.  This kernel exercises that path without any
// fault: one thread waits, with a short bound, on an mbarrier phase that
// nothing completes.
#include "tq_internal.cuh"

namespace {

__global__ void tq_selftest_wait_kernel(unsigned long long *status, unsigned long long timeout_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        tqdev::mbar_init(&bar, 1);   // one expected arrival, which never comes
        tqdev::fence_barrier_init();
        if (!tqdev::mbar_wait_bounded(&bar, 0, timeout_ns))
            atomicOr(reinterpret_cast<unsigned int *>(status + 1), TQ_FLAG_WAIT_TIMEOUT);
    }
}

}  // namespace

tq_status tq_check_cuda(cudaError_t e);
tq_status tq_check_device(const tq_ctx *ctx);

extern "C" tq_status tq_selftest_wait_timeout(tq_ctx *ctx, uint32_t timeout_us, void *stream) {
    if (!ctx) return TQ_ERR_NULL;
    if (timeout_us == 0 || timeout_us > 100000) return TQ_ERR_LIMIT;
    tq_status st = tq_check_device(ctx);
    if (st != TQ_OK) return st;
    tq_selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(ctx->d_status,
                                                                             (unsigned long long)timeout_us * 1000ull);
    return tq_check_cuda(cudaGetLastError());
}
