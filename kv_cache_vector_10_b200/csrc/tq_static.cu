// tq_static.cu -- decode attention that allocates nothing.
//
// Some callers cannot call cudaMalloc: a plug-in loaded into a host
// application that owns all device memory through its own allocator and
// hands the plug-in no allocation hook, or a serving loop that must not
// allocate on the decode path because cudaMalloc may synchronize the device.
// tq_decode_attention_static gives them the same decode as
// tq_decode_attention, with its scratch (prepared queries and split-K
// partials) in a fixed array compiled into the library instead of a
// caller-provided workspace.
//
// The array is a file-scope __device__ object of TQ_STATIC_SCRATCH_BYTES; every
// GPU that loads the library holds it until the process exits.  All calls on
// a device share it and it keeps the last call's contents; the decode writes
// every scratch byte it reads, so nothing needs clearing.  Calls that overlap
// on the GPU (different streams, no ordering between them) race on it.
#include <mutex>

#include "tq_internal.cuh"

size_t tq_decode_ws(const tq_segment *segs, int n_segs, int batch, int Hq, int Hkv, int n_sms);
struct TqAppend;
tq_status tq_launch_decode(const tq_segment *segs, int n_segs, const void *q, tq_dtype q_dtype, int batch,
                           int Hq, int Hkv, void *out, tq_dtype out_dtype, void *ws, size_t ws_bytes,
                           cudaStream_t stream, int n_sms, const TqAppend *app = nullptr);
tq_status tq_validate_decode(const tq_segment *segs, int n_segs, const void *q, tq_dtype q_dtype, int batch, int Hq,
                             int Hkv, const void *out, tq_dtype out_dtype, bool build_tables);
int tq_device_sms(int dev);

static __device__ __align__(256) unsigned char g_tq_static_scratch[TQ_STATIC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices];   // device address of the array, per device
}  // namespace

extern "C" tq_status tq_decode_attention_static(const tq_segment *segs, int n_segs, const void *q, tq_dtype q_dtype,
                                                int batch, int n_q_heads, int n_kv_heads, void *out,
                                                tq_dtype out_dtype, void *stream) {
    tq_status st = tq_validate_decode(segs, n_segs, q, q_dtype, batch, n_q_heads, n_kv_heads, out, out_dtype, false);
    if (st != TQ_OK) return st;
    int dev = -1;
    if ((st = tq_check_cuda(cudaGetDevice(&dev))) != TQ_OK) return st;
    if (dev < 0 || dev >= kMaxDevices) return TQ_ERR_DEVICE;
    const int sms = tq_device_sms(dev);
    const size_t need = tq_decode_ws(segs, n_segs, batch, n_q_heads, n_kv_heads, sms);
    if (need > (size_t)TQ_STATIC_SCRATCH_BYTES) return TQ_ERR_LIMIT;
    void *scratch = nullptr;
    {
        // One-time set-up per device, with that device current: the host-side
        // name of the array is not a device address, so ask the runtime.
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_scratch_addr[dev]) {
            void *p = nullptr;
            if ((st = tq_check_cuda(cudaGetSymbolAddress(&p, g_tq_static_scratch))) != TQ_OK) return st;
            g_scratch_addr[dev] = p;
        }
        scratch = g_scratch_addr[dev];
    }
    return tq_launch_decode(segs, n_segs, q, q_dtype, batch, n_q_heads, n_kv_heads, out, out_dtype, scratch,
                            (size_t)TQ_STATIC_SCRATCH_BYTES, static_cast<cudaStream_t>(stream), sms);
}
