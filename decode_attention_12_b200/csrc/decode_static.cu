// decode_static.cu -- lla_decode_attn_static: decode attention whose scratch lives in
// a fixed-size device array inside the library, for callers that cannot allocate
// device memory.  The computation is exactly lla_decode_attn's; only the origin of the
// scratch differs.
//
// The array is a file-scope __device__ object, so every GPU that loads the library
// holds LLA_STATIC_SCRATCH_BYTES until the process exits.  In host code its name is
// only a host-side stand-in, never a device address: the address is looked up with
// cudaGetSymbolAddress, with the device current, and cached together with the context
// it was looked up in; a call made in another context of that device (after a
// cudaDeviceReset, say) looks it up again.
#include <mutex>

#include "decode.cuh"
#include "tmap.cuh"

namespace {

constexpr size_t kStaticScratchBytes = LLA_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void *g_scratch_addr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

// The driver's cuCtxGetCurrent, through the runtime's entry-point query (the library
// does not link libcuda directly); nullptr when unavailable.
PFN_cuCtxGetCurrent_v4000 ctx_get_current()
{
    static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    });
    return fn;
}

// Device address of g_static_scratch in the current device's current context (looked
// up on first use in that context).
int static_scratch_of_current_device(void **addr)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return LLA_ERR_CUDA;
    auto get_ctx = ctx_get_current();
    if (get_ctx == nullptr)
        return LLA_ERR_CUDA;
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS)
        return LLA_ERR_CUDA;
    if (ctx == nullptr) {
        // no context bound to this thread yet: the runtime binds the device's primary
        // context on its first call that needs one, such as this lookup
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || get_ctx(&ctx) != CUDA_SUCCESS ||
            ctx == nullptr)
            return LLA_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_addr[dev] == nullptr || g_scratch_ctx[dev] != ctx) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess || p == nullptr)
            return LLA_ERR_CUDA;
        g_scratch_addr[dev] = p;
        g_scratch_ctx[dev] = ctx;
    }
    *addr = g_scratch_addr[dev];
    return LLA_OK;
}

} // namespace

extern "C" int lla_decode_attn_static(const lla_dims *dims, int32_t layer, int32_t t0, int32_t Tq,
                                      const void *q, const lla_cache *cache, const int64_t *seq_start,
                                      const int32_t *ctx_lens, int32_t B, int32_t max_ctx,
                                      const lla_codec *codec, float softmax_scale, int32_t variant,
                                      int32_t num_splits, void *out, float *lse, lla_stream_t stream)
{
    const int splits = lla_decode_num_splits(dims, B, Tq, max_ctx, variant, num_splits);
    if (splits < 0)
        return splits;
    const size_t need = lla_decode_workspace_bytes(dims, B, Tq, max_ctx, variant, num_splits);
    if (need == 0 || need > kStaticScratchBytes)
        return LLA_ERR_WORKSPACE;
    void *scratch = nullptr;
    const int rc = static_scratch_of_current_device(&scratch);
    if (rc != LLA_OK)
        return rc;
    // The array keeps the previous call's contents.  The partial records are fully
    // rewritten by every launch; the status word is cleared on `stream` once the
    // arguments have passed every check, so a refused call queues nothing.
    return lla::decode_attn_clearing_status(dims, layer, t0, Tq, q, cache, seq_start, ctx_lens, B, max_ctx, codec,
                                            softmax_scale, variant, num_splits, out, lse, scratch,
                                            kStaticScratchBytes, stream);
}

extern "C" int lla_status_fetch_static(lla_stream_t stream, int32_t *status_host)
{
    if (status_host == nullptr)
        return LLA_ERR_INVALID;
    void *scratch = nullptr;
    const int rc = static_scratch_of_current_device(&scratch);
    if (rc != LLA_OK)
        return rc;
    return lla_status_fetch(scratch, stream, status_host);
}
