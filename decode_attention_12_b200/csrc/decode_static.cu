// decode_static.cu -- lla_decode_attn_static: decode attention whose scratch lives in
// a fixed-size device array inside the library, for callers that cannot allocate
// device memory.  The computation is exactly lla_decode_attn's; only the origin of the
// scratch differs.
//
// The array is a file-scope __device__ object, so every GPU that loads the library
// holds LLA_STATIC_SCRATCH_BYTES until the process exits.  In host code its name is
// only a host-side stand-in, never a device address: the address is looked up with
// cudaGetSymbolAddress, once per device, with that device current, and cached.
#include <mutex>

#include "decode.cuh"

namespace {

constexpr size_t kStaticScratchBytes = LLA_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device (looked up on first use).
int static_scratch_of_current_device(void **addr)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return LLA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess || p == nullptr)
            return LLA_ERR_CUDA;
        g_scratch_addr[dev] = p;
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
    // rewritten by every launch; the status word must start at zero.
    if (cudaMemsetAsync(scratch, 0, sizeof(int32_t), (cudaStream_t)stream) != cudaSuccess)
        return LLA_ERR_CUDA;
    return lla_decode_attn(dims, layer, t0, Tq, q, cache, seq_start, ctx_lens, B, max_ctx, codec,
                           softmax_scale, variant, num_splits, out, lse, scratch, kStaticScratchBytes,
                           stream);
}
