// lla_api.cu -- the C ABI of liblla (declared in include/lla.h): argument checks,
// kernel selection, workspace carving, status handling.  Every arithmetic step of
// the path runs in the kernels; this file only validates and launches.
#include <atomic>
#include <climits>
#include <cmath>
#include <cstring>

#include "decode.cuh"
#include "encode.cuh"

namespace lla {
// decode_simt.cu: whether the combine can hold W_up,t^V for this shape
bool decode_combine_supported(int r_v, int d, bool recon);
} // namespace lla

using namespace lla;

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_bytes(int dtype) { return dtype == LLA_BF16 ? 2 : 4; }

// Basic validity of the problem description.
int check_dims(const lla_dims *d)
{
    if (d == nullptr)
        return LLA_ERR_INVALID;
    if (d->T <= 0 || d->L <= 0 || d->H <= 0 || d->d_head <= 0 || d->r_k <= 0 || d->r_v <= 0)
        return LLA_ERR_INVALID;
    if (d->fold != LLA_PER_HEAD && d->fold != LLA_FOLD_2D)
        return LLA_ERR_INVALID;
    if (d->dtype != LLA_F32 && d->dtype != LLA_BF16)
        return LLA_ERR_INVALID;
    if (d->out_dtype != LLA_F32 && d->out_dtype != LLA_BF16)
        return LLA_ERR_INVALID;
    const int64_t W = (int64_t)d->T * d->d_head * (d->fold ? d->H : 1);
    if (W > INT32_MAX / 2 || d->r_k > W || d->r_v > W)
        return LLA_ERR_INVALID;
    // every latent row and every W_down row must be a whole number of 16-byte chunks
    const int e = elem_bytes(d->dtype);
    if ((d->r_k * e) % 16 != 0 || (d->r_v * e) % 16 != 0 || (W * e) % 16 != 0)
        return LLA_ERR_UNSUPPORTED;
    return LLA_OK;
}

int heads_stored(const lla_dims *d) { return d->fold ? 1 : d->H; }
int64_t stack_width(const lla_dims *d) { return (int64_t)d->T * d->d_head * (d->fold ? d->H : 1); }
int64_t loop_width(const lla_dims *d) { return (int64_t)d->d_head * (d->fold ? d->H : 1); }

// SM count of the current device, looked up once per device (atomic: the library may be
// called from several host threads at once).
int sm_count()
{
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return 148;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// Plan of one decode call: the work split of the persistent decode kernel and the
// workspace regions (header | counts | q_tilde | partial records).
struct Plan {
    int32_t seg_max, chunk_min;
    size_t off_counts, off_qt, off_part, off_win, bytes;
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

Plan make_plan(const lla_dims *d, int32_t B, int32_t Tq, int32_t max_ctx, int32_t num_splits, int32_t variant,
               bool window = false, int32_t d_rope = 0)
{
    Plan p;
    const int64_t units = (int64_t)B * d->H;
    const int64_t ctas = (int64_t)sm_count() * kDecodeCtasPerSm;
    int64_t segs = num_splits > 0 ? num_splits : (units > 0 ? (2 * ctas + units - 1) / units : 1);
    if (segs < 1) segs = 1;
    if (segs > 64) segs = 64;
    int64_t chunk_min = (max_ctx + segs - 1) / segs;
    if (chunk_min < 128) chunk_min = 128;
    // LLA-2D: units are whole sequences and each segment writes H x Tq records; by default a
    // share holds at least 256 tokens (four whole 64-token tiles): for 16 sequences of
    // 4096 tokens this measured the shortest decode grid (22.7 us against 29.1 us at 384,
    // and 26.9-27.1 us at 171 or 128, where partial tiles and records cost more)
    if (num_splits == 0 && variant == LLA_ABSORB &&
        decode_mma2d_supported(d->dtype, d->r_k, d->r_v, d->fold, d->H))
        chunk_min = 256;
    p.chunk_min = (int32_t)chunk_min;
    p.seg_max = (int32_t)((max_ctx + chunk_min - 1) / chunk_min + 1);
    p.off_counts = kWorkspaceHeader;
    p.off_qt = align256(p.off_counts + (size_t)units * sizeof(int32_t));
    p.off_part = align256(p.off_qt + (size_t)units * Tq * (d->r_k + d_rope) * sizeof(float));
    // reconstruct-form records carry d-wide outputs, absorbed-form records r_v-wide latents
    const int rec_w = variant == LLA_RECONSTRUCT ? d->d_head : d->r_v;
    p.bytes = p.off_part + (size_t)units * Tq * p.seg_max * part_stride(rec_w) * sizeof(float);
    p.off_win = 0;
    if (window) { // hybrid form: one d-wide window record per (unit, loop query)
        p.off_win = align256(p.bytes);
        p.bytes = p.off_win + (size_t)units * Tq * part_stride(d->d_head) * sizeof(float);
    }
    return p;
}

} // namespace

extern "C" {

const char *lla_status_string(int code)
{
    switch (code) {
    case LLA_OK: return "ok";
    case LLA_ERR_INVALID: return "invalid argument";
    case LLA_ERR_UNSUPPORTED: return "unsupported rank, dtype or shape";
    case LLA_ERR_MISALIGNED: return "device pointer not 16-byte aligned";
    case LLA_ERR_WORKSPACE: return "workspace missing or too small";
    case LLA_ERR_CUDA: return "CUDA launch or copy failed";
    case LLA_ERR_DEVICE_TIMEOUT: return "a kernel gave up a bounded wait";
    case LLA_ERR_NO_CONVERGENCE: return "the codec fit's eigen-solver did not converge";
    default: return "unknown status";
    }
}

int lla_cache_bytes(const lla_dims *dims, const int32_t *ctx_lens_host, int32_t B,
                    uint64_t *latent_bytes, uint64_t *uncompressed_bytes, uint64_t *rho_num,
                    uint64_t *rho_den)
{
    if (dims == nullptr || B < 0 || (B > 0 && ctx_lens_host == nullptr))
        return LLA_ERR_INVALID;
    if (dims->T <= 0 || dims->L <= 0 || dims->H <= 0 || dims->d_head <= 0 || dims->r_k <= 0 ||
        dims->r_v <= 0 || (dims->fold != 0 && dims->fold != 1) || (dims->dtype != 0 && dims->dtype != 1))
        return LLA_ERR_INVALID;
    unsigned __int128 S = 0;
    for (int32_t b = 0; b < B; ++b) {
        if (ctx_lens_host[b] < 0)
            return LLA_ERR_INVALID;
        S += (unsigned)ctx_lens_host[b];
    }
    const unsigned __int128 e = (unsigned)elem_bytes(dims->dtype);
    const unsigned __int128 per_unc = (unsigned __int128)2 * dims->T * dims->H * dims->d_head;
    const unsigned __int128 per_lat = (unsigned __int128)heads_stored(dims) * (dims->r_k + dims->r_v);
    const unsigned __int128 unc = S * dims->L * per_unc * e;
    const unsigned __int128 lat = S * dims->L * per_lat * e;
    if (unc > (unsigned __int128)UINT64_MAX || lat > (unsigned __int128)UINT64_MAX)
        return LLA_ERR_INVALID;
    uint64_t a = (uint64_t)per_unc, b = (uint64_t)per_lat;
    while (b != 0) {
        const uint64_t t = a % b;
        a = b;
        b = t;
    }
    if (latent_bytes) *latent_bytes = (uint64_t)lat;
    if (uncompressed_bytes) *uncompressed_bytes = (uint64_t)unc;
    if (rho_num) *rho_num = (uint64_t)per_unc / a;
    if (rho_den) *rho_den = (uint64_t)per_lat / a;
    return LLA_OK;
}

int lla_slot_layout(const int32_t *ctx_lens_host, int32_t B, int64_t gap, int64_t *seq_start_host,
                    int64_t *total_slots)
{
    if (B < 0 || gap < 0 || (B > 0 && (ctx_lens_host == nullptr || seq_start_host == nullptr)))
        return LLA_ERR_INVALID;
    int64_t pos = 0;
    for (int32_t b = 0; b < B; ++b) {
        if (ctx_lens_host[b] < 0)
            return LLA_ERR_INVALID;
        seq_start_host[b] = pos;
        if (pos > INT64_MAX - ctx_lens_host[b] - gap)
            return LLA_ERR_INVALID;
        pos += ctx_lens_host[b] + gap;
    }
    if (total_slots)
        *total_slots = pos;
    return LLA_OK;
}

int lla_codec_bias(const lla_dims *dims, const lla_codec *codec, float *bias_k_out, float *bias_v_out,
                   lla_stream_t stream)
{
    int rc = check_dims(dims);
    if (rc != LLA_OK)
        return rc;
    if (codec == nullptr || codec->W_down_k == nullptr || codec->W_down_v == nullptr ||
        codec->mu_k == nullptr || codec->mu_v == nullptr || bias_k_out == nullptr || bias_v_out == nullptr)
        return LLA_ERR_INVALID;
    const int64_t groups = (int64_t)dims->L * heads_stored(dims);
    const int W = (int)stack_width(dims);
    cudaError_t e = launch_codec_bias(codec->W_down_k, codec->mu_k, bias_k_out, groups, dims->r_k, W,
                                      dims->dtype, (cudaStream_t)stream);
    if (e == cudaSuccess)
        e = launch_codec_bias(codec->W_down_v, codec->mu_v, bias_v_out, groups, dims->r_v, W, dims->dtype,
                              (cudaStream_t)stream);
    return e == cudaSuccess ? LLA_OK : LLA_ERR_CUDA;
}

int lla_encode(const lla_dims *dims, int32_t layer0, int32_t n_layers, const void *x_k, const void *x_v,
               int64_t n_tok, const int64_t *slot_idx, const lla_codec *codec, const lla_cache *cache,
               lla_stream_t stream)
{
    int rc = check_dims(dims);
    if (rc != LLA_OK)
        return rc;
    if (layer0 < 0 || n_layers < 0 || layer0 + (int64_t)n_layers > dims->L || n_tok < 0)
        return LLA_ERR_INVALID;
    if (n_tok == 0 || n_layers == 0)
        return LLA_OK;
    if (x_k == nullptr || x_v == nullptr || slot_idx == nullptr || codec == nullptr || cache == nullptr ||
        codec->W_down_k == nullptr || codec->W_down_v == nullptr || codec->bias_k == nullptr ||
        codec->bias_v == nullptr || cache->k == nullptr || cache->v == nullptr || cache->slots < 0)
        return LLA_ERR_INVALID;
    if (!aligned16(x_k) || !aligned16(x_v) || !aligned16(slot_idx) || !aligned16(codec->W_down_k) ||
        !aligned16(codec->W_down_v) || !aligned16(codec->bias_k) || !aligned16(codec->bias_v) ||
        !aligned16(cache->k) || !aligned16(cache->v))
        return LLA_ERR_MISALIGNED;
    if (dims->r_k > 256 || dims->r_v > 256)
        return LLA_ERR_UNSUPPORTED;
    EncodeArgs a;
    a.x_k = x_k; a.x_v = x_v;
    a.W_down_k = codec->W_down_k; a.W_down_v = codec->W_down_v;
    a.bias_k = codec->bias_k; a.bias_v = codec->bias_v;
    a.cache_k = cache->k; a.cache_v = cache->v;
    a.slot_idx = slot_idx;
    a.n_tok = n_tok; a.slots = cache->slots;
    a.layer0 = layer0; a.n_layers = n_layers;
    a.T = dims->T; a.H = dims->H; a.d = dims->d_head; a.Hs = heads_stored(dims);
    a.W = (int32_t)stack_width(dims);
    a.r_k = dims->r_k; a.r_v = dims->r_v; a.fold = dims->fold;
    cudaError_t e;
    if (dims->dtype == LLA_BF16 && encode_tc_supported(a))
        e = launch_encode_tc(a, (cudaStream_t)stream);   // tcgen05 tensor cores
    else
        e = launch_encode_simt(a, dims->dtype, (cudaStream_t)stream);
    return e == cudaSuccess ? LLA_OK : LLA_ERR_CUDA;
}

size_t lla_codec_fit_workspace_bytes(const lla_dims *dims, int32_t n_layers, int64_t n_cal)
{
    if (check_dims(dims) != LLA_OK || n_layers <= 0 || n_cal < 2)
        return 0;
    const int r_max = dims->r_k > dims->r_v ? dims->r_k : dims->r_v;
    return kWorkspaceHeader +
           codec_fit_scratch_bytes((int64_t)n_layers * heads_stored(dims), n_cal, stack_width(dims), r_max) + 1536;
}

int lla_codec_fit(const lla_dims *dims, int32_t layer0, int32_t n_layers, const void *x_k, const void *x_v,
                  int64_t n_cal, const lla_codec *codec, float *sigma_k, float *sigma_v, void *workspace,
                  size_t ws_bytes, lla_stream_t stream)
{
    int rc = check_dims(dims);
    if (rc != LLA_OK)
        return rc;
    if (layer0 < 0 || n_layers < 0 || layer0 + (int64_t)n_layers > dims->L)
        return LLA_ERR_INVALID;
    if (n_layers == 0)
        return LLA_OK;
    if (n_cal < 2 || n_cal > 1024 || (n_cal & 1) || dims->r_k > n_cal - 1 || dims->r_v > n_cal - 1)
        return LLA_ERR_INVALID;
    if (x_k == nullptr || x_v == nullptr || codec == nullptr || codec->W_down_k == nullptr ||
        codec->W_down_v == nullptr || codec->W_up_k == nullptr || codec->W_up_v == nullptr ||
        codec->mu_k == nullptr || codec->mu_v == nullptr)
        return LLA_ERR_INVALID;
    if (!aligned16(x_k) || !aligned16(x_v) || !aligned16(codec->W_down_k) || !aligned16(codec->W_down_v) ||
        !aligned16(codec->W_up_k) || !aligned16(codec->W_up_v) || !aligned16(codec->mu_k) ||
        !aligned16(codec->mu_v))
        return LLA_ERR_MISALIGNED;
    const size_t need = lla_codec_fit_workspace_bytes(dims, n_layers, n_cal);
    if (workspace == nullptr || ws_bytes < need)
        return LLA_ERR_WORKSPACE;
    if (!aligned16(workspace))
        return LLA_ERR_MISALIGNED;
    CodecFitArgs a;
    a.x_k = x_k; a.x_v = x_v;
    a.W_down_k = const_cast<void *>(codec->W_down_k); a.W_down_v = const_cast<void *>(codec->W_down_v);
    a.W_up_k = const_cast<float *>(codec->W_up_k); a.W_up_v = const_cast<float *>(codec->W_up_v);
    a.mu_k = const_cast<float *>(codec->mu_k); a.mu_v = const_cast<float *>(codec->mu_v);
    a.sigma_k = sigma_k; a.sigma_v = sigma_v;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    a.status = reinterpret_cast<int32_t *>(ws);
    a.scratch = ws + kWorkspaceHeader;
    a.n = n_cal;
    a.layer0 = layer0; a.n_layers = n_layers;
    a.T = dims->T; a.H = dims->H; a.d = dims->d_head; a.Dp = (int32_t)loop_width(dims); a.Hs = heads_stored(dims);
    a.W = (int32_t)stack_width(dims); a.fold = dims->fold; a.r_k = dims->r_k; a.r_v = dims->r_v;
    a.dtype = dims->dtype;
    return launch_codec_fit(a, (cudaStream_t)stream) == cudaSuccess ? LLA_OK : LLA_ERR_CUDA;
}

int lla_codec_residual(const lla_dims *dims, int32_t layer0, int32_t n_layers, const void *x_k, const void *x_v,
                       int64_t n_tok, const lla_codec *codec, float *err_k, float *norm_k, float *err_v,
                       float *norm_v, lla_stream_t stream)
{
    int rc = check_dims(dims);
    if (rc != LLA_OK)
        return rc;
    if (layer0 < 0 || n_layers < 0 || layer0 + (int64_t)n_layers > dims->L || n_tok < 0)
        return LLA_ERR_INVALID;
    if (n_tok == 0 || n_layers == 0)
        return LLA_OK;
    if (x_k == nullptr || x_v == nullptr || codec == nullptr || codec->W_down_k == nullptr ||
        codec->W_down_v == nullptr || codec->bias_k == nullptr || codec->bias_v == nullptr ||
        codec->W_up_k == nullptr || codec->W_up_v == nullptr || codec->mu_k == nullptr || codec->mu_v == nullptr ||
        err_k == nullptr || norm_k == nullptr || err_v == nullptr || norm_v == nullptr)
        return LLA_ERR_INVALID;
    if (!aligned16(x_k) || !aligned16(x_v) || !aligned16(codec->W_down_k) || !aligned16(codec->W_down_v) ||
        !aligned16(codec->bias_k) || !aligned16(codec->bias_v) || !aligned16(codec->W_up_k) ||
        !aligned16(codec->W_up_v) || !aligned16(codec->mu_k) || !aligned16(codec->mu_v))
        return LLA_ERR_MISALIGNED;
    const int Dp = (int)loop_width(dims);
    if (!codec_residual_supported(dims->dtype, dims->r_k, dims->r_v, Dp))
        return LLA_ERR_UNSUPPORTED;
    CodecResidualArgs a;
    a.x_k = x_k; a.x_v = x_v;
    a.W_down_k = codec->W_down_k; a.W_down_v = codec->W_down_v;
    a.bias_k = codec->bias_k; a.bias_v = codec->bias_v;
    a.W_up_k = codec->W_up_k; a.W_up_v = codec->W_up_v;
    a.mu_k = codec->mu_k; a.mu_v = codec->mu_v;
    a.err_k = err_k; a.norm_k = norm_k; a.err_v = err_v; a.norm_v = norm_v;
    a.n_tok = n_tok;
    a.layer0 = layer0; a.n_layers = n_layers;
    a.T = dims->T; a.H = dims->H; a.d = dims->d_head; a.Dp = Dp; a.Hs = heads_stored(dims);
    a.W = (int32_t)stack_width(dims); a.fold = dims->fold; a.r_k = dims->r_k; a.r_v = dims->r_v;
    return launch_codec_residual(a, (cudaStream_t)stream) == cudaSuccess ? LLA_OK : LLA_ERR_CUDA;
}

int lla_decode_num_splits(const lla_dims *dims, int32_t B, int32_t Tq, int32_t max_ctx, int32_t variant,
                          int32_t num_splits)
{
    int rc = check_dims(dims);
    if (rc != LLA_OK)
        return rc;
    if (B < 0 || Tq < 1 || max_ctx < 0 || num_splits < 0 ||
        (variant != LLA_ABSORB && variant != LLA_RECONSTRUCT))
        return LLA_ERR_INVALID;
    return make_plan(dims, B, Tq, max_ctx, num_splits, variant).seg_max;
}

size_t lla_decode_workspace_bytes(const lla_dims *dims, int32_t B, int32_t Tq, int32_t max_ctx,
                                  int32_t variant, int32_t num_splits)
{
    if (lla_decode_num_splits(dims, B, Tq, max_ctx, variant, num_splits) < 1)
        return 0;
    return make_plan(dims, B, Tq, max_ctx, num_splits, variant).bytes;
}

} // extern "C"

namespace {

// Body of lla_decode_attn and lla_decode_attn_hybrid (window == NULL: latents only).
int decode_call(const lla_dims *dims, int32_t layer, int32_t t0, int32_t Tq, const void *q,
                const lla_cache *cache, const int64_t *seq_start, const int32_t *ctx_lens, int32_t B,
                int32_t max_ctx, const lla_codec *codec, const lla_window *window, const lla_rope *rope,
                float softmax_scale, int32_t variant, int32_t num_splits, void *out, float *lse,
                void *workspace, size_t ws_bytes, lla_stream_t stream, const lla_decoupled *dec = nullptr,
                lla_event_t ev_start = nullptr, lla_event_t ev_end = nullptr, bool clear_status = false)
{
    int rc = check_dims(dims);
    if (rc != LLA_OK)
        return rc;
    if (layer < 0 || layer >= dims->L || t0 < 0 || Tq < 1 || t0 + (int64_t)Tq > dims->T || B < 0 ||
        max_ctx < 0 || num_splits < 0 || (variant != LLA_ABSORB && variant != LLA_RECONSTRUCT))
        return LLA_ERR_INVALID;
    if (B == 0) { // nothing to compute; a status word the caller asked to clear is cleared
        if (!clear_status)
            return LLA_OK;
        if (workspace == nullptr || !aligned16(workspace))
            return LLA_ERR_INVALID;
        return cudaMemsetAsync(workspace, 0, sizeof(int32_t), (cudaStream_t)stream) == cudaSuccess ? LLA_OK
                                                                                                   : LLA_ERR_CUDA;
    }
    if (q == nullptr || cache == nullptr || cache->k == nullptr || cache->v == nullptr || cache->slots < 0 ||
        seq_start == nullptr || ctx_lens == nullptr || codec == nullptr || codec->W_up_k == nullptr ||
        codec->W_up_v == nullptr || codec->mu_k == nullptr || codec->mu_v == nullptr || out == nullptr)
        return LLA_ERR_INVALID;
    if (!aligned16(q) || !aligned16(cache->k) || !aligned16(cache->v) || !aligned16(out) ||
        !aligned16(codec->W_up_k) || !aligned16(codec->W_up_v) || !aligned16(codec->mu_k) ||
        !aligned16(codec->mu_v) || !aligned16(seq_start) || !aligned16(ctx_lens) ||
        (lse != nullptr && !aligned16(lse)))
        return LLA_ERR_MISALIGNED;
    if ((dims->d_head * elem_bytes(dims->dtype)) % 16 != 0)
        return LLA_ERR_UNSUPPORTED; // query / output rows are moved in 16-byte pieces
    if (dec != nullptr) {
        if (rope == nullptr || dec->k_rope == nullptr || dec->q_rope == nullptr || dec->d_rope <= 0)
            return LLA_ERR_INVALID;
        if (!aligned16(dec->k_rope) || !aligned16(dec->q_rope))
            return LLA_ERR_MISALIGNED;
    }
    if (rope != nullptr) {
        if (variant != (dec != nullptr ? LLA_ABSORB : LLA_RECONSTRUCT) || rope->q_pos == nullptr || !std::isfinite(rope->base) ||
            rope->base <= 1.0f || (rope->style != LLA_ROPE_HALF && rope->style != LLA_ROPE_INTERLEAVED))
            return LLA_ERR_INVALID;
        if (!aligned16(rope->q_pos))
            return LLA_ERR_MISALIGNED;
    }
    if (dec != nullptr && !decode_mma_rope_supported(dims->dtype, dims->r_k, dims->r_v, dec->d_rope, dims->fold))
        return LLA_ERR_UNSUPPORTED;
    if (window != nullptr) {
        if (window->w_max < 0 || window->seqs < B || window->len == nullptr ||
            (window->w_max > 0 && (window->k == nullptr || window->v == nullptr)))
            return LLA_ERR_INVALID;
        if (!aligned16(window->len) || !aligned16(window->k) || !aligned16(window->v))
            return LLA_ERR_MISALIGNED;
        if (!decode_window_supported(dims->dtype, dims->d_head))
            return LLA_ERR_UNSUPPORTED;
    }
    const Plan plan = make_plan(dims, B, Tq, max_ctx, num_splits, variant, window != nullptr,
                                dec != nullptr ? dec->d_rope : 0);
    if (workspace == nullptr || ws_bytes < plan.bytes)
        return LLA_ERR_WORKSPACE;
    if (!aligned16(workspace))
        return LLA_ERR_MISALIGNED;
    if (variant == LLA_RECONSTRUCT &&
        !decode_reconstruct_supported(dims->dtype, dims->r_k, dims->r_v, dims->d_head))
        return LLA_ERR_UNSUPPORTED;
    const bool use_mma = decode_mma_supported(dims->dtype, dims->r_k, dims->r_v, dims->fold, Tq);
    if (!use_mma && !decode_absorb_supported(dims->dtype, dims->r_k, dims->r_v, dims->d_head, dims->fold))
        return LLA_ERR_UNSUPPORTED;
    if (B > 16384 || !decode_combine_supported(dims->r_v, dims->d_head, variant == LLA_RECONSTRUCT))
        return LLA_ERR_UNSUPPORTED;

    const int Hs = heads_stored(dims);
    const int64_t Dp = loop_width(dims);
    const int e = elem_bytes(dims->dtype);
    DecodeArgs a;
    a.q = q;
    a.k = static_cast<const uint8_t *>(cache->k) + (int64_t)layer * Hs * cache->slots * dims->r_k * e;
    a.v = static_cast<const uint8_t *>(cache->v) + (int64_t)layer * Hs * cache->slots * dims->r_v * e;
    a.slots = cache->slots;
    a.seq_start = seq_start;
    a.ctx_lens = ctx_lens;
    a.W_up_k = codec->W_up_k + (int64_t)layer * Hs * dims->T * dims->r_k * Dp;
    a.W_up_v = codec->W_up_v + (int64_t)layer * Hs * dims->T * dims->r_v * Dp;
    a.mu_k = codec->mu_k + (int64_t)layer * Hs * dims->T * Dp;
    a.mu_v = codec->mu_v + (int64_t)layer * Hs * dims->T * Dp;
    a.B = B; a.H = dims->H; a.d = dims->d_head; a.T = dims->T; a.t0 = t0; a.Tq = Tq;
    a.fold = dims->fold; a.r_k = dims->r_k; a.r_v = dims->r_v;
    a.recon = variant == LLA_RECONSTRUCT;
    a.seg_max = plan.seg_max;
    a.chunk_min = plan.chunk_min;
    a.scale = softmax_scale;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    a.status = reinterpret_cast<int32_t *>(ws);
    a.counts = reinterpret_cast<int32_t *>(ws + plan.off_counts);
    a.qt = reinterpret_cast<float *>(ws + plan.off_qt);
    a.part = reinterpret_cast<float *>(ws + plan.off_part);
    a.out = out;
    a.lse = lse;
    a.win_k = a.win_v = nullptr;
    a.win_len = nullptr;
    a.w_max = 0;
    a.win_part = nullptr;
    a.q_pos = rope != nullptr ? rope->q_pos : nullptr;
    a.rope_base = rope != nullptr ? rope->base : 0.f;
    a.rope_style = rope != nullptr ? rope->style : 0;
    a.k_rope = a.q_rope = nullptr;
    a.d_rope = 0;
    // timing aid: events around the latent-streaming grid, every grid launched in order
    a.serial = ev_start != nullptr || ev_end != nullptr;
    cudaEvent_t e0 = reinterpret_cast<cudaEvent_t>(ev_start), e1 = reinterpret_cast<cudaEvent_t>(ev_end);
    auto mark = [&](cudaEvent_t ev) -> cudaError_t { return ev != nullptr ? cudaEventRecord(ev, (cudaStream_t)stream) : cudaSuccess; };
    if (dec != nullptr) {
        a.k_rope = static_cast<const uint8_t *>(dec->k_rope) + (int64_t)layer * Hs * cache->slots * dec->d_rope * e;
        a.q_rope = dec->q_rope;
        a.d_rope = dec->d_rope;
    }
    if (window != nullptr) {
        // window planes [L][seqs][H][T][w_max][d]: select the layer
        const int64_t plane = (int64_t)window->seqs * dims->H * dims->T * window->w_max * dims->d_head * e;
        a.win_k = window->w_max > 0 ? static_cast<const uint8_t *>(window->k) + layer * plane : nullptr;
        a.win_v = window->w_max > 0 ? static_cast<const uint8_t *>(window->v) + layer * plane : nullptr;
        a.win_len = window->len;
        a.w_max = window->w_max;
        a.win_part = reinterpret_cast<float *>(ws + plan.off_win);
    }

    a.Tq_all = Tq;
    a.tq_off = 0;
    cudaStream_t s = (cudaStream_t)stream;
    // every check has passed: only now is anything queued on the caller's stream
    if (clear_status && cudaMemsetAsync(workspace, 0, sizeof(int32_t), s) != cudaSuccess)
        return LLA_ERR_CUDA;
    cudaError_t err = cudaSuccess;
    // hybrid form: the window pass runs after the decode grid, before the combine
    auto window_pass = [&](const DecodeArgs &ac) -> cudaError_t {
        return window != nullptr ? launch_decode_window(ac, dims->dtype, s) : cudaSuccess;
    };
    if (variant == LLA_RECONSTRUCT &&
        decode_recon_tc_supported(dims->dtype, dims->r_k, dims->r_v, dims->d_head, dims->fold, B, rope != nullptr)) {
        // tensor-memory kernel: one pass over the latents per (up to 4) loop queries
        const int per = decode_recon_tc_loops_per_pass();
        for (int32_t c = 0; c < Tq && err == cudaSuccess; c += per) {
            DecodeArgs ac = a;
            ac.tq_off = c;
            ac.Tq = Tq - c < per ? Tq - c : per;
            err = mark(c == 0 ? e0 : nullptr);
            if (err == cudaSuccess)
                err = launch_decode_recon_tc(ac, s);
            if (err == cudaSuccess && c + per >= Tq)
                err = mark(e1);
        }
        if (err == cudaSuccess)
            err = window_pass(a);
        if (err == cudaSuccess)
            err = launch_decode_combine(a, dims->dtype, dims->out_dtype, s);
        return err == cudaSuccess ? LLA_OK : LLA_ERR_CUDA;
    }
    if (variant == LLA_RECONSTRUCT) {
        // one pass over the latents per loop query, then one merge of all records
        for (int32_t c = 0; c < Tq && err == cudaSuccess; ++c) {
            DecodeArgs ac = a;
            ac.tq_off = c;
            ac.Tq = 1;
            err = mark(c == 0 ? e0 : nullptr);
            if (err == cudaSuccess)
                err = launch_decode_reconstruct(ac, s);
            if (err == cudaSuccess && c == Tq - 1)
                err = mark(e1);
        }
        if (err == cudaSuccess)
            err = window_pass(a);
        if (err == cudaSuccess)
            err = launch_decode_combine(a, dims->dtype, dims->out_dtype, s);
        return err == cudaSuccess ? LLA_OK : LLA_ERR_CUDA;
    }
    if (decode_mma2d_supported(dims->dtype, dims->r_k, dims->r_v, dims->fold, dims->H)) {
        // LLA-2D: all heads of a sequence share each latent tile; passes of H * loops <= 64
        // query rows
        const int per = decode_mma2d_loops_per_pass(dims->H);
        for (int32_t c = 0; c < Tq && err == cudaSuccess; c += per) {
            DecodeArgs ac = a;
            ac.tq_off = c;
            ac.Tq = Tq - c < per ? Tq - c : per;
            err = launch_absorb_prologue(ac, dims->dtype, s);
            if (err == cudaSuccess && c == 0)
                err = mark(e0);
            if (err == cudaSuccess)
                err = launch_decode_absorb_2d(ac, s);
            if (err == cudaSuccess && c + per >= Tq)
                err = mark(e1);
            if (err == cudaSuccess)
                err = window_pass(ac);
            if (err == cudaSuccess)
                err = launch_decode_combine(ac, dims->dtype, dims->out_dtype, s);
        }
        return err == cudaSuccess ? LLA_OK : LLA_ERR_CUDA;
    }
    if (use_mma) {
        // tensor-core kernel: up to 32 loop queries (two m16 row tiles) per pass over the latents
        const int per = decode_mma_loops_per_pass(a.d_rope);
        for (int32_t c = 0; c < Tq && err == cudaSuccess; c += per) {
            DecodeArgs ac = a;
            ac.tq_off = c;
            ac.Tq = Tq - c < per ? Tq - c : per;
            err = launch_absorb_prologue(ac, dims->dtype, s);
            if (err == cudaSuccess && c == 0)
                err = mark(e0);
            if (err == cudaSuccess)
                err = launch_decode_absorb_mma(ac, 0, s);
            if (err == cudaSuccess && c + per >= Tq)
                err = mark(e1);
            if (err == cudaSuccess)
                err = window_pass(ac);
            if (err == cudaSuccess)
                err = launch_decode_combine(ac, dims->dtype, dims->out_dtype, s);
        }
        return err == cudaSuccess ? LLA_OK : LLA_ERR_CUDA;
    }
    // The CUDA-core kernel serves up to 4 loop queries per pass over the latents.
    for (int32_t c = 0; c < Tq && err == cudaSuccess; c += 4) {
        DecodeArgs ac = a;
        ac.tq_off = c;
        ac.Tq = Tq - c < 4 ? Tq - c : 4;
        err = launch_absorb_prologue(ac, dims->dtype, s);
        bool supported = false;
        if (err == cudaSuccess && c == 0)
            err = mark(e0);
        if (err == cudaSuccess)
            err = launch_decode_absorb(ac, dims->dtype, 0, s, &supported);
        if (err == cudaSuccess && c + 4 >= Tq)
            err = mark(e1);
        if (!supported)
            return LLA_ERR_UNSUPPORTED;
        if (err == cudaSuccess)
            err = window_pass(ac);
        if (err == cudaSuccess)
            err = launch_decode_combine(ac, dims->dtype, dims->out_dtype, s);
    }
    return err == cudaSuccess ? LLA_OK : LLA_ERR_CUDA;
}

} // namespace

int lla::decode_attn_clearing_status(const lla_dims *dims, int32_t layer, int32_t t0, int32_t Tq, const void *q,
                                     const lla_cache *cache, const int64_t *seq_start, const int32_t *ctx_lens,
                                     int32_t B, int32_t max_ctx, const lla_codec *codec, float softmax_scale,
                                     int32_t variant, int32_t num_splits, void *out, float *lse, void *workspace,
                                     size_t ws_bytes, lla_stream_t stream)
{
    return decode_call(dims, layer, t0, Tq, q, cache, seq_start, ctx_lens, B, max_ctx, codec, nullptr, nullptr,
                       softmax_scale, variant, num_splits, out, lse, workspace, ws_bytes, stream, nullptr, nullptr,
                       nullptr, true);
}

extern "C" {

int lla_decode_attn(const lla_dims *dims, int32_t layer, int32_t t0, int32_t Tq, const void *q,
                    const lla_cache *cache, const int64_t *seq_start, const int32_t *ctx_lens, int32_t B,
                    int32_t max_ctx, const lla_codec *codec, float softmax_scale, int32_t variant,
                    int32_t num_splits, void *out, float *lse, void *workspace, size_t ws_bytes,
                    lla_stream_t stream)
{
    return decode_call(dims, layer, t0, Tq, q, cache, seq_start, ctx_lens, B, max_ctx, codec, nullptr,
                       nullptr, softmax_scale, variant, num_splits, out, lse, workspace, ws_bytes, stream);
}

int lla_decode_attn_rope(const lla_dims *dims, int32_t layer, int32_t t0, int32_t Tq, const void *q,
                         const lla_cache *cache, const int64_t *seq_start, const int32_t *ctx_lens, int32_t B,
                         int32_t max_ctx, const lla_codec *codec, const lla_rope *rope, float softmax_scale,
                         int32_t num_splits, void *out, float *lse, void *workspace, size_t ws_bytes,
                         lla_stream_t stream)
{
    if (rope == nullptr)
        return LLA_ERR_INVALID;
    return decode_call(dims, layer, t0, Tq, q, cache, seq_start, ctx_lens, B, max_ctx, codec, nullptr, rope,
                       softmax_scale, LLA_RECONSTRUCT, num_splits, out, lse, workspace, ws_bytes, stream);
}

int lla_decode_attn_timed(const lla_dims *dims, int32_t layer, int32_t t0, int32_t Tq, const void *q,
                          const lla_cache *cache, const int64_t *seq_start, const int32_t *ctx_lens, int32_t B,
                          int32_t max_ctx, const lla_codec *codec, float softmax_scale, int32_t variant,
                          int32_t num_splits, void *out, float *lse, void *workspace, size_t ws_bytes,
                          lla_stream_t stream, lla_event_t ev_start, lla_event_t ev_end)
{
    if (ev_start == nullptr || ev_end == nullptr)
        return LLA_ERR_INVALID;
    return decode_call(dims, layer, t0, Tq, q, cache, seq_start, ctx_lens, B, max_ctx, codec, nullptr, nullptr,
                       softmax_scale, variant, num_splits, out, lse, workspace, ws_bytes, stream, nullptr, ev_start,
                       ev_end);
}

int lla_decode_attn_hybrid(const lla_dims *dims, int32_t layer, int32_t t0, int32_t Tq, const void *q,
                           const lla_cache *cache, const int64_t *seq_start, const int32_t *ctx_lens,
                           int32_t B, int32_t max_ctx, const lla_codec *codec, const lla_window *window,
                           float softmax_scale, int32_t variant, int32_t num_splits, void *out, float *lse,
                           void *workspace, size_t ws_bytes, lla_stream_t stream)
{
    if (window == nullptr)
        return LLA_ERR_INVALID;
    return decode_call(dims, layer, t0, Tq, q, cache, seq_start, ctx_lens, B, max_ctx, codec, window, nullptr,
                       softmax_scale, variant, num_splits, out, lse, workspace, ws_bytes, stream);
}

int lla_decode_attn_decoupled(const lla_dims *dims, int32_t layer, int32_t t0, int32_t Tq, const void *q,
                              const lla_cache *cache, const int64_t *seq_start, const int32_t *ctx_lens, int32_t B,
                              int32_t max_ctx, const lla_codec *codec, const lla_decoupled *dec,
                              const lla_rope *rope, float softmax_scale, int32_t num_splits, void *out, float *lse,
                              void *workspace, size_t ws_bytes, lla_stream_t stream)
{
    if (dec == nullptr || rope == nullptr)
        return LLA_ERR_INVALID;
    return decode_call(dims, layer, t0, Tq, q, cache, seq_start, ctx_lens, B, max_ctx, codec, nullptr, rope,
                       softmax_scale, LLA_ABSORB, num_splits, out, lse, workspace, ws_bytes, stream, dec);
}

size_t lla_decode_decoupled_workspace_bytes(const lla_dims *dims, int32_t B, int32_t Tq, int32_t max_ctx,
                                            int32_t d_rope, int32_t num_splits)
{
    if (d_rope <= 0 || lla_decode_num_splits(dims, B, Tq, max_ctx, LLA_ABSORB, num_splits) < 1)
        return 0;
    return make_plan(dims, B, Tq, max_ctx, num_splits, LLA_ABSORB, false, d_rope).bytes;
}

size_t lla_decode_hybrid_workspace_bytes(const lla_dims *dims, int32_t B, int32_t Tq, int32_t max_ctx,
                                         int32_t variant, int32_t num_splits)
{
    if (lla_decode_num_splits(dims, B, Tq, max_ctx, variant, num_splits) < 1)
        return 0;
    return make_plan(dims, B, Tq, max_ctx, num_splits, variant, true).bytes;
}

int lla_status_fetch(void *workspace, lla_stream_t stream, int32_t *status_host)
{
    if (status_host == nullptr)
        return LLA_ERR_INVALID;
    if (workspace == nullptr) { // the encode kernels' status word of the current device
        workspace = encode_status_address();
        if (workspace == nullptr)
            return LLA_ERR_CUDA;
    }
    cudaStream_t s = (cudaStream_t)stream;
    int32_t v = 0;
    if (cudaMemcpyAsync(&v, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return LLA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess)
        return LLA_ERR_CUDA;
    if (cudaMemsetAsync(workspace, 0, sizeof(int32_t), s) != cudaSuccess)
        return LLA_ERR_CUDA;
    *status_host = v;
    return LLA_OK;
}

} // extern "C"
