// encode.cuh -- shared declarations of the LLA write-path kernels.
#pragma once

#include "common.cuh"

namespace lla {

struct EncodeArgs {
    const void *x_k, *x_v;         // T [n_layers][n_tok][T][H][d]
    const void *W_down_k, *W_down_v; // T [L][H'][r][W]
    const float *bias_k, *bias_v;  // [L][H'][r]
    void *cache_k, *cache_v;       // T [L][H'][slots][r]
    const int64_t *slot_idx;       // [n_tok]
    int64_t n_tok, slots;
    int32_t layer0, n_layers, T, H, d, Hs, W, r_k, r_v, fold;
};

cudaError_t launch_encode_simt(const EncodeArgs &a, int dtype, cudaStream_t stream);
bool encode_tc_supported(const EncodeArgs &a);
cudaError_t launch_encode_tc(const EncodeArgs &a, cudaStream_t stream);
void *encode_status_address(); // device address of the encode status word, current device
// Per-token reconstruction residual of the codec (lla_codec_residual).
struct CodecResidualArgs {
    const void *x_k, *x_v;             // bf16 [n_layers][n_tok][T][H][d]
    const void *W_down_k, *W_down_v;   // bf16 [L][H'][r][W]
    const float *bias_k, *bias_v;      // [L][H'][r]
    const float *W_up_k, *W_up_v;      // [L][H'][T][r][Dp]
    const float *mu_k, *mu_v;          // [L][H'][T][Dp]
    float *err_k, *norm_k, *err_v, *norm_v; // [n_layers][n_tok][H']
    int64_t n_tok;
    int32_t layer0, n_layers, T, H, d, Dp, Hs, W, fold, r_k, r_v;
};
bool codec_residual_supported(int dtype, int r_k, int r_v, int Dp);
cudaError_t launch_codec_residual(const CodecResidualArgs &a, cudaStream_t stream);

// SVD initialisation of the codec (lla_codec_fit).
struct CodecFitArgs {
    const void *x_k, *x_v;             // T [n_layers][n][T][H][d]
    void *W_down_k, *W_down_v;         // T [L][H'][r][W] (written)
    float *W_up_k, *W_up_v;            // [L][H'][T][r][Dp] (written)
    float *mu_k, *mu_v;                // [L][H'][T][Dp] (written)
    float *sigma_k, *sigma_v;          // [n_layers][H'][n] or null
    void *scratch;                     // codec_fit_scratch_bytes(...)
    int32_t *status;
    int64_t n;
    int32_t layer0, n_layers, T, H, d, Dp, Hs, W, fold, r_k, r_v, dtype;
};
size_t codec_fit_scratch_bytes(int64_t groups, int64_t n, int64_t W, int64_t r_max);
cudaError_t launch_codec_fit(const CodecFitArgs &a, cudaStream_t stream);

cudaError_t launch_codec_bias(const void *Wd, const float *mu, float *bias, int64_t groups, int r, int W,
                              int dtype, cudaStream_t stream);

} // namespace lla
