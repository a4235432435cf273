// decode.cuh -- shared declarations of the LLA decode kernels.
#pragma once

#include "common.cuh"

namespace lla {

// Arguments of one decode pass for one layer (pointers already offset to the layer).
struct DecodeArgs {
    const void *q;            // T [B][Tq_all][H][d]
    const void *k;            // T [H'][slots][r_k]
    const void *v;            // T [H'][slots][r_v]
    int64_t slots;
    const int64_t *seq_start; // [B]
    const int32_t *ctx_lens;  // [B]
    const float *W_up_k;      // [H'][T][r_k][D']
    const float *mu_k;        // [H'][T][D']
    const float *W_up_v;      // [H'][T][r_v][D']
    const float *mu_v;        // [H'][T][D']
    int32_t B, H, d, T, t0, Tq, fold, r_k, r_v;
    int32_t Tq_all, tq_off;   // q/out/lse/records hold Tq_all loop queries; this pass
                              // serves queries tq_off .. tq_off+Tq-1 (loop t0 + tq_off + i)
    int32_t recon;            // records hold d-wide reconstruct-form outputs (no projection)
    int32_t seg_max;          // partial-record slots per (unit, query)
    int32_t chunk_min;        // smallest token share of one decode CTA
    float scale;              // softmax scale
    float *qt;                // [B*H][Tq_all][r_k] absorbed queries, pre-scaled by log2(e)
    int32_t *counts;          // [B*H] partial records written for each unit by this pass
    float *part;              // [B*H][Tq_all][seg_max][r_v + 4] partial records
    int32_t *status;          // sticky device status word
    void *out;                // O [B][Tq_all][H][d] (O = out_dtype)
    float *lse;               // [B][Tq_all][H] or null
    // hybrid form: exact loop keys / values of each sequence's window tokens
    const void *win_k;        // T [B][H][T][w_max][d] (layer already selected) or null
    const void *win_v;        // T [B][H][T][w_max][d]
    const int32_t *win_len;   // [B] window rows in use
    int32_t w_max;
    float *win_part;          // [B*H][Tq_all][d + 4] window output and lse (log2 units);
                              // null: no window, the combine writes the latent result alone
    // faithful read (reconstruct form only): rotary embedding after reconstruction
    const int32_t *q_pos;     // [B] query position of each sequence; null: no rotation
    float rope_base;          // pair i turns by pos * rope_base^(-2i/d)
    int32_t rope_style;       // LLA_ROPE_HALF or LLA_ROPE_INTERLEAVED
    // decoupled rotary sub-key beside the latent (absorbed form, tensor-core kernel)
    const void *k_rope;       // T [H'][slots][d_rope], stored rotated at each token's position
    const void *q_rope;       // T [B][Tq_all][H][d_rope], rotated at q_pos by the prologue
    int32_t d_rope;           // 0: none; q_tilde rows then hold r_k + d_rope values
    int32_t serial;           // launch every grid without programmatic overlap (timing aid)
};

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Partial record stride (floats) for value rank r_v: acc[r_v], m, l, 2 pad.
__host__ __device__ constexpr int part_stride(int r_v) { return r_v + 4; }

// Decode CTAs resident per SM that the persistent kernel is shaped for.
constexpr int kDecodeCtasPerSm = 4;

cudaError_t launch_decode_absorb(const DecodeArgs &a, int dtype, int ctas, cudaStream_t stream,
                                 bool *supported);
cudaError_t launch_absorb_prologue(const DecodeArgs &a, int dtype, cudaStream_t stream);
cudaError_t launch_decode_combine(const DecodeArgs &a, int dtype, int out_dtype, cudaStream_t stream);
bool decode_absorb_supported(int dtype, int r_k, int r_v, int d, int fold);
bool decode_mma_supported(int dtype, int r_k, int r_v, int fold, int Tq);
// loop queries one pass of the tensor-core kernel serves (two m16 row tiles; 16 with a
// decoupled rotary sub-key)
int decode_mma_loops_per_pass(int d_rope);
bool decode_mma_rope_supported(int dtype, int r_k, int r_v, int d_rope, int fold);
cudaError_t launch_decode_absorb_mma(const DecodeArgs &a, int ctas, cudaStream_t stream);
bool decode_reconstruct_supported(int dtype, int r_k, int r_v, int d);
// LLA-2D: every latent tile read once for all heads of a sequence (H * loops <= 64 rows
// per pass); records in the per-(sequence, head) layout of the other kernels.
bool decode_mma2d_supported(int dtype, int r_k, int r_v, int fold, int H);
int decode_mma2d_loops_per_pass(int H);
cudaError_t launch_decode_absorb_2d(const DecodeArgs &a, cudaStream_t stream);
cudaError_t launch_decode_reconstruct(const DecodeArgs &a, cudaStream_t stream);
// Reconstruct form on tcgen05 tensor cores: one latent read serves up to
// decode_recon_tc_loops_per_pass() loop queries (a.Tq per launch); d = 128, bf16.
bool decode_recon_tc_supported(int dtype, int r_k, int r_v, int d, int fold, int B, bool rope);
int decode_recon_tc_loops_per_pass();
int decode_recon_tc_smem_bytes(int r_k, int r_v, bool rope, int lp, int B);
cudaError_t launch_decode_recon_tc(const DecodeArgs &a, cudaStream_t stream);
// Hybrid form: attention of every loop query over its exact window rows, written to
// a.win_part for the combine to merge (launched between the decode and the combine).
bool decode_window_supported(int dtype, int d);
cudaError_t launch_decode_window(const DecodeArgs &a, int dtype, cudaStream_t stream);

// lla_decode_attn that, once its arguments have passed every check, clears the first
// word of `workspace` (the sticky device status) on `stream` before its launches; a
// refused call queues nothing.
int decode_attn_clearing_status(const lla_dims *dims, int32_t layer, int32_t t0, int32_t Tq, const void *q,
                                const lla_cache *cache, const int64_t *seq_start, const int32_t *ctx_lens,
                                int32_t B, int32_t max_ctx, const lla_codec *codec, float softmax_scale,
                                int32_t variant, int32_t num_splits, void *out, float *lse, void *workspace,
                                size_t ws_bytes, lla_stream_t stream);

} // namespace lla
