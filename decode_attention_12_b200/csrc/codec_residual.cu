// codec_residual.cu -- per-token reconstruction residual of the cross-loop codec.
//
// "Looped Latent Attention: Cross-Loop KV Compression for Looped Transformers", Pith
// verdict record: the skeptic's concrete test measures, on held-out tokens,
//     ||x - ((x - mu) W_down) W_up^T - mu|| / ||x||,
// i.e. how much of a token's stacked T-loop trajectory the shared codec loses (Eq. 2 then
// Eq. 3 for every loop).  This kernel returns err = ||x - x_hat|| and norm = ||x|| for
// every (layer, token, stored head) of a batch laid out like the encode input.
//
// Both products are dense contractions over a batch of tokens, so both run on tensor
// cores (warp-level MMAs):
//   pass 1  c [16 x r] = X [16 x W] . W_down [W x r] + b    bf16 m16n8k16, exact products
//           (x and W_down are stored bf16), fp32 accumulation; b = -mu W_down (fp32).
//   pass 2  x_hat [16 x W] = c . W_up [r x W] + mu          3xTF32 m16n8k8 (hi/lo parts of
//           c and of the fp32 W_up), so the rebuild keeps fp32 accuracy; the epilogue
//           accumulates (x - x_hat)^2 and x^2 per token.
// One CTA = 4 warps = 64 tokens of one (layer, stored head); each warp owns 16 tokens.
// The stacked vector is walked in 64-column chunks (a chunk never crosses a loop block,
// since the loop width is a multiple of 64), staged with 16-byte cp.async into XOR-
// swizzled shared memory (X and W_down, 128-byte rows) or padded rows (W_up, fp32),
// double-buffered when the rank leaves room.  Pass 2 reads X again; for the per-head
// stack (W = T d) the CTA's 64 KB tile is still in L2.
#include <climits>

#include "encode.cuh"
#include "mma_common.cuh"

namespace lla {
namespace {
using namespace mma;

constexpr int kResWarps = 4;
constexpr int kResThreads = 32 * kResWarps;
constexpr int kResTok = 16 * kResWarps; // tokens per CTA
constexpr int kChunk = 64;              // stacked-vector columns per chunk

template <int R> struct ResCfg {
    static constexpr int STAGES = R <= 64 ? 2 : 1;
    static constexpr int X_BYTES = kResTok * kChunk * 2;    // bf16, 128-byte rows
    static constexpr int WD_BYTES = R * kChunk * 2;         // bf16, 128-byte rows
    static constexpr int WU_LD = kChunk + 8;                // fp32 row stride (bank spread)
    static constexpr int WU_BYTES = R * WU_LD * 4;
    static constexpr int MU_BYTES = kChunk * 4;
    static constexpr int P1 = X_BYTES + WD_BYTES;           // one pass-1 stage
    static constexpr int P2 = X_BYTES + WU_BYTES + MU_BYTES; // one pass-2 stage
    static constexpr int STAGE = P1 > P2 ? P1 : P2;
    static constexpr int CS_LD = R + 4;                     // fp32 row stride of c
    static constexpr int CS_OFF = STAGES * STAGE;
    static constexpr int SMEM = CS_OFF + kResWarps * 16 * CS_LD * 4;
};

struct ResArgs {
    const __nv_bfloat16 *x;  // [n_layers][n_tok][T][H][d]
    const __nv_bfloat16 *Wd; // [L][H'][R][W] (layer already selected by layer0 below)
    const float *bias;       // [L][H'][R]
    const float *Wu;         // [L][H'][T][R][Dp]
    const float *mu;         // [L][H'][T][Dp]
    float *err, *norm;       // [n_layers][n_tok][H']
    int64_t n_tok;
    int32_t layer0, T, H, d, Dp, Hs, W, fold;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint32_t to_tf32(float x)
{
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void split_tf32(float x, uint32_t &hi, uint32_t &lo)
{
    hi = to_tf32(x);
    lo = to_tf32(x - __uint_as_float(hi));
}
__device__ __forceinline__ void mma1688(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                 "{%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of 16-byte chunk q of row r in a 128-byte-row swizzled tile.
__device__ __forceinline__ uint32_t swz(int r, int q) { return (uint32_t)(r * 128 + ((q ^ (r & 7)) << 4)); }

template <int R>
__global__ void __launch_bounds__(kResThreads) codec_residual_kernel(const ResArgs a)
{
    using C = ResCfg<R>;
    extern __shared__ __align__(128) uint8_t rsm[];
    const uint32_t sb = smem_u32(rsm);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, tq = lane & 3;
    const int64_t i0 = (int64_t)blockIdx.x * kResTok;
    const int hs = blockIdx.y, l = blockIdx.z;
    const int64_t grp = (int64_t)(a.layer0 + l) * a.Hs + hs; // codec group (layer, stored head)
    const __nv_bfloat16 *Wd = a.Wd + grp * R * a.W;
    const float *bias = a.bias + grp * R;
    const float *Wu = a.Wu + grp * a.T * R * a.Dp;
    const float *mu = a.mu + grp * a.W;
    const int NQ = a.W / kChunk;

    // global element offset of stacked column c of token i (chunks never cross a loop block)
    auto x_off = [&](int64_t i, int c) -> int64_t {
        const int t = c / a.Dp, k = c - t * a.Dp;
        return (((int64_t)l * a.n_tok + i) * a.T + t) * a.H * a.d + (a.fold ? 0 : hs * a.d) + k;
    };
    auto stage_x = [&](uint32_t dst, int c0) {
        for (int e = tid; e < kResTok * 8; e += kResThreads) {
            const int r = e >> 3, q = e & 7;
            const int64_t i = i0 + r;
            const bool ok = i < a.n_tok;
            cp_async16(dst + swz(r, q), a.x + x_off(ok ? i : 0, c0 + 8 * q), ok);
        }
    };
    auto stage_pass1 = [&](int st, int qc) {
        const uint32_t base = sb + st * C::STAGE;
        stage_x(base, qc * kChunk);
        for (int e = tid; e < R * 8; e += kResThreads) {
            const int j = e >> 3, q = e & 7;
            cp_async16(base + C::X_BYTES + swz(j, q), Wd + (int64_t)j * a.W + qc * kChunk + 8 * q, true);
        }
        cp_async_commit();
    };
    auto stage_pass2 = [&](int st, int qc) {
        const uint32_t base = sb + st * C::STAGE;
        const int c0 = qc * kChunk, t = c0 / a.Dp, k0 = c0 - t * a.Dp;
        stage_x(base, c0);
        const float *wu = Wu + (int64_t)t * R * a.Dp + k0;
        for (int e = tid; e < R * 16; e += kResThreads) {
            const int j = e >> 4, q = e & 15;
            cp_async16(base + C::X_BYTES + (j * C::WU_LD + 4 * q) * 4, wu + (int64_t)j * a.Dp + 4 * q, true);
        }
        if (tid < 16)
            cp_async16(base + C::X_BYTES + C::WU_BYTES + 16 * tid, mu + c0 + 4 * tid, true);
        cp_async_commit();
    };
    // waits for chunk qc's stage (and issues the next one first when double-buffered)
    auto pipeline_step = [&](int qc, auto &&stage) {
        if (C::STAGES == 2 && qc + 1 < NQ) {
            stage((qc + 1) & 1, qc + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
    };

    // ---- pass 1: c = X W_down (+ b)
    constexpr int NT = R / 8;
    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
        acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    stage_pass1(0, 0);
    for (int qc = 0; qc < NQ; ++qc) {
        pipeline_step(qc, stage_pass1);
        const uint32_t xs = sb + (C::STAGES == 2 ? (qc & 1) : 0) * C::STAGE, ws = xs + C::X_BYTES;
#pragma unroll
        for (int ks = 0; ks < kChunk / 16; ++ks) {
            uint32_t af[4];
            ldsm_x4(xs + swz(16 * warp + (lane & 15), 2 * ks + (lane >> 4)), af);
#pragma unroll
            for (int n2 = 0; n2 < NT / 2; ++n2) {
                uint32_t bf[4];
                ldsm_x4(ws + swz(16 * n2 + ((lane >> 4) << 3) + (lane & 7), 2 * ks + ((lane >> 3) & 1)), bf);
                mma16816(acc[2 * n2], af[0], af[1], af[2], af[3], bf[0], bf[1]);
                mma16816(acc[2 * n2 + 1], af[0], af[1], af[2], af[3], bf[2], bf[3]);
            }
        }
        __syncthreads(); // stage reusable
        if (C::STAGES == 1 && qc + 1 < NQ)
            stage_pass1(0, qc + 1);
    }
    float *cs = reinterpret_cast<float *>(rsm + C::CS_OFF) + warp * 16 * C::CS_LD;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const int j = 8 * n + 2 * tq;
        const float b0 = bias[j], b1 = bias[j + 1];
        cs[g * C::CS_LD + j] = acc[n][0] + b0;
        cs[g * C::CS_LD + j + 1] = acc[n][1] + b1;
        cs[(g + 8) * C::CS_LD + j] = acc[n][2] + b0;
        cs[(g + 8) * C::CS_LD + j + 1] = acc[n][3] + b1;
    }
    __syncwarp();

    // ---- pass 2: x_hat = c W_up + mu, residual and norm per token
    float e2[2] = {0.f, 0.f}, n2s[2] = {0.f, 0.f};
    stage_pass2(0, 0);
    for (int qc = 0; qc < NQ; ++qc) {
        pipeline_step(qc, stage_pass2);
        const uint32_t xs = sb + (C::STAGES == 2 ? (qc & 1) : 0) * C::STAGE;
        const uint8_t *xg = rsm + (xs - sb);
        const float *wu = reinterpret_cast<const float *>(xg + C::X_BYTES);
        const float *mus = reinterpret_cast<const float *>(xg + C::X_BYTES + C::WU_BYTES);
        float o[8][4];
#pragma unroll
        for (int n = 0; n < 8; ++n)
            o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
#pragma unroll 2
        for (int ks = 0; ks < R / 8; ++ks) {
            uint32_t ah[4], al[4];
            split_tf32(cs[g * C::CS_LD + 8 * ks + tq], ah[0], al[0]);
            split_tf32(cs[(g + 8) * C::CS_LD + 8 * ks + tq], ah[1], al[1]);
            split_tf32(cs[g * C::CS_LD + 8 * ks + tq + 4], ah[2], al[2]);
            split_tf32(cs[(g + 8) * C::CS_LD + 8 * ks + tq + 4], ah[3], al[3]);
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                uint32_t bh0, bl0, bh1, bl1;
                split_tf32(wu[(8 * ks + tq) * C::WU_LD + 8 * n + g], bh0, bl0);
                split_tf32(wu[(8 * ks + tq + 4) * C::WU_LD + 8 * n + g], bh1, bl1);
                mma1688(o[n], ah, bh0, bh1);
                mma1688(o[n], ah, bl0, bl1);
                mma1688(o[n], al, bh0, bh1);
            }
        }
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            const int c = 8 * n + 2 * tq;
#pragma unroll
            for (int hrow = 0; hrow < 2; ++hrow) {
                const int r = 16 * warp + g + 8 * hrow;
                const uint32_t xv = *reinterpret_cast<const uint32_t *>(xg + swz(r, n) + 4 * tq);
                const float x0 = bf16_lo(xv), x1 = bf16_hi(xv);
                const float d0 = x0 - (o[n][2 * hrow] + mus[c]), d1 = x1 - (o[n][2 * hrow + 1] + mus[c + 1]);
                e2[hrow] = fmaf(d0, d0, fmaf(d1, d1, e2[hrow]));
                n2s[hrow] = fmaf(x0, x0, fmaf(x1, x1, n2s[hrow]));
            }
        }
        __syncthreads();
        if (C::STAGES == 1 && qc + 1 < NQ)
            stage_pass2(0, qc + 1);
    }
#pragma unroll
    for (int hrow = 0; hrow < 2; ++hrow) {
        e2[hrow] += __shfl_xor_sync(0xffffffffu, e2[hrow], 1);
        e2[hrow] += __shfl_xor_sync(0xffffffffu, e2[hrow], 2);
        n2s[hrow] += __shfl_xor_sync(0xffffffffu, n2s[hrow], 1);
        n2s[hrow] += __shfl_xor_sync(0xffffffffu, n2s[hrow], 2);
        const int64_t i = i0 + 16 * warp + g + 8 * hrow;
        if (tq == 0 && i < a.n_tok) {
            const int64_t o_idx = ((int64_t)l * a.n_tok + i) * a.Hs + hs;
            a.err[o_idx] = sqrtf(e2[hrow]);
            a.norm[o_idx] = sqrtf(n2s[hrow]);
        }
    }
}

template <int R> cudaError_t launch_res(const ResArgs &a, int n_layers, cudaStream_t stream)
{
    using C = ResCfg<R>;
    auto k = codec_residual_kernel<R>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess)
        return e;
    const dim3 grid((unsigned)((a.n_tok + kResTok - 1) / kResTok), (unsigned)a.Hs, (unsigned)n_layers);
    k<<<grid, kResThreads, C::SMEM, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_res_rank(const ResArgs &a, int r, int n_layers, cudaStream_t stream)
{
    switch (r) {
    case 16: return launch_res<16>(a, n_layers, stream);
    case 32: return launch_res<32>(a, n_layers, stream);
    case 64: return launch_res<64>(a, n_layers, stream);
    case 96: return launch_res<96>(a, n_layers, stream);
    case 128: return launch_res<128>(a, n_layers, stream);
    case 160: return launch_res<160>(a, n_layers, stream);
    default: return cudaErrorNotSupported;
    }
}

} // namespace

bool codec_residual_supported(int dtype, int r_k, int r_v, int Dp)
{
    auto rank_ok = [](int r) { return r == 16 || r == 32 || r == 64 || r == 96 || r == 128 || r == 160; };
    return dtype == LLA_BF16 && rank_ok(r_k) && rank_ok(r_v) && Dp % kChunk == 0;
}

cudaError_t launch_codec_residual(const CodecResidualArgs &c, cudaStream_t stream)
{
    if (c.n_layers > 65535 || c.Hs > 65535 || (c.n_tok + kResTok - 1) / kResTok > INT32_MAX)
        return cudaErrorInvalidValue;
    for (int axis = 0; axis < 2; ++axis) {
        ResArgs a;
        a.x = static_cast<const __nv_bfloat16 *>(axis ? c.x_v : c.x_k);
        a.Wd = static_cast<const __nv_bfloat16 *>(axis ? c.W_down_v : c.W_down_k);
        a.bias = axis ? c.bias_v : c.bias_k;
        a.Wu = axis ? c.W_up_v : c.W_up_k;
        a.mu = axis ? c.mu_v : c.mu_k;
        a.err = axis ? c.err_v : c.err_k;
        a.norm = axis ? c.norm_v : c.norm_k;
        a.n_tok = c.n_tok;
        a.layer0 = c.layer0;
        a.T = c.T; a.H = c.H; a.d = c.d; a.Dp = c.Dp; a.Hs = c.Hs; a.W = c.W; a.fold = c.fold;
        const cudaError_t e = launch_res_rank(a, axis ? c.r_v : c.r_k, c.n_layers, stream);
        if (e != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

} // namespace lla
