// encode_simt.cu -- LLA write path on CUDA cores (fp32 storage), and the encode bias.
//
// "Looped Latent Attention: Cross-Loop KV Compression for Looped Transformers",
// Pith review page, "What carries the argument", Eq. 2: the T per-loop vectors of a
// (token, layer, head, axis) are stacked and centred, then projected to the latent
// c = (x - mu) W_down.  Written as c = x W_down + b with b = -mu W_down.
//
// The fp32 path keeps fp32 end to end (tf32 tensor cores would round the inputs to
// 10 mantissa bits), so it is a tiled SIMT GEMM: a CTA computes a 32-token x r tile
// for one (layer, head', axis), staging 32-wide K slices of x and W_down^T in shared
// memory.  The bf16 path runs on tcgen05 tensor cores (encode_tc.cu).
#include "encode.cuh"

namespace lla {
namespace {

constexpr int kEncThreads = 128;
constexpr int kEncM = 32;  // tokens per CTA
constexpr int kEncK = 32;  // K slice

// x element (token i, stacked index kk) of stored head hs for layer-slot li.
template <typename T>
__device__ __forceinline__ float load_x(const EncodeArgs &a, const T *x, int li, int64_t i, int hs,
                                        int kk)
{
    if (a.fold) // LLA-2D: the stacked row is x[li][i][T][H][d] itself
        return Elem<T>::to_f(x[((int64_t)li * a.n_tok + i) * a.W + kk]);
    const int t = kk / a.d, dd = kk - t * a.d;
    return Elem<T>::to_f(x[(((int64_t)li * a.n_tok + i) * a.T + t) * a.H * a.d + (int64_t)hs * a.d + dd]);
}

template <typename T>
__global__ void __launch_bounds__(kEncThreads) encode_simt_kernel(const EncodeArgs a)
{
    // grid: x = token tile, y = stored head, z = layer-slot * 2 + axis
    extern __shared__ float esm[];
    float *xs = esm;                        // [kEncM][kEncK + 1]
    float *ws = xs + kEncM * (kEncK + 1);   // [r_max][kEncK + 1]
    const int hs = blockIdx.y, li = blockIdx.z >> 1, axis = blockIdx.z & 1;
    const int l = a.layer0 + li;
    const int r = axis ? a.r_v : a.r_k;
    const T *x = static_cast<const T *>(axis ? a.x_v : a.x_k);
    const T *Wd = static_cast<const T *>(axis ? a.W_down_v : a.W_down_k) +
                  ((int64_t)l * a.Hs + hs) * r * a.W;
    const float *bias = (axis ? a.bias_v : a.bias_k) + ((int64_t)l * a.Hs + hs) * r;
    T *plane = static_cast<T *>(axis ? a.cache_v : a.cache_k) + ((int64_t)l * a.Hs + hs) * a.slots * r;
    const int64_t i0 = (int64_t)blockIdx.x * kEncM;
    const int tid = threadIdx.x;
    // thread -> (token row tr, output columns j = jc, jc + 4, ...)
    const int tr = tid >> 2, jc = tid & 3;
    float acc[64];
    const int nj = (r - jc + 3) / 4;
#pragma unroll
    for (int q = 0; q < 64; ++q)
        acc[q] = 0.f;
    for (int k0 = 0; k0 < a.W; k0 += kEncK) {
        for (int e = tid; e < kEncM * kEncK; e += kEncThreads) {
            const int ii = e / kEncK, kk = e % kEncK;
            const int64_t i = i0 + ii;
            xs[ii * (kEncK + 1) + kk] =
                (i < a.n_tok && k0 + kk < a.W) ? load_x<T>(a, x, li, i, hs, k0 + kk) : 0.f;
        }
        for (int e = tid; e < r * kEncK; e += kEncThreads) {
            const int j = e / kEncK, kk = e % kEncK;
            ws[j * (kEncK + 1) + kk] =
                (k0 + kk < a.W) ? Elem<T>::to_f(Wd[(int64_t)j * a.W + k0 + kk]) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int kk = 0; kk < kEncK; ++kk) {
            const float xv = xs[tr * (kEncK + 1) + kk];
#pragma unroll
            for (int q = 0; q < 64; ++q)
                if (q < nj)
                    acc[q] = fmaf(xv, ws[(jc + 4 * q) * (kEncK + 1) + kk], acc[q]);
        }
        __syncthreads();
    }
    const int64_t i = i0 + tr;
    if (i < a.n_tok) {
        const int64_t slot = a.slot_idx[i];
        if (slot >= 0 && slot < a.slots) {
#pragma unroll
            for (int q = 0; q < 64; ++q)
                if (q < nj)
                    plane[slot * r + jc + 4 * q] = Elem<T>::from_f(acc[q] + bias[jc + 4 * q]);
        }
    }
}

// b[l][h'][j] = -sum_k mu[l][h'][k] W_down[l][h'][j][k], fp64 accumulation.  One warp
// per output.
template <typename T>
__global__ void codec_bias_kernel(const T *Wd, const float *mu, float *bias, int64_t n_out, int r,
                                  int W)
{
    const int64_t o = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (o >= n_out)
        return;
    const int64_t g = o / r; // (layer, head') group
    const int j = (int)(o - g * r);
    const T *w = Wd + (g * r + j) * W;
    const float *m = mu + g * W;
    double acc = 0.0;
    for (int k = lane; k < W; k += 32)
        acc += (double)m[k] * (double)Elem<T>::to_f(w[k]);
    for (int off = 16; off > 0; off >>= 1)
        acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0)
        bias[o] = (float)(-acc);
}

} // namespace

cudaError_t launch_encode_simt(const EncodeArgs &a, int dtype, cudaStream_t stream)
{
    const int r_max = a.r_k > a.r_v ? a.r_k : a.r_v;
    if (r_max > 256)
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(float) * (size_t)(kEncM + r_max) * (kEncK + 1);
    dim3 grid((unsigned)((a.n_tok + kEncM - 1) / kEncM), a.Hs, a.n_layers * 2);
    if (dtype == LLA_BF16) {
        auto k = encode_simt_kernel<__nv_bfloat16>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<grid, kEncThreads, smem, stream>>>(a);
    } else {
        auto k = encode_simt_kernel<float>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<grid, kEncThreads, smem, stream>>>(a);
    }
    return cudaGetLastError();
}

cudaError_t launch_codec_bias(const void *Wd, const float *mu, float *bias, int64_t groups, int r, int W,
                              int dtype, cudaStream_t stream)
{
    const int64_t n_out = groups * r;
    const int threads = 256;
    const int64_t blocks = (n_out * 32 + threads - 1) / threads;
    if (dtype == LLA_BF16)
        codec_bias_kernel<__nv_bfloat16><<<(unsigned)blocks, threads, 0, stream>>>(
            static_cast<const __nv_bfloat16 *>(Wd), mu, bias, n_out, r, W);
    else
        codec_bias_kernel<float><<<(unsigned)blocks, threads, 0, stream>>>(static_cast<const float *>(Wd),
                                                                          mu, bias, n_out, r, W);
    return cudaGetLastError();
}

} // namespace lla
