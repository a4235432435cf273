// decode_window.cu -- the exact-window half of hybrid latent attention.
//
// "Hybrid Latent Attention for Looped Language Models", abstract: the keys and values
// of the W most recent tokens are kept exact (one K_t, V_t pair per loop t, as in an
// uncompressed looped cache), older tokens live only as latents, and each loop query
// reads both.  With one softmax over the union, the output splits into two partial
// attentions merged by their log-sum-exp:
//     out = (e^{lse_lat} out_lat + e^{lse_win} out_win) / (e^{lse_lat} + e^{lse_win}).
// This kernel computes (out_win, lse_win) for every (sequence b, head h, loop query t)
// and writes them to the workspace; the combine kernel of the latent path merges them
// into its own result.
//
// Roofline: every window row is read exactly once (a loop-t key or value belongs to one
// query), so the kernel is a streaming read of 2 * len_b * d elements per unit, bound by
// HBM bandwidth; the dot products cost 2 flops per element read.  There is no operand
// reuse for tensor cores to exploit.
//
// Layout of the work: one CTA of 4 warps per unit.  A row of d elements is LPR 16-byte
// chunks held by LPR consecutive lanes (LPR = d * sizeof(T) / 16, rounded up to a power of
// two; lanes past the row's chunks idle), so one warp load instruction covers 32 / LPR
// whole rows.  Each lane group keeps its own online-softmax state (running max, sum and a
// chunk-wide accumulator, in log2 units); groups, then warps, are merged at the end.
//
// Launch position: after the decode grid and before the combine grid, with programmatic
// dependent launch.  The window inputs are the call's own, so CTAs start streaming as soon
// as decode CTAs leave SM slots free, filling the decode's tail.  Before exiting, every
// CTA waits for the decode grid, so the combine grid's own wait (on this grid) also covers
// the decode's records.
#include "decode.cuh"

namespace lla {
namespace {

constexpr int kWinWarps = 4;
constexpr int kWinThreads = 32 * kWinWarps;
constexpr int kWinUnroll = 2; // rows per lane group and block (x2 in flight: double buffered)

// Streaming 16-byte load: the data is read once, keep it out of L1.
__device__ __forceinline__ uint4 ld_stream_u4(const void *p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Folds the state (mo, lo, ao) into (m, l, acc); all in log2 units, m = -inf when empty.
template <int N>
__device__ __forceinline__ void merge_state(float &m, float &l, float (&acc)[N], float mo, float lo,
                                            const float (&ao)[N])
{
    const float mn = fmaxf(m, mo);
    if (mn == -INFINITY)
        return;
    const float a = exp2f(m - mn), b = exp2f(mo - mn); // exp2(-inf) = 0
    l = a * l + b * lo;
#pragma unroll
    for (int i = 0; i < N; ++i)
        acc[i] = a * acc[i] + b * ao[i];
    m = mn;
}

template <typename T, int LPR>
__global__ void __launch_bounds__(kWinThreads) decode_window_kernel(const DecodeArgs a)
{
    constexpr int N = Chunk<T>::N; // elements per 16-byte chunk
    constexpr int RPW = 32 / LPR;  // rows per warp load instruction
    constexpr int ROWS = kWinWarps * kWinUnroll * RPW;
    __shared__ float red[kWinWarps][2];
    extern __shared__ __align__(16) float wacc[]; // [kWinWarps][d]

    grid_launch_dependents(); // the combine grid may stage its own inputs meanwhile

    const int h = blockIdx.x, tl = blockIdx.y, b = blockIdx.z;
    const int t = a.tq_off + tl;
    const int tg = a.t0 + t;
    const int d = a.d;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane / LPR, sub = lane % LPR;
    const int chunks = d / N; // 16-byte chunks per row (<= LPR)
    const bool has_chunk = sub < chunks;
    const int len = min(max(a.win_len[b], 0), a.w_max);

    const int64_t unit_row0 = (((int64_t)b * a.H + h) * a.T + tg) * a.w_max;
    const T *K = static_cast<const T *>(a.win_k) + unit_row0 * d + sub * N;
    const T *V = static_cast<const T *>(a.win_v) + unit_row0 * d + sub * N;

    // this lane's query chunk, scaled into log2 units
    float qf[N];
    {
        const T *qrow = static_cast<const T *>(a.q) + (((int64_t)b * a.Tq_all + t) * a.H + h) * d;
        uint4 u = make_uint4(0u, 0u, 0u, 0u);
        if (has_chunk)
            u = *reinterpret_cast<const uint4 *>(qrow + sub * N);
        Chunk<T>::unpack(u, qf);
        const float s = a.scale * kLog2e;
#pragma unroll
        for (int i = 0; i < N; ++i)
            qf[i] *= s;
    }

    float m = -INFINITY, l = 0.f, acc[N];
#pragma unroll
    for (int i = 0; i < N; ++i)
        acc[i] = 0.f;

    // Row block r0 covers rows r0 + (warp * kWinUnroll + u) * RPW + g.  The loads of block
    // r0 + ROWS are issued before block r0 is computed (register double buffering), so a
    // lane always has a block of K and V chunks in flight.
    uint4 kk[kWinUnroll], vv[kWinUnroll];
    auto load_block = [&](int r0, uint4 (&kb)[kWinUnroll], uint4 (&vb)[kWinUnroll]) {
#pragma unroll
        for (int u = 0; u < kWinUnroll; ++u) {
            const int row = r0 + (warp * kWinUnroll + u) * RPW + g;
            kb[u] = vb[u] = make_uint4(0u, 0u, 0u, 0u);
            if (row < len && has_chunk) {
                kb[u] = ld_stream_u4(K + (int64_t)row * d);
                vb[u] = ld_stream_u4(V + (int64_t)row * d);
            }
        }
    };
    load_block(0, kk, vv);
    for (int r0 = 0; r0 < len; r0 += ROWS) {
        uint4 nk[kWinUnroll], nv[kWinUnroll];
        load_block(r0 + ROWS, nk, nv); // rows past len load nothing
        float s[kWinUnroll];
        float mx = m;
#pragma unroll
        for (int u = 0; u < kWinUnroll; ++u) {
            float kf[N];
            Chunk<T>::unpack(kk[u], kf);
            float p = 0.f;
#pragma unroll
            for (int i = 0; i < N; ++i)
                p = fmaf(qf[i], kf[i], p);
#pragma unroll
            for (int off = LPR / 2; off > 0; off >>= 1)
                p += __shfl_xor_sync(0xffffffffu, p, off);
            s[u] = r0 + (warp * kWinUnroll + u) * RPW + g < len ? p : -INFINITY;
            mx = fmaxf(mx, s[u]);
        }
        if (mx != -INFINITY) { // else this group had no rows in this block (m stays -inf)
            const float al = exp2f(m - mx);
            l *= al;
#pragma unroll
            for (int i = 0; i < N; ++i)
                acc[i] *= al;
#pragma unroll
            for (int u = 0; u < kWinUnroll; ++u) {
                const float p = exp2f(s[u] - mx);
                float vf[N];
                Chunk<T>::unpack(vv[u], vf);
                l += p;
#pragma unroll
                for (int i = 0; i < N; ++i)
                    acc[i] = fmaf(p, vf[i], acc[i]);
            }
            m = mx;
        }
#pragma unroll
        for (int u = 0; u < kWinUnroll; ++u) {
            kk[u] = nk[u];
            vv[u] = nv[u];
        }
    }

    // merge the lane groups of this warp (lanes sub, sub + LPR, ... hold the same columns)
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m, off);
        const float lo = __shfl_xor_sync(0xffffffffu, l, off);
        float ao[N];
#pragma unroll
        for (int i = 0; i < N; ++i)
            ao[i] = __shfl_xor_sync(0xffffffffu, acc[i], off);
        merge_state<N>(m, l, acc, mo, lo, ao);
    }
    if (g == 0) {
        if (has_chunk) {
#pragma unroll
            for (int i = 0; i < N; ++i)
                wacc[warp * d + sub * N + i] = acc[i];
        }
        if (sub == 0) {
            red[warp][0] = m;
            red[warp][1] = l;
        }
    }
    __syncthreads();

    // merge the warps: thread c owns output column c
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWinWarps; ++w)
        M = fmaxf(M, red[w][0]);
    float L = 0.f, f[kWinWarps];
#pragma unroll
    for (int w = 0; w < kWinWarps; ++w) {
        f[w] = M == -INFINITY ? 0.f : exp2f(red[w][0] - M);
        L = fmaf(f[w], red[w][1], L);
    }
    const float invL = L > 0.f ? 1.f / L : 0.f;
    float *rec = a.win_part + (((int64_t)b * a.H + h) * a.Tq_all + t) * part_stride(d);
    for (int c = threadIdx.x; c < d; c += kWinThreads) {
        float o = 0.f;
#pragma unroll
        for (int w = 0; w < kWinWarps; ++w)
            o = fmaf(f[w], wacc[w * d + c], o);
        rec[c] = o * invL;
    }
    if (threadIdx.x == 0)
        rec[d] = L > 0.f ? M + log2f(L) : -INFINITY; // lse_win in log2 units

    grid_dependency_wait(); // the decode grid has finished: the combine may read its records
}

template <typename T, int LPR>
cudaError_t launch_window_t(const DecodeArgs &a, cudaStream_t stream)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.H, a.Tq, a.B);
    cfg.blockDim = dim3(kWinThreads);
    cfg.dynamicSmemBytes = sizeof(float) * kWinWarps * a.d;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization; // fill the decode's tail
    attr[0].val.programmaticStreamSerializationAllowed = a.serial ? 0 : 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_window_kernel<T, LPR>, a);
}

template <typename T> cudaError_t launch_window_lpr(const DecodeArgs &a, int chunks, cudaStream_t stream)
{
    if (chunks <= 1) return launch_window_t<T, 1>(a, stream);
    if (chunks <= 2) return launch_window_t<T, 2>(a, stream);
    if (chunks <= 4) return launch_window_t<T, 4>(a, stream);
    if (chunks <= 8) return launch_window_t<T, 8>(a, stream);
    if (chunks <= 16) return launch_window_t<T, 16>(a, stream);
    return launch_window_t<T, 32>(a, stream);
}

} // namespace

bool decode_window_supported(int dtype, int d)
{
    const int e = dtype == LLA_BF16 ? 2 : 4;
    return d > 0 && (d * e) % 16 == 0 && d * e <= 512 && d <= 128 * 4;
}

cudaError_t launch_decode_window(const DecodeArgs &a, int dtype, cudaStream_t stream)
{
    if (a.B > 65535 || a.Tq > 65535)
        return cudaErrorInvalidValue;
    const int e = dtype == LLA_BF16 ? 2 : 4;
    const int chunks = a.d * e / 16;
    if (dtype == LLA_BF16)
        return launch_window_lpr<__nv_bfloat16>(a, chunks, stream);
    return launch_window_lpr<float>(a, chunks, stream);
}

} // namespace lla
