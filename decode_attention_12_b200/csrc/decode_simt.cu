// decode_simt.cu -- LLA decode attention, query-absorbed form, on CUDA cores.
//
// "Looped Latent Attention: Cross-Loop KV Compression for Looped Transformers":
// Pith review page, "What carries the argument" (Eq. 3, x_hat_t = c W_up,t + mu_t)
// and the Pith verdict record's desk-editor letter (the absorbed-attention
// variant).  Substituting Eq. 3 into a loop-t attention read gives
//     l_n = q_tilde . c_K[n] + scale * q . mu_t^K,   q_tilde = scale * q W_up,t^K^T
//     out = (sum_n p_n c_V[n]) W_up,t^V + mu_t^V,
// so one pass over the latents (r_k + r_v values per cached token) serves every
// loop query of the (sequence, head) at once.
//
// Kernel shape (per-head latents, r_k, r_v <= 32):
//  * grid (split, head, sequence); 128 threads; each CTA streams a contiguous
//    token range of one (sequence, head) latent stream, HBM -> shared memory with
//    1-D bulk (TMA) copies into a 4-stage mbarrier ring;
//  * a1 (absorb prologue) is computed per CTA while the first tiles are in
//    flight: q_tilde for the Tq loop queries, pre-scaled by log2(e);
//  * a2/a3: one token per thread per step; the thread keeps its own online-softmax
//    state (running reference m, sum l, r_v-wide latent accumulator) for all Tq
//    queries, with a lazy rescale (only when a score exceeds the reference by
//    more than 2^8); rows are read from shared memory in a per-lane rotated chunk
//    order that makes every 16-byte load conflict-free;
//  * the CTA merges its 128 thread states through shared memory and writes one
//    partial record (acc, m, l) per query; the combine kernel (a4) merges splits
//    and applies W_up,t^V + mu_t^V.
#include "decode.cuh"

namespace lla {
namespace {

constexpr int kThreads = 128;
constexpr int kTokensPerThread = 2;
constexpr int kStages = 4;
constexpr int kTile = kThreads * kTokensPerThread;
constexpr float kRescaleThreshold = 8.0f; // log2 units

template <typename T, int RK, int RV, int TQ> struct SimtCfg {
    static constexpr int KB = RK * (int)sizeof(T); // bytes per key-latent row
    static constexpr int VB = RV * (int)sizeof(T);
    static constexpr int N = Chunk<T>::N;           // values per 16-byte chunk
    static constexpr int NCK = KB / 16;
    static constexpr int NCV = VB / 16;
    static constexpr int RING = kStages * kTile * (KB + VB);
    static constexpr int RED_STRIDE = TQ * (RV + 1) + 1; // floats per thread row
    static constexpr int RED = kThreads * RED_STRIDE * 4;
    static constexpr int BODY = RING > RED ? RING : RED;
    static constexpr int QT_OFF = BODY;                      // q_tilde [TQ][RK] fp32
    static constexpr int MRED_OFF = QT_OFF + TQ * RK * 4;    // [4 warps][TQ]
    static constexpr int BAR_OFF = (MRED_OFF + 4 * TQ * 4 + 15) & ~15;
    static constexpr int FLAG_OFF = BAR_OFF + kStages * 8;
    static constexpr int SMEM = FLAG_OFF + 16;
    static_assert(KB % 16 == 0 && VB % 16 == 0, "rows must be 16-byte multiples");
    static_assert(NCK <= 8 && NCV <= 8, "rank too large for the SIMT kernel");
};

// Rotation of the 16-byte chunk order for shared-memory row `row` of `nc` chunks
// so that 8 consecutive rows touch 8 distinct 16-byte bank groups.
__device__ __forceinline__ int chunk_rotation(int row, int nc)
{
    return nc <= 1 ? 0 : (row / (8 / nc)) % nc;
}

template <typename T, int RK, int RV, int TQ>
__global__ void __launch_bounds__(kThreads, 2) decode_absorb_simt_kernel(const DecodeArgs a)
{
    using C = SimtCfg<T, RK, RV, TQ>;
    extern __shared__ __align__(128) uint8_t smem[];
    float *qt_s = reinterpret_cast<float *>(smem + C::QT_OFF);
    float *mred = reinterpret_cast<float *>(smem + C::MRED_OFF);
    int *flag = reinterpret_cast<int *>(smem + C::FLAG_OFF);
    const uint32_t bar0 = smem_u32(smem + C::BAR_OFF);

    const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int len = a.ctx_lens[b];
    int n0, n1;
    split_range(len, split, a.num_splits, n0, n1);
    const int ntok = n1 - n0;
    const int ntiles = (ntok + kTile - 1) / kTile;
    const int64_t row0 = a.seq_start[b] + n0;
    const uint8_t *gK = static_cast<const uint8_t *>(a.k) + ((int64_t)h * a.slots + row0) * C::KB;
    const uint8_t *gV = static_cast<const uint8_t *>(a.v) + ((int64_t)h * a.slots + row0) * C::VB;
    uint8_t *ringK = smem;
    uint8_t *ringV = smem + kStages * kTile * C::KB;

    auto issue = [&](int tile, int stage) {
        const int rows = min(kTile, ntok - tile * kTile);
        const uint32_t kb = rows * C::KB, vb = rows * C::VB;
        const uint32_t bar = bar0 + 8 * stage;
        mbar_arrive_expect_tx(bar, kb + vb);
        bulk_copy_g2s(smem_u32(ringK + stage * kTile * C::KB), gK + (int64_t)tile * kTile * C::KB,
                      kb, bar);
        bulk_copy_g2s(smem_u32(ringV + stage * kTile * C::VB), gV + (int64_t)tile * kTile * C::VB,
                      vb, bar);
    };

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s)
            mbar_init(bar0 + 8 * s, 1);
        *flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (tid == 0) {
        for (int s = 0; s < kStages && s < ntiles; ++s)
            issue(s, s);
    }

    // ---- a1: absorb prologue, q_tilde[t][j] = scale*log2e * sum_k q[t][k] W_up,t^K[j][k]
    {
        const T *qb = static_cast<const T *>(a.q);
        for (int o = warp; o < TQ * RK; o += kThreads / 32) {
            const int t = o / RK, j = o % RK;
            float acc = 0.f;
            if (t < a.Tq) {
                const T *qrow = qb + (((int64_t)b * a.Tq_all + a.tq_off + t) * a.H + h) * a.d;
                const float *w = a.W_up_k + (((int64_t)h * a.T + a.t0 + a.tq_off + t) * RK + j) * a.d;
                for (int k = lane; k < a.d; k += 32)
                    acc = fmaf(Elem<T>::to_f(qrow[k]), w[k], acc);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (lane == 0)
                qt_s[o] = acc * a.scale * kLog2e;
        }
    }
    __syncthreads();

    // Per-lane rotated copies of q_tilde (see chunk_rotation) and the online state.
    const int rotK = chunk_rotation(tid, C::NCK);
    const int rotV = chunk_rotation(tid, C::NCV);
    float qreg[TQ][C::NCK][C::N];
#pragma unroll
    for (int t = 0; t < TQ; ++t)
#pragma unroll
        for (int c = 0; c < C::NCK; ++c)
#pragma unroll
            for (int e = 0; e < C::N; ++e)
                qreg[t][c][e] = qt_s[t * RK + ((c + rotK) % C::NCK) * C::N + e];

    float m[TQ], l[TQ], acc[TQ][C::NCV][C::N];
#pragma unroll
    for (int t = 0; t < TQ; ++t) {
        m[t] = -INFINITY;
        l[t] = 0.f;
#pragma unroll
        for (int c = 0; c < C::NCV; ++c)
#pragma unroll
            for (int e = 0; e < C::N; ++e)
                acc[t][c][e] = 0.f;
    }

    int failed_at = -1;
    for (int i = 0; i < ntiles; ++i) {
        const int stage = i % kStages;
        if (!mbar_wait_bounded(bar0 + 8 * stage, (i / kStages) & 1)) {
            *flag = 1; // benign race: every writer stores 1
        } else {
            const int rows = min(kTile, ntok - i * kTile);
            const uint8_t *sK = ringK + stage * kTile * C::KB;
            const uint8_t *sV = ringV + stage * kTile * C::VB;
#pragma unroll
            for (int tt = 0; tt < kTokensPerThread; ++tt) {
                const int row = tt * kThreads + tid;
                if (row < rows) {
                    // a2: scores (log2 domain, without the constant q.mu_t^K term)
                    float s[TQ];
#pragma unroll
                    for (int t = 0; t < TQ; ++t)
                        s[t] = 0.f;
#pragma unroll
                    for (int c = 0; c < C::NCK; ++c) {
                        const uint4 u = *reinterpret_cast<const uint4 *>(
                            sK + row * C::KB + 16 * ((c + rotK) % C::NCK));
                        float f[C::N];
                        Chunk<T>::unpack(u, f);
#pragma unroll
                        for (int t = 0; t < TQ; ++t)
#pragma unroll
                            for (int e = 0; e < C::N; ++e)
                                s[t] = fmaf(qreg[t][c][e], f[e], s[t]);
                    }
                    // a3: online softmax with lazy rescale
                    float p[TQ];
#pragma unroll
                    for (int t = 0; t < TQ; ++t) {
                        if (s[t] > m[t] + kRescaleThreshold) {
                            const float alpha = exp2f(m[t] - s[t]);
                            l[t] *= alpha;
#pragma unroll
                            for (int c = 0; c < C::NCV; ++c)
#pragma unroll
                                for (int e = 0; e < C::N; ++e)
                                    acc[t][c][e] *= alpha;
                            m[t] = s[t];
                        }
                        p[t] = exp2f(s[t] - m[t]);
                        l[t] += p[t];
                    }
#pragma unroll
                    for (int c = 0; c < C::NCV; ++c) {
                        const uint4 u = *reinterpret_cast<const uint4 *>(
                            sV + row * C::VB + 16 * ((c + rotV) % C::NCV));
                        float f[C::N];
                        Chunk<T>::unpack(u, f);
#pragma unroll
                        for (int t = 0; t < TQ; ++t)
#pragma unroll
                            for (int e = 0; e < C::N; ++e)
                                acc[t][c][e] = fmaf(p[t], f[e], acc[t][c][e]);
                    }
                }
            }
        }
        __syncthreads();
        if (*flag) {
            failed_at = i;
            break;
        }
        if (tid == 0 && i + kStages < ntiles)
            issue(i + kStages, stage);
    }

    if (failed_at >= 0) {
        // Wind down: wait (bounded) for this CTA's own copies still in flight
        // (tiles failed_at .. failed_at+kStages-1 were issued and not consumed).
        if (tid == 0) {
            report_status(a.status, LLA_ERR_DEVICE_TIMEOUT);
            for (int j = failed_at; j < ntiles && j < failed_at + kStages; ++j)
                (void)mbar_wait_bounded(bar0 + 8 * (j % kStages), (j / kStages) & 1);
        }
        return;
    }

    // ---- merge the 128 thread states: common reference M[t] = max of references
#pragma unroll
    for (int t = 0; t < TQ; ++t) {
        float mm = m[t];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, off));
        if (lane == 0)
            mred[warp * TQ + t] = mm;
    }
    __syncthreads(); // also: ring no longer read, reuse it for the reduction
#pragma unroll
    for (int t = 0; t < TQ; ++t) {
        const float Mt = fmaxf(fmaxf(mred[t], mred[TQ + t]), fmaxf(mred[2 * TQ + t], mred[3 * TQ + t]));
        const float f = (m[t] == -INFINITY) ? 0.f : exp2f(m[t] - Mt);
        l[t] *= f;
#pragma unroll
        for (int c = 0; c < C::NCV; ++c)
#pragma unroll
            for (int e = 0; e < C::N; ++e)
                acc[t][c][e] *= f;
    }
    float *red = reinterpret_cast<float *>(smem);
    float *myrow = red + tid * C::RED_STRIDE;
#pragma unroll
    for (int t = 0; t < TQ; ++t) {
#pragma unroll
        for (int c = 0; c < C::NCV; ++c)
#pragma unroll
            for (int e = 0; e < C::N; ++e)
                myrow[t * (RV + 1) + ((c + rotV) % C::NCV) * C::N + e] = acc[t][c][e];
        myrow[t * (RV + 1) + RV] = l[t];
    }
    __syncthreads();
    for (int col = tid; col < TQ * (RV + 1); col += kThreads) {
        const int t = col / (RV + 1), j = col % (RV + 1);
        float sum = 0.f;
        for (int r = 0; r < kThreads; ++r)
            sum += red[r * C::RED_STRIDE + col];
        if (t < a.Tq) {
            // record layout: acc[0..RV), reference m at RV, sum l at RV+1
            float *rec = a.part + ((((int64_t)b * a.H + h) * a.Tq_all + a.tq_off + t) * a.num_splits + split) *
                                      part_stride(RV);
            if (j < RV) {
                rec[j] = sum;
            } else {
                rec[RV] = fmaxf(fmaxf(mred[t], mred[TQ + t]), fmaxf(mred[2 * TQ + t], mred[3 * TQ + t]));
                rec[RV + 1] = sum;
            }
        }
    }
}

template <typename T, int RK, int RV, int TQ>
cudaError_t launch_simt(const DecodeArgs &a, cudaStream_t stream)
{
    using C = SimtCfg<T, RK, RV, TQ>;
    auto kern = decode_absorb_simt_kernel<T, RK, RV, TQ>;
    static bool configured = false; // attribute set once per process (same value every time)
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess)
            return e;
        configured = true;
    }
    dim3 grid(a.num_splits, a.H, a.B);
    kern<<<grid, kThreads, C::SMEM, stream>>>(a);
    return cudaGetLastError();
}

template <typename T, int RK, int RV>
cudaError_t launch_simt_tq(const DecodeArgs &a, cudaStream_t stream)
{
    if (a.Tq == 1)
        return launch_simt<T, RK, RV, 1>(a, stream);
    if (a.Tq == 2)
        return launch_simt<T, RK, RV, 2>(a, stream);
    return launch_simt<T, RK, RV, 4>(a, stream);
}

// ---------------------------------------------------------------------------------
// a4: cross-split combine + output projection.
//   M = max_s m_s,  L = sum_s l_s 2^(m_s - M),  o_lat = sum_s acc_s 2^(m_s - M) / L
//   out = o_lat W_up,t^V + mu_t^V,   lse = ln2 (M + log2 L) + scale * q . mu_t^K
// One CTA per (query loop, head, sequence); thread k owns output dims k, k+128, ...
// ---------------------------------------------------------------------------------
constexpr int kCombineThreads = 128;

template <typename T, typename O>
__global__ void __launch_bounds__(kCombineThreads) decode_combine_kernel(const DecodeArgs a)
{
    extern __shared__ float csm[]; // o_lat [r_v], w [S], misc
    const int t = a.tq_off + blockIdx.x, h = blockIdx.y, b = blockIdx.z; // t indexes q/out/lse
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int S = a.num_splits, RV = a.r_v;
    const int ps = part_stride(RV);
    float *olat = csm;
    float *w = csm + RV;
    float *red = w + S;
    const float *rec0 = a.part + (((int64_t)b * a.H + h) * a.Tq_all + t) * S * ps;

    float Mloc = -INFINITY;
    for (int s = tid; s < S; s += kCombineThreads)
        Mloc = fmaxf(Mloc, rec0[s * ps + RV]);
    for (int off = 16; off > 0; off >>= 1)
        Mloc = fmaxf(Mloc, __shfl_xor_sync(0xffffffffu, Mloc, off));
    if (lane == 0)
        red[warp] = Mloc;
    __syncthreads();
    const float M = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    __syncthreads();
    float Lloc = 0.f;
    for (int s = tid; s < S; s += kCombineThreads) {
        const float ms = rec0[s * ps + RV];
        const float ws = (ms == -INFINITY) ? 0.f : exp2f(ms - M);
        w[s] = ws;
        Lloc += ws * rec0[s * ps + RV + 1];
    }
    for (int off = 16; off > 0; off >>= 1)
        Lloc += __shfl_xor_sync(0xffffffffu, Lloc, off);
    if (lane == 0)
        red[warp] = Lloc;
    __syncthreads();
    const float L = red[0] + red[1] + red[2] + red[3];
    const float invL = L > 0.f ? 1.f / L : 0.f;
    for (int j = tid; j < RV; j += kCombineThreads) {
        float sum = 0.f;
        for (int s = 0; s < S; ++s)
            sum = fmaf(w[s], rec0[s * ps + j], sum);
        olat[j] = sum * invL;
    }
    __syncthreads();

    // output projection; per-head: W_up [H][T][RV][d]; LLA-2D: [T][RV][H*d], cols h*d..
    const int tg = a.t0 + t;
    const int ld = a.fold ? a.H * a.d : a.d;
    const int64_t wbase = a.fold ? (int64_t)tg * RV * ld + (int64_t)h * a.d
                                 : ((int64_t)h * a.T + tg) * RV * ld;
    const int64_t mbase = a.fold ? (int64_t)tg * ld + (int64_t)h * a.d : ((int64_t)h * a.T + tg) * ld;
    const T *qrow = static_cast<const T *>(a.q) + (((int64_t)b * a.Tq_all + t) * a.H + h) * a.d;
    O *orow = static_cast<O *>(a.out) + (((int64_t)b * a.Tq_all + t) * a.H + h) * a.d;
    float qmu = 0.f;
    for (int k = tid; k < a.d; k += kCombineThreads) {
        float o = 0.f;
        if (L > 0.f) {
            o = a.mu_v[mbase + k];
            for (int j = 0; j < RV; ++j)
                o = fmaf(olat[j], a.W_up_v[wbase + (int64_t)j * ld + k], o);
        }
        orow[k] = Elem<O>::from_f(o);
        qmu = fmaf(Elem<T>::to_f(qrow[k]), a.mu_k[mbase + k], qmu);
    }
    if (a.lse != nullptr) {
        for (int off = 16; off > 0; off >>= 1)
            qmu += __shfl_xor_sync(0xffffffffu, qmu, off);
        __syncthreads();
        if (lane == 0)
            red[warp] = qmu;
        __syncthreads();
        if (tid == 0) {
            const float qm = red[0] + red[1] + red[2] + red[3];
            a.lse[((int64_t)b * a.Tq_all + t) * a.H + h] =
                L > 0.f ? kLn2 * (M + log2f(L)) + a.scale * qm : -INFINITY;
        }
    }
}

} // namespace

bool decode_absorb_simt_supported(int dtype, int r_k, int r_v, int d, int fold)
{
    if (fold != LLA_PER_HEAD || d % 32 != 0 || d > 1024)
        return false;
    if (dtype == LLA_BF16)
        return (r_k == 16 && r_v == 32) || (r_k == 8 && r_v == 16) || (r_k == 16 && r_v == 16);
    return (r_k == 8 && r_v == 16) || (r_k == 16 && r_v == 32) || (r_k == 4 && r_v == 8);
}

cudaError_t launch_decode_absorb_simt(const DecodeArgs &a, int dtype, cudaStream_t stream,
                                      bool *supported)
{
    *supported = true;
    if (dtype == LLA_BF16) {
        using B = __nv_bfloat16;
        if (a.r_k == 16 && a.r_v == 32) return launch_simt_tq<B, 16, 32>(a, stream);
        if (a.r_k == 8 && a.r_v == 16) return launch_simt_tq<B, 8, 16>(a, stream);
        if (a.r_k == 16 && a.r_v == 16) return launch_simt_tq<B, 16, 16>(a, stream);
    } else {
        if (a.r_k == 8 && a.r_v == 16) return launch_simt_tq<float, 8, 16>(a, stream);
        if (a.r_k == 16 && a.r_v == 32) return launch_simt_tq<float, 16, 32>(a, stream);
        if (a.r_k == 4 && a.r_v == 8) return launch_simt_tq<float, 4, 8>(a, stream);
    }
    *supported = false;
    return cudaSuccess;
}

cudaError_t launch_decode_combine(const DecodeArgs &a, int dtype, int out_dtype, cudaStream_t stream)
{
    dim3 grid(a.Tq, a.H, a.B);
    const size_t smem = sizeof(float) * (a.r_v + a.num_splits + 8);
    if (smem > 48 * 1024)
        return cudaErrorInvalidValue;
    using BF = __nv_bfloat16;
    if (dtype == LLA_BF16 && out_dtype == LLA_BF16)
        decode_combine_kernel<BF, BF><<<grid, kCombineThreads, smem, stream>>>(a);
    else if (dtype == LLA_BF16)
        decode_combine_kernel<BF, float><<<grid, kCombineThreads, smem, stream>>>(a);
    else if (out_dtype == LLA_BF16)
        decode_combine_kernel<float, BF><<<grid, kCombineThreads, smem, stream>>>(a);
    else
        decode_combine_kernel<float, float><<<grid, kCombineThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

} // namespace lla
