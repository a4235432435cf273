// decode_simt.cu -- LLA decode attention, query-absorbed form, on CUDA cores.
//
// "Looped Latent Attention: Cross-Loop KV Compression for Looped Transformers":
// Pith review page, "What carries the argument" (Eq. 3, x_hat_t = c W_up,t + mu_t),
// and the Pith verdict record's desk-editor letter (the absorbed-attention variant).
// Substituting Eq. 3 into a loop-t attention read gives
//     l_n = q_tilde . c_K[n] + scale * q . mu_t^K,   q_tilde = scale * q W_up,t^K^T
//     out = (sum_n p_n c_V[n]) W_up,t^V + mu_t^V,
// so one pass over the latents (r_k + r_v values per cached token) serves every
// loop query of a (sequence, head) unit at once.  Three kernels:
//
//  a1  absorb_prologue_kernel: q_tilde for every (unit, loop query), pre-scaled by
//      log2(e), into the workspace (one warp per output element).
//  a2/a3 decode_absorb_kernel (persistent, load-balanced): the grid holds exactly the
//      resident CTAs; the concatenated token stream of all (sequence, head) units is
//      cut into equal shares, one per CTA, so ragged lengths leave no tail wave.  A
//      share may cross unit boundaries; every unit segment it covers becomes one
//      partial record (acc, m, l).  One thread walks the share and streams tiles of
//      128 tokens with 1-D bulk (TMA) copies into a 3-stage mbarrier ring; the
//      unit's q_tilde rides along with its first tile.  Each of the 64 threads owns
//      two tokens per tile and keeps its own online-softmax state for all loop
//      queries (running reference m, sum l, r_v-wide latent accumulator) with a lazy
//      rescale; dot products use packed fp32x2 FMAs; rows are read in a per-lane
//      rotated chunk order so every 16-byte shared load is conflict-free.
//  a4  decode_combine_kernel: log-sum-exp merge of a unit's records, then
//      out = o_lat W_up,t^V + mu_t^V and lse.
#include "decode_sched.cuh"

namespace lla {
namespace {

constexpr int kThreads = 64;
constexpr int kWarps = kThreads / 32;
constexpr int kTokensPerThread = 2;
constexpr int kStages = 3;
constexpr int kTile = kThreads * kTokensPerThread;
constexpr float kRescaleThreshold = 8.0f; // log2 units

template <typename T, int RK, int RV, int TQ> struct Cfg {
    static constexpr int KB = RK * (int)sizeof(T); // bytes per key-latent row
    static constexpr int VB = RV * (int)sizeof(T);
    static constexpr int N = Chunk<T>::N;           // values per 16-byte chunk
    static constexpr int NCK = KB / 16;
    static constexpr int NCV = VB / 16;
    static constexpr int QB = TQ * RK * 4;          // q_tilde slot of one unit (Tq <= TQ used)
    static constexpr int STAGE = kTile * (KB + VB) + QB;
    static constexpr int RING = kStages * STAGE;
    static constexpr int RED_STRIDE = RV + 1;
    static constexpr int RED_OFF = RING;                                    // [warps][32][RV+1]
    static constexpr int WSUM_OFF = RED_OFF + kWarps * 32 * RED_STRIDE * 4; // [warps][TQ][RV]
    static constexpr int LSUM_OFF = WSUM_OFF + kWarps * TQ * RV * 4;        // [warps][TQ]
    static constexpr int MRED_OFF = LSUM_OFF + kWarps * TQ * 4;             // [warps][TQ]
    static constexpr int DESC_OFF = (MRED_OFF + kWarps * TQ * 4 + 15) & ~15; // [stages]
    static constexpr int BAR_OFF = DESC_OFF + kStages * (int)sizeof(TileDesc);
    static constexpr int MISC_OFF = BAR_OFF + kStages * 8;                 // ntiles, flag
    static constexpr int PREF_OFF = (MISC_OFF + 16 + 15) & ~15;             // int64 [B+1]
    static_assert(KB % 16 == 0 && VB % 16 == 0, "rows must be 16-byte multiples");
    static_assert(NCK <= 8 && NCV <= 8 && RV <= 32, "rank too large for the SIMT kernel");
    static_assert(N % 2 == 0 && RK % 2 == 0 && RV % 2 == 0, "packed pairs");
};

__device__ __forceinline__ int chunk_rotation(int row, int nc)
{
    return nc <= 1 ? 0 : (row / (8 / nc)) % nc;
}

template <typename T, int RK, int RV, int TQ>
__global__ void __launch_bounds__(kThreads, kDecodeCtasPerSm) decode_absorb_kernel(const DecodeArgs a)
{
    using C = Cfg<T, RK, RV, TQ>;
    extern __shared__ __align__(128) uint8_t smem[];
    float *red = reinterpret_cast<float *>(smem + C::RED_OFF);
    float *wsum = reinterpret_cast<float *>(smem + C::WSUM_OFF);
    float *lsum = reinterpret_cast<float *>(smem + C::LSUM_OFF);
    float *mred = reinterpret_cast<float *>(smem + C::MRED_OFF);
    TileDesc *descs = reinterpret_cast<TileDesc *>(smem + C::DESC_OFF);
    int *misc = reinterpret_cast<int *>(smem + C::MISC_OFF);
    int64_t *pref = reinterpret_cast<int64_t *>(smem + C::PREF_OFF);
    const uint32_t bar0 = smem_u32(smem + C::BAR_OFF);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int B = a.B, H = a.H;

    // ---- work split: prefix of the context lengths, this CTA's token share
    if (tid == 0) {
        for (int s2 = 0; s2 < kStages; ++s2)
            mbar_init(bar0 + 8 * s2, 1);
        misc[1] = 0;
        fence_barrier_init();
    }
    block_length_prefix<kThreads>(a.ctx_lens, B, pref, reinterpret_cast<int64_t *>(red));
    int64_t s0, s1, chunk;
    cta_share(pref, B, H, a.chunk_min, s0, s1, chunk);
    if (s0 >= s1)
        return; // uniform: nothing for this CTA

    const T *gk = static_cast<const T *>(a.k);
    const T *gv = static_cast<const T *>(a.v);
    uint8_t *ring = smem;
    ShareWalk<kTile> walk; // producer state (thread 0 only)
    auto issue = [&](int stage) -> bool {
        TileDesc d;
        if (!walk.next(pref, a.seq_start, B, H, d))
            return false;
        descs[stage] = d;
        uint8_t *st = ring + stage * C::STAGE;
        const uint32_t kb = d.rows * C::KB, vb = d.rows * C::VB;
        const uint32_t qb = (d.flags & 1) ? (uint32_t)(a.Tq * RK * 4) : 0u; // this pass's queries only
        const uint32_t bar = bar0 + 8 * stage;
        mbar_arrive_expect_tx(bar, kb + vb + qb);
        const int64_t row = (int64_t)d.h * a.slots + d.row;
        bulk_copy_g2s(smem_u32(st), gk + row * RK, kb, bar);
        bulk_copy_g2s(smem_u32(st + kTile * C::KB), gv + row * RV, vb, bar);
        if (qb)
            bulk_copy_g2s(smem_u32(st + kTile * (C::KB + C::VB)),
                          a.qt + ((int64_t)d.u * a.Tq_all + a.tq_off) * RK, qb, bar);
        return true;
    };
    if (tid == 0) {
        // count this share's tiles, then start the ring
        int nt = 0;
        TileDesc d;
        walk.start(s0, s1, chunk);
        while (walk.next(pref, a.seq_start, B, H, d))
            ++nt;
        misc[0] = nt;
        walk.start(s0, s1, chunk);
        for (int s2 = 0; s2 < kStages && s2 < nt; ++s2)
            issue(s2);
    }
    __syncthreads();
    const int ntiles = misc[0];

    const int rotK = chunk_rotation(tid, C::NCK);
    const int rotV = chunk_rotation(tid, C::NCV);
    float2 q2[TQ][RK / 2];
    float m[TQ], l[TQ];
    float2 acc[TQ][RV / 2];

    int failed_at = -1;
    for (int i = 0; i < ntiles; ++i) {
        const int stage = i % kStages;
        __syncthreads(); // every thread is done with tile i - 1: its stage may be refilled
        if (tid == 0 && i >= 1 && i - 1 + kStages < ntiles)
            issue((i - 1) % kStages);
        if (!mbar_wait_bounded(bar0 + 8 * stage, (i / kStages) & 1))
            misc[1] = 1; // every writer stores 1
        __syncthreads(); // all threads agree on the outcome before reading the descriptor
        if (misc[1]) {
            failed_at = i;
            break;
        }
        {
            const TileDesc d = descs[stage];
            const uint8_t *sK = ring + stage * C::STAGE;
            const uint8_t *sV = sK + kTile * C::KB;
            if (d.flags & 1) { // a new unit segment: its q_tilde (rotated per lane), fresh state
                const float *qs = reinterpret_cast<const float *>(sV + kTile * C::VB);
#pragma unroll
                for (int t = 0; t < TQ; ++t) {
#pragma unroll
                    for (int c = 0; c < C::NCK; ++c)
#pragma unroll
                        for (int e = 0; e < C::N; e += 2) {
                            const int k = ((c + rotK) % C::NCK) * C::N + e;
                            q2[t][(c * C::N + e) / 2] =
                                t < a.Tq ? make_float2(qs[t * RK + k], qs[t * RK + k + 1]) : make_float2(0.f, 0.f);
                        }
                    m[t] = -INFINITY;
                    l[t] = 0.f;
#pragma unroll
                    for (int c = 0; c < RV / 2; ++c)
                        acc[t][c] = make_float2(0.f, 0.f);
                }
            }
#pragma unroll
            for (int tt = 0; tt < kTokensPerThread; ++tt) {
                const int row = tt * kThreads + tid;
                if (row < d.rows) {
                    // a2: scores in the log2 domain (the constant q.mu_t^K term is left out)
                    float2 s2[TQ];
#pragma unroll
                    for (int t = 0; t < TQ; ++t)
                        s2[t] = make_float2(0.f, 0.f);
#pragma unroll
                    for (int c = 0; c < C::NCK; ++c) {
                        const uint4 u = *reinterpret_cast<const uint4 *>(
                            sK + row * C::KB + 16 * ((c + rotK) % C::NCK));
                        float f[C::N];
                        Chunk<T>::unpack(u, f);
#pragma unroll
                        for (int t = 0; t < TQ; ++t)
#pragma unroll
                            for (int e = 0; e < C::N; e += 2)
                                s2[t] = __ffma2_rn(q2[t][(c * C::N + e) / 2], make_float2(f[e], f[e + 1]), s2[t]);
                    }
                    // a3: online softmax with a lazy rescale
                    float p[TQ];
#pragma unroll
                    for (int t = 0; t < TQ; ++t) {
                        const float s = s2[t].x + s2[t].y;
                        if (s > m[t] + kRescaleThreshold) {
                            const float alpha = fast_exp2(m[t] - s);
                            l[t] *= alpha;
                            const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
                            for (int c = 0; c < RV / 2; ++c)
                                acc[t][c] = __fmul2_rn(acc[t][c], a2);
                            m[t] = s;
                        }
                        p[t] = fast_exp2(s - m[t]);
                        l[t] += p[t];
                    }
#pragma unroll
                    for (int c = 0; c < C::NCV; ++c) {
                        const uint4 u = *reinterpret_cast<const uint4 *>(
                            sV + row * C::VB + 16 * ((c + rotV) % C::NCV));
                        float f[C::N];
                        Chunk<T>::unpack(u, f);
#pragma unroll
                        for (int t = 0; t < TQ; ++t) {
                            const float2 pp = make_float2(p[t], p[t]);
#pragma unroll
                            for (int e = 0; e < C::N; e += 2)
                                acc[t][(c * C::N + e) / 2] =
                                    __ffma2_rn(pp, make_float2(f[e], f[e + 1]), acc[t][(c * C::N + e) / 2]);
                        }
                    }
                }
            }
            if (d.flags & 2) {
                // ---- end of a unit segment: merge the 64 thread states into one record
#pragma unroll
                for (int t = 0; t < TQ; ++t) {
                    float mm = m[t];
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1)
                        mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, off));
                    if (lane == 0)
                        mred[warp * TQ + t] = mm;
                }
                __syncthreads();
                float *wred = red + warp * 32 * C::RED_STRIDE;
#pragma unroll
                for (int t = 0; t < TQ; ++t) {
                    float Mt = mred[t];
#pragma unroll
                    for (int w = 1; w < kWarps; ++w)
                        Mt = fmaxf(Mt, mred[w * TQ + t]);
                    const float f = (m[t] == -INFINITY) ? 0.f : fast_exp2(m[t] - Mt);
                    float lt = l[t] * f;
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1)
                        lt += __shfl_xor_sync(0xffffffffu, lt, off);
                    if (lane == 0)
                        lsum[warp * TQ + t] = lt;
#pragma unroll
                    for (int c = 0; c < C::NCV; ++c)
#pragma unroll
                        for (int e = 0; e < C::N; e += 2) {
                            const float2 v2 = acc[t][(c * C::N + e) / 2];
                            const int dim = ((c + rotV) % C::NCV) * C::N + e;
                            wred[lane * C::RED_STRIDE + dim] = v2.x * f;
                            wred[lane * C::RED_STRIDE + dim + 1] = v2.y * f;
                        }
                    __syncwarp();
                    if (lane < RV) {
                        float sum = 0.f;
#pragma unroll 8
                        for (int r = 0; r < 32; ++r)
                            sum += wred[r * C::RED_STRIDE + lane];
                        wsum[(warp * TQ + t) * RV + lane] = sum;
                    }
                    __syncwarp();
                }
                __syncthreads();
                if (d.j < a.seg_max) {
                    for (int idx = tid; idx < TQ * (RV + 2); idx += kThreads) {
                        const int t = idx / (RV + 2), jj = idx % (RV + 2);
                        if (t >= a.Tq)
                            continue;
                        float val;
                        if (jj < RV) {
                            val = 0.f;
                            for (int w = 0; w < kWarps; ++w)
                                val += wsum[(w * TQ + t) * RV + jj];
                        } else if (jj == RV) {
                            val = mred[t];
                            for (int w = 1; w < kWarps; ++w)
                                val = fmaxf(val, mred[w * TQ + t]);
                        } else {
                            val = 0.f;
                            for (int w = 0; w < kWarps; ++w)
                                val += lsum[w * TQ + t];
                        }
                        a.part[(((int64_t)d.u * a.Tq_all + a.tq_off + t) * a.seg_max + d.j) * part_stride(RV) + jj] =
                            val;
                    }
                    if (tid == 0 && d.j == 0)
                        a.counts[d.u] = d.n_u;
                } else if (tid == 0) {
                    report_status(a.status, LLA_ERR_INVALID); // a context longer than max_ctx
                }
            }
        }
    }
    if (failed_at >= 0 && tid == 0) {
        // wind down: wait (bounded) for this CTA's own copies still in flight
        report_status(a.status, LLA_ERR_DEVICE_TIMEOUT);
        for (int jt = failed_at; jt < ntiles && jt < failed_at + kStages; ++jt)
            (void)mbar_wait_bounded(bar0 + 8 * (jt % kStages), (jt / kStages) & 1);
    }
}

template <typename T, int RK, int RV, int TQ>
cudaError_t launch_persistent(const DecodeArgs &a, int ctas, cudaStream_t stream)
{
    using C = Cfg<T, RK, RV, TQ>;
    auto kern = decode_absorb_kernel<T, RK, RV, TQ>;
    const int smem = C::PREF_OFF + 8 * (a.B + 1);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
        return e;
    int dev = 0, sms = 148, occ = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kThreads, smem);
    if (e != cudaSuccess)
        return e;
    if (occ < 1)
        return cudaErrorInvalidConfiguration;
    int grid = sms * occ;
    if (ctas > 0 && ctas < grid)
        grid = ctas;
    kern<<<grid, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

template <typename T, int RK, int RV>
cudaError_t launch_tq(const DecodeArgs &a, int ctas, cudaStream_t stream)
{
    if (a.Tq == 1)
        return launch_persistent<T, RK, RV, 1>(a, ctas, stream);
    if (a.Tq == 2)
        return launch_persistent<T, RK, RV, 2>(a, ctas, stream);
    return launch_persistent<T, RK, RV, 4>(a, ctas, stream);
}

// ---------------------------------------------------------------------------------
// a1: q_tilde[u][tq_off + t][j] = scale * log2(e) * sum_k q[b][t][h][k] W_up,t^K[j][k]
// One CTA per (head h, loop query t, chunk of 8 sequences).  Lane l of a warp owns the
// components k = 128 c + 4 l .. + 3 of the reduction axis: the 8 query rows sit in its
// registers and each W_up,t^K row (r_k rows, LLA-2D: head h's columns) is read from
// global memory once per CTA as coalesced 16-byte loads, a warp taking every 8th row.
// A row's 8 partial sums are closed across the warp by recursive halving (9 shuffles),
// leaving sequence lane / 4's sum in lanes 4 (lane / 4) .. + 3.  d is covered in
// passes of 128 NCH components (NCH = 1 for d <= 128, so only the registers a head needs
// are held); the results gather in shared memory and leave as whole q_tilde rows.
// ---------------------------------------------------------------------------------
// sequences per combine CTA (one warp each): 16 when W_up,t^V is large enough that staging
// it once for more sequences pays, else 8 (smaller CTAs take SM slots sooner at the
// decode grid's tail)
constexpr int kBatchSmall = 8, kBatchLarge = 16;
constexpr int kPrologueSeqs = 8; // sequences per prologue CTA (the 8 partial sums of a lane)
constexpr int kPrologueThreads = 256;
constexpr int kPrologueWarps = kPrologueThreads / 32;
// W rows a warp keeps in flight per step: the kernel is bound by load latency, so a warp
// requests 8 rows (4 when a lane holds two 128-wide chunks) before it sums any of them
template <int NCH> constexpr int prologue_rows() { return NCH == 1 ? 8 : 4; }

// Sum over the warp of s[0..7] (one partial per sequence): returns the total of sequence
// lane / 4 (the same in the 4 lanes of a quad).
__device__ __forceinline__ float warp_sum8(float (&s)[8], int lane)
{
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
    float h4[4], h2[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) { // keep sequences 4 b4 + i, hand over the other half
        const float keep = b4 ? s[i + 4] : s[i], give = b4 ? s[i] : s[i + 4];
        h4[i] = keep + __shfl_xor_sync(0xffffffffu, give, 16);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float keep = b3 ? h4[i + 2] : h4[i], give = b3 ? h4[i] : h4[i + 2];
        h2[i] = keep + __shfl_xor_sync(0xffffffffu, give, 8);
    }
    float v = (b2 ? h2[1] : h2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? h2[0] : h2[1], 4);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    return v + __shfl_xor_sync(0xffffffffu, v, 1);
}

// 4 consecutive query components as floats (bf16: one 8-byte load; fp32: one 16-byte load)
template <typename T> __device__ __forceinline__ float4 load4(const T *p);
template <> __device__ __forceinline__ float4 load4<float>(const float *p)
{
    return *reinterpret_cast<const float4 *>(p);
}
template <> __device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16 *p)
{
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    return make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y));
}

__device__ __forceinline__ float dot4(float4 a, float4 b, float s)
{
    return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, fmaf(a.w, b.w, s))));
}

// ROPEQ: also append the rotated rotary query part (decoupled sub-key form).
template <typename T, bool ROPEQ, int NCH>
__global__ void __launch_bounds__(kPrologueThreads, 2) absorb_prologue_kernel(const DecodeArgs a)
{
    extern __shared__ float psm[]; // [kPrologueSeqs][r_k]: q_tilde rows of the chunk
    grid_launch_dependents();      // the decode grid may start streaming latents right away
    const int h = blockIdx.x, t = blockIdx.y, b0 = blockIdx.z * kPrologueSeqs;
    const int RK = a.r_k, d = a.d;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int tg = a.t0 + a.tq_off + t;
    const int ld = a.fold ? a.H * d : d;
    const float *wsrc = a.W_up_k + (a.fold ? (int64_t)tg * RK * ld + (int64_t)h * d
                                           : ((int64_t)h * a.T + tg) * RK * ld);
    const int nb = min(kPrologueSeqs, a.B - b0);
    const T *qbase = static_cast<const T *>(a.q) + ((int64_t)b0 * a.Tq_all + a.tq_off + t) * a.H * d + (int64_t)h * d;
    const int64_t qstride = (int64_t)a.Tq_all * a.H * d; // next sequence
    for (int k0 = 0; k0 < d; k0 += 128 * NCH) {
        // this lane's components of the pass: k0 + 128 c + 4 lane, c < NCH
        float4 qv[kPrologueSeqs][NCH];
        bool kin[NCH];
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int k = k0 + 128 * c + 4 * lane;
            kin[c] = k < d;
#pragma unroll
            for (int b = 0; b < kPrologueSeqs; ++b)
                qv[b][c] = kin[c] && b < nb ? load4<T>(qbase + b * qstride + k) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        // rows j = warp, warp + 8, ...; R rows' loads in flight per step
        constexpr int R = prologue_rows<NCH>();
        for (int j0 = warp; j0 < RK; j0 += R * kPrologueWarps) {
            float4 w[R][NCH];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int j = j0 + r * kPrologueWarps;
#pragma unroll
                for (int c = 0; c < NCH; ++c) {
                    const int k = k0 + 128 * c + 4 * lane;
                    w[r][c] = j < RK && kin[c] ? *reinterpret_cast<const float4 *>(wsrc + (int64_t)j * ld + k)
                                               : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int j = j0 + r * kPrologueWarps;
                if (j >= RK)
                    break; // warp-uniform: no sums (and no shuffles) for rows past r_k
                float s[kPrologueSeqs];
#pragma unroll
                for (int b = 0; b < kPrologueSeqs; ++b) {
                    s[b] = 0.f;
#pragma unroll
                    for (int c = 0; c < NCH; ++c)
                        s[b] = dot4(qv[b][c], w[r][c], s[b]);
                }
                const float tot = warp_sum8(s, lane); // uniform control flow: every lane shuffles
                if ((lane & 3) == 0) {
                    float *dst = psm + (lane >> 2) * RK + j;
                    *dst = k0 == 0 ? tot : *dst + tot; // the same lane owns (sequence, j) in every pass
                }
            }
        }
    }
    __syncthreads();
    const float sc = a.scale * kLog2e;
    const int qt_ld = RK + a.d_rope;
    for (int e = threadIdx.x; e < nb * RK; e += kPrologueThreads) {
        const int bl = e / RK, j = e - bl * RK;
        const int64_t u = (int64_t)(b0 + bl) * a.H + h;
        a.qt[(u * a.Tq_all + a.tq_off + t) * qt_ld + j] = psm[bl * RK + j] * sc;
    }
    if (ROPEQ) {
        // decoupled rotary part: q_rope rotated at the query position, appended to q_tilde;
        // pair i (i, i + d_r/2 or 2i, 2i+1) turns by q_pos * base^(-2i/d_r), angle in fp64
        const int dr = a.d_rope, np = dr / 2;
        for (int o = threadIdx.x; o < nb * np; o += kPrologueThreads) {
            const int bl = o / np, i = o - bl * np;
            const int b = b0 + bl;
            const int ia = a.rope_style == LLA_ROPE_INTERLEAVED ? 2 * i : i;
            const int ib = a.rope_style == LLA_ROPE_INTERLEAVED ? 2 * i + 1 : i + np;
            const T *qr = static_cast<const T *>(a.q_rope) + (((int64_t)b * a.Tq_all + a.tq_off + t) * a.H + h) * dr;
            const float xa = Elem<T>::to_f(qr[ia]), xb = Elem<T>::to_f(qr[ib]);
            const double ang = (double)a.q_pos[b] * pow((double)a.rope_base, -2.0 * i / dr);
            const float red = (float)(ang - 6.283185307179586 * rint(ang * 0.15915494309189535));
            float sn, cs;
            sincosf(red, &sn, &cs);
            const int64_t u = (int64_t)b * a.H + h;
            float *dst = a.qt + (u * a.Tq_all + a.tq_off + t) * qt_ld + RK;
            dst[ia] = (xa * cs - xb * sn) * sc;
            dst[ib] = (xa * sn + xb * cs) * sc;
        }
    }
}

// ---------------------------------------------------------------------------------
// a4: cross-segment combine + output projection.  A CTA holds NSEQ sequences of one
// (head h, loop query t); warp w merges the records of sequence b0 + w:
//   M = max_s m_s,  L = sum_s l_s 2^(m_s - M),  o_lat = sum_s acc_s 2^(m_s - M) / L,
//   lse = ln2 (M + log2 L) + scale * q . mu_t^K   (-inf and out = 0 for an empty context)
// (lane c owns record columns 4c + 128 i), then the CTA projects all of them at once:
//   out[b] = o_lat W_up,t^V + mu_t^V,
// W_up,t^V (r_v x d) read once into shared memory by bulk copies.
// Latency design: everything that does not come from the decode grid (W_up,t^V,
// mu_t^V, mu_t^K, q, ctx_lens) is requested before the programmatic-launch wait; after
// it, the unit's record count and its first kSpecRecords records are loaded in one
// round (slots past the count lie inside the workspace and are ignored), so the
// combine adds two dependent global-load latencies to the end of the decode.
// ---------------------------------------------------------------------------------

constexpr int kSpecRecords = 4;      // records fetched before the count is known
constexpr int kMaxOutGroups = 4;     // d <= 512

template <typename T> struct Vec4;
template <> struct Vec4<float> {
    static __device__ __forceinline__ float4 load(const float *p) { return *reinterpret_cast<const float4 *>(p); }
    static __device__ __forceinline__ void store(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
};
template <> struct Vec4<__nv_bfloat16> {
    static __device__ __forceinline__ float4 load(const __nv_bfloat16 *p)
    {
        const uint2 u = *reinterpret_cast<const uint2 *>(p);
        return make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y));
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, float4 v)
    {
        const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
        uint2 u;
        u.x = *reinterpret_cast<const uint32_t *>(&lo);
        u.y = *reinterpret_cast<const uint32_t *>(&hi);
        *reinterpret_cast<uint2 *>(p) = u;
    }
};

__device__ __forceinline__ float4 f4_fma(float s, float4 x, float4 y)
{
    return make_float4(fmaf(s, x.x, y.x), fmaf(s, x.y, y.y), fmaf(s, x.z, y.z), fmaf(s, x.w, y.w));
}
__device__ __forceinline__ float4 f4_scale(float s, float4 x) { return make_float4(s * x.x, s * x.y, s * x.z, s * x.w); }

// Records [s0, s0 + n) of one unit in registers: (m, l) and this lane's RG column groups.
template <int RG, int SPEC> struct RecBatch {
    float2 ml[SPEC];
    float4 rv[SPEC][RG];

    // Loads the records s0 + k < lim (k < SPEC); lane c holds columns 4c + 128 g.
    __device__ __forceinline__ void load(const float *rec0, int s0, int lim, int ps, int RV, int lane)
    {
#pragma unroll
        for (int k = 0; k < SPEC; ++k) {
            const int s = s0 + k;
            ml[k] = make_float2(-INFINITY, 0.f);
#pragma unroll
            for (int g = 0; g < RG; ++g)
                rv[k][g] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (s < lim) {
                ml[k] = *reinterpret_cast<const float2 *>(rec0 + (int64_t)s * ps + RV);
#pragma unroll
                for (int g = 0; g < RG; ++g) {
                    const int c = 4 * lane + 128 * g;
                    if (c < RV)
                        rv[k][g] = Vec4<float>::load(rec0 + (int64_t)s * ps + c);
                }
            }
        }
    }

    // Folds records k < n into the running (M, L, acc).
    __device__ __forceinline__ void merge(int n, float &M, float &L, float4 (&acc)[RG]) const
    {
        float Mn = M;
#pragma unroll
        for (int k = 0; k < SPEC; ++k)
            if (k < n)
                Mn = fmaxf(Mn, ml[k].x);
        if (Mn == -INFINITY)
            return; // nothing but empty records so far
        const float al = M == -INFINITY ? 0.f : exp2f(M - Mn);
        L *= al;
#pragma unroll
        for (int g = 0; g < RG; ++g)
            acc[g] = f4_scale(al, acc[g]);
#pragma unroll
        for (int k = 0; k < SPEC; ++k) {
            if (k < n && ml[k].x != -INFINITY) {
                const float w = exp2f(ml[k].x - Mn);
                L = fmaf(w, ml[k].y, L);
#pragma unroll
                for (int g = 0; g < RG; ++g)
                    acc[g] = f4_fma(w, rv[k][g], acc[g]);
            }
        }
        M = Mn;
    }
};

// REC: records carry d-wide outputs of the reconstruct form (mu and the q.mu_t^K score term
// already included), so the output is the merged record itself.  RG = record width / 128,
// rounded up.  WIN: hybrid form, merge the window part (a.win_part) as well.
// Registers per thread the launch bounds allow: 64 only for the plain bf16 form; wide record
// batches, the window merge and fp32 inputs get 128 so that nothing spills -- their grids
// (H x Tq x B / NSEQ CTAs) are far below that many CTAs per SM anyway.
template <typename T, bool WIN, int RG, int SPEC, int NSEQ> constexpr int combine_min_blocks()
{
    return (RG == 1 && !WIN && SPEC == kSpecRecords && sizeof(T) == 2 ? 2 : 1) * (NSEQ == kBatchSmall ? 2 : 1);
}

template <typename T, typename O, bool REC, int RG, bool WIN, int SPEC, int NSEQ>
__global__ void __launch_bounds__(32 * NSEQ, (combine_min_blocks<T, WIN, RG, SPEC, NSEQ>()))
    decode_combine_kernel(const DecodeArgs a)
{
    constexpr int kBatchSeqs = NSEQ, kCombineThreads = 32 * NSEQ;
    extern __shared__ __align__(16) float csm[];
    const int h = blockIdx.x, tl = blockIdx.y, b0 = blockIdx.z * kBatchSeqs;
    const int t = a.tq_off + tl; // indexes q / out / lse / records
    const int d = a.d, RV = REC ? a.d : a.r_v, ps = part_stride(RV);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int b = b0 + warp;
    const bool active = b < a.B;
    // shared memory of the projection: W_up,t^V [RV][d] | mu_t^V [d] | o_lat [8][RV + 4] |
    // per sequence (valid, fa, fw, -) [8][4] | mbarrier of the W copy
    const int osl = RV + 4; // row stride of o_lat: 8 rows fall in distinct 16-byte bank groups
    float *W = csm;
    float *muv = W + RV * d;
    float *os = muv + d;
    float *sq = os + kBatchSeqs * osl;
    const uint32_t wbar = smem_u32(sq + kBatchSeqs * 4);
    const int tg = a.t0 + t;
    const int ld = a.fold ? a.H * d : d;
    const int64_t wbase = a.fold ? (int64_t)tg * RV * ld + (int64_t)h * d : ((int64_t)h * a.T + tg) * RV * ld;
    const int64_t mbase = a.fold ? (int64_t)tg * ld + (int64_t)h * d : ((int64_t)h * a.T + tg) * ld;
    const int64_t u = (int64_t)b * a.H + h;

    // ---- inputs of the call (not written by the decode grid)
    if (!REC) {
        // W_up,t^V rows (d fp32 each, 16-byte aligned) come in by bulk copies issued by
        // warp 0; they land while the records are merged
        if (threadIdx.x == 0) {
            mbar_init(wbar, 1);
            fence_barrier_init();
        }
        __syncthreads();
        if (warp == 0) {
            if (lane == 0)
                mbar_arrive_expect_tx(wbar, (uint32_t)(RV * d * 4));
            __syncwarp();
            if (!a.fold) {
                // per-head layout: the (head, loop) block is contiguous -- a few large copies
                constexpr uint32_t kPiece = 64 * 1024;
                const uint32_t total = (uint32_t)(RV * d * 4);
                for (uint32_t o = (uint32_t)lane * kPiece; o < total; o += 32u * kPiece)
                    bulk_copy_g2s(smem_u32(W) + o, reinterpret_cast<const uint8_t *>(a.W_up_v + wbase) + o,
                                  total - o < kPiece ? total - o : kPiece, wbar);
            } else {
                // LLA-2D: head h's d columns of each folded row
                for (int j = lane; j < RV; j += 32)
                    bulk_copy_g2s(smem_u32(W + j * d), a.W_up_v + wbase + (int64_t)j * ld, (uint32_t)(d * 4), wbar);
            }
        }
        for (int k = threadIdx.x; k < d; k += kCombineThreads)
            muv[k] = a.mu_v[mbase + k];
    }
    int len = 0;
    float qm = 0.f;
    if (active) {
        len = a.ctx_lens[b];
        if (!REC) {
            const T *qrow = static_cast<const T *>(a.q) + (((int64_t)b * a.Tq_all + t) * a.H + h) * d;
            for (int c = 4 * lane; c < d; c += 128) {
                const float4 qv = Vec4<T>::load(qrow + c);
                const float4 mk = Vec4<float>::load(a.mu_k + mbase + c);
                qm = fmaf(qv.x, mk.x, fmaf(qv.y, mk.y, fmaf(qv.z, mk.z, fmaf(qv.w, mk.w, qm))));
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                qm += __shfl_xor_sync(0xffffffffu, qm, off);
        }
    }

    grid_dependency_wait(); // records and counts come from the preceding decode grid

    // hybrid form: the window part of this (unit, query), complete before this grid's wait
    // returns; its first column group is fetched here, wider rows group by group below
    constexpr bool win = WIN;
    const float *wrec = win ? a.win_part + (u * a.Tq_all + t) * part_stride(d) : nullptr;
    float wl = -INFINITY;
    float4 wo0 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (win && active) {
        wl = wrec[d];
        if (REC && 4 * lane < d)
            wo0 = Vec4<float>::load(wrec + 4 * lane);
    }

    float M = -INFINITY, L = 0.f;
    float4 acc[RG];
#pragma unroll
    for (int g = 0; g < RG; ++g)
        acc[g] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (active && len > 0) {
        const float *rec0 = a.part + (u * a.Tq_all + t) * a.seg_max * ps;
        const int cnt = a.counts[u];
        RecBatch<RG, SPEC> rb;
        rb.load(rec0, 0, a.seg_max, ps, RV, lane); // issued together with the count
        const int S = min(cnt, a.seg_max);
        rb.merge(min(S, SPEC), M, L, acc);
        for (int s0 = SPEC; s0 < S; s0 += SPEC) { // long contexts / many splits
            rb.load(rec0, s0, S, ps, RV, lane);
            rb.merge(min(S - s0, SPEC), M, L, acc);
        }
    }
    const float invL = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
    for (int g = 0; g < RG; ++g)
        acc[g] = f4_scale(invL, acc[g]); // o_lat (or the output itself for REC)
    float lse = L > 0.f ? kLn2 * (M + log2f(L)) + (REC ? 0.f : a.scale * qm) : -INFINITY;
    // hybrid form: out = fa * out_lat + fw * out_win, weights from the two log-sum-exps
    float fa = 1.f, fw = 0.f;
    if (win) {
        const float l2 = L > 0.f ? M + log2f(L) + (REC ? 0.f : a.scale * qm * kLog2e) : -INFINITY;
        const float mm = fmaxf(l2, wl);
        fa = 0.f;
        lse = -INFINITY;
        if (mm != -INFINITY) {
            const float ea = exp2f(l2 - mm), ew = exp2f(wl - mm), sum = ea + ew;
            fa = ea / sum;
            fw = ew / sum;
            lse = kLn2 * (mm + log2f(sum));
        }
    }
    if (active && lane == 0 && a.lse != nullptr)
        a.lse[((int64_t)b * a.Tq_all + t) * a.H + h] = lse;

    if (REC) {
        O *orow = static_cast<O *>(a.out) + (((int64_t)b * a.Tq_all + t) * a.H + h) * d;
        if (active) {
#pragma unroll
            for (int g = 0; g < RG; ++g) {
                const int c = 4 * lane + 128 * g;
                if (c < d) {
                    float4 o = acc[g];
                    if (win)
                        o = f4_fma(fw, g == 0 ? wo0 : Vec4<float>::load(wrec + c), f4_scale(fa, o));
                    Vec4<O>::store(orow + c, o);
                }
            }
        }
        return;
    }

    // ---- projection out[b] = o_lat[b] W_up,t^V + mu_t^V for the CTA's NSEQ sequences at
    // once: lane l works for sequence l / (32 / NSEQ) and column group l % (32 / NSEQ) of
    // the warp's; warp w owns the groups (32 / NSEQ) (w + NSEQ i) + l % (32 / NSEQ) (4
    // columns each), so a W row's columns of a warp are one shared-memory wavefront
    // serving all NSEQ sequences
    const bool valid = active && L > 0.f;
#pragma unroll
    for (int g = 0; g < RG; ++g) {
        const int c = 4 * lane + 128 * g;
        if (c < RV)
            *reinterpret_cast<float4 *>(os + warp * osl + c) = valid ? acc[g] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (lane == 0)
        *reinterpret_cast<float4 *>(sq + 4 * warp) = make_float4(valid ? 1.f : 0.f, fa, fw, 0.f);
    const bool landed = mbar_wait_bounded(wbar, 0);
    if (__syncthreads_or(!landed)) { // o_lat, flags and W all in place, or a copy never landed
        if (threadIdx.x == 0)
            report_status(a.status, LLA_ERR_DEVICE_TIMEOUT);
        return;
    }
    constexpr int GPL = 32 / NSEQ; // column groups per warp and W row
    const int bs = lane / GPL, qd = lane % GPL, sb = b0 + bs;
    const float4 flags = *reinterpret_cast<const float4 *>(sq + 4 * bs);
    const int ncg = d >> 2;
    float4 o4[kMaxOutGroups];
#pragma unroll
    for (int i = 0; i < kMaxOutGroups; ++i)
        o4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (flags.x != 0.f) {
        const float *orow = os + bs * osl;
#pragma unroll 2
        for (int j = 0; j < RV; j += 4) {
            const float4 ov = *reinterpret_cast<const float4 *>(orow + j);
#pragma unroll
            for (int i = 0; i < kMaxOutGroups; ++i) {
                const int cg = GPL * (warp + NSEQ * i) + qd;
                if (cg < ncg) {
                    const float *wc = W + j * d + 4 * cg;
                    o4[i] = f4_fma(ov.x, *reinterpret_cast<const float4 *>(wc), o4[i]);
                    o4[i] = f4_fma(ov.y, *reinterpret_cast<const float4 *>(wc + d), o4[i]);
                    o4[i] = f4_fma(ov.z, *reinterpret_cast<const float4 *>(wc + 2 * d), o4[i]);
                    o4[i] = f4_fma(ov.w, *reinterpret_cast<const float4 *>(wc + 3 * d), o4[i]);
                }
            }
        }
    }
    if (sb >= a.B)
        return;
    O *orow = static_cast<O *>(a.out) + (((int64_t)sb * a.Tq_all + t) * a.H + h) * d;
    const float *wrow = win ? a.win_part + (((int64_t)sb * a.H + h) * a.Tq_all + t) * part_stride(d) : nullptr;
#pragma unroll
    for (int i = 0; i < kMaxOutGroups; ++i) {
        const int cg = GPL * (warp + NSEQ * i) + qd;
        if (cg < ncg) {
            const int c = 4 * cg;
            float4 o = o4[i];
            if (flags.x != 0.f) {
                const float4 m = *reinterpret_cast<const float4 *>(muv + c);
                o = make_float4(o.x + m.x, o.y + m.y, o.z + m.z, o.w + m.w);
            }
            if (win)
                o = f4_fma(flags.z, Vec4<float>::load(wrow + c), f4_scale(flags.y, o));
            Vec4<O>::store(orow + c, o);
        }
    }
}

} // namespace

bool decode_absorb_supported(int dtype, int r_k, int r_v, int d, int fold)
{
    if (fold != LLA_PER_HEAD || d % 32 != 0 || d > 1024)
        return false;
    if (dtype == LLA_BF16)
        return (r_k == 16 && r_v == 32) || (r_k == 8 && r_v == 16) || (r_k == 16 && r_v == 16);
    return (r_k == 8 && r_v == 16) || (r_k == 16 && r_v == 32) || (r_k == 4 && r_v == 8);
}

cudaError_t launch_decode_absorb(const DecodeArgs &a, int dtype, int ctas, cudaStream_t stream,
                                 bool *supported)
{
    *supported = true;
    if (dtype == LLA_BF16) {
        using B = __nv_bfloat16;
        if (a.r_k == 16 && a.r_v == 32) return launch_tq<B, 16, 32>(a, ctas, stream);
        if (a.r_k == 8 && a.r_v == 16) return launch_tq<B, 8, 16>(a, ctas, stream);
        if (a.r_k == 16 && a.r_v == 16) return launch_tq<B, 16, 16>(a, ctas, stream);
    } else {
        if (a.r_k == 8 && a.r_v == 16) return launch_tq<float, 8, 16>(a, ctas, stream);
        if (a.r_k == 16 && a.r_v == 32) return launch_tq<float, 16, 32>(a, ctas, stream);
        if (a.r_k == 4 && a.r_v == 8) return launch_tq<float, 4, 8>(a, ctas, stream);
    }
    *supported = false;
    return cudaSuccess;
}

cudaError_t launch_absorb_prologue(const DecodeArgs &a, int dtype, cudaStream_t stream)
{
    dim3 grid(a.H, a.Tq, (a.B + kPrologueSeqs - 1) / kPrologueSeqs);
    const size_t smem = sizeof(float) * (size_t)kPrologueSeqs * a.r_k; // q_tilde rows of the chunk
    if (smem > 200 * 1024)
        return cudaErrorInvalidValue;
    auto pick = [&](auto tag) {
        using T = decltype(tag);
        if (a.d <= 128)
            return a.d_rope > 0 ? absorb_prologue_kernel<T, true, 1> : absorb_prologue_kernel<T, false, 1>;
        return a.d_rope > 0 ? absorb_prologue_kernel<T, true, 2> : absorb_prologue_kernel<T, false, 2>;
    };
    auto k = dtype == LLA_BF16 ? pick(__nv_bfloat16{}) : pick(float{});
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, kPrologueThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

template <typename T, typename O, int RG, int SPEC, int NSEQ>
static cudaError_t launch_combine_n(const DecodeArgs &a, cudaStream_t stream)
{
    const int rv = a.recon ? a.d : a.r_v;
    // W_up,t^V + mu_t^V + o_lat rows + per-sequence flags + the copy's mbarrier
    const size_t smem = a.recon ? 16
                                : sizeof(float) * ((size_t)rv * a.d + a.d + (size_t)NSEQ * (rv + 4) + 4 * NSEQ) + 16;
    if (smem > 200 * 1024)
        return cudaErrorInvalidValue;
    const bool win = a.win_part != nullptr;
    auto k = a.recon ? (win ? decode_combine_kernel<T, O, true, RG, true, SPEC, NSEQ>
                            : decode_combine_kernel<T, O, true, RG, false, SPEC, NSEQ>)
                     : (win ? decode_combine_kernel<T, O, false, RG, true, SPEC, NSEQ>
                            : decode_combine_kernel<T, O, false, RG, false, SPEC, NSEQ>);
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.H, a.Tq, (a.B + NSEQ - 1) / NSEQ);
    cfg.blockDim = dim3(32 * NSEQ);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization; // stage W_up while decode ends
    attr[0].val.programmaticStreamSerializationAllowed = a.serial ? 0 : 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, a);
}

template <typename T, typename O, int RG, int SPEC>
static cudaError_t launch_combine_t(const DecodeArgs &a, cudaStream_t stream)
{
    // a W_up,t^V of 32 KB or more is worth staging once for 16 sequences
    const bool large = !a.recon && (size_t)a.r_v * a.d * sizeof(float) >= 32 * 1024;
    return large ? launch_combine_n<T, O, RG, SPEC, kBatchLarge>(a, stream)
                 : launch_combine_n<T, O, RG, SPEC, kBatchSmall>(a, stream);
}

template <typename T, typename O>
static cudaError_t launch_combine_rg(const DecodeArgs &a, int rv, cudaStream_t stream)
{
    // many record slots per unit (LLA-2D's short shares, long contexts): 8 records per load
    // round instead of 4, so fewer dependent rounds; the small batch keeps the register count
    // (and the CTAs resident beside a finishing decode grid) when a unit has <= 4 records
    if (rv > 128)
        return launch_combine_t<T, O, 2, kSpecRecords>(a, stream);
    return a.seg_max > kSpecRecords ? launch_combine_t<T, O, 1, 2 * kSpecRecords>(a, stream)
                                    : launch_combine_t<T, O, 1, kSpecRecords>(a, stream);
}

// The combine holds W_up,t^V (r_v x d fp32) in shared memory for its CTA's sequences:
// shapes whose W does not fit are refused before anything is queued.
bool decode_combine_supported(int r_v, int d, bool recon)
{
    const int rv = recon ? d : r_v;
    if (rv > 256 || d > 128 * kMaxOutGroups || rv % 4 != 0 || d % 4 != 0)
        return false;
    if (recon)
        return true;
    const int nseq = (size_t)r_v * d * sizeof(float) >= 32 * 1024 ? kBatchLarge : kBatchSmall;
    const size_t smem = sizeof(float) * ((size_t)rv * d + d + (size_t)nseq * (rv + 4) + 4 * nseq) + 16;
    return smem <= 200 * 1024;
}

cudaError_t launch_decode_combine(const DecodeArgs &a, int dtype, int out_dtype, cudaStream_t stream)
{
    const int rv = a.recon ? a.d : a.r_v;
    if (rv > 256 || a.d > 128 * kMaxOutGroups || rv % 4 != 0 || a.d % 4 != 0)
        return cudaErrorInvalidValue; // a lane holds 16-byte groups of a record / output row
    using BF = __nv_bfloat16;
    if (dtype == LLA_BF16 && out_dtype == LLA_BF16)
        return launch_combine_rg<BF, BF>(a, rv, stream);
    if (dtype == LLA_BF16)
        return launch_combine_rg<BF, float>(a, rv, stream);
    if (out_dtype == LLA_BF16)
        return launch_combine_rg<float, BF>(a, rv, stream);
    return launch_combine_rg<float, float>(a, rv, stream);
}

} // namespace lla
