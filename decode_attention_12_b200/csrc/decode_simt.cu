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
#include "decode.cuh"

namespace lla {
namespace {

constexpr int kThreads = 64;
constexpr int kWarps = kThreads / 32;
constexpr int kTokensPerThread = 2;
constexpr int kStages = 3;
constexpr int kTile = kThreads * kTokensPerThread;
constexpr float kRescaleThreshold = 8.0f; // log2 units

__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

struct TileDesc {
    int64_t row;            // first cache row of the tile within the head's plane
    int32_t b, h, n0, rows; // sequence, head, first token (within the sequence), rows
    int32_t u, j, n_u;      // unit id, record slot within the unit, records of the unit
    int32_t flags;          // bit 0: first tile of a segment, bit 1: last tile of a segment
};

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

// Largest b in [0, B) with H * pref[b] <= pos (pref is the exclusive prefix of lengths).
__device__ __forceinline__ int find_seq(const int64_t *pref, int B, int H, int64_t pos)
{
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((int64_t)H * pref[mid] <= pos)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// Walks the token share [pos, end) of one CTA, unit segment by unit segment, tile by tile.
struct ShareWalk {
    int64_t pos, end, chunk, seq0;
    int32_t b, h, n, seg_end, u, j, n_u;
    bool in_seg;

    __device__ void start(int64_t p, int64_t e, int64_t ch)
    {
        pos = p;
        end = e;
        chunk = ch;
        in_seg = false;
    }
    // Next tile; false when the share is exhausted.
    __device__ bool next(const int64_t *pref, const int64_t *starts, int B, int H, TileDesc &d)
    {
        if (!in_seg) {
            if (pos >= end)
                return false;
            b = find_seq(pref, B, H, pos);
            const int len = (int)(pref[b + 1] - pref[b]);
            seq0 = starts[b];
            const int64_t off = pos - (int64_t)H * pref[b];
            h = (int)(off / len);
            n = (int)(off - (int64_t)h * len);
            const int64_t take = min((int64_t)(len - n), end - pos);
            seg_end = n + (int)take;
            pos += take;
            u = b * H + h;
            const int64_t U = (int64_t)H * pref[b] + (int64_t)h * len; // unit start in the stream
            const int64_t c_first = U / chunk, c_last = (U + len - 1) / chunk;
            j = (int)(blockIdx.x - c_first);
            n_u = (int)(c_last - c_first + 1);
            in_seg = true;
            d.flags = 1;
        } else {
            d.flags = 0;
        }
        d.row = seq0 + n;
        d.b = b;
        d.h = h;
        d.n0 = n;
        d.rows = min(kTile, seg_end - n);
        d.u = u;
        d.j = j;
        d.n_u = n_u;
        n += d.rows;
        if (n >= seg_end) {
            d.flags |= 2;
            in_seg = false;
        }
        return true;
    }
};

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

    // ---- exclusive prefix of the context lengths (work split of the token stream):
    // each thread sums a contiguous slice, a warp scan and a cross-warp offset follow.
    {
        const int per = (B + kThreads - 1) / kThreads;
        const int b0 = min(B, tid * per), b1 = min(B, b0 + per);
        int64_t local = 0;
        for (int b = b0; b < b1; ++b)
            local += a.ctx_lens[b];
        int64_t x = local;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off)
                x += y;
        }
        int64_t *wtot = reinterpret_cast<int64_t *>(red);
        if (lane == 31)
            wtot[warp] = x;
        if (tid == 0) {
            for (int s2 = 0; s2 < kStages; ++s2)
                mbar_init(bar0 + 8 * s2, 1);
            misc[1] = 0;
            fence_barrier_init();
        }
        __syncthreads();
        int64_t run = x - local;
        for (int w = 0; w < warp; ++w)
            run += wtot[w];
        for (int b = b0; b < b1; ++b) {
            pref[b] = run;
            run += a.ctx_lens[b];
        }
        if (tid == kThreads - 1)
            pref[B] = run;
    }
    __syncthreads();
    const int64_t total = (int64_t)H * pref[B];
    int64_t chunk = (total + gridDim.x - 1) / gridDim.x;
    if (chunk < a.chunk_min)
        chunk = a.chunk_min;
    const int64_t s0 = (int64_t)blockIdx.x * chunk;
    const int64_t s1 = min(total, s0 + chunk);
    if (s0 >= s1)
        return; // uniform: nothing for this CTA

    const T *gk = static_cast<const T *>(a.k);
    const T *gv = static_cast<const T *>(a.v);
    uint8_t *ring = smem;
    ShareWalk walk; // producer state (thread 0 only)
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
        if (!mbar_wait_bounded(bar0 + 8 * stage, (i / kStages) & 1)) {
            misc[1] = 1; // every writer stores 1
        } else {
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
        __syncthreads();
        if (misc[1]) {
            failed_at = i;
            break;
        }
        if (tid == 0 && i + kStages < ntiles)
            issue(stage);
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
// grid (B*H, Tq); one warp per latent dimension j.  LLA-2D reads head h's columns.
// ---------------------------------------------------------------------------------
template <typename T>
__global__ void absorb_prologue_kernel(const DecodeArgs a)
{
    const int u = blockIdx.x, t = blockIdx.y;
    const int b = u / a.H, h = u - b * a.H;
    const int j = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (j >= a.r_k)
        return;
    const int tg = a.t0 + a.tq_off + t;
    const int ld = a.fold ? a.H * a.d : a.d;
    const float *w = a.W_up_k + (a.fold ? ((int64_t)tg * a.r_k + j) * ld + (int64_t)h * a.d
                                        : (((int64_t)h * a.T + tg) * a.r_k + j) * ld);
    const T *qrow = static_cast<const T *>(a.q) + (((int64_t)b * a.Tq_all + a.tq_off + t) * a.H + h) * a.d;
    float acc = 0.f;
    for (int k = lane; k < a.d; k += 32)
        acc = fmaf(Elem<T>::to_f(qrow[k]), w[k], acc);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0)
        a.qt[((int64_t)u * a.Tq_all + a.tq_off + t) * a.r_k + j] = acc * a.scale * kLog2e;
}

// ---------------------------------------------------------------------------------
// a4: cross-segment combine + output projection.
//   M = max_s m_s,  L = sum_s l_s 2^(m_s - M),  o_lat = sum_s acc_s 2^(m_s - M) / L
//   out = o_lat W_up,t^V + mu_t^V,   lse = ln2 (M + log2 L) + scale * q . mu_t^K
// One CTA per (loop query, head, sequence); thread k owns output dims k, k+128, ...
// ---------------------------------------------------------------------------------
constexpr int kCombineThreads = 128;

template <typename T, typename O>
__global__ void __launch_bounds__(kCombineThreads) decode_combine_kernel(const DecodeArgs a)
{
    extern __shared__ float csm[]; // o_lat [r_v], w [seg_max], red [8]
    const int t = a.tq_off + blockIdx.x, h = blockIdx.y, b = blockIdx.z; // t indexes q/out/lse
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int RV = a.r_v, ps = part_stride(RV);
    const int u = b * a.H + h;
    const int len = a.ctx_lens[b];
    const int S = len > 0 ? min(a.counts[u], a.seg_max) : 0;
    float *olat = csm;
    float *w = csm + RV;
    float *red = w + a.seg_max;
    const float *rec0 = a.part + ((int64_t)u * a.Tq_all + t) * a.seg_max * ps;

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
    if (a.r_k > 32)
        return cudaErrorInvalidValue;
    dim3 grid(a.B * a.H, a.Tq);
    const int threads = 32 * a.r_k;
    if (dtype == LLA_BF16)
        absorb_prologue_kernel<__nv_bfloat16><<<grid, threads, 0, stream>>>(a);
    else
        absorb_prologue_kernel<float><<<grid, threads, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_decode_combine(const DecodeArgs &a, int dtype, int out_dtype, cudaStream_t stream)
{
    dim3 grid(a.Tq, a.H, a.B);
    const size_t smem = sizeof(float) * (a.r_v + a.seg_max + 8);
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
