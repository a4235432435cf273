// decode_mma2d.cu -- LLA-2D decode attention on warp-level tensor cores: one latent per
// (token, layer) serves all H heads, so every latent tile is read once for all of a
// sequence's queries.
//
// "Looped Latent Attention: Cross-Loop KV Compression for Looped Transformers": review
// page abstract (LLA-2D folds the head axis into the cross-loop latent), "What carries
// the argument" (Eq. 3) and the Pith verdict record's desk-editor letter (absorbed form):
// head h uses the d columns h*d .. h*d+d-1 of the folded W_up,t and mu_t, so per sequence
// the queries of this pass form one matrix
//     Q_tilde [H*Tq x r_k],  row h*Tq + t = scale * q[b][t][h] W_up,t,h^K^T  (prologue grid)
// and the two contractions of a token tile are tensor-core MMAs on 16-row tiles of it:
//     S[rows x tok] = Q_tilde . C_K^T,   O[rows x r_v] += P . C_V
// with the bf16 hi + lo parts of q_tilde and p (all 16 fragment rows are queries).  Partial
// records go to the per-(sequence, head) layout of the other decode kernels, so the same
// combine applies the head-h slice of W_up,t^V.
//
// Four consumer warps: warp w owns row tile w % RT (RT = ceil(H*Tq / 16) <= 4) and token
// groups of 32 of every tile; with RT < 4 the warps of one row tile split the tile's
// tokens and merge their online-softmax states at a segment end.  A producer warp streams
// tiles of the folded plane with 2-D TMA copies (128-byte swizzle) into a 3-stage ring.
// Units of the persistent work split are sequences.
#include "mma_common.cuh"

namespace lla {
namespace {
using namespace mma;

template <int RK, int RV, int RT> struct M2Cfg {
    static constexpr int NW = 4;
    static constexpr int TG = NW / RT;          // warps per row tile
    static constexpr int BPW = RT == 4 ? 2 : 1; // 32-token blocks per warp and tile
    static constexpr int TILE = 32 * BPW * TG;  // 64, 64, 128 tokens for RT = 4, 2, 1
    static constexpr int THREADS = (NW + 1) * 32;
    static constexpr int CONSUMERS = NW * 32;
    using LK = TileLayout<RK, TILE>;
    using LV = TileLayout<RV, TILE>;
    static constexpr int KS = RK / 16, NTV = RV / 8;
    static constexpr int K_BYTES = LK::BYTES, V_BYTES = LV::BYTES;
    static constexpr int STAGE = align1024(K_BYTES + V_BYTES);
    static constexpr int STAGES = 3;
    static constexpr int RING = STAGES * STAGE;
    static constexpr int MRG_FLOATS = TG > 1 ? NW * 16 * (RV + 2) : 0; // [NW][16][RV + 2]
    static constexpr int MRG_OFF = RING;
    static constexpr int BAR_OFF = (MRG_OFF + MRG_FLOATS * 4 + 15) & ~15; // full[S], empty[S]
    static constexpr int MISC_OFF = BAR_OFF + 2 * STAGES * 8;
    static constexpr int SCR_OFF = (MISC_OFF + 16 + 15) & ~15; // int64 [NW + 1]
    static constexpr int PREF_OFF = SCR_OFF + (NW + 1) * 8;    // int64 [B + 1]
    static int smem_bytes(int B) { return PREF_OFF + 8 * (B + 1) + 1024; }
    static_assert(RK % 16 == 0 && RV % 16 == 0, "ranks in whole k16 steps / n8 pairs");
};

// A record of one (sequence, head, loop) row: acc[RV], m, l.
__device__ __forceinline__ float *rec_row(const DecodeArgs &a, int b, int r, int j, int RV)
{
    const int h = r / a.Tq, t = r - h * a.Tq;
    const int64_t u = (int64_t)b * a.H + h;
    return a.part + ((u * a.Tq_all + a.tq_off + t) * a.seg_max + j) * part_stride(RV);
}

template <int RK, int RV, int RT>
__global__ void __launch_bounds__(160, 2)
    decode_absorb_2d_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_kt,
                            const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_vt,
                            const DecodeArgs a)
{
    using C = M2Cfg<RK, RV, RT>;
    constexpr int kWarps = C::NW, kThreads = C::THREADS, kConsumers = C::CONSUMERS, kTile = C::TILE;
    constexpr int kStages = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    // aligned by arithmetic on the shared array itself, so accesses stay shared-space loads
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float *mrg = reinterpret_cast<float *>(smem + C::MRG_OFF);
    volatile int *misc = reinterpret_cast<volatile int *>(smem + C::MISC_OFF); // [0] error flag
    int64_t *pref = reinterpret_cast<int64_t *>(smem + C::PREF_OFF);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t full0 = sbase + C::BAR_OFF, empty0 = full0 + 8 * kStages;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, tq = lane & 3;
    const int B = a.B, rows_all = a.H * a.Tq; // query rows of one sequence in this pass

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, kWarps);
        }
        misc[0] = 0;
        fence_barrier_init();
    }
    block_length_prefix<kThreads>(a.ctx_lens, B, pref, reinterpret_cast<int64_t *>(smem + C::SCR_OFF));
    grid_launch_dependents(); // the combine grid may take SM slots as these CTAs exit
    int64_t s0, s1, chunk;
    cta_share(pref, B, 1, a.chunk_min, s0, s1, chunk); // units: sequences
    if (s0 >= s1)
        return;

    ShareWalk<kTile> walk;
    walk.start(s0, s1, chunk);
    TileDesc d;
    int issued = 0;

    if (warp == kWarps) {
        // ================= producer warp: one lane streams the folded plane =================
        if (lane == 0) {
            while (walk.next(pref, a.seq_start, B, 1, d)) {
                const int i = issued, stage = i % kStages;
                if (i >= kStages && !mbar_wait_bounded(empty0 + 8 * stage, ((i / kStages) - 1) & 1)) {
                    misc[0] = 1;
                    break;
                }
                if (misc[0])
                    break;
                const uint32_t st = sbase + stage * C::STAGE, bar = full0 + 8 * stage;
                const int nbox = (d.rows + kBox - 1) / kBox;
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(bar, nbox * kBox * (RK + RV) * 2);
                const int y0 = (int)d.row;
                for (int bx = 0; bx < nbox; ++bx) {
                    const int y = y0 + bx * kBox;
#pragma unroll
                    for (int blk = 0; blk < C::LK::NBLK; ++blk)
                        tma_load_2d(st + blk * kTile * 128 + bx * kBox * 128, &map_k, 64 * blk, y, bar);
                    if (C::LK::TAIL)
                        tma_load_2d(st + C::LK::NBLK * kTile * 128 + bx * kBox * C::LK::TB, &map_kt,
                                    64 * C::LK::NBLK, y, bar);
                    const uint32_t sv0 = st + C::K_BYTES;
#pragma unroll
                    for (int blk = 0; blk < C::LV::NBLK; ++blk)
                        tma_load_2d(sv0 + blk * kTile * 128 + bx * kBox * 128, &map_v, 64 * blk, y, bar);
                    if (C::LV::TAIL)
                        tma_load_2d(sv0 + C::LV::NBLK * kTile * 128 + bx * kBox * C::LV::TB, &map_vt,
                                    64 * C::LV::NBLK, y, bar);
                }
                ++issued;
            }
        }
    } else {
        // ================= consumer warps =================
        const int rt = warp % RT, grp = warp / RT; // row tile, token group
        uint32_t qa[C::KS][2][4];                  // [k16 step][hi/lo][a0..a3]
        float o[C::NTV][4];
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
        bool q_ready = false; // q_tilde comes from the prologue grid
        int i = 0;
        while (walk.next(pref, a.seq_start, B, 1, d)) {
            const int stage = i % kStages;
            if (d.flags & 1) {
                // a new sequence segment: its q_tilde rows straight into A fragments
                if (!q_ready) {
                    grid_dependency_wait();
                    q_ready = true;
                }
#pragma unroll
                for (int kk = 0; kk < C::KS; ++kk) {
                    const int c0 = 16 * kk + 2 * tq;
                    float x[4][2];
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr) { // rows g, g + 8 of the row tile
                        const int r = rt * 16 + g + 8 * rr;
                        float2 lo = make_float2(0.f, 0.f), hi = make_float2(0.f, 0.f);
                        if (r < rows_all) {
                            const int h = r / a.Tq, t = r - h * a.Tq;
                            const float *qr =
                                a.qt + (((int64_t)d.b * a.H + h) * a.Tq_all + a.tq_off + t) * RK + c0;
                            lo = *reinterpret_cast<const float2 *>(qr);
                            hi = *reinterpret_cast<const float2 *>(qr + 8);
                        }
                        x[rr][0] = lo.x;
                        x[rr][1] = lo.y;
                        x[2 + rr][0] = hi.x;
                        x[2 + rr][1] = hi.y;
                    }
#pragma unroll
                    for (int f = 0; f < 4; ++f)
                        split_bf16_rn(x[f][0], x[f][1], qa[kk][0][f], qa[kk][1][f]);
                }
#pragma unroll
                for (int j = 0; j < C::NTV; ++j)
                    o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
                m0 = m1 = -INFINITY;
                l0 = l1 = 0.f;
            }
            bool ok = misc[0] == 0 && mbar_wait_bounded(full0 + 8 * stage, (i / kStages) & 1);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok)
                misc[0] = 1;
            const uint32_t sk = sbase + stage * C::STAGE, sv = sk + C::K_BYTES;
            if (ok) {
#pragma unroll
                for (int bb = 0; bb < C::BPW; ++bb) {
                    const int tbase = 32 * (grp * C::BPW + bb);
                    if (tbase >= d.rows)
                        break;
                    if (tbase + 32 > d.rows) {
                        // value rows past the segment in this block: p = 0 there, but 0 * NaN
                        // would poison the MMA (every warp of the block writes the same zeros)
                        C::LV::zero_rows(smem + stage * C::STAGE + C::K_BYTES, d.rows, tbase + 32, lane);
                        __syncwarp();
                    }
                    // ---- scores of 32 tokens (4 n8 tiles) for this warp's 16 rows
                    float s[4][4];
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
#pragma unroll
                        for (int kk = 0; kk < C::KS; ++kk) {
                            uint32_t kb[4];
                            const int tok = tbase + 16 * half + ((lane >> 4) << 3) + (lane & 7);
                            ldsm_x4(sk + C::LK::off(tok, 2 * kk + ((lane >> 3) & 1)), kb);
#pragma unroll
                            for (int hl = 0; hl < 2; ++hl) {
                                mma16816(s[2 * half], qa[kk][hl][0], qa[kk][hl][1], qa[kk][hl][2], qa[kk][hl][3],
                                         kb[0], kb[1]);
                                mma16816(s[2 * half + 1], qa[kk][hl][0], qa[kk][hl][1], qa[kk][hl][2],
                                         qa[kk][hl][3], kb[2], kb[3]);
                            }
                        }
                    }
                    if (tbase + 32 > d.rows) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int tok = tbase + 8 * j + 2 * tq;
                            if (tok >= d.rows)
                                s[j][0] = s[j][2] = -INFINITY;
                            if (tok + 1 >= d.rows)
                                s[j][1] = s[j][3] = -INFINITY;
                        }
                    }
                    // ---- online softmax (log2 domain), rows g and g + 8
                    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        mx0 = fmaxf(mx0, fmaxf(s[j][0], s[j][1]));
                        mx1 = fmaxf(mx1, fmaxf(s[j][2], s[j][3]));
                    }
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
                    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
                    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
                    if (mx0 > m0 + kRescaleThreshold) {
                        const float al = fast_exp2(m0 - mx0);
                        l0 *= al;
#pragma unroll
                        for (int j = 0; j < C::NTV; ++j)
                            o[j][0] *= al, o[j][1] *= al;
                        m0 = mx0;
                    }
                    if (mx1 > m1 + kRescaleThreshold) {
                        const float al = fast_exp2(m1 - mx1);
                        l1 *= al;
#pragma unroll
                        for (int j = 0; j < C::NTV; ++j)
                            o[j][2] *= al, o[j][3] *= al;
                        m1 = mx1;
                    }
                    uint32_t pa[2][2][4]; // [k16 step][hi/lo][a0..a3]
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float p0 = fast_exp2(s[j][0] - m0), p1 = fast_exp2(s[j][1] - m0);
                        const float p2 = fast_exp2(s[j][2] - m1), p3 = fast_exp2(s[j][3] - m1);
                        l0 += p0 + p1;
                        l1 += p2 + p3;
                        const int ks = j >> 1, f = (j & 1) * 2;
                        split_bf16(p0, p1, pa[ks][0][f], pa[ks][1][f]);
                        split_bf16(p2, p3, pa[ks][0][f + 1], pa[ks][1][f + 1]);
                    }
                    // ---- O += P . C_V for the 32 tokens
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
                        const int t16 = tbase + 16 * ks;
#pragma unroll
                        for (int pr = 0; pr < C::NTV / 2; ++pr) {
                            uint32_t vb[4];
                            const int tok = t16 + (((lane >> 3) & 1) << 3) + (lane & 7);
                            ldsm_x4_t(sv + C::LV::off(tok, 2 * pr + (lane >> 4)), vb);
#pragma unroll
                            for (int hl = 0; hl < 2; ++hl) {
                                mma16816(o[2 * pr], pa[ks][hl][0], pa[ks][hl][1], pa[ks][hl][2], pa[ks][hl][3],
                                         vb[0], vb[1]);
                                mma16816(o[2 * pr + 1], pa[ks][hl][0], pa[ks][hl][1], pa[ks][hl][2],
                                         pa[ks][hl][3], vb[2], vb[3]);
                            }
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(empty0 + 8 * stage);
            if (d.flags & 2) {
                // ---- segment end: one partial record per (head, loop) row
                float lq0 = l0 + __shfl_xor_sync(0xffffffffu, l0, 1);
                lq0 += __shfl_xor_sync(0xffffffffu, lq0, 2);
                float lq1 = l1 + __shfl_xor_sync(0xffffffffu, l1, 1);
                lq1 += __shfl_xor_sync(0xffffffffu, lq1, 2);
                const bool rec_ok = misc[0] == 0 && d.j < a.seg_max;
                if constexpr (C::TG == 1) {
                    if (rec_ok) {
#pragma unroll
                        for (int rr = 0; rr < 2; ++rr) {
                            const int r = rt * 16 + g + 8 * rr;
                            if (r < rows_all) {
                                float *rec = rec_row(a, d.b, r, d.j, RV);
#pragma unroll
                                for (int j = 0; j < C::NTV; ++j)
                                    *reinterpret_cast<float2 *>(rec + 8 * j + 2 * tq) =
                                        make_float2(o[j][2 * rr], o[j][2 * rr + 1]);
                                if (tq == 0)
                                    *reinterpret_cast<float2 *>(rec + RV) =
                                        make_float2(rr ? m1 : m0, rr ? lq1 : lq0);
                            }
                        }
                    }
                } else {
                    // merge the TG token groups of each row tile through shared memory
                    float *mw = mrg + warp * 16 * (RV + 2);
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr) {
                        const int row = g + 8 * rr;
#pragma unroll
                        for (int j = 0; j < C::NTV; ++j) {
                            mw[row * (RV + 2) + 8 * j + 2 * tq] = o[j][2 * rr];
                            mw[row * (RV + 2) + 8 * j + 2 * tq + 1] = o[j][2 * rr + 1];
                        }
                        if (tq == 0) {
                            mw[row * (RV + 2) + RV] = rr ? m1 : m0;
                            mw[row * (RV + 2) + RV + 1] = rr ? lq1 : lq0;
                        }
                    }
                    asm volatile("bar.sync 1, %0;" ::"r"(kConsumers) : "memory");
                    if (rec_ok) {
                        for (int idx = tid; idx < RT * 16 * (RV + 2); idx += kConsumers) {
                            const int rowa = idx / (RV + 2), jj = idx - rowa * (RV + 2);
                            const int rtt = rowa >> 4, row = rowa & 15, r = rtt * 16 + row;
                            if (r >= rows_all)
                                continue;
                            float M = -INFINITY;
#pragma unroll
                            for (int gq = 0; gq < C::TG; ++gq)
                                M = fmaxf(M, mrg[((gq * RT + rtt) * 16 + row) * (RV + 2) + RV]);
                            float val = 0.f;
                            if (jj == RV) {
                                val = M;
                            } else {
#pragma unroll
                                for (int gq = 0; gq < C::TG; ++gq) {
                                    const float mg = mrg[((gq * RT + rtt) * 16 + row) * (RV + 2) + RV];
                                    if (mg != -INFINITY)
                                        val += fast_exp2(mg - M) * mrg[((gq * RT + rtt) * 16 + row) * (RV + 2) + jj];
                                }
                            }
                            rec_row(a, d.b, r, d.j, RV)[jj] = val;
                        }
                    }
                    asm volatile("bar.sync 1, %0;" ::"r"(kConsumers) : "memory");
                }
                if (rec_ok && d.j == 0)
                    for (int h = tid; h < a.H; h += kConsumers)
                        a.counts[(int64_t)d.b * a.H + h] = d.n_u;
                if (tid == 0 && misc[0] == 0 && d.j >= a.seg_max)
                    report_status(a.status, LLA_ERR_INVALID); // a context longer than max_ctx
            }
            ++i;
        }
    }
    __syncwarp();
    __syncthreads();
    if (misc[0] != 0 && warp == kWarps && lane == 0) {
        report_status(a.status, LLA_ERR_DEVICE_TIMEOUT);
        for (int i = issued - kStages < 0 ? 0 : issued - kStages; i < issued; ++i)
            (void)mbar_wait_bounded(full0 + 8 * (i % kStages), (i / kStages) & 1);
    }
}

template <int RK, int RV, int RT>
cudaError_t launch_2d_t(const DecodeArgs &a, cudaStream_t stream)
{
    using C = M2Cfg<RK, RV, RT>;
    CUtensorMap mk, mkt, mv, mvt;
    if (!plane_maps(&mk, &mkt, a.k, RK, a.slots) || !plane_maps(&mv, &mvt, a.v, RV, a.slots))
        return cudaErrorInvalidValue;
    auto kern = decode_absorb_2d_kernel<RK, RV, RT>;
    const int smem = C::smem_bytes(a.B);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
        return e;
    int dev = 0, sms = 148, occ = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, C::THREADS, smem);
    if (e != cudaSuccess)
        return e;
    if (occ < 1)
        return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sms * occ);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization; // overlap the prologue
    attr[0].val.programmaticStreamSerializationAllowed = a.serial ? 0 : 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, mk, mkt, mv, mvt, a);
}

} // namespace

bool decode_mma2d_supported(int dtype, int r_k, int r_v, int fold, int H)
{
    return dtype == LLA_BF16 && fold == LLA_FOLD_2D && H <= 64 && r_k == 64 && r_v == 128 &&
           tensor_map_encoder() != nullptr;
}

int decode_mma2d_loops_per_pass(int H) { return H >= 64 ? 1 : 64 / H; }

cudaError_t launch_decode_absorb_2d(const DecodeArgs &a, cudaStream_t stream)
{
    const int rows = a.H * a.Tq;
    if (a.r_k == 64 && a.r_v == 128) {
        if (rows > 32)
            return launch_2d_t<64, 128, 4>(a, stream);
        if (rows > 16)
            return launch_2d_t<64, 128, 2>(a, stream);
        return launch_2d_t<64, 128, 1>(a, stream);
    }
    return cudaErrorNotSupported;
}

} // namespace lla
