// decode_mma.cu -- LLA decode attention, query-absorbed form, on warp-level tensor cores.
//
// "Looped Latent Attention: Cross-Loop KV Compression for Looped Transformers": Pith
// review page, "What carries the argument" (Eq. 3) and the Pith verdict record's
// desk-editor letter (absorbed-attention variant):
//     l_n = q_tilde . c_K[n] + scale * q . mu_t^K,   out = (sum_n p_n c_V[n]) W_up,t^V + mu_t^V.
// Per (sequence, head) unit the Tq <= 16 loop queries form the 16 rows of an m16n8k16
// tile, so both contractions of one token tile are tensor-core MMAs:
//     S[16 x 16 tok]   = Q_tilde[16 x r_k] . C_K^T          (bf16 hi + lo parts of q_tilde)
//     O[16 x r_v]     += P[16 x 16 tok] . C_V[16 tok x r_v]  (bf16 hi + lo parts of p)
// The hi/lo split keeps about 16 mantissa bits for q_tilde and p, so the result matches
// fp32 accumulation to within the parity tolerance while the latents stay exact bf16.
//
// Scheduling is the persistent, load-balanced split of decode_sched.cuh.  One thread
// streams tiles of 128 tokens with 2-D TMA tensor copies (boxes of 16 rows) into a
// 3-stage mbarrier ring; the swizzled shared layout (32 B rows: 32B swizzle, 64 B rows:
// 64B swizzle) makes every ldmatrix conflict-free.  Each of the 4 warps owns 32 tokens of
// a tile: 8 (r_k = 16) MMAs for the scores, an online softmax on the accumulator
// fragments (row max over a quad of lanes, lazy rescale), then 16 (r_v = 32) MMAs for
// P.C_V with P taken straight from the score fragments.  At a segment end the 4 warp
// states are merged through shared memory into one partial record (acc, m, l).
#include "mma_common.cuh"

namespace lla {
namespace {
using namespace mma;

// NW consumer warps (32 tokens of a tile each) + one producer warp.  DR > 0: every cached
// token also carries a decoupled rotary sub-key of DR values in a plane of its own (the
// Pith verdict record's decoupled RoPE for the absorbed variant); its tile sits beside
// the key tile and adds DR / 16 k16 steps to the score MMA, with the rotated rotary query
// part appended to q_tilde (rows of RK + DR).
// RT row tiles: the loop queries of a pass fill RT m16 tiles (RT = 2: up to 32 queries), each
// taken by its own NW consumer warps over the same staged latent tile, so one read of the
// latents serves them all.
template <int RK, int RV, int NW, int DR = 0, int RT = 1> struct MCfg {
    static constexpr int TILE = 32 * NW;
    static constexpr int CW = NW * RT; // consumer warps
    static constexpr int THREADS = (CW + 1) * 32;
    static constexpr int CONSUMERS = CW * 32;
    static constexpr int STAGES = RT > 1 ? 3 : ((RK + RV + DR) * 2 * TILE > 24 * 1024 ? 2 : 3);
    using LK = TileLayout<RK, TILE>;
    using LV = TileLayout<RV, TILE>;
    using LR = TileLayout<(DR > 0 ? DR : 16), TILE>;
    static constexpr int RKT = RK + DR; // q_tilde row
    static constexpr int KS = RK / 16;  // k16 steps of the score MMA over the latent
    static constexpr int KSR = DR / 16; // k16 steps over the rotary sub-key
    static constexpr int NTV = RV / 8;  // n8 tiles of the output
    static constexpr int K_BYTES = LK::BYTES, V_BYTES = LV::BYTES, R_BYTES = DR > 0 ? LR::BYTES : 0;
    static constexpr int Q_OFF = K_BYTES + V_BYTES + R_BYTES;
    static constexpr int Q_BYTES = 16 * RT * RKT * 4;
    static constexpr int STAGE = align1024(Q_OFF + Q_BYTES);
    static constexpr int RING = STAGES * STAGE;
    static constexpr int MRG_OFF = RING;                              // [NW][16 RT][RV + 2]
    static constexpr int BAR_OFF = (MRG_OFF + NW * 16 * RT * (RV + 2) * 4 + 15) & ~15; // full[S], empty[S]
    static constexpr int MISC_OFF = BAR_OFF + 2 * STAGES * 8;
    static constexpr int SCR_OFF = (MISC_OFF + 16 + 15) & ~15;        // int64 [CW + 2]
    static constexpr int PREF_OFF = SCR_OFF + (CW + 2) * 8;           // int64 [B + 1]
};

// TQ16: the tile carries more than 8 loop queries, so fragment rows g + 8 are real.
template <int RK, int RV, bool TQ16, int NW, int DR, int RT = 1>
__device__ __forceinline__ void decode_mma_body(const CUtensorMap *map_k, const CUtensorMap *map_kt,
                                                const CUtensorMap *map_v, const CUtensorMap *map_vt,
                                                const CUtensorMap *map_r, const CUtensorMap *map_rt,
                                                const DecodeArgs &a)
{
    using C = MCfg<RK, RV, NW, DR, RT>;
    constexpr int kWarps = C::CW, kThreads = C::THREADS, kConsumers = C::CONSUMERS, kTile = C::TILE;
    constexpr int kStages = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float *mrg = reinterpret_cast<float *>(smem + C::MRG_OFF);
    volatile int *misc = reinterpret_cast<volatile int *>(smem + C::MISC_OFF); // [0] error flag
    int64_t *pref = reinterpret_cast<int64_t *>(smem + C::PREF_OFF);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t full0 = sbase + C::BAR_OFF, empty0 = full0 + 8 * kStages;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, tq = lane & 3; // fragment row group / thread-in-group
    const int B = a.B, H = a.H, Tq = a.Tq;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full0 + 8 * s, 1);       // producer's expect_tx + TMA bytes
            mbar_init(empty0 + 8 * s, kWarps); // one arrival per consumer warp
        }
        misc[0] = 0;
        fence_barrier_init();
    }
    block_length_prefix<kThreads>(a.ctx_lens, B, pref, reinterpret_cast<int64_t *>(smem + C::SCR_OFF));
    // The combine grid may take SM slots (and stage its inputs) as this grid's CTAs exit;
    // it reads nothing of ours before its own programmatic-launch wait.
    grid_launch_dependents();
    int64_t s0, s1, chunk;
    cta_share(pref, B, H, a.chunk_min, s0, s1, chunk);
    if (s0 >= s1)
        return; // uniform: nothing for this CTA

    // Every warp walks the same tile sequence of this CTA's share, so segment ends (and the
    // consumer-only barriers at them) happen in the same order in every warp.
    ShareWalk<kTile> walk;
    walk.start(s0, s1, chunk);
    TileDesc d;
    int issued = 0;

    if (warp == kWarps) {
        // ================= producer warp: one lane streams the tiles =================
        if (lane == 0) {
            bool q_ready = false; // q_tilde comes from the preceding (prologue) grid
            while (walk.next(pref, a.seq_start, B, H, d)) {
                const int i = issued, stage = i % kStages;
                if (i >= kStages && !mbar_wait_bounded(empty0 + 8 * stage, ((i / kStages) - 1) & 1)) {
                    misc[0] = 1;
                    break;
                }
                if (misc[0])
                    break;
                const uint32_t st = sbase + stage * C::STAGE;
                const int nbox = (d.rows + kBox - 1) / kBox;
                const uint32_t qb = (d.flags & 1) ? (uint32_t)(Tq * C::RKT * 4) : 0u;
                const uint32_t bar = full0 + 8 * stage;
                fence_proxy_async_smem(); // consumers' generic writes to this stage come first
                mbar_arrive_expect_tx(bar, nbox * kBox * (RK + RV + DR) * 2 + qb);
                const int hs = a.fold ? 0 : d.h; // LLA-2D: every head reads the one folded plane
                const int y0 = (int)((int64_t)hs * a.slots + d.row);
                for (int bx = 0; bx < nbox; ++bx) {
                    const int y = y0 + bx * kBox;
#pragma unroll
                    for (int blk = 0; blk < C::LK::NBLK; ++blk)
                        tma_load_2d(st + blk * kTile * 128 + bx * kBox * 128, map_k, 64 * blk, y, bar);
                    if (C::LK::TAIL)
                        tma_load_2d(st + C::LK::NBLK * kTile * 128 + bx * kBox * C::LK::TB, map_kt,
                                    64 * C::LK::NBLK, y, bar);
                    const uint32_t sv0 = st + C::K_BYTES;
#pragma unroll
                    for (int blk = 0; blk < C::LV::NBLK; ++blk)
                        tma_load_2d(sv0 + blk * kTile * 128 + bx * kBox * 128, map_v, 64 * blk, y, bar);
                    if (C::LV::TAIL)
                        tma_load_2d(sv0 + C::LV::NBLK * kTile * 128 + bx * kBox * C::LV::TB, map_vt,
                                    64 * C::LV::NBLK, y, bar);
                    if constexpr (DR > 0) { // the rotary sub-key plane, same rows
                        const uint32_t sr0 = sv0 + C::V_BYTES;
#pragma unroll
                        for (int blk = 0; blk < C::LR::NBLK; ++blk)
                            tma_load_2d(sr0 + blk * kTile * 128 + bx * kBox * 128, map_r, 64 * blk, y, bar);
                        if (C::LR::TAIL)
                            tma_load_2d(sr0 + C::LR::NBLK * kTile * 128 + bx * kBox * C::LR::TB, map_rt,
                                        64 * C::LR::NBLK, y, bar);
                    }
                }
                if (qb) {
                    if (!q_ready) {
                        grid_dependency_wait();
                        q_ready = true;
                    }
                    bulk_copy_g2s(st + C::Q_OFF, a.qt + ((int64_t)d.u * a.Tq_all + a.tq_off) * C::RKT, qb, bar);
                }
                ++issued;
            }
        }
    } else {
        // ================= consumer warps =================
        // warp = rt * NW + tw: token group tw (32 tokens of the tile), row tile rt (queries
        // 16 rt .. 16 rt + 15)
        const int tw = warp % NW, rt = warp / NW;
        uint32_t qa[C::KS + C::KSR][2][4]; // q_tilde A fragments, [k16 step][hi/lo][a0..a3]
        float o[C::NTV][4];       // output accumulator fragments (rows g, g + 8)
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
        int i = 0;
        while (walk.next(pref, a.seq_start, B, H, d)) {
            const int stage = i % kStages;
            bool ok = misc[0] == 0 && mbar_wait_bounded(full0 + 8 * stage, (i / kStages) & 1);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok)
                misc[0] = 1;
            const uint32_t sk = sbase + stage * C::STAGE, sv = sk + C::K_BYTES;
            if (ok) {
                // Tokens past the segment in the last active warp's 32-token group (loaded
                // from beyond the segment, or never written): their p is 0, but 0 * NaN is NaN
                // in the MMA, so that warp zeroes those value rows.
                const int r0 = d.rows, r1 = (d.rows + 31) & ~31;
                if (r0 < r1 && tw == (r0 >> 5)) { // (each row tile's warp zeroes the same rows)
                    C::LV::zero_rows(smem + stage * C::STAGE + C::K_BYTES, r0, r1, lane);
                    __syncwarp();
                }
                if (d.flags & 1) { // new unit segment: its q_tilde, fresh state
                    const float *qs = reinterpret_cast<const float *>(smem + stage * C::STAGE + C::Q_OFF);
                    constexpr int QL = C::RKT;
#pragma unroll
                    for (int kk = 0; kk < C::KS + C::KSR; ++kk) {
                        const int c0 = 16 * kk + 2 * tq;
                        float x[4][2];
#pragma unroll
                        for (int r = 0; r < 2; ++r) { // rows g, g + 8 of the row tile
                            const int row = 16 * rt + g + 8 * r;
                            const bool in = row < Tq;
                            x[r][0] = in ? qs[row * QL + c0] : 0.f;
                            x[r][1] = in ? qs[row * QL + c0 + 1] : 0.f;
                            x[2 + r][0] = in ? qs[row * QL + c0 + 8] : 0.f;
                            x[2 + r][1] = in ? qs[row * QL + c0 + 9] : 0.f;
                        }
                        // a0: (g, c0..), a1: (g+8, c0..), a2: (g, c0+8..), a3: (g+8, c0+8..)
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
                const int tbase = tw * 32; // this warp's 32 tokens of the tile
                if (tbase < d.rows) {
                    // ---- a2: scores for 32 tokens (4 n8 tiles)
                    float s[4][4];
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const int t16 = tbase + 16 * half;
#pragma unroll
                        for (int kk = 0; kk < C::KS; ++kk) {
                            uint32_t kb[4];
                            const int tok = t16 + ((lane >> 4) << 3) + (lane & 7);
                            const int ch = 2 * kk + ((lane >> 3) & 1);
                            ldsm_x4(sk + C::LK::off(tok, ch), kb);
#pragma unroll
                            for (int hl = 0; hl < 2; ++hl) {
                                mma16816(s[2 * half], qa[kk][hl][0], qa[kk][hl][1], qa[kk][hl][2], qa[kk][hl][3],
                                         kb[0], kb[1]);
                                mma16816(s[2 * half + 1], qa[kk][hl][0], qa[kk][hl][1], qa[kk][hl][2],
                                         qa[kk][hl][3], kb[2], kb[3]);
                            }
                        }
                        if constexpr (DR > 0) { // + rotated q_rope . k_rope
                            const uint32_t sr = sv + C::V_BYTES;
#pragma unroll
                            for (int kr = 0; kr < C::KSR; ++kr) {
                                uint32_t rb[4];
                                const int tok = t16 + ((lane >> 4) << 3) + (lane & 7);
                                const int ch = 2 * kr + ((lane >> 3) & 1);
                                ldsm_x4(sr + C::LR::off(tok, ch), rb);
                                const int kq = C::KS + kr;
#pragma unroll
                                for (int hl = 0; hl < 2; ++hl) {
                                    mma16816(s[2 * half], qa[kq][hl][0], qa[kq][hl][1], qa[kq][hl][2],
                                             qa[kq][hl][3], rb[0], rb[1]);
                                    mma16816(s[2 * half + 1], qa[kq][hl][0], qa[kq][hl][1], qa[kq][hl][2],
                                             qa[kq][hl][3], rb[2], rb[3]);
                                }
                            }
                        }
                    }
                    if (tbase + 32 > d.rows) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) { // mask tokens beyond the tile's rows
                            const int tok = tbase + 8 * j + 2 * tq;
                            if (tok >= d.rows)
                                s[j][0] = s[j][2] = -INFINITY;
                            if (tok + 1 >= d.rows)
                                s[j][1] = s[j][3] = -INFINITY;
                        }
                    }
                    // ---- a3: online softmax (log2 domain) for rows g (and g + 8)
                    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        mx0 = fmaxf(mx0, fmaxf(s[j][0], s[j][1]));
                        if constexpr (TQ16)
                            mx1 = fmaxf(mx1, fmaxf(s[j][2], s[j][3]));
                    }
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
                    if constexpr (TQ16) {
                        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
                        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
                    }
                    if (mx0 > m0 + kRescaleThreshold) {
                        const float al = fast_exp2(m0 - mx0);
                        l0 *= al;
#pragma unroll
                        for (int j = 0; j < C::NTV; ++j)
                            o[j][0] *= al, o[j][1] *= al;
                        m0 = mx0;
                    }
                    if constexpr (TQ16) {
                        if (mx1 > m1 + kRescaleThreshold) {
                            const float al = fast_exp2(m1 - mx1);
                            l1 *= al;
#pragma unroll
                            for (int j = 0; j < C::NTV; ++j)
                                o[j][2] *= al, o[j][3] *= al;
                            m1 = mx1;
                        }
                    }
                    uint32_t pa[2][2][4]; // [k16 step][hi/lo][a0..a3]
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float p0 = fast_exp2(s[j][0] - m0), p1 = fast_exp2(s[j][1] - m0);
                        l0 += p0 + p1;
                        // n8 tile j -> k16 step j/2: a0/a1 for the first tile, a2/a3 for the second
                        const int ks = j >> 1, f = (j & 1) * 2;
                        split_bf16(p0, p1, pa[ks][0][f], pa[ks][1][f]);
                        if constexpr (TQ16) {
                            const float p2 = fast_exp2(s[j][2] - m1), p3 = fast_exp2(s[j][3] - m1);
                            l1 += p2 + p3;
                            split_bf16(p2, p3, pa[ks][0][f + 1], pa[ks][1][f + 1]);
                        } else {
                            pa[ks][0][f + 1] = pa[ks][1][f + 1] = 0u; // rows 8..15 are padding
                        }
                    }
                    // ---- O += P . C_V for the 32 tokens
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
                        const int t16 = tbase + 16 * ks;
#pragma unroll
                        for (int pr = 0; pr < C::NTV / 2; ++pr) {
                            uint32_t vb[4];
                            const int tok = t16 + (((lane >> 3) & 1) << 3) + (lane & 7);
                            const int ch = 2 * pr + (lane >> 4);
                            ldsm_x4_t(sv + C::LV::off(tok, ch), vb);
#pragma unroll
                            for (int hl = 0; hl < 2; ++hl) {
                                mma16816(o[2 * pr], pa[ks][hl][0], pa[ks][hl][1], pa[ks][hl][2], pa[ks][hl][3], vb[0],
                                         vb[1]);
                                mma16816(o[2 * pr + 1], pa[ks][hl][0], pa[ks][hl][1], pa[ks][hl][2], pa[ks][hl][3],
                                         vb[2], vb[3]);
                            }
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(empty0 + 8 * stage); // this warp is done with the stage
            if (d.flags & 2) {
                // ---- segment end: merge the 4 consumer warps' states into one record
                float lq0 = l0 + __shfl_xor_sync(0xffffffffu, l0, 1);
                lq0 += __shfl_xor_sync(0xffffffffu, lq0, 2);
                float lq1 = l1 + __shfl_xor_sync(0xffffffffu, l1, 1);
                lq1 += __shfl_xor_sync(0xffffffffu, lq1, 2);
                float *mw = mrg + tw * 16 * RT * (RV + 2); // [token group][query row][RV + 2]
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int row = 16 * rt + g + 8 * r;
                    if (row < Tq) {
#pragma unroll
                        for (int j = 0; j < C::NTV; ++j) {
                            mw[row * (RV + 2) + 8 * j + 2 * tq] = o[j][2 * r];
                            mw[row * (RV + 2) + 8 * j + 2 * tq + 1] = o[j][2 * r + 1];
                        }
                        if (tq == 0) {
                            mw[row * (RV + 2) + RV] = r ? m1 : m0;
                            mw[row * (RV + 2) + RV + 1] = r ? lq1 : lq0;
                        }
                    }
                }
                asm volatile("bar.sync 1, %0;" ::"r"(kConsumers) : "memory");
                if (misc[0] == 0 && d.j < a.seg_max) {
                    for (int idx = tid; idx < Tq * (RV + 2); idx += kConsumers) {
                        const int row = idx / (RV + 2), jj = idx - row * (RV + 2);
                        float M = -INFINITY;
#pragma unroll
                        for (int w = 0; w < NW; ++w)
                            M = fmaxf(M, mrg[(w * 16 * RT + row) * (RV + 2) + RV]);
                        float val = 0.f;
                        if (jj == RV) {
                            val = M;
                        } else {
#pragma unroll
                            for (int w = 0; w < NW; ++w) {
                                const float mwv = mrg[(w * 16 * RT + row) * (RV + 2) + RV];
                                if (mwv != -INFINITY)
                                    val += fast_exp2(mwv - M) * mrg[(w * 16 * RT + row) * (RV + 2) + jj];
                            }
                        }
                        a.part[(((int64_t)d.u * a.Tq_all + a.tq_off + row) * a.seg_max + d.j) * part_stride(RV) + jj] =
                            val;
                    }
                    if (tid == 0 && d.j == 0)
                        a.counts[d.u] = d.n_u;
                } else if (tid == 0 && d.j >= a.seg_max) {
                    report_status(a.status, LLA_ERR_INVALID); // a context longer than max_ctx
                }
                asm volatile("bar.sync 1, %0;" ::"r"(kConsumers) : "memory"); // mrg free again
            }
            ++i;
        }
    }
    __syncwarp(); // the producer warp's lanes reconverge before the CTA barrier
    __syncthreads();
    if (misc[0] != 0 && warp == kWarps && lane == 0) {
        // wind down: wait (bounded) for this CTA's own copies still in flight
        report_status(a.status, LLA_ERR_DEVICE_TIMEOUT);
        for (int i = issued - kStages < 0 ? 0 : issued - kStages; i < issued; ++i)
            (void)mbar_wait_bounded(full0 + 8 * (i % kStages), (i / kStages) & 1);
    }
}

template <int RK, int RV, bool TQ16, int NW, int MINB, int RT = 1>
__global__ void __launch_bounds__((NW * RT + 1) * 32, MINB)
    decode_absorb_mma_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_kt,
                             const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_vt,
                             const DecodeArgs a)
{
    decode_mma_body<RK, RV, TQ16, NW, 0, RT>(&map_k, &map_kt, &map_v, &map_vt, nullptr, nullptr, a);
}

// With the decoupled rotary sub-key plane (two more tensor maps).
template <int RK, int RV, bool TQ16, int NW, int MINB, int DR>
__global__ void __launch_bounds__((NW + 1) * 32, MINB)
    decode_absorb_mma_rope_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_kt,
                                  const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_vt,
                                  const __grid_constant__ CUtensorMap map_r, const __grid_constant__ CUtensorMap map_rt,
                                  const DecodeArgs a)
{
    decode_mma_body<RK, RV, TQ16, NW, DR>(&map_k, &map_kt, &map_v, &map_vt, &map_r, &map_rt, a);
}

// ---- host ------------------------------------------------------------------------------
template <int RK, int RV, bool TQ16, int NW, int MINB, int DR, int RT = 1>
cudaError_t launch_mma_t(const DecodeArgs &a, int ctas, cudaStream_t stream)
{
    using C = MCfg<RK, RV, NW, DR, RT>;
    const int Hs = a.fold ? 1 : a.H;
    CUtensorMap mk, mkt, mv, mvt, mr, mrt;
    if (!plane_maps(&mk, &mkt, a.k, RK, (int64_t)Hs * a.slots) ||
        !plane_maps(&mv, &mvt, a.v, RV, (int64_t)Hs * a.slots) ||
        (DR > 0 && !plane_maps(&mr, &mrt, a.k_rope, DR, (int64_t)Hs * a.slots)))
        return cudaErrorInvalidValue;
    const void *kern;
    if constexpr (DR > 0)
        kern = (const void *)decode_absorb_mma_rope_kernel<RK, RV, TQ16, NW, MINB, DR>;
    else
        kern = (const void *)decode_absorb_mma_kernel<RK, RV, TQ16, NW, MINB, RT>;
    const int smem = C::PREF_OFF + 8 * (a.B + 1) + 1024;
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
    int grid = sms * occ;
    if (ctas > 0 && ctas < grid)
        grid = ctas;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization; // overlap the prologue's tail
    attr[0].val.programmaticStreamSerializationAllowed = a.serial ? 0 : 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if constexpr (DR > 0)
        return cudaLaunchKernelEx(&cfg, decode_absorb_mma_rope_kernel<RK, RV, TQ16, NW, MINB, DR>, mk, mkt, mv, mvt,
                                  mr, mrt, a);
    else
        return cudaLaunchKernelEx(&cfg, decode_absorb_mma_kernel<RK, RV, TQ16, NW, MINB, RT>, mk, mkt, mv, mvt, a);
}

// Small ranks: 128-token tiles, 4 consumer warps, 4 CTAs per SM.  Ranks >= 64: 64-token
// tiles, 2 consumer warps, 2 CTAs per SM (larger register and shared-memory footprint).
template <int RK, int RV, int DR = 0>
cudaError_t launch_mma(const DecodeArgs &a, int ctas, cudaStream_t stream)
{
    constexpr bool big = RK >= 64 || RV >= 64;
    // a 64-wide rotary sub-key adds 32 registers of q_tilde fragments: 3 CTAs per SM
    constexpr int NW = big ? 2 : 4, MINB = big ? 2 : (DR >= 64 ? 3 : 4);
    if constexpr (DR == 0) {
        // 17 .. 32 loop queries: two row tiles over one staged latent tile (one pass)
        if (a.Tq > 16)
            return launch_mma_t<RK, RV, true, NW, big ? 1 : 2, 0, 2>(a, ctas, stream);
    }
    return a.Tq > 8 ? launch_mma_t<RK, RV, true, NW, MINB, DR>(a, ctas, stream)
                    : launch_mma_t<RK, RV, false, NW, MINB, DR>(a, ctas, stream);
}

} // namespace

int decode_mma_loops_per_pass(int d_rope) { return d_rope > 0 ? 16 : 32; }

bool decode_mma_supported(int dtype, int r_k, int r_v, int fold, int Tq)
{
    (void)Tq; // more than decode_mma_loops_per_pass() loop queries run as several passes
    const bool pair = (r_k == 16 && r_v == 32) || (r_k == 16 && r_v == 16) || (r_k == 32 && r_v == 32) ||
                      (r_k == 64 && r_v == 128) || (r_k == 96 && r_v == 160) || (r_k == 128 && r_v == 128);
    return dtype == LLA_BF16 && pair && tensor_map_encoder() != nullptr;
}

bool decode_mma_rope_supported(int dtype, int r_k, int r_v, int d_rope, int fold)
{
    return dtype == LLA_BF16 && fold == LLA_PER_HEAD && r_k == 16 && r_v == 32 && (d_rope == 32 || d_rope == 64) &&
           tensor_map_encoder() != nullptr;
}

cudaError_t launch_decode_absorb_mma(const DecodeArgs &a, int ctas, cudaStream_t stream)
{
    if (a.d_rope > 0) {
        if (a.r_k == 16 && a.r_v == 32 && a.d_rope == 32)
            return launch_mma<16, 32, 32>(a, ctas, stream);
        if (a.r_k == 16 && a.r_v == 32 && a.d_rope == 64)
            return launch_mma<16, 32, 64>(a, ctas, stream);
        return cudaErrorNotSupported;
    }
#define LLA_MMA_CASE(RK, RV) \
    if (a.r_k == RK && a.r_v == RV) \
        return launch_mma<RK, RV>(a, ctas, stream);
    LLA_MMA_CASE(16, 32)
    LLA_MMA_CASE(16, 16)
    LLA_MMA_CASE(32, 32)
    LLA_MMA_CASE(64, 128)
    LLA_MMA_CASE(96, 160)
    LLA_MMA_CASE(128, 128)
#undef LLA_MMA_CASE
    return cudaErrorNotSupported;
}

} // namespace lla
