// decode_reconstruct.cu -- LLA decode attention, reconstruct-on-read form.
//
// "Looped Latent Attention: Cross-Loop KV Compression for Looped Transformers": Pith
// review page, "What carries the argument" (Eq. 3: loop t reads x_hat_t = c W_up,t + mu_t)
// and arXiv abstract (K/V vectors are reconstructed only when attention reads them).
// For one loop t this kernel rebuilds, per 32-token slice of every latent tile,
//     K_hat^T [d x 32] = W_up,t^K^T [d x r_k] . C_K^T   (+ mu_t^K),
//     V_hat^T [d x 32] = W_up,t^V^T [d x r_v] . C_V^T   (+ mu_t^V)
// on warp-level tensor cores (m16n8k16, d rows as M, bf16 hi/lo parts of W_up,t), and
// runs plain flash decoding on the rebuilt vectors: the scores q . k_hat come from the
// K_hat fragments, and O^T [d x 1] += V_hat^T . p is another MMA (V_hat and p split
// into bf16 hi/lo parts).  It costs about d flop per latent byte per loop against the
// absorbed form's ~1, which is the Pith verdict record's desk-editor point that the
// latent store read this way is compute-bound.  It exists for that comparison.
//
// Faithful read (ROPE): the pages' model applies rotary embedding after reconstruction
// (Pith verdict record: the codec is fitted on pre-RoPE K and a token has one position at
// every loop).  Query and rebuilt key are rotated at their positions, which for the score
// is one rotation of the key by the relative angle (pos_n - pos_q) * omega_i per component
// pair.  Both elements of a pair sit in the same thread: the staged W_up,t^K rows (and q,
// mu_t^K) are ordered so that pair i is (row i, row i + d/2) -- the identity for the
// half-split pairing, an even-first reordering for RoFormer's (2i, 2i+1) -- and row i of
// m16 tile md pairs with the same fragment slot of tile md + d/32.  Angles: the warp's
// first token gets its base angle in double precision (reduced to [-pi, pi]), the 32
// tokens of a block add a per-CTA table of cos/sin(j * omega_i); mu_t^K is rotated with
// the key, so the constant q . mu term is not used.
//
// One launch serves one loop query (Tq = 1); the host launches it per loop.  The
// scheduling (persistent token shares, producer warp, swizzled TMA tiles) is the one
// of the absorbed kernel; each CTA stages W_up,t (transposed, bf16 hi/lo), mu_t and q_t
// of a unit in shared memory when a segment of that unit starts.  Records hold the
// d-wide output, so the combine kernel only merges them.
#include "mma_common.cuh"

namespace lla {
namespace {
using namespace mma;

constexpr int kWarps = 4;
constexpr int kThreads = (kWarps + 1) * 32;
constexpr int kConsumers = kWarps * 32;
constexpr int kTile = 128;
constexpr int kStages = 3;

template <int RK, int RV, int D, bool ROPE> struct RCfg {
    using LK = TileLayout<RK, kTile>;
    using LV = TileLayout<RV, kTile>;
    static constexpr int MD = D / 16;       // m16 tiles over the head dimension
    static constexpr int KSK = RK / 16, KSV = RV / 16;
    static constexpr int WK_LD = RK * 2 + 16; // padded bf16 row bytes of W_up^K^T (conflict-free ldmatrix)
    static constexpr int WV_LD = RV * 2 + 16;
    static constexpr int STAGE = align1024(LK::BYTES + LV::BYTES);
    static constexpr int RING = kStages * STAGE;
    static constexpr int WK_OFF = RING;                      // [2 hi/lo][D][WK_LD bytes]
    static constexpr int WV_OFF = WK_OFF + 2 * D * WK_LD;    // [2 hi/lo][D][WV_LD bytes]
    static constexpr int VEC_OFF = WV_OFF + 2 * D * WV_LD;   // q[D], mu_k[D], mu_v[D] fp32, qmu
    static constexpr int MRG_OFF = VEC_OFF + (3 * D + 4) * 4; // [warps][D + 2]
    static constexpr int BAR_OFF = (MRG_OFF + kWarps * (D + 2) * 4 + 15) & ~15;
    static constexpr int MISC_OFF = BAR_OFF + 2 * kStages * 8;
    static constexpr int SCR_OFF = (MISC_OFF + 16 + 15) & ~15;
    static constexpr int ROT_LD = D / 2 + 4;                  // float2 per table row (bank spread)
    static constexpr int ROT_OFF = (SCR_OFF + (kWarps + 1) * 8 + 15) & ~15; // [32][ROT_LD] cos/sin(j w_i)
    static constexpr int OMG_OFF = ROT_OFF + (ROPE ? 32 * ROT_LD * 8 : 0); // double w_i [D/2]
    static constexpr int PREF_OFF = OMG_OFF + (ROPE ? D / 2 * 8 : 0);
};

// Kernel row of d-index k in the staged K side: pair i is (row i, row i + D/2).
template <int D> __device__ __forceinline__ int rope_row(int k, int style)
{
    return style == LLA_ROPE_INTERLEAVED ? (k & 1) * (D / 2) + (k >> 1) : k;
}

template <int RK, int RV, int D, bool ROPE>
__global__ void __launch_bounds__(kThreads, 2)
    decode_reconstruct_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_kt,
                              const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_vt,
                              const DecodeArgs a)
{
    using C = RCfg<RK, RV, D, ROPE>;
    extern __shared__ uint8_t smem_raw[];
    // aligned by arithmetic on the shared array itself, so accesses stay shared-space loads
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float *vq = reinterpret_cast<float *>(smem + C::VEC_OFF);
    float *vmk = vq + D, *vmv = vq + 2 * D, *vqmu = vq + 3 * D;
    float *mrg = reinterpret_cast<float *>(smem + C::MRG_OFF);
    volatile int *misc = reinterpret_cast<volatile int *>(smem + C::MISC_OFF);
    int64_t *pref = reinterpret_cast<int64_t *>(smem + C::PREF_OFF);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t full0 = sbase + C::BAR_OFF, empty0 = full0 + 8 * kStages;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, tq = lane & 3;
    const int B = a.B, H = a.H;
    const int tl = a.t0 + a.tq_off; // the loop this launch serves

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, kWarps);
        }
        misc[0] = 0;
        fence_barrier_init();
    }
    if (ROPE) { // cos/sin(j w_i) for the 32 token offsets of a block, and w_i in double
        float2 *rot = reinterpret_cast<float2 *>(smem + C::ROT_OFF);
        double *omg = reinterpret_cast<double *>(smem + C::OMG_OFF);
        const float lb = log2f(a.rope_base);
        for (int e = tid; e < 32 * (D / 2); e += kThreads) {
            const int j = e / (D / 2), i = e - j * (D / 2);
            float sn, cs;
            sincosf((float)j * exp2f(-2.0f * (float)i / (float)D * lb), &sn, &cs);
            rot[j * C::ROT_LD + i] = make_float2(cs, sn);
        }
        for (int i = tid; i < D / 2; i += kThreads)
            omg[i] = pow((double)a.rope_base, -2.0 * i / D);
        __syncthreads();
    }
    block_length_prefix<kThreads>(a.ctx_lens, B, pref, reinterpret_cast<int64_t *>(smem + C::SCR_OFF));
    int64_t s0, s1, chunk;
    cta_share(pref, B, H, a.chunk_min, s0, s1, chunk);
    if (s0 >= s1)
        return;

    ShareWalk<kTile> walk;
    walk.start(s0, s1, chunk);
    TileDesc d;
    int issued = 0;

    if (warp == kWarps) {
        if (lane == 0) { // producer: stream the latent tiles
            while (walk.next(pref, a.seq_start, B, H, d)) {
                const int i = issued, stage = i % kStages;
                if (i >= kStages && !mbar_wait_bounded(empty0 + 8 * stage, ((i / kStages) - 1) & 1)) {
                    misc[0] = 1;
                    break;
                }
                if (misc[0])
                    break;
                const uint32_t st = sbase + stage * C::STAGE, sv0 = st + C::LK::BYTES;
                const int nbox = (d.rows + kBox - 1) / kBox;
                const uint32_t bar = full0 + 8 * stage;
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(bar, nbox * kBox * (RK + RV) * 2);
                const int y0 = (int)((int64_t)(a.fold ? 0 : d.h) * a.slots + d.row);
                for (int bx = 0; bx < nbox; ++bx) {
                    const int y = y0 + bx * kBox;
#pragma unroll
                    for (int blk = 0; blk < C::LK::NBLK; ++blk)
                        tma_load_2d(st + blk * kTile * 128 + bx * kBox * 128, &map_k, 64 * blk, y, bar);
                    if (C::LK::TAIL)
                        tma_load_2d(st + C::LK::NBLK * kTile * 128 + bx * kBox * C::LK::TB, &map_kt, 64 * C::LK::NBLK,
                                    y, bar);
#pragma unroll
                    for (int blk = 0; blk < C::LV::NBLK; ++blk)
                        tma_load_2d(sv0 + blk * kTile * 128 + bx * kBox * 128, &map_v, 64 * blk, y, bar);
                    if (C::LV::TAIL)
                        tma_load_2d(sv0 + C::LV::NBLK * kTile * 128 + bx * kBox * C::LV::TB, &map_vt, 64 * C::LV::NBLK,
                                    y, bar);
                }
                ++issued;
            }
        }
    } else {
        float o[C::MD][4]; // O^T fragments: rows d = 16 md + g (+8), column 0 real (tq == 0)
        float m = -INFINITY, l = 0.f;
        int64_t rope_off = 0; // seq_start[b] + q_pos[b]: a tile row's relative position is row - rope_off
        int i = 0;
        while (walk.next(pref, a.seq_start, B, H, d)) {
            const int stage = i % kStages;
            if (d.flags & 1) {
                // ---- new unit segment: stage W_up,t^T (bf16 hi/lo), mu_t, scaled q_t
                const int ld = a.fold ? a.H * D : D;
                const int64_t col0 = a.fold ? (int64_t)d.h * D : 0;
                const float *wk = a.W_up_k + (a.fold ? (int64_t)tl * RK * ld : ((int64_t)d.h * a.T + tl) * RK * ld) + col0;
                const float *wv = a.W_up_v + (a.fold ? (int64_t)tl * RV * ld : ((int64_t)d.h * a.T + tl) * RV * ld) + col0;
                const float *mk = a.mu_k + (a.fold ? (int64_t)tl * ld : ((int64_t)d.h * a.T + tl) * ld) + col0;
                const float *mv = a.mu_v + (a.fold ? (int64_t)tl * ld : ((int64_t)d.h * a.T + tl) * ld) + col0;
                for (int e = tid; e < D * RK; e += kConsumers) { // read [j][k] coalesced, store [k][j]
                    const int j = e / D, k = e - j * D;
                    const int kr = ROPE ? rope_row<D>(k, a.rope_style) : k;
                    const float x = wk[(int64_t)j * ld + k];
                    const __nv_bfloat16 hi = __float2bfloat16_rn(x);
                    const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
                    *reinterpret_cast<__nv_bfloat16 *>(smem + C::WK_OFF + kr * C::WK_LD + 2 * j) = hi;
                    *reinterpret_cast<__nv_bfloat16 *>(smem + C::WK_OFF + D * C::WK_LD + kr * C::WK_LD + 2 * j) = lo;
                }
                for (int e = tid; e < D * RV; e += kConsumers) {
                    const int j = e / D, k = e - j * D;
                    const float x = wv[(int64_t)j * ld + k];
                    const __nv_bfloat16 hi = __float2bfloat16_rn(x);
                    const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
                    *reinterpret_cast<__nv_bfloat16 *>(smem + C::WV_OFF + k * C::WV_LD + 2 * j) = hi;
                    *reinterpret_cast<__nv_bfloat16 *>(smem + C::WV_OFF + D * C::WV_LD + k * C::WV_LD + 2 * j) = lo;
                }
                const __nv_bfloat16 *qrow =
                    static_cast<const __nv_bfloat16 *>(a.q) + (((int64_t)d.b * a.Tq_all + a.tq_off) * a.H + d.h) * D;
                for (int k = tid; k < D; k += kConsumers) {
                    const int kr = ROPE ? rope_row<D>(k, a.rope_style) : k;
                    vq[kr] = __bfloat162float(qrow[k]) * a.scale * kLog2e;
                    vmk[kr] = mk[k];
                    vmv[k] = mv[k];
                }
                if (ROPE)
                    rope_off = a.seq_start[d.b] + (int64_t)a.q_pos[d.b];
                asm volatile("bar.sync 1, %0;" ::"r"(kConsumers) : "memory");
                if (warp == 0) { // constant score term q . mu_t^K (log2 units)
                    float qm = 0.f;
                    for (int k = lane; k < D; k += 32)
                        qm = fmaf(vq[k], vmk[k], qm);
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1)
                        qm += __shfl_xor_sync(0xffffffffu, qm, off);
                    if (lane == 0)
                        vqmu[0] = qm;
                }
                asm volatile("bar.sync 1, %0;" ::"r"(kConsumers) : "memory");
#pragma unroll
                for (int md = 0; md < C::MD; ++md)
                    o[md][0] = o[md][1] = o[md][2] = o[md][3] = 0.f;
                m = -INFINITY;
                l = 0.f;
            }
            bool ok = misc[0] == 0 && mbar_wait_bounded(full0 + 8 * stage, (i / kStages) & 1);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok)
                misc[0] = 1;
            const uint32_t sk = sbase + stage * C::STAGE, sv = sk + C::LK::BYTES;
            const int tbase = warp * 32;
            if (ok && tbase < d.rows) {
                const int r0 = d.rows, r1 = (d.rows + 31) & ~31;
                if (r0 < r1 && warp == (r0 >> 5)) { // 0 * NaN guard for rows past the segment
                    C::LV::zero_rows(smem + stage * C::STAGE + C::LK::BYTES, r0, r1, lane);
                    C::LK::zero_rows(smem + stage * C::STAGE, r0, r1, lane);
                    __syncwarp();
                }
                // B fragments of C_K^T and C_V^T for the warp's 32 tokens
                uint32_t kb[2][C::KSK][4], vb[2][C::KSV][4];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int tok = tbase + 16 * half + ((lane >> 4) << 3) + (lane & 7);
#pragma unroll
                    for (int kk = 0; kk < C::KSK; ++kk)
                        ldsm_x4(sk + C::LK::off(tok, 2 * kk + ((lane >> 3) & 1)), kb[half][kk]);
#pragma unroll
                    for (int kv = 0; kv < C::KSV; ++kv)
                        ldsm_x4(sv + C::LV::off(tok, 2 * kv + ((lane >> 3) & 1)), vb[half][kv]);
                }
                // ---- scores: s[tok] = q . (K_hat[tok]) over d, from K_hat^T fragments
                float sp[4][2];
#pragma unroll
                for (int n = 0; n < 4; ++n)
                    sp[n][0] = sp[n][1] = 0.f;
                // K_hat^T tile md (rows d = 16 md + g (+8), 32 token columns), without mu
                auto k_tile = [&](int md, float (&acc)[4][4]) {
#pragma unroll
                    for (int n = 0; n < 4; ++n)
                        acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
#pragma unroll
                    for (int kk = 0; kk < C::KSK; ++kk) {
#pragma unroll
                        for (int hl = 0; hl < 2; ++hl) {
                            uint32_t wa[4];
                            const int row = 16 * md + (lane & 15);
                            ldsm_x4(sbase + C::WK_OFF + hl * D * C::WK_LD + row * C::WK_LD + 32 * kk + 16 * (lane >> 4), wa);
                            // ldmatrix x4 order: (rows 0-7, k 0-7), (rows 8-15, k 0-7), (rows 0-7, k 8-15), (rows 8-15, k 8-15)
#pragma unroll
                            for (int half = 0; half < 2; ++half) {
                                mma16816(acc[2 * half], wa[0], wa[1], wa[2], wa[3], kb[half][kk][0], kb[half][kk][1]);
                                mma16816(acc[2 * half + 1], wa[0], wa[1], wa[2], wa[3], kb[half][kk][2], kb[half][kk][3]);
                            }
                        }
                    }
                };
                if (!ROPE) {
#pragma unroll
                    for (int md = 0; md < C::MD; ++md) {
                        float acc[4][4];
                        k_tile(md, acc);
                        const float q0 = vq[16 * md + g], q1 = vq[16 * md + g + 8];
#pragma unroll
                        for (int n = 0; n < 4; ++n) {
                            sp[n][0] = fmaf(q0, acc[n][0], fmaf(q1, acc[n][2], sp[n][0]));
                            sp[n][1] = fmaf(q0, acc[n][1], fmaf(q1, acc[n][3], sp[n][1]));
                        }
                    }
                } else {
                    // pair (row i, row i + D/2): tile mp and tile mp + MD/2, same fragment slot
                    const float2 *rot = reinterpret_cast<const float2 *>(smem + C::ROT_OFF);
                    const double *omg = reinterpret_cast<const double *>(smem + C::OMG_OFF);
                    const int64_t rel0 = d.row + tbase - rope_off; // relative position of token 0
#pragma unroll
                    for (int mp = 0; mp < C::MD / 2; ++mp) {
                        float ka[4][4], kc[4][4];
                        k_tile(mp, ka);
                        k_tile(mp + C::MD / 2, kc);
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int i = 16 * mp + g + 8 * e;
                            const double ang = (double)rel0 * omg[i];
                            const float red = (float)(ang - 6.283185307179586 * rint(ang * 0.15915494309189535));
                            float s0, c0;
                            sincosf(red, &s0, &c0);
                            const float qa = vq[i], qb = vq[i + D / 2];
                            const float ma = vmk[i], mb = vmk[i + D / 2];
#pragma unroll
                            for (int n = 0; n < 4; ++n)
#pragma unroll
                                for (int c = 0; c < 2; ++c) {
                                    const float2 cj = rot[(8 * n + 2 * tq + c) * C::ROT_LD + i];
                                    const float cp = c0 * cj.x - s0 * cj.y, sp_ = s0 * cj.x + c0 * cj.y;
                                    const float x = ka[n][c + 2 * e] + ma, y = kc[n][c + 2 * e] + mb;
                                    // q_a (x cos - y sin) + q_b (x sin + y cos)
                                    sp[n][c] = fmaf(x, fmaf(qa, cp, qb * sp_), fmaf(y, fmaf(qb, cp, -qa * sp_), sp[n][c]));
                                }
                        }
                    }
                }
#pragma unroll
                for (int n = 0; n < 4; ++n)
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        float x = sp[n][c];
                        x += __shfl_xor_sync(0xffffffffu, x, 4);
                        x += __shfl_xor_sync(0xffffffffu, x, 8);
                        x += __shfl_xor_sync(0xffffffffu, x, 16);
                        sp[n][c] = ROPE ? x : x + vqmu[0]; // ROPE: mu_t^K was rotated with the key
                        if (tbase + 8 * n + 2 * tq + c >= d.rows)
                            sp[n][c] = -INFINITY;
                    }
                // ---- online softmax over the 32 scores (one query row)
                float mx = -INFINITY;
#pragma unroll
                for (int n = 0; n < 4; ++n)
                    mx = fmaxf(mx, fmaxf(sp[n][0], sp[n][1]));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                if (mx > m + 8.0f) {
                    const float al = fast_exp2(m - mx);
                    l *= al;
#pragma unroll
                    for (int md = 0; md < C::MD; ++md)
                        o[md][0] *= al, o[md][1] *= al, o[md][2] *= al, o[md][3] *= al;
                    m = mx;
                }
                uint32_t pb[2][2][2]; // [k16 step][hi/lo][b0/b1], column 0 only (lanes g == 0)
#pragma unroll
                for (int n = 0; n < 4; ++n) {
                    const float p0 = fast_exp2(sp[n][0] - m), p1 = fast_exp2(sp[n][1] - m);
                    l += p0 + p1;
                    uint32_t h, lo;
                    split_bf16(p0, p1, h, lo);
                    pb[n >> 1][0][n & 1] = g == 0 ? h : 0u;
                    pb[n >> 1][1][n & 1] = g == 0 ? lo : 0u;
                }
                // ---- V_hat^T per d tile, then O^T += V_hat^T . p
#pragma unroll
                for (int md = 0; md < C::MD; ++md) {
                    float acc[4][4];
#pragma unroll
                    for (int n = 0; n < 4; ++n)
                        acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
#pragma unroll
                    for (int kv = 0; kv < C::KSV; ++kv) {
#pragma unroll
                        for (int hl = 0; hl < 2; ++hl) {
                            uint32_t wa[4];
                            const int row = 16 * md + (lane & 15);
                            ldsm_x4(sbase + C::WV_OFF + hl * D * C::WV_LD + row * C::WV_LD + 32 * kv + 16 * (lane >> 4), wa);
#pragma unroll
                            for (int half = 0; half < 2; ++half) {
                                mma16816(acc[2 * half], wa[0], wa[1], wa[2], wa[3], vb[half][kv][0], vb[half][kv][1]);
                                mma16816(acc[2 * half + 1], wa[0], wa[1], wa[2], wa[3], vb[half][kv][2], vb[half][kv][3]);
                            }
                        }
                    }
                    const float mu0 = vmv[16 * md + g], mu1 = vmv[16 * md + g + 8];
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
                        uint32_t ah[4], al[4]; // V_hat^T A fragments (rows d, cols tokens of k16 step ks)
                        split_bf16(acc[2 * ks][0] + mu0, acc[2 * ks][1] + mu0, ah[0], al[0]);
                        split_bf16(acc[2 * ks][2] + mu1, acc[2 * ks][3] + mu1, ah[1], al[1]);
                        split_bf16(acc[2 * ks + 1][0] + mu0, acc[2 * ks + 1][1] + mu0, ah[2], al[2]);
                        split_bf16(acc[2 * ks + 1][2] + mu1, acc[2 * ks + 1][3] + mu1, ah[3], al[3]);
                        mma16816(o[md], ah[0], ah[1], ah[2], ah[3], pb[ks][0][0], pb[ks][0][1]);
                        mma16816(o[md], ah[0], ah[1], ah[2], ah[3], pb[ks][1][0], pb[ks][1][1]);
                        mma16816(o[md], al[0], al[1], al[2], al[3], pb[ks][0][0], pb[ks][0][1]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(empty0 + 8 * stage);
            if (d.flags & 2) {
                // ---- segment end: merge the warps into one d-wide record
                float lq = l + __shfl_xor_sync(0xffffffffu, l, 1);
                lq += __shfl_xor_sync(0xffffffffu, lq, 2);
                float *mw = mrg + warp * (D + 2);
                if (tq == 0) {
#pragma unroll
                    for (int md = 0; md < C::MD; ++md) {
                        mw[16 * md + g] = o[md][0];
                        mw[16 * md + g + 8] = o[md][2];
                    }
                }
                if (lane == 0) {
                    mw[D] = m;
                    mw[D + 1] = lq;
                }
                asm volatile("bar.sync 1, %0;" ::"r"(kConsumers) : "memory");
                if (misc[0] == 0 && d.j < a.seg_max) {
                    float M = -INFINITY;
#pragma unroll
                    for (int w = 0; w < kWarps; ++w)
                        M = fmaxf(M, mrg[w * (D + 2) + D]);
                    for (int jj = tid; jj < D + 2; jj += kConsumers) {
                        float val = 0.f;
                        if (jj == D) {
                            val = M;
                        } else {
#pragma unroll
                            for (int w = 0; w < kWarps; ++w) {
                                const float mwv = mrg[w * (D + 2) + D];
                                if (mwv != -INFINITY)
                                    val += fast_exp2(mwv - M) * mrg[w * (D + 2) + jj];
                            }
                        }
                        a.part[(((int64_t)d.u * a.Tq_all + a.tq_off) * a.seg_max + d.j) * part_stride(D) + jj] = val;
                    }
                    if (tid == 0 && d.j == 0)
                        a.counts[d.u] = d.n_u;
                } else if (tid == 0 && d.j >= a.seg_max) {
                    report_status(a.status, LLA_ERR_INVALID);
                }
                asm volatile("bar.sync 1, %0;" ::"r"(kConsumers) : "memory");
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

template <int RK, int RV, int D, bool ROPE>
cudaError_t launch_rec(const DecodeArgs &a, cudaStream_t stream)
{
    using C = RCfg<RK, RV, D, ROPE>;
    const int Hs = a.fold ? 1 : a.H;
    CUtensorMap mk, mkt, mv, mvt;
    if (!plane_maps(&mk, &mkt, a.k, RK, (int64_t)Hs * a.slots) ||
        !plane_maps(&mv, &mvt, a.v, RV, (int64_t)Hs * a.slots))
        return cudaErrorInvalidValue;
    auto kern = decode_reconstruct_kernel<RK, RV, D, ROPE>;
    const int smem = C::PREF_OFF + 8 * (a.B + 1) + 1024;
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
    kern<<<sms * occ, kThreads, smem, stream>>>(mk, mkt, mv, mvt, a);
    return cudaGetLastError();
}

} // namespace

bool decode_reconstruct_supported(int dtype, int r_k, int r_v, int d)
{
    return dtype == LLA_BF16 && (r_k == 16 || r_k == 32) && (r_v == 16 || r_v == 32) && (d == 64 || d == 128) &&
           tensor_map_encoder() != nullptr;
}

cudaError_t launch_decode_reconstruct(const DecodeArgs &a, cudaStream_t stream)
{
#define LLA_REC_CASE(RK, RV, D) \
    if (a.r_k == RK && a.r_v == RV && a.d == D) \
        return a.q_pos != nullptr ? launch_rec<RK, RV, D, true>(a, stream) : launch_rec<RK, RV, D, false>(a, stream);
    LLA_REC_CASE(16, 32, 128)
    LLA_REC_CASE(16, 16, 128)
    LLA_REC_CASE(32, 32, 128)
    LLA_REC_CASE(16, 32, 64)
    LLA_REC_CASE(32, 32, 64)
    LLA_REC_CASE(16, 16, 64)
#undef LLA_REC_CASE
    return cudaErrorNotSupported;
}

} // namespace lla
