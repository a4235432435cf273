// decode_absorb_tc.cu -- LLA decode attention, query-absorbed form, on tcgen05 tensor
// cores, for passes in which many query rows share every latent tile: LLA-2D (the H
// heads x the pass's loops of a sequence all read the one folded latent) and deep loop
// stacks (up to 32 loop queries of one (sequence, head) per pass).
//
// "Looped Latent Attention: Cross-Loop KV Compression for Looped Transformers": review
// page abstract (LLA-2D folds the head axis into the cross-loop latent), "What carries
// the argument" (Eq. 3, x_hat_t = c W_up,t + mu_t) and the Pith verdict record's
// desk-editor letter (absorbed attention): with q_tilde = scale * q W_up,t^K^T (pre-scaled
// by log2 e, from the prologue grid) a loop query's logits over the cached latents are
// q_tilde . c_K[n] (+ a per-query constant added by the combine) and its output is
// (sum_n p_n c_V[n]) W_up,t^V + mu_t^V, projected by the combine.
//
// Orientation: tokens on the tensor-memory lanes.  Per tile of 128 tokens, with the NQ
// query rows of the unit's pass split into bf16 hi + lo parts (stacked along N, so both
// parts of a query land in the same lane and one thread adds them):
//     S^T [128 tok x 2NQ] = C_K . [q_hi ; q_lo]^T          M = tokens, N = 2 NQ, K = r_k
//     O^T [r_v x 2NQ]    += C_V^T . [p_hi | p_lo]^T        M = r_v,    N = 2 NQ, K = tokens
// C_V^T and the weights are read MN-major straight from the tiles the TMA and the softmax
// threads wrote; O^T stays in tensor memory for a whole unit segment and its hi and lo
// halves are added at the segment end.  Thread k of a softmax group owns token k of the
// tile, so every score a thread needs sits in its own lane: no cross-thread work per
// tile.  The running max per query is a reference m kept in registers (identical in the
// group's 128 threads): p = 2^(s - m) as long as no score passes m + 8; otherwise the
// group votes (barrier reduction), takes the tile's column maxima, rescales its partial
// sums and its columns of O^T (tensor-memory load, scale, store) and moves m.  The first
// tile of every segment takes this path; later ones rarely do.
//
// Warps: 4 NQ / 16 softmax warps (group g = warps 4g .. 4g + 3 serves queries 16 g ..
// 16 g + 15 over all 128 lanes), then a producer (TMA 2-D boxes of the folded or per-head
// plane into a ring of stages), an MMA issuer (one elected lane; S of tile i is issued
// before the output MMAs of tile i - 1, so the softmax of a tile overlaps the previous
// output MMAs and the next scores) and two warps that build each unit's [q_hi ; q_lo]
// tile from the prologue's fp32 q_tilde.  Work split: the persistent equal-share walk of the other decode kernels
// (units are sequences for LLA-2D, (sequence, head) pairs otherwise); records have the
// shared (acc, m, l) layout, so the combine projects them.  Every wait is bounded.
#include "mma_common.cuh"
#include "tc_mn.cuh"

namespace lla {
namespace {
using namespace mma;

constexpr int kTile = 128;
constexpr int kGroupThreads = 128; // a softmax group: 4 warps, one per tensor-memory lane quarter
constexpr int kBuildThreads = 64;
constexpr float kMargin = 8.0f; // log2 units: scores up to 2^8 above the reference are taken as they are

// barriers after the rings' kfull[NK], kempty[NK], vfull[NV], vempty[NV]
enum { SFULL0 = 0, SFULL1, SEMPTY0, SEMPTY1, PFULL0, PFULL1, PVDONE0, PVDONE1, QFULL, QEMPTY, DRAIN, NBAR };
// Latent rings: a K tile is free as soon as its scores are computed, a V tile only after the
// output MMAs, so V needs the depth: with three V stages two V tiles (80 KB at r_v = 160)
// stay in flight while one is consumed, enough to cover the HBM latency under full load.
constexpr int kKStages = 2, kVStages = 3;

template <int RK, int RV, int NQ> struct ACfg {
    using LK = TileLayout<RK, kTile>;
    using LV = TileLayout<RV, kTile>;
    using LQ = TileLayout<RK, 2 * NQ>;          // rows: q_hi of the NQ queries, then q_lo
    static constexpr int NS = 2 * NQ;            // columns of S^T and of each O^T block
    static constexpr int QG = 16;                // queries per softmax group
    static constexpr int GROUPS = NQ / QG;       // softmax groups
    static constexpr int SOFT_WARPS = 4 * GROUPS;
    static constexpr int PRODUCER = SOFT_WARPS, MMA = SOFT_WARPS + 1, BUILD = SOFT_WARPS + 2; // + 1 more builder
    static constexpr int THREADS = (SOFT_WARPS + 4) * 32;
    // With 640 threads (96 registers each at launch) the issue warpgroup gives registers to
    // the softmax warps: 512 x 104 + 128 x 64 = 61,440, all of the registers launched.  The host
    // checks the launch's register count before enabling the kernel.
    static constexpr bool SPLIT = THREADS > 384;
    static constexpr int SOFT_REGS = 104, ISSUE_REGS = 64;
    static constexpr int SPLIT_REGS = SOFT_WARPS * 32 * SOFT_REGS + 128 * ISSUE_REGS;
    static constexpr int VB = (RV + 127) / 128;  // O^T blocks of 128 r_v rows
    static constexpr int KSTAGE = (LK::BYTES + 1023) / 1024 * 1024;
    static constexpr int VSTAGE = (LV::BYTES + 1023) / 1024 * 1024;
    static constexpr int P_BYTES = kTile * NS * 2; // MN-major [NS / 64 atoms][128 tokens][128 B]
    static constexpr int Q_BYTES = (LQ::BYTES + 1023) / 1024 * 1024;
    static constexpr uint32_t COL_S = 0;          // S^T buffer b at COL_S + b NS
    static constexpr uint32_t COL_O = 2 * NS;     // O^T block vb at COL_O + vb NS
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(NQ == 32 || NQ == 64, "query rows per pass: 32 or 64");
    static_assert(COL_O + VB * NS <= TMEM_COLS, "tensor memory");
    static_assert(RK % 16 == 0, "r_k in whole K steps");
    // r_v: whole 128-row blocks of 64-wide SW128 atoms, or a last block that is one 32-wide
    // SW64 tail (read with a zero atom stride: its lanes past 32 repeat it and are ignored)
    static_assert(RV % 128 == 0 || (RV % 128 == 32 && LV::TAIL == 32), "r_v layout");
};

struct ALayout {
    uint32_t kring, vring, p, q, cm, bar, misc, scr, ring, pref, total;
};

__host__ __device__ inline uint32_t up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

// Shared-memory layout (byte offsets from a 1024-aligned base): the K ring, the V ring, two
// weights tiles (tile i writes buffer i & 1), the query tile, then the small arrays.
template <int RK, int RV, int NQ> __host__ __device__ inline ALayout alayout(int B)
{
    using C = ACfg<RK, RV, NQ>;
    ALayout L;
    uint32_t o = 0;
    L.kring = o;
    o += kKStages * C::KSTAGE;
    L.vring = o;
    o += kVStages * C::VSTAGE;
    L.p = o;
    o += 2 * C::P_BYTES;
    L.q = o;
    o += C::Q_BYTES;
    // [groups][4 warps][QG] column maxima / sums, [groups][QG] record references,
    // [groups][QG] rescale factors, [groups][2][QG] running references (double buffer)
    L.cm = o;
    o += C::GROUPS * 8 * C::QG * 4;
    L.bar = up(o, 8);
    o = L.bar + (2 * kKStages + 2 * kVStages + NBAR) * 8;
    L.misc = o;
    o += 16;
    L.scr = up(o, 8);
    o = L.scr + (C::THREADS / 32 + 1) * 8;
    L.ring = o; // producer's tiles between the K and V cursors: {plane row, rows}
    o += kKStages * 8;
    L.pref = up(o, 8);
    o = L.pref + 8 * (B + 1);
    L.total = o;
    return L;
}

// Non-blocking test: has the phase of `bar` with parity `parity` completed?
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok)
                 : "r"(bar), "r"(parity)
                 : "memory");
    return ok != 0;
}

__device__ __forceinline__ void group_sync(int g)
{
    asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "r"(kGroupThreads) : "memory");
}
template <int NT> __device__ __forceinline__ void all_sync() { asm volatile("bar.sync 15, %0;" ::"r"(NT) : "memory"); }

// Named barriers: 1 + g group g's sync, 8 + g its vote, 15 the whole CTA (g < 4).
// OR of `pred` over the 128 threads of softmax group g (a barrier with a reduction).
__device__ __forceinline__ bool group_any(int g, bool pred)
{
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
                 "barrier.cta.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r)
                 : "r"((uint32_t)pred), "r"(8 + g), "r"(kGroupThreads)
                 : "memory");
    return r != 0;
}

// Column reduction across the warp by recursive halving: v[0..N) per lane (N = 16 or 32)
// becomes, in lane l, the reduction over the 32 lanes of column l * N / 32.
template <int N, bool MAX> __device__ __forceinline__ float warp_columns(float (&v)[N], int lane)
{
    static_assert(N == 16 || N == 32, "16 or 32 columns");
    auto op = [](float x, float y) { return MAX ? fmaxf(x, y) : x + y; };
#pragma unroll
    for (int w = N / 2, bit = 16; w >= 1; w >>= 1, bit >>= 1) {
        const bool up = lane & bit; // keep the upper half of the live columns
#pragma unroll
        for (int i = 0; i < w; ++i) {
            const float keep = up ? v[i + w] : v[i], give = up ? v[i] : v[i + w];
            v[i] = op(keep, __shfl_xor_sync(0xffffffffu, give, bit));
        }
    }
    float x = v[0];
    if (N == 16) // one column per lane pair: close over the last lane bit
        x = op(x, __shfl_xor_sync(0xffffffffu, x, 1));
    return x;
}

// Byte offset of (token k, column n) in the MN-major weights tile: 64-column atoms of
// [128 tokens][128 B], 16-byte chunks swizzled by token mod 8.
__device__ __forceinline__ uint32_t p_off(int k, int n)
{
    return (uint32_t)((n >> 6) * (kTile * 128) + k * 128 + 16 * (((n & 63) >> 3) ^ (k & 7)) + 2 * (n & 7));
}

// bf16 hi and lo parts of 8 consecutive values, packed for one 16-byte store each
__device__ __forceinline__ void split8(const float (&x)[8], uint4 &hi, uint4 &lo)
{
    uint32_t h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        split_bf16(x[2 * i], x[2 * i + 1], h[i], l[i]);
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

template <int RK, int RV, int NQ>
__global__ void __launch_bounds__(ACfg<RK, RV, NQ>::THREADS, 1)
    decode_absorb_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_kt,
                            const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_vt,
                            const DecodeArgs a)
{
    using C = ACfg<RK, RV, NQ>;
    using LK = typename C::LK;
    using LV = typename C::LV;
    using LQ = typename C::LQ;
    constexpr int NS = C::NS, QG = C::QG, kSoftWarps = C::SOFT_WARPS, kThreads = C::THREADS;
    constexpr int kProducerWarp = C::PRODUCER, kMmaWarp = C::MMA, kBuildWarp = C::BUILD;
    extern __shared__ uint8_t smem_raw[];
    // aligned by arithmetic on the shared array itself, so accesses stay shared-space loads
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const ALayout Ly = alayout<RK, RV, NQ>(a.B);
    const uint32_t sbase = smem_u32(smem);
    volatile int *misc = reinterpret_cast<volatile int *>(smem + Ly.misc); // [0] error, [1] tmem, [2] [3] K/V issued
    int64_t *pref = reinterpret_cast<int64_t *>(smem + Ly.pref);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int B = a.B;
    const int HU = a.fold ? 1 : a.H;              // latent planes: units are (sequence, plane)
    const int lp = a.Tq;                          // loop queries of this pass
    const int nq = a.fold ? a.H * lp : lp;        // query rows of a unit (<= NQ)
    const uint32_t bar0 = sbase + Ly.bar;
    auto kfull = [&](int st) { return bar0 + 8u * st; };
    auto kempty = [&](int st) { return bar0 + 8u * (kKStages + st); };
    auto vfull = [&](int st) { return bar0 + 8u * (2 * kKStages + st); };
    auto vempty = [&](int st) { return bar0 + 8u * (2 * kKStages + kVStages + st); };
    auto bar = [&](int k) { return bar0 + 8u * (2 * kKStages + 2 * kVStages + k); };

    if (tid == 0) {
        for (int st = 0; st < kKStages; ++st) {
            mbar_init(kfull(st), 1);  // producer's expect_tx + TMA bytes
            mbar_init(kempty(st), 1); // the tile's score MMAs completed (commit)
        }
        for (int st = 0; st < kVStages; ++st) {
            mbar_init(vfull(st), 1);
            mbar_init(vempty(st), 1); // the tile's output MMAs completed (commit)
        }
        mbar_init(bar(SFULL0), 1);
        mbar_init(bar(SFULL1), 1);
        mbar_init(bar(SEMPTY0), kSoftWarps); // one arrival per softmax warp
        mbar_init(bar(SEMPTY1), kSoftWarps);
        mbar_init(bar(PFULL0), kSoftWarps);
        mbar_init(bar(PFULL1), kSoftWarps);
        mbar_init(bar(PVDONE0), 1);
        mbar_init(bar(PVDONE1), 1);
        mbar_init(bar(QFULL), kBuildThreads / 32);
        mbar_init(bar(QEMPTY), 1);
        mbar_init(bar(DRAIN), 1);
        misc[0] = 0;
        misc[2] = 0;
        misc[3] = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp)
        tc::alloc(reinterpret_cast<uint32_t *>(smem + Ly.misc + 4), C::TMEM_COLS);
    for (int e = tid; e < C::GROUPS * 2 * C::QG; e += kThreads) // running references: none yet
        reinterpret_cast<float *>(smem + Ly.cm)[C::GROUPS * 6 * C::QG + e] = -INFINITY;
    tc::fence_before();
    block_length_prefix<kThreads>(a.ctx_lens, B, pref, reinterpret_cast<int64_t *>(smem + Ly.scr));
    tc::fence_after();
    const uint32_t tmem = (uint32_t)misc[1];
    // The combine grid may take SM slots as this grid's CTAs exit; it reads nothing of
    // ours before its own programmatic-launch wait.
    grid_launch_dependents();
    int64_t s0, s1, chunk;
    cta_share(pref, B, HU, a.chunk_min, s0, s1, chunk);
    bool err = false;
    // bounded wait of the whole warp; a failure anywhere winds every role down
    auto wait_all = [&](uint32_t b, uint32_t parity) -> bool {
        bool ok = !err && misc[0] == 0 && mbar_wait_bounded(b, parity);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) {
            err = true;
            misc[0] = 1;
        }
        return ok;
    };

    if (warp >= kProducerWarp) {
      // ======== the issue warpgroup: producer, MMA issuer, two query builders ========
      if constexpr (C::SPLIT)
          asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::ISSUE_REGS));
      if (warp == kProducerWarp) {
        // ================= producer: one lane streams the latent tiles =================
        // Two cursors over the same tile sequence: K tiles go into their ring as soon as a
        // K stage frees (its scores computed), V tiles as a V stage frees (its outputs
        // computed); K may run up to the whole K ring ahead of V.  The tiles between the
        // cursors are remembered in a small ring (plane row, rows).
        if (lane == 0 && s0 < s1) {
            ShareWalk<kTile> walk;
            walk.start(s0, s1, chunk);
            TileDesc d;
            int2 *tring = reinterpret_cast<int2 *>(smem + Ly.ring);
            bool more = walk.next(pref, a.seq_start, B, HU, d);
            int kt = 0, vt = 0;
            uint64_t t_idle = 0;
            uint32_t spins = 0;
            while (misc[0] == 0 && (more || vt < kt)) {
                bool progress = false;
                if (more && kt - vt < kKStages) {
                    const int st = kt % kKStages;
                    if (kt < kKStages || mbar_test(kempty(st), ((kt / kKStages) - 1) & 1)) {
                        const int y0 = (int)((int64_t)d.h * a.slots + d.row), nbox = (d.rows + kBox - 1) / kBox;
                        const uint32_t sk = sbase + Ly.kring + st * C::KSTAGE;
                        fence_proxy_async_smem();
                        mbar_arrive_expect_tx(kfull(st), nbox * kBox * RK * 2);
                        for (int bx = 0; bx < nbox; ++bx) {
                            const int y = y0 + bx * kBox;
#pragma unroll
                            for (int blk = 0; blk < LK::NBLK; ++blk)
                                tma_load_2d(sk + blk * kTile * 128 + bx * kBox * 128, &map_k, 64 * blk, y, kfull(st));
                            if (LK::TAIL)
                                tma_load_2d(sk + LK::NBLK * kTile * 128 + bx * kBox * LK::TB, &map_kt, 64 * LK::NBLK,
                                            y, kfull(st));
                        }
                        tring[st] = make_int2(y0, d.rows);
                        ++kt;
                        more = walk.next(pref, a.seq_start, B, HU, d);
                        progress = true;
                    }
                }
                if (vt < kt) {
                    const int st = vt % kVStages;
                    if (vt < kVStages || mbar_test(vempty(st), ((vt / kVStages) - 1) & 1)) {
                        const int2 t = tring[vt % kKStages];
                        const int nbox = (t.y + kBox - 1) / kBox;
                        const uint32_t sv = sbase + Ly.vring + st * C::VSTAGE;
                        fence_proxy_async_smem();
                        mbar_arrive_expect_tx(vfull(st), nbox * kBox * RV * 2);
                        for (int bx = 0; bx < nbox; ++bx) {
                            const int y = t.x + bx * kBox;
#pragma unroll
                            for (int blk = 0; blk < LV::NBLK; ++blk)
                                tma_load_2d(sv + blk * kTile * 128 + bx * kBox * 128, &map_v, 64 * blk, y, vfull(st));
                            if (LV::TAIL)
                                tma_load_2d(sv + LV::NBLK * kTile * 128 + bx * kBox * LV::TB, &map_vt, 64 * LV::NBLK,
                                            y, vfull(st));
                        }
                        ++vt;
                        progress = true;
                    }
                }
                if (progress) {
                    spins = 0;
                    t_idle = 0;
                } else if ((++spins & 63u) == 0u) {
                    const uint64_t now = global_timer_ns();
                    if (t_idle == 0)
                        t_idle = now;
                    else if (now - t_idle > kWaitLimitNs)
                        misc[0] = 1;
                }
            }
            misc[2] = kt;
            misc[3] = vt;
        }
    } else if (warp >= kBuildWarp) {
        // ================= query tile of each unit: [q_hi ; q_lo] rows, bf16, K-major ====
        // Each thread fetches its share of the unit's fp32 q_tilde rows before waiting for
        // the tile to be free, so the loads overlap the previous unit's last scores.
        const int bt = tid - kBuildWarp * 32;
        constexpr int C8 = RK / 8;                                  // 8-value chunks of a row
        constexpr int PER = (NQ * C8 + kBuildThreads - 1) / kBuildThreads; // chunks per thread
        constexpr int PRE = C::SPLIT ? (PER + 1) / 2 : PER; // fetched before the wait (register budget)
        if (s0 < s1) {
            ShareWalk<kTile> walk;
            walk.start(s0, s1, chunk);
            TileDesc d;
            int k = 0;
            while (walk.next(pref, a.seq_start, B, HU, d)) {
                if (!(d.flags & 1))
                    continue;
                if (k == 0)
                    grid_dependency_wait(); // q_tilde comes from the prologue grid
                auto fetch = [&](int r, float4 (&w)[2]) {
                    const int e = bt + r * kBuildThreads, n = e / C8, c = e - n * C8;
                    w[0] = w[1] = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (e < NQ * C8 && n < nq) {
                        const int hq = a.fold ? n / lp : d.h, t = a.fold ? n - (n / lp) * lp : n;
                        const int64_t u = (int64_t)d.b * a.H + hq;
                        const float *src = a.qt + (u * a.Tq_all + a.tq_off + t) * RK + 8 * c;
                        w[0] = *reinterpret_cast<const float4 *>(src);
                        w[1] = *reinterpret_cast<const float4 *>(src + 4);
                    }
                };
                uint8_t *qt_s = smem + Ly.q;
                // chunk r of this thread: round-to-nearest bf16 hi, then the remainder, into
                // row n (hi) and row NQ + n (lo) of the tile
                auto store = [&](int r, const float4 (&w)[2]) {
                    const int e = bt + r * kBuildThreads, n = e / C8, c = e - n * C8;
                    if (e >= NQ * C8)
                        return;
                    const float x[8] = {w[0].x, w[0].y, w[0].z, w[0].w, w[1].x, w[1].y, w[1].z, w[1].w};
                    uint32_t h4[4], l4[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const __nv_bfloat162 hh = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
                        const float2 hf = __bfloat1622float2(hh);
                        const __nv_bfloat162 ll = __floats2bfloat162_rn(x[2 * i] - hf.x, x[2 * i + 1] - hf.y);
                        h4[i] = *reinterpret_cast<const uint32_t *>(&hh);
                        l4[i] = *reinterpret_cast<const uint32_t *>(&ll);
                    }
                    *reinterpret_cast<uint4 *>(qt_s + LQ::off(n, c)) = make_uint4(h4[0], h4[1], h4[2], h4[3]);
                    *reinterpret_cast<uint4 *>(qt_s + LQ::off(NQ + n, c)) = make_uint4(l4[0], l4[1], l4[2], l4[3]);
                };
                float4 v[PRE][2];
#pragma unroll
                for (int r = 0; r < PRE; ++r)
                    fetch(r, v[r]);
                // the previous unit's last score MMAs have read the tile
                if (k >= 1 && !wait_all(bar(QEMPTY), (k - 1) & 1))
                    break;
#pragma unroll
                for (int r = 0; r < PRE; ++r)
                    store(r, v[r]);
#pragma unroll
                for (int r = PRE; r < PER; ++r) {
                    float4 w[2];
                    fetch(r, w);
                    store(r, w);
                }
                fence_proxy_async_smem(); // generic writes -> tensor-core reads
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(bar(QFULL));
                ++k;
            }
        }
    } else if (warp == kMmaWarp) {
        // ================= MMA issuer: the whole warp runs the loop, one elected lane issues =========
        if (s0 < s1) {
            constexpr uint32_t idS = tc::idesc_major(tc::kFmtBf16, 128, NS, false, false);
            constexpr uint32_t idPV = tc::idesc_major(tc::kFmtBf16, 128, NS, true, true);
            const uint32_t qbase = sbase + Ly.q, pbase = sbase + Ly.p;
            // K step kk (16 values of r_k) of a K-major [rows][RK] tile laid out by TileLayout
            auto kdesc = [&](uint32_t base, int rows, int kk) -> uint64_t {
                if ((kk >> 2) < LK::NBLK)
                    return tc::smem_desc(base + (kk >> 2) * rows * 128 + 32 * (kk & 3), 128);
                return tc::smem_desc(base + LK::NBLK * rows * 128 + 32 * (kk - 4 * LK::NBLK), LK::TB);
            };
            // C_V^T block vb (r_v rows 128 vb ..), token step kk, read MN-major from the V tile:
            // 64-wide SW128 atoms a whole tile (128 rows x 128 B) apart, 8-token groups 1 KB
            // apart; the SW64 tail of 32 values repeats across the block (atom stride 0)
            auto vdesc = [&](uint32_t vbase, int vb, int kk) -> uint64_t {
                if (2 * vb < LV::NBLK)
                    return tc::smem_desc_explicit(vbase + 2 * vb * kTile * 128 + kk * 2048, kTile * 128, 1024,
                                                  tc::kSw128);
                return tc::smem_desc_explicit(vbase + LV::NBLK * kTile * 128 + kk * 1024, 0, 512, tc::kSw64);
            };
            // weights [p_hi | p_lo]^T of buffer pb, token step kk, MN-major
            auto pdesc = [&](int pb, int kk) -> uint64_t {
                return tc::smem_desc_explicit(pbase + pb * C::P_BYTES + kk * 2048, kTile * 128, 1024, tc::kSw128);
            };
            // Event loop: the scores of the next tile go out as soon as its K tile, its score
            // buffer and its unit's query tile are ready; the output MMAs of a tile as soon as
            // its weights and its V tile are -- neither waits for the other.  Readiness comes
            // from non-blocking tests (made warp-uniform by lane 0); a stretch with no
            // progress at all is bounded.
            ShareWalk<kTile> walk;
            walk.start(s0, s1, chunk);
            TileDesc nxt, hist[2]; // the next tile for scores; tiles with scores out, no output yet
            bool more = walk.next(pref, a.seq_start, B, HU, nxt);
            int ns = 0, npv = 0, k = 0; // tiles with scores issued, with outputs issued; units begun
            uint64_t t_idle = 0;
            uint32_t spins = 0;
            auto ready = [&](uint32_t b, uint32_t parity) -> bool {
                return __shfl_sync(0xffffffffu, mbar_test(b, parity) ? 1 : 0, 0) != 0;
            };
            while (!err && (more || npv < ns)) {
                bool progress = false;
                if (more && ns - npv < 2) {
                    const int st = ns % kKStages, sb = ns & 1;
                    if ((!(nxt.flags & 1) || ready(bar(QFULL), k & 1)) && ready(kfull(st), (ns / kKStages) & 1) &&
                        (ns < 2 || ready(bar(SEMPTY0 + sb), ((ns >> 1) - 1) & 1))) {
                        uint8_t *kt_s = smem + Ly.kring + st * C::KSTAGE;
                        if (nxt.rows < kTile) { // rows past the segment: zeros, never stale or NaN data
                            LK::zero_rows(kt_s, nxt.rows, kTile, lane);
                            fence_proxy_async_smem();
                            __syncwarp();
                        }
                        tc::fence_after();
                        const uint32_t kbase = smem_u32(kt_s);
                        if (tc::elect_one()) {
#pragma unroll
                            for (int kk = 0; kk < RK / 16; ++kk)
                                tc::mma_bf16(tmem + C::COL_S + sb * NS, kdesc(kbase, kTile, kk), kdesc(qbase, NS, kk),
                                             idS, kk > 0 ? 1u : 0u);
                            tc::commit(bar(SFULL0 + sb));
                            tc::commit(kempty(st)); // the K stage is free once the scores are computed
                            if (nxt.flags & 2)
                                tc::commit(bar(QEMPTY)); // the unit's query tile is free after these
                        }
                        __syncwarp();
                        if (nxt.flags & 1)
                            ++k;
                        hist[ns & 1] = nxt;
                        ++ns;
                        more = walk.next(pref, a.seq_start, B, HU, nxt);
                        progress = true;
                    }
                }
                if (npv < ns) {
                    const int st = npv % kVStages, pb = npv & 1;
                    if (ready(bar(PFULL0 + pb), (npv >> 1) & 1) && ready(vfull(st), (npv / kVStages) & 1)) {
                        // output MMAs of tile npv: O^T (+)= C_V^T P^T; the first tile of a segment
                        // overwrites what the previous segment left
                        const TileDesc &dd = hist[npv & 1];
                        uint8_t *vt_s = smem + Ly.vring + st * C::VSTAGE;
                        if (dd.rows < kTile) {
                            LV::zero_rows(vt_s, dd.rows, kTile, lane);
                            fence_proxy_async_smem();
                            __syncwarp();
                        }
                        tc::fence_after();
                        const uint32_t vbase = smem_u32(vt_s);
                        if (tc::elect_one()) {
                            // a token step moves both descriptors' start fields by its byte offset / 16
#pragma unroll
                            for (int vb = 0; vb < C::VB; ++vb) {
                                const uint64_t v0 = vdesc(vbase, vb, 0), p0 = pdesc(pb, 0);
                                const uint32_t vstep = (2 * vb < LV::NBLK ? 2048u : 1024u) >> 4;
#pragma unroll 1
                                for (int kk = 0; kk < kTile / 16; ++kk)
                                    tc::mma_bf16(tmem + C::COL_O + vb * NS, v0 + kk * vstep, p0 + kk * (2048u >> 4),
                                                 idPV, (kk > 0 || !(dd.flags & 1)) ? 1u : 0u);
                            }
                            tc::commit(bar(PVDONE0 + pb));
                            tc::commit(vempty(st)); // the V stage is free once these complete
                        }
                        __syncwarp();
                        ++npv;
                        progress = true;
                    }
                }
                if (progress) {
                    spins = 0;
                    t_idle = 0;
                } else if ((++spins & 63u) == 0u) { // the clock only every 64 idle rounds
                    const uint64_t now = global_timer_ns();
                    if (t_idle == 0)
                        t_idle = now;
                    else if (now - t_idle > kWaitLimitNs)
                        err = true;
                }
                if (misc[0] != 0)
                    err = true;
            }
            if (err)
                misc[0] = 1;
        }
      }
    } else {
        // ================= softmax: group g = warps 4g .. 4g + 3; thread kq owns token kq ==========
        if constexpr (C::SPLIT)
            asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::SOFT_REGS));
        // A warp never leaves the loop early: on an error its waits fail at once and it only
        // keeps meeting the group's barriers, so the group stays in step.
        const int g = warp >> 2, q = warp & 3, kq = 32 * q + lane;
        const uint32_t tq_ = tmem + ((uint32_t)(32 * q) << 16); // this warp's lane quarter
        float *cm = reinterpret_cast<float *>(smem + Ly.cm);    // see alayout
        uint8_t *pt = smem + Ly.p;
        // the group's running reference per query lives in shared memory (the same for
        // all 128 threads), double-buffered: read buffer mc, a move writes the other one
        float *mref = cm + C::GROUPS * 6 * QG + g * 2 * QG;
        int mc = 0;
        float l[QG];
#pragma unroll
        for (int n = 0; n < QG; ++n)
            l[n] = 0.f;
        // x[n] = hi + lo of the group's columns of a tensor-memory block starting at `col`
        // (hi part; the lo part is NQ further), read in rounds of 8 columns
        auto ld_sum = [&](uint32_t col, float (&x)[QG]) {
#pragma unroll
            for (int c = 0; c < QG; c += 8) {
                uint32_t rh[8], rl[8];
                tc::ld_x8(tq_ + col + g * QG + c, rh);
                tc::ld_x8(tq_ + col + NQ + g * QG + c, rl);
                tc::wait_ld();
#pragma unroll
                for (int n = 0; n < 8; ++n)
                    x[c + n] = __uint_as_float(rh[n]) + __uint_as_float(rl[n]);
            }
        };
        float *alf = cm + C::GROUPS * 5 * QG + g * QG; // the group's rescale factors
        // record of query row nn of the current unit, slot j
        auto rec_of = [&](const TileDesc &dd, int nn) -> float * {
            const int hq = a.fold ? nn / lp : dd.h, t = a.fold ? nn - (nn / lp) * lp : nn;
            const int64_t u = (int64_t)dd.b * a.H + hq;
            return a.part + ((u * a.Tq_all + a.tq_off + t) * a.seg_max + dd.j) * part_stride(RV);
        };
        if (s0 < s1) {
            ShareWalk<kTile> walk;
            walk.start(s0, s1, chunk);
            TileDesc d;
            int i = 0;
            while (walk.next(pref, a.seq_start, B, HU, d)) {
                const int sb = i & 1;
                const bool first = d.flags & 1;
                // ---- scores of token kq against the group's queries: hi + lo columns.  The
                // buffer is held to the end of the tile (the MMA warp refills it only after
                // this tile's output MMAs anyway), so the rare rescale path can read it again.
                float s[QG];
                const bool s_ok = wait_all(bar(SFULL0 + sb), (i >> 1) & 1);
                auto load_scores = [&]() {
                    if (s_ok) {
                        ld_sum(C::COL_S + sb * NS, s);
#pragma unroll
                        for (int n = 0; n < QG; ++n)
                            s[n] = kq < d.rows ? s[n] : -INFINITY;
                    } else {
#pragma unroll
                        for (int n = 0; n < QG; ++n)
                            s[n] = -INFINITY;
                    }
                };
                if (s_ok)
                    tc::fence_after();
                load_scores();
                bool over = false;
                {
                    const float *mr = mref + mc * QG;
#pragma unroll
                    for (int n = 0; n < QG; ++n)
                        over |= s[n] > mr[n] + kMargin;
                }
                // the output MMAs of tile i - 2 have read weights buffer i & 1
                const int pb = i & 1;
                const bool pv_ok = s_ok && (i < 2 || wait_all(bar(PVDONE0 + pb), ((i >> 1) - 1) & 1));
                if (group_any(g, over)) {
                    // ---- the reference moves: column maxima of the tile over the group's tokens
                    // (the reduction consumes s; it is read again from tensor memory below)
                    const float wm = warp_columns<QG, true>(s, lane);
                    if (QG == 32 || (lane & 1) == 0)
                        cm[(g * 4 + q) * QG + lane * QG / 32] = wm;
                    group_sync(g);
                    bool drop = false;
                    const float *mr = mref + mc * QG;
                    float *mw = mref + (mc ^ 1) * QG;
#pragma unroll
                    for (int n = 0; n < QG; ++n) {
                        const float mx = fmaxf(fmaxf(cm[(g * 4 + 0) * QG + n], cm[(g * 4 + 1) * QG + n]),
                                               fmaxf(cm[(g * 4 + 2) * QG + n], cm[(g * 4 + 3) * QG + n]));
                        const float mo = mr[n], mn = fmaxf(mo, mx);
                        const float al = mo == -INFINITY ? 0.f : (mn == mo ? 1.f : fast_exp2(mo - mn));
                        drop |= al != 1.f;
                        l[n] *= al;
                        if (q == 0 && lane == 0) { // the same in every thread of the group
                            alf[n] = al;
                            mw[n] = mn;
                        }
                    }
                    group_sync(g); // the column maxima are read, the factors and references written
                    mc ^= 1;
                    // O^T: the group's columns shrink with the reference (the first tile of a
                    // segment overwrites them instead)
                    // (every earlier output MMA, tile i - 1's included, has to be complete)
                    if (!first && drop && pv_ok && wait_all(bar(PVDONE0 + (pb ^ 1)), ((i - 1) >> 1) & 1)) {
#pragma unroll
                        for (int vb = 0; vb < C::VB; ++vb) {
                            if (vb > 0 && q != 0)
                                continue; // a tail block holds r_v rows in lanes 0..31 only
#pragma unroll
                            for (int half = 0; half < 2; ++half)
#pragma unroll
                                for (int c = 0; c < QG; c += 16) {
                                    const uint32_t col = C::COL_O + vb * NS + half * NQ + g * QG + c;
                                    uint32_t r[16];
                                    tc::ld_x16(tq_ + col, r);
                                    tc::wait_ld();
#pragma unroll
                                    for (int n = 0; n < 16; ++n)
                                        r[n] = __float_as_uint(__uint_as_float(r[n]) * alf[c + n]);
                                    tc::st_x16(tq_ + col, r);
                                }
                        }
                        tc::wait_st();
                    }
                    load_scores();
                }
                // ---- weights of token kq: p = 2^(s - m), bf16 hi and lo into the MN-major tile
                if (pv_ok) {
                    const float *mr = mref + mc * QG;
#pragma unroll
                    for (int c = 0; c < QG / 8; ++c) {
                        float x[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int n = 8 * c + e;
                            x[e] = fast_exp2(s[n] - mr[n]); // masked tokens: 2^-inf = 0
                            l[n] += x[e];
                        }
                        uint4 hi, lo;
                        split8(x, hi, lo);
                        *reinterpret_cast<uint4 *>(pt + pb * C::P_BYTES + p_off(kq, g * QG + 8 * c)) = hi;
                        *reinterpret_cast<uint4 *>(pt + pb * C::P_BYTES + p_off(kq, NQ + g * QG + 8 * c)) = lo;
                    }
                }
                fence_proxy_async_smem(); // generic writes -> tensor-core reads
                tc::fence_before();       // the score reads and O^T stores before the arrivals
                __syncwarp();
                if (lane == 0 && s_ok)
                    mbar_arrive(bar(SEMPTY0 + sb));
                if (lane == 0 && pv_ok)
                    mbar_arrive(bar(PFULL0 + pb));
                if (d.flags & 2) {
                    // ---- segment end: O^T complete once this tile's output MMAs are
                    const bool fin = pv_ok && wait_all(bar(PVDONE0 + pb), (i >> 1) & 1);
                    tc::fence_after();
                    const float wl = warp_columns<QG, false>(l, lane); // l is reset below
                    if (QG == 32 || (lane & 1) == 0)
                        cm[(g * 4 + q) * QG + lane * QG / 32] = wl;
                    if (q == 0 && lane == 0) {
#pragma unroll
                        for (int n = 0; n < QG; ++n) {
                            cm[C::GROUPS * 4 * QG + g * QG + n] = mref[mc * QG + n];
                            mref[(mc ^ 1) * QG + n] = -INFINITY; // the next segment starts without one
                        }
                    }
                    group_sync(g);
                    const bool rec_ok = fin && misc[0] == 0 && d.j < a.seg_max;
                    if (rec_ok) {
#pragma unroll
                        for (int vb = 0; vb < C::VB; ++vb) {
                            const int v = 128 * vb + kq;
                            if (vb > 0 && q != 0)
                                continue;
                            float o[QG];
                            ld_sum(C::COL_O + vb * NS, o);
                            if (v < RV) {
#pragma unroll
                                for (int n = 0; n < QG; ++n) {
                                    const int nn = g * QG + n;
                                    if (nn < nq)
                                        rec_of(d, nn)[v] = o[n];
                                }
                            }
                        }
                        if (q == 0 && lane < QG && g * QG + lane < nq) {
                            const int nn = g * QG + lane;
                            const float L = cm[(g * 4 + 0) * QG + lane] + cm[(g * 4 + 1) * QG + lane] +
                                            cm[(g * 4 + 2) * QG + lane] + cm[(g * 4 + 3) * QG + lane];
                            float *rec = rec_of(d, nn);
                            rec[RV] = cm[C::GROUPS * 4 * QG + g * QG + lane];
                            rec[RV + 1] = L;
                        }
                        if (g == 0 && q == 0 && d.j == 0) {
                            if (a.fold) {
                                for (int h = lane; h < a.H; h += 32)
                                    a.counts[(int64_t)d.b * a.H + h] = d.n_u;
                            } else if (lane == 0) {
                                a.counts[d.u] = d.n_u;
                            }
                        }
                    } else if (g == 0 && kq == 0 && fin && d.j >= a.seg_max) {
                        report_status(a.status, LLA_ERR_INVALID); // a context longer than max_ctx
                    }
                    tc::fence_before();
                    group_sync(g); // the sums and references are read: the array is free again
                    mc ^= 1;
#pragma unroll
                    for (int n = 0; n < QG; ++n)
                        l[n] = 0.f;
                }
                ++i;
            }
        }
    }
    __syncwarp();
    all_sync<kThreads>(); // every role is done with tensor memory and the barriers
    if (warp == kMmaWarp) { // every MMA complete before tensor memory is released
        if (lane == 0)
            tc::commit(bar(DRAIN));
        __syncwarp();
        (void)mbar_wait_bounded(bar(DRAIN), 0);
        __syncwarp();
        tc::fence_after();
        tc::dealloc(tmem, C::TMEM_COLS);
    }
    if (misc[0] != 0 && warp == kProducerWarp && lane == 0) {
        // wind down: every copy still in flight lands before the CTA exits
        report_status(a.status, LLA_ERR_DEVICE_TIMEOUT);
        const int kt = misc[2], vt = misc[3];
        for (int i = kt - kKStages < 0 ? 0 : kt - kKStages; i < kt; ++i)
            (void)mbar_wait_bounded(kfull(i % kKStages), (i / kKStages) & 1);
        for (int i = vt - kVStages < 0 ? 0 : vt - kVStages; i < vt; ++i)
            (void)mbar_wait_bounded(vfull(i % kVStages), (i / kVStages) & 1);
    }
}

template <int RK, int RV, int NQ> int atc_smem_bytes(int B) { return (int)alayout<RK, RV, NQ>(B).total + 1024; }

template <int RK, int RV, int NQ> cudaError_t launch_atc(const DecodeArgs &a, cudaStream_t stream)
{
    CUtensorMap mk, mkt, mv, mvt;
    const int64_t rows = (int64_t)(a.fold ? 1 : a.H) * a.slots; // the folded plane, or H per-head planes
    if (!plane_maps(&mk, &mkt, a.k, RK, rows) || !plane_maps(&mv, &mvt, a.v, RV, rows))
        return cudaErrorInvalidValue;
    const int nq = a.fold ? a.H * a.Tq : a.Tq;
    if (nq < 1 || nq > NQ)
        return cudaErrorInvalidValue;
    auto kern = decode_absorb_tc_kernel<RK, RV, NQ>;
    const int smem = atc_smem_bytes<RK, RV, NQ>(a.B);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
        return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sms); // one persistent CTA per SM (tensor memory: 512 columns each)
    cfg.blockDim = dim3(ACfg<RK, RV, NQ>::THREADS);
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

// Ranks served: LLA-2D r 64/128 (H * loops <= 64 query rows per pass), per head r 96/160
// (up to 32 loop queries per pass).
int decode_absorb_tc_loops_per_pass(int fold, int H) { return fold == LLA_FOLD_2D ? (H >= 64 ? 1 : 64 / H) : 32; }

// The register split of an instantiation fits the registers it launches with (setmaxnreg.inc
// would wait forever otherwise).
template <int RK, int RV, int NQ> static bool atc_regs_fit()
{
    using C = ACfg<RK, RV, NQ>;
    if (!C::SPLIT)
        return true;
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, decode_absorb_tc_kernel<RK, RV, NQ>) != cudaSuccess)
        return false;
    return fa.numRegs * C::THREADS >= C::SPLIT_REGS;
}

bool decode_absorb_tc_supported(int dtype, int r_k, int r_v, int d_rope, int fold, int H, int B)
{
    if (dtype != LLA_BF16 || d_rope != 0 || tensor_map_encoder() == nullptr)
        return false;
    int smem = -1;
    bool regs = false;
    if (fold == LLA_FOLD_2D && r_k == 64 && r_v == 128 && H <= 64) {
        smem = std::max(atc_smem_bytes<64, 128, 64>(B), atc_smem_bytes<64, 128, 32>(B));
        regs = atc_regs_fit<64, 128, 64>() && atc_regs_fit<64, 128, 32>();
    } else if (fold == LLA_PER_HEAD && r_k == 96 && r_v == 160) {
        smem = atc_smem_bytes<96, 160, 32>(B);
        regs = atc_regs_fit<96, 160, 32>();
    }
    return regs && smem > 0 && smem <= 227 * 1024;
}

cudaError_t launch_decode_absorb_tc(const DecodeArgs &a, cudaStream_t stream)
{
    const int nq = a.fold ? a.H * a.Tq : a.Tq;
    if (a.fold && a.r_k == 64 && a.r_v == 128)
        return nq > 32 ? launch_atc<64, 128, 64>(a, stream) : launch_atc<64, 128, 32>(a, stream);
    if (!a.fold && a.r_k == 96 && a.r_v == 160)
        return launch_atc<96, 160, 32>(a, stream);
    return cudaErrorNotSupported;
}

} // namespace lla
