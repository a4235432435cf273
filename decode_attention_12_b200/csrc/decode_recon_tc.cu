// decode_recon_tc.cu -- LLA decode attention, reconstruct-on-read form (and the faithful
// read with rotary embedding), on tcgen05 tensor cores with tensor-memory accumulators.
//
// "Looped Latent Attention: Cross-Loop KV Compression for Looped Transformers": Pith
// review page, "What carries the argument" (Eq. 3: loop t reads x_hat_t = c W_up,t + mu_t)
// and arXiv abstract (K/V vectors are reconstructed only when attention reads them); the
// faithful read rotates query and rebuilt key at their positions after reconstruction
// (Pith verdict record, key_machinery; RoFormer's rotation).
//
// One latent tile of 128 tokens is read from HBM once and serves every loop query t of
// the pass (up to 4).  Per (tile, loop) step one thread issues, on the tensor cores,
//     K_hat   [128 tok x d] = C_K . W_up,t^K       M = tokens, N = d, K = r_k
//     V_hat^T [d x 128 tok] = W_up,t^V^T . C_V^T   M = d, N = tokens, K = r_v
// into tensor memory.  W_up,t enters as bf16 hi + lo parts (two MMAs whose products are
// exact in the fp32 accumulator), so the rebuilt vectors carry about 16 mantissa bits of
// W_up against exact bf16 latents.  mu_t^V is left out of V_hat and added once per record
// (sum_n p_n (v_hat_n - mu) + mu sum_n p_n); the score term q . mu_t^K is one constant per
// (unit, loop) -- with rotation the key's mean turns with the key, so there K_hat takes
// mu_t^K from one more MMA (a ones column against mu's hi/lo parts).
//
// Two groups of 8 warps take alternate steps, each with its own K_hat and V_hat^T
// buffers (4 x 128 of the 512 tensor-memory columns), so one group's scores overlap the
// other's output sums and the tensor cores' next rebuild.  Tensor memory is read in
// 16-lane x 256-bit fragments: each warp of a group owns a 16-row block of the buffers,
// and its lane holds two rows (rq and rq + 8 of the block, rq = lane / 4) and a quarter of
// their columns, so each shared-memory operand a lane loads serves two rows and a row's
// dot product closes over the 4 lanes of a quad.  Per step a warp:
//   * forms the scores of its 16 token rows of K_hat against the loop's query, picks a
//     warp reference (the group's running max, or its own max when that is more than a
//     lazy-rescale margin higher) and writes p to shared memory;
//   * after the group's barrier reconciles the 8 warps' references and reads its 16
//     d-rows of V_hat^T, forming sum_n p_n v_hat_n[d] over all 128 tokens of the tile.
// Records (acc, m, l) are merged across the two groups at segment ends and have the
// layout of the other reconstruct kernels, so the combine is shared.
//
// Faithful read: a query at position p and the rebuilt key of token n = n0 + r (tile row
// r) give <R(p) q, R(n) k> = <R(p - n0) q, R(r) k>: each group turns the query once per
// tile by (p - n0) (angles in double precision), and every thread keeps cos/sin(r w_i) of
// its row in registers for the whole kernel.  Component pairs (i, i + d/2) sit in one
// thread: the rows of W_up,t^K, q and mu_t^K are staged pair-major (identity for the
// half-split pairing, even-first for RoFormer's interleaved one).
//
// Work split: the token stream of all (head, sequence) units in head-major order is cut
// into equal shares, one per CTA (one CTA per SM), so a CTA's share mostly stays within
// one head and W_up is staged rarely.  Every wait is bounded; a timeout records
// LLA_ERR_DEVICE_TIMEOUT and the CTA winds down (tensor memory is always released).
#include "mma_common.cuh"
#include "tc_common.cuh"

namespace lla {
namespace {
using namespace mma;

constexpr int kD = 128;         // head dimension served
constexpr int kTile = 128;      // tokens per latent tile (M of the K_hat MMA)
constexpr int kMaxLoops = 4;    // loop queries per pass
constexpr int kGroups = 2;      // softmax warpgroups, alternate steps
constexpr int kGroupWarps = 8;  // two per tensor-memory lane quarter, one per 16-lane half
constexpr int kGroupThreads = kGroupWarps * 32;
constexpr int kSoftWarps = kGroups * kGroupWarps;
constexpr int kSoftThreads = kSoftWarps * 32;
constexpr int kProducerWarp = kSoftWarps, kMmaWarp = kSoftWarps + 1; // + 2 idle warps: a fifth warpgroup
constexpr int kThreads = (kSoftWarps + 4) * 32;
// Register split (setmaxnreg): 640 threads launch with 96 registers each (61,440 of the
// SM's 65,536); the producer/MMA warpgroup gives back to 56 and the four softmax warpgroups
// take 104: 512 x 104 + 128 x 56 = 60,416.  The host checks the count the kernel was built
// with before enabling it, so a split above the launch's total never runs.
constexpr int kSoftRegs = 104, kIssueRegs = 56;
constexpr int kSplitRegs = kSoftThreads * kSoftRegs + 128 * kIssueRegs;
constexpr float kRescale = 8.0f; // lazy rescale margin (log2 units)

// tensor-memory columns: K_hat of group g at 128 g, V_hat^T of group g at 256 + 128 g
constexpr uint32_t kTmemCols = 512;
__device__ __forceinline__ uint32_t col_k(int g) { return 128u * g; }
__device__ __forceinline__ uint32_t col_v(int g) { return 256u + 128u * g; }

// barriers after the ring's full[NST] and empty[NST]
enum { BKFULL0 = 0, BKFULL1, BKEMPTY0, BKEMPTY1, BVFULL0, BVFULL1, BVEMPTY0, BVEMPTY1, BWREADY, BDRAIN, BCOUNT };

struct RLayout {
    uint32_t nst, stage, wk, wv, wk_part, wv_part, ones, muk_t, qv, qt4, muk, muv, pv, alpha, xch, qmu, mrg,
        omg, bar, misc, scr, pref, total;
};

__host__ __device__ inline uint32_t round_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

// Shared-memory layout (byte offsets from a 1024-aligned base) for lp loops per pass and
// B sequences.  Every operand tile starts on a 1024-byte boundary.
template <int RK, int RV, bool ROPE> __host__ __device__ inline RLayout rlayout(int lp, int B)
{
    using LK = TileLayout<RK, kTile>;
    using LV = TileLayout<RV, kTile>;
    RLayout L;
    L.nst = (RK + RV) >= 64 ? 3 : 4;
    L.stage = align1024(LK::BYTES + LV::BYTES);
    uint32_t o = L.nst * L.stage;
    L.wk_part = kD * RK * 2;
    L.wv_part = kD * RV * 2;
    L.wk = o;
    o += lp * 2 * L.wk_part;
    L.wv = o;
    o += lp * 2 * L.wv_part;
    L.ones = o;
    o += ROPE ? kTile * 32 : 0;
    L.muk_t = o;
    o += ROPE ? lp * kD * 32 : 0;
    L.qv = o;                       // [lp][d] scaled query (kernel row order)
    o += lp * kD * 4;
    L.qt4 = o;                      // [group][lp][2 row offsets][32] turned query, pairs 2c, 2c+1
    o += ROPE ? kGroups * lp * 2 * 32 * 16 : 0;
    L.muk = o;                      // [lp][d]
    o += lp * kD * 4;
    L.muv = o;                      // [lp][d]
    o += lp * kD * 4;
    L.pv = o;                       // [group][2][128] softmax weights of a step
    o += kGroups * 2 * kTile * 4;
    L.alpha = o;                    // [group][2][8 warps] max references of a step
    o += kGroups * 2 * kGroupWarps * 4;
    L.xch = o;                      // [lp][d] group 1's share of a record
    o += lp * kD * 4;
    L.qmu = o;
    o += 16;
    L.mrg = o;                      // [16 warps][4 loops][m, l]
    o += kSoftWarps * kMaxLoops * 2 * 4;
    L.omg = round_up(o, 8);
    o = L.omg + (ROPE ? kD / 2 * 8 : 0);
    L.bar = round_up(o, 8);
    o = L.bar + (2 * L.nst + BCOUNT) * 8;
    L.misc = o;
    o += 16;
    L.scr = round_up(o, 8);
    o = L.scr + (kThreads / 32 + 1) * 8;
    L.pref = o;
    o += 8 * (B + 1);
    L.total = o;
    return L;
}

// Kernel row of d-index k on the key side: pair i is (row i, row i + d/2).
__device__ __forceinline__ int pair_row(int k, int style)
{
    return style == LLA_ROPE_INTERLEAVED ? (k & 1) * (kD / 2) + (k >> 1) : k;
}

// Walks a CTA's share of the head-major token stream (position p: head p / S, token
// p mod S of the concatenated sequences), unit segment by unit segment, tile by tile.
// The record slot of a segment is j = share - first share of its unit, as in the
// sequence-major walk of the other kernels, so the combine reads it the same way.
template <int TILE> struct HeadWalk {
    int64_t pos, end, chunk, S, seq0;
    int32_t b, h, n, seg_end, u, j, n_u;
    bool in_seg;

    __device__ void start(int64_t p, int64_t e, int64_t ch, int64_t s_tot)
    {
        pos = p;
        end = e;
        chunk = ch;
        S = s_tot;
        b = 0;
        in_seg = false;
    }
    __device__ bool next(const int64_t *pref, const int64_t *starts, int B, int H, TileDesc &d)
    {
        if (!in_seg) {
            if (pos >= end)
                return false;
            h = (int)(pos / S);
            const int64_t q = pos - (int64_t)h * S;
            if (!(pref[b] <= q && q < pref[b + 1])) {
                if (b + 2 <= B && pref[b + 1] <= q && q < pref[b + 2]) {
                    ++b;
                } else { // largest b with pref[b] <= q (skips empty sequences)
                    int lo = 0, hi = B - 1;
                    while (lo < hi) {
                        const int mid = (lo + hi + 1) >> 1;
                        if (pref[mid] <= q)
                            lo = mid;
                        else
                            hi = mid - 1;
                    }
                    b = lo;
                }
            }
            const int len = (int)(pref[b + 1] - pref[b]);
            seq0 = starts[b];
            n = (int)(q - pref[b]);
            const int64_t take = min((int64_t)(len - n), end - pos);
            seg_end = n + (int)take;
            pos += take;
            u = b * H + h;
            const int64_t U = (int64_t)h * S + pref[b]; // unit start in the stream
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
        d.rows = min(TILE, seg_end - n);
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

__device__ __forceinline__ float2 f2(uint32_t x, uint32_t y) { return make_float2(__uint_as_float(x), __uint_as_float(y)); }

__device__ __forceinline__ void group_sync(int g)
{
    asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "r"(kGroupThreads) : "memory");
}
__device__ __forceinline__ void soft_sync() { asm volatile("bar.sync 3, %0;" ::"r"(kSoftThreads) : "memory"); }
__device__ __forceinline__ void all_sync() { asm volatile("bar.sync 4, %0;" ::"r"(kThreads) : "memory"); }

template <int RK, int RV, bool ROPE>
__global__ void __launch_bounds__(kThreads, 1)
    decode_recon_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                           const DecodeArgs a)
{
    using LK = TileLayout<RK, kTile>;
    using LV = TileLayout<RV, kTile>;
    using L16 = TileLayout<16, kTile>;
    extern __shared__ uint8_t smem_raw[];
    // aligned by arithmetic on the shared array itself, so accesses stay shared-space loads
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int lp = a.Tq;
    const RLayout Ly = rlayout<RK, RV, ROPE>(lp, a.B);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + Ly.bar;
    const uint32_t nst = Ly.nst;
    volatile int *misc = reinterpret_cast<volatile int *>(smem + Ly.misc); // [0] error, [1] tmem, [2] issued
    int64_t *pref = reinterpret_cast<int64_t *>(smem + Ly.pref);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int B = a.B, H = a.H;
    auto full_bar = [&](int st) { return bar0 + 8u * st; };
    auto empty_bar = [&](int st) { return bar0 + 8u * (nst + st); };
    auto bar = [&](int k) { return bar0 + 8u * (2 * nst + k); };

    if (tid == 0) {
        for (uint32_t st = 0; st < nst; ++st) {
            mbar_init(full_bar(st), 1);  // producer's expect_tx + TMA bytes
            mbar_init(empty_bar(st), 1); // the tile's last MMAs completed (commit)
        }
        for (int g = 0; g < kGroups; ++g) {
            mbar_init(bar(BKFULL0 + g), 1);
            mbar_init(bar(BKEMPTY0 + g), kGroupWarps); // one arrival per warp of the group
            mbar_init(bar(BVFULL0 + g), 1);
            mbar_init(bar(BVEMPTY0 + g), kGroupWarps);
        }
        mbar_init(bar(BWREADY), 1);
        mbar_init(bar(BDRAIN), 1);
        misc[0] = 0;
        misc[2] = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp)
        tc::alloc(reinterpret_cast<uint32_t *>(smem + Ly.misc + 4), kTmemCols);
    if (ROPE) {
        // ones tile [128 rows][16]: columns 0 and 1 are 1 (they meet mu's hi and lo parts)
        const __nv_bfloat162 one2 = __floats2bfloat162_rn(1.f, 1.f);
        for (int r = tid; r < kTile; r += kThreads) {
            *reinterpret_cast<uint4 *>(smem + Ly.ones + L16::off(r, 0)) =
                make_uint4(*reinterpret_cast<const uint32_t *>(&one2), 0u, 0u, 0u);
            *reinterpret_cast<uint4 *>(smem + Ly.ones + L16::off(r, 1)) = make_uint4(0u, 0u, 0u, 0u);
        }
        double *omg = reinterpret_cast<double *>(smem + Ly.omg);
        for (int i = tid; i < kD / 2; i += kThreads)
            omg[i] = pow((double)a.rope_base, -2.0 * i / kD);
        fence_proxy_async_smem(); // the ones tile is read by the tensor cores
    }
    tc::fence_before();
    block_length_prefix<kThreads>(a.ctx_lens, B, pref, reinterpret_cast<int64_t *>(smem + Ly.scr));
    tc::fence_after();
    const uint32_t tmem = (uint32_t)misc[1];
    // The combine grid may take SM slots as this grid's CTAs exit; it reads nothing of
    // ours before its own programmatic-launch wait.
    grid_launch_dependents();
    int64_t s0, s1, chunk;
    cta_share(pref, B, H, a.chunk_min, s0, s1, chunk);
    const int64_t S_tot = pref[B];
    if (warp >= kSoftWarps) {
      // ======== fifth warpgroup: producer warp, MMA warp, two idle warps ========
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kIssueRegs));
      if (s0 < s1 && warp == kProducerWarp) {
        // ================= producer: one lane streams the latent tiles =================
        if (lane == 0) {
            HeadWalk<kTile> walk;
            walk.start(s0, s1, chunk, S_tot);
            TileDesc d;
            int issued = 0;
            while (walk.next(pref, a.seq_start, B, H, d)) {
                const int i = issued, st = i % (int)nst;
                if (i >= (int)nst && !mbar_wait_bounded(empty_bar(st), ((i / nst) - 1) & 1)) {
                    misc[0] = 1;
                    break;
                }
                if (misc[0])
                    break;
                const uint32_t sk = sbase + st * Ly.stage, sv = sk + LK::BYTES;
                const int nbox = (d.rows + kBox - 1) / kBox;
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(full_bar(st), nbox * kBox * (RK + RV) * 2);
                const int y0 = (int)((int64_t)d.h * a.slots + d.row);
                for (int bx = 0; bx < nbox; ++bx) {
                    tma_load_2d(sk + bx * kBox * LK::TB, &map_k, 0, y0 + bx * kBox, full_bar(st));
                    tma_load_2d(sv + bx * kBox * LV::TB, &map_v, 0, y0 + bx * kBox, full_bar(st));
                }
                ++issued;
            }
            misc[2] = issued;
        }
      } else if (s0 < s1 && warp == kMmaWarp) {
        // ================= MMA issuer: the whole warp runs the loop, one elected lane issues =================
        // Shared-memory descriptors are formed once; moving a descriptor's start address by
        // `bytes` adds bytes / 16 to its low field (every operand lies below 256 KB).
        {
            constexpr uint32_t kIdKV = tc::idesc(tc::kFmtBf16, 128, 128);
            const uint64_t dK0 = tc::smem_desc(sbase, 2 * RK);                // latent K tile of stage 0
            const uint64_t dV0 = tc::smem_desc(sbase + LK::BYTES, 2 * RV);    // latent V tile of stage 0
            const uint64_t dWk = tc::smem_desc(sbase + Ly.wk, 2 * RK);        // W_up^K^T parts
            const uint64_t dWv = tc::smem_desc(sbase + Ly.wv, 2 * RV);        // W_up^V^T parts
            const uint64_t dOnes = tc::smem_desc(sbase + Ly.ones, 32);
            const uint64_t dMu = tc::smem_desc(sbase + Ly.muk_t, 32);
            const uint32_t stage_units = Ly.stage >> 4, wk_units = Ly.wk_part >> 4, wv_units = Ly.wv_part >> 4;
            bool err = false;
            auto wait_all = [&](uint32_t b, uint32_t parity) -> bool {
                bool ok = !err && misc[0] == 0 && mbar_wait_bounded(b, parity);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) {
                    err = true;
                    misc[0] = 1;
                }
                return ok;
            };
            HeadWalk<kTile> walk;
            walk.start(s0, s1, chunk, S_tot);
            TileDesc d;
            int s = 0, ti = 0, wc = 0, prev_h = -1;
            while (!err && walk.next(pref, a.seq_start, B, H, d)) {
                const int st = ti % (int)nst;
                if ((d.flags & 1) && d.h != prev_h) {
                    // a new head's W_up: staged once every MMA of the old one has been consumed
                    if (!wait_all(bar(BWREADY), wc & 1))
                        break;
                    ++wc;
                    prev_h = d.h;
                }
                if (!wait_all(full_bar(st), (ti / nst) & 1))
                    break;
                if (d.rows < kTile) { // rows past the segment: zeros, never stale or NaN data
                    LK::zero_rows(smem + st * Ly.stage, d.rows, kTile, lane);
                    LV::zero_rows(smem + st * Ly.stage + LK::BYTES, d.rows, kTile, lane);
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                const uint64_t dK = dK0 + st * stage_units, dV = dV0 + st * stage_units;
                for (int t = 0; t < lp && !err; ++t, ++s) {
                    const int g = s & 1, use = s >> 1; // group g's use number of its buffers
                    // the group has read both buffers of its previous step (V after K)
                    if (use >= 1 && !wait_all(bar(BVEMPTY0 + g), (use - 1) & 1))
                        break;
                    tc::fence_after();
                    const uint64_t wk = dWk + 2 * t * wk_units, wv = dWv + 2 * t * wv_units;
                    const uint32_t dk_t = tmem + col_k(g), dv_t = tmem + col_v(g);
                    if (tc::elect_one()) {
#pragma unroll
                        for (int kk = 0; kk < RK / 16; ++kk)
#pragma unroll
                            for (int hl = 0; hl < 2; ++hl)
                                tc::mma_bf16(dk_t, dK + 2 * kk, wk + hl * wk_units + 2 * kk, kIdKV, (kk | hl) != 0);
                        if (ROPE)
                            tc::mma_bf16(dk_t, dOnes, dMu + t * (kD * 32 / 16), kIdKV, 1);
                        tc::commit(bar(BKFULL0 + g));
#pragma unroll
                        for (int kk = 0; kk < RV / 16; ++kk)
#pragma unroll
                            for (int hl = 0; hl < 2; ++hl)
                                tc::mma_bf16(dv_t, wv + hl * wv_units + 2 * kk, dV + 2 * kk, kIdKV, (kk | hl) != 0);
                        tc::commit(bar(BVFULL0 + g));
                        if (t == lp - 1)
                            tc::commit(empty_bar(st)); // the tile's stage is free once these complete
                    }
                    __syncwarp();
                }
                ++ti;
            }
        }
      }
      __syncwarp();
      all_sync(); // the softmax groups have consumed every MMA result
      if (warp == kMmaWarp) { // every MMA complete before tensor memory is released
          if (lane == 0)
              tc::commit(bar(BDRAIN));
          __syncwarp();
          (void)mbar_wait_bounded(bar(BDRAIN), 0);
          __syncwarp();
          tc::fence_after();
          tc::dealloc(tmem, kTmemCols);
      }
      if (misc[0] != 0 && warp == kProducerWarp && lane == 0) {
          report_status(a.status, LLA_ERR_DEVICE_TIMEOUT);
          const int issued = misc[2];
          for (int i = issued - (int)nst < 0 ? 0 : issued - (int)nst; i < issued; ++i)
              (void)mbar_wait_bounded(full_bar(i % nst), (i / nst) & 1);
      }
    } else {
      // ======== two groups of 8 warps, alternate steps ========
      // Tensor memory is read in 16-lane x 256-bit fragments.  Warp (wq, hh) of a group owns
      // lanes 32 wq + 16 hh .. + 15 of the buffers; its lane t holds rows rq and rq + 8
      // (rq = t / 4) of those 16 and columns 8 i + 2 j + {0, 1} (j = t % 4), so a query or
      // weight pair it loads from shared memory serves two rows, and a row's sum closes over
      // the 4 lanes of a quad.
      asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftRegs));
      if (s0 < s1) {
        const int g = warp / kGroupWarps, gw = warp % kGroupWarps, wq = gw & 3, hh = gw >> 2;
        const int r = tid % kGroupThreads, j = lane & 3, rq = lane >> 2;
        const int tb = 2 * wq + hh;                      // this warp's 16-row block of the tile
        const uint32_t tq = tmem + ((uint32_t)(32 * wq + 16 * hh) << 16);
        auto row_of = [&](int e) { return 16 * tb + 8 * e + rq; }; // tile row / d-index of row e
        bool err = false;
        auto wait_all = [&](uint32_t b, uint32_t parity) -> bool {
            bool ok = !err && misc[0] == 0 && mbar_wait_bounded(b, parity);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) {
                err = true;
                misc[0] = 1;
            }
            return ok;
        };
        auto quad_sum = [&](float x) {
            x += __shfl_xor_sync(0xffffffffu, x, 1);
            return x + __shfl_xor_sync(0xffffffffu, x, 2);
        };
        // rotation of the thread's base row b0 = 16 tb + rq: (cos, sin)(b0 w_P) for the pairs
        // P = 8 i + 2 j + {0, 1}, i = 0..7 (row b0 + 8 takes a query turned 8 steps further)
        float2 rc[ROPE ? 8 : 1], rs[ROPE ? 8 : 1];
        if (ROPE) {
            const float lb = log2f(a.rope_base);
            const float b0 = (float)(16 * tb + rq);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float sa, ca, sb, cb;
                sincosf(b0 * exp2f(-2.0f * (float)(8 * i + 2 * j) / (float)kD * lb), &sa, &ca);
                sincosf(b0 * exp2f(-2.0f * (float)(8 * i + 2 * j + 1) / (float)kD * lb), &sb, &cb);
                rc[i] = make_float2(ca, cb);
                rs[i] = make_float2(sa, sb);
            }
        }
        // per loop: the group's running max (uniform), this thread's share of the sum of
        // weights (the row it writes), output sums of its 2 d-rows
        float m[kMaxLoops], l[kMaxLoops], oacc[kMaxLoops][2];
        const float *qv = reinterpret_cast<const float *>(smem + Ly.qv);
        const float *qmu = reinterpret_cast<const float *>(smem + Ly.qmu);
        const float *muv = reinterpret_cast<const float *>(smem + Ly.muv);
        float *mrg = reinterpret_cast<float *>(smem + Ly.mrg);
        float *xch = reinterpret_cast<float *>(smem + Ly.xch);

        // segment end: merge the two groups' states into one record per loop
        auto flush = [&](const TileDesc &dd) {
#pragma unroll
            for (int t = 0; t < kMaxLoops; ++t) {
                if (t < lp) {
                    float lq = l[t];
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1)
                        lq += __shfl_xor_sync(0xffffffffu, lq, off);
                    if (lane == 0) {
                        mrg[(warp * kMaxLoops + t) * 2] = m[t];
                        mrg[(warp * kMaxLoops + t) * 2 + 1] = lq;
                    }
                }
            }
            soft_sync();
            float M[kMaxLoops], wg[kMaxLoops];
#pragma unroll
            for (int t = 0; t < kMaxLoops; ++t) {
                M[t] = -INFINITY;
                wg[t] = 0.f;
                if (t < lp) {
                    const float m0 = mrg[(0 * kMaxLoops + t) * 2], m1 = mrg[(kGroupWarps * kMaxLoops + t) * 2];
                    M[t] = fmaxf(m0, m1);
                    const float mine = g == 0 ? m0 : m1;
                    wg[t] = mine == -INFINITY ? 0.f : fast_exp2(mine - M[t]);
                    if (g == 1 && j < 2)
                        xch[t * kD + row_of(j)] = wg[t] * (j == 0 ? oacc[t][0] : oacc[t][1]);
                }
            }
            soft_sync();
            if (g == 0 && misc[0] == 0 && dd.j < a.seg_max) {
#pragma unroll
                for (int t = 0; t < kMaxLoops; ++t) {
                    if (t < lp) {
                        float L = 0.f;
#pragma unroll
                        for (int w = 0; w < kSoftWarps; ++w) {
                            const float mw = mrg[(w * kMaxLoops + t) * 2];
                            if (mw != -INFINITY)
                                L = fmaf(fast_exp2(mw - M[t]), mrg[(w * kMaxLoops + t) * 2 + 1], L);
                        }
                        float *rec = a.part + (((int64_t)dd.u * a.Tq_all + a.tq_off + t) * a.seg_max + dd.j) *
                                                  part_stride(kD);
                        if (j < 2) {
                            const int d = row_of(j);
                            // + L mu_t^V: the mean left out of V_hat
                            rec[d] = fmaf(L, muv[t * kD + d],
                                          fmaf(wg[t], j == 0 ? oacc[t][0] : oacc[t][1], xch[t * kD + d]));
                        }
                        if (r == 0) {
                            rec[kD] = M[t];
                            rec[kD + 1] = L;
                        }
                    }
                }
                if (r == 0 && dd.j == 0)
                    a.counts[dd.u] = dd.n_u;
            } else if (g == 0 && r == 0 && dd.j >= a.seg_max) {
                report_status(a.status, LLA_ERR_INVALID); // a context longer than max_ctx
            }
            soft_sync(); // mrg and xch free again
        };

        HeadWalk<kTile> walk;
        walk.start(s0, s1, chunk, S_tot);
        TileDesc d, dseg;
        bool have_seg = false;
        int s = 0, prev_h = -1;
        int32_t qpos = 0;
        const int st_ = tid; // 0 .. kSoftThreads - 1
        while (walk.next(pref, a.seq_start, B, H, d)) {
            if (d.flags & 1) {
                // ---- new unit segment: close the previous one, stage this one's inputs
                if (have_seg)
                    flush(dseg);
                dseg = d;
                have_seg = true;
                const bool wchange = d.h != prev_h;
                const int style = a.rope_style;
                for (int t = 0; t < lp; ++t) {
                    const int tl = a.t0 + a.tq_off + t;
                    const int64_t gi = ((int64_t)d.h * a.T + tl);
                    if (wchange) {
                        // W_up,t^K^T and W_up,t^V^T as bf16 hi/lo K-major tiles (rows = d)
                        const float *wk = a.W_up_k + gi * RK * kD;
                        const float *wv = a.W_up_v + gi * RV * kD;
                        uint8_t *dk = smem + Ly.wk + t * 2 * Ly.wk_part;
                        uint8_t *dv = smem + Ly.wv + t * 2 * Ly.wv_part;
                        for (int e = st_; e < RK * kD; e += kSoftThreads) {
                            const int jj = e / kD, k = e - jj * kD;
                            const int row = ROPE ? pair_row(k, style) : k;
                            const float x = wk[e];
                            const __nv_bfloat16 hi = __float2bfloat16_rn(x);
                            const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
                            const uint32_t off = LK::off(row, jj >> 3) + (jj & 7) * 2;
                            *reinterpret_cast<__nv_bfloat16 *>(dk + off) = hi;
                            *reinterpret_cast<__nv_bfloat16 *>(dk + Ly.wk_part + off) = lo;
                        }
                        for (int e = st_; e < RV * kD; e += kSoftThreads) {
                            const int jj = e / kD, k = e - jj * kD;
                            const float x = wv[e];
                            const __nv_bfloat16 hi = __float2bfloat16_rn(x);
                            const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
                            const uint32_t off = LV::off(k, jj >> 3) + (jj & 7) * 2;
                            *reinterpret_cast<__nv_bfloat16 *>(dv + off) = hi;
                            *reinterpret_cast<__nv_bfloat16 *>(dv + Ly.wv_part + off) = lo;
                        }
                        if (st_ < kD) {
                            const int k = st_;
                            const float mk = a.mu_k[gi * kD + k];
                            const int row = ROPE ? pair_row(k, style) : k;
                            reinterpret_cast<float *>(smem + Ly.muk)[t * kD + row] = mk;
                            reinterpret_cast<float *>(smem + Ly.muv)[t * kD + k] = a.mu_v[gi * kD + k];
                            if (ROPE) { // mu_t^K as the B tile of the ones MMA: columns 0, 1 = hi, lo
                                const __nv_bfloat16 hi = __float2bfloat16_rn(mk);
                                const __nv_bfloat16 lo = __float2bfloat16_rn(mk - __bfloat162float(hi));
                                const __nv_bfloat162 hl = __halves2bfloat162(hi, lo);
                                uint8_t *mt = smem + Ly.muk_t + t * kD * 32;
                                *reinterpret_cast<uint4 *>(mt + L16::off(row, 0)) =
                                    make_uint4(*reinterpret_cast<const uint32_t *>(&hl), 0u, 0u, 0u);
                                *reinterpret_cast<uint4 *>(mt + L16::off(row, 1)) = make_uint4(0u, 0u, 0u, 0u);
                            }
                        }
                    }
                    if (st_ >= kD && st_ < 2 * kD) { // scaled query of this (sequence, head) and loop
                        const int k = st_ - kD;
                        const __nv_bfloat16 *qrow = static_cast<const __nv_bfloat16 *>(a.q) +
                                                    (((int64_t)d.b * a.Tq_all + a.tq_off + t) * H + d.h) * kD;
                        reinterpret_cast<float *>(smem + Ly.qv)[t * kD + (ROPE ? pair_row(k, style) : k)] =
                            __bfloat162float(qrow[k]) * a.scale * kLog2e;
                    }
                }
                if (wchange)
                    fence_proxy_async_smem(); // W and mu tiles are read by the tensor cores
                soft_sync();
                if (wchange && tid == 0)
                    mbar_arrive(bar(BWREADY));
                prev_h = d.h;
                if (!ROPE && warp < lp) { // constant score term q . mu_t^K (log2 units)
                    const float *mk = reinterpret_cast<const float *>(smem + Ly.muk) + warp * kD;
                    float qm = 0.f;
                    for (int k = lane; k < kD; k += 32)
                        qm = fmaf(qv[warp * kD + k], mk[k], qm);
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1)
                        qm += __shfl_xor_sync(0xffffffffu, qm, off);
                    if (lane == 0)
                        reinterpret_cast<float *>(smem + Ly.qmu)[warp] = qm;
                }
                if (ROPE)
                    qpos = a.q_pos[d.b];
                soft_sync();
#pragma unroll
                for (int t = 0; t < kMaxLoops; ++t) {
                    m[t] = -INFINITY;
                    l[t] = 0.f;
                    oacc[t][0] = oacc[t][1] = 0.f;
                }
            }
            // does this group take any step of the tile?
            const bool mine = lp > 1 || (s & 1) == g;
            if (ROPE && mine) {
                // the tile's query, once per row offset 8 v (v = 0, 1) within a 16-row block:
                // R((p - n0 - 8 v) w) q for pairs 2c, 2c + 1; entry [loop][v][couple c]; the
                // block offset 16 tb sits in the thread's own rotation
                const double *omg = reinterpret_cast<const double *>(smem + Ly.omg);
                float4 *qt = reinterpret_cast<float4 *>(smem + Ly.qt4) + g * lp * 2 * 32;
                for (int e = r; e < lp * 2 * 32; e += kGroupThreads) {
                    const int c = e & 31, v = (e >> 5) & 1, t = e >> 6;
                    const int64_t rel = (int64_t)qpos - d.n0 - 8 * v;
                    float qa2[2], qb2[2];
#pragma unroll
                    for (int ee = 0; ee < 2; ++ee) {
                        const int i = 2 * c + ee;
                        const double ang = (double)rel * omg[i];
                        const float red = (float)(ang - 6.283185307179586 * rint(ang * 0.15915494309189535));
                        float sn, cs;
                        sincosf(red, &sn, &cs);
                        const float x = qv[t * kD + i], y = qv[t * kD + i + kD / 2];
                        qa2[ee] = x * cs - y * sn;
                        qb2[ee] = x * sn + y * cs;
                    }
                    qt[e] = make_float4(qa2[0], qa2[1], qb2[0], qb2[1]);
                }
                group_sync(g);
            }
#pragma unroll
            for (int t = 0; t < kMaxLoops; ++t) {
                if (t >= lp)
                    break;
                const int ss = s + t;
                if ((ss & 1) != g)
                    continue;
                const int use = ss >> 1;
                const int pb = use & 1; // this group's weight / reference buffer of the step
                // ---- scores of loop t for the thread's 2 token rows
                float sc[2] = {-INFINITY, -INFINITY};
                if (wait_all(bar(BKFULL0 + g), use & 1)) {
                    tc::fence_after();
                    float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                    if (!ROPE) {
                        const float2 *q2 = reinterpret_cast<const float2 *>(qv + t * kD + 2 * j); // q pairs
#pragma unroll
                        for (int c = 0; c < 2; ++c) { // columns 64 c .. 64 c + 63
                            uint32_t kr[32];
                            tc::ld_16x256b_x8(tq + col_k(g) + 64 * c, kr);
                            tc::wait_ld();
                            if (c == 1) {
                                tc::fence_before();
                                __syncwarp();
                                if (lane == 0)
                                    mbar_arrive(bar(BKEMPTY0 + g));
                            }
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const float2 qq = q2[4 * (8 * c + i)];
                                acc[0] = __ffma2_rn(qq, f2(kr[4 * i], kr[4 * i + 1]), acc[0]);
                                acc[1] = __ffma2_rn(qq, f2(kr[4 * i + 2], kr[4 * i + 3]), acc[1]);
                            }
                        }
                        sc[0] = quad_sum(acc[0].x + acc[0].y) + qmu[t];
                        sc[1] = quad_sum(acc[1].x + acc[1].y) + qmu[t];
                    } else {
                        // row e uses the query turned by its row offset 8 e
                        const float4 *qt = reinterpret_cast<const float4 *>(smem + Ly.qt4) + (g * lp + t) * 2 * 32;
#pragma unroll
                        for (int c = 0; c < 2; ++c) { // pairs 32 c .. 32 c + 31: columns i and i + 8
                            uint32_t ka[16], kb[16];
                            tc::ld_16x256b_x4(tq + col_k(g) + 32 * c, ka);
                            tc::ld_16x256b_x4(tq + col_k(g) + kD / 2 + 32 * c, kb);
                            tc::wait_ld();
                            if (c == 1) {
                                tc::fence_before();
                                __syncwarp();
                                if (lane == 0)
                                    mbar_arrive(bar(BKEMPTY0 + g));
                            }
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
#pragma unroll
                                for (int ii = 0; ii < 4; ++ii) {
                                    const int i = 4 * c + ii;
                                    const float4 qq = qt[e * 32 + 4 * i + j];
                                    const float2 qa = make_float2(qq.x, qq.y), qb = make_float2(qq.z, qq.w);
                                    const float2 qas = __fmul2_rn(qa, rs[i]);
                                    // x (qa cos + qb sin) + y (qb cos - qa sin)
                                    const float2 t1 = __ffma2_rn(qa, rc[i], __fmul2_rn(qb, rs[i]));
                                    const float2 t2 = __ffma2_rn(qb, rc[i], make_float2(-qas.x, -qas.y));
                                    acc[e] = __ffma2_rn(f2(ka[4 * ii + 2 * e], ka[4 * ii + 2 * e + 1]), t1, acc[e]);
                                    acc[e] = __ffma2_rn(f2(kb[4 * ii + 2 * e], kb[4 * ii + 2 * e + 1]), t2, acc[e]);
                                }
                            }
                        }
                        sc[0] = quad_sum(acc[0].x + acc[0].y);
                        sc[1] = quad_sum(acc[1].x + acc[1].y);
                    }
                } else {
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(bar(BKEMPTY0 + g));
                }
                if (row_of(0) >= d.rows)
                    sc[0] = -INFINITY;
                if (row_of(1) >= d.rows)
                    sc[1] = -INFINITY;
                // ---- online softmax: each warp picks a reference (the group's running max, or
                // its own max when that is more than the margin higher), the group reconciles
                float mx = fmaxf(sc[0], sc[1]);
#pragma unroll
                for (int off = 4; off < 32; off <<= 1)
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                const float ref = mx > m[t] + kRescale ? mx : m[t];
                const float sm_ = j == 0 ? sc[0] : sc[1];
                const float pmine = sm_ == -INFINITY ? 0.f : fast_exp2(sm_ - ref); // rows j = 0, 1 write
                float *pw = reinterpret_cast<float *>(smem + Ly.pv) + (g * 2 + pb) * kTile;
                float *rw = reinterpret_cast<float *>(smem + Ly.alpha) + (g * 2 + pb) * kGroupWarps;
                if (j < 2)
                    pw[row_of(j)] = pmine;
                if (lane == 0)
                    rw[tb] = ref;
                group_sync(g);
                const float4 ra = *reinterpret_cast<const float4 *>(rw), rb = *reinterpret_cast<const float4 *>(rw + 4);
                const float Mn = fmaxf(fmaxf(fmaxf(ra.x, ra.y), fmaxf(ra.z, ra.w)), fmaxf(fmaxf(rb.x, rb.y), fmaxf(rb.z, rb.w)));
                float f[8] = {1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f};
                const bool same = ra.x == Mn && ra.y == Mn && ra.z == Mn && ra.w == Mn && rb.x == Mn && rb.y == Mn &&
                                  rb.z == Mn && rb.w == Mn;
                if (Mn != -INFINITY && !same) {
                    f[0] = fast_exp2(ra.x - Mn);
                    f[1] = fast_exp2(ra.y - Mn);
                    f[2] = fast_exp2(ra.z - Mn);
                    f[3] = fast_exp2(ra.w - Mn);
                    f[4] = fast_exp2(rb.x - Mn);
                    f[5] = fast_exp2(rb.y - Mn);
                    f[6] = fast_exp2(rb.z - Mn);
                    f[7] = fast_exp2(rb.w - Mn);
                }
                if (Mn > m[t]) { // the group's max rose: rescale what was summed so far
                    const float al = fast_exp2(m[t] - Mn);
                    l[t] *= al;
                    oacc[t][0] *= al;
                    oacc[t][1] *= al;
                    m[t] = Mn;
                }
                if (j < 2)
                    l[t] = fmaf(f[tb], pmine, l[t]);
                // ---- output: sum over the tile's tokens of p v_hat at the thread's 2 d-rows
                float2 pacc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                if (wait_all(bar(BVFULL0 + g), use & 1)) {
                    tc::fence_after();
                    const float2 *p2 = reinterpret_cast<const float2 *>(pw + 2 * j); // tokens 8 i + 2 j
#pragma unroll
                    for (int c = 0; c < 2; ++c) { // tokens 64 c .. 64 c + 63
                        uint32_t vr[32];
                        tc::ld_16x256b_x8(tq + col_v(g) + 64 * c, vr);
                        tc::wait_ld();
                        if (c == 1) {
                            tc::fence_before();
                            __syncwarp();
                            if (lane == 0)
                                mbar_arrive(bar(BVEMPTY0 + g));
                        }
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int ti = 8 * c + i; // tokens 8 ti + 2 j: 16-row block ti / 2
                            float2 pq = p2[4 * ti];
                            if (!same)
                                pq = make_float2(pq.x * f[ti >> 1], pq.y * f[ti >> 1]);
                            pacc[0] = __ffma2_rn(pq, f2(vr[4 * i], vr[4 * i + 1]), pacc[0]);
                            pacc[1] = __ffma2_rn(pq, f2(vr[4 * i + 2], vr[4 * i + 3]), pacc[1]);
                        }
                    }
                } else {
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(bar(BVEMPTY0 + g));
                }
                oacc[t][0] += quad_sum(pacc[0].x + pacc[0].y);
                oacc[t][1] += quad_sum(pacc[1].x + pacc[1].y);
            }
            s += lp;
        }
        if (have_seg)
            flush(dseg);
      }
      __syncwarp();
      all_sync();
    }
}

template <int RK, int RV, bool ROPE> cudaError_t launch_rtc(const DecodeArgs &a, cudaStream_t stream)
{
    CUtensorMap mk, mkt, mv, mvt;
    if (!plane_maps(&mk, &mkt, a.k, RK, (int64_t)a.H * a.slots) ||
        !plane_maps(&mv, &mvt, a.v, RV, (int64_t)a.H * a.slots))
        return cudaErrorInvalidValue;
    if (a.Tq < 1 || a.Tq > kMaxLoops)
        return cudaErrorInvalidValue;
    auto kern = decode_recon_tc_kernel<RK, RV, ROPE>;
    const int smem = (int)rlayout<RK, RV, ROPE>(a.Tq, a.B).total + 1024;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
        return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // tail maps only: ranks up to 32 are one 32- or 64-byte box column
    kern<<<sms, kThreads, smem, stream>>>(mkt, mvt, a);
    return cudaGetLastError();
}

} // namespace

int decode_recon_tc_smem_bytes(int r_k, int r_v, bool rope, int lp, int B)
{
#define LLA_RTC_SMEM(RK, RV) \
    if (r_k == RK && r_v == RV) \
        return (int)(rope ? rlayout<RK, RV, true>(lp, B).total : rlayout<RK, RV, false>(lp, B).total) + 1024;
    LLA_RTC_SMEM(16, 32)
    LLA_RTC_SMEM(16, 16)
    LLA_RTC_SMEM(32, 32)
#undef LLA_RTC_SMEM
    return -1;
}

// Registers per thread the kernel instantiation launches with (0 when unknown).
static int rtc_launch_regs(int r_k, int r_v, bool rope)
{
    cudaFuncAttributes fa;
    cudaError_t e = cudaErrorInvalidValue;
#define LLA_RTC_REGS(RK, RV) \
    if (r_k == RK && r_v == RV) \
        e = rope ? cudaFuncGetAttributes(&fa, decode_recon_tc_kernel<RK, RV, true>) \
                 : cudaFuncGetAttributes(&fa, decode_recon_tc_kernel<RK, RV, false>);
    LLA_RTC_REGS(16, 32)
    LLA_RTC_REGS(16, 16)
    LLA_RTC_REGS(32, 32)
#undef LLA_RTC_REGS
    return e == cudaSuccess ? fa.numRegs : 0;
}

bool decode_recon_tc_supported(int dtype, int r_k, int r_v, int d, int fold, int B, bool rope)
{
    if (dtype != LLA_BF16 || d != kD || fold != LLA_PER_HEAD || tensor_map_encoder() == nullptr)
        return false;
    const int smem = decode_recon_tc_smem_bytes(r_k, r_v, rope, kMaxLoops, B);
    if (smem <= 0 || smem > 227 * 1024)
        return false;
    // setmaxnreg redistributes the registers the CTA was launched with: the split must fit
    return rtc_launch_regs(r_k, r_v, rope) * kThreads >= kSplitRegs;
}

int decode_recon_tc_loops_per_pass() { return kMaxLoops; }

cudaError_t launch_decode_recon_tc(const DecodeArgs &a, cudaStream_t stream)
{
#define LLA_RTC_CASE(RK, RV) \
    if (a.r_k == RK && a.r_v == RV) \
        return a.q_pos != nullptr ? launch_rtc<RK, RV, true>(a, stream) : launch_rtc<RK, RV, false>(a, stream);
    LLA_RTC_CASE(16, 32)
    LLA_RTC_CASE(16, 16)
    LLA_RTC_CASE(32, 32)
#undef LLA_RTC_CASE
    return cudaErrorNotSupported;
}

} // namespace lla
