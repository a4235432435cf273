// encode_tc.cu -- LLA write path (Eq. 2) on tcgen05 tensor cores, bf16 in, fp32
// accumulation in tensor memory, one rounding to bf16 on the way out.
//
// "Looped Latent Attention: Cross-Loop KV Compression for Looped Transformers", Pith
// review page, "What carries the argument": the T per-loop vectors of a finished
// (token, layer, head, axis) are stacked and centred and projected to the latent
// c = (x - mu) W_down, here c = x W_down + b with b = -mu W_down (lla_codec_bias).
// Per (layer, stored head, axis) this is a dense GEMM [n_tok, W] x [W, r]:
//
//  * one CTA computes a 128-token x r tile (M = 128, N = r, K = W in 64-element slabs);
//  * A (tokens) and B (W_down^T rows) are loaded by TMA with 128-byte swizzle into a
//    multi-stage mbarrier ring; for per-head codecs a 5-D tensor map over
//    [layers][tokens][T][H][d] gathers head h's [T][d] row of every token directly;
//  * one thread issues tcgen05.mma (kind::f16, bf16 x bf16 -> fp32) into a tensor
//    memory accumulator of 128 lanes x r columns; tcgen05.commit frees ring stages;
//  * the 4 warps read the accumulator with tcgen05.ld (warp w owns lanes 32w..32w+31,
//    i.e. tokens), add the bias, round to bf16 and store each token's latent row to
//    its cache slot.
// Every wait is bounded; a timeout records LLA_ERR_DEVICE_TIMEOUT in the library's
// encode status word and the CTA winds down (tensor memory is always released).
#include <cstring>
#include <mutex>

#include "encode.cuh"
#include "tmap.cuh"

namespace lla {

__device__ int32_t g_encode_status; // sticky status of the encode kernels (per device)

namespace {

constexpr int kThreads = 128;
constexpr int kBlockM = 128;
constexpr int kSlabK = 64; // bf16 elements per K slab = 128 bytes (one swizzle row)

// ---- tcgen05 / TMA helpers ---------------------------------------------------------------
__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap *map, int c0, int c1, int c2,
                                            int c3, int c4, uint32_t bar)
{
    asm volatile("cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int c0, int c1, int c2,
                                            uint32_t bar)
{
    asm volatile("cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// K-major operand tile with 128-byte swizzle: rows of 128 B, 8-row atoms of 1024 B.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr)
{
    uint64_t desc = 0;
    desc |= (uint64_t)((addr >> 4) & 0x3FFF);      // start address
    desc |= (uint64_t)1 << 16;                      // leading byte offset (16 B; unused for SW128 K-major)
    desc |= (uint64_t)(1024 >> 4) << 32;            // stride byte offset: 8 rows x 128 B
    desc |= (uint64_t)1 << 46;                      // descriptor version (sm_100)
    desc |= (uint64_t)2 << 61;                      // layout: SWIZZLE_128B
    return desc;
}

// Instruction descriptor: kind::f16, A = B = bf16 (K-major), D = fp32, M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int n)
{
    return (1u << 4)            // D format: f32
           | (1u << 7)          // A format: bf16
           | (1u << 10)         // B format: bf16
           | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kBlockM >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tc_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
                 "%12, %13, %14, %15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
                   "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

struct EncTcAxis {
    const float *bias;     // [L][H'][N]
    void *plane;           // [L][H'][slots][N]
};

struct EncTcArgs {
    EncTcAxis ax[2];       // K, V
    const int64_t *slot_idx;
    int64_t n_tok, slots;
    int32_t layer0, Hs, nk, d_slabs, fold, axis0;
    int32_t ksplit;        // CTAs of a cluster sharing one tile's K slabs (1: no split)
};

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float4 ld_peer_f4(uint32_t local_addr, uint32_t rank)
{
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(remote)
                 : "memory");
    return v;
}

// Ring depth: a shallow ring (~110 KB) leaves room for two CTAs per SM on large grids;
// a grid smaller than the GPU gets every K slab in flight at once (<= 8 stages).
template <int N, bool DEEP> struct EncCfg {
    static constexpr int A_BYTES = kBlockM * 128;
    static constexpr int B_BYTES = N * 128;
    static constexpr int STAGE = (A_BYTES + B_BYTES + 1023) & ~1023;
    static constexpr int BUDGET = DEEP ? 200 * 1024 : 110 * 1024;
    static constexpr int FIT = BUDGET / STAGE;
    static constexpr int CAP = DEEP ? 8 : 4;
    static constexpr int STAGES = FIT >= CAP ? CAP : (FIT >= 2 ? FIT : 2);
    static constexpr int TMEM_COLS = N <= 32 ? 32 : (N <= 64 ? 64 : (N <= 128 ? 128 : 256));
    static constexpr int BAR_OFF = STAGES * STAGE;         // full[S], empty[S], acc
    static constexpr int HOLD_OFF = BAR_OFF + (2 * STAGES + 1) * 8;
    static constexpr int BIAS_OFF = (HOLD_OFF + 16 + 15) & ~15;
    static constexpr int SMEM = BIAS_OFF + N * 4 + 1024;   // + alignment slack
    static_assert(N % 16 == 0 && N >= 16 && N <= 256, "tcgen05 N for M = 128");
};

// One 128-token x N tile of one (layer, stored head, axis).  With a.ksplit > 1 the CTAs of
// a cluster each take a contiguous share of the K slabs; their fp32 partial tiles meet in
// shared memory (the idle ring) and every CTA reduces a share of the rows across the
// cluster (distributed shared memory) before the bias and the bf16 store.
template <int N, bool DEEP>
__device__ __forceinline__ void encode_tile(uint8_t *smem, const CUtensorMap *map_a, const CUtensorMap *map_b,
                                            const EncTcArgs &a, const EncTcAxis &ax, int m0, int hs, int li)
{
    using C = EncCfg<N, DEEP>;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t full0 = sbase + C::BAR_OFF, empty0 = full0 + 8 * C::STAGES, accb = empty0 + 8 * C::STAGES;
    uint32_t *hold = reinterpret_cast<uint32_t *>(smem + C::HOLD_OFF);
    float *bias_s = reinterpret_cast<float *>(smem + C::BIAS_OFF);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int l = a.layer0 + li;

    // destination slot of this thread's token (accumulator lane), fetched up front
    const int64_t tok = (int64_t)m0 + warp * 32 + lane;
    int64_t slot = -1;
    if (tok < a.n_tok) {
        slot = a.slot_idx[tok];
        if (slot < 0 || slot >= a.slots)
            slot = -1;
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        mbar_init(accb, 1);
        hold[1] = 0; // error flag
        fence_barrier_init();
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(hold)),
                     "r"(C::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = hold[0];
    const int krank = a.ksplit > 1 ? (int)cluster_ctarank() : 0;
    const int kper = (a.nk + a.ksplit - 1) / a.ksplit;
    const int kb0 = krank * kper, nkl = min(a.nk, kb0 + kper) - kb0; // this CTA's K slabs

    if (warp == 0 && lane == 0) {
        // ---- TMA producer
        for (int kl = 0; kl < nkl; ++kl) {
            const int kb = kb0 + kl, s = kl % C::STAGES;
            if (kl >= C::STAGES && !mbar_wait_bounded(empty0 + 8 * s, ((kl / C::STAGES) - 1) & 1)) {
                hold[1] = 1;
                break;
            }
            const uint32_t dst = sbase + s * C::STAGE;
            mbar_arrive_expect_tx(full0 + 8 * s, C::A_BYTES + C::B_BYTES);
            if (a.fold)
                tma_load_3d(dst, map_a, kb * kSlabK, m0, li, full0 + 8 * s);
            else
                tma_load_5d(dst, map_a, (kb % a.d_slabs) * kSlabK, hs, kb / a.d_slabs, m0, li, full0 + 8 * s);
            tma_load_3d(dst + C::A_BYTES, map_b, kb * kSlabK, 0, l * a.Hs + hs, full0 + 8 * s);
        }
    } else if (warp == 1 && lane == 0) {
        // ---- MMA issuer
        constexpr uint32_t idesc = idesc_bf16_f32(N);
        bool ok = true;
        for (int kl = 0; kl < nkl; ++kl) {
            const int s = kl % C::STAGES;
            if (!mbar_wait_bounded(full0 + 8 * s, (kl / C::STAGES) & 1)) {
                hold[1] = 1;
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t a_addr = sbase + s * C::STAGE, b_addr = a_addr + C::A_BYTES;
#pragma unroll
            for (int k = 0; k < kSlabK / 16; ++k)
                tc_mma(tmem, smem_desc_sw128(a_addr + 32 * k), smem_desc_sw128(b_addr + 32 * k), idesc,
                       (kl | k) != 0);
            tc_commit(empty0 + 8 * s); // frees the stage once these MMAs have read it
        }
        if (ok)
            tc_commit(accb); // accumulator complete
        else
            mbar_arrive(accb);
    } else if (warp >= 2) {
        // the bias row, while the tiles stream in
        for (int j = threadIdx.x - 64; j < N; j += kThreads - 64)
            bias_s[j] = ax.bias[((int64_t)l * a.Hs + hs) * N + j];
    }
    __syncwarp();
    __syncthreads(); // bias staged; roles done issuing

    // ---- epilogue: all 4 warps, warp w owns accumulator lanes (tokens) 32w .. 32w+31
    const bool acc_ok = mbar_wait_bounded(accb, 0);
    tc_fence_after();
    const bool good = acc_ok && !hold[1] && nkl > 0;
    if (!good && nkl > 0 && threadIdx.x == 0)
        report_status(&g_encode_status, LLA_ERR_DEVICE_TIMEOUT);
    if (a.ksplit > 1) {
        // ---- split K: partial rows into the (idle) ring, reduction across the cluster
        static_assert(!DEEP || C::STAGES * C::STAGE >= kBlockM * N * 4, "ring holds the fp32 partial tile");
        float *red = reinterpret_cast<float *>(smem); // [128][N]
        const int row = warp * 32 + lane;
#pragma unroll 1
        for (int c = 0; c < N / 16; ++c) {
            uint32_t r[16];
            tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + c * 16, r);
#pragma unroll
            for (int e = 0; e < 16; e += 4)
                *reinterpret_cast<float4 *>(red + row * N + c * 16 + e) =
                    good ? make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]), __uint_as_float(r[e + 2]),
                                       __uint_as_float(r[e + 3]))
                         : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        cluster_sync_all(); // every partial tile is written
        const int rows = (int)min((int64_t)kBlockM, a.n_tok - m0);
        const int per = (rows + a.ksplit - 1) / a.ksplit, r0 = krank * per, r1 = min(rows, r0 + per);
        __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(ax.plane) + (((int64_t)l * a.Hs + hs) * a.slots) * N;
        const uint32_t red_addr = smem_u32(red);
        for (int it = threadIdx.x; it < (r1 - r0) * (N / 4); it += kThreads) {
            const int rr = r0 + it / (N / 4), c4 = 4 * (it % (N / 4));
            float4 acc = make_float4(bias_s[c4], bias_s[c4 + 1], bias_s[c4 + 2], bias_s[c4 + 3]);
            for (int p = 0; p < a.ksplit; ++p) {
                const float4 v = ld_peer_f4(red_addr + (uint32_t)(rr * N + c4) * 4u, (uint32_t)p);
                acc.x += v.x, acc.y += v.y, acc.z += v.z, acc.w += v.w;
            }
            int64_t sl = a.slot_idx[m0 + rr];
            if (sl >= 0 && sl < a.slots) {
                const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
                uint2 w;
                w.x = *reinterpret_cast<const uint32_t *>(&lo);
                w.y = *reinterpret_cast<const uint32_t *>(&hi);
                *reinterpret_cast<uint2 *>(dst + sl * N + c4) = w;
            }
        }
        cluster_sync_all(); // peers are done reading this CTA's partial tile
    } else if (good) {
        __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(ax.plane) + (((int64_t)l * a.Hs + hs) * a.slots) * N;
#pragma unroll 1
        for (int c = 0; c < N / 16; ++c) {
            uint32_t r[16];
            tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + c * 16, r);
            if (slot >= 0) {
                uint32_t packed[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float lo = __uint_as_float(r[2 * e]) + bias_s[c * 16 + 2 * e];
                    const float hi = __uint_as_float(r[2 * e + 1]) + bias_s[c * 16 + 2 * e + 1];
                    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
                    packed[e] = *reinterpret_cast<const uint32_t *>(&v);
                }
                uint4 *out = reinterpret_cast<uint4 *>(dst + slot * N + c * 16);
                out[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                out[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS)
                     : "memory");
}

// grid (token tiles, axes x stored heads, layers); blockIdx.y / Hs selects K (rank NK) or
// V (rank NV) counted from a.axis0, so one launch can cover both axes.
template <int NK, int NV, bool DEEP>
__global__ void __launch_bounds__(kThreads, 1)
    encode_tc_kernel(const __grid_constant__ CUtensorMap map_ak, const __grid_constant__ CUtensorMap map_bk,
                     const __grid_constant__ CUtensorMap map_av, const __grid_constant__ CUtensorMap map_bv,
                     const EncTcArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    // aligned by arithmetic on the shared array itself, so accesses stay shared-space loads
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int axis = a.axis0 + (int)blockIdx.y / a.Hs, hs = (int)blockIdx.y % a.Hs;
    const int m0 = (int)(blockIdx.x / a.ksplit) * kBlockM; // a cluster of ksplit CTAs per tile
    if (axis == 0)
        encode_tile<NK, DEEP>(smem, &map_ak, &map_bk, a, a.ax[0], m0, hs, blockIdx.z);
    else
        encode_tile<NV, DEEP>(smem, &map_av, &map_bv, a, a.ax[1], m0, hs, blockIdx.z);
}

// ---- host: tensor maps ------------------------------------------------------------------------
bool make_map(CUtensorMap *map, const void *base, int rank, const uint64_t *dims, const uint64_t *strides_bytes,
              const uint32_t *box)
{
    auto fn = tensor_map_encoder();
    if (fn == nullptr)
        return false;
    uint32_t estr[5] = {1, 1, 1, 1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims, strides_bytes,
                          box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool axis_maps(const EncodeArgs &e, int axis, int N, CUtensorMap *ma, CUtensorMap *mb)
{
    const void *x = axis ? e.x_v : e.x_k;
    const void *wd = axis ? e.W_down_v : e.W_down_k;
    const uint64_t el = 2;
    if (e.fold) {
        const uint64_t dims[3] = {(uint64_t)e.W, (uint64_t)e.n_tok, (uint64_t)e.n_layers};
        const uint64_t str[2] = {(uint64_t)e.W * el, (uint64_t)e.n_tok * e.W * el};
        const uint32_t box[3] = {kSlabK, kBlockM, 1};
        if (!make_map(ma, x, 3, dims, str, box))
            return false;
    } else {
        const uint64_t dims[5] = {(uint64_t)e.d, (uint64_t)e.H, (uint64_t)e.T, (uint64_t)e.n_tok,
                                  (uint64_t)e.n_layers};
        const uint64_t str[4] = {(uint64_t)e.d * el, (uint64_t)e.H * e.d * el, (uint64_t)e.T * e.H * e.d * el,
                                 (uint64_t)e.n_tok * e.T * e.H * e.d * el};
        const uint32_t box[5] = {kSlabK, 1, 1, kBlockM, 1};
        if (!make_map(ma, x, 5, dims, str, box))
            return false;
    }
    const int L_total = e.layer0 + e.n_layers; // rows of W_down needed: up to the last layer used
    const uint64_t dims[3] = {(uint64_t)e.W, (uint64_t)N, (uint64_t)L_total * e.Hs};
    const uint64_t str[2] = {(uint64_t)e.W * el, (uint64_t)N * e.W * el};
    const uint32_t box[3] = {kSlabK, (uint32_t)N, 1};
    return make_map(mb, wd, 3, dims, str, box);
}

// Launch axes [axis0, axis0 + n_axes) of one encode in one grid; ksplit > 1 runs every tile
// as a cluster of ksplit CTAs that share its K slabs (deep ring only).
template <int NK, int NV, bool DEEP>
cudaError_t launch_tc(const EncodeArgs &e, int axis0, int n_axes, cudaStream_t stream, int ksplit = 1)
{
    CUtensorMap mak, mbk, mav, mbv;
    std::memset(&mak, 0, sizeof(mak));
    std::memset(&mbk, 0, sizeof(mbk));
    std::memset(&mav, 0, sizeof(mav));
    std::memset(&mbv, 0, sizeof(mbv));
    if (axis0 == 0 && !axis_maps(e, 0, NK, &mak, &mbk))
        return cudaErrorInvalidValue;
    if (axis0 + n_axes > 1 && !axis_maps(e, 1, NV, &mav, &mbv))
        return cudaErrorInvalidValue;
    EncTcArgs a;
    a.ax[0].bias = e.bias_k;
    a.ax[0].plane = e.cache_k;
    a.ax[1].bias = e.bias_v;
    a.ax[1].plane = e.cache_v;
    a.slot_idx = e.slot_idx;
    a.n_tok = e.n_tok;
    a.slots = e.slots;
    a.layer0 = e.layer0;
    a.Hs = e.Hs;
    a.nk = e.W / kSlabK;
    a.d_slabs = e.d / kSlabK;
    a.fold = e.fold;
    a.axis0 = axis0;
    a.ksplit = DEEP ? ksplit : 1;
    auto kern = encode_tc_kernel<NK, NV, DEEP>;
    const int smem = EncCfg<NK, DEEP>::SMEM > EncCfg<NV, DEEP>::SMEM ? EncCfg<NK, DEEP>::SMEM
                                                                       : EncCfg<NV, DEEP>::SMEM;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess)
        return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((e.n_tok + kBlockM - 1) / kBlockM) * a.ksplit, n_axes * e.Hs, e.n_layers);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = a.ksplit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.ksplit > 1 ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, mak, mbk, mav, mbv, a);
}

template <bool DEEP>
cudaError_t launch_tc_single(const EncodeArgs &e, int axis, int r, cudaStream_t stream, int ks)
{
    switch (r) {
    case 16: return launch_tc<16, 16, DEEP>(e, axis, 1, stream, ks);
    case 32: return launch_tc<32, 32, DEEP>(e, axis, 1, stream, ks);
    case 48: return launch_tc<48, 48, DEEP>(e, axis, 1, stream, ks);
    case 64: return launch_tc<64, 64, DEEP>(e, axis, 1, stream, ks);
    case 96: return launch_tc<96, 96, DEEP>(e, axis, 1, stream, ks);
    case 128: return launch_tc<128, 128, DEEP>(e, axis, 1, stream, ks);
    case 160: return launch_tc<160, 160, DEEP>(e, axis, 1, stream, ks);
    case 192: return launch_tc<192, 192, DEEP>(e, axis, 1, stream, ks);
    case 256: return launch_tc<256, 256, DEEP>(e, axis, 1, stream, ks);
    default: return cudaErrorNotSupported;
    }
}

// Both axes in one grid for the rank pairs of the decode kernels; otherwise one grid per axis.
template <bool DEEP> cudaError_t launch_tc_pair(const EncodeArgs &e, cudaStream_t stream, int ks)
{
    const int rk = e.r_k, rv = e.r_v;
    if (rk == 16 && rv == 32) return launch_tc<16, 32, DEEP>(e, 0, 2, stream, ks);
    if (rk == 16 && rv == 16) return launch_tc<16, 16, DEEP>(e, 0, 2, stream, ks);
    if (rk == 32 && rv == 32) return launch_tc<32, 32, DEEP>(e, 0, 2, stream, ks);
    if (rk == 64 && rv == 128) return launch_tc<64, 128, DEEP>(e, 0, 2, stream, ks);
    if (rk == 96 && rv == 160) return launch_tc<96, 160, DEEP>(e, 0, 2, stream, ks);
    if (rk == 128 && rv == 128) return launch_tc<128, 128, DEEP>(e, 0, 2, stream, ks);
    cudaError_t err = launch_tc_single<DEEP>(e, 0, rk, stream, ks);
    if (err == cudaSuccess)
        err = launch_tc_single<DEEP>(e, 1, rv, stream, ks);
    return err;
}

bool tc_rank_ok(int r) { return r == 16 || r == 32 || r == 48 || r == 64 || r == 96 || r == 128 || r == 160 || r == 192 || r == 256; }

int device_sms()
{
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 148;
    return n;
}

} // namespace

bool encode_tc_supported(const EncodeArgs &e)
{
    return tc_rank_ok(e.r_k) && tc_rank_ok(e.r_v) && e.W % kSlabK == 0 && (e.fold || e.d % kSlabK == 0) &&
           tensor_map_encoder() != nullptr;
}

cudaError_t launch_encode_tc(const EncodeArgs &e, cudaStream_t stream)
{
    // A grid that does not fill the GPU twice over gets the deep ring (latency-bound).  One
    // that leaves most SMs idle, with more K slabs than one ring pass (8), also splits each
    // tile's slabs over a cluster of up to 8 CTAs, so every CTA's slabs are in flight at once.
    const int64_t ctas = ((e.n_tok + kBlockM - 1) / kBlockM) * (int64_t)e.Hs * e.n_layers * 2;
    const int sms = device_sms();
    if (ctas >= 2 * sms)
        return launch_tc_pair<false>(e, stream, 1);
    const int nk = e.W / kSlabK, passes = (nk + 7) / 8;
    int ks = ctas < sms ? (int)(sms / ctas < 8 ? sms / ctas : 8) : 1;
    ks = ks < passes ? ks : passes;
    return launch_tc_pair<true>(e, stream, ks < 1 ? 1 : ks);
}

namespace {
std::mutex g_status_mutex;
void *g_status_addr[64] = {};
} // namespace

// Device address of g_encode_status on the current device (looked up once per device).
void *encode_status_address()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return nullptr;
    std::lock_guard<std::mutex> lock(g_status_mutex);
    if (g_status_addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_encode_status) != cudaSuccess)
            return nullptr;
        g_status_addr[dev] = p;
    }
    return g_status_addr[dev];
}

} // namespace lla
