// mma_common.cuh -- pieces shared by the warp-level tensor-core decode kernels:
// swizzled latent tile layout, ldmatrix / mma.sync wrappers, bf16 hi/lo splits,
// 2-D TMA loads and the tensor maps of a latent plane.
#pragma once

#include "decode_sched.cuh"
#include "tmap.cuh"

namespace lla {
namespace mma {

constexpr int kBox = 32; // rows per TMA box
constexpr float kRescaleThreshold = 8.0f;

__host__ __device__ constexpr int align1024(int x) { return (x + 1023) & ~1023; }

// Shared-memory layout of a tile of TILE rows of R bf16 latents.  The columns are cut
// into NBLK blocks of 64 (128-byte rows, 128B swizzle) and a tail of TAIL = R % 64
// columns (32- or 64-byte rows with the matching swizzle); each block is a separate
// TMA box, so every ldmatrix row group touches 8 distinct bank groups.
template <int R, int TILE> struct TileLayout {
    static constexpr int NBLK = R / 64;
    static constexpr int TAIL = R % 64;
    static constexpr int TB = TAIL * 2; // tail row bytes
    static constexpr int BYTES = TILE * R * 2;
    static_assert(TAIL == 0 || TAIL == 16 || TAIL == 32, "rank must be 64k, 64k + 16 or 64k + 32");
    // byte offset of (row, 16-byte chunk c) in the tile
    __device__ static __forceinline__ uint32_t off(int row, int c)
    {
        if (c < 8 * NBLK)
            return (uint32_t)((c >> 3) * TILE * 128 + row * 128 + 16 * ((c & 7) ^ (row & 7)));
        const int cc = c - 8 * NBLK;
        return (uint32_t)(NBLK * TILE * 128 + row * TB + 16 * (cc ^ ((row * TB >> 7) & (TB / 16 - 1))));
    }
    // zero rows [r0, r1) of the tile (all column blocks), strided over `n` threads (a warp's
    // lanes by default; n = 1: one thread does it all)
    __device__ static __forceinline__ void zero_rows(uint8_t *tile, int r0, int r1, int lane, int n = 32)
    {
        for (int blk = 0; blk < NBLK; ++blk) {
            uint4 *z = reinterpret_cast<uint4 *>(tile + blk * TILE * 128 + r0 * 128);
            for (int e = lane; e < (r1 - r0) * 8; e += n)
                z[e] = make_uint4(0u, 0u, 0u, 0u);
        }
        if (TAIL) {
            uint4 *z = reinterpret_cast<uint4 *>(tile + NBLK * TILE * 128 + r0 * TB);
            for (int e = lane; e < (r1 - r0) * TB / 16; e += n)
                z[e] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                 "{%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

// x = hi + lo with hi and lo exactly representable in bf16: hi keeps the top 16 bits of x
// (truncation), lo = x - hi is exact in fp32 and is truncated to bf16 in turn, so hi + lo
// carries about 15 mantissa bits of x.  Packs (x0, x1) into two bf16x2 words using only
// integer/FMA-pipe instructions (byte permutes, masks, subtractions).
__device__ __forceinline__ uint32_t pack_top16(float a, float b)
{
    return __byte_perm(__float_as_uint(a), __float_as_uint(b), 0x7632);
}

// Round-to-nearest split (hi = bf16(x), lo = bf16(x - hi)): about 17 bits, for q_tilde,
// whose error scales with the logits.  Used once per unit segment, so cost does not matter.
__device__ __forceinline__ void split_bf16_rn(float x0, float x1, uint32_t &hi, uint32_t &lo)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    const float2 hf = __bfloat1622float2(h);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = pack_bf16(x0 - hf.x, x1 - hf.y);
}

// Truncating split for the softmax weights p in the hot loop (p <= 2^8, relative error
// below 2^-14 is far inside the tolerance).
__device__ __forceinline__ void split_bf16(float x0, float x1, uint32_t &hi, uint32_t &lo)
{
    hi = pack_top16(x0, x1);
    const float h0 = __uint_as_float(__float_as_uint(x0) & 0xffff0000u);
    const float h1 = __uint_as_float(__float_as_uint(x1) & 0xffff0000u);
    lo = pack_top16(x0 - h0, x1 - h1);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
                 : "memory");
}


bool plane_maps(CUtensorMap *main, CUtensorMap *tail, const void *base, int r, int64_t rows);

} // namespace mma
} // namespace lla
