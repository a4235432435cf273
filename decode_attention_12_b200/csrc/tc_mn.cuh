// tc_mn.cuh -- tcgen05 helpers for operands read MN-major (the M or N index contiguous in
// shared memory) and for tensor-memory stores, on top of tc_common.cuh.
#pragma once

#include "tc_common.cuh"

namespace lla {
namespace tc {

// Descriptor of an operand tile with explicit byte offsets: `lbo` and `sbo` fill the
// leading- and stride-dimension fields (bits 16-29 and 32-45, in 16-byte units) and `sw`
// the layout code.  For an MN-major operand with a swizzled layout, an atom holds 8 rows
// of K, each row one swizzle width (32/64/128 bytes) of consecutive MN values; `lbo` is the
// distance between atoms along MN and `sbo` the distance between 8-row groups along K.
__host__ __device__ constexpr uint64_t smem_desc_explicit(uint32_t addr, uint32_t lbo, uint32_t sbo, int sw)
{
    return (uint64_t)((addr >> 4) & 0x3FFFu) | (uint64_t)((lbo >> 4) & 0x3FFFu) << 16 |
           (uint64_t)((sbo >> 4) & 0x3FFFu) << 32 | (uint64_t)1 << 46 | (uint64_t)sw << 61;
}

// As idesc, with A and/or B read MN-major (bits 15 and 16: the operand is transposed).
__host__ __device__ constexpr uint32_t idesc_major(int fmt, int m, int n, bool a_mn, bool b_mn)
{
    return idesc(fmt, m, n) | (a_mn ? 1u << 15 : 0u) | (b_mn ? 1u << 16 : 0u);
}

// Tensor-memory stores: thread i of the warp writes lane (warp's lane quarter) + i, 16
// consecutive 32-bit columns from `taddr` on.  Visible to later tensor-core work after
// wait_st() and a fence_before / thread sync / fence_after sequence.
__device__ __forceinline__ void st_x16(uint32_t taddr, const uint32_t (&r)[16])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
                 "%12, %13, %14, %15, %16};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
                 "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
                 : "memory");
}

__device__ __forceinline__ void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

} // namespace tc
} // namespace lla
