// decode_sched.cuh -- work split of the persistent decode kernels.
//
// The concatenated token stream of all (sequence, head) units -- unit u = b*H + h holds
// ctx_lens[b] tokens -- is cut into equal shares of `chunk` tokens, one per CTA of a
// grid sized to the resident CTAs, so ragged context lengths leave no tail wave.  A
// share may cross unit boundaries; every unit segment it covers is streamed as tiles
// and yields one partial record.  Unit u is covered by shares c_first .. c_last and the
// share of CTA c writes record slot j = c - c_first of that unit.
#pragma once

#include "decode.cuh"

namespace lla {

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

// Walks the token share [pos, end) of one CTA (shares of `chunk` tokens), unit segment by
// unit segment, tile by tile; each segment's record slot j = share - first share of the
// unit and the unit's record count n_u come from the share geometry.
template <int TILE> struct ShareWalk {
    int64_t pos, end, chunk, seq0;
    int32_t b = 0, h, n, seg_end, u, j, n_u;
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
            // the sequence holding pos: the previous one or its successor, else bisect
            const int64_t HH = H;
            if (!(HH * pref[b] <= pos && pos < HH * pref[b + 1])) {
                if (b + 2 <= B && HH * pref[b + 1] <= pos && pos < HH * pref[b + 2])
                    ++b;
                else
                    b = find_seq(pref, B, H, pos);
            }
            const int len = (int)(pref[b + 1] - pref[b]);
            seq0 = starts[b];
            const int64_t off = pos - HH * pref[b];
            if (off < 0x7fffffff) {
                h = (int)off / len;
                n = (int)off - h * len;
            } else {
                h = (int)(off / len);
                n = (int)(off - (int64_t)h * len);
            }
            const int64_t take = min((int64_t)(len - n), end - pos);
            seg_end = n + (int)take;
            pos += take;
            u = b * H + h;
            const int64_t U = HH * pref[b] + (int64_t)h * len; // unit start in the stream
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

// Exclusive prefix of ctx_lens[0..B) into pref[0..B] (pref[B] = total), by a whole CTA
// of NT threads: contiguous slices per thread, a warp scan, a cross-warp offset.
// `scratch` holds NT/32 int64.  Ends with __syncthreads().
template <int NT>
__device__ __forceinline__ void block_length_prefix(const int32_t *lens, int B, int64_t *pref, int64_t *scratch)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (B + NT - 1) / NT;
    const int b0 = min(B, tid * per), b1 = min(B, b0 + per);
    int64_t local = 0;
    for (int b = b0; b < b1; ++b)
        local += lens[b];
    int64_t x = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int64_t y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off)
            x += y;
    }
    if (lane == 31)
        scratch[warp] = x;
    __syncthreads();
    int64_t run = x - local;
    for (int w = 0; w < warp; ++w)
        run += scratch[w];
    for (int b = b0; b < b1; ++b) {
        pref[b] = run;
        run += lens[b];
    }
    if (tid == NT - 1)
        pref[B] = run;
    __syncthreads();
}

// This CTA's share of the token stream: [s0, s1) with share size `chunk`.
__device__ __forceinline__ void cta_share(const int64_t *pref, int B, int H, int chunk_min, int64_t &s0, int64_t &s1,
                                          int64_t &chunk)
{
    const int64_t total = (int64_t)H * pref[B];
    chunk = (total + gridDim.x - 1) / gridDim.x;
    if (chunk < chunk_min)
        chunk = chunk_min;
    s0 = (int64_t)blockIdx.x * chunk;
    s1 = min(total, s0 + chunk);
}

} // namespace lla
