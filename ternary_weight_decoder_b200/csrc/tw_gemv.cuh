// tw_gemv.cuh — the register-level ternary GEMV step shared by the decode
// sweep (tw_decode.cu) and the fused decoder-layer chain (tw_chain.cu):
// one 16 x 128 tile of 2-bit codes against up to NT x 8 int8 token columns
// on m16n8k32 integer MMAs.
//
// A tile's 16-byte lane slot holds 4 words: rows g and g + 8 at k 16t.. and
// 64 + 16t..; (word & (3 << 2s per byte)) are the codes + 1 of k = 16t + 4s
// + b (resp. 64 + 16t + 4s + b), times 4^s, as unsigned bytes.  MMA s pairs
// them with the token bytes at the same k, one accumulator per s; at the
// end acc = sum_s (acc_s >> 2s) - sum(q) (exact: sum (c + 1) q - sum q).
#pragma once

#include <cstdint>

#include "tw_device.cuh"
#include "tw_internal.h"

namespace tw {

// D(16x8, s32) += A(16x32, u8, row) * B(32x8, s8, col).
__device__ __forceinline__ void mma_u8s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t comp(const uint4 &v, int s)
{
    return s == 0 ? v.x : s == 1 ? v.y : s == 2 ? v.z : v.w;
}

// One 16x128 tile.  Lane slot a holds 4 words: rows g and g+8 at k 16t.. and
// 64+16t..; (word & (3 << 2s per byte)) are the codes + 1 of k = 16t+4s+b
// (resp. 64+16t+4s+b), times 4^s.  MMA s pairs them with the token bytes at
// the same k: component s of the 16-byte loads at xrow + koff (+ 64).
template <int NT>
__device__ __forceinline__ void tile_mma(int (&acc)[NT][4][4], const uint4 &a,
                                         const uint32_t (&xrow)[NT], uint32_t koff)
{
    uint4 b0[NT], b1[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        b0[nt] = lds128(xrow[nt] + koff);
        b1[nt] = lds128(xrow[nt] + koff + 64);
    }
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const uint32_t mk = 0x03030303u << (2 * s);
        const uint32_t a0 = a.x & mk, a1 = a.y & mk, a2 = a.z & mk, a3 = a.w & mk;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
            mma_u8s8(acc[nt][s], a0, a1, a2, a3, comp(b0[nt], s), comp(b1[nt], s));
    }
}

// The n tiles of one ring chunk (lane slots at ra + 512 i, token k offset
// kbase + 128 i).  A full chunk is one straight-line block, so the loads of
// later tiles can be scheduled ahead of the MMAs of earlier ones; the last,
// shorter chunk of a row block runs as 4 + 2 + 1 tiles without a branch per
// tile.  Both measured on B200 against a loop that tests every tile
// (M = 1: 74.9 -> 70.5 us per sweep).
template <int NT, int CT>
__device__ __forceinline__ void chunk_mma(int (&acc)[NT][4][4], uint32_t ra,
                                          const uint32_t (&xrow)[NT], uint32_t kbase, int n)
{
    static_assert(CT <= 8, "a partial chunk is at most 4 + 2 + 1 tiles");
    if (n == CT) {
#pragma unroll
        for (int i = 0; i < CT; ++i)
            tile_mma<NT>(acc, lds128(ra + i * kTileBytes), xrow, kbase + i * kTileK);
        return;
    }
    if (n & 4) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            tile_mma<NT>(acc, lds128(ra + i * kTileBytes), xrow, kbase + i * kTileK);
        ra += 4 * kTileBytes;
        kbase += 4 * kTileK;
    }
    if (n & 2) {
#pragma unroll
        for (int i = 0; i < 2; ++i)
            tile_mma<NT>(acc, lds128(ra + i * kTileBytes), xrow, kbase + i * kTileK);
        ra += 2 * kTileBytes;
        kbase += 2 * kTileK;
    }
    if (n & 1)
        tile_mma<NT>(acc, lds128(ra), xrow, kbase);
}

}  // namespace tw
