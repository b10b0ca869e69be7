// Device helpers for reading packed code records two coordinates at a time
// (the layout is the one documented in tq.h): byte offsets into tables with one
// entry per *pair field* (the 2b bits of coordinates 2m, 2m + 1 of a
// 32-coordinate block), stored as 8 interleaved copies of 16-byte entries
// (entry f, copy c at byte f * 128 + c * 16) so that a quarter-warp's 16-byte
// loads never share a bank.
#pragma once

#include <stdint.h>

namespace tq {

// (w >> S) for S >= 0, (w << -S) for S < 0.
template <int S>
__device__ __forceinline__ uint32_t shr(uint32_t w) {
    if constexpr (S >= 0) return w >> S;
    else return w << (-S);
}

// Byte offset (pair field * 128) of the table entry of coordinates 2M, 2M + 1
// (M < 16) of the block whose B words are w[0..B).  Pair fields: b = 4, the
// byte of two [idx|z] nibbles; b = 2, two [idx|z] 2-bit fields; b = 3, the two
// 2-bit cells then the two sign bits (bits 4, 5); b = 1, the two sign bits.
template <int B, int M>
__device__ __forceinline__ uint32_t pair_offset_m(const uint32_t (&w)[4]) {
    if constexpr (B == 4) {
        return shr<8 * (M & 3) - 7>(w[M >> 2]) & (0xFFu << 7);
    } else if constexpr (B == 2) {
        return shr<4 * (M & 7) - 7>(w[M >> 3]) & (0xFu << 7);
    } else if constexpr (B == 3) {
        return (shr<4 * (M & 7) - 7>(w[M >> 3]) & (0xFu << 7)) |
               (shr<2 * M - 11>(w[2]) & (0x3u << 11));
    } else {
        return shr<2 * M - 7>(w[0]) & (0x3u << 7);
    }
}

template <int B>
__device__ __forceinline__ uint32_t pair_offset(const uint32_t (&w)[4], int m) {
    switch (m) {
#define TQ_PO(M) case M: return pair_offset_m<B, M>(w);
        TQ_PO(0) TQ_PO(1) TQ_PO(2) TQ_PO(3) TQ_PO(4) TQ_PO(5) TQ_PO(6) TQ_PO(7)
        TQ_PO(8) TQ_PO(9) TQ_PO(10) TQ_PO(11) TQ_PO(12) TQ_PO(13) TQ_PO(14) TQ_PO(15)
#undef TQ_PO
    }
    return 0u;
}

// A pair field split into the single-coordinate fields of its low (2m) and
// high (2m + 1) coordinate, each in the per-coordinate field encoding
// (b = 4: [idx(3)|z]; b = 3: idx(2) | z << 2; b = 2: [idx|z]; b = 1: z).
template <int B>
__device__ __forceinline__ void pair_split(uint32_t f, uint32_t& lo, uint32_t& hi) {
    if (B == 4) {
        lo = f & 15u;
        hi = f >> 4;
    } else if (B == 3) {
        lo = (f & 3u) | (((f >> 4) & 1u) << 2);
        hi = ((f >> 2) & 3u) | (((f >> 5) & 1u) << 2);
    } else if (B == 2) {
        lo = f & 3u;
        hi = f >> 2;
    } else {
        lo = f & 1u;
        hi = f >> 1;
    }
}

// Number of pair fields.
template <int B>
constexpr int pair_fields() { return 1 << (2 * B); }

}  // namespace tq
