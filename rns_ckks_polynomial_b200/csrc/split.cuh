// Exact sums of 60-bit products in three 64-bit partial sums ("split form"), for primes
// q = 2^60 - delta with delta < 2^32 and operands below 2^60 (every residue).
//
// With a = a1 2^30 + a0 and b = b1 2^30 + b0 (halves below 2^30),
//     a b = a1 b1 2^60 + (a1 b0 + a0 b1) 2^30 + a0 b0,
// each partial product below 2^60, so one 32 x 32 -> 64-bit multiply-add adds it into one of the
// sums s2, s1, s0 without any carry handling.  Every kSplitFold products per sum, split_fold brings
// the sums back under their bounds: s1 moves into s2 and s0, s0's bits from 2^60 up into s2, and
// s2's bits from 2^60 up (its 2^120 part) come back as (s2 >> 60) delta, since 2^60 = delta (mod q).
// Bounds: after a fold s0 < 2^60, s1 = 0 and s2 < 2^60 + 2^36; a block of kSplitFold = 8 products
// adds below 8 2^60 to s0 and s2 and below 16 2^60 to s1, all below 2^64.  The value is then
// s2 2^60 + s0 (s0 < 2^60), a 128-bit number with words (s2 >> 4, s2 << 60 | s0).
#pragma once
#include "common.cuh"

namespace ckks {

constexpr int kSplitFold = 8;

__device__ __forceinline__ u32 lo30(u64 a) { return (u32)a & 0x3FFFFFFFu; }
__device__ __forceinline__ u32 hi30(u64 a) { return __funnelshift_r((u32)a, (u32)(a >> 32), 30); }

__device__ __forceinline__ void madw(u64 &acc, u32 a, u32 b)
{
    asm("mad.wide.u32 %0, %1, %2, %0;" : "+l"(acc) : "r"(a), "r"(b));
}

// (s2, s1, s0) += a b for a = (a1, a0), b = (b1, b0) in 30-bit halves.
__device__ __forceinline__ void split_mac(u64 &s0, u64 &s1, u64 &s2, u32 a0, u32 a1, u32 b0, u32 b1)
{
    madw(s2, a1, b1);
    madw(s1, a1, b0);
    madw(s1, a0, b1);
    madw(s0, a0, b0);
}

__device__ __forceinline__ void split_fold(u64 &s0, u64 &s1, u64 &s2, u32 delta)
{
    constexpr u64 kM60 = (1ull << 60) - 1;
    s2 += s1 >> 30;
    s0 += (s1 & 0x3FFFFFFFull) << 30;
    s1 = 0;
    s2 += s0 >> 60;
    s0 &= kM60;
    u64 f = s2 & kM60;
    madw(f, (u32)(s2 >> 60), delta);
    s2 = f;
}

// The folded sums reduced into [0, q).
__device__ __forceinline__ u64 split_reduce(u64 s0, u64 s2, const PrimeConst &c)
{
    return reduce128(s2 >> 4, (s2 << 60) | s0, c);
}

}  // namespace ckks
