// Exact sums of 60-bit products in three 64-bit partial sums ("split form"), for primes
// q = 2^60 - delta with delta < 2^32 and operands below 2^60 (every residue).
//
// With a = a1 2^30 + a0 and b = b1 2^30 + b0 (halves below 2^30),
//     a b = a1 b1 2^60 + (a1 b0 + a0 b1) 2^30 + a0 b0,
// and the middle term is taken the Karatsuba way, (a0 + a1)(b0 + b1) - a0 b0 - a1 b1, so a product
// costs three 32 x 32 -> 64-bit multiply-adds: a0 b0 into s0, a1 b1 into s2 and (a0 + a1)(b0 + b1)
// (below 2^62) into s1.  The subtractions wait for split_fold, which runs every kSplitFold products
// per sum: at the start of a block s1 is set to s0 + s2, so at its end s1 - s0 - s2 (mod 2^64) is
// exactly the block's middle sum, which is below 8 (2^61 - 2^32 + 2) < 2^64 however s1 wrapped.
// The fold moves that middle sum into s2 and s0, s0's bits from 2^60 up into s2, and brings s2's
// bits from 2^60 up (its 2^120 part) back as (s2 >> 60) delta, since 2^60 = delta (mod q).
// Bounds: after a fold s0 < 2^60 and s2 < 2^60 + 2^36; a block of 8 products adds below 8 2^60 to
// each, so both stay below 2^64.  The value is then s2 2^60 + s0 (s0 < 2^60), a 128-bit number with
// words (s2 >> 4, s2 << 60 | s0).
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

// Operand halves and their sum: (x0, x1, x0 + x1).
struct Split30 {
    u32 lo, hi, sum;
};

__device__ __forceinline__ Split30 split30(u64 a)
{
    const u32 lo = lo30(a), hi = hi30(a);
    return {lo, hi, lo + hi};
}

// (s2, s1, s0) += a b, the middle sum taking (a0 + a1)(b0 + b1).
__device__ __forceinline__ void split_mac(u64 &s0, u64 &s1, u64 &s2, const Split30 &a, const Split30 &b)
{
    madw(s2, a.hi, b.hi);
    madw(s1, a.sum, b.sum);
    madw(s0, a.lo, b.lo);
}

__device__ __forceinline__ void split_fold(u64 &s0, u64 &s1, u64 &s2, u32 delta)
{
    constexpr u64 kM60 = (1ull << 60) - 1;
    const u64 mid = s1 - s0 - s2;  // the block's sum of a0 b1 + a1 b0
    s2 += mid >> 30;
    s0 += (mid & 0x3FFFFFFFull) << 30;
    s2 += s0 >> 60;
    s0 &= kM60;
    u64 f = s2 & kM60;
    madw(f, (u32)(s2 >> 60), delta);
    s2 = f;
    s1 = s0 + s2;
}

// The folded sums reduced into [0, q).
__device__ __forceinline__ u64 split_reduce(u64 s0, u64 s2, const PrimeConst &c)
{
    return reduce128(s2 >> 4, (s2 << 60) | s0, c);
}

}  // namespace ckks
