// RNS basis conversion on the int8 tensor cores (tcgen05.mma, kind::i8).
//
// The conversion out[t][c] = (sum_s M[t][s] y[s][c]) mod q_t is a dense integer contraction:
// targets x sources times sources x coefficients, with 60-bit operands.  It is computed exactly by
// splitting both operands into bytes: M = sum_u M_u 2^(8u), y = sum_v y_v 2^(8v), u, v < 8, so that
//     sum_s M y = sum_{d=0}^{14} 2^(8d) P_d,   P_d = sum_{u+v=d} sum_s M_u[t][s] y_v[s][c].
// Each P_d is an unsigned 8-bit matrix product with at most 8 * 64 * 255^2 < 2^25 per entry, so it
// fits an int32 tensor-memory accumulator.
//
// One CTA (one per SM, owning all 512 TMEM columns) converts one block of 128 targets (the MMA's M)
// for a run of coefficient tiles of 32 (the MMA's N):
//  - the block's M byte planes (64 KiB) stay in shared memory for the whole run;
//  - the 15 accumulators P_d take TMEM columns 32 d .. 32 d + 31, in two groups: X = P_0..P_7
//    (36 plane pairs) and Y = P_8..P_14 (28 pairs);
//  - the y bytes of a tile are staged in one of two shared-memory buffers, two tiles ahead.
// With both operands in shared memory a tcgen05.mma reads its whole A tile (128 x 32 bytes) and
// N x 32 bytes of B per K-step, at about 128 bytes per SM cycle: about 40 cycles at N = 32 against
// 16 cycles of arithmetic, so the tile is as wide as the 15 accumulators allow (15 x 32 of the 512
// columns), and four warps issue.
// Warp roles: 16 epilogue warps and 4 MMA warps, synchronised by mbarriers only.
//  - MMA warps (one elected lane each) own disjoint sets of accumulators: two split group X (P_d sets
//    {0, 1, 6, 7} and {2, 3, 4, 5}, 18 plane pairs each), two split group Y ({8, 11, 12} and
//    {9, 10, 13, 14}, 14 pairs each).  For tile i an issuer waits until the tile's y bytes are
//    staged and the epilogue has read its group of tile i - 1, issues its products and commits to
//    its group's barrier (which completes after both of the group's issuers commit).
//  - Epilogue warps: wait for group X of tile i, fold it and release it (the tensor cores meanwhile
//    form group Y); wait for group Y, fold it, rebuild the exact 128-bit sums, reduce them once mod
//    q_t, release Y and store (the tensor cores meanwhile run group X of tile i + 1); then stage
//    tile i + 2 into the buffer tile i used.  Warp w reads TMEM lane quadrant w & 3 (targets
//    32 (w & 3) ..) and columns 8 (w >> 2) .. of each accumulator: eight coefficients of one target.
//
// Operand layout in shared memory (A and B): K-major, no swizzle, 8-row x 16-byte core matrices,
// K-direction core-matrix stride (LBO) 128 bytes, 8-row-group stride (SBO) 512 bytes, for a K extent
// of 64 sources (a digit or the special basis holds at most 64 primes).  The M byte planes are built
// on the host at context creation in exactly this layout; the y planes are packed by the threads.
//
// Every mbarrier wait is bounded: on expiry a thread records an error flag and leaves its loop (the
// others then run out of arrivals and leave theirs), the MMA warps wait (bounded again) for the
// products they issued, the CTA frees its tensor memory and returns; the host reports CKKS_ECUDA.
#include "internal.cuh"

namespace ckks {
namespace {

constexpr int kTM = 128, kTN = 32, kKP = 64, kPlanes = 8;
constexpr int kAPlane = kTM * kKP;         // 8 KiB per A byte plane
constexpr int kATile = kPlanes * kAPlane;  // 64 KiB per block of 128 targets
constexpr int kBPlane = kTN * kKP;         // 2 KiB per staged B byte plane
constexpr int kBTile = kPlanes * kBPlane;  // 16 KiB per staged coefficient tile
constexpr int kEpiWarps = 16, kEpiThreads = 32 * kEpiWarps;  // epilogue and staging
constexpr int kThreads = kEpiThreads + 128;                   // plus four MMA-issue warps
constexpr int kTmemCols = 512;
constexpr int kSmemB = kATile;             // two B buffers follow the A planes
constexpr int kSmemBar = kSmemB + 2 * kBTile;
constexpr int kSmemBytes = 116 * 1024;     // keeps one CTA per SM (it owns all of TMEM)
static_assert(kSmemBar + 8 * 8 + 4 <= kSmemBytes, "shared-memory layout");

__host__ __device__ __forceinline__ int cm_off(int row, int k)
{
    return (row >> 3) * 512 + (k >> 4) * 128 + (row & 7) * 16 + (k & 15);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Shared-memory matrix descriptor: start address >> 4, LBO 128 B, SBO 512 B, descriptor version 1,
// no swizzle.
__device__ __forceinline__ u64 smem_desc(uint32_t addr)
{
    return (u64)((addr >> 4) & 0x3FFF) | ((u64)(128 >> 4) << 16) | ((u64)(512 >> 4) << 32) | (1ull << 46);
}

// Instruction descriptor: int32 accumulate, unsigned 8-bit A and B, both K-major, N = 32, M = 128.
constexpr uint32_t kIdesc = (2u << 4) | ((uint32_t)(kTN >> 3) << 17) | ((uint32_t)(kTM >> 4) << 24);

// D[tmem_d] (+)= A[adesc] x B[bdesc], both from shared memory.
__device__ __forceinline__ void mma_ss(uint32_t tmem_d, u64 adesc, u64 bdesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
        :: "r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate), "r"(0), "r"(0), "r"(0),
           "r"(0));
}

__device__ __forceinline__ void commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(smem_u32(bar)) : "memory");
}

// Bounded wait for the given phase parity of an mbarrier.
__device__ __forceinline__ bool mbar_wait(const uint64_t *bar, uint32_t parity)
{
    const uint32_t a = smem_u32(bar);
    for (int i = 0; i < (1 << 18); ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(done) : "r"(a), "r"(parity) : "memory");
        if (done) return true;
    }
    return false;
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

// True in exactly one lane of the (converged) warp.  The MMA warps issue from this lane with every
// operand computed warp-wide, so the operands stay warp-uniform and the products issue back to back.
__device__ __forceinline__ bool elect_one()
{
    uint32_t pred;
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}" : "=r"(pred));
    return pred != 0;
}
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// The products of the y tile at `bdesc` into the accumulators P_d whose bit d is set in kMask.  The
// first product into each P_d (u = max(0, d - 7), K-step 0) overwrites it.
template <int kMask>
__device__ __forceinline__ void issue_set(uint32_t tmem, u64 adesc, u64 bdesc, bool two_k)
{
#pragma unroll
    for (int u = 0; u < kPlanes; ++u)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            if (h == 1 && !two_k) break;
            const u64 ad = adesc + ((u * kAPlane + h * 256) >> 4);
#pragma unroll
            for (int v = 0; v < kPlanes; ++v) {
                const int d = u + v;
                if (!((kMask >> d) & 1)) continue;
                const uint32_t acc = (h == 0 && u == (d > 7 ? d - 7 : 0)) ? 0u : 1u;
                mma_ss(tmem + d * kTN, ad, bdesc + ((v * kBPlane + h * 256) >> 4), acc);
            }
        }
}

// CNT accumulators from P_D0 on, four columns each.
template <int D0, int CNT>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&r)[CNT][4])
{
#pragma unroll
    for (int i = 0; i < CNT; ++i)
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(r[i][0]), "=r"(r[i][1]), "=r"(r[i][2]), "=r"(r[i][3])
                     : "r"(taddr + (D0 + i) * kTN));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// p0 + p1 2^8 + p2 2^16 + p3 2^24 (each p < 2^25).
__device__ __forceinline__ u64 fold4(uint32_t p0, uint32_t p1, uint32_t p2, uint32_t p3)
{
    return (u64)p0 + ((u64)p1 << 8) + ((u64)p2 << 16) + ((u64)p3 << 24);
}

// x = hi 2^64 + lo (x < 2^126) mod q for q = 2^60 - delta, delta < 2^28.  Since 2^60 = delta
// (mod q): fold the bits from 2^64 on with 2^64 = 16 delta, then twice the bits from 2^60 on.
__device__ __forceinline__ u64 reduce_special(u64 hi, u64 lo, const PrimeConst &c)
{
    constexpr u64 kMask60 = ((u64)1 << 60) - 1;
    const uint32_t c16 = (uint32_t)c.delta << 4;
    const u64 p0 = (u64)(uint32_t)hi * c16, p1 = (u64)(uint32_t)(hi >> 32) * c16;
    const u64 t = p0 + (p1 << 32);
    const u64 yl = t + lo;
    const u64 yh = (p1 >> 32) + (t < p0) + (yl < t);    // y = hi 16 delta + lo < 2^95
    const u64 a = (yh << 4) | (yl >> 60);               // floor(y / 2^60) < 2^35
    const u64 z = (yl & kMask60) + a * c.delta;         // < 2^64
    const u64 w = (z & kMask60) + (z >> 60) * c.delta;  // < 2^60 + 2^32 < 2q
    return w >= c.q ? w - c.q : w;
}

// Job geometry of one launch (kind 0: ModUp over (ciphertext, digit); kind 1: ModDown over
// (job, component)).
struct TcJobs {
    int kind;
    const u64 *y;         // sources, coefficient form
    u64 *out;             // digits (ModUp) or conversion output (ModDown)
    const uint8_t *apl;   // A rows
    int L, LK, alpha, dnum, K, tb_per_digit;
    int csplit;           // coefficient runs per target block
    __device__ __forceinline__ void geometry(int z, int &S, int &T, int &lo, const u64 *&ybase,
                                             const uint8_t *&abase) const
    {
        if (kind == 0) {
            const int b = z / dnum, jd = z - b * dnum;
            lo = jd * alpha;
            S = min(alpha, L - lo);
            T = LK - S;
            ybase = y + ((size_t)b * L + lo) * kN;
            abase = apl + (size_t)jd * tb_per_digit * kATile;
        } else {
            lo = 0;
            S = K;
            T = L;
            ybase = y + (size_t)z * K * kN;
            abase = apl;
        }
    }
    __device__ __forceinline__ int prime(int ti, int lo, int S) const
    {
        return kind == 0 ? (ti < lo ? ti : ti + S) : ti;
    }
    __device__ __forceinline__ u64 *row(int z, int t) const
    {
        return kind == 0 ? out + ((size_t)z * LK + t) * kN : out + ((size_t)z * L + t) * kN;
    }
};

// Byte planes of sources s0 .. s0 + 3 of coefficient n into a staged B tile.
__device__ __forceinline__ void stage4(uint8_t *buf, const u64 (&v)[4], int n, int s0)
{
    uint8_t *p = buf + cm_off(n, s0);
    const uint32_t x0 = (uint32_t)v[0], x1 = (uint32_t)v[1], x2 = (uint32_t)v[2], x3 = (uint32_t)v[3];
    const uint32_t y0 = (uint32_t)(v[0] >> 32), y1 = (uint32_t)(v[1] >> 32), y2 = (uint32_t)(v[2] >> 32),
                   y3 = (uint32_t)(v[3] >> 32);
    // bytes b of the four values, packed low to high: interleave pairs, then pairs of pairs
    const uint32_t lo01 = __byte_perm(x0, x1, 0x5140), hi01 = __byte_perm(x0, x1, 0x7362);
    const uint32_t lo23 = __byte_perm(x2, x3, 0x5140), hi23 = __byte_perm(x2, x3, 0x7362);
    const uint32_t Lo01 = __byte_perm(y0, y1, 0x5140), Hi01 = __byte_perm(y0, y1, 0x7362);
    const uint32_t Lo23 = __byte_perm(y2, y3, 0x5140), Hi23 = __byte_perm(y2, y3, 0x7362);
    *reinterpret_cast<uint32_t *>(p + 0 * kBPlane) = __byte_perm(lo01, lo23, 0x5410);
    *reinterpret_cast<uint32_t *>(p + 1 * kBPlane) = __byte_perm(lo01, lo23, 0x7632);
    *reinterpret_cast<uint32_t *>(p + 2 * kBPlane) = __byte_perm(hi01, hi23, 0x5410);
    *reinterpret_cast<uint32_t *>(p + 3 * kBPlane) = __byte_perm(hi01, hi23, 0x7632);
    *reinterpret_cast<uint32_t *>(p + 4 * kBPlane) = __byte_perm(Lo01, Lo23, 0x5410);
    *reinterpret_cast<uint32_t *>(p + 5 * kBPlane) = __byte_perm(Lo01, Lo23, 0x7632);
    *reinterpret_cast<uint32_t *>(p + 6 * kBPlane) = __byte_perm(Hi01, Hi23, 0x5410);
    *reinterpret_cast<uint32_t *>(p + 7 * kBPlane) = __byte_perm(Hi01, Hi23, 0x7632);
}

// Four outputs of group X: g0 = P_0 + .. + P_3 2^24, g1 = P_4 + .. + P_7 2^24 (columns col .. col + 3).
__device__ __forceinline__ void fold_x(uint32_t taddr, u64 *g0, u64 *g1)
{
    uint32_t r[8][4];
    tmem_ld<0, 8>(taddr, r);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        g0[c] = fold4(r[0][c], r[1][c], r[2][c], r[3][c]);
        g1[c] = fold4(r[4][c], r[5][c], r[6][c], r[7][c]);
    }
}

// Four outputs completed with group Y: the exact 128-bit sum, reduced mod the row's prime.
template <bool kSpecial>
__device__ __forceinline__ void finish_y(uint32_t taddr, const u64 *g0, const u64 *g1, const PrimeConst &p,
                                         u64 *res)
{
    uint32_t r[7][4];
    tmem_ld<8, 7>(taddr, r);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const u64 g2 = fold4(r[0][c], r[1][c], r[2][c], r[3][c]);
        const u64 g3 = fold4(r[4][c], r[5][c], r[6][c], 0);
        const u64 lo64 = g0[c] + (g1[c] << 32);
        const u64 hi64 = (g1[c] >> 32) + g2 + (g3 << 32) + (lo64 < g0[c]);
        if constexpr (kSpecial)
            res[c] = reduce_special(hi64, lo64, p);
        else
            res[c] = reduce128(hi64, lo64, p);
    }
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, int count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" :: "r"(smem_u32(bar))
                 : "memory");
}

// Barriers in shared memory after the B buffers.
enum { kBarMmaX, kBarMmaY, kBarFreeX, kBarFreeY, kBarFull0, kBarFull1, kBarDrain, kNumBars };

template <bool kSpecial>
__global__ void __launch_bounds__(kThreads, 1) conv_tc_kernel(TcJobs jobs, const PrimeConst *__restrict__ pc,
                                                               int *err)
{
    extern __shared__ __align__(1024) uint8_t sm[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tb = blockIdx.x / jobs.csplit, run = blockIdx.x - tb * jobs.csplit, z = blockIdx.y;
    int S, T, lo;
    const u64 *ybase;
    const uint8_t *abase;
    jobs.geometry(z, S, T, lo, ybase, abase);
    if (tb * kTM >= T) return;  // uniform per CTA
    const int ntiles = kN / kTN / jobs.csplit;  // 16, 32 or 64
    const int cbase = run * ntiles * kTN;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + kSmemBar);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + kSmemBar + 8 * kNumBars);
    const bool mma_warp = warp >= kEpiWarps;
    const int issuer = warp - kEpiWarps;  // 0, 1: group X; 2, 3: group Y
    const bool y_issuer = issuer >= 2;

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(tslot)), "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        mbar_init(bar + kBarMmaX, 2);
        mbar_init(bar + kBarMmaY, 2);
        mbar_init(bar + kBarFreeX, kEpiThreads);
        mbar_init(bar + kBarFreeY, kEpiThreads);
        mbar_init(bar + kBarFull0, kEpiThreads);
        mbar_init(bar + kBarFull1, kEpiThreads);
        mbar_init(bar + kBarDrain, 4);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // Staging share of an epilogue thread: coefficient n of each tile, sources s0 .. s0 + 3.  A warp
    // covers 8 coefficients x 4 source quads, so its 32-bit stores into the core-matrix layout fall
    // in 32 different banks (bank = 4 (n & 7) + ((s0 & 15) >> 2)).
    const int n = ((warp & 3) << 3) | (lane & 7), s0 = ((warp >> 2) << 4) | ((lane >> 3) << 2);
    const u64 *ysrc = ybase + (size_t)s0 * kN + cbase + n;
    auto fetch = [&](int i, u64 (&v)[4]) {
#pragma unroll
        for (int k = 0; k < 4; ++k) v[k] = s0 + k < S ? __ldg(ysrc + (size_t)k * kN + i * kTN) : 0;
    };
    u64 pre[4];
    if (!mma_warp) {
        const uint4 *src = reinterpret_cast<const uint4 *>(abase + (size_t)tb * kATile);
        uint4 *dst = reinterpret_cast<uint4 *>(sm);
        for (int i = tid; i < kATile / 16; i += kEpiThreads) dst[i] = __ldg(src + i);
        u64 w[4];
        fetch(0, pre);
        fetch(1, w);
        stage4(sm + kSmemB, pre, n, s0);
        stage4(sm + kSmemB + kBTile, w, n, s0);
        fetch(2, pre);  // ntiles >= 16
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *tslot;
    bool ok = true;

    if (mma_warp) {
        // ------------------------------------------------ MMA issue (one elected lane per warp)
        const bool two_k = S > 32;
        const u64 adesc = smem_desc(smem_u32(sm)), bdesc0 = smem_desc(smem_u32(sm + kSmemB));
        for (int i = 0; i < ntiles && ok; ++i) {
            const u64 bdesc = bdesc0 + (((i & 1) * kBTile) >> 4);
            ok = __all_sync(0xffffffffu, mbar_wait(bar + kBarFull0 + (i & 1), (i >> 1) & 1));
            if (ok && i > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar + (y_issuer ? kBarFreeY : kBarFreeX), (i - 1) & 1));
            if (!ok) break;
            fence_after();
            if (elect_one()) {
                // P_d sets of 18, 18, 14 and 14 plane pairs
                if (issuer == 0) issue_set<(1 << 0) | (1 << 1) | (1 << 6) | (1 << 7)>(tmem, adesc, bdesc, two_k);
                if (issuer == 1) issue_set<(1 << 2) | (1 << 3) | (1 << 4) | (1 << 5)>(tmem, adesc, bdesc, two_k);
                if (issuer == 2) issue_set<(1 << 8) | (1 << 11) | (1 << 12)>(tmem, adesc, bdesc, two_k);
                if (issuer == 3) issue_set<(1 << 9) | (1 << 10) | (1 << 13) | (1 << 14)>(tmem, adesc, bdesc, two_k);
                commit(bar + (y_issuer ? kBarMmaY : kBarMmaX));
            }
            __syncwarp();
        }
        // every product issued here has completed before tensor memory is freed (bounded)
        if (lane == 0) commit(bar + kBarDrain);
        __syncwarp();
        ok = mbar_wait(bar + kBarDrain, 0) && ok;
    } else {
        // ------------------------------------------------ epilogue and staging
        const int quad = warp & 3, part = warp >> 2;
        const int row = quad * 32 + lane, ti = tb * kTM + row;
        const bool valid = ti < T;
        const int t = valid ? jobs.prime(ti, lo, S) : 0;
        const PrimeConst p = pc[t];
        u64 *row_out = jobs.row(z, t) + cbase + part * 8;
        const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + part * 8;
        mbar_arrive(bar + kBarFull0);  // tiles 0 and 1 were staged before the block barrier
        mbar_arrive(bar + kBarFull1);
        for (int i = 0; i < ntiles; ++i) {
            ok = mbar_wait(bar + kBarMmaX, i & 1) && ok;
            fence_after();
            u64 g0[8], g1[8];
            fold_x(taddr, g0, g1);
            fold_x(taddr + 4, g0 + 4, g1 + 4);
            fence_before();
            mbar_arrive(bar + kBarFreeX);
            ok = mbar_wait(bar + kBarMmaY, i & 1) && ok;
            fence_after();
            u64 res[8];
            finish_y<kSpecial>(taddr, g0, g1, p, res);
            finish_y<kSpecial>(taddr + 4, g0 + 4, g1 + 4, p, res + 4);
            fence_before();
            mbar_arrive(bar + kBarFreeY);
            if (valid && ok) {
                ulonglong2 *o = reinterpret_cast<ulonglong2 *>(row_out + i * kTN);
#pragma unroll
                for (int k = 0; k < 4; ++k) o[k] = make_ulonglong2(res[2 * k], res[2 * k + 1]);
            }
            // both groups of tile i are complete: its buffer takes tile i + 2
            if (i + 2 < ntiles) {
                stage4(sm + kSmemB + (i & 1) * kBTile, pre, n, s0);
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive(bar + kBarFull0 + (i & 1));
                if (i + 3 < ntiles) fetch(i + 3, pre);
            }
            if (!ok) break;
        }
    }
    if (!ok) atomicExch(err, 1);
    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(kTmemCols));
}

// Host: byte planes of a (targets x sources) matrix given by `at(ti, s)`, one block of 128 targets
// after another, in the shared-memory core-matrix layout.
template <class F>
void build_planes(std::vector<uint8_t> &dst, size_t base, int T, int S, F at)
{
    const int tbs = (T + kTM - 1) / kTM;
    for (int tb = 0; tb < tbs; ++tb)
        for (int r = 0; r < kTM; ++r) {
            const int ti = tb * kTM + r;
            for (int s = 0; s < kKP; ++s) {
                const u64 m = (ti < T && s < S) ? at(ti, s) : 0;
                for (int u = 0; u < kPlanes; ++u)
                    dst[base + (size_t)tb * kATile + (size_t)u * kAPlane + cm_off(r, s)] = (uint8_t)(m >> (8 * u));
            }
        }
}

int upload_bytes(ckks_ctx *ctx, const std::vector<uint8_t> &h, const uint8_t **out)
{
    void *d = nullptr;
    if (cudaMalloc(&d, h.size()) != cudaSuccess) {
        cudaGetLastError();
        return set_error(CKKS_ENOMEM, "tensor-core table allocation failed");
    }
    ctx->allocations.push_back(d);
    cudaError_t e = cudaMemcpy(d, h.data(), h.size(), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_status(e, "cudaMemcpy(tensor-core tables)");
    *out = static_cast<const uint8_t *>(d);
    return CKKS_OK;
}

int launch(const ckks_ctx *ctx, TcJobs j, int tbs, int jobs, cudaStream_t s)
{
    if (jobs <= 0) return CKKS_OK;
    // enough CTAs for the machine: split each block's coefficients into runs when blocks are few
    const long ctas = (long)tbs * jobs;
    j.csplit = ctas >= 148 * 16 ? 1 : ctas >= 148 * 8 ? 2 : 4;  // 64, 32 or 16 tiles per run
    const dim3 grid(tbs * j.csplit, jobs);
    if (ctx->t.tc_special)
        conv_tc_kernel<true><<<grid, kThreads, kSmemBytes, s>>>(j, ctx->t.pc, ctx->tc_err);
    else
        conv_tc_kernel<false><<<grid, kThreads, kSmemBytes, s>>>(j, ctx->t.pc, ctx->tc_err);
    CKKS_CHECK_LAUNCH("conv_tc_kernel");
    return CKKS_OK;
}

// ---------------------------------------------------------------- tensor-pipe microbenchmark
// Back-to-back tcgen05.mma (kind::i8, M = 128, K = 32, both operands in shared memory) from one
// elected thread per CTA (warp-uniform operands), one CTA per SM: the fixed cost per MMA at a given N (the conversion's own tile is
// N = 32) and the dense int8 rate (N = 256).  Operand values do not matter; the products accumulate
// into one TMEM region.
constexpr int kBenchSmem = kTM * kKP + 256 * kKP + 64;  // A 8 KiB, B up to 16 KiB, barrier, slot

template <int N>
__global__ void __launch_bounds__(128, 1) mma_rate_kernel(int iters, int *err)
{
    extern __shared__ __align__(1024) uint8_t sm[];
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + kTM * kKP + 256 * kKP);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + kTM * kKP + 256 * kKP + 8);
    for (int i = threadIdx.x; i < (kTM + 256) * kKP / 4; i += blockDim.x)
        reinterpret_cast<uint32_t *>(sm)[i] = 0x01010101u;
    if (threadIdx.x < 32) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(tslot)), "r"(256));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *tslot;
    if (threadIdx.x < 32) {
        constexpr uint32_t idesc = (2u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(kTM >> 4) << 24);
        const u64 ad = smem_desc(smem_u32(sm)), bd = smem_desc(smem_u32(sm + kTM * kKP));
        if (elect_one()) {
            for (int r = 0; r < iters; r += 8) {
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    asm volatile(
                        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
                        :: "r"(tmem), "l"(ad + ((k & 1) * 256 >> 4)), "l"(bd + ((k & 1) * 256 >> 4)), "r"(idesc),
                           "r"(k | r), "r"(0), "r"(0), "r"(0), "r"(0));
            }
            commit(bar);
            if (!mbar_wait(bar, 0)) atomicExch(err, 1);
        }
        __syncwarp();
    }
    fence_before();
    __syncthreads();
    fence_after();
    if (threadIdx.x < 32)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(256));
}

// Failure-path self-test: one thread waits, with the same bound as every other wait in this file, on
// an mbarrier that nothing ever completes, and raises the context's flag when the bound expires.
__global__ void wait_expiry_kernel(int *err)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if (!mbar_wait(&bar, 0)) atomicExch(err, 1);
    }
}

}  // namespace

ConvKind conv_kind(const ckks_ctx *ctx, int sources)
{
    switch (ctx->conv_engine.load(std::memory_order_relaxed)) {
    case CKKS_CONV_INTEGER: return kConvInteger;
    case CKKS_CONV_TENSOR: return kConvTensor;
    case CKKS_CONV_FOLDED: return kConvFolded;
    default: return sources > kTcMinSources ? kConvFolded : kConvInteger;
    }
}

int build_tc_tables(ckks_ctx *ctx, const std::vector<u64> &up_mat, const std::vector<u64> &dn_mat)
{
    Tables &T = ctx->t;
    const int L = ctx->L, K = ctx->K, LK = L + K, alpha = ctx->alpha, dnum = ctx->dnum;
    T.tc_tb_per_digit = (LK - 1 + kTM - 1) / kTM;
    T.tc_special = true;
    for (int i = 0; i < LK; ++i) {
        const u64 q = ctx->mods[i], top = (u64)1 << 60;
        T.tc_special = T.tc_special && q < top && top - q < ((u64)1 << 28);
    }
    {
        const size_t per_digit = (size_t)T.tc_tb_per_digit * kATile;
        std::vector<uint8_t> h(per_digit * dnum, 0);
        for (int j = 0; j < dnum; ++j) {
            const int lo = j * alpha, S = std::min(alpha, L - lo);
            build_planes(h, per_digit * j, LK - S, S, [&](int ti, int s) {
                const int t = ti < lo ? ti : ti + S;
                return up_mat[((size_t)j * alpha + s) * LK + t];
            });
        }
        CKKS_TRY(upload_bytes(ctx, h, &T.tc_up));
    }
    {
        std::vector<uint8_t> h((size_t)((L + kTM - 1) / kTM) * kATile, 0);
        build_planes(h, 0, L, K, [&](int ti, int s) { return dn_mat[(size_t)s * L + ti]; });
        CKKS_TRY(upload_bytes(ctx, h, &T.tc_dn));
    }
    cudaError_t e = cudaMalloc(&ctx->tc_err, sizeof(int));
    if (e != cudaSuccess) {
        cudaGetLastError();
        return set_error(CKKS_ENOMEM, "flag allocation failed");
    }
    ctx->allocations.push_back(ctx->tc_err);
    e = cudaMemset(ctx->tc_err, 0, sizeof(int));
    if (e != cudaSuccess) return cuda_status(e, "cudaMemset(flag)");
    e = cudaFuncSetAttribute(conv_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(conv_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemBytes);
    if (e != cudaSuccess) return cuda_status(e, "cudaFuncSetAttribute(conv_tc_kernel)");
    return CKKS_OK;
}

int launch_conv_tc_up(const ckks_ctx *ctx, const u64 *y, u64 *digits, int batch, cudaStream_t s)
{
    const Tables &T = ctx->t;
    TcJobs j{0, y, digits, T.tc_up, T.L, T.LK, T.alpha, T.dnum, T.K, T.tc_tb_per_digit, 1};
    return launch(ctx, j, T.tc_tb_per_digit, batch * T.dnum, s);
}

int launch_conv_tc_down(const ckks_ctx *ctx, const u64 *zsrc, u64 *cv, int jobs2, cudaStream_t s)
{
    const Tables &T = ctx->t;
    TcJobs j{1, zsrc, cv, T.tc_dn, T.L, T.LK, T.alpha, T.dnum, T.K, 0, 1};
    return launch(ctx, j, (T.L + kTM - 1) / kTM, jobs2, s);
}

int bench_mma(const ckks_ctx *ctx, int n, int blocks, int iters, double *ms, double *ops)
{
    iters = (iters + 7) / 8 * 8;
    cudaError_t e = n == 32 ? cudaFuncSetAttribute(mma_rate_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   kBenchSmem)
                            : cudaFuncSetAttribute(mma_rate_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   kBenchSmem);
    if (e != cudaSuccess) return cuda_status(e, "cudaFuncSetAttribute(mma_rate_kernel)");
    auto launch_n = [&](int it) {
        if (n == 32)
            mma_rate_kernel<32><<<blocks, 128, kBenchSmem>>>(it, ctx->tc_err);
        else
            mma_rate_kernel<256><<<blocks, 128, kBenchSmem>>>(it, ctx->tc_err);
    };
    cudaEvent_t a, b;
    cudaEventCreate(&a);
    cudaEventCreate(&b);
    launch_n(8);  // warm-up
    cudaEventRecord(a);
    launch_n(iters);
    cudaEventRecord(b);
    e = cudaEventSynchronize(b);
    float t = 0;
    cudaEventElapsedTime(&t, a, b);
    cudaEventDestroy(a);
    cudaEventDestroy(b);
    if (e != cudaSuccess) return cuda_status(e, "mma_rate_kernel");
    *ms = t;
    *ops = 2.0 * kTM * n * 32 * (double)blocks * iters;
    return CKKS_OK;
}

int selftest_wait_expiry(const ckks_ctx *ctx)
{
    wait_expiry_kernel<<<1, 32>>>(ctx->tc_err);
    CKKS_CHECK_LAUNCH("wait_expiry_kernel");
    return CKKS_OK;
}

}  // namespace ckks
