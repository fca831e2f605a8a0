// RNS basis conversion on the int8 tensor cores, folded form (tcgen05.mma kind::i8 with the data
// operand in tensor memory).
//
// The conversion out[t][c] = (sum_s M[s][t] y[s][c]) mod q_t (the step the Kestrel engine write-up,
// section 3 table, names "RNS basis conversion") is computed exactly, but with the byte weights of
// the data folded into the matrix modulo each target prime:
//     y_s = sum_v y_{s,v} 2^(8v)  (bytes),   F[(s,v)][t] = 2^(8v) M[s][t] mod q_t  (60 bits),
//     out_t = sum_{s,v} y_{s,v} F[(s,v)][t]  (mod q_t).
// F is split into byte planes F_u, so that
//     sum_{s,v} y_{s,v} F = sum_{u<8} 2^(8u) P_u,   P_u = sum_{k'} y_{k'} F_u[k'][t],  k' = 8s + v,
// an unsigned 8-bit contraction of K' = 8 S terms: P_u <= 512 * 255^2 < 2^25, so eight int32
// accumulators hold the exact sum, and the epilogue rebuilds the (< 2^82) value and reduces it once.
// The K' index 8s + v makes the data operand the raw 64-bit words: the four bytes of a 32-bit half
// of y_s are consecutive K' entries, so staging writes the words unchanged.
//
// One CTA (one per SM, owning all 512 TMEM columns) converts one block of 32 targets (the MMA's N)
// for a run of coefficient tiles of 128 (the MMA's M, the TMEM lanes):
//  - the block's eight F planes (8 x 32 targets x 512 bytes = 128 KiB) stay in shared memory (the B
//    operand, K-major core matrices) for the whole run; the CTA copies only the K' chunks its
//    products read (16-byte cp.async, issued together with tile 0's data words);
//  - each staging thread copies its 16 words of the next data tile (cp.async, 8 bytes each) into
//    its own shared-memory slots one tile ahead, and moves them (one coefficient per TMEM lane) into
//    the A operand in tensor memory when a buffer frees up: double-buffered, columns 256..383 and
//    384..511, two 32-bit columns per source;
//  - accumulator P_u takes columns 32 u .. 32 u + 31.
// Warp roles (20 warps, so that 96 registers fit), synchronised by mbarriers only:
//  - 4 MMA warps (one elected lane each) own planes {k, k + 4}: for tile i each waits until its
//    data is staged, then per plane group g (P_0..P_3, then P_4..P_7) until the epilogue has read
//    group g of tile i - 1, issues the ceil(S / 4) K-steps of its plane in that group and commits.
//    All four warps issue group 0 before group 1, so group 0 completes half-way through the tile
//    and the epilogue reads it while group 1 runs;
//  - 16 epilogue / staging warps: for tile i they read plane group 0 as soon as it completes and
//    release it (the next tile's products into it can start) and fold it to the low 50 bits of each
//    sum; read and release group 1 as soon as it completes, rebuild each (< 2^83) sum, reduce it
//    once and store it while the tensor cores run the next tile; then stage tile i + 2 from shared
//    memory into the data buffer tile i used (every product of tile i is complete by then).
//    Warp w reads TMEM lane quadrant w & 3 (coefficients 32 (w & 3) ..) and columns 8 (w >> 2) ..
//    8 (w >> 2) + 7 of each plane: eight targets of one coefficient; for staging it owns sources
//    16 (w >> 2) .. + 15.
// Three job geometries: ModUp (a digit into its L + K - S other primes), ModDown (the special
// primes into the ciphertext primes) and a window of ModUp (a digit into the primes of one window
// of the streamed rotation, its own table layout).
// Per output the epilogue spends 8 tensor-memory words, two folds and one reduction: for primes
// 2^60 - delta (delta < 2^28) a funnel shift and one 32 x 32 multiply-add leave the value in
// [0, 2q), which the forward NTT that consumes every converted limb accepts (it takes inputs below
// 8q); other primes get the full 128-bit reduction.
//
// Every mbarrier wait is bounded: on expiry a thread records an error flag and leaves its loop, the
// MMA warps wait (bounded again) for the products they issued, the CTA frees its tensor memory and
// returns; the host reports CKKS_ECUDA.
#include "internal.cuh"

namespace ckks {
namespace {

constexpr int kFM = 128;                          // coefficients per tile (MMA M, TMEM lanes)
constexpr int kFN = 32;                           // targets per CTA (MMA N)
constexpr int kWinBlocks = (kWinMax + kFN - 1) / kFN;  // target blocks per streamed window
constexpr int kFKP = 512;                         // K' extent in bytes: 64 sources x 8 bytes
constexpr int kFPlanes = 8;
constexpr int kFPlaneBytes = kFN * kFKP;          // 16 KiB
constexpr int kFBlock = kFPlanes * kFPlaneBytes;  // 128 KiB per block of 32 targets
constexpr int kFSbo = (kFKP / 16) * 128;          // 8-row-group stride of the core-matrix layout
constexpr int kFEpiWarps = 16, kFEpiThreads = 32 * kFEpiWarps;
constexpr int kFMmaWarp0 = kFEpiWarps;
constexpr int kFThreads = kFEpiThreads + 128;  // 20 warps: at most 5 per SM partition keeps 96 registers
constexpr int kFTmemCols = 512;
constexpr int kFAcol = 256;                       // first data-buffer column
constexpr int kFSmemY = kFBlock;                  // staging slots: 16 words per epilogue thread (64 KiB)
constexpr int kFSmemDelta = kFSmemY + 16 * kFEpiThreads * 8;  // 32 target deltas 2^60 - q
constexpr int kFSmemBar = kFSmemDelta + 32 * 4;
constexpr int kFSmemBytes = kFSmemBar + 256;

enum { kFBarMma = 0, kFBarFree = 2, kFBarFull = 4, kFBarDrain = 6, kFNumBars = 7 };
static_assert(kFSmemBar + 8 * kFNumBars + 4 <= kFSmemBytes, "shared-memory layout");
static_assert(kFSmemBytes <= 227 * 1024, "shared memory per CTA");

__host__ __device__ __forceinline__ int fcm_off(int row, int k)
{
    return (row >> 3) * kFSbo + (k >> 4) * 128 + (row & 7) * 16 + (k & 15);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Shared-memory matrix descriptor: start address >> 4, LBO 128 B, SBO kFSbo, version 1, no swizzle.
__device__ __forceinline__ u64 fsmem_desc(uint32_t addr)
{
    return (u64)((addr >> 4) & 0x3FFF) | ((u64)(128 >> 4) << 16) | ((u64)(kFSbo >> 4) << 32) | (1ull << 46);
}

// Instruction descriptor: int32 accumulate, unsigned 8-bit A and B, both K-major, N = 32, M = 128.
constexpr uint32_t kFIdesc = (2u << 4) | ((uint32_t)(kFN >> 3) << 17) | ((uint32_t)(kFM >> 4) << 24);

// D[tmem_d] (+)= A[tmem_a] x B[bdesc]: A from tensor memory, B from shared memory.
__device__ __forceinline__ void mma_ts(uint32_t tmem_d, uint32_t tmem_a, u64 bdesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
        :: "r"(tmem_d), "r"(tmem_a), "l"(bdesc), "r"(kFIdesc), "r"(accumulate), "r"(0), "r"(0), "r"(0),
           "r"(0));
}

// True in exactly one lane of the (converged) warp.
__device__ __forceinline__ bool elect_one()
{
    uint32_t pred;
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}" : "=r"(pred));
    return pred != 0;
}
__device__ __forceinline__ void fcommit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(smem_u32(bar)) : "memory");
}

// Bounded wait for a phase parity: each poll lets the hardware suspend the thread for up to
// kFSuspendNs (it resumes as soon as the phase completes), so waiting warps take no issue slots
// from the working ones; kFPolls polls bound the whole wait to about a second.
constexpr uint32_t kFSuspendNs = 1000000;
constexpr int kFPolls = 1024;

__device__ __forceinline__ bool fbar_wait(const uint64_t *bar, uint32_t parity)
{
    const uint32_t a = smem_u32(bar);
    for (int i = 0; i < kFPolls; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(done) : "r"(a), "r"(parity), "r"(kFSuspendNs) : "memory");
        if (done) return true;
    }
    return false;
}

__device__ __forceinline__ void fbar_init(uint64_t *bar, int count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fbar_arrive(uint64_t *bar)
{
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" :: "r"(smem_u32(bar))
                 : "memory");
}

// Asynchronous 8-byte copy from global into this thread's own shared-memory slot (no register
// holds the word while it is in flight); completion per thread by commit / wait groups.
__device__ __forceinline__ void fcp8(void *dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" :: "r"(smem_u32(dst)), "l"(src) : "memory");
}

// The same for 16 bytes, through L2 only (a table block is read once per CTA).
__device__ __forceinline__ void fcp16(void *dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(smem_u32(dst)), "l"(src) : "memory");
}

__device__ __forceinline__ void fcp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void fcp_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void ffence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void ffence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 columns (16 source words) of the data operand for the warp's 32 lanes, as two stores of 16.
__device__ __forceinline__ void fst32(uint32_t taddr, const u64 (&v)[16])
{
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const u64 *w = v + 8 * h;
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
            "%16};"
            :: "r"(taddr + 16 * h), "r"((uint32_t)w[0]), "r"((uint32_t)(w[0] >> 32)), "r"((uint32_t)w[1]),
               "r"((uint32_t)(w[1] >> 32)), "r"((uint32_t)w[2]), "r"((uint32_t)(w[2] >> 32)), "r"((uint32_t)w[3]),
               "r"((uint32_t)(w[3] >> 32)), "r"((uint32_t)w[4]), "r"((uint32_t)(w[4] >> 32)), "r"((uint32_t)w[5]),
               "r"((uint32_t)(w[5] >> 32)), "r"((uint32_t)w[6]), "r"((uint32_t)(w[6] >> 32)), "r"((uint32_t)w[7]),
               "r"((uint32_t)(w[7] >> 32))
            : "memory");
    }
}

// Job geometry (kind 0: ModUp over (ciphertext, digit), the ciphertext fastest in the grid so the
// CTAs that share a digit's F block run together; kind 1: ModDown over (job, component); kind 2:
// ModUp of one prime window (primes w0 .. w0 + wn - 1, in tb_per_digit blocks of 32) over
// (ciphertext, digit), into the window buffer [batch][dnum][wbuf][n]; the window's own digit (wown)
// has no conversion).
struct FoldJobs {
    int kind;
    const u64 *y;
    u64 *out;
    const uint8_t *fpl;   // F blocks
    int L, LK, alpha, dnum, K, tb_per_digit, batch;
    int csplit;
    int win, w0, wn, wown, wbuf;  // kind 2
    __device__ __forceinline__ void geometry(int z, int &S, int &T, int &lo, const u64 *&ybase,
                                             const uint8_t *&fbase, int &zrow) const
    {
        if (kind == 0) {
            const int b = z % batch, jd = z / batch;
            lo = jd * alpha;
            S = min(alpha, L - lo);
            T = LK - S;
            ybase = y + ((size_t)b * L + lo) * kN;
            fbase = fpl + (size_t)jd * tb_per_digit * kFBlock;
            zrow = b * dnum + jd;
        } else if (kind == 2) {
            const int b = z % batch, jd = z / batch;
            lo = jd * alpha;
            S = min(alpha, L - lo);
            T = jd == wown ? 0 : wn;
            ybase = y + ((size_t)b * L + lo) * kN;
            fbase = fpl + ((size_t)win * dnum + jd) * tb_per_digit * kFBlock;
            zrow = b * dnum + jd;
        } else {
            lo = 0;
            S = K;
            T = L;
            ybase = y + (size_t)z * K * kN;
            fbase = fpl;
            zrow = z;
        }
    }
    // the prime of target ti, and its row in the output block of job zrow
    __device__ __forceinline__ int prime(int ti, int lo, int S) const
    {
        return kind == 0 ? (ti < lo ? ti : ti + S) : kind == 2 ? w0 + ti : ti;
    }
    __device__ __forceinline__ int orow(int ti, int lo, int S) const { return kind == 2 ? ti : prime(ti, lo, S); }
    __device__ __forceinline__ u64 *row(int zrow, int t) const
    {
        return kind == 0   ? out + ((size_t)zrow * LK + t) * kN
               : kind == 2 ? out + ((size_t)zrow * wbuf + t) * kN
                           : out + ((size_t)zrow * L + t) * kN;
    }
};

// p0 + p1 2^8 + p2 2^16 + p3 2^24 (each p < 2^25, sum < 2^50) as four 32 x 32 -> 64-bit
// multiply(-add)s on the multiply pipe.
__device__ __forceinline__ u64 ffold4(uint32_t p0, uint32_t p1, uint32_t p2, uint32_t p3)
{
    u64 g;
    asm("mul.wide.u32 %0, %1, 1;" : "=l"(g) : "r"(p0));
    asm("mad.wide.u32 %0, %1, 256, %0;" : "+l"(g) : "r"(p1));
    asm("mad.wide.u32 %0, %1, 65536, %0;" : "+l"(g) : "r"(p2));
    asm("mad.wide.u32 %0, %1, 16777216, %0;" : "+l"(g) : "r"(p3));
    return g;
}

// A value in [0, 2q) congruent to g0 + g1 2^32 mod q, for g0, g1 < 2^50 and q = 2^60 - delta,
// delta < 2^28.  The sum x < 2^83 is a 2^60 + b with a < 2^23; 2^60 = delta (mod q), so x = a delta
// + b < 2^60 + 2^51 < 2q.  The forward NTT that consumes every converted limb (ModUp's new limbs,
// ModDown's correction) accepts inputs below 8q and returns them fully reduced.
__device__ __forceinline__ u64 freduce_fold_lazy(u64 g0, u64 g1, uint32_t delta)
{
    uint32_t xm, xh;  // bits 32..63 and 64..95 of x (bits 0..31 are g0's low word)
    asm("add.cc.u32 %0, %2, %3;\n\taddc.u32 %1, %4, 0;"
        : "=r"(xm), "=r"(xh) : "r"((uint32_t)(g0 >> 32)), "r"((uint32_t)g1), "r"((uint32_t)(g1 >> 32)));
    const uint32_t a = __funnelshift_l(xm, xh, 4);                  // x >> 60
    const u64 b = ((u64)(xm & 0x0FFFFFFFu) << 32) | (uint32_t)g0;  // x mod 2^60
    u64 w;
    asm("mad.wide.u32 %0, %1, %2, %3;" : "=l"(w) : "r"(a), "r"(delta), "l"(b));
    return w;
}

// The same sum reduced by the generic 128-bit reduction (primes not of the 2^60 - delta form).
__device__ __forceinline__ u64 freduce_fold_generic(u64 g0, u64 g1, const PrimeConst &p)
{
    const u64 lo64 = g0 + (g1 << 32);
    const u64 hi64 = (g1 >> 32) + (lo64 < g0);
    return reduce128(hi64, lo64, p);
}

// Four planes (P_g4 .. P_g4+3) x eight columns of the warp's lanes, one wait for all loads.
__device__ __forceinline__ void fld4x8(uint32_t taddr, uint32_t (&r)[4][8])
{
#pragma unroll
    for (int u = 0; u < 4; ++u)
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(r[u][0]), "=r"(r[u][1]), "=r"(r[u][2]), "=r"(r[u][3]), "=r"(r[u][4]), "=r"(r[u][5]),
                       "=r"(r[u][6]), "=r"(r[u][7])
                     : "r"(taddr + u * kFN));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Four planes (P_g4 .. P_g4+3) x four columns of the warp's lanes, one wait for all loads.
__device__ __forceinline__ void fld4x4(uint32_t taddr, uint32_t (&r)[4][4])
{
#pragma unroll
    for (int u = 0; u < 4; ++u)
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(r[u][0]), "=r"(r[u][1]), "=r"(r[u][2]), "=r"(r[u][3])
                     : "r"(taddr + u * kFN));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Barriers: kFBarMma + g (g < 2) completes when the four commits of plane group g of a tile are in;
// kFBarFree + g (g < 2) when the epilogue has read plane group g (planes 4g .. 4g+3) of a tile;
// kFBarFull + b when tensor-memory data buffer b is staged; kFBarDrain when every issued product
// is done.
template <bool kSpecial>
__global__ void __launch_bounds__(kFThreads, 1) conv_fold_kernel(FoldJobs jobs, const PrimeConst *__restrict__ pc,
                                                                  int *err)
{
    extern __shared__ __align__(1024) uint8_t sm[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tb = blockIdx.x / jobs.csplit, run = blockIdx.x - tb * jobs.csplit, z = blockIdx.y;
    int S, T, lo, zrow;
    const u64 *ybase;
    const uint8_t *fbase;
    jobs.geometry(z, S, T, lo, ybase, fbase, zrow);
    if (tb * kFN >= T) return;  // uniform per CTA
    const int ntiles = kN / kFM / jobs.csplit;  // 16, 8 or 4
    const int cbase = run * ntiles * kFM;
    const int nks = (S + 3) >> 2;                // K-steps of 32 bytes (4 sources)
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + kFSmemBar);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + kFSmemBar + 8 * kFNumBars);
    uint32_t *dsm = reinterpret_cast<uint32_t *>(sm + kFSmemDelta);

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(tslot)), "r"(kFTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        for (int k = 0; k < 2; ++k) fbar_init(bar + kFBarMma + k, 4);
        fbar_init(bar + kFBarFree + 0, kFEpiThreads);
        fbar_init(bar + kFBarFree + 1, kFEpiThreads);
        fbar_init(bar + kFBarFull + 0, kFEpiThreads);
        fbar_init(bar + kFBarFull + 1, kFEpiThreads);
        fbar_init(bar + kFBarDrain, 4);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // Epilogue / staging threads: thread (quad, part) owns coefficient m = 32 quad + lane of a tile
    // and sources s0 .. s0 + 15.  Each copies its 16 words of a tile into its own shared-memory
    // slots one tile ahead, so the words are waiting when the tensor-memory buffer frees up, and no
    // register or other thread is involved while they travel.
    const int quad = warp & 3, part = warp >> 2;
    const int m = quad * 32 + lane, s0 = part * 16;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    u64 *slot = reinterpret_cast<u64 *>(sm + kFSmemY) + tid;  // word k at slot[k * 512]
    const u64 *ysrc = ybase + (size_t)s0 * kN + cbase + m;
    const bool full16 = s0 + 16 <= S;  // warp-uniform: all 16 of this thread's sources exist
    auto issue = [&](int t) {
        const u64 *src = ysrc + t * kFM;
        if (full16) {
#pragma unroll
            for (int k = 0; k < 16; ++k) fcp8(slot + k * kFEpiThreads, src + (size_t)k * kN);
        } else {
#pragma unroll
            for (int k = 0; k < 16; ++k)
                if (s0 + k < S) fcp8(slot + k * kFEpiThreads, src + (size_t)k * kN);
        }
        fcp_commit();
    };
    if (warp < kFEpiWarps) {
        // tile 0's words and the table block travel together: only the K' chunks the products read,
        // 2 nks chunks of 16 bytes in each 8-row group of each plane (the table is zero past 8 S, so
        // the last K-step's padding comes in as zeros)
        issue(0);
        const uint4 *src = reinterpret_cast<const uint4 *>(fbase + (size_t)tb * kFBlock);
        uint4 *dst = reinterpret_cast<uint4 *>(sm);
        const int nkc = 2 * nks, per_group = 8 * nkc;  // 16-byte words per 8-row group
        for (int i = tid; i < kFPlanes * (kFN / 8) * per_group; i += kFEpiThreads) {
            const int ug = i / per_group, w = i - ug * per_group;
            const int off = ug * (kFSbo / 16) + w;  // chunk w / 8, word w % 8 of group ug
            fcp16(dst + off, src + off);
        }
        fcp_commit();
        fcp_wait_all();
        if (tid < kFN) {
            const int ti = tb * kFN + tid;
            const PrimeConst &p = pc[ti < T ? jobs.prime(ti, lo, S) : 0];
            dsm[tid] = (uint32_t)p.delta;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    ffence_before();
    __syncthreads();
    ffence_after();
    const uint32_t tmem = *tslot;
    bool ok = true;

    if (warp >= kFMmaWarp0) {
        // ------------------------------------------------ MMA issue (one elected lane per warp)
        const int issuer = warp - kFMmaWarp0;  // planes issuer (group 0) and issuer + 4 (group 1)
        const u64 bdesc0 = fsmem_desc(smem_u32(sm));
        for (int i = 0; i < ntiles && ok; ++i) {
            const int buf = i & 1;
            ok = __all_sync(0xffffffffu, fbar_wait(bar + kFBarFull + buf, (i >> 1) & 1));
            const uint32_t ta = tmem + kFAcol + buf * 128;
            for (int g = 0; g < 2 && ok; ++g) {
                if (i > 0) ok = __all_sync(0xffffffffu, fbar_wait(bar + kFBarFree + g, (i - 1) & 1));
                if (!ok) break;
                ffence_after();
                const int u = issuer + 4 * g;
                const uint32_t td = tmem + u * kFN;
                const u64 bd = bdesc0 + (((size_t)u * kFPlaneBytes) >> 4);
                // Every operand is warp-uniform and one lane is elected by elect.sync: the products
                // then issue back to back, where a lane-divergent issue cost about 120 cycles each.
                if (elect_one()) {
                    mma_ts(td, ta, bd, 0u);
                    for (int ks = 1; ks < nks; ++ks) mma_ts(td, ta + ks * 8, bd + ks * 16, 1u);
                    fcommit(bar + kFBarMma + g);
                }
                __syncwarp();
            }
        }
        // every product issued here has completed before tensor memory is freed (bounded)
        if (lane == 0) fcommit(bar + kFBarDrain);
        __syncwarp();
        ok = fbar_wait(bar + kFBarDrain, 0) && ok;
    } else {
        // ------------------------------------------------ epilogue and staging
        // tile t's words: own slots -> tensor-memory buffer t & 1 (the caller knows it is free); the
        // copies of tile t + 1 then start into the same slots
        auto stage = [&](int t) -> bool {
            fcp_wait_all();
            u64 v[16];
            if (full16) {
#pragma unroll
                for (int k = 0; k < 16; ++k) v[k] = slot[k * kFEpiThreads];
            } else {
#pragma unroll
                for (int k = 0; k < 16; ++k) v[k] = s0 + k < S ? slot[k * kFEpiThreads] : 0;
            }
            fst32(tmem + lane_base + kFAcol + (t & 1) * 128 + part * 32, v);
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            ffence_before();
            fbar_arrive(bar + kFBarFull + (t & 1));
            if (t + 1 < ntiles) issue(t + 1);
            return true;
        };
        ok = stage(0);  // tile 0's copies were issued with the table block
        if (ok && ntiles > 1) ok = stage(1);
        // the eight targets of this thread, tb * 32 + part * 8 + c: element offset of its output word
        // in tile 0 from the job's first output row (-1 for a target past the end)
        u64 *const jobrow = jobs.row(zrow, 0);
        int toff[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int ti = tb * kFN + part * 8 + c;
            toff[c] = ti < T ? jobs.orow(ti, lo, S) * kN + cbase + m : -1;
        }
        const uint32_t tcol = tmem + lane_base + part * 8;
        for (int i = 0; i < ntiles && ok; ++i) {
            // plane group 0 (P_0 .. P_3): the low 50 bits of each sum
            ok = fbar_wait(bar + kFBarMma + 0, i & 1) && ok;
            ok = __all_sync(0xffffffffu, ok);  // warp-uniform: the loads below are warp-collective
            ffence_after();
            u64 g0[8];
#pragma unroll
            for (int hc = 0; hc < 2; ++hc) {
                uint32_t r[4][4];
                fld4x4(tcol + 4 * hc, r);
#pragma unroll
                for (int c = 0; c < 4; ++c) g0[4 * hc + c] = ffold4(r[0][c], r[1][c], r[2][c], r[3][c]);
            }
            ffence_before();
            fbar_arrive(bar + kFBarFree + 0);
            // plane group 1 (P_4 .. P_7), released as soon as it is read: the next tile's products
            // into both groups then run while this tile's outputs are finished
            ok = fbar_wait(bar + kFBarMma + 1, i & 1) && ok;
            ok = __all_sync(0xffffffffu, ok);
            ffence_after();
            uint32_t r1[4][8];
            fld4x8(tcol + 4 * kFN, r1);
            ffence_before();
            fbar_arrive(bar + kFBarFree + 1);
            u64 *const out_i = jobrow + i * kFM;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const u64 g1 = ffold4(r1[0][c], r1[1][c], r1[2][c], r1[3][c]);
                if (toff[c] < 0 || !ok) continue;
                u64 res;
                if constexpr (kSpecial)
                    res = freduce_fold_lazy(g0[c], g1, dsm[part * 8 + c]);
                else
                    res = freduce_fold_generic(g0[c], g1, pc[jobs.prime(tb * kFN + part * 8 + c, lo, S)]);
                out_i[toff[c]] = res;
            }
            // every product of tile i is complete: its data buffer takes tile i + 2
            if (i + 2 < ntiles && ok) ok = stage(i + 2);
        }
        fcp_wait_all();  // no copy of this thread is still in flight when the CTA exits
    }
    if (!ok) atomicExch(err, 1);
    ffence_before();
    __syncthreads();
    ffence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(kFTmemCols));
}

// Host: the F blocks of a (targets x sources) matrix given by `at(ti, s)` over target primes
// `prime(ti)`, one block of 32 targets after another, each in the shared-memory layout:
// plane u, row r (target 32 tb + r), byte k' = 8 s + v holds byte u of 2^(8v) at(ti, s) mod q.
// One block of 32 targets: targets ti0 .. ti0 + 31 (those below T) of F = 2^(8v) M mod q_t, at(ti, s)
// giving M[s][target ti] and prime(ti) its prime index.
template <class F, class P>
void build_fold_block(uint8_t *blk, int ti0, int T, int S, const std::vector<u64> &mods, F at, P prime)
{
    for (int r = 0; r < kFN; ++r) {
        const int ti = ti0 + r;
        if (ti >= T) continue;
        const u64 q = mods[prime(ti)];
        for (int s = 0; s < S; ++s) {
            u64 f = at(ti, s) % q;
            for (int v = 0; v < 8; ++v) {
                const int k = 8 * s + v;
                for (int u = 0; u < kFPlanes; ++u)
                    blk[(size_t)u * kFPlaneBytes + fcm_off(r, k)] = (uint8_t)(f >> (8 * u));
                f = host_mulmod(f, 256 % q, q);
            }
        }
    }
}

template <class F, class P>
void build_fold(std::vector<uint8_t> &dst, size_t base, int T, int S, const std::vector<u64> &mods, F at,
                P prime)
{
    const int tbs = (T + kFN - 1) / kFN;
    parallel_for(tbs, [&](int tb) {
        build_fold_block(dst.data() + base + (size_t)tb * kFBlock, tb * kFN, T, S, mods, at, prime);
    });
}

int upload_fold(ckks_ctx *ctx, const std::vector<uint8_t> &h, const uint8_t **out)
{
    void *d = nullptr;
    if (cudaMalloc(&d, std::max<size_t>(h.size(), 16)) != cudaSuccess) {
        cudaGetLastError();
        return set_error(CKKS_ENOMEM, "folded conversion table allocation failed");
    }
    ctx->allocations.push_back(d);
    cudaError_t e = cudaMemcpy(d, h.data(), h.size(), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_status(e, "cudaMemcpy(folded conversion tables)");
    *out = static_cast<const uint8_t *>(d);
    return CKKS_OK;
}

int launch_fold(const ckks_ctx *ctx, FoldJobs j, int tbs, int jobs, cudaStream_t s)
{
    if (jobs <= 0) return CKKS_OK;
    const long ctas = (long)tbs * jobs;
    // 16, 8 or 4 tiles per run; a window's conversion (kind 2) keeps whole runs down to one wave,
    // since every CTA pays the table load and the pipeline fill once
    if (j.kind == 2)
        j.csplit = ctas >= 148 ? 1 : ctas >= 74 ? 2 : 4;
    else
        j.csplit = ctas >= 148 * 4 ? 1 : ctas >= 148 * 2 ? 2 : 4;
    const dim3 grid(tbs * j.csplit, jobs);
    if (ctx->t.tc_special)
        conv_fold_kernel<true><<<grid, kFThreads, kFSmemBytes, s>>>(j, ctx->t.pc, ctx->tc_err);
    else
        conv_fold_kernel<false><<<grid, kFThreads, kFSmemBytes, s>>>(j, ctx->t.pc, ctx->tc_err);
    CKKS_CHECK_LAUNCH("conv_fold_kernel");
    return CKKS_OK;
}

}  // namespace

static int build_fold_tables(ckks_ctx *ctx)
{
    Tables &T = ctx->t;
    const std::vector<u64> &up_mat = ctx->up_mat_host, &dn_mat = ctx->dn_mat_host;
    const int L = ctx->L, K = ctx->K, LK = L + K, alpha = ctx->alpha, dnum = ctx->dnum;
    T.fold_tb_per_digit = (LK - 1 + kFN - 1) / kFN;
    if (alpha > 64 || K > 64) return set_error(CKKS_EUNSUPPORTED, "more than 64 sources per conversion");
    {
        const size_t per_digit = (size_t)T.fold_tb_per_digit * kFBlock;
        std::vector<uint8_t> h(per_digit * dnum, 0);
        for (int j = 0; j < dnum; ++j) {
            const int lo = j * alpha, S = std::min(alpha, L - lo);
            build_fold(h, per_digit * j, LK - S, S, ctx->mods,
                       [&](int ti, int s) {
                           const int t = ti < lo ? ti : ti + S;
                           return up_mat[((size_t)j * alpha + s) * LK + t];
                       },
                       [&](int ti) { return ti < lo ? ti : ti + S; });
        }
        CKKS_TRY(upload_fold(ctx, h, &T.fold_up));
    }
    {
        std::vector<uint8_t> h((size_t)((L + kFN - 1) / kFN) * kFBlock, 0);
        build_fold(h, 0, L, K, ctx->mods, [&](int ti, int s) { return dn_mat[(size_t)s * L + ti]; },
                   [&](int ti) { return ti; });
        CKKS_TRY(upload_fold(ctx, h, &T.fold_dn));
    }
    cudaError_t e = cudaFuncSetAttribute(conv_fold_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kFSmemBytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(conv_fold_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kFSmemBytes);
    if (e != cudaSuccess) return cuda_status(e, "cudaFuncSetAttribute(conv_fold_kernel)");
    return CKKS_OK;
}

// The folded tables, built once per context on the first call that needs them.
static int ensure_fold_tables(ckks_ctx *ctx)
{
    std::lock_guard<std::mutex> lock(ctx->mu);
    if (ctx->fold_built) return CKKS_OK;
    CKKS_TRY(build_fold_tables(ctx));
    ctx->fold_built = true;
    return CKKS_OK;
}

bool fold_tables_ready(const ckks_ctx *ctx)
{
    std::lock_guard<std::mutex> lock(const_cast<ckks_ctx *>(ctx)->mu);
    return ctx->fold_built;
}

// Windows of at most kWinMax primes: each digit's range and the special primes, each cut into
// near-equal pieces.
static void make_windows(const ckks_ctx *ctx, std::vector<ckks_ctx::Window> &out)
{
    auto split = [&](int a, int b, int own) {
        const int len = b - a;
        if (len <= 0) return;
        const int cnt = (len + kWinMax - 1) / kWinMax;
        for (int i = 0; i < cnt; ++i) {
            const int s0 = a + (int)((long)len * i / cnt), s1 = a + (int)((long)len * (i + 1) / cnt);
            out.push_back({s0, s1 - s0, own});
        }
    };
    for (int j = 0; j < ctx->dnum; ++j) split(j * ctx->alpha, std::min(ctx->L, (j + 1) * ctx->alpha), j);
    split(ctx->L, ctx->L + ctx->K, -1);
}

// The windows and their folded blocks: blocks (w, j, 0 .. kWinBlocks - 1) hold digit j's conversion
// into window w's primes (none for the window's own digit), built once per context on the first
// streamed call.
static int ensure_window_tables(ckks_ctx *ctx)
{
    CKKS_TRY(ensure_fold_tables(ctx));
    std::lock_guard<std::mutex> lock(ctx->mu);
    if (ctx->win_built) return CKKS_OK;
    std::vector<ckks_ctx::Window> win;
    make_windows(ctx, win);
    const int nw = (int)win.size(), dnum = ctx->dnum, L = ctx->L, LK = L + ctx->K, alpha = ctx->alpha;
    const std::vector<u64> &up_mat = ctx->up_mat_host;
    std::vector<uint8_t> h((size_t)nw * dnum * kWinBlocks * kFBlock, 0);
    parallel_for(nw * dnum * kWinBlocks, [&](int idx) {
        const int tb = idx % kWinBlocks, wj = idx / kWinBlocks, w = wj / dnum, j = wj - w * dnum;
        const ckks_ctx::Window wd = win[w];
        if (wd.own == j) return;
        const int S = std::min(alpha, L - j * alpha);
        build_fold_block(h.data() + (size_t)idx * kFBlock, tb * kFN, wd.n, S, ctx->mods,
                         [&](int ti, int s2) { return up_mat[((size_t)j * alpha + s2) * LK + wd.t0 + ti]; },
                         [&](int ti) { return wd.t0 + ti; });
    });
    CKKS_TRY(upload_fold(ctx, h, &ctx->fold_win));
    ctx->windows = std::move(win);
    ctx->win_built = true;
    return CKKS_OK;
}

int stream_windows(ckks_ctx *ctx, const std::vector<ckks_ctx::Window> **out)
{
    CKKS_TRY(ensure_window_tables(ctx));
    *out = &ctx->windows;
    return CKKS_OK;
}

int launch_conv_fold_window(ckks_ctx *ctx, const u64 *y, u64 *buf, int batch, int w, cudaStream_t s)
{
    CKKS_TRY(ensure_window_tables(ctx));
    const Tables &T = ctx->t;
    const ckks_ctx::Window wd = ctx->windows[w];
    FoldJobs j{2, y, buf, ctx->fold_win, T.L, T.LK, T.alpha, T.dnum, T.K, kWinBlocks, batch, 1,
               w, wd.t0, wd.n, wd.own, kWinMax};
    return launch_fold(ctx, j, (wd.n + kFN - 1) / kFN, batch * T.dnum, s);
}

int launch_conv_fold_up(ckks_ctx *ctx, const u64 *y, u64 *digits, int batch, cudaStream_t s)
{
    CKKS_TRY(ensure_fold_tables(ctx));
    const Tables &T = ctx->t;
    FoldJobs j{0, y, digits, T.fold_up, T.L, T.LK, T.alpha, T.dnum, T.K, T.fold_tb_per_digit, batch, 1};
    return launch_fold(ctx, j, T.fold_tb_per_digit, batch * T.dnum, s);
}

int launch_conv_fold_down(ckks_ctx *ctx, const u64 *zsrc, u64 *cv, int jobs2, cudaStream_t s)
{
    CKKS_TRY(ensure_fold_tables(ctx));
    const Tables &T = ctx->t;
    FoldJobs j{1, zsrc, cv, T.fold_dn, T.L, T.LK, T.alpha, T.dnum, T.K, 0, 1, 1};
    return launch_fold(ctx, j, (T.L + kFN - 1) / kFN, jobs2, s);
}

}  // namespace ckks
