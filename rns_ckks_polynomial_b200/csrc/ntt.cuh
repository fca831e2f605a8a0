// Limb-batched negacyclic NTT / INTT for n = 2048 with 60-bit primes.
//
// One CTA of 128 threads transforms one limb-polynomial at a time (and loops
// over a few consecutive jobs of the same prime, so its twiddles stay in L1).
// Each thread holds 16 coefficients in registers; the 11 butterfly stages run
// as two radix-16 passes and one double radix-8 pass, with the data exchanged
// between passes through a swizzled 32 KiB shared-memory tile (two alternating
// 16 KiB buffers) whose three access patterns are all bank-conflict free.
//
// Arithmetic: Harvey-style lazy butterflies with Shoup twiddles whose
// quotient comes from a three-product approximation of the high half
// (shoup4: result in [0, 4q)).  The forward (Cooley-Tukey) pass keeps values
// in [0, 8q), the inverse (Gentleman-Sande) pass in [0, 4q); 8q < 2^63 for
// q < 2^60.  Both end fully reduced to [0, q).  The inverse folds n^-1 into
// its last stage.  kS selects the cheaper quotient product for primes of the
// form 2^60 - delta, delta < 2^32.
//
// Ordering (the library's reading of the pages, which name NTT/INTT but not
// the convention): forward output slot k holds a(psi^(2 brv(k) + 1)); the
// stage with half-size h uses twiddle psi^brv((n + e) / (2h)) for the pair
// starting at element e.
//
// What happens to each element on its way in and out is supplied by a Job
// type, so ModUp, ModDown and rescale fuse their per-element arithmetic
// (copies, constant products, final combines) into the transform's own
// loads and stores.  A Job provides:
//   int count;                                  number of limb jobs
//   struct Ref { ...; int prime; };             job j decoded once (rows, constants)
//   __device__ Ref ref(int j) const;
//   fwd:  __device__ u64  load(const Ref &, int e)    element e (value < 8q)
//         __device__ void store4(const Ref &, int e, const u64 v[4])   e % 4 == 0
//   inv:  __device__ void load4(const Ref &, int e, u64 v[4])           values < 4q
//         __device__ void store(const Ref &, int e, u64 v)
#pragma once

#include "common.cuh"

namespace ckks {

constexpr int kNttThreads = 128;

// Shared-memory swizzle: bits 0..2 of the element index flip with bits 4..6 and
// bit 3 with bit 7, which makes the three access patterns of the passes
// conflict free for 64-bit words (every half-warp touches 16 distinct banks).
__device__ __forceinline__ int swz(int e) { return e ^ ((e >> 4) & 7) ^ (((e >> 7) & 1) << 3); }

__device__ __forceinline__ ulonglong2 ldtw(const ulonglong2 *tw, int i) { return __ldg(tw + i); }

struct Mod {
    u64 q, q2, q4, delta;
};

// Cooley-Tukey butterfly, inputs and outputs in [0, 8q).
template <bool kS>
__device__ __forceinline__ void ct_bfly(u64 &x, u64 &y, ulonglong2 w, const Mod &m)
{
    const u64 a = csub(x, m.q4);
    const u64 t = shoup4<kS>(y, w.x, w.y, m.q, m.delta);
    x = a + t;
    y = a - t + m.q4;
}

// Gentleman-Sande butterfly, inputs and outputs in [0, 4q).
template <bool kS>
__device__ __forceinline__ void gs_bfly(u64 &x, u64 &y, ulonglong2 w, const Mod &m)
{
    const u64 s = x + y;
    const u64 d = x - y + m.q4;
    x = csub(s, m.q4);
    y = shoup4<kS>(d, w.x, w.y, m.q, m.delta);
}

// Four forward stages (half-sizes 8S, 4S, 2S, S) on v[k] = a[base + r + S k],
// base a multiple of 16S; m1 = (n + base) / (16S).
template <bool kS>
__device__ __forceinline__ void fwd_radix16(u64 v[16], int m1, const ulonglong2 *tw, const Mod &m)
{
    {
        const ulonglong2 w = ldtw(tw, m1);
#pragma unroll
        for (int k = 0; k < 8; ++k) ct_bfly<kS>(v[k], v[k + 8], w, m);
    }
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        const ulonglong2 w = ldtw(tw, 2 * m1 + g);
#pragma unroll
        for (int k = 0; k < 4; ++k) ct_bfly<kS>(v[8 * g + k], v[8 * g + k + 4], w, m);
    }
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const ulonglong2 w = ldtw(tw, 4 * m1 + g);
        ct_bfly<kS>(v[4 * g], v[4 * g + 2], w, m);
        ct_bfly<kS>(v[4 * g + 1], v[4 * g + 3], w, m);
    }
#pragma unroll
    for (int g = 0; g < 8; ++g) ct_bfly<kS>(v[2 * g], v[2 * g + 1], ldtw(tw, 8 * m1 + g), m);
}

// Three forward stages (half-sizes 4, 2, 1) on eight consecutive elements
// 8g .. 8g+7; m1 = (n + 8g) / 8.
template <bool kS>
__device__ __forceinline__ void fwd_radix8c(u64 *v, int g, const ulonglong2 *tw, const Mod &m)
{
    const int m1 = (kN >> 3) + g;
    {
        const ulonglong2 w = ldtw(tw, m1);
#pragma unroll
        for (int k = 0; k < 4; ++k) ct_bfly<kS>(v[k], v[k + 4], w, m);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const ulonglong2 w = ldtw(tw, 2 * m1 + h);
        ct_bfly<kS>(v[4 * h], v[4 * h + 2], w, m);
        ct_bfly<kS>(v[4 * h + 1], v[4 * h + 3], w, m);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) ct_bfly<kS>(v[2 * k], v[2 * k + 1], ldtw(tw, 4 * m1 + k), m);
}

template <bool kS>
__device__ __forceinline__ void inv_radix8c(u64 *v, int g, const ulonglong2 *tw, const Mod &m)
{
    const int m1 = (kN >> 3) + g;
#pragma unroll
    for (int k = 0; k < 4; ++k) gs_bfly<kS>(v[2 * k], v[2 * k + 1], ldtw(tw, 4 * m1 + k), m);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const ulonglong2 w = ldtw(tw, 2 * m1 + h);
        gs_bfly<kS>(v[4 * h], v[4 * h + 2], w, m);
        gs_bfly<kS>(v[4 * h + 1], v[4 * h + 3], w, m);
    }
    const ulonglong2 w = ldtw(tw, m1);
#pragma unroll
    for (int k = 0; k < 4; ++k) gs_bfly<kS>(v[k], v[k + 4], w, m);
}

// Four inverse stages (half-sizes S, 2S, 4S, 8S).  kLast folds n^-1 into the
// final stage (half-size n/2): tw[0] holds psi^-brv(1) n^-1.
template <bool kS, bool kLast>
__device__ __forceinline__ void inv_radix16(u64 v[16], int m1, const ulonglong2 *tw, const Mod &m,
                                            u64 ninv, u64 ninvp)
{
#pragma unroll
    for (int g = 0; g < 8; ++g) gs_bfly<kS>(v[2 * g], v[2 * g + 1], ldtw(tw, 8 * m1 + g), m);
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const ulonglong2 w = ldtw(tw, 4 * m1 + g);
        gs_bfly<kS>(v[4 * g], v[4 * g + 2], w, m);
        gs_bfly<kS>(v[4 * g + 1], v[4 * g + 3], w, m);
    }
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        const ulonglong2 w = ldtw(tw, 2 * m1 + g);
#pragma unroll
        for (int k = 0; k < 4; ++k) gs_bfly<kS>(v[8 * g + k], v[8 * g + k + 4], w, m);
    }
    if (kLast) {
        const ulonglong2 w = ldtw(tw, 0);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const u64 x = v[k], y = v[k + 8];
            v[k] = shoup4<kS>(x + y, ninv, ninvp, m.q, m.delta);
            v[k + 8] = shoup4<kS>(x - y + m.q4, w.x, w.y, m.q, m.delta);
        }
    } else {
        const ulonglong2 w = ldtw(tw, m1);
#pragma unroll
        for (int k = 0; k < 8; ++k) gs_bfly<kS>(v[k], v[k + 8], w, m);
    }
}

// Full reduction of a lazy value v < 8q (forward) or v < 4q (inverse).  For q = 2^60 - delta with
// delta < 2^32: v = k 2^60 + (v mod 2^60) with k = v >> 60 < 8, and 2^60 = delta (mod q), so
// r = (v mod 2^60) + k delta < 2^60 + 2^35 < 2q is congruent to v and one conditional subtraction
// finishes (one shift, one mask and one 32 x 32 multiply-add in place of a chain of subtractions).
template <bool kS, int kRange>
__device__ __forceinline__ u64 reduce_lazy(u64 v, const Mod &m)
{
    if (kS) {
        const uint32_t k = (uint32_t)(v >> 60);
        u64 r;
        asm("mad.wide.u32 %0, %1, %2, %3;" : "=l"(r) : "r"(k), "r"((uint32_t)m.delta), "l"(v & ((1ull << 60) - 1)));
        return csub(r, m.q);
    }
    if (kRange == 8) v = csub(v, m.q4);
    return csub(csub(v, m.q2), m.q);
}

// Element index held in register k by thread `t` in each of the three passes.
struct IdxA { __device__ static __forceinline__ int at(int t, int k) { return t + 128 * k; } };
struct IdxB { __device__ static __forceinline__ int at(int t, int k) { return (t >> 3) * 128 + (t & 7) + 8 * k; } };
struct IdxC { __device__ static __forceinline__ int at(int t, int k) { return 8 * (t + 128 * (k >> 3)) + (k & 7); } };

template <class F, class G>
__device__ __forceinline__ void exchange(u64 v[16], u64 *buf, int tid)
{
#pragma unroll
    for (int k = 0; k < 16; ++k) buf[swz(F::at(tid, k))] = v[k];
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; ++k) v[k] = buf[swz(G::at(tid, k))];
}

template <class Job, bool kS>
__global__ void __launch_bounds__(kNttThreads, 4) ntt_fwd_kernel(Job job, Tables T, int per_block)
{
    __shared__ u64 sm[2][kN];
    const int tid = threadIdx.x;
    const int j0 = blockIdx.x * per_block;
    for (int jj = 0; jj < per_block; ++jj) {
        const int j = j0 + jj;
        if (j >= job.count) break;
        const typename Job::Ref r = job.ref(j);
        const PrimeConst &pc = T.pc[r.prime];
        const Mod m{pc.q, pc.two_q, 2 * pc.two_q, pc.delta};
        const ulonglong2 *tw = T.tw_fwd + (size_t)r.prime * kN;
        u64 v[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) v[k] = job.load(r, IdxA::at(tid, k));
        fwd_radix16<kS>(v, 1, tw, m);
        exchange<IdxA, IdxB>(v, sm[0], tid);
        fwd_radix16<kS>(v, 16 + (tid >> 3), tw, m);
        exchange<IdxB, IdxC>(v, sm[1], tid);
        fwd_radix8c<kS>(v, tid, tw, m);
        fwd_radix8c<kS>(v + 8, tid + 128, tw, m);
#pragma unroll
        for (int k = 0; k < 16; ++k) v[k] = reduce_lazy<kS, 8>(v[k], m);
        job.store4(r, 8 * tid, v);
        job.store4(r, 8 * tid + 4, v + 4);
        job.store4(r, 8 * (tid + 128), v + 8);
        job.store4(r, 8 * (tid + 128) + 4, v + 12);
        if (jj + 1 < per_block) __syncthreads();
    }
}

template <class Job, bool kS>
__global__ void __launch_bounds__(kNttThreads, 4) ntt_inv_kernel(Job job, Tables T, int per_block)
{
    __shared__ u64 sm[2][kN];
    const int tid = threadIdx.x;
    const int j0 = blockIdx.x * per_block;
    for (int jj = 0; jj < per_block; ++jj) {
        const int j = j0 + jj;
        if (j >= job.count) break;
        const typename Job::Ref r = job.ref(j);
        const PrimeConst &pc = T.pc[r.prime];
        const Mod m{pc.q, pc.two_q, 2 * pc.two_q, pc.delta};
        const ulonglong2 *tw = T.tw_inv + (size_t)r.prime * kN;
        u64 v[16];
        job.load4(r, 8 * tid, v);
        job.load4(r, 8 * tid + 4, v + 4);
        job.load4(r, 8 * (tid + 128), v + 8);
        job.load4(r, 8 * (tid + 128) + 4, v + 12);
        inv_radix8c<kS>(v, tid, tw, m);
        inv_radix8c<kS>(v + 8, tid + 128, tw, m);
        exchange<IdxC, IdxB>(v, sm[0], tid);
        inv_radix16<kS, false>(v, 16 + (tid >> 3), tw, m, 0, 0);
        exchange<IdxB, IdxA>(v, sm[1], tid);
        inv_radix16<kS, true>(v, 1, tw, m, pc.ninv, pc.ninvp);
#pragma unroll
        for (int k = 0; k < 16; ++k) job.store(r, IdxA::at(tid, k), reduce_lazy<kS, 4>(v[k], m));
        if (jj + 1 < per_block) __syncthreads();
    }
}

// Jobs per CTA: a few once the count is large, so consecutive jobs of one
// prime reuse its L1-resident twiddles.
inline int ntt_per_block(int count)
{
    const int target = 148 * 4 * 2;
    int per = (count + target - 1) / target;
    return per < 1 ? 1 : (per > 4 ? 4 : per);
}

template <class Job>
inline int launch_ntt_fwd(const Job &job, const Tables &T, cudaStream_t s)
{
    if (job.count <= 0) return CKKS_OK;
    int per = ntt_per_block(job.count);
    int blocks = (job.count + per - 1) / per;
    if (T.special)
        ntt_fwd_kernel<Job, true><<<blocks, kNttThreads, 0, s>>>(job, T, per);
    else
        ntt_fwd_kernel<Job, false><<<blocks, kNttThreads, 0, s>>>(job, T, per);
    CKKS_CHECK_LAUNCH("ntt_fwd_kernel");
    return CKKS_OK;
}

template <class Job>
inline int launch_ntt_inv(const Job &job, const Tables &T, cudaStream_t s)
{
    if (job.count <= 0) return CKKS_OK;
    int per = ntt_per_block(job.count);
    int blocks = (job.count + per - 1) / per;
    if (T.special)
        ntt_inv_kernel<Job, true><<<blocks, kNttThreads, 0, s>>>(job, T, per);
    else
        ntt_inv_kernel<Job, false><<<blocks, kNttThreads, 0, s>>>(job, T, per);
    CKKS_CHECK_LAUNCH("ntt_inv_kernel");
    return CKKS_OK;
}

// ---------------------------------------------------------------- plain batched job
// x[batch][limbs][n], limb l with prime limb_begin + l.  Jobs are ordered
// limb-major (all batch entries of one limb are consecutive).
struct BatchJob {
    u64 *x;
    int limbs, batch, limb_begin, count;
    struct Ref {
        u64 *row;
        int prime;
    };
    __device__ __forceinline__ Ref ref(int j) const
    {
        const int l = j / batch, b = j - l * batch;
        return {x + ((size_t)b * limbs + l) * kN, limb_begin + l};
    }
    __device__ __forceinline__ u64 load(const Ref &r, int e) const { return r.row[e]; }
    __device__ __forceinline__ void store4(const Ref &r, int e, const u64 *v) const
    {
        ulonglong2 *d = reinterpret_cast<ulonglong2 *>(r.row + e);
        d[0] = make_ulonglong2(v[0], v[1]);
        d[1] = make_ulonglong2(v[2], v[3]);
    }
    __device__ __forceinline__ void load4(const Ref &r, int e, u64 *v) const
    {
        const ulonglong2 *s = reinterpret_cast<const ulonglong2 *>(r.row + e);
        ulonglong2 a = s[0], b = s[1];
        v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
    }
    __device__ __forceinline__ void store(const Ref &r, int e, u64 v) const { r.row[e] = v; }
};

__device__ __forceinline__ void ld4(const u64 *p, u64 *v)
{
    const ulonglong2 *s = reinterpret_cast<const ulonglong2 *>(p);
    ulonglong2 a = s[0], b = s[1];
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}

__device__ __forceinline__ void st4(u64 *p, const u64 *v)
{
    ulonglong2 *d = reinterpret_cast<ulonglong2 *>(p);
    d[0] = make_ulonglong2(v[0], v[1]);
    d[1] = make_ulonglong2(v[2], v[3]);
}

}  // namespace ckks
