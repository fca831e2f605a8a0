// Limb-batched negacyclic NTT / INTT for n = 2048 with 60-bit primes.
//
// One CTA of 256 threads transforms one limb-polynomial at a time (and loops
// over a few consecutive jobs of the same prime, so its twiddles stay in L1).
// Each thread holds 8 coefficients in registers; the 11 butterfly stages run
// as three radix-8 passes and one double radix-4 pass, with the data
// exchanged between passes through a swizzled 32 KiB shared-memory tile
// (two alternating 16 KiB buffers), so every exchange is bank-conflict free.
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
//   __device__ int prime(int j) const;          prime index of job j
//   fwd:  __device__ u64  load(int j, int e)    element e (value < 8q)
//         __device__ void store4(int j, int e, const u64 v[4])   e % 4 == 0
//   inv:  __device__ void load4(int j, int e, u64 v[4])           values < 4q
//         __device__ void store(int j, int e, u64 v)
#pragma once

#include "common.cuh"

namespace ckks {

constexpr int kNttThreads = 256;

// Shared-memory swizzle: flips bits 0..3 of the element index by bits 4..6,
// which makes all four access patterns of the passes conflict free for
// 64-bit words.
__device__ __forceinline__ int swz(int e) { return e ^ ((e >> 4) & 3) ^ (((e >> 5) & 3) << 2); }

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

// Three forward stages (half-sizes 4S, 2S, S) on v[k] = a[base + r + S k],
// base a multiple of 8S; m1 = (n + base) / (8S).
template <bool kS>
__device__ __forceinline__ void fwd_radix8(u64 v[8], int m1, const ulonglong2 *tw, const Mod &m)
{
    const ulonglong2 w = ldtw(tw, m1);
#pragma unroll
    for (int k = 0; k < 4; ++k) ct_bfly<kS>(v[k], v[k + 4], w, m);
    const ulonglong2 w0 = ldtw(tw, 2 * m1), w1 = ldtw(tw, 2 * m1 + 1);
    ct_bfly<kS>(v[0], v[2], w0, m);
    ct_bfly<kS>(v[1], v[3], w0, m);
    ct_bfly<kS>(v[4], v[6], w1, m);
    ct_bfly<kS>(v[5], v[7], w1, m);
#pragma unroll
    for (int k = 0; k < 4; ++k) ct_bfly<kS>(v[2 * k], v[2 * k + 1], ldtw(tw, 4 * m1 + k), m);
}

// Two forward stages (half-sizes 2, 1) on four consecutive elements 4g..4g+3.
template <bool kS>
__device__ __forceinline__ void fwd_radix4(u64 *v, int g, const ulonglong2 *tw, const Mod &m)
{
    const int m1 = (kN >> 2) + g;
    const ulonglong2 w = ldtw(tw, m1);
    ct_bfly<kS>(v[0], v[2], w, m);
    ct_bfly<kS>(v[1], v[3], w, m);
    ct_bfly<kS>(v[0], v[1], ldtw(tw, 2 * m1), m);
    ct_bfly<kS>(v[2], v[3], ldtw(tw, 2 * m1 + 1), m);
}

template <bool kS>
__device__ __forceinline__ void inv_radix4(u64 *v, int g, const ulonglong2 *tw, const Mod &m)
{
    const int m1 = (kN >> 2) + g;
    gs_bfly<kS>(v[0], v[1], ldtw(tw, 2 * m1), m);
    gs_bfly<kS>(v[2], v[3], ldtw(tw, 2 * m1 + 1), m);
    const ulonglong2 w = ldtw(tw, m1);
    gs_bfly<kS>(v[0], v[2], w, m);
    gs_bfly<kS>(v[1], v[3], w, m);
}

// Three inverse stages (half-sizes S, 2S, 4S).  kLast folds n^-1 into the
// final stage (half-size n/2): tw[0] holds psi^-brv(1) n^-1.
template <bool kS, bool kLast>
__device__ __forceinline__ void inv_radix8(u64 v[8], int m1, const ulonglong2 *tw, const Mod &m,
                                           u64 ninv, u64 ninvp)
{
#pragma unroll
    for (int k = 0; k < 4; ++k) gs_bfly<kS>(v[2 * k], v[2 * k + 1], ldtw(tw, 4 * m1 + k), m);
    const ulonglong2 w0 = ldtw(tw, 2 * m1), w1 = ldtw(tw, 2 * m1 + 1);
    gs_bfly<kS>(v[0], v[2], w0, m);
    gs_bfly<kS>(v[1], v[3], w0, m);
    gs_bfly<kS>(v[4], v[6], w1, m);
    gs_bfly<kS>(v[5], v[7], w1, m);
    if (kLast) {
        const ulonglong2 w = ldtw(tw, 0);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const u64 x = v[k], y = v[k + 4];
            v[k] = shoup4<kS>(x + y, ninv, ninvp, m.q, m.delta);
            v[k + 4] = shoup4<kS>(x - y + m.q4, w.x, w.y, m.q, m.delta);
        }
    } else {
        const ulonglong2 w = ldtw(tw, m1);
#pragma unroll
        for (int k = 0; k < 4; ++k) gs_bfly<kS>(v[k], v[k + 4], w, m);
    }
}

// Element index held in register k by thread `tid` in each of the four passes.
struct IdxA { __device__ static __forceinline__ int at(int t, int k) { return t + 256 * k; } };
struct IdxB { __device__ static __forceinline__ int at(int t, int k) { return (t >> 5) * 256 + (t & 31) + 32 * k; } };
struct IdxC { __device__ static __forceinline__ int at(int t, int k) { return (t >> 2) * 32 + (t & 3) + 4 * k; } };
struct IdxD { __device__ static __forceinline__ int at(int t, int k) { return 4 * (t + 256 * (k >> 2)) + (k & 3); } };

template <class F, class G>
__device__ __forceinline__ void exchange(u64 v[8], u64 *buf, int tid)
{
#pragma unroll
    for (int k = 0; k < 8; ++k) buf[swz(F::at(tid, k))] = v[k];
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = buf[swz(G::at(tid, k))];
}

template <class Job, bool kS>
__global__ void __launch_bounds__(kNttThreads) ntt_fwd_kernel(Job job, Tables T, int per_block)
{
    __shared__ u64 sm[2][kN];
    const int tid = threadIdx.x;
    const int j0 = blockIdx.x * per_block;
    for (int jj = 0; jj < per_block; ++jj) {
        const int j = j0 + jj;
        if (j >= job.count) break;
        const int p = job.prime(j);
        const PrimeConst &pc = T.pc[p];
        const Mod m{pc.q, pc.two_q, 2 * pc.two_q, pc.delta};
        const ulonglong2 *tw = T.tw_fwd + (size_t)p * kN;
        u64 v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = job.load(j, IdxA::at(tid, k));
        fwd_radix8<kS>(v, 1, tw, m);
        exchange<IdxA, IdxB>(v, sm[0], tid);
        fwd_radix8<kS>(v, 8 + (tid >> 5), tw, m);
        exchange<IdxB, IdxC>(v, sm[1], tid);
        fwd_radix8<kS>(v, 64 + (tid >> 2), tw, m);
        exchange<IdxC, IdxD>(v, sm[0], tid);
        fwd_radix4<kS>(v, tid, tw, m);
        fwd_radix4<kS>(v + 4, tid + 256, tw, m);
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = csub(csub(csub(v[k], m.q4), m.q2), m.q);
        job.store4(j, 4 * tid, v);
        job.store4(j, 4 * (tid + 256), v + 4);
        if (jj + 1 < per_block) __syncthreads();
    }
}

template <class Job, bool kS>
__global__ void __launch_bounds__(kNttThreads) ntt_inv_kernel(Job job, Tables T, int per_block)
{
    __shared__ u64 sm[2][kN];
    const int tid = threadIdx.x;
    const int j0 = blockIdx.x * per_block;
    for (int jj = 0; jj < per_block; ++jj) {
        const int j = j0 + jj;
        if (j >= job.count) break;
        const int p = job.prime(j);
        const PrimeConst &pc = T.pc[p];
        const Mod m{pc.q, pc.two_q, 2 * pc.two_q, pc.delta};
        const ulonglong2 *tw = T.tw_inv + (size_t)p * kN;
        u64 v[8];
        job.load4(j, 4 * tid, v);
        job.load4(j, 4 * (tid + 256), v + 4);
        inv_radix4<kS>(v, tid, tw, m);
        inv_radix4<kS>(v + 4, tid + 256, tw, m);
        exchange<IdxD, IdxC>(v, sm[0], tid);
        inv_radix8<kS, false>(v, 64 + (tid >> 2), tw, m, 0, 0);
        exchange<IdxC, IdxB>(v, sm[1], tid);
        inv_radix8<kS, false>(v, 8 + (tid >> 5), tw, m, 0, 0);
        exchange<IdxB, IdxA>(v, sm[0], tid);
        inv_radix8<kS, true>(v, 1, tw, m, pc.ninv, pc.ninvp);
#pragma unroll
        for (int k = 0; k < 8; ++k) job.store(j, IdxA::at(tid, k), csub(csub(v[k], m.q2), m.q));
        if (jj + 1 < per_block) __syncthreads();
    }
}

// Jobs per CTA: enough CTAs for several waves on 148 SMs, a few jobs each
// once the count is large so that consecutive jobs reuse L1-resident twiddles.
inline int ntt_per_block(int count)
{
    const int target = 148 * 6 * 4;
    int per = (count + target - 1) / target;
    return per < 1 ? 1 : (per > 8 ? 8 : per);
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
    __device__ __forceinline__ u64 *row(int j) const
    {
        const int l = j / batch, b = j - l * batch;
        return x + ((size_t)b * limbs + l) * kN;
    }
    __device__ __forceinline__ int prime(int j) const { return limb_begin + j / batch; }
    __device__ __forceinline__ u64 load(int j, int e) const { return row(j)[e]; }
    __device__ __forceinline__ void store4(int j, int e, const u64 *v) const
    {
        ulonglong2 *d = reinterpret_cast<ulonglong2 *>(row(j) + e);
        d[0] = make_ulonglong2(v[0], v[1]);
        d[1] = make_ulonglong2(v[2], v[3]);
    }
    __device__ __forceinline__ void load4(int j, int e, u64 *v) const
    {
        const ulonglong2 *s = reinterpret_cast<const ulonglong2 *>(row(j) + e);
        ulonglong2 a = s[0], b = s[1];
        v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
    }
    __device__ __forceinline__ void store(int j, int e, u64 v) const { row(j)[e] = v; }
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
