// Hybrid key switching: ModUp, key inner product, ModDown, and the key
// switch / hoisted rotation entry points built from them.
//
// The pages name the operations (RNS basis conversion as the core of the
// coeff<->slot transforms, Kestrel engine write-up, section 3 table; rotation
// = transform + key switch and relinearisation with an evaluation key,
// EncryptedLLM GPU article, section 2.5; the basis-conversion index mapping as
// the error-prone GPU kernel, same article, section 3.4) but not their
// formulas.  This file implements the standard full-RNS hybrid method with
// contiguous digits: approximate ModUp without overflow correction, floor
// ModDown, and rotation with ModUp hoisted before the automorphism.
//
// Kernels:
//  - INTT of the input limbs with the digit copy and the factor
//    [(Q_j/q_i)^-1]_{q_i} fused into its load/store (ntt.cuh);
//  - the basis-conversion product out_t = sum_s y_s M[s][t], a (targets x
//    sources) x (sources x coefficients) matrix product reduced once per
//    output: conv_kernel below on the integer pipes (exact 128-bit
//    accumulation), or conv_tc_kernel (conv_tc.cu) on the int8 tensor cores,
//    as the context's conversion engine selects;
//  - forward NTT of the new limbs in place;
//  - key_inner_kernel: the dnum-term inner product with the key, the Galois
//    permutation applied as a gather on the digit load;
//  - ModDown: INTT of the special limbs (times [(P/p_k)^-1]), conversion,
//    forward NTT whose store computes (acc - conv) P^-1 and any fused extra
//    term (phi_g(c0) for a rotation, the tensor terms for relinearisation).
#include <algorithm>

#include "internal.cuh"
#include "ntt.cuh"
#include "split.cuh"

namespace ckks {

// ---------------------------------------------------------------- basis conversion
constexpr int kConvThreads = 128;
constexpr int kConvTT = 8;  // targets per thread (and per CTA)

template <class Map>
__global__ void __launch_bounds__(kConvThreads) conv_kernel(Map m, const PrimeConst *__restrict__ pc)
{
    __shared__ __align__(16) u64 msm[kMaxDigit * kConvTT];
    const int z = blockIdx.z;
    const int S = m.sources(z), T = m.targets(z);
    const int t0 = blockIdx.y * kConvTT;
    if (t0 >= T) return;
    for (int i = threadIdx.x; i < S * kConvTT; i += kConvThreads) {
        const int s = i / kConvTT, tt = i - s * kConvTT;
        msm[i] = (t0 + tt < T) ? m.mat(z, s, t0 + tt) : 0;
    }
    __syncthreads();
    const int c = blockIdx.x * kConvThreads + threadIdx.x;
    const u64 *y = m.src(z) + c;
    u64 hi[kConvTT], lo[kConvTT];
#pragma unroll
    for (int tt = 0; tt < kConvTT; ++tt) hi[tt] = lo[tt] = 0;
    for (int s = 0; s < S; ++s) {
        const u64 ys = __ldg(y + (size_t)s * kN);
        const u64 *mr = msm + s * kConvTT;
#pragma unroll
        for (int tt = 0; tt < kConvTT; ++tt) mac128(hi[tt], lo[tt], ys, mr[tt]);
    }
#pragma unroll
    for (int tt = 0; tt < kConvTT; ++tt) {
        const int ti = t0 + tt;
        if (ti < T) m.dst(z, ti)[c] = reduce128(hi[tt], lo[tt], pc[m.prime(z, ti)]);
    }
}

// ModUp conversion: job z = (b, digit jd); sources are the digit's primes,
// targets every other prime (ciphertext and special), in index order.
struct UpConvMap {
    const u64 *y;
    u64 *digits;
    const u64 *matp;
    int L, LK, alpha, dnum;
    __device__ __forceinline__ int lo(int z) const { return (z % dnum) * alpha; }
    __device__ __forceinline__ int sources(int z) const { return min(alpha, L - lo(z)); }
    __device__ __forceinline__ int targets(int z) const { return LK - sources(z); }
    __device__ __forceinline__ const u64 *src(int z) const
    {
        return y + ((size_t)(z / dnum) * L + lo(z)) * kN;
    }
    __device__ __forceinline__ int prime(int z, int ti) const
    {
        const int l = lo(z);
        return ti < l ? ti : ti + sources(z);
    }
    __device__ __forceinline__ u64 mat(int z, int s, int ti) const
    {
        return matp[(size_t)((z % dnum) * alpha + s) * LK + prime(z, ti)];
    }
    __device__ __forceinline__ u64 *dst(int z, int ti) const
    {
        return digits + ((size_t)z * LK + prime(z, ti)) * kN;
    }
};

// ModDown conversion: job z = (J, component); sources the K special primes,
// targets the L ciphertext primes.
struct DownConvMap {
    const u64 *zsrc;
    u64 *cv;
    const u64 *matp;
    int L, K;
    __device__ __forceinline__ int sources(int) const { return K; }
    __device__ __forceinline__ int targets(int) const { return L; }
    __device__ __forceinline__ const u64 *src(int z) const { return zsrc + (size_t)z * K * kN; }
    __device__ __forceinline__ int prime(int, int ti) const { return ti; }
    __device__ __forceinline__ u64 mat(int, int s, int ti) const { return matp[(size_t)s * L + ti]; }
    __device__ __forceinline__ u64 *dst(int z, int ti) const { return cv + ((size_t)z * L + ti) * kN; }
};

template <class Map>
static int launch_conv(const Map &m, int max_targets, int jobs, const Tables &T, cudaStream_t s)
{
    if (jobs <= 0 || max_targets <= 0) return CKKS_OK;
    dim3 grid(kN / kConvThreads, (max_targets + kConvTT - 1) / kConvTT, jobs);
    conv_kernel<Map><<<grid, kConvThreads, 0, s>>>(m, T.pc);
    CKKS_CHECK_LAUNCH("conv_kernel");
    return CKKS_OK;
}

// modraise conversion: job z = polynomial; sources its l Garner digits and the
// sign row; targets the primes l..L-1.  matp[s][t] = [q_0..q_{s-1}]_{q_t} for
// s < l and [-Q]_{q_t} for s = l, so the exact sum is the centred lift.
struct RaiseConvMap {
    const u64 *dg;
    u64 *out;
    const u64 *matp;  // [l+1][L]
    int l, L;
    __device__ __forceinline__ int sources(int) const { return l + 1; }
    __device__ __forceinline__ int targets(int) const { return L - l; }
    __device__ __forceinline__ const u64 *src(int z) const { return dg + (size_t)z * (l + 1) * kN; }
    __device__ __forceinline__ u64 mat(int, int s, int t) const { return matp[(size_t)s * L + l + t]; }
    __device__ __forceinline__ u64 *dst(int z, int t) const { return out + ((size_t)z * L + l + t) * kN; }
    __device__ __forceinline__ int prime(int, int t) const { return l + t; }
};

int raise_conv(const Tables &T, const u64 *dg, u64 *out, const u64 *matp, int l, int P, cudaStream_t s)
{
    RaiseConvMap m{dg, out, matp, l, T.L};
    return launch_conv(m, T.L - l, P, T, s);
}

// ---------------------------------------------------------------- ModUp
// INTT of source limb i of polynomial b; the load also writes the input limb
// (NTT domain) into its own digit, the store multiplies by [(Q_j/q_i)^-1].
template <bool kProduct>
struct UpInttJob {
    const u64 *in, *in2;
    size_t in_bstride;
    u64 *digits, *y;
    const ulonglong2 *hatinv;
    const PrimeConst *pc;
    int L, LK, alpha, dnum, batch, count;
    struct Ref {
        const u64 *src, *src2;
        u64 *copy, *yrow;
        ulonglong2 h;
        u64 q;
        int prime;
    };
    __device__ __forceinline__ Ref ref(int j) const
    {
        const int i = j / batch, b = j - i * batch;
        const size_t off = (size_t)b * in_bstride + (size_t)i * kN;
        Ref r;
        r.src = in + off;
        r.src2 = kProduct ? in2 + off : nullptr;
        r.copy = digits ? digits + (((size_t)b * dnum + i / alpha) * LK + i) * kN : nullptr;
        r.yrow = y + ((size_t)b * L + i) * kN;
        r.h = hatinv[i];
        r.q = pc[i].q;
        r.prime = i;
        return r;
    }
    __device__ __forceinline__ void load4(const Ref &r, int e, u64 *v) const
    {
        ld4(r.src + e, v);
        if (kProduct) {
            u64 w[4];
            ld4(r.src2 + e, w);
            const PrimeConst c = pc[r.prime];
#pragma unroll
            for (int k = 0; k < 4; ++k) v[k] = mulmod(v[k], w[k], c);
        }
        if (r.copy) st4(r.copy + e, v);
    }
    __device__ __forceinline__ void store(const Ref &r, int e, u64 v) const
    {
        r.yrow[e] = shoup(v, r.h.x, r.h.y, r.q);
    }
};

// Forward NTT of the converted limbs, in place.  Jobs are ordered by target
// prime: for a ciphertext prime t the dnum-1 digits not containing it, for a
// special prime all dnum digits; batch entries innermost.
struct UpNttJob {
    u64 *digits;
    int L, LK, alpha, dnum, batch, count;
    struct Ref {
        u64 *row;
        int prime;
    };
    __device__ __forceinline__ Ref ref(int j) const
    {
        const int b = j % batch;
        int r = j / batch, t, jd;
        const int per_q = dnum - 1;
        if (r < L * per_q) {
            t = r / per_q;
            const int d = r - t * per_q, own = t / alpha;
            jd = d < own ? d : d + 1;
        } else {
            r -= L * per_q;
            t = L + r / dnum;
            jd = r - (t - L) * dnum;
        }
        return {digits + (((size_t)b * dnum + jd) * LK + t) * kN, t};
    }
    __device__ __forceinline__ u64 load(const Ref &r, int e) const { return r.row[e]; }
    __device__ __forceinline__ void store4(const Ref &r, int e, const u64 *v) const { st4(r.row + e, v); }
};

// Forward NTT of one window's converted limbs: buf[b][j][tw][n] for every digit j but the window's
// own (whose limbs are copies of the input, already in the NTT domain), prime t0 + tw.  Jobs run
// ciphertext fastest, then digit, so consecutive jobs share a prime.
struct WinNttJob {
    u64 *buf;
    int wbuf, t0, n, own, dnum, batch, count;
    struct Ref {
        u64 *row;
        int prime;
    };
    __device__ __forceinline__ Ref ref(int j) const
    {
        const int b = j % batch, ndig = own >= 0 ? dnum - 1 : dnum;
        const int r = j / batch, jj = r % ndig, tw = r / ndig;
        const int jd = own >= 0 && jj >= own ? jj + 1 : jj;
        return {buf + (((size_t)b * dnum + jd) * wbuf + tw) * kN, t0 + tw};
    }
    __device__ __forceinline__ u64 load(const Ref &r, int e) const { return r.row[e]; }
    __device__ __forceinline__ void store4(const Ref &r, int e, const u64 *v) const { st4(r.row + e, v); }
};

size_t modup_ws_bytes(const ckks_ctx *ctx, int batch) { return limbs_bytes((size_t)batch * ctx->L); }

int modup_stage(const ckks_ctx *ctx, const u64 *in, const u64 *in2, size_t in_bstride, u64 *digits,
                int batch, void *ws, cudaStream_t s)
{
    if (batch <= 0) return CKKS_OK;
    const Tables &T = ctx->t;
    Carve cv(ws);
    u64 *y = cv.take<u64>((size_t)batch * T.L * kN);
    if (in2) {
        UpInttJob<true> j{in, in2, in_bstride, digits, y, T.up_hatinv, T.pc,
                          T.L, T.LK, T.alpha, T.dnum, batch, T.L * batch};
        CKKS_TRY(launch_ntt_inv(j, T, s));
    } else {
        UpInttJob<false> j{in, nullptr, in_bstride, digits, y, T.up_hatinv, T.pc,
                           T.L, T.LK, T.alpha, T.dnum, batch, T.L * batch};
        CKKS_TRY(launch_ntt_inv(j, T, s));
    }
    const ConvKind ck = conv_kind(ctx, T.alpha);
    if (ck == kConvFolded) {
        CKKS_TRY(launch_conv_fold_up(const_cast<ckks_ctx *>(ctx), y, digits, batch, s));
    } else if (ck == kConvTensor) {
        CKKS_TRY(launch_conv_tc_up(ctx, y, digits, batch, s));
    } else {
        UpConvMap m{y, digits, T.up_mat, T.L, T.LK, T.alpha, T.dnum};
        CKKS_TRY(launch_conv(m, T.LK - 1, batch * T.dnum, T, s));
    }
    UpNttJob nj{digits, T.L, T.LK, T.alpha, T.dnum, batch, batch * (T.dnum * T.LK - T.L)};
    return launch_ntt_fwd(nj, T, s);
}

// ---------------------------------------------------------------- key inner product
// One thread per output coefficient k of one (prime t, key r) pair and a chunk of up to kB
// ciphertexts b: per digit j it loads the two key words once and the chunk's gathered digit words,
// and keeps 2 kB exact sums (three 64-bit partial sums each in the split form below, taken when
// every prime is 2^60 - delta, whose words arrive by cp.async ki_depth(kB) digits ahead; 128-bit
// sums otherwise).  The 1-D grid is ordered coefficient tile fastest, then key,
// then ciphertext chunk, then prime, so the CTAs that read the same digit rows (all keys of one
// chunk at one prime) run back to back and re-read them from L2.  The Galois permutation is the
// gather on the digit load (it maps each aligned tile of 32 coefficients onto one, so a warp's
// gathered loads stay within one 256-byte segment).
constexpr int kKiB = 4;       // ciphertexts per thread: the 128-bit form, and batches below kKiBWide
constexpr int kKiBWide = 8;   // ciphertexts per thread in the split form from 8 ciphertexts per key
constexpr int kKiThreads = 128;
constexpr int kKiFold = 256;  // digits summed exactly in 128 bits between reductions
// Split form: each thread copies its 2 + kB words of a digit (cp.async, 8 bytes each) into its
// own shared-memory slots ki_depth(kB) digits ahead, so the loads in flight hold no registers.
// Chunks of 4: 8 digits ahead, 48 KiB and 4 CTAs per SM; chunks of 8 (the key's two words split
// once for 8 ciphertexts, more registers): 4 digits ahead, 40 KiB and 3 CTAs per SM.
__host__ __device__ constexpr int ki_depth(int b) { return b == kKiBWide ? 4 : 8; }
__host__ __device__ constexpr int ki_min_blocks(int b) { return b == kKiBWide ? 3 : 4; }
constexpr size_t ki_smem(int b) { return (size_t)ki_depth(b) * (2 + b) * kKiThreads * sizeof(u64); }

// Asynchronous 8-byte copy from global into this thread's shared-memory slot.
__device__ __forceinline__ void kcp8(void *dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" :: "r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
                 : "memory");
}

template <bool kSplit, int kB>
__global__ void __launch_bounds__(kKiThreads, ki_min_blocks(kB)) key_inner_kernel(const u64 *__restrict__ digits, KeyList kl,
                                                        int per_key, int nkeys, int hoisted,
                                                        u64 *__restrict__ acc, Tables T, DigitView dv)
{
    constexpr int kDepth = ki_depth(kB), kSlots = 2 + kB;
    const int nchunks = (per_key + kB - 1) / kB;
    int id = blockIdx.x;
    const int tile = id % (kN / kKiThreads);
    id /= kN / kKiThreads;
    const int r = id % nkeys;
    id /= nkeys;
    const int chunk = id % nchunks;
    const int t = dv.t_lo + id / nchunks;
    const int b0 = chunk * kB, nb = min(kB, per_key - b0);
    const int k = tile * kKiThreads + threadIdx.x;
    const u32 g = kl.galois[r];
    const int src = g == 1u ? k : (int)galois_src((u32)k, g);
    const size_t LKn = (size_t)T.LK * kN;
    const size_t bstride = dv.ct_stride;  // between the digit sets of consecutive ciphertexts
    const u64 *dg = digits + (size_t)(hoisted ? b0 : r * per_key + b0) * bstride + (size_t)(t - dv.t_lo) * kN + src;
    const size_t kLKn = (size_t)T.key_LK * kN;  // key rows per (digit, component)
    const int kt = t < T.L ? t : t - T.L + T.key_L;
    const u64 *kp = kl.key[r] + (size_t)kt * kN + k;
    const PrimeConst pc = T.pc[t];
    if constexpr (kSplit) {
        u64 s0[2][kB], s1[2][kB], s2[2][kB];
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int b = 0; b < kB; ++b) s0[c][b] = s1[c][b] = s2[c][b] = 0;
        const u32 delta = (u32)pc.delta;
        // this thread's slots: word w of digit j at slot[((j % kDepth) kSlots + w) kKiThreads];
        // words 0, 1: the key's two components, 2 + b: ciphertext b's digit word (zero past nb)
        extern __shared__ u64 kism[];
        u64 *const slot = kism + threadIdx.x;
        for (int st = 0; st < kDepth; ++st)
            for (int b = nb; b < kB; ++b) slot[(st * kSlots + 2 + b) * kKiThreads] = 0;
        auto fetch = [&](int j) {  // one commit group per digit, empty past the last
            if (j < T.dnum) {
                u64 *sl = slot + (j % kDepth) * kSlots * kKiThreads;
                kcp8(sl, kp + (size_t)(2 * j) * kLKn);
                kcp8(sl + kKiThreads, kp + (size_t)(2 * j + 1) * kLKn);
                const u64 *dj = dg + (size_t)j * dv.j_stride;
#pragma unroll
                for (int b = 0; b < kB; ++b)
                    if (b < nb) kcp8(sl + (2 + b) * kKiThreads, dj + (size_t)b * bstride);
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
        };
#pragma unroll
        for (int j = 0; j < kDepth; ++j) fetch(j);
        for (int j0 = 0; j0 < T.dnum; j0 += kSplitFold) {
            const int j1 = min(T.dnum, j0 + kSplitFold);
#pragma unroll 2
            for (int j = j0; j < j1; ++j) {
                asm volatile("cp.async.wait_group %0;" :: "n"(kDepth - 1) : "memory");  // digit j is in
                const u64 *sl = slot + (j % kDepth) * kSlots * kKiThreads;
                const u64 kb = sl[0], ka = sl[kKiThreads];
                const Split30 kw[2] = {split30(kb), split30(ka)};
                u64 d[kB];
#pragma unroll
                for (int b = 0; b < kB; ++b) d[b] = sl[(2 + b) * kKiThreads];
#pragma unroll
                for (int b = 0; b < kB; ++b) {
                    const Split30 dw = split30(d[b]);
#pragma unroll
                    for (int c = 0; c < 2; ++c) split_mac(s0[c][b], s1[c][b], s2[c][b], dw, kw[c]);
                }
                fetch(j + kDepth);  // into the slots just read: their values are consumed
            }
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int b = 0; b < kB; ++b) split_fold(s0[c][b], s1[c][b], s2[c][b], delta);
        }
#pragma unroll
        for (int b = 0; b < kB; ++b) {
            if (b < nb) {
                u64 *o = acc + ((size_t)(r * per_key + b0 + b) * 2 * T.LK + t) * kN + k;
                o[0] = split_reduce(s0[0][b], s2[0][b], pc);
                o[LKn] = split_reduce(s0[1][b], s2[1][b], pc);
            }
        }
    } else {
        u64 h0[kB], l0[kB], h1[kB], l1[kB];
#pragma unroll
        for (int b = 0; b < kB; ++b) h0[b] = l0[b] = h1[b] = l1[b] = 0;
        // 256 products below 2^120 plus a folded value below 2^60 stay below
        // 2^128: past 256 digits the sums are reduced once per block of 256
        for (int j0 = 0; j0 < T.dnum; j0 += kKiFold) {
            if (j0 > 0) {
#pragma unroll
                for (int b = 0; b < kB; ++b) {
                    l0[b] = reduce128(h0[b], l0[b], pc);
                    l1[b] = reduce128(h1[b], l1[b], pc);
                    h0[b] = h1[b] = 0;
                }
            }
            const int j1 = min(T.dnum, j0 + kKiFold);
#pragma unroll 4
            for (int j = j0; j < j1; ++j) {
                const u64 kb = __ldg(kp + (size_t)(2 * j) * kLKn), ka = __ldg(kp + (size_t)(2 * j + 1) * kLKn);
                const u64 *dj = dg + (size_t)j * dv.j_stride;
                u64 d[kB];
#pragma unroll
                for (int b = 0; b < kB; ++b) d[b] = b < nb ? __ldg(dj + (size_t)b * bstride) : 0;
#pragma unroll
                for (int b = 0; b < kB; ++b) {
                    mac128(h0[b], l0[b], d[b], kb);
                    mac128(h1[b], l1[b], d[b], ka);
                }
            }
        }
#pragma unroll
        for (int b = 0; b < kB; ++b) {
            if (b < nb) {
                u64 *o = acc + ((size_t)(r * per_key + b0 + b) * 2 * T.LK + t) * kN + k;
                o[0] = reduce128(h0[b], l0[b], pc);
                o[LKn] = reduce128(h1[b], l1[b], pc);
            }
        }
    }
}

int key_inner_stage(const ckks_ctx *ctx, const u64 *digits, const KeyList &kl, int per_key,
                    bool hoisted, u64 *acc, int jobs, cudaStream_t s, const DigitView &dv)
{
    if (jobs <= 0 || dv.nt <= 0) return CKKS_OK;
    const Tables &T = ctx->t;
    const int nkeys = jobs / per_key;
    const bool wide = T.special && per_key >= kKiBWide;
    const int cb = wide ? kKiBWide : kKiB;
    const size_t blocks = (size_t)(kN / kKiThreads) * nkeys * ((per_key + cb - 1) / cb) * dv.nt;
    if (blocks > 0x7fffffffull) return set_error(CKKS_EUNSUPPORTED, "key inner product grid too large");
    if (wide)
        key_inner_kernel<true, kKiBWide><<<(unsigned)blocks, kKiThreads, ki_smem(kKiBWide), s>>>(
            digits, kl, per_key, nkeys, hoisted ? 1 : 0, acc, T, dv);
    else if (T.special)
        key_inner_kernel<true, kKiB><<<(unsigned)blocks, kKiThreads, ki_smem(kKiB), s>>>(
            digits, kl, per_key, nkeys, hoisted ? 1 : 0, acc, T, dv);
    else
        key_inner_kernel<false, kKiB><<<(unsigned)blocks, kKiThreads, 0, s>>>(digits, kl, per_key, nkeys,
                                                                              hoisted ? 1 : 0, acc, T, dv);
    CKKS_CHECK_LAUNCH("key_inner_kernel");
    return CKKS_OK;
}

int key_inner_stage(const ckks_ctx *ctx, const u64 *digits, const KeyList &kl, int per_key,
                    bool hoisted, u64 *acc, int jobs, cudaStream_t s)
{
    const Tables &T = ctx->t;
    const DigitView dv{(size_t)T.dnum * T.LK * kN, (size_t)T.LK * kN, 0, T.LK};
    return key_inner_stage(ctx, digits, kl, per_key, hoisted, acc, jobs, s, dv);
}

// ---------------------------------------------------------------- ModDown
struct DownInttJob {
    const u64 *acc;
    u64 *zdst;
    const ulonglong2 *hatinv;
    const PrimeConst *pc;
    int L, K, LK, jobs2, count;
    struct Ref {
        const u64 *src;
        u64 *dst;
        ulonglong2 h;
        u64 q;
        int prime;
    };
    __device__ __forceinline__ Ref ref(int j) const
    {
        const int k = j / jobs2, zz = j - k * jobs2;
        return {acc + ((size_t)zz * LK + L + k) * kN, zdst + ((size_t)zz * K + k) * kN, hatinv[k],
                pc[L + k].q, L + k};
    }
    __device__ __forceinline__ void load4(const Ref &r, int e, u64 *v) const { ld4(r.src + e, v); }
    __device__ __forceinline__ void store(const Ref &r, int e, u64 v) const
    {
        r.dst[e] = shoup(v, r.h.x, r.h.y, r.q);
    }
};

template <int kKind>
struct DownFinalJob {
    u64 *cv;
    const u64 *acc;
    u64 *out;
    const ulonglong2 *pinv;
    const PrimeConst *pc;
    int L, LK, jobs2, count;
    DownExtra ex;
    struct Ref {
        const u64 *cv, *acc, *c0, *a, *b;
        u64 *out;
        ulonglong2 pv;
        u64 q;
        u32 g;
        int prime, comp;
    };
    __device__ __forceinline__ Ref ref(int j) const
    {
        const int i = j / jobs2, zz = j - i * jobs2;
        const int z = zz >> 1;
        Ref r;
        r.cv = cv + ((size_t)zz * L + i) * kN;
        r.acc = acc + ((size_t)zz * LK + i) * kN;
        r.out = out + ((size_t)zz * L + i) * kN;
        r.pv = pinv[i];
        r.q = pc[i].q;
        r.prime = i;
        r.comp = zz & 1;
        r.c0 = nullptr;
        r.a = r.b = nullptr;
        r.g = 1;
        if (kKind == 1) {
            const int ci = ex.ct_mod ? z % ex.ct_mod : z;
            r.c0 = ex.ct + (size_t)ci * ex.ct_bstride + (size_t)i * kN;
            r.g = ex.gal[z / ex.per];
        }
        if (kKind == 2) {
            const size_t base = (size_t)z * 2 * L * kN + (size_t)i * kN;
            r.a = ex.a + base;
            r.b = ex.b + base;
        }
        return r;
    }
    __device__ __forceinline__ u64 load(const Ref &r, int e) const { return r.cv[e]; }
    __device__ __forceinline__ void store4(const Ref &r, int e, const u64 *v) const
    {
        const u64 q = r.q;
        u64 a[4], o[4];
        ld4(r.acc + e, a);
#pragma unroll
        for (int c = 0; c < 4; ++c) o[c] = shoup(submod(a[c], v[c], q), r.pv.x, r.pv.y, q);
        if (kKind == 1 && r.comp == 0) {
#pragma unroll
            for (int c = 0; c < 4; ++c) o[c] = addmod(o[c], __ldg(r.c0 + galois_src((u32)(e + c), r.g)), q);
        }
        if (kKind == 2) {
            const PrimeConst pcc = pc[r.prime];
            const size_t Ln = (size_t)L * kN;
            u64 a0[4], b0[4], a1[4], b1[4];
            ld4(r.a + e, a0);
            ld4(r.b + e, b0);
            if (r.comp == 0) {
#pragma unroll
                for (int c = 0; c < 4; ++c) o[c] = addmod(o[c], mulmod(a0[c], b0[c], pcc), q);
            } else {
                ld4(r.a + Ln + e, a1);
                ld4(r.b + Ln + e, b1);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    u64 hi = 0, lo = 0;
                    mac128(hi, lo, a0[c], b1[c]);
                    mac128(hi, lo, a1[c], b0[c]);
                    o[c] = addmod(o[c], reduce128(hi, lo, pcc), q);
                }
            }
        }
        st4(r.out + e, o);
    }
};

size_t moddown_ws_bytes(const ckks_ctx *ctx, int jobs)
{
    return limbs_bytes((size_t)jobs * 2 * ctx->K) + limbs_bytes((size_t)jobs * 2 * ctx->L);
}

int moddown_stage(const ckks_ctx *ctx, const u64 *acc, u64 *out, int jobs, const DownExtra &ex,
                  void *ws, cudaStream_t s)
{
    if (jobs <= 0) return CKKS_OK;
    const Tables &T = ctx->t;
    const int jobs2 = 2 * jobs;
    Carve c(ws);
    u64 *zb = c.take<u64>((size_t)jobs2 * T.K * kN);
    u64 *cvb = c.take<u64>((size_t)jobs2 * T.L * kN);
    DownInttJob ij{acc, zb, T.dn_hatinv, T.pc, T.L, T.K, T.LK, jobs2, T.K * jobs2};
    CKKS_TRY(launch_ntt_inv(ij, T, s));
    const ConvKind ck = conv_kind(ctx, T.K);
    if (ck == kConvFolded) {
        CKKS_TRY(launch_conv_fold_down(const_cast<ckks_ctx *>(ctx), zb, cvb, jobs2, s));
    } else if (ck == kConvTensor) {
        CKKS_TRY(launch_conv_tc_down(ctx, zb, cvb, jobs2, s));
    } else {
        DownConvMap m{zb, cvb, T.dn_mat, T.L, T.K};
        CKKS_TRY(launch_conv(m, T.L, jobs2, T, s));
    }
    switch (ex.kind) {
    case 1: {
        DownFinalJob<1> fj{cvb, acc, out, T.dn_pinv, T.pc, T.L, T.LK, jobs2, T.L * jobs2, ex};
        return launch_ntt_fwd(fj, T, s);
    }
    case 2: {
        DownFinalJob<2> fj{cvb, acc, out, T.dn_pinv, T.pc, T.L, T.LK, jobs2, T.L * jobs2, ex};
        return launch_ntt_fwd(fj, T, s);
    }
    default: {
        DownFinalJob<0> fj{cvb, acc, out, T.dn_pinv, T.pc, T.L, T.LK, jobs2, T.L * jobs2, ex};
        return launch_ntt_fwd(fj, T, s);
    }
    }
}

}  // namespace ckks

// ---------------------------------------------------------------- entry points
using namespace ckks;

namespace {

int check_batch(int batch)
{
    if (batch < 0) return set_error(CKKS_EINVAL, "negative batch");
    if (batch > 65535) return set_error(CKKS_EUNSUPPORTED, "batch above 65535");
    return CKKS_OK;
}

size_t keyswitch_ws(const ckks_ctx *ctx, int batch)
{
    return limbs_bytes((size_t)batch * ctx->dnum * (ctx->L + ctx->K)) +
           limbs_bytes((size_t)batch * 2 * (ctx->L + ctx->K)) +
           std::max(modup_ws_bytes(ctx, batch), moddown_ws_bytes(ctx, batch));
}

size_t rotate_ws(const ckks_ctx *ctx, int batch, int nkeys)
{
    const int chunk = std::min(std::max(nkeys, 1), kMaxKeys);
    return limbs_bytes((size_t)batch * ctx->dnum * (ctx->L + ctx->K)) +
           limbs_bytes((size_t)chunk * batch * 2 * (ctx->L + ctx->K)) +
           std::max(modup_ws_bytes(ctx, batch), moddown_ws_bytes(ctx, chunk * batch));
}

constexpr int kLanes = 2;  // streams the windows of a streamed rotation alternate between

// ModUp's sources y, one window buffer per lane, the accumulators of a key chunk and ModDown's
// scratch.
size_t rotate_streamed_ws(const ckks_ctx *ctx, int batch, int nkeys)
{
    const int chunk = std::min(std::max(nkeys, 1), kMaxKeys);
    return limbs_bytes((size_t)batch * ctx->L) + kLanes * limbs_bytes((size_t)batch * ctx->dnum * kWinMax) +
           limbs_bytes((size_t)chunk * batch * 2 * (ctx->L + ctx->K)) + moddown_ws_bytes(ctx, chunk * batch);
}

}  // namespace

namespace ckks {
size_t keyswitch_ws_bytes(const ckks_ctx *ctx, int batch) { return keyswitch_ws(ctx, batch); }
size_t rotate_ws_bytes(const ckks_ctx *ctx, int batch, int nkeys) { return rotate_ws(ctx, batch, nkeys); }
size_t rotate_streamed_ws_bytes(const ckks_ctx *ctx, int batch, int nkeys)
{
    return rotate_streamed_ws(ctx, batch, nkeys);
}
}  // namespace ckks

extern "C" int ckks_modup(const ckks_ctx *ctx, const uint64_t *c_ntt, uint64_t *digits, int batch,
                          void *ws, ckks_stream_t stream)
{
    CKKS_TRY(check_ctx(ctx));
    CKKS_TRY(check_batch(batch));
    if (batch == 0) return CKKS_OK;
    CKKS_TRY(check_ptr(c_ntt, "c_ntt"));
    CKKS_TRY(check_ptr(digits, "digits"));
    CKKS_TRY(set_device(ctx));
    void *w;
    ckks_ctx *mctx = const_cast<ckks_ctx *>(ctx);
    CKKS_TRY(resolve_ws(mctx, ws, modup_ws_bytes(ctx, batch), &w));
    return modup_stage(ctx, c_ntt, nullptr, (size_t)ctx->L * kN, digits, batch, w,
                       (cudaStream_t)stream);
}

extern "C" int ckks_key_inner(const ckks_ctx *ctx, const uint64_t *digits, const uint64_t *key,
                              uint32_t galois, uint64_t *acc, int batch, ckks_stream_t stream)
{
    CKKS_TRY(check_ctx(ctx));
    CKKS_TRY(check_batch(batch));
    if ((galois & 1u) == 0) return set_error(CKKS_EINVAL, "galois element must be odd");
    if (batch == 0) return CKKS_OK;
    CKKS_TRY(check_ptr(digits, "digits"));
    CKKS_TRY(check_ptr(key, "key"));
    CKKS_TRY(check_ptr(acc, "acc"));
    CKKS_TRY(set_device(ctx));
    KeyList kl{};
    kl.key[0] = key;
    kl.galois[0] = galois & (2u * kN - 1u);
    return key_inner_stage(ctx, digits, kl, batch, true, acc, batch, (cudaStream_t)stream);
}

extern "C" int ckks_moddown(const ckks_ctx *ctx, const uint64_t *acc, uint64_t *out, int batch,
                            void *ws, ckks_stream_t stream)
{
    CKKS_TRY(check_ctx(ctx));
    CKKS_TRY(check_batch(batch));
    if (batch == 0) return CKKS_OK;
    CKKS_TRY(check_ptr(acc, "acc"));
    CKKS_TRY(check_ptr(out, "out"));
    CKKS_TRY(set_device(ctx));
    void *w;
    CKKS_TRY(resolve_ws(const_cast<ckks_ctx *>(ctx), ws, moddown_ws_bytes(ctx, batch), &w));
    DownExtra ex;
    return moddown_stage(ctx, acc, out, batch, ex, w, (cudaStream_t)stream);
}

extern "C" int ckks_keyswitch(const ckks_ctx *ctx, const uint64_t *d, const uint64_t *key,
                              uint64_t *out, int batch, void *ws, ckks_stream_t stream)
{
    CKKS_TRY(check_ctx(ctx));
    CKKS_TRY(check_batch(batch));
    if (batch == 0) return CKKS_OK;
    CKKS_TRY(check_ptr(d, "d"));
    CKKS_TRY(check_ptr(key, "key"));
    CKKS_TRY(check_ptr(out, "out"));
    CKKS_TRY(set_device(ctx));
    void *w;
    CKKS_TRY(resolve_ws(const_cast<ckks_ctx *>(ctx), ws, keyswitch_ws(ctx, batch), &w));
    const cudaStream_t s = (cudaStream_t)stream;
    const int LK = ctx->L + ctx->K;
    Carve c(w);
    u64 *digits = c.take<u64>((size_t)batch * ctx->dnum * LK * kN);
    u64 *acc = c.take<u64>((size_t)batch * 2 * LK * kN);
    void *scratch = c.base + c.off;
    CKKS_TRY(modup_stage(ctx, d, nullptr, (size_t)ctx->L * kN, digits, batch, scratch, s));
    KeyList kl{};
    kl.key[0] = key;
    kl.galois[0] = 1;
    CKKS_TRY(key_inner_stage(ctx, digits, kl, batch, true, acc, batch, s));
    DownExtra ex;
    return moddown_stage(ctx, acc, out, batch, ex, scratch, s);
}

extern "C" int ckks_rotate(const ckks_ctx *ctx, const uint64_t *ct, const uint64_t *const *keys,
                           const uint32_t *galois, int nkeys, uint64_t *out, int batch, void *ws,
                           ckks_stream_t stream)
{
    CKKS_TRY(check_ctx(ctx));
    CKKS_TRY(check_batch(batch));
    if (nkeys < 0) return set_error(CKKS_EINVAL, "negative key count");
    if (batch == 0 || nkeys == 0) return CKKS_OK;
    if (!keys || !galois) return set_error(CKKS_EINVAL, "null key or galois array");
    for (int r = 0; r < nkeys; ++r) {
        CKKS_TRY(check_ptr(keys[r], "keys[r]"));
        if ((galois[r] & 1u) == 0) return set_error(CKKS_EINVAL, "galois element must be odd");
    }
    if ((size_t)nkeys * batch > 32767) return set_error(CKKS_EUNSUPPORTED, "nkeys * batch above 32767");
    CKKS_TRY(check_ptr(ct, "ct"));
    CKKS_TRY(check_ptr(out, "out"));
    CKKS_TRY(set_device(ctx));
    void *w;
    CKKS_TRY(resolve_ws(const_cast<ckks_ctx *>(ctx), ws, rotate_ws(ctx, batch, nkeys), &w));
    const cudaStream_t s = (cudaStream_t)stream;
    const int L = ctx->L, LK = L + ctx->K;
    const size_t ct_elems = (size_t)2 * L * kN;
    const int chunk = std::min(nkeys, kMaxKeys);
    Carve c(w);
    u64 *digits = c.take<u64>((size_t)batch * ctx->dnum * LK * kN);
    u64 *acc = c.take<u64>((size_t)chunk * batch * 2 * LK * kN);
    void *scratch = c.base + c.off;
    CKKS_TRY(modup_stage(ctx, ct + (size_t)L * kN, nullptr, ct_elems, digits, batch, scratch, s));
    for (int r0 = 0; r0 < nkeys; r0 += chunk) {
        const int nk = std::min(chunk, nkeys - r0);
        KeyList kl{};
        DownExtra ex;
        ex.kind = 1;
        ex.ct = ct;
        ex.ct_bstride = ct_elems;
        ex.ct_mod = batch;
        ex.per = batch;
        for (int r = 0; r < nk; ++r) {
            kl.key[r] = keys[r0 + r];
            kl.galois[r] = ex.gal[r] = galois[r0 + r] & (2u * kN - 1u);
        }
        CKKS_TRY(key_inner_stage(ctx, digits, kl, batch, true, acc, nk * batch, s));
        CKKS_TRY(moddown_stage(ctx, acc, out + (size_t)r0 * batch * ct_elems, nk * batch, ex,
                               scratch, s));
    }
    return CKKS_OK;
}

// The rotation of ckks_rotate with ModUp -> NTT -> inner product streamed over windows of at most
// kWinMax primes: per window, the folded conversion writes every digit's limbs at the window's
// primes into a window buffer (the window's own digit gets the input's limbs), the forward NTT runs
// over it and the key inner product consumes it, so the extended digits never exist as a whole.
// Consecutive windows go round kLanes streams (the caller's and kLanes - 1 of its own), each with
// its own buffer (they write disjoint accumulator rows and only read y), so one window's launches
// fill the others' partial waves.  ModDown then runs as in ckks_rotate.
extern "C" int ckks_rotate_streamed(const ckks_ctx *ctx, const uint64_t *ct, const uint64_t *const *keys,
                                    const uint32_t *galois, int nkeys, uint64_t *out, int batch, void *ws,
                                    ckks_stream_t stream)
{
    CKKS_TRY(check_ctx(ctx));
    CKKS_TRY(check_batch(batch));
    if (nkeys < 0) return set_error(CKKS_EINVAL, "negative key count");
    if (batch == 0 || nkeys == 0) return CKKS_OK;
    if (!keys || !galois) return set_error(CKKS_EINVAL, "null key or galois array");
    for (int r = 0; r < nkeys; ++r) {
        CKKS_TRY(check_ptr(keys[r], "keys[r]"));
        if ((galois[r] & 1u) == 0) return set_error(CKKS_EINVAL, "galois element must be odd");
    }
    if ((size_t)nkeys * batch > 32767) return set_error(CKKS_EUNSUPPORTED, "nkeys * batch above 32767");
    CKKS_TRY(check_ptr(ct, "ct"));
    CKKS_TRY(check_ptr(out, "out"));
    CKKS_TRY(set_device(ctx));
    ckks_ctx *mctx = const_cast<ckks_ctx *>(ctx);
    const std::vector<ckks_ctx::Window> *wins = nullptr;
    CKKS_TRY(stream_windows(mctx, &wins));
    void *w;
    CKKS_TRY(resolve_ws(mctx, ws, rotate_streamed_ws(ctx, batch, nkeys), &w));
    const cudaStream_t s = (cudaStream_t)stream;
    const Tables &T = ctx->t;
    const int L = ctx->L, LK = L + ctx->K, dnum = ctx->dnum;
    const size_t ct_elems = (size_t)2 * L * kN;
    const int chunk = std::min(nkeys, kMaxKeys);
    Carve c(w);
    u64 *y = c.take<u64>((size_t)batch * L * kN);
    u64 *bufs[kLanes];
    for (u64 *&bp : bufs) bp = c.take<u64>((size_t)batch * dnum * kWinMax * kN);
    u64 *acc = c.take<u64>((size_t)chunk * batch * 2 * LK * kN);
    void *scratch = c.base + c.off;
    // the other lanes' streams and the fork / join events live for this call only; on every way
    // out (an error after the fork included) the caller's stream first waits for every lane, so no
    // window work outlives the call's view of the workspace
    cudaStream_t lane[kLanes] = {};
    cudaEvent_t ev[kLanes] = {};  // ev[0]: fork; ev[l]: lane l done
    struct Release {
        cudaStream_t *st;
        cudaEvent_t *e;
        ~Release()
        {
            for (int i = 1; i < kLanes; ++i) {
                if (!st[i]) continue;
                if (e[i] && cudaEventRecord(e[i], st[i]) == cudaSuccess) cudaStreamWaitEvent(st[0], e[i], 0);
                cudaStreamDestroy(st[i]);
            }
            for (int i = 0; i < kLanes; ++i)
                if (e[i]) cudaEventDestroy(e[i]);
        }
    } release{lane, ev};
    // a stream being captured into a graph keeps every window on itself (one lane)
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t ce = cudaStreamIsCapturing(s, &cap);
    const bool multi = ce == cudaSuccess && cap == cudaStreamCaptureStatusNone;
    if (ce != cudaSuccess) return cuda_status(ce, "cudaStreamIsCapturing");
    const int nl = multi ? kLanes : 1;
    lane[0] = s;
    for (int i = 1; i < nl && ce == cudaSuccess; ++i) ce = cudaStreamCreateWithFlags(&lane[i], cudaStreamNonBlocking);
    for (int i = 0; i < nl && ce == cudaSuccess; ++i) ce = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
    if (ce != cudaSuccess) return cuda_status(ce, "stream/event for the streamed rotation");
    // ModUp's sources: y = INTT(c1) times [(Q_j/q_i)^-1]
    const u64 *c1 = ct + (size_t)L * kN;
    UpInttJob<false> ij{c1, nullptr, ct_elems, nullptr, y, T.up_hatinv, T.pc, L, LK, T.alpha, dnum, batch,
                        L * batch};
    CKKS_TRY(launch_ntt_inv(ij, T, s));
    for (int r0 = 0; r0 < nkeys; r0 += chunk) {
        const int nk = std::min(chunk, nkeys - r0);
        KeyList kl{};
        DownExtra ex;
        ex.kind = 1;
        ex.ct = ct;
        ex.ct_bstride = ct_elems;
        ex.ct_mod = batch;
        ex.per = batch;
        for (int r = 0; r < nk; ++r) {
            kl.key[r] = keys[r0 + r];
            kl.galois[r] = ex.gal[r] = galois[r0 + r] & (2u * kN - 1u);
        }
        // fork: the second lane starts once y (and, from the second key chunk on, the previous
        // ModDown's reads of acc) are done on the caller's stream
        if (nl > 1) {
            ce = cudaEventRecord(ev[0], s);
            for (int i = 1; i < nl && ce == cudaSuccess; ++i) ce = cudaStreamWaitEvent(lane[i], ev[0], 0);
            if (ce != cudaSuccess) return cuda_status(ce, "fork of the streamed rotation");
        }
        for (int wi = 0; wi < (int)wins->size(); ++wi) {
            const ckks_ctx::Window wd = (*wins)[wi];
            const cudaStream_t ls = lane[wi % nl];
            u64 *buf = bufs[wi % nl];
            CKKS_TRY(launch_conv_fold_window(mctx, y, buf, batch, wi, ls));
            if (wd.own >= 0) {
                cudaError_t e = cudaMemcpy2DAsync(buf + (size_t)wd.own * kWinMax * kN,
                                                  (size_t)dnum * kWinMax * kN * sizeof(u64), c1 + (size_t)wd.t0 * kN,
                                                  ct_elems * sizeof(u64), (size_t)wd.n * kN * sizeof(u64), batch,
                                                  cudaMemcpyDeviceToDevice, ls);
                if (e != cudaSuccess) return cuda_status(e, "cudaMemcpy2DAsync(window digit copy)");
            }
            WinNttJob nj{buf, kWinMax, wd.t0, wd.n, wd.own, dnum, batch,
                         batch * (wd.own >= 0 ? dnum - 1 : dnum) * wd.n};
            CKKS_TRY(launch_ntt_fwd(nj, T, ls));
            const DigitView dv{(size_t)dnum * kWinMax * kN, (size_t)kWinMax * kN, wd.t0, wd.n};
            CKKS_TRY(key_inner_stage(ctx, buf, kl, batch, true, acc, nk * batch, ls, dv));
        }
        // join: ModDown reads every window's accumulator rows
        for (int i = 1; i < nl && ce == cudaSuccess; ++i) {
            ce = cudaEventRecord(ev[i], lane[i]);
            if (ce == cudaSuccess) ce = cudaStreamWaitEvent(s, ev[i], 0);
        }
        if (ce != cudaSuccess) return cuda_status(ce, "join of the streamed rotation");
        CKKS_TRY(moddown_stage(ctx, acc, out + (size_t)r0 * batch * ct_elems, nk * batch, ex, scratch, s));
    }
    return CKKS_OK;
}
