// NTT entry points, pointwise arithmetic, the Galois automorphism, rescale,
// ct x ct multiply with relinearisation, the BSGS linear transform, workspace
// sizing and the integer-pipe microbenchmarks.
#include <algorithm>

#include "internal.cuh"
#include "ntt.cuh"
#include "split.cuh"

namespace ckks {

size_t keyswitch_ws_bytes(const ckks_ctx *ctx, int batch);
size_t rotate_ws_bytes(const ckks_ctx *ctx, int batch, int nkeys);
size_t rotate_unhoisted_ws(const ckks_ctx *ctx, int batch);

static int check_batch(int batch)
{
    if (batch < 0) return set_error(CKKS_EINVAL, "negative batch");
    if (batch > 65535) return set_error(CKKS_EUNSUPPORTED, "batch above 65535");
    return CKKS_OK;
}

static int check_limbs(const ckks_ctx *ctx, int limb_begin, int limbs)
{
    // compared without forming limb_begin + limbs, which could overflow an int
    const int total = ctx->L + ctx->K;
    if (limb_begin < 0 || limbs < 0 || limb_begin > total || limbs > total - limb_begin)
        return set_error(CKKS_EINVAL, "limb range outside the context's primes");
    return CKKS_OK;
}

// ---------------------------------------------------------------- pointwise
__global__ void pointwise_kernel(int op, const u64 *__restrict__ a, const u64 *__restrict__ b,
                                 u64 *__restrict__ out, int limbs, int limb_begin, size_t pairs,
                                 const PrimeConst *__restrict__ pc)
{
    for (size_t p = blockIdx.x * (size_t)blockDim.x + threadIdx.x; p < pairs;
         p += (size_t)gridDim.x * blockDim.x) {
        const size_t e = 2 * p;
        const int limb = (int)((e / kN) % limbs);
        const PrimeConst c = pc[limb_begin + limb];
        const ulonglong2 x = *reinterpret_cast<const ulonglong2 *>(a + e);
        const ulonglong2 y = *reinterpret_cast<const ulonglong2 *>(b + e);
        ulonglong2 r;
        if (op == CKKS_PW_MUL) {
            r.x = mulmod(x.x, y.x, c);
            r.y = mulmod(x.y, y.y, c);
        } else if (op == CKKS_PW_ADD) {
            r.x = addmod(x.x, y.x, c.q);
            r.y = addmod(x.y, y.y, c.q);
        } else {
            r.x = submod(x.x, y.x, c.q);
            r.y = submod(x.y, y.y, c.q);
        }
        *reinterpret_cast<ulonglong2 *>(out + e) = r;
    }
}

static int grid_for(size_t work, int threads)
{
    size_t blocks = (work + threads - 1) / threads;
    return (int)std::min<size_t>(std::max<size_t>(blocks, 1), 148 * 32);
}

// ---------------------------------------------------------------- automorphism
// One CTA per limb row: stage the row in shared memory with coalesced loads,
// gather through the Galois index map, store coalesced.
__global__ void __launch_bounds__(256) automorph_kernel(const u64 *__restrict__ in,
                                                        u64 *__restrict__ out, u32 g)
{
    __shared__ u64 row[kN];
    const size_t base = (size_t)blockIdx.x * kN;
    for (int k = threadIdx.x; k < kN / 2; k += 256) {
        const ulonglong2 v = *reinterpret_cast<const ulonglong2 *>(in + base + 2 * k);
        row[2 * k] = v.x;
        row[2 * k + 1] = v.y;
    }
    __syncthreads();
    for (int k = threadIdx.x; k < kN / 2; k += 256) {
        ulonglong2 v;
        v.x = row[galois_src(2 * k, g)];
        v.y = row[galois_src(2 * k + 1, g)];
        *reinterpret_cast<ulonglong2 *>(out + base + 2 * k) = v;
    }
}

// ---------------------------------------------------------------- rescale
// INTT of the dropped limb of every (ciphertext, component) into w[.][n].
struct RescInttJob {
    const u64 *ct;
    u64 *w;
    int lp1, count;
    struct Ref {
        const u64 *src;
        u64 *dst;
        int prime;
    };
    __device__ __forceinline__ Ref ref(int j) const
    {
        return {ct + ((size_t)j * lp1 + lp1 - 1) * kN, w + (size_t)j * kN, lp1 - 1};
    }
    __device__ __forceinline__ void load4(const Ref &r, int e, u64 *v) const { ld4(r.src + e, v); }
    __device__ __forceinline__ void store(const Ref &r, int e, u64 v) const { r.dst[e] = v; }
};

// Forward NTT of [w]_{q_i} for every kept limb i; the store forms
// (c_i - NTT([w]_{q_i})) q_l^-1.
struct RescFwdJob {
    const u64 *w, *ct;
    u64 *out;
    const ulonglong2 *qinv;
    const PrimeConst *pc;
    int lp1, jobs2, count;
    struct Ref {
        const u64 *w, *ct;
        u64 *out;
        ulonglong2 qi;
        u64 q, mu;
        int prime;
    };
    __device__ __forceinline__ Ref ref(int j) const
    {
        const int i = j / jobs2, zz = j - i * jobs2;
        return {w + (size_t)zz * kN, ct + ((size_t)zz * lp1 + i) * kN, out + ((size_t)zz * (lp1 - 1) + i) * kN,
                qinv[i], pc[i].q, pc[i].mu64, i};
    }
    __device__ __forceinline__ u64 load(const Ref &r, int e) const
    {
        const u64 v = r.w[e];
        return v - mulhi(v, r.mu) * r.q;  // [0, 2 q_i)
    }
    __device__ __forceinline__ void store4(const Ref &r, int e, const u64 *v) const
    {
        u64 c[4], o[4];
        ld4(r.ct + e, c);
#pragma unroll
        for (int k = 0; k < 4; ++k) o[k] = shoup(submod(c[k], v[k], r.q), r.qi.x, r.qi.y, r.q);
        st4(r.out + e, o);
    }
};

size_t rescale_ws_bytes(int batch) { return limbs_bytes((size_t)batch * 2); }

int rescale_stage(ckks_ctx *ctx, const u64 *ct, u64 *out, int lp1, int batch, void *ws, cudaStream_t s)
{
    if (batch <= 0) return CKKS_OK;
    int rc;
    const ulonglong2 *qinv = rescale_table(ctx, lp1, &rc);
    if (!qinv) return rc;
    const Tables &T = ctx->t;
    Carve c(ws);
    u64 *w = c.take<u64>((size_t)batch * 2 * kN);
    RescInttJob ij{ct, w, lp1, 2 * batch};
    CKKS_TRY(launch_ntt_inv(ij, T, s));
    RescFwdJob fj{w, ct, out, qinv, T.pc, lp1, 2 * batch, (lp1 - 1) * 2 * batch};
    return launch_ntt_fwd(fj, T, s);
}

// ---------------------------------------------------------------- BSGS pieces
// inner[g][b][c][i][e] = sum_r diags[g][r][i][e] * baby_r[b][c][i][e], where
// baby_0 = x and baby_r (r >= 1) = baby[r-1].  One CTA per (32 coefficients,
// limb i, group of kBC ciphertext-components bc): the group's bb baby values
// sit in shared memory, 8 warps split the giant index g, and each diagonal
// word loaded serves the kBC components.  The grid runs the component groups
// of one (coefficients, limb) back to back, so the diagonals cross HBM once
// and are re-read from L2 by the other groups.
constexpr int kMaxBaby = 64;

template <int kBC>
__global__ void __launch_bounds__(256) bsgs_inner_kernel(const u64 *__restrict__ diags,
                                                         const u64 *__restrict__ x,
                                                         const u64 *__restrict__ baby,
                                                         u64 *__restrict__ inner, int bb, int gg,
                                                         int B, int L, const PrimeConst *__restrict__ pc)
{
    extern __shared__ u64 sb[];  // [kBC][bb][32]
    const int lane = threadIdx.x & 31, gw = threadIdx.x >> 5;
    const int ngrp = (2 * B + kBC - 1) / kBC;
    const int grp = blockIdx.x % ngrp, ech = blockIdx.x / ngrp, i = blockIdx.y;
    const int e = ech * 32 + lane;
    const int bc0 = grp * kBC, nbc = min(kBC, 2 * B - bc0);
    const size_t Ln = (size_t)L * kN;
    const size_t off0 = (size_t)bc0 * Ln + (size_t)i * kN + e;  // within one [B][2][L][n] block
    for (int idx = gw; idx < kBC * bb; idx += 8) {
        const int q = idx / bb, r = idx - q * bb;
        u64 v = 0;
        if (q < nbc) {
            const size_t off = off0 + (size_t)q * Ln;
            v = r == 0 ? x[off] : baby[(size_t)(r - 1) * B * 2 * Ln + off];
        }
        sb[(q * bb + r) * 32 + lane] = v;
    }
    __syncthreads();
    const PrimeConst c = pc[i];
    for (int g = gw; g < gg; g += 8) {
        const u64 *d = diags + ((size_t)g * bb * L + i) * kN + e;
        u64 hi[kBC], lo[kBC];
#pragma unroll
        for (int q = 0; q < kBC; ++q) hi[q] = lo[q] = 0;
#pragma unroll 8  // eight diagonal words in flight per thread
        for (int r = 0; r < bb; ++r) {
            const u64 dv = __ldg(d + (size_t)r * Ln);
#pragma unroll
            for (int q = 0; q < kBC; ++q) mac128(hi[q], lo[q], dv, sb[(q * bb + r) * 32 + lane]);
        }
#pragma unroll
        for (int q = 0; q < kBC; ++q)
            if (q < nbc) inner[(size_t)g * B * 2 * Ln + off0 + (size_t)q * Ln] = reduce128(hi[q], lo[q], c);
    }
}

// total[b] = (first ? first[b] : total[b]) + sum_{t < nterms} terms[t B + b],
// arrays of ciphertexts [.][2][L][n].
__global__ void accum_kernel(u64 *__restrict__ total, const u64 *__restrict__ first,
                             const u64 *__restrict__ terms, int nterms, int B, int L,
                             const PrimeConst *__restrict__ pc)
{
    const size_t ct = (size_t)2 * L * kN, n_all = (size_t)B * ct;
    for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < n_all;
         idx += (size_t)gridDim.x * blockDim.x) {
        const int i = (int)((idx / kN) % L);
        const u64 q = pc[i].q;
        u64 v = first ? first[idx] : total[idx];
        for (int t = 0; t < nterms; ++t) v = addmod(v, terms[(size_t)t * n_all + idx], q);
        total[idx] = v;
    }
}

static u32 galois_pow5(long long r)
{
    u32 g = 1;
    const u32 m = 2 * kN;
    r %= kN / 2;  // 5 has order n/2 modulo 2n
    if (r < 0) r += kN / 2;
    for (long long k = 0; k < r; ++k) g = (g * 5u) % m;
    return g;
}

struct BsgsLayout {
    int gchunk;
    size_t digits, acc, baby, inner, rot, total, scratch;
};

static BsgsLayout bsgs_layout(const ckks_ctx *ctx, int B, int bb, int gg)
{
    BsgsLayout l{};
    const size_t LK = ctx->L + ctx->K, L = ctx->L;
    l.gchunk = std::max(1, std::min(std::min(gg - 1, kMaxKeys), std::max(1, 64 / std::max(B, 1))));
    const int babyk = std::min(std::max(bb - 1, 1), kMaxKeys);
    const size_t up_batch = std::max<size_t>(B, (size_t)l.gchunk * B);
    const size_t acc_jobs = std::max<size_t>((size_t)babyk * B, (size_t)l.gchunk * B);
    l.digits = limbs_bytes(up_batch * ctx->dnum * LK);
    l.acc = limbs_bytes(acc_jobs * 2 * LK);
    l.baby = limbs_bytes((size_t)std::max(bb - 1, 0) * B * 2 * L);
    l.inner = limbs_bytes((size_t)gg * B * 2 * L);
    l.rot = limbs_bytes((size_t)l.gchunk * B * 2 * L);
    l.total = limbs_bytes((size_t)B * 2 * L);
    l.scratch = std::max({modup_ws_bytes(ctx, (int)up_batch), moddown_ws_bytes(ctx, (int)acc_jobs),
                          rescale_ws_bytes(B)});
    return l;
}

static size_t bsgs_ws(const ckks_ctx *ctx, int B, int bb, int gg)
{
    BsgsLayout l = bsgs_layout(ctx, B, bb, gg);
    return l.digits + l.acc + l.baby + l.inner + l.rot + l.total + l.scratch;
}

static size_t mrr_ws(const ckks_ctx *ctx, int B)
{
    const size_t LK = ctx->L + ctx->K;
    return limbs_bytes((size_t)B * ctx->dnum * LK) + limbs_bytes((size_t)B * 2 * LK) +
           limbs_bytes((size_t)B * 2 * ctx->L) +
           std::max({modup_ws_bytes(ctx, B), moddown_ws_bytes(ctx, B), rescale_ws_bytes(B)});
}

}  // namespace ckks

using namespace ckks;

// ---------------------------------------------------------------- entry points
extern "C" size_t ckks_workspace_bytes(const ckks_ctx *ctx, int op, int batch, int aux)
{
    if (!ctx || batch < 0) return 0;
    switch (op) {
    case CKKS_OP_MODUP: return modup_ws_bytes(ctx, batch);
    case CKKS_OP_MODDOWN: return moddown_ws_bytes(ctx, batch);
    case CKKS_OP_KEYSWITCH: return keyswitch_ws_bytes(ctx, batch);
    case CKKS_OP_ROTATE: return rotate_ws_bytes(ctx, batch, aux);
    case CKKS_OP_ROTATE_STREAMED: return rotate_streamed_ws_bytes(ctx, batch, aux);
    case CKKS_OP_ROTATE_UNHOISTED: return rotate_unhoisted_ws(ctx, batch);
    case CKKS_OP_MODRAISE: return aux >= 1 ? modraise_ws_bytes(ctx, batch, aux) : 0;
    case CKKS_OP_CONJ_EXTRACT: return conj_extract_ws_bytes(ctx, batch);
    case CKKS_OP_RESCALE: return rescale_ws_bytes(batch);
    case CKKS_OP_MUL_RELIN_RESCALE: return mrr_ws(ctx, batch);
    case CKKS_OP_BSGS: {
        const int bb = aux / 1000, gg = aux % 1000;
        if (bb < 1 || gg < 1) return 0;
        return bsgs_ws(ctx, batch, bb, gg);
    }
    default: return 0;
    }
}

static int ntt_common(const ckks_ctx *ctx, uint64_t *x, int batch, int limb_begin, int limbs)
{
    CKKS_TRY(check_ctx(ctx));
    CKKS_TRY(check_limbs(ctx, limb_begin, limbs));
    if (batch < 0) return set_error(CKKS_EINVAL, "negative batch");
    if ((long long)batch * limbs > (1LL << 30)) return set_error(CKKS_EUNSUPPORTED, "too many limbs");
    if (batch == 0 || limbs == 0) return 1;
    CKKS_TRY(check_ptr(x, "x"));
    CKKS_TRY(set_device(ctx));
    return CKKS_OK;
}

extern "C" int ckks_ntt_fwd(const ckks_ctx *ctx, uint64_t *x, int batch, int limb_begin, int limbs,
                            ckks_stream_t stream)
{
    int rc = ntt_common(ctx, x, batch, limb_begin, limbs);
    if (rc != CKKS_OK) return rc > 0 ? CKKS_OK : rc;
    BatchJob j{x, limbs, batch, limb_begin, limbs * batch};
    return launch_ntt_fwd(j, ctx->t, (cudaStream_t)stream);
}

extern "C" int ckks_ntt_inv(const ckks_ctx *ctx, uint64_t *x, int batch, int limb_begin, int limbs,
                            ckks_stream_t stream)
{
    int rc = ntt_common(ctx, x, batch, limb_begin, limbs);
    if (rc != CKKS_OK) return rc > 0 ? CKKS_OK : rc;
    BatchJob j{x, limbs, batch, limb_begin, limbs * batch};
    return launch_ntt_inv(j, ctx->t, (cudaStream_t)stream);
}

// Several tensors in one launch: group g is x[g][batch][limbs][n], limb l with prime
// limb_begin + l; its jobs follow those of the groups before it, limb-major within the group (the
// order BatchJob uses), so a CTA's consecutive jobs still share a prime.
constexpr int kMaxNttGroups = 8;

struct GroupJob {
    u64 *x[kMaxNttGroups];
    int limbs[kMaxNttGroups], batch[kMaxNttGroups], begin[kMaxNttGroups], start[kMaxNttGroups + 1];
    int groups, count;
    struct Ref {
        u64 *row;
        int prime;
    };
    __device__ __forceinline__ Ref ref(int j) const
    {
        int g = 0;
#pragma unroll
        for (int i = 1; i < kMaxNttGroups; ++i) g += (i < groups && j >= start[i]) ? 1 : 0;
        const int jj = j - start[g];
        const int l = jj / batch[g], b = jj - l * batch[g];
        return {x[g] + ((size_t)b * limbs[g] + l) * kN, begin[g] + l};
    }
    __device__ __forceinline__ u64 load(const Ref &r, int e) const { return r.row[e]; }
    __device__ __forceinline__ void store4(const Ref &r, int e, const u64 *v) const { st4(r.row + e, v); }
    __device__ __forceinline__ void load4(const Ref &r, int e, u64 *v) const { ld4(r.row + e, v); }
    __device__ __forceinline__ void store(const Ref &r, int e, u64 v) const { r.row[e] = v; }
};

static int ntt_group_job(const ckks_ctx *ctx, uint64_t *const *x, const int *batch, const int *limb_begin,
                         const int *limbs, int groups, GroupJob *job)
{
    CKKS_TRY(check_ctx(ctx));
    if (groups < 0 || groups > kMaxNttGroups) return set_error(CKKS_EINVAL, "need 0 <= groups <= 8");
    if (groups > 0 && (!x || !batch || !limb_begin || !limbs)) return set_error(CKKS_EINVAL, "null group array");
    long long total = 0;
    int n = 0;
    for (int g = 0; g < groups; ++g) {
        CKKS_TRY(check_limbs(ctx, limb_begin[g], limbs[g]));
        if (batch[g] < 0) return set_error(CKKS_EINVAL, "negative batch");
        if ((long long)batch[g] * limbs[g] == 0) continue;
        CKKS_TRY(check_ptr(x[g], "x[g]"));
        job->x[n] = x[g];
        job->limbs[n] = limbs[g];
        job->batch[n] = batch[g];
        job->begin[n] = limb_begin[g];
        job->start[n] = (int)total;
        total += (long long)batch[g] * limbs[g];
        if (total > (1LL << 30)) return set_error(CKKS_EUNSUPPORTED, "too many limbs");
        ++n;
    }
    for (int g = n; g <= kMaxNttGroups; ++g) job->start[g] = (int)total;
    job->groups = n;
    job->count = (int)total;
    if (total == 0) return 1;
    CKKS_TRY(set_device(ctx));
    return CKKS_OK;
}

extern "C" int ckks_ntt_fwd_group(const ckks_ctx *ctx, uint64_t *const *x, const int *batch,
                                  const int *limb_begin, const int *limbs, int groups, ckks_stream_t stream)
{
    GroupJob j{};
    int rc = ntt_group_job(ctx, x, batch, limb_begin, limbs, groups, &j);
    if (rc != CKKS_OK) return rc > 0 ? CKKS_OK : rc;
    return launch_ntt_fwd(j, ctx->t, (cudaStream_t)stream);
}

extern "C" int ckks_ntt_inv_group(const ckks_ctx *ctx, uint64_t *const *x, const int *batch,
                                  const int *limb_begin, const int *limbs, int groups, ckks_stream_t stream)
{
    GroupJob j{};
    int rc = ntt_group_job(ctx, x, batch, limb_begin, limbs, groups, &j);
    if (rc != CKKS_OK) return rc > 0 ? CKKS_OK : rc;
    return launch_ntt_inv(j, ctx->t, (cudaStream_t)stream);
}

extern "C" int ckks_pointwise(const ckks_ctx *ctx, int op, const uint64_t *a, const uint64_t *b,
                              uint64_t *out, int batch, int limb_begin, int limbs,
                              ckks_stream_t stream)
{
    CKKS_TRY(check_ctx(ctx));
    if (op != CKKS_PW_MUL && op != CKKS_PW_ADD && op != CKKS_PW_SUB)
        return set_error(CKKS_EINVAL, "unknown pointwise op");
    CKKS_TRY(check_limbs(ctx, limb_begin, limbs));
    CKKS_TRY(check_batch(batch));
    if (batch == 0 || limbs == 0) return CKKS_OK;
    CKKS_TRY(check_ptr(a, "a"));
    CKKS_TRY(check_ptr(b, "b"));
    CKKS_TRY(check_ptr(out, "out"));
    CKKS_TRY(set_device(ctx));
    const size_t pairs = (size_t)batch * limbs * kN / 2;
    pointwise_kernel<<<grid_for(pairs, 256), 256, 0, (cudaStream_t)stream>>>(
        op, a, b, out, limbs, limb_begin, pairs, ctx->t.pc);
    CKKS_CHECK_LAUNCH("pointwise_kernel");
    return CKKS_OK;
}

extern "C" int ckks_automorph(const ckks_ctx *ctx, const uint64_t *in, uint64_t *out, int batch,
                              int limbs, uint32_t galois, ckks_stream_t stream)
{
    CKKS_TRY(check_ctx(ctx));
    CKKS_TRY(check_batch(batch));
    if (limbs < 0) return set_error(CKKS_EINVAL, "negative limb count");
    if ((galois & 1u) == 0) return set_error(CKKS_EINVAL, "galois element must be odd");
    const long long rows = (long long)batch * limbs;
    if (rows == 0) return CKKS_OK;
    if (rows > 0x7fffffffLL) return set_error(CKKS_EUNSUPPORTED, "too many rows");
    CKKS_TRY(check_ptr(in, "in"));
    CKKS_TRY(check_ptr(out, "out"));
    if (in == out) return set_error(CKKS_EINVAL, "automorphism cannot run in place");
    CKKS_TRY(set_device(ctx));
    automorph_kernel<<<(unsigned)rows, 256, 0, (cudaStream_t)stream>>>(in, out, galois & (2u * kN - 1u));
    CKKS_CHECK_LAUNCH("automorph_kernel");
    return CKKS_OK;
}

namespace ckks {
size_t rotate_unhoisted_ws(const ckks_ctx *ctx, int batch)
{
    return limbs_bytes((size_t)batch * 2 * ctx->L) + rotate_ws_bytes(ctx, batch, 1);
}
}  // namespace ckks

// The other rotation order: for each key, phi_g of the whole ciphertext batch (one automorphism
// launch over both components), then a key switch of the rotated c1 with the Galois key (ModUp,
// inner product without a gather, ModDown) whose final store adds the rotated c0.
extern "C" int ckks_rotate_unhoisted(const ckks_ctx *ctx, const uint64_t *ct, const uint64_t *const *keys,
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
    if (batch > 32767) return set_error(CKKS_EUNSUPPORTED, "batch above 32767");
    CKKS_TRY(check_ptr(ct, "ct"));
    CKKS_TRY(check_ptr(out, "out"));
    CKKS_TRY(set_device(ctx));
    void *w;
    CKKS_TRY(resolve_ws(const_cast<ckks_ctx *>(ctx), ws, rotate_unhoisted_ws(ctx, batch), &w));
    const cudaStream_t s = (cudaStream_t)stream;
    const int L = ctx->L, LK = L + ctx->K;
    const size_t ct_elems = (size_t)2 * L * kN;
    Carve c(w);
    u64 *rct = c.take<u64>((size_t)batch * 2 * L * kN);
    u64 *digits = c.take<u64>((size_t)batch * ctx->dnum * LK * kN);
    u64 *acc = c.take<u64>((size_t)batch * 2 * LK * kN);
    void *scratch = c.base + c.off;
    for (int r = 0; r < nkeys; ++r) {
        const u32 g = galois[r] & (2u * kN - 1u);
        automorph_kernel<<<(unsigned)((size_t)batch * 2 * L), 256, 0, s>>>(ct, rct, g);
        CKKS_CHECK_LAUNCH("automorph_kernel");
        CKKS_TRY(modup_stage(ctx, rct + (size_t)L * kN, nullptr, ct_elems, digits, batch, scratch, s));
        KeyList kl{};
        kl.key[0] = keys[r];
        kl.galois[0] = 1;
        CKKS_TRY(key_inner_stage(ctx, digits, kl, batch, true, acc, batch, s));
        DownExtra ex;
        ex.kind = 1;
        ex.ct = rct;
        ex.ct_bstride = ct_elems;
        ex.ct_mod = batch;
        ex.per = batch;
        ex.gal[0] = 1;
        CKKS_TRY(moddown_stage(ctx, acc, out + (size_t)r * batch * ct_elems, batch, ex, scratch, s));
    }
    return CKKS_OK;
}

extern "C" int ckks_rescale(const ckks_ctx *ctx, const uint64_t *ct, uint64_t *out, int lp1, int batch,
                            void *ws, ckks_stream_t stream)
{
    CKKS_TRY(check_ctx(ctx));
    CKKS_TRY(check_batch(batch));
    if (lp1 < 2 || lp1 > ctx->L) return set_error(CKKS_EINVAL, "lp1 must be in [2, L]");
    if (batch == 0) return CKKS_OK;
    CKKS_TRY(check_ptr(ct, "ct"));
    CKKS_TRY(check_ptr(out, "out"));
    if (ct == out) return set_error(CKKS_EINVAL, "rescale cannot run in place");
    CKKS_TRY(set_device(ctx));
    ckks_ctx *m = const_cast<ckks_ctx *>(ctx);
    void *w;
    CKKS_TRY(resolve_ws(m, ws, rescale_ws_bytes(batch), &w));
    return rescale_stage(m, ct, out, lp1, batch, w, (cudaStream_t)stream);
}

extern "C" int ckks_mul_relin_rescale(const ckks_ctx *ctx, const uint64_t *a, const uint64_t *b,
                                      const uint64_t *rlk, uint64_t *out, int batch, void *ws,
                                      ckks_stream_t stream)
{
    CKKS_TRY(check_ctx(ctx));
    CKKS_TRY(check_batch(batch));
    if (ctx->L < 2) return set_error(CKKS_EUNSUPPORTED, "rescale needs L >= 2");
    if (batch == 0) return CKKS_OK;
    CKKS_TRY(check_ptr(a, "a"));
    CKKS_TRY(check_ptr(b, "b"));
    CKKS_TRY(check_ptr(rlk, "rlk"));
    CKKS_TRY(check_ptr(out, "out"));
    CKKS_TRY(set_device(ctx));
    ckks_ctx *m = const_cast<ckks_ctx *>(ctx);
    void *w;
    CKKS_TRY(resolve_ws(m, ws, mrr_ws(ctx, batch), &w));
    const cudaStream_t s = (cudaStream_t)stream;
    const int L = ctx->L, LK = L + ctx->K;
    const size_t Ln = (size_t)L * kN;
    Carve c(w);
    u64 *digits = c.take<u64>((size_t)batch * ctx->dnum * LK * kN);
    u64 *acc = c.take<u64>((size_t)batch * 2 * LK * kN);
    u64 *cr = c.take<u64>((size_t)batch * 2 * Ln);
    void *scratch = c.base + c.off;
    // d2 = a1 b1 is formed inside ModUp's first transform
    CKKS_TRY(modup_stage(ctx, a + Ln, b + Ln, 2 * Ln, digits, batch, scratch, s));
    KeyList kl{};
    kl.key[0] = rlk;
    kl.galois[0] = 1;
    CKKS_TRY(key_inner_stage(ctx, digits, kl, batch, true, acc, batch, s));
    DownExtra ex;
    ex.kind = 2;  // + (a0 b0, a0 b1 + a1 b0)
    ex.a = a;
    ex.b = b;
    CKKS_TRY(moddown_stage(ctx, acc, cr, batch, ex, scratch, s));
    return rescale_stage(m, cr, out, L, batch, scratch, s);
}

// The BSGS transform for diagonals at offsets stride (t0 + bb g + b), g < gg,
// b < bb (the dense form is stride 1, t0 0):
//   y = Rescale( sum_g Rot_{G_g}( sum_b diags[g][b] * Rot_{stride b}(x) ) ),
//   G_g = stride (t0 + bb g) mod n/2.
// giant_keys[g] serves G_g (unused where G_g = 0, which needs no rotation).
static int bsgs_core(const ckks_ctx *ctx, const uint64_t *x, const uint64_t *diags,
                     const uint64_t *const *baby_keys, const uint64_t *const *giant_keys, int stride,
                     int t0, int bb, int gg, uint64_t *y, int batch, void *ws, cudaStream_t s)
{
    ckks_ctx *m = const_cast<ckks_ctx *>(ctx);
    void *w;
    CKKS_TRY(resolve_ws(m, ws, bsgs_ws(ctx, batch, bb, gg), &w));
    const Tables &T = ctx->t;
    const int L = ctx->L, B = batch;
    const size_t Ln = (size_t)L * kN, ctn = 2 * Ln;
    const BsgsLayout lay = bsgs_layout(ctx, B, bb, gg);
    char *base = static_cast<char *>(w);
    u64 *digits = reinterpret_cast<u64 *>(base);
    u64 *acc = reinterpret_cast<u64 *>(base + lay.digits);
    u64 *baby = reinterpret_cast<u64 *>(base + lay.digits + lay.acc);
    u64 *inner = reinterpret_cast<u64 *>(base + lay.digits + lay.acc + lay.baby);
    u64 *rot = reinterpret_cast<u64 *>(base + lay.digits + lay.acc + lay.baby + lay.inner);
    u64 *total = reinterpret_cast<u64 *>(base + lay.digits + lay.acc + lay.baby + lay.inner + lay.rot);
    void *scratch = base + lay.digits + lay.acc + lay.baby + lay.inner + lay.rot + lay.total;

    // baby steps: Rot_{stride r}(x), r = 1..bb-1, on one hoisted ModUp
    if (bb > 1) {
        CKKS_TRY(modup_stage(ctx, x + Ln, nullptr, ctn, digits, B, scratch, s));
        for (int r0 = 1; r0 < bb; r0 += kMaxKeys) {
            const int nk = std::min(kMaxKeys, bb - r0);
            KeyList kl{};
            DownExtra ex;
            ex.kind = 1;
            ex.ct = x;
            ex.ct_bstride = ctn;
            ex.ct_mod = B;
            ex.per = B;
            for (int r = 0; r < nk; ++r) {
                kl.key[r] = baby_keys[r0 + r - 1];
                kl.galois[r] = ex.gal[r] = galois_pow5((long long)stride * (r0 + r));
            }
            CKKS_TRY(key_inner_stage(ctx, digits, kl, B, true, acc, nk * B, s));
            CKKS_TRY(moddown_stage(ctx, acc, baby + (size_t)(r0 - 1) * B * ctn, nk * B, ex, scratch, s));
        }
    }
    // inner sums for every giant index
    {
        // 4 components per CTA while the baby values fit 32 KiB of shared memory, else 2
        if (bb <= 32) {
            const dim3 grid((kN / 32) * ((2 * B + 3) / 4), L);
            bsgs_inner_kernel<4><<<grid, 256, (size_t)4 * bb * 32 * sizeof(u64), s>>>(diags, x, baby, inner, bb,
                                                                                       gg, B, L, T.pc);
        } else {
            const dim3 grid((kN / 32) * ((2 * B + 1) / 2), L);
            bsgs_inner_kernel<2><<<grid, 256, (size_t)2 * bb * 32 * sizeof(u64), s>>>(diags, x, baby, inner, bb,
                                                                                       gg, B, L, T.pc);
        }
        CKKS_CHECK_LAUNCH("bsgs_inner_kernel");
    }
    // giant steps: total = (the unrotated inner sum, if any) + sum of the rotated ones
    const int S = kN / 2;
    auto giant = [&](int g) {
        long long v = (long long)stride * (t0 + (long long)bb * g) % S;
        return (int)(v < 0 ? v + S : v);
    };
    int gz = -1;
    for (int g = 0; g < gg && gz < 0; ++g)
        if (giant(g) == 0) gz = g;
    const size_t all = (size_t)B * ctn;
    if (gz >= 0) {
        accum_kernel<<<grid_for(all, 256), 256, 0, s>>>(total, inner + (size_t)gz * B * ctn, nullptr, 0, B, L,
                                                        T.pc);
        CKKS_CHECK_LAUNCH("accum_kernel");
    } else {
        cudaError_t e = cudaMemsetAsync(total, 0, all * sizeof(u64), s);
        if (e != cudaSuccess) return cuda_status(e, "cudaMemsetAsync(bsgs total)");
    }
    // the rotated giant steps form at most two runs of consecutive g, around gz
    const int run_lo[2] = {0, gz + 1}, run_hi[2] = {gz < 0 ? gg : gz, gz < 0 ? 0 : gg};
    for (int run = 0; run < 2; ++run) {
        for (int g0 = run_lo[run]; g0 < run_hi[run]; g0 += lay.gchunk) {
            const int ng = std::min(lay.gchunk, run_hi[run] - g0);
            const u64 *src = inner + (size_t)g0 * B * ctn;
            CKKS_TRY(modup_stage(ctx, src + Ln, nullptr, ctn, digits, ng * B, scratch, s));
            KeyList kl{};
            DownExtra ex;
            ex.kind = 1;
            ex.ct = src;
            ex.ct_bstride = ctn;
            ex.ct_mod = 0;
            ex.per = B;
            for (int g = 0; g < ng; ++g) {
                kl.key[g] = giant_keys[g0 + g];
                kl.galois[g] = ex.gal[g] = galois_pow5(giant(g0 + g));
            }
            CKKS_TRY(key_inner_stage(ctx, digits, kl, B, false, acc, ng * B, s));
            CKKS_TRY(moddown_stage(ctx, acc, rot, ng * B, ex, scratch, s));
            accum_kernel<<<grid_for(all, 256), 256, 0, s>>>(total, nullptr, rot, ng, B, L, T.pc);
            CKKS_CHECK_LAUNCH("accum_kernel");
        }
    }
    return rescale_stage(m, total, y, L, B, scratch, s);
}

static int bsgs_checks(const ckks_ctx *ctx, const uint64_t *x, const uint64_t *diags, uint64_t *y, int bb,
                       int gg, int batch)
{
    CKKS_TRY(check_ctx(ctx));
    CKKS_TRY(check_batch(batch));
    if (ctx->L < 2) return set_error(CKKS_EUNSUPPORTED, "rescale needs L >= 2");
    if (bb < 1 || gg < 1 || bb > kMaxBaby || gg > 999)
        return set_error(CKKS_EINVAL, "need 1 <= bb <= 64 and 1 <= gg <= 999");
    if ((size_t)batch * std::max(bb - 1, 1) > 32767)
        return set_error(CKKS_EUNSUPPORTED, "batch * (bb - 1) above 32767");
    if (batch == 0) return CKKS_OK;
    CKKS_TRY(check_ptr(x, "x"));
    CKKS_TRY(check_ptr(diags, "diags"));
    CKKS_TRY(check_ptr(y, "y"));
    return CKKS_OK;
}

extern "C" int ckks_bsgs_lintrans(const ckks_ctx *ctx, const uint64_t *x, const uint64_t *diags,
                                  const uint64_t *const *baby_keys, const uint64_t *const *giant_keys,
                                  int bb, int gg, uint64_t *y, int batch, void *ws,
                                  ckks_stream_t stream)
{
    CKKS_TRY(bsgs_checks(ctx, x, diags, y, bb, gg, batch));
    if (batch == 0) return CKKS_OK;
    if (bb > 1 && !baby_keys) return set_error(CKKS_EINVAL, "null baby key array");
    if (gg > 1 && !giant_keys) return set_error(CKKS_EINVAL, "null giant key array");
    for (int r = 0; r + 1 < bb; ++r) CKKS_TRY(check_ptr(baby_keys[r], "baby_keys[r]"));
    for (int g = 0; g + 1 < gg; ++g) CKKS_TRY(check_ptr(giant_keys[g], "giant_keys[g]"));
    CKKS_TRY(set_device(ctx));
    // giant step g >= 1 uses giant_keys[g - 1]; step 0 is unrotated
    std::vector<const uint64_t *> gk(gg, nullptr);
    for (int g = 1; g < gg; ++g) gk[g] = giant_keys[g - 1];
    return bsgs_core(ctx, x, diags, baby_keys, gk.data(), 1, 0, bb, gg, y, batch, ws, (cudaStream_t)stream);
}

extern "C" int ckks_bsgs_lintrans_plan(const ckks_ctx *ctx, const uint64_t *x, const uint64_t *diags,
                                       const uint64_t *const *baby_keys, const uint64_t *const *giant_keys,
                                       int stride, int t0, int bb, int gg, uint64_t *y, int batch, void *ws,
                                       ckks_stream_t stream)
{
    CKKS_TRY(bsgs_checks(ctx, x, diags, y, bb, gg, batch));
    if (stride < 1 || (long long)stride * (bb - 1) >= kN / 2)
        return set_error(CKKS_EINVAL, "need stride >= 1 and stride * (bb - 1) < n/2");
    if (t0 < -(kN / 2) || t0 > kN / 2) return set_error(CKKS_EINVAL, "t0 outside [-n/2, n/2]");
    if (batch == 0) return CKKS_OK;
    if (bb > 1 && !baby_keys) return set_error(CKKS_EINVAL, "null baby key array");
    if (!giant_keys) return set_error(CKKS_EINVAL, "null giant key array");
    for (int r = 0; r + 1 < bb; ++r) CKKS_TRY(check_ptr(baby_keys[r], "baby_keys[r]"));
    // only the first giant step with G_g = 0 is summed unrotated; any other
    // step (including a later one with G_g = 0) is a key switch and needs a key
    const int S = kN / 2;
    bool unrotated_seen = false;
    for (int g = 0; g < gg; ++g) {
        long long v = (long long)stride * (t0 + (long long)bb * g) % S;
        if (v == 0 && !unrotated_seen) {
            unrotated_seen = true;
            continue;
        }
        CKKS_TRY(check_ptr(giant_keys[g], "giant_keys[g]"));
    }
    CKKS_TRY(set_device(ctx));
    return bsgs_core(ctx, x, diags, baby_keys, giant_keys, stride, t0, bb, gg, y, batch, ws,
                     (cudaStream_t)stream);
}

// ---------------------------------------------------------------- microbenchmarks
// The forward NTT's own butterfly (ct_bfly: the three-partial-product Shoup
// quotient, the cheap q h product for 2^60 - delta primes when kS, and the
// lazy add/sub), 4 independent butterflies over 8 registers per iteration.
template <bool kS>
__device__ __forceinline__ void bfly_loop(u64 x[8], int iters, u64 q, u64 w, u64 wp)
{
    const Mod md{q, 2 * q, 4 * q, (1ull << 60) - q};
    const ulonglong2 tw = make_ulonglong2(w, wp);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int k = 0; k < 4; ++k) ct_bfly<kS>(x[k], x[k + 4], tw, md);
    }
}

// Kind 6, the key inner product's split form without its loads, in a kernel of its own so that its
// 48 sums do not raise the register count (and lower the occupancy) of the other kinds: per step a
// new word per chain, split once and multiplied into the sums of two key words (the kernel's two
// components), the sums folded every kSplitFold words.
__global__ void splitmac_kernel(int iters, u64 q, u64 w, u64 *sink)
{
    u64 x[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) x[k] = (threadIdx.x * 8 + k + 1) * 0x9E3779B97F4A7C15ull % q;
    const Split30 kw0 = split30(w), kw1 = split30(q - 1 - w);
    const u32 delta = (u32)(((u64)1 << 60) - q);
    u64 s[8][2][3];
#pragma unroll
    for (int k = 0; k < 8; ++k)
#pragma unroll
        for (int c = 0; c < 2; ++c) s[k][c][0] = s[k][c][1] = s[k][c][2] = 0;
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int u = 0; u < kSplitFold; ++u) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const Split30 d = split30(x[k] ^ (u64)(it * kSplitFold + u));  // stays below 2^60
                split_mac(s[k][0][0], s[k][0][1], s[k][0][2], d, kw0);
                split_mac(s[k][1][0], s[k][1][1], s[k][1][2], d, kw1);
            }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
#pragma unroll
            for (int c = 0; c < 2; ++c) split_fold(s[k][c][0], s[k][c][1], s[k][c][2], delta);
    }
    u64 acc = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) acc ^= s[k][0][0] ^ s[k][0][2] ^ s[k][1][0] ^ s[k][1][2];
    if (acc == 0x1234567ull) sink[threadIdx.x] = acc;  // keeps the loop alive
}

__global__ void intpipe_kernel(int kind, int iters, u64 q, u64 w, u64 wp, int special, u64 *sink)
{
    u64 x[8], h[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        x[k] = (threadIdx.x * 8 + k + 1) * 0x9E3779B97F4A7C15ull % q;
        h[k] = 0;
    }
    if (kind == 0) {
        for (int it = 0; it < iters; ++it) {
#pragma unroll
            for (int k = 0; k < 8; ++k) x[k] = shoup(x[k], w, wp, q);
        }
    } else if (kind == 1) {
        u64 y[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) y[k] = x[k] ^ 0x5555555555ull;
        for (int it = 0; it < iters; ++it) {
            const u64 m = w ^ (u64)it;  // a new multiplier every iteration: nothing to hoist
#pragma unroll
            for (int k = 0; k < 8; ++k) mac128(h[k], x[k], y[k], m);  // 8 independent chains
        }
    } else if (kind == 2) {
        for (int it = 0; it < iters; ++it) {
#pragma unroll
            for (int k = 0; k < 8; ++k) x[k] = mulhi(x[k], wp) + w;
        }
    } else if (special) {
        bfly_loop<true>(x, iters, q, w, wp);
    } else {
        bfly_loop<false>(x, iters, q, w, wp);
    }
    u64 acc = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) acc ^= x[k] ^ h[k];
    if (acc == 0x1234567ull) sink[threadIdx.x] = acc;  // keeps the loops alive
}

extern "C" int ckks_bench_intpipe(const ckks_ctx *ctx, int kind, int blocks, int iters, double *ms,
                                  double *ops)
{
    CKKS_TRY(check_ctx(ctx));
    if (kind < 0 || kind > 6 || blocks < 1 || blocks > 148 * 64 || iters < 1 || !ms || !ops)
        return set_error(CKKS_EINVAL, "bad microbenchmark arguments");
    if (kind == 6 && !ctx->t.special)
        return set_error(CKKS_EUNSUPPORTED, "the split-form microbenchmark needs primes 2^60 - delta");
    if (kind == 6 && iters > (1 << 26)) return set_error(CKKS_EINVAL, "too many iterations for kind 6");
    CKKS_TRY(set_device(ctx));
    if (kind == 3 || kind == 4) return bench_mma(ctx, kind == 3 ? 256 : 32, blocks, iters, ms, ops);
    const u64 q = ctx->mods[0];
    const u64 w = 0x0123456789abcdefull % q, wp = host_shoup(w, q);
    u64 *sink = nullptr;
    cudaError_t e = cudaMalloc(&sink, 256 * sizeof(u64));
    if (e != cudaSuccess) return cuda_status(e, "cudaMalloc(sink)");
    cudaEvent_t a, b;
    cudaEventCreate(&a);
    cudaEventCreate(&b);
    const int special = ctx->t.special ? 1 : 0;
    if (kind == 6)
        splitmac_kernel<<<blocks, 256>>>(std::max(1, iters / 16), q, w, sink);  // warm-up
    else
        intpipe_kernel<<<blocks, 256>>>(kind, std::max(1, iters / 16), q, w, wp, special, sink);
    cudaEventRecord(a);
    if (kind == 6)
        splitmac_kernel<<<blocks, 256>>>(iters, q, w, sink);
    else
        intpipe_kernel<<<blocks, 256>>>(kind, iters, q, w, wp, special, sink);
    cudaEventRecord(b);
    e = cudaEventSynchronize(b);
    float t = 0;
    cudaEventElapsedTime(&t, a, b);
    cudaEventDestroy(a);
    cudaEventDestroy(b);
    cudaFree(sink);
    if (e != cudaSuccess) return cuda_status(e, "intpipe_kernel");
    *ms = t;
    *ops = (double)blocks * 256.0 * iters * (kind == 5 ? 4.0 : kind == 6 ? 8.0 * 2 * kSplitFold : 8.0);
    return CKKS_OK;
}
