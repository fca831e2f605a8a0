// Building blocks of the bootstrapping refresh that the hot-path calls do not
// already provide (Kestrel engine write-up, the boot profile in section 5.3:
// modraise, conj_extract, restore_merge, and the constant products and sums
// of sin_fold).  Readings of the pages, as in the oracle:
//  - X^{n/2} multiplies every slot by i; in the NTT domain it is the
//    pointwise product by psi^{n/2} on the first n/2 evaluation slots and by
//    -psi^{n/2} on the others (NTT(X^{n/2})[k] = psi^{(n/2)(2 brv(k)+1)}).
//  - conj_extract: re = ct + conj(ct), im = X^{n/2} (conj(ct) - ct), with
//    conj the hoisted rotation by g = 2n - 1; slots 2 Re w and 2 Im w.
//  - restore_merge: re + X^{n/2} im.
//  - modraise: each coefficient over q_0..q_{l-1} read as its centred integer
//    X in (-Q/2, Q/2] and reduced modulo every prime of the context.  X comes
//    from Garner's mixed-radix digits d_i (word-size arithmetic only); the
//    comparison with the digits of (Q-1)/2 gives the sign; the conversion
//    sum_i d_i [q_0..q_{i-1}]_p - neg [Q]_p runs on conv_kernel with the sign
//    as one more source row.
#include <algorithm>

#include "internal.cuh"
#include "ntt.cuh"

extern "C" int ckks_rotate(const ckks_ctx *ctx, const uint64_t *ct, const uint64_t *const *keys,
                           const uint32_t *galois, int nkeys, uint64_t *out, int batch, void *ws,
                           ckks_stream_t stream);

namespace ckks {

constexpr int kMaxRaise = kMaxDigit - 1;  // input primes of modraise (one source row is the sign)

static int grid_1d(size_t work, int threads)
{
    size_t blocks = (work + threads - 1) / threads;
    return (int)std::min<size_t>(std::max<size_t>(blocks, 1), 148 * 32);
}

static int check_batch_b(int batch)
{
    if (batch < 0) return set_error(CKKS_EINVAL, "negative batch");
    if (batch > 65535) return set_error(CKKS_EUNSUPPORTED, "batch above 65535");
    return CKKS_OK;
}

// v * (+-psi^{n/2}) for evaluation slot k of prime `prime`: X^{n/2} in the NTT domain.
__device__ __forceinline__ u64 times_i(u64 v, int k, int prime, const ulonglong2 *__restrict__ iq, u64 q)
{
    const ulonglong2 w = iq[2 * prime + (k >= kN / 2 ? 1 : 0)];
    return shoup(v, w.x, w.y, q);
}

// ---------------------------------------------------------------- elementwise kernels
// out[p][l][k] = a[p][l][k] op kv[l]; kv holds residues in [0, q) of prime limb_begin + l.
__global__ void scalar_kernel(int op, const u64 *__restrict__ a, const u64 *__restrict__ kv,
                              u64 *__restrict__ out, int limbs, int limb_begin, size_t count,
                              const PrimeConst *__restrict__ pc)
{
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < count;
         e += (size_t)gridDim.x * blockDim.x) {
        const int limb = (int)((e / kN) % limbs);
        const PrimeConst c = pc[limb_begin + limb];
        const u64 x = a[e], y = kv[limb];
        out[e] = op == CKKS_PW_MUL ? mulmod(x, y, c) : op == CKKS_PW_ADD ? addmod(x, y, c.q)
                                                                          : submod(x, y, c.q);
    }
}

// ct[b][0][l][k] += kv[l] for every ciphertext b of [B][2][L][n] (component 0 only).
__global__ void c0_add_kernel(u64 *__restrict__ ct, const u64 *__restrict__ kv, int L, size_t count,
                              const PrimeConst *__restrict__ pc)
{
    const size_t Ln = (size_t)L * kN;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < count;
         e += (size_t)gridDim.x * blockDim.x) {
        const size_t b = e / Ln, r = e - b * Ln;
        const int limb = (int)(r / kN);
        u64 *p = ct + b * 2 * Ln + r;
        *p = addmod(*p, kv[limb], pc[limb].q);
    }
}

__global__ void muli_kernel(const u64 *__restrict__ in, u64 *__restrict__ out, int limbs, int limb_begin,
                            size_t count, const ulonglong2 *__restrict__ iq,
                            const PrimeConst *__restrict__ pc)
{
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < count;
         e += (size_t)gridDim.x * blockDim.x) {
        const int prime = limb_begin + (int)((e / kN) % limbs);
        out[e] = times_i(in[e], (int)(e % kN), prime, iq, pc[prime].q);
    }
}

// re = ct + cj, im = X^{n/2} (cj - ct) over [B][2][L][n].
__global__ void extract_kernel(const u64 *__restrict__ ct, const u64 *__restrict__ cj, u64 *__restrict__ re,
                               u64 *__restrict__ im, int L, size_t count, const ulonglong2 *__restrict__ iq,
                               const PrimeConst *__restrict__ pc)
{
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < count;
         e += (size_t)gridDim.x * blockDim.x) {
        const int prime = (int)((e / kN) % L);
        const u64 q = pc[prime].q, a = ct[e], c = cj[e];
        re[e] = addmod(a, c, q);
        im[e] = times_i(submod(c, a, q), (int)(e % kN), prime, iq, q);
    }
}

// out = re + X^{n/2} im over [B][2][L][n].
__global__ void merge_kernel(const u64 *__restrict__ re, const u64 *__restrict__ im, u64 *__restrict__ out,
                             int L, size_t count, const ulonglong2 *__restrict__ iq,
                             const PrimeConst *__restrict__ pc)
{
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < count;
         e += (size_t)gridDim.x * blockDim.x) {
        const int prime = (int)((e / kN) % L);
        const u64 q = pc[prime].q;
        out[e] = addmod(re[e], times_i(im[e], (int)(e % kN), prime, iq, q), q);
    }
}

// ---------------------------------------------------------------- modraise
// Garner digits of every coefficient: coef[P][l][n] (reduced residues) ->
// dg[P][l+1][n], rows 0..l-1 the digits d_i in [0, q_i) and row l the sign
// (1 where X > (Q-1)/2).  inv[i][j] = {q_j^-1 mod q_i, Shoup} for j < i;
// hd = the digits of (Q-1)/2.
__global__ void __launch_bounds__(128) garner_kernel(const u64 *__restrict__ coef, u64 *__restrict__ dg,
                                                     const ulonglong2 *__restrict__ inv,
                                                     const u64 *__restrict__ hd, int l, int P,
                                                     const PrimeConst *__restrict__ pc)
{
    const size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
    if (idx >= (size_t)P * kN) return;
    const size_t z = idx / kN;
    const int k = (int)(idx - z * kN);
    u64 d[kMaxRaise];
    for (int i = 0; i < l; ++i) {
        const u64 qi = pc[i].q;
        u64 t = coef[(z * l + i) * kN + k];
        for (int j = 0; j < i; ++j) {
            const ulonglong2 w = inv[(size_t)i * l + j];
            const u64 dj = csub(d[j] - mulhi(d[j], pc[i].mu64) * qi, qi);  // d_j mod q_i
            t = shoup(submod(t, dj, qi), w.x, w.y, qi);
        }
        d[i] = t;
        dg[(z * (l + 1) + i) * kN + k] = t;
    }
    u64 neg = 0;
    for (int i = l - 1; i >= 0; --i) {
        if (d[i] != hd[i]) {
            neg = d[i] > hd[i] ? 1 : 0;
            break;
        }
    }
    dg[(z * (l + 1) + l) * kN + k] = neg;
}

// Forward NTT of rows l..L-1 of every polynomial of out[P][L][n].
struct RaiseNttJob : BatchJob {
    int l, L;
    __device__ __forceinline__ Ref ref(int j) const
    {
        const int tr = j / batch, z = j - tr * batch;
        return {x + ((size_t)z * L + l + tr) * kN, l + tr};
    }
};

struct RaiseTab {
    ulonglong2 *inv = nullptr;
    u64 *hd = nullptr, *mat = nullptr;
};

static int upload_raw(const void *h, size_t bytes, void **d)
{
    cudaError_t e = cudaMalloc(d, std::max<size_t>(bytes, 16));
    if (e != cudaSuccess) {
        cudaGetLastError();
        *d = nullptr;
        return set_error(CKKS_ENOMEM, "modraise table allocation failed");
    }
    e = cudaMemcpy(*d, h, bytes, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_status(e, "cudaMemcpy(modraise table)");
    return CKKS_OK;
}

// Tables for raising from q_0..q_{l-1}, built once per l and kept by the context.
static const RaiseTab *raise_table(ckks_ctx *ctx, int l, int *rc)
{
    std::lock_guard<std::mutex> lock(ctx->mu);
    auto it = ctx->raise_tab.find(l);
    if (it != ctx->raise_tab.end()) {
        *rc = CKKS_OK;
        return static_cast<const RaiseTab *>(it->second);
    }
    const std::vector<u64> &m = ctx->mods;
    const int L = ctx->L;
    std::vector<ulonglong2> inv((size_t)l * l, make_ulonglong2(0, 0));
    for (int i = 0; i < l; ++i)
        for (int j = 0; j < i; ++j) {
            const u64 v = host_invmod(m[j] % m[i], m[i]);
            inv[(size_t)i * l + j] = make_ulonglong2(v, host_shoup(v, m[i]));
        }
    std::vector<u64> hd(l);
    for (int i = 0; i < l; ++i) {
        u64 t = (m[i] - 1) / 2;  // (Q-1)/2 = -1/2 mod q_i
        for (int j = 0; j < i; ++j) {
            const u64 dj = hd[j] % m[i];
            t = host_mulmod((t + m[i] - dj) % m[i], inv[(size_t)i * l + j].x, m[i]);
        }
        hd[i] = t;
    }
    std::vector<u64> mat((size_t)(l + 1) * L, 0);
    for (int t = l; t < L; ++t) {
        const u64 p = m[t];
        u64 pre = 1 % p;
        for (int s = 0; s < l; ++s) {
            mat[(size_t)s * L + t] = pre;
            pre = host_mulmod(pre, m[s] % p, p);
        }
        mat[(size_t)l * L + t] = (p - pre) % p;  // -Q mod p
    }
    RaiseTab *tab = new RaiseTab();
    *rc = upload_raw(inv.data(), inv.size() * sizeof(ulonglong2), reinterpret_cast<void **>(&tab->inv));
    if (*rc == CKKS_OK) *rc = upload_raw(hd.data(), hd.size() * sizeof(u64), reinterpret_cast<void **>(&tab->hd));
    if (*rc == CKKS_OK) *rc = upload_raw(mat.data(), mat.size() * sizeof(u64), reinterpret_cast<void **>(&tab->mat));
    if (*rc != CKKS_OK) {
        cudaFree(tab->inv);
        cudaFree(tab->hd);
        cudaFree(tab->mat);
        delete tab;
        return nullptr;
    }
    ctx->raise_tab[l] = tab;
    return tab;
}

void free_raise_tables(ckks_ctx *ctx)
{
    for (auto &kv : ctx->raise_tab) {
        RaiseTab *t = static_cast<RaiseTab *>(kv.second);
        cudaFree(t->inv);
        cudaFree(t->hd);
        cudaFree(t->mat);
        delete t;
    }
    ctx->raise_tab.clear();
}

size_t modraise_ws_bytes(const ckks_ctx *, int batch, int l)
{
    const size_t P = (size_t)2 * batch;
    return limbs_bytes(P * l) + limbs_bytes(P * (l + 1));
}

size_t conj_extract_ws_bytes(const ckks_ctx *ctx, int batch)
{
    return limbs_bytes((size_t)batch * 2 * ctx->L) + rotate_ws_bytes(ctx, batch, 1);
}

}  // namespace ckks

using namespace ckks;

extern "C" int ckks_pointwise_scalar(const ckks_ctx *ctx, int op, const uint64_t *a, const uint64_t *k,
                                     uint64_t *out, int batch, int limb_begin, int limbs,
                                     ckks_stream_t stream)
{
    CKKS_TRY(check_ctx(ctx));
    if (op != CKKS_PW_MUL && op != CKKS_PW_ADD && op != CKKS_PW_SUB)
        return set_error(CKKS_EINVAL, "unknown pointwise op");
    const int total = ctx->L + ctx->K;
    if (limb_begin < 0 || limbs < 0 || limb_begin > total || limbs > total - limb_begin)
        return set_error(CKKS_EINVAL, "limb range outside the context's primes");
    CKKS_TRY(check_batch_b(batch));
    if (batch == 0 || limbs == 0) return CKKS_OK;
    CKKS_TRY(check_ptr(a, "a"));
    CKKS_TRY(check_ptr(k, "k"));
    CKKS_TRY(check_ptr(out, "out"));
    CKKS_TRY(set_device(ctx));
    const size_t count = (size_t)batch * limbs * kN;
    scalar_kernel<<<grid_1d(count, 256), 256, 0, (cudaStream_t)stream>>>(op, a, k, out, limbs, limb_begin,
                                                                          count, ctx->t.pc);
    CKKS_CHECK_LAUNCH("scalar_kernel");
    return CKKS_OK;
}

extern "C" int ckks_add_const_c0(const ckks_ctx *ctx, uint64_t *ct, const uint64_t *k, int batch,
                                 ckks_stream_t stream)
{
    CKKS_TRY(check_ctx(ctx));
    CKKS_TRY(check_batch_b(batch));
    if (batch == 0) return CKKS_OK;
    CKKS_TRY(check_ptr(ct, "ct"));
    CKKS_TRY(check_ptr(k, "k"));
    CKKS_TRY(set_device(ctx));
    const size_t count = (size_t)batch * ctx->L * kN;
    c0_add_kernel<<<grid_1d(count, 256), 256, 0, (cudaStream_t)stream>>>(ct, k, ctx->L, count, ctx->t.pc);
    CKKS_CHECK_LAUNCH("c0_add_kernel");
    return CKKS_OK;
}

extern "C" int ckks_mul_i(const ckks_ctx *ctx, const uint64_t *in, uint64_t *out, int batch, int limb_begin,
                          int limbs, ckks_stream_t stream)
{
    CKKS_TRY(check_ctx(ctx));
    const int total = ctx->L + ctx->K;
    if (limb_begin < 0 || limbs < 0 || limb_begin > total || limbs > total - limb_begin)
        return set_error(CKKS_EINVAL, "limb range outside the context's primes");
    CKKS_TRY(check_batch_b(batch));
    if (batch == 0 || limbs == 0) return CKKS_OK;
    CKKS_TRY(check_ptr(in, "in"));
    CKKS_TRY(check_ptr(out, "out"));
    CKKS_TRY(set_device(ctx));
    const size_t count = (size_t)batch * limbs * kN;
    muli_kernel<<<grid_1d(count, 256), 256, 0, (cudaStream_t)stream>>>(in, out, limbs, limb_begin, count,
                                                                         ctx->t.mul_i, ctx->t.pc);
    CKKS_CHECK_LAUNCH("muli_kernel");
    return CKKS_OK;
}

extern "C" int ckks_conj_extract(const ckks_ctx *ctx, const uint64_t *ct, const uint64_t *conj_key,
                                 uint64_t *re, uint64_t *im, int batch, void *ws, ckks_stream_t stream)
{
    CKKS_TRY(check_ctx(ctx));
    CKKS_TRY(check_batch_b(batch));
    if (batch > 32767) return set_error(CKKS_EUNSUPPORTED, "batch above 32767");
    if (batch == 0) return CKKS_OK;
    CKKS_TRY(check_ptr(ct, "ct"));
    CKKS_TRY(check_ptr(conj_key, "conj_key"));
    CKKS_TRY(check_ptr(re, "re"));
    CKKS_TRY(check_ptr(im, "im"));
    CKKS_TRY(set_device(ctx));
    void *w;
    CKKS_TRY(resolve_ws(const_cast<ckks_ctx *>(ctx), ws, conj_extract_ws_bytes(ctx, batch), &w));
    Carve c(w);
    u64 *cj = c.take<u64>((size_t)batch * 2 * ctx->L * kN);
    void *rest = c.base + c.off;
    const uint32_t g = 2u * kN - 1u;
    const uint64_t *keys[1] = {conj_key};
    CKKS_TRY(ckks_rotate(ctx, ct, keys, &g, 1, cj, batch, rest, stream));
    const size_t count = (size_t)batch * 2 * ctx->L * kN;
    extract_kernel<<<grid_1d(count, 256), 256, 0, (cudaStream_t)stream>>>(ct, cj, re, im, ctx->L, count,
                                                                            ctx->t.mul_i, ctx->t.pc);
    CKKS_CHECK_LAUNCH("extract_kernel");
    return CKKS_OK;
}

extern "C" int ckks_restore_merge(const ckks_ctx *ctx, const uint64_t *re, const uint64_t *im, uint64_t *out,
                                  int batch, ckks_stream_t stream)
{
    CKKS_TRY(check_ctx(ctx));
    CKKS_TRY(check_batch_b(batch));
    if (batch == 0) return CKKS_OK;
    CKKS_TRY(check_ptr(re, "re"));
    CKKS_TRY(check_ptr(im, "im"));
    CKKS_TRY(check_ptr(out, "out"));
    CKKS_TRY(set_device(ctx));
    const size_t count = (size_t)batch * 2 * ctx->L * kN;
    merge_kernel<<<grid_1d(count, 256), 256, 0, (cudaStream_t)stream>>>(re, im, out, ctx->L, count,
                                                                          ctx->t.mul_i, ctx->t.pc);
    CKKS_CHECK_LAUNCH("merge_kernel");
    return CKKS_OK;
}

extern "C" int ckks_modraise(const ckks_ctx *ctx, const uint64_t *in, int l, uint64_t *out, int batch,
                             void *ws, ckks_stream_t stream)
{
    CKKS_TRY(check_ctx(ctx));
    CKKS_TRY(check_batch_b(batch));
    if (l < 1 || l > ctx->L || l > kMaxRaise)
        return set_error(CKKS_EUNSUPPORTED, "need 1 <= l <= min(L, 63)");
    if (batch > 32767) return set_error(CKKS_EUNSUPPORTED, "batch above 32767");
    if (batch == 0) return CKKS_OK;
    CKKS_TRY(check_ptr(in, "in"));
    CKKS_TRY(check_ptr(out, "out"));
    CKKS_TRY(set_device(ctx));
    int rc;
    const RaiseTab *tab = raise_table(const_cast<ckks_ctx *>(ctx), l, &rc);
    if (!tab) return rc;
    void *w;
    CKKS_TRY(resolve_ws(const_cast<ckks_ctx *>(ctx), ws, modraise_ws_bytes(ctx, batch, l), &w));
    const cudaStream_t s = (cudaStream_t)stream;
    const Tables &T = ctx->t;
    const int L = ctx->L, P = 2 * batch;
    Carve c(w);
    u64 *coef = c.take<u64>((size_t)P * l * kN);
    u64 *dg = c.take<u64>((size_t)P * (l + 1) * kN);
    cudaError_t e = cudaMemcpyAsync(coef, in, (size_t)P * l * kN * sizeof(u64), cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_status(e, "cudaMemcpyAsync(modraise input)");
    BatchJob ij{coef, l, P, 0, l * P};
    CKKS_TRY(launch_ntt_inv(ij, T, s));
    garner_kernel<<<(unsigned)(((size_t)P * kN + 127) / 128), 128, 0, s>>>(coef, dg, tab->inv, tab->hd, l, P,
                                                                          T.pc);
    CKKS_CHECK_LAUNCH("garner_kernel");
    if (l < L) {
        CKKS_TRY(raise_conv(T, dg, out, tab->mat, l, P, s));
        RaiseNttJob nj{{out, L - l, P, 0, (L - l) * P}, l, L};
        CKKS_TRY(launch_ntt_fwd(nj, T, s));
    }
    // below q_l the centred integer keeps its residues: copy the input limbs (NTT domain)
    e = cudaMemcpy2DAsync(out, (size_t)L * kN * sizeof(u64), in, (size_t)l * kN * sizeof(u64),
                          (size_t)l * kN * sizeof(u64), P, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_status(e, "cudaMemcpy2DAsync(modraise kept limbs)");
    return CKKS_OK;
}
