// Context creation, validation, host-side number theory and error plumbing.
//
// The tables follow the library's readings of the pages (60-bit primes with
// q = 1 mod 2n; the smallest primitive 2n-th root; hybrid key switching with
// contiguous digits).  Everything here runs once per context on the host; the
// hot path only reads the uploaded tables.
#include <string.h>

#include <algorithm>
#include <functional>
#include <thread>

#include "internal.cuh"

namespace ckks {

typedef unsigned __int128 u128;

static thread_local std::string g_last_error = "";

int set_error(int code, const std::string &msg)
{
    g_last_error = msg;
    return code;
}

int cuda_status(cudaError_t e, const char *what)
{
    return set_error(CKKS_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

int check_ctx(const ckks_ctx *ctx)
{
    if (!ctx) return set_error(CKKS_EINVAL, "null context");
    return CKKS_OK;
}

int check_ptr(const void *p, const char *name)
{
    if (!p) return set_error(CKKS_EINVAL, std::string("null pointer: ") + name);
    if (reinterpret_cast<uintptr_t>(p) % 16 != 0)
        return set_error(CKKS_EINVAL, std::string("pointer not 16-byte aligned: ") + name);
    return CKKS_OK;
}

int set_device(const ckks_ctx *ctx)
{
    cudaError_t e = cudaSetDevice(ctx->device);
    if (e != cudaSuccess) return cuda_status(e, "cudaSetDevice");
    return CKKS_OK;
}

int resolve_ws(ckks_ctx *ctx, void *ws, size_t bytes, void **out)
{
    if (ws) {
        if (reinterpret_cast<uintptr_t>(ws) % 16 != 0)
            return set_error(CKKS_EINVAL, "workspace not 16-byte aligned");
        *out = ws;
        return CKKS_OK;
    }
    std::lock_guard<std::mutex> lock(ctx->mu);
    if (ctx->own_ws_bytes < bytes) {
        cudaError_t e = cudaDeviceSynchronize();
        if (e != cudaSuccess) return cuda_status(e, "cudaDeviceSynchronize");
        if (ctx->own_ws) cudaFree(ctx->own_ws);
        ctx->own_ws = nullptr;
        ctx->own_ws_bytes = 0;
        e = cudaMalloc(&ctx->own_ws, bytes);
        if (e != cudaSuccess) {
            ctx->own_ws = nullptr;
            cudaGetLastError();
            return set_error(CKKS_ENOMEM, "workspace allocation failed");
        }
        ctx->own_ws_bytes = bytes;
    }
    *out = ctx->own_ws;
    return CKKS_OK;
}

// ---------------------------------------------------------------- host number theory
u64 host_mulmod(u64 a, u64 b, u64 q) { return (u64)(((u128)a * b) % q); }

u64 host_powmod(u64 a, u64 e, u64 q)
{
    u64 r = 1 % q;
    a %= q;
    for (; e; e >>= 1) {
        if (e & 1) r = host_mulmod(r, a, q);
        a = host_mulmod(a, a, q);
    }
    return r;
}

// Extended Euclid; q need not be prime but gcd(a, q) must be 1.
u64 host_invmod(u64 a, u64 q)
{
    __int128 t = 0, nt = 1, r = q, nr = a % q;
    while (nr != 0) {
        __int128 quo = r / nr, tmp;
        tmp = t - quo * nt; t = nt; nt = tmp;
        tmp = r - quo * nr; r = nr; nr = tmp;
    }
    if (t < 0) t += q;
    return (u64)t;
}

u64 host_shoup(u64 w, u64 q) { return (u64)(((u128)w << 64) / q); }

bool host_is_prime(u64 m)
{
    if (m < 2) return false;
    static const u64 small[] = {2, 3, 5, 7, 11, 13, 17, 19, 23, 29, 31, 37};
    for (u64 p : small) {
        if (m % p == 0) return m == p;
    }
    u64 d = m - 1;
    int s = 0;
    while (!(d & 1)) { d >>= 1; ++s; }
    for (u64 a : small) {  // deterministic for all 64-bit m
        u64 x = host_powmod(a, d, m);
        if (x == 1 || x == m - 1) continue;
        bool comp = true;
        for (int r = 1; r < s && comp; ++r) {
            x = host_mulmod(x, x, m);
            if (x == m - 1) comp = false;
        }
        if (comp) return false;
    }
    return true;
}

// Smallest primitive 2n-th root of unity mod prime q (q = 1 mod 2n).
u64 host_find_psi(u64 q, int n)
{
    const u64 two_n = 2 * (u64)n;
    u64 root = 0;
    for (u64 g = 2; g < q && !root; ++g) {
        u64 x = host_powmod(g, (q - 1) / two_n, q);
        if (host_powmod(x, (u64)n, q) == q - 1) root = x;
    }
    // the primitive 2n-th roots are the odd powers of any one of them
    u64 best = root, sq = host_mulmod(root, root, q), cur = root;
    for (u64 k = 3; k < two_n; k += 2) {
        cur = host_mulmod(cur, sq, q);
        best = std::min(best, cur);
    }
    return best;
}

void parallel_for(int count, const std::function<void(int)> &fn)
{
    unsigned hw = std::max(1u, std::min(32u, std::thread::hardware_concurrency()));
    int nt = std::min<int>((int)hw, count);
    if (nt <= 1) {
        for (int i = 0; i < count; ++i) fn(i);
        return;
    }
    std::vector<std::thread> th;
    for (int w = 0; w < nt; ++w)
        th.emplace_back([&, w] {
            for (int i = w; i < count; i += nt) fn(i);
        });
    for (auto &x : th) x.join();
}

template <class T>
static int upload(ckks_ctx *ctx, const std::vector<T> &h, const T **dst)
{
    void *d = nullptr;
    size_t bytes = std::max<size_t>(sizeof(T), h.size() * sizeof(T));
    cudaError_t e = cudaMalloc(&d, bytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return set_error(CKKS_ENOMEM, "table allocation failed");
    }
    ctx->allocations.push_back(d);
    if (!h.empty()) {
        e = cudaMemcpy(d, h.data(), h.size() * sizeof(T), cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_status(e, "cudaMemcpy(tables)");
    }
    *dst = static_cast<const T *>(d);
    return CKKS_OK;
}

static u32 bitrev(u32 x, int bits)
{
    u32 r = 0;
    for (int i = 0; i < bits; ++i) r |= ((x >> i) & 1u) << (bits - 1 - i);
    return r;
}

// Rescale constants for input level lp1: {q_l^-1 mod q_i, Shoup} for i < l.
const ulonglong2 *rescale_table(ckks_ctx *ctx, int lp1, int *rc)
{
    std::lock_guard<std::mutex> lock(ctx->mu);
    auto it = ctx->rescale_tab.find(lp1);
    if (it != ctx->rescale_tab.end()) {
        *rc = CKKS_OK;
        return it->second;
    }
    const int l = lp1 - 1;
    std::vector<ulonglong2> h(l);
    for (int i = 0; i < l; ++i) {
        u64 qi = ctx->mods[i];
        u64 inv = host_invmod(ctx->mods[l] % qi, qi);
        h[i] = make_ulonglong2(inv, host_shoup(inv, qi));
    }
    void *d = nullptr;
    cudaError_t e = cudaMalloc(&d, std::max<size_t>(16, h.size() * sizeof(ulonglong2)));
    if (e != cudaSuccess) {
        cudaGetLastError();
        *rc = set_error(CKKS_ENOMEM, "rescale table allocation failed");
        return nullptr;
    }
    e = cudaMemcpy(d, h.data(), h.size() * sizeof(ulonglong2), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        cudaFree(d);
        *rc = cuda_status(e, "cudaMemcpy(rescale table)");
        return nullptr;
    }
    ctx->rescale_tab[lp1] = static_cast<ulonglong2 *>(d);
    *rc = CKKS_OK;
    return ctx->rescale_tab[lp1];
}

static int build_tables(ckks_ctx *ctx)
{
    const int L = ctx->L, K = ctx->K, LK = L + K, n = ctx->n, alpha = ctx->alpha;
    const int dnum = ctx->dnum;
    const std::vector<u64> &m = ctx->mods;
    Tables &T = ctx->t;
    T.L = L; T.K = K; T.alpha = alpha; T.dnum = dnum; T.LK = LK;
    T.key_L = L; T.key_LK = LK;

    std::vector<PrimeConst> pc(LK);
    std::vector<ulonglong2> fw((size_t)LK * n), iw((size_t)LK * n), iq((size_t)2 * LK);
    parallel_for(LK, [&](int t) {
        const u64 q = m[t];
        PrimeConst &c = pc[t];
        c.q = q;
        c.r64 = (u64)(((u128)1 << 64) % q);
        c.r64p = host_shoup(c.r64, q);
        c.mu64 = (u64)(((u128)1 << 64) / q);
        c.ninv = host_invmod((u64)n, q);
        c.ninvp = host_shoup(c.ninv, q);
        c.two_q = 2 * q;
        c.delta = (((u64)1 << 60) - q) < ((u64)1 << 32) ? ((u64)1 << 60) - q : 0;
        const u64 psi = host_find_psi(q, n), psi_inv = host_invmod(psi, q);
        std::vector<u64> pw(n), pwi(n);
        pw[0] = pwi[0] = 1;
        for (int k = 1; k < n; ++k) {
            pw[k] = host_mulmod(pw[k - 1], psi, q);
            pwi[k] = host_mulmod(pwi[k - 1], psi_inv, q);
        }
        ulonglong2 *f = &fw[(size_t)t * n], *v = &iw[(size_t)t * n];
        for (int k = 1; k < n; ++k) {
            u32 e = bitrev((u32)k, kLogN);
            f[k] = make_ulonglong2(pw[e], host_shoup(pw[e], q));
            v[k] = make_ulonglong2(pwi[e], host_shoup(pwi[e], q));
        }
        f[0] = make_ulonglong2(1, host_shoup(1, q));
        iq[2 * t] = make_ulonglong2(pw[n / 2], host_shoup(pw[n / 2], q));
        iq[2 * t + 1] = make_ulonglong2(q - pw[n / 2], host_shoup(q - pw[n / 2], q));
        u64 last = host_mulmod(v[1].x, c.ninv, q);  // psi^-brv(1) n^-1
        v[0] = make_ulonglong2(last, host_shoup(last, q));
    });

    // ModUp: per digit j, sources i in D_j, targets t over all primes.
    std::vector<ulonglong2> up_hatinv(L);
    std::vector<u64> up_mat((size_t)dnum * alpha * LK, 0);
    parallel_for(dnum, [&](int j) {
        const int lo = j * alpha, hi = std::min(L, lo + alpha), S = hi - lo;
        for (int i = lo; i < hi; ++i) {
            u64 prod = 1;
            for (int i2 = lo; i2 < hi; ++i2)
                if (i2 != i) prod = host_mulmod(prod, m[i2] % m[i], m[i]);
            u64 inv = host_invmod(prod, m[i]);
            up_hatinv[i] = make_ulonglong2(inv, host_shoup(inv, m[i]));
        }
        std::vector<u64> pre(S + 1), suf(S + 1);
        for (int t = 0; t < LK; ++t) {
            const u64 qt = m[t];
            pre[0] = 1 % qt;
            for (int s = 0; s < S; ++s) pre[s + 1] = host_mulmod(pre[s], m[lo + s] % qt, qt);
            suf[S] = 1 % qt;
            for (int s = S - 1; s >= 0; --s) suf[s] = host_mulmod(suf[s + 1], m[lo + s] % qt, qt);
            for (int s = 0; s < S; ++s)
                up_mat[((size_t)j * alpha + s) * LK + t] = host_mulmod(pre[s], suf[s + 1], qt);
        }
    });

    // ModDown: sources p_k, targets q_i.
    std::vector<ulonglong2> dn_hatinv(K), dn_pinv(L);
    std::vector<u64> dn_mat((size_t)K * L);
    for (int k = 0; k < K; ++k) {
        const u64 pk = m[L + k];
        u64 prod = 1;
        for (int k2 = 0; k2 < K; ++k2)
            if (k2 != k) prod = host_mulmod(prod, m[L + k2] % pk, pk);
        u64 inv = host_invmod(prod, pk);
        dn_hatinv[k] = make_ulonglong2(inv, host_shoup(inv, pk));
    }
    parallel_for(L, [&](int i) {
        const u64 qi = m[i];
        std::vector<u64> pre(K + 1), suf(K + 1);
        pre[0] = 1;
        for (int k = 0; k < K; ++k) pre[k + 1] = host_mulmod(pre[k], m[L + k] % qi, qi);
        suf[K] = 1;
        for (int k = K - 1; k >= 0; --k) suf[k] = host_mulmod(suf[k + 1], m[L + k] % qi, qi);
        for (int k = 0; k < K; ++k) dn_mat[(size_t)k * L + i] = host_mulmod(pre[k], suf[k + 1], qi);
        u64 pinv = host_invmod(pre[K], qi);
        dn_pinv[i] = make_ulonglong2(pinv, host_shoup(pinv, qi));
    });

    T.special = true;
    for (const PrimeConst &c : pc) T.special = T.special && c.delta != 0;
    CKKS_TRY(upload(ctx, pc, &T.pc));
    CKKS_TRY(upload(ctx, fw, &T.tw_fwd));
    CKKS_TRY(upload(ctx, iw, &T.tw_inv));
    CKKS_TRY(upload(ctx, iq, &T.mul_i));
    CKKS_TRY(upload(ctx, up_hatinv, &T.up_hatinv));
    CKKS_TRY(upload(ctx, up_mat, &T.up_mat));
    CKKS_TRY(upload(ctx, dn_hatinv, &T.dn_hatinv));
    CKKS_TRY(upload(ctx, dn_mat, &T.dn_mat));
    CKKS_TRY(upload(ctx, dn_pinv, &T.dn_pinv));
    CKKS_TRY(build_tc_tables(ctx, up_mat, dn_mat));
    ctx->up_mat_host = std::move(up_mat);
    ctx->dn_mat_host = std::move(dn_mat);
    return CKKS_OK;
}

static void free_ctx(ckks_ctx *ctx)
{
    for (void *p : ctx->allocations) cudaFree(p);
    for (auto &kv : ctx->rescale_tab) cudaFree(kv.second);
    free_raise_tables(ctx);
    if (ctx->own_ws) cudaFree(ctx->own_ws);
    delete ctx;
}

}  // namespace ckks

using namespace ckks;

extern "C" const char *ckks_last_error(void) { return g_last_error.c_str(); }

extern "C" int ckks_primes(int n, int count, uint64_t *out)
{
    if (!out && count > 0) return set_error(CKKS_EINVAL, "null output");
    if (count < 0) return set_error(CKKS_EINVAL, "negative count");
    if (n < 2 || n > (1 << 16) || (n & (n - 1))) return set_error(CKKS_EINVAL, "n must be a power of two");
    const u64 step = 2 * (u64)n, top = (u64)1 << 60, bottom = (u64)1 << 59;
    u64 c = (top - 1) / step * step + 1;
    for (int k = 0; k < count; c -= step) {
        if (c <= bottom) return set_error(CKKS_EUNSUPPORTED, "ran out of primes in (2^59, 2^60)");
        if (host_is_prime(c)) out[k++] = c;
    }
    return CKKS_OK;
}

extern "C" int ckks_ctx_create(const uint64_t *q, int L, const uint64_t *p, int K, int alpha,
                               int n, int device, ckks_ctx **out)
{
    if (!out) return set_error(CKKS_EINVAL, "null output pointer");
    if (!q || !p) return set_error(CKKS_EINVAL, "null prime list");
    if (n != kN) return set_error(CKKS_EUNSUPPORTED, "only n = 2048 is supported");
    if (L < 1 || L > 4096) return set_error(CKKS_EUNSUPPORTED, "L must be in [1, 4096]");
    if (K < 1 || K > kMaxDigit) return set_error(CKKS_EUNSUPPORTED, "K must be in [1, 64]");
    if (alpha < 1 || alpha > kMaxDigit || alpha > L)
        return set_error(CKKS_EUNSUPPORTED, "alpha must be in [1, min(64, L)]");
    std::vector<u64> mods(q, q + L);
    mods.insert(mods.end(), p, p + K);
    for (size_t i = 0; i < mods.size(); ++i) {
        const u64 m = mods[i];
        if (m >= ((u64)1 << 60) || m % (2 * (u64)n) != 1 || !host_is_prime(m))
            return set_error(CKKS_EINVAL, "prime " + std::to_string(i) +
                                              " is not a prime q = 1 mod 2n below 2^60");
    }
    std::vector<u64> sorted = mods;
    std::sort(sorted.begin(), sorted.end());
    if (std::adjacent_find(sorted.begin(), sorted.end()) != sorted.end())
        return set_error(CKKS_EINVAL, "primes must be distinct");
    int ndev = 0;
    cudaError_t e = cudaGetDeviceCount(&ndev);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetDeviceCount");
    if (device < 0 || device >= ndev) return set_error(CKKS_EINVAL, "no such CUDA device");
    e = cudaSetDevice(device);
    if (e != cudaSuccess) return cuda_status(e, "cudaSetDevice");

    ckks_ctx *ctx = new ckks_ctx();
    ctx->device = device;
    ctx->n = n;
    ctx->L = L;
    ctx->K = K;
    ctx->alpha = alpha;
    ctx->dnum = (L + alpha - 1) / alpha;
    ctx->mods = mods;
    int rc = build_tables(ctx);
    if (rc == CKKS_OK && L >= 2) rescale_table(ctx, L, &rc);
    if (rc != CKKS_OK) {
        free_ctx(ctx);
        return rc;
    }
    *out = ctx;
    return CKKS_OK;
}

extern "C" void ckks_ctx_destroy(ckks_ctx *ctx)
{
    if (!ctx) return;
    cudaSetDevice(ctx->device);
    cudaDeviceSynchronize();
    free_ctx(ctx);
}

extern "C" int ckks_device_status(const ckks_ctx *ctx)
{
    CKKS_TRY(check_ctx(ctx));
    CKKS_TRY(set_device(ctx));
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_status(e, "cudaDeviceSynchronize");
    if (!ctx->tc_err) return CKKS_OK;
    int flag = 0;
    e = cudaMemcpy(&flag, ctx->tc_err, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(e, "cudaMemcpy(flag)");
    if (flag) {
        cudaMemset(ctx->tc_err, 0, sizeof(int));
        return set_error(CKKS_ECUDA, "a tensor-core conversion gave up waiting for its matrix products");
    }
    return CKKS_OK;
}

extern "C" int ckks_selftest_wait_expiry(const ckks_ctx *ctx)
{
    CKKS_TRY(check_ctx(ctx));
    CKKS_TRY(set_device(ctx));
    return selftest_wait_expiry(ctx);
}

extern "C" int ckks_ctx_set_conversion(ckks_ctx *ctx, int engine)
{
    CKKS_TRY(check_ctx(ctx));
    if (engine != CKKS_CONV_AUTO && engine != CKKS_CONV_INTEGER && engine != CKKS_CONV_TENSOR &&
        engine != CKKS_CONV_FOLDED)
        return set_error(CKKS_EINVAL, "unknown conversion engine");
    ctx->conv_engine.store(engine, std::memory_order_relaxed);
    return CKKS_OK;
}

extern "C" int ckks_ctx_set_key_chain(ckks_ctx *ctx, int key_L)
{
    CKKS_TRY(check_ctx(ctx));
    if (key_L < ctx->L || key_L > 4096)
        return set_error(CKKS_EINVAL, "key_L must be in [L, 4096]");
    ctx->t.key_L = key_L;
    ctx->t.key_LK = key_L + ctx->K;
    return CKKS_OK;
}

extern "C" int ckks_ctx_params(const ckks_ctx *ctx, int *L, int *K, int *alpha, int *dnum, int *n)
{
    CKKS_TRY(check_ctx(ctx));
    if (L) *L = ctx->L;
    if (K) *K = ctx->K;
    if (alpha) *alpha = ctx->alpha;
    if (dnum) *dnum = ctx->dnum;
    if (n) *n = ctx->n;
    return CKKS_OK;
}
