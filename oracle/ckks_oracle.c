/*
 * ckks_oracle.c -- plain, slow CPU oracle for the RNS-CKKS hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product (the CUDA library, its
 * Python binding, bench.py's GPU legs) may link, load or call this file.
 * Only the test suite, the package smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or constant
 * generator with the CUDA path.
 *
 * Every operation is written as its definition: modular products are
 * (a*b) % q over unsigned __int128, sums of products are accumulated
 * exactly in 128 bits and reduced once, tables are recomputed per call.
 * OpenMP is used only as a parallel-for over independent limbs / targets;
 * it never changes the arithmetic or its order within one output.
 *
 * Sources (the pages give the parameters and the operation list, not the
 * formulas; where they are silent the plainest textbook reading is used):
 *  - Kestrel FHE relay README, section 1 ("what we are doing"): n = 2048,
 *    slots = 1024, scale 2^60, 112 RNS primes for a layer, 2100 for boot.
 *  - Kestrel engine write-up (wzjinhao.cn/news/17831), section 3 (technology
 *    table: NTT/INTT, RNS decomposition with 60-bit primes, rescale, Galois
 *    rotation, baby-step giant-step matmul, basis conversion as the core of
 *    bootstrapping) and section 4.1 (key parameters).
 *  - EncryptedLLM GPU article (m.lqnn.cn/news/239961), section 2.5 (a
 *    rotation is a transform plus a key switch; relinearisation consumes an
 *    evaluation key) and section 3.4 (NTT and basis conversion as the GPU
 *    operator core).
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes of the repository):
 *  R1 primes: q = 1 mod 2n, 2^59 < q < 2^60, scanned downward from 2^60;
 *     the first L are the ciphertext primes, the next K the special primes.
 *  R2 psi: the smallest primitive 2n-th root of unity mod q.
 *  R3 NTT: ahat[k] = sum_j a_j psi^(j (2 brv(k) + 1)), bit-reversed order.
 *  R4 automorphism: X -> X^g; slot j sits at zeta^(5^j), so g = 5^r rotates
 *     the slots left by r.
 *  R5 hybrid key switching with contiguous digits, approximate ModUp,
 *     floor ModDown.
 *  R6 keys: b_j = -a_j s + e_j + g_j s', stored [dnum][2][L+K][n].
 *  R7 rotation: ModUp(c1) first, the automorphism is applied to the
 *     extended digits, then inner product, ModDown, plus phi_g(c0).
 *  R8 rescale: floor form (c - [c]_{q_l}) / q_l.
 *  R14 bootstrapping steps (Kestrel engine write-up, the boot profile in
 *     section 5.3, names them; the forms are the textbook ones): modraise is
 *     the centred lift of each coefficient from q_0..q_{l-1} to the longer
 *     chain; conj_extract gives (ct + conj ct, X^{n/2}(conj ct - ct));
 *     restore_merge gives re + X^{n/2} im.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef uint64_t u64;
typedef int64_t i64;
typedef unsigned __int128 u128;

/* ------------------------------------------------------------------ */
/* scalar modular arithmetic (q < 2^60 throughout)                     */
/* ------------------------------------------------------------------ */

static u64 mulmod(u64 a, u64 b, u64 q) { return (u64)(((u128)a * b) % q); }
static u64 addmod(u64 a, u64 b, u64 q) { return (a + b) % q; }
static u64 submod(u64 a, u64 b, u64 q) { return (a + q - b) % q; }

static u64 powmod(u64 a, u64 e, u64 q)
{
    u64 r = 1 % q;
    a %= q;
    while (e) {
        if (e & 1) r = mulmod(r, a, q);
        a = mulmod(a, a, q);
        e >>= 1;
    }
    return r;
}

/* inverse modulo a prime, by Fermat's little theorem */
static u64 invmod(u64 a, u64 q) { return powmod(a % q, q - 2, q); }

/* reduce a signed 64-bit integer into [0, q) */
static u64 reduce_signed(i64 v, u64 q)
{
    i64 r = v % (i64)q;
    if (r < 0) r += (i64)q;
    return (u64)r;
}

/* ------------------------------------------------------------------ */
/* R1: primes                                                          */
/* ------------------------------------------------------------------ */

/* Deterministic Miller-Rabin; the first twelve prime bases decide every
 * 64-bit integer. */
int oracle_is_prime(u64 m)
{
    static const u64 bases[12] = {2, 3, 5, 7, 11, 13, 17, 19, 23, 29, 31, 37};
    if (m < 2) return 0;
    for (int i = 0; i < 12; ++i) {
        if (m == bases[i]) return 1;
        if (m % bases[i] == 0) return 0;
    }
    u64 d = m - 1;
    int s = 0;
    while ((d & 1) == 0) { d >>= 1; ++s; }
    for (int i = 0; i < 12; ++i) {
        u64 x = powmod(bases[i], d, m);
        if (x == 1 || x == m - 1) continue;
        int witness = 1;
        for (int r = 1; r < s; ++r) {
            x = mulmod(x, x, m);
            if (x == m - 1) { witness = 0; break; }
        }
        if (witness) return 0;
    }
    return 1;
}

/* The first `count` primes q = 1 (mod 2n) below 2^60, largest first. */
int oracle_gen_primes(int n, int count, u64 *out)
{
    const u64 m = 2 * (u64)n;
    const u64 top = (u64)1 << 60;
    u64 c = (top - 1) / m * m + 1;
    if (c >= top) c -= m;
    int k = 0;
    while (k < count) {
        if (c <= ((u64)1 << 59)) return -1;
        if (oracle_is_prime(c)) out[k++] = c;
        c -= m;
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* R2: the 2n-th root psi                                              */
/* ------------------------------------------------------------------ */

u64 oracle_find_psi(u64 q, int n)
{
    const u64 two_n = 2 * (u64)n;
    u64 x = 0;
    for (u64 g = 2; g < q; ++g) {
        x = powmod(g, (q - 1) / two_n, q);
        if (powmod(x, (u64)n, q) == q - 1) break;   /* order exactly 2n */
    }
    /* every primitive 2n-th root is an odd power of x; take the smallest */
    u64 best = x, x2 = mulmod(x, x, q), cur = x;
    for (u64 k = 3; k < two_n; k += 2) {
        cur = mulmod(cur, x2, q);
        if (cur < best) best = cur;
    }
    return best;
}

static int log2i(int n) { int l = 0; while ((1 << l) < n) ++l; return l; }

static u64 bitrev(u64 x, int bits)
{
    u64 r = 0;
    for (int i = 0; i < bits; ++i) r |= ((x >> i) & 1) << (bits - 1 - i);
    return r;
}

/* Per-prime tables: psi^{brv(k)} and psi^{-brv(k)} for k < n, n^{-1}. */
typedef struct {
    u64 q, psi, n_inv;
    u64 *fw;   /* fw[k] = psi^{brv(k)}  */
    u64 *iw;   /* iw[k] = psi^{-brv(k)} */
} ptab;

static void ptab_init(ptab *t, u64 q, int n)
{
    int lg = log2i(n);
    t->q = q;
    t->psi = oracle_find_psi(q, n);
    t->n_inv = invmod((u64)n, q);
    t->fw = (u64 *)malloc(sizeof(u64) * n);
    t->iw = (u64 *)malloc(sizeof(u64) * n);
    u64 psi_inv = invmod(t->psi, q);
    for (int k = 0; k < n; ++k) {
        u64 e = bitrev((u64)k, lg);
        t->fw[k] = powmod(t->psi, e, q);
        t->iw[k] = powmod(psi_inv, e, q);
    }
}

static void ptab_free(ptab *t) { free(t->fw); free(t->iw); }

static ptab *ptabs_make(const u64 *mods, int count, int n)
{
    ptab *t = (ptab *)malloc(sizeof(ptab) * (count > 0 ? count : 1));
    #pragma omp parallel for schedule(dynamic)
    for (int i = 0; i < count; ++i) ptab_init(&t[i], mods[i], n);
    return t;
}

static void ptabs_free(ptab *t, int count)
{
    for (int i = 0; i < count; ++i) ptab_free(&t[i]);
    free(t);
}

/* ------------------------------------------------------------------ */
/* R3: NTT / INTT                                                      */
/* ------------------------------------------------------------------ */

/* Definition, O(n^2): out[k] = sum_j a_j psi^{j (2 brv(k) + 1)} mod q. */
void oracle_ntt_naive(const u64 *a, u64 *out, u64 q, int n)
{
    int lg = log2i(n);
    u64 psi = oracle_find_psi(q, n);
    for (int k = 0; k < n; ++k) {
        u64 w = powmod(psi, 2 * bitrev((u64)k, lg) + 1, q);
        u64 acc = 0, wj = 1;
        for (int j = 0; j < n; ++j) {
            acc = addmod(acc, mulmod(a[j] % q, wj, q), q);
            wj = mulmod(wj, w, q);
        }
        out[k] = acc;
    }
}

/* Cooley-Tukey, natural order in, bit-reversed evaluation order out. */
static void ntt_fwd_one(u64 *a, const ptab *t, int n)
{
    const u64 q = t->q;
    for (int m = 1, h = n / 2; m < n; m *= 2, h /= 2) {
        for (int i = 0; i < m; ++i) {
            u64 w = t->fw[m + i];
            for (int j = 2 * i * h; j < 2 * i * h + h; ++j) {
                u64 u = a[j], v = mulmod(a[j + h], w, q);
                a[j] = addmod(u, v, q);
                a[j + h] = submod(u, v, q);
            }
        }
    }
}

/* Gentleman-Sande, the exact inverse of ntt_fwd_one, including n^{-1}. */
static void ntt_inv_one(u64 *a, const ptab *t, int n)
{
    const u64 q = t->q;
    for (int m = n / 2, h = 1; m >= 1; m /= 2, h *= 2) {
        for (int i = 0; i < m; ++i) {
            u64 w = t->iw[m + i];
            for (int j = 2 * i * h; j < 2 * i * h + h; ++j) {
                u64 u = a[j], v = a[j + h];
                a[j] = addmod(u, v, q);
                a[j + h] = mulmod(submod(u, v, q), w, q);
            }
        }
    }
    for (int j = 0; j < n; ++j) a[j] = mulmod(a[j], t->n_inv, q);
}

/* In place over x[batch][limbs][n]; limb l uses mods[l]. */
void oracle_ntt_fwd(u64 *x, const u64 *mods, int limbs, int batch, int n)
{
    ptab *t = ptabs_make(mods, limbs, n);
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < batch; ++b)
        for (int l = 0; l < limbs; ++l)
            ntt_fwd_one(x + ((size_t)b * limbs + l) * n, &t[l], n);
    ptabs_free(t, limbs);
}

void oracle_ntt_inv(u64 *x, const u64 *mods, int limbs, int batch, int n)
{
    ptab *t = ptabs_make(mods, limbs, n);
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < batch; ++b)
        for (int l = 0; l < limbs; ++l)
            ntt_inv_one(x + ((size_t)b * limbs + l) * n, &t[l], n);
    ptabs_free(t, limbs);
}

/* ------------------------------------------------------------------ */
/* pointwise operations in the NTT domain                              */
/* ------------------------------------------------------------------ */

/* op: 0 = a*b, 1 = a+b, 2 = a-b; arrays [batch][limbs][n] */
void oracle_pointwise(int op, const u64 *a, const u64 *b, u64 *out,
                      const u64 *mods, int limbs, int batch, int n)
{
    #pragma omp parallel for collapse(2) schedule(static)
    for (int bb = 0; bb < batch; ++bb)
        for (int l = 0; l < limbs; ++l) {
            size_t off = ((size_t)bb * limbs + l) * n;
            u64 q = mods[l];
            for (int k = 0; k < n; ++k) {
                u64 x = a[off + k], y = b[off + k];
                out[off + k] = op == 0 ? mulmod(x, y, q)
                             : op == 1 ? addmod(x, y, q) : submod(x, y, q);
            }
        }
}

/* ------------------------------------------------------------------ */
/* Galois automorphism phi_g : a(X) -> a(X^g)                         */
/* ------------------------------------------------------------------ */

/* Coefficient-domain definition, one limb: X^j -> X^{j g mod 2n}, with a
 * sign flip when the exponent lands in [n, 2n) because X^n = -1. */
void oracle_automorph_coeff(const u64 *in, u64 *out, u64 q, int n, u64 g)
{
    const u64 two_n = 2 * (u64)n;
    for (int j = 0; j < n; ++j) out[j] = 0;
    for (int j = 0; j < n; ++j) {
        u64 e = ((u64)j * g) % two_n;
        if (e < (u64)n) out[e] = addmod(out[e], in[j], q);
        else out[e - n] = submod(out[e - n], in[j], q);
    }
}

/* NTT-domain index map: slot k holds a(psi^{2 brv(k)+1}); phi_g(a) there
 * equals a(psi^{g (2 brv(k)+1)}), found at the slot k' whose odd exponent
 * 2 brv(k')+1 equals g (2 brv(k)+1) mod 2n. */
static int automorph_src(int k, u64 g, int n)
{
    int lg = log2i(n);
    u64 e = (g * (2 * bitrev((u64)k, lg) + 1)) % (2 * (u64)n);
    return (int)bitrev((e - 1) / 2, lg);
}

/* x[batch][limbs][n] in the NTT domain */
void oracle_automorph_ntt(const u64 *in, u64 *out, int limbs, int batch,
                          int n, u64 g)
{
    int *src = (int *)malloc(sizeof(int) * n);
    for (int k = 0; k < n; ++k) src[k] = automorph_src(k, g, n);
    for (size_t r = 0; r < (size_t)batch * limbs; ++r)
        for (int k = 0; k < n; ++k) out[r * n + k] = in[r * n + src[k]];
    free(src);
}

/* ------------------------------------------------------------------ */
/* R5: hybrid key switching                                            */
/* ------------------------------------------------------------------ */

/* mods = q_0..q_{L-1}, p_0..p_{K-1}; digit j covers q_{j alpha} ..
 * q_{min((j+1) alpha, L) - 1}. */
static int digit_count(int L, int alpha) { return (L + alpha - 1) / alpha; }

/* Fast basis conversion, coefficient domain (approximate: no overflow
 * correction).  For source primes s_0..s_{S-1} with product S_all, input
 * residues x_i of one integer X in [0, S_all):
 *     y_i  = [x_i * (S_all/s_i)^{-1}]_{s_i}
 *     out_t = sum_i y_i * [S_all/s_i]_t   mod t
 * which equals X + u S_all (mod t) with an integer 0 <= u < S. */
void oracle_basis_convert(const u64 *x /*[S][n]*/, const u64 *src, int S,
                          u64 *out /*[T][n]*/, const u64 *dst, int T, int n)
{
    u64 *hat_inv = (u64 *)malloc(sizeof(u64) * (S > 0 ? S : 1));
    u64 *hat = (u64 *)malloc(sizeof(u64) * (size_t)(S > 0 ? S : 1) * (T > 0 ? T : 1));
    u64 *y = (u64 *)malloc(sizeof(u64) * (size_t)(S > 0 ? S : 1) * n);
    for (int i = 0; i < S; ++i) {
        u64 prod = 1;
        for (int i2 = 0; i2 < S; ++i2)
            if (i2 != i) prod = mulmod(prod, src[i2] % src[i], src[i]);
        hat_inv[i] = invmod(prod, src[i]);
        for (int t = 0; t < T; ++t) {
            u64 pt = 1;
            for (int i2 = 0; i2 < S; ++i2)
                if (i2 != i) pt = mulmod(pt, src[i2] % dst[t], dst[t]);
            hat[(size_t)i * T + t] = pt;
        }
    }
    for (int i = 0; i < S; ++i)
        for (int k = 0; k < n; ++k)
            y[(size_t)i * n + k] = mulmod(x[(size_t)i * n + k], hat_inv[i], src[i]);
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t)
        for (int k = 0; k < n; ++k) {
            u128 acc = 0;       /* S products < 2^120 each: exact for S < 256 */
            for (int i = 0; i < S; ++i)
                acc += (u128)y[(size_t)i * n + k] * hat[(size_t)i * T + t];
            out[(size_t)t * n + k] = (u64)(acc % dst[t]);
        }
    free(hat_inv); free(hat); free(y);
}

/* ModUp of one polynomial: c_ntt[L][n] (NTT domain over q) ->
 * digits[dnum][L+K][n] (NTT domain over q and p).  Digit j's own limbs are
 * copies of the input; the others come from basis conversion of the
 * digit's coefficients followed by a forward NTT. */
static void modup_one(const u64 *c_ntt, u64 *digits, const u64 *mods,
                      const ptab *tabs, int L, int K, int alpha, int n)
{
    const int dnum = digit_count(L, alpha), LK = L + K;
    u64 *coef = (u64 *)malloc(sizeof(u64) * (size_t)L * n);
    memcpy(coef, c_ntt, sizeof(u64) * (size_t)L * n);
    #pragma omp parallel for schedule(static)
    for (int l = 0; l < L; ++l) ntt_inv_one(coef + (size_t)l * n, &tabs[l], n);

    for (int j = 0; j < dnum; ++j) {
        int lo = j * alpha, hi = lo + alpha < L ? lo + alpha : L, S = hi - lo;
        int T = LK - S;
        u64 *dst = (u64 *)malloc(sizeof(u64) * T);
        int *dst_idx = (int *)malloc(sizeof(int) * T);
        for (int t = 0, c = 0; t < LK; ++t)
            if (t < lo || t >= hi) { dst[c] = mods[t]; dst_idx[c] = t; ++c; }
        u64 *conv = (u64 *)malloc(sizeof(u64) * (size_t)T * n);
        oracle_basis_convert(coef + (size_t)lo * n, mods + lo, S, conv, dst, T, n);
        u64 *dj = digits + (size_t)j * LK * n;
        #pragma omp parallel for schedule(static)
        for (int c = 0; c < T; ++c) {
            u64 *row = dj + (size_t)dst_idx[c] * n;
            memcpy(row, conv + (size_t)c * n, sizeof(u64) * n);
            ntt_fwd_one(row, &tabs[dst_idx[c]], n);
        }
        for (int t = lo; t < hi; ++t)
            memcpy(dj + (size_t)t * n, c_ntt + (size_t)t * n, sizeof(u64) * n);
        free(dst); free(dst_idx); free(conv);
    }
    free(coef);
}

void oracle_modup(const u64 *c_ntt /*[B][L][n]*/, u64 *digits /*[B][dnum][L+K][n]*/,
                  const u64 *mods, int L, int K, int alpha, int batch, int n)
{
    const int dnum = digit_count(L, alpha), LK = L + K;
    ptab *tabs = ptabs_make(mods, LK, n);
    for (int b = 0; b < batch; ++b)
        modup_one(c_ntt + (size_t)b * L * n, digits + (size_t)b * dnum * LK * n,
                  mods, tabs, L, K, alpha, n);
    ptabs_free(tabs, LK);
}

/* Key inner product with the automorphism applied to the digits:
 * acc_c[t][k] = sum_j phi_g(D_j)[t][k] * key[j][c][t][k]  mod t. */
static void inner_one(const u64 *digits, const u64 *key, u64 g, u64 *acc,
                      const u64 *mods, int L, int K, int alpha, int n)
{
    const int dnum = digit_count(L, alpha), LK = L + K;
    int *src = (int *)malloc(sizeof(int) * n);
    for (int k = 0; k < n; ++k) src[k] = automorph_src(k, g, n);
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < LK; ++t)
        for (int c = 0; c < 2; ++c)
            for (int k = 0; k < n; ++k) {
                u128 s = 0;   /* dnum products < 2^120: exact for dnum < 256 */
                for (int j = 0; j < dnum; ++j) {
                    u64 d = digits[((size_t)j * LK + t) * n + src[k]];
                    u64 kv = key[(((size_t)j * 2 + c) * LK + t) * n + k];
                    s += (u128)d * kv;
                }
                acc[((size_t)c * LK + t) * n + k] = (u64)(s % mods[t]);
            }
    free(src);
}

void oracle_key_inner(const u64 *digits /*[B][dnum][L+K][n]*/,
                      const u64 *key /*[dnum][2][L+K][n]*/, u64 galois,
                      u64 *acc /*[B][2][L+K][n]*/, const u64 *mods,
                      int L, int K, int alpha, int batch, int n)
{
    const int dnum = digit_count(L, alpha), LK = L + K;
    for (int b = 0; b < batch; ++b)
        inner_one(digits + (size_t)b * dnum * LK * n, key, galois,
                  acc + (size_t)b * 2 * LK * n, mods, L, K, alpha, n);
}

/* ModDown of one polynomial pair acc[2][L+K][n] -> out[2][L][n]:
 * x = INTT of the special limbs, conv = basis conversion P -> q_i,
 * out_i = (acc_i - NTT(conv_i)) * P^{-1}  mod q_i. */
static void moddown_one(const u64 *acc, u64 *out, const u64 *mods,
                        const ptab *tabs, int L, int K, int n)
{
    const int LK = L + K;
    u64 *sp = (u64 *)malloc(sizeof(u64) * (size_t)K * n);
    u64 *conv = (u64 *)malloc(sizeof(u64) * (size_t)L * n);
    u64 *pinv = (u64 *)malloc(sizeof(u64) * L);
    for (int i = 0; i < L; ++i) {
        u64 P = 1;
        for (int k = 0; k < K; ++k) P = mulmod(P, mods[L + k] % mods[i], mods[i]);
        pinv[i] = invmod(P, mods[i]);
    }
    for (int c = 0; c < 2; ++c) {
        const u64 *a = acc + (size_t)c * LK * n;
        memcpy(sp, a + (size_t)L * n, sizeof(u64) * (size_t)K * n);
        for (int k = 0; k < K; ++k) ntt_inv_one(sp + (size_t)k * n, &tabs[L + k], n);
        oracle_basis_convert(sp, mods + L, K, conv, mods, L, n);
        #pragma omp parallel for schedule(static)
        for (int i = 0; i < L; ++i) {
            u64 *ci = conv + (size_t)i * n;
            ntt_fwd_one(ci, &tabs[i], n);
            for (int k = 0; k < n; ++k)
                out[((size_t)c * L + i) * n + k] =
                    mulmod(submod(a[(size_t)i * n + k], ci[k], mods[i]), pinv[i], mods[i]);
        }
    }
    free(sp); free(conv); free(pinv);
}

void oracle_moddown(const u64 *acc /*[B][2][L+K][n]*/, u64 *out /*[B][2][L][n]*/,
                    const u64 *mods, int L, int K, int batch, int n)
{
    ptab *tabs = ptabs_make(mods, L + K, n);
    for (int b = 0; b < batch; ++b)
        moddown_one(acc + (size_t)b * 2 * (L + K) * n, out + (size_t)b * 2 * L * n,
                    mods, tabs, L, K, n);
    ptabs_free(tabs, L + K);
}

/* KeySwitch(d) = ModDown(<ModUp(d), key>), no automorphism. */
void oracle_keyswitch(const u64 *d /*[B][L][n]*/, const u64 *key,
                      u64 *out /*[B][2][L][n]*/, const u64 *mods,
                      int L, int K, int alpha, int batch, int n)
{
    const int dnum = digit_count(L, alpha), LK = L + K;
    ptab *tabs = ptabs_make(mods, LK, n);
    u64 *dig = (u64 *)malloc(sizeof(u64) * (size_t)dnum * LK * n);
    u64 *acc = (u64 *)malloc(sizeof(u64) * (size_t)2 * LK * n);
    for (int b = 0; b < batch; ++b) {
        modup_one(d + (size_t)b * L * n, dig, mods, tabs, L, K, alpha, n);
        inner_one(dig, key, 1, acc, mods, L, K, alpha, n);
        moddown_one(acc, out + (size_t)b * 2 * L * n, mods, tabs, L, K, n);
    }
    free(dig); free(acc);
    ptabs_free(tabs, LK);
}

/* R7 rotation with hoisted ModUp: for every key r,
 * out[r][b] = (phi_g(c0) + KS0, KS1), KS = ModDown(<phi_g(ModUp(c1)), key_r>). */
void oracle_rotate(const u64 *ct /*[B][2][L][n]*/, const u64 *const *keys,
                   const u64 *galois, int nkeys, u64 *out /*[nkeys][B][2][L][n]*/,
                   const u64 *mods, int L, int K, int alpha, int batch, int n)
{
    const int dnum = digit_count(L, alpha), LK = L + K;
    ptab *tabs = ptabs_make(mods, LK, n);
    u64 *dig = (u64 *)malloc(sizeof(u64) * (size_t)dnum * LK * n);
    u64 *acc = (u64 *)malloc(sizeof(u64) * (size_t)2 * LK * n);
    u64 *ks = (u64 *)malloc(sizeof(u64) * (size_t)2 * L * n);
    u64 *rot0 = (u64 *)malloc(sizeof(u64) * (size_t)L * n);
    for (int b = 0; b < batch; ++b) {
        const u64 *c0 = ct + (size_t)b * 2 * L * n, *c1 = c0 + (size_t)L * n;
        modup_one(c1, dig, mods, tabs, L, K, alpha, n);
        for (int r = 0; r < nkeys; ++r) {
            inner_one(dig, keys[r], galois[r], acc, mods, L, K, alpha, n);
            moddown_one(acc, ks, mods, tabs, L, K, n);
            oracle_automorph_ntt(c0, rot0, L, 1, n, galois[r]);
            u64 *o = out + ((size_t)r * batch + b) * 2 * L * n;
            for (int i = 0; i < L; ++i)
                for (int k = 0; k < n; ++k) {
                    size_t at = (size_t)i * n + k;
                    o[at] = addmod(rot0[at], ks[at], mods[i]);
                    o[(size_t)L * n + at] = ks[(size_t)L * n + at];
                }
        }
    }
    free(dig); free(acc); free(ks); free(rot0);
    ptabs_free(tabs, LK);
}

/* The other rotation order (automorphism first, no hoisting): for every key,
 * phi_g(c1) is key-switched with the Galois key -- ModUp of the rotated c1,
 * inner product without a gather, ModDown -- and phi_g(c0) is added.  The
 * Galois key is the same (it switches from phi_g(s) to s); the approximate
 * ModUp of phi_g(c1) is not phi_g of the ModUp of c1, so the low bits differ
 * from oracle_rotate while both decrypt to the rotated slots. */
void oracle_rotate_unhoisted(const u64 *ct /*[B][2][L][n]*/, const u64 *const *keys,
                             const u64 *galois, int nkeys, u64 *out /*[nkeys][B][2][L][n]*/,
                             const u64 *mods, int L, int K, int alpha, int batch, int n)
{
    const int dnum = digit_count(L, alpha), LK = L + K;
    ptab *tabs = ptabs_make(mods, LK, n);
    u64 *dig = (u64 *)malloc(sizeof(u64) * (size_t)dnum * LK * n);
    u64 *acc = (u64 *)malloc(sizeof(u64) * (size_t)2 * LK * n);
    u64 *ks = (u64 *)malloc(sizeof(u64) * (size_t)2 * L * n);
    u64 *rot0 = (u64 *)malloc(sizeof(u64) * (size_t)L * n);
    u64 *rot1 = (u64 *)malloc(sizeof(u64) * (size_t)L * n);
    for (int b = 0; b < batch; ++b) {
        const u64 *c0 = ct + (size_t)b * 2 * L * n, *c1 = c0 + (size_t)L * n;
        for (int r = 0; r < nkeys; ++r) {
            oracle_automorph_ntt(c1, rot1, L, 1, n, galois[r]);
            modup_one(rot1, dig, mods, tabs, L, K, alpha, n);
            inner_one(dig, keys[r], 1, acc, mods, L, K, alpha, n);
            moddown_one(acc, ks, mods, tabs, L, K, n);
            oracle_automorph_ntt(c0, rot0, L, 1, n, galois[r]);
            u64 *o = out + ((size_t)r * batch + b) * 2 * L * n;
            for (int i = 0; i < L; ++i)
                for (int k = 0; k < n; ++k) {
                    size_t at = (size_t)i * n + k;
                    o[at] = addmod(rot0[at], ks[at], mods[i]);
                    o[(size_t)L * n + at] = ks[(size_t)L * n + at];
                }
        }
    }
    free(dig); free(acc); free(ks); free(rot0); free(rot1);
    ptabs_free(tabs, LK);
}

/* ------------------------------------------------------------------ */
/* R8: rescale                                                         */
/* ------------------------------------------------------------------ */

/* ct[B][2][l+1][n] -> out[B][2][l][n]: c'_i = (c_i - NTT_{q_i}([c]_{q_l})) q_l^{-1}.
 * Coefficients of the dropped limb lie in [0, q_l) and are reduced mod q_i. */
void oracle_rescale(const u64 *ct, u64 *out, const u64 *mods, int lp1,
                    int batch, int n)
{
    const int l = lp1 - 1;
    ptab *tabs = ptabs_make(mods, lp1, n);
    u64 *last = (u64 *)malloc(sizeof(u64) * n);
    for (int b = 0; b < batch; ++b)
        for (int c = 0; c < 2; ++c) {
            const u64 *in = ct + ((size_t)b * 2 + c) * lp1 * n;
            u64 *o = out + ((size_t)b * 2 + c) * l * n;
            memcpy(last, in + (size_t)l * n, sizeof(u64) * n);
            ntt_inv_one(last, &tabs[l], n);
            #pragma omp parallel for schedule(static)
            for (int i = 0; i < l; ++i) {
                u64 qi = mods[i];
                u64 inv = invmod(mods[l] % qi, qi);
                u64 *row = o + (size_t)i * n;
                for (int k = 0; k < n; ++k) row[k] = last[k] % qi;
                ntt_fwd_one(row, &tabs[i], n);
                for (int k = 0; k < n; ++k)
                    row[k] = mulmod(submod(in[(size_t)i * n + k], row[k], qi), inv, qi);
            }
        }
    free(last);
    ptabs_free(tabs, lp1);
}

/* ------------------------------------------------------------------ */
/* ct x ct multiply, relinearisation, rescale                          */
/* ------------------------------------------------------------------ */

/* a, b [B][2][L][n]; rlk [dnum][2][L+K][n]; out [B][2][L-1][n].
 * d0 = a0 b0, d1 = a0 b1 + a1 b0, d2 = a1 b1; (d0, d1) + KeySwitch(d2);
 * then rescale by q_{L-1}. */
void oracle_mul_relin_rescale(const u64 *a, const u64 *b, const u64 *rlk,
                              u64 *out, const u64 *mods, int L, int K,
                              int alpha, int batch, int n)
{
    const size_t Ln = (size_t)L * n;
    u64 *d = (u64 *)malloc(sizeof(u64) * 3 * Ln);
    u64 *ks = (u64 *)malloc(sizeof(u64) * 2 * Ln);
    u64 *c = (u64 *)malloc(sizeof(u64) * 2 * Ln);
    for (int bb = 0; bb < batch; ++bb) {
        const u64 *a0 = a + (size_t)bb * 2 * Ln, *a1 = a0 + Ln;
        const u64 *b0 = b + (size_t)bb * 2 * Ln, *b1 = b0 + Ln;
        for (int i = 0; i < L; ++i) {
            u64 q = mods[i];
            for (int k = 0; k < n; ++k) {
                size_t at = (size_t)i * n + k;
                d[at] = mulmod(a0[at], b0[at], q);
                d[Ln + at] = addmod(mulmod(a0[at], b1[at], q), mulmod(a1[at], b0[at], q), q);
                d[2 * Ln + at] = mulmod(a1[at], b1[at], q);
            }
        }
        oracle_keyswitch(d + 2 * Ln, rlk, ks, mods, L, K, alpha, 1, n);
        for (int i = 0; i < L; ++i)
            for (int k = 0; k < n; ++k) {
                size_t at = (size_t)i * n + k;
                c[at] = addmod(d[at], ks[at], mods[i]);
                c[Ln + at] = addmod(d[Ln + at], ks[Ln + at], mods[i]);
            }
        oracle_rescale(c, out + (size_t)bb * 2 * (L - 1) * n, mods, L, 1, n);
    }
    free(d); free(ks); free(c);
}

/* ------------------------------------------------------------------ */
/* baby-step giant-step diagonal matrix-vector product                 */
/* ------------------------------------------------------------------ */

static u64 galois_power(u64 r, int n)
{
    return powmod(5, r, 2 * (u64)n);
}

/* x [B][2][L][n]; diags [gg][bb][L][n] (pt_{g,b}, NTT domain);
 * baby_keys[b-1] rotates by b (galois 5^b), b = 1..bb-1;
 * giant_keys[g-1] rotates by bb*g (galois 5^{bb g}), g = 1..gg-1;
 * y [B][2][L-1][n] = Rescale( sum_g Rot_{bb g}( sum_b pt_{g,b} * Rot_b(x) ) ). */
void oracle_bsgs(const u64 *x, const u64 *diags, const u64 *const *baby_keys,
                 const u64 *const *giant_keys, int bb, int gg, u64 *y,
                 const u64 *mods, int L, int K, int alpha, int batch, int n)
{
    const size_t Ln = (size_t)L * n, ctsz = 2 * Ln;
    u64 *baby = (u64 *)malloc(sizeof(u64) * (size_t)bb * ctsz);
    u64 *inner = (u64 *)malloc(sizeof(u64) * ctsz);
    u64 *acc = (u64 *)malloc(sizeof(u64) * ctsz);
    u64 *rot = (u64 *)malloc(sizeof(u64) * ctsz);
    u64 *galb = (u64 *)malloc(sizeof(u64) * (bb > 1 ? bb - 1 : 1));
    for (int r = 1; r < bb; ++r) galb[r - 1] = galois_power((u64)r, n);
    for (int b = 0; b < batch; ++b) {
        const u64 *xb = x + (size_t)b * ctsz;
        memcpy(baby, xb, sizeof(u64) * ctsz);
        if (bb > 1)
            oracle_rotate(xb, baby_keys, galb, bb - 1, baby + ctsz, mods, L, K, alpha, 1, n);
        memset(acc, 0, sizeof(u64) * ctsz);
        for (int g = 0; g < gg; ++g) {
            memset(inner, 0, sizeof(u64) * ctsz);
            for (int r = 0; r < bb; ++r) {
                const u64 *pt = diags + ((size_t)g * bb + r) * Ln;
                const u64 *br = baby + (size_t)r * ctsz;
                for (int c = 0; c < 2; ++c)
                    for (int i = 0; i < L; ++i)
                        for (int k = 0; k < n; ++k) {
                            size_t at = (size_t)i * n + k;
                            u64 q = mods[i];
                            inner[c * Ln + at] = addmod(inner[c * Ln + at],
                                                        mulmod(pt[at], br[c * Ln + at], q), q);
                        }
            }
            const u64 *term = inner;
            if (g > 0) {
                u64 gal = galois_power((u64)bb * g, n);
                const u64 *key = giant_keys[g - 1];
                oracle_rotate(inner, &key, &gal, 1, rot, mods, L, K, alpha, 1, n);
                term = rot;
            }
            for (int c = 0; c < 2; ++c)
                for (int i = 0; i < L; ++i)
                    for (int k = 0; k < n; ++k) {
                        size_t at = c * Ln + (size_t)i * n + k;
                        acc[at] = addmod(acc[at], term[at], mods[i]);
                    }
        }
        oracle_rescale(acc, y + (size_t)b * 2 * (L - 1) * n, mods, L, 1, n);
    }
    free(baby); free(inner); free(acc); free(rot); free(galb);
}

/* ------------------------------------------------------------------ */
/* R14: the bootstrapping steps around the two linear transforms       */
/* ------------------------------------------------------------------ */

/* Multiplication by the monomial X^e, 0 <= e < 2n, in Z_q[X]/(X^n + 1),
 * coefficient domain, one limb: X^j goes to X^{j+e}, negated once for every
 * time the exponent passes n (X^n = -1). */
static void monomial_coeff(const u64 *in, u64 *out, u64 q, int n, int e)
{
    for (int j = 0; j < n; ++j) {
        int t = j + e;
        int neg = 0;
        while (t >= n) { t -= n; neg ^= 1; }
        out[t] = neg ? submod(0, in[j], q) : in[j] % q;
    }
}

/* x[batch][limbs][n] NTT domain -> X^e * x, NTT domain: INTT, the
 * coefficient shift above, NTT. */
void oracle_mul_monomial(const u64 *in, u64 *out, const u64 *mods, int limbs,
                         int batch, int n, int e)
{
    ptab *tabs = ptabs_make(mods, limbs, n);
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < batch; ++b)
        for (int l = 0; l < limbs; ++l) {
            size_t off = ((size_t)b * limbs + l) * n;
            u64 *tmp = (u64 *)malloc(sizeof(u64) * n);
            memcpy(tmp, in + off, sizeof(u64) * n);
            ntt_inv_one(tmp, &tabs[l], n);
            monomial_coeff(tmp, out + off, mods[l], n, e);
            ntt_fwd_one(out + off, &tabs[l], n);
            free(tmp);
        }
    ptabs_free(tabs, limbs);
}

/* ModRaise: polynomials x[P][l][n] over q_0..q_{l-1} (NTT domain) ->
 * out[P][Lf][n] over q_0..q_{Lf-1} (NTT domain), Lf >= l.  Each coefficient
 * is read as the centred integer X in (-Q/2, Q/2], Q = q_0 ... q_{l-1}, and
 * X is reduced modulo every prime of the longer chain.
 *
 * X is found in Garner's mixed-radix form X = d_0 + d_1 q_0 + d_2 q_0 q_1 +
 * ..., with digits d_i in [0, q_i): d_i = (...((x_i - d_0) q_0^{-1} - d_1)
 * q_1^{-1} ... - d_{i-1}) q_{i-1}^{-1} mod q_i.  H = (Q - 1) / 2 has residue
 * (q_i - 1) / 2 at every q_i (2H = -1 mod q_i); X > H is decided by comparing
 * the two digit strings from the most significant digit down, and in that
 * case Q is subtracted.  X mod p is evaluated from the digits by Horner's
 * rule.  Only word-size modular arithmetic is involved. */
void oracle_modraise(const u64 *x, u64 *out, const u64 *mods, int l, int Lf,
                     int P, int n)
{
    ptab *tabs = ptabs_make(mods, Lf, n);
    /* inv[i][k] = q_k^{-1} mod q_i, k < i */
    u64 *inv = (u64 *)malloc(sizeof(u64) * (size_t)l * l);
    for (int i = 0; i < l; ++i)
        for (int k = 0; k < i; ++k) inv[(size_t)i * l + k] = invmod(mods[k] % mods[i], mods[i]);
    /* Garner digits of H = (Q - 1) / 2 */
    u64 *hd = (u64 *)malloc(sizeof(u64) * l);
    for (int i = 0; i < l; ++i) {
        u64 t = (mods[i] - 1) / 2;
        for (int k = 0; k < i; ++k)
            t = mulmod(submod(t, hd[k] % mods[i], mods[i]), inv[(size_t)i * l + k], mods[i]);
        hd[i] = t;
    }
    /* Q mod p for every prime of the longer chain */
    u64 *qmod = (u64 *)malloc(sizeof(u64) * Lf);
    for (int t = 0; t < Lf; ++t) {
        u64 r = 1 % mods[t];
        for (int i = 0; i < l; ++i) r = mulmod(r, mods[i] % mods[t], mods[t]);
        qmod[t] = r;
    }
    for (int pi = 0; pi < P; ++pi) {
        const u64 *src = x + (size_t)pi * l * n;
        u64 *dst = out + (size_t)pi * Lf * n;
        u64 *coef = (u64 *)malloc(sizeof(u64) * (size_t)l * n);
        memcpy(coef, src, sizeof(u64) * (size_t)l * n);
        #pragma omp parallel for schedule(static)
        for (int i = 0; i < l; ++i) ntt_inv_one(coef + (size_t)i * n, &tabs[i], n);
        #pragma omp parallel for schedule(static)
        for (int k = 0; k < n; ++k) {
            u64 d[l > 0 ? l : 1];
            for (int i = 0; i < l; ++i) {
                u64 t = coef[(size_t)i * n + k];
                for (int j = 0; j < i; ++j)
                    t = mulmod(submod(t, d[j] % mods[i], mods[i]), inv[(size_t)i * l + j], mods[i]);
                d[i] = t;
            }
            int neg = 0;
            for (int i = l - 1; i >= 0; --i)
                if (d[i] != hd[i]) { neg = d[i] > hd[i]; break; }
            for (int t = l; t < Lf; ++t) {
                u64 p = mods[t], r = 0;
                for (int i = l - 1; i >= 0; --i)
                    r = addmod(mulmod(r, mods[i] % p, p), d[i] % p, p);
                if (neg) r = submod(r, qmod[t], p);
                dst[(size_t)t * n + k] = r;
            }
        }
        #pragma omp parallel for schedule(static)
        for (int t = l; t < Lf; ++t) ntt_fwd_one(dst + (size_t)t * n, &tabs[t], n);
        /* below q_l the centred integer keeps its residues */
        memcpy(dst, src, sizeof(u64) * (size_t)l * n);
        free(coef);
    }
    free(inv); free(hd); free(qmod);
    ptabs_free(tabs, Lf);
}

/* conj_extract: ct[B][2][L][n] with slots w -> re, im [B][2][L][n] with
 * slots 2 Re(w) and 2 Im(w), at the input's scale:
 *     c* = the conjugate of ct (hoisted rotation by g = 2n - 1, key conj_key),
 *     re = ct + c*,   im = X^{n/2} (c* - ct).
 * X^{n/2} multiplies every slot by i (slot j sits at zeta^{5^j} and 5^j = 1
 * mod 4), so im's slots are i (conj(w) - w) = 2 Im(w). */
void oracle_conj_extract(const u64 *ct, const u64 *conj_key, u64 *re, u64 *im,
                         const u64 *mods, int L, int K, int alpha, int batch, int n)
{
    const size_t csz = (size_t)2 * L * n;
    u64 *cj = (u64 *)malloc(sizeof(u64) * csz);
    u64 *dif = (u64 *)malloc(sizeof(u64) * csz);
    const u64 g = 2 * (u64)n - 1;
    for (int b = 0; b < batch; ++b) {
        const u64 *c = ct + (size_t)b * csz;
        const u64 *keys[1] = {conj_key};
        oracle_rotate(c, keys, &g, 1, cj, mods, L, K, alpha, 1, n);
        for (size_t at = 0; at < csz; ++at) {
            u64 q = mods[(at / n) % L];
            re[(size_t)b * csz + at] = addmod(c[at], cj[at], q);
            dif[at] = submod(cj[at], c[at], q);
        }
        for (int comp = 0; comp < 2; ++comp)
            oracle_mul_monomial(dif + (size_t)comp * L * n,
                                im + (size_t)b * csz + (size_t)comp * L * n, mods, L, 1, n, n / 2);
    }
    free(cj); free(dif);
}

/* restore_merge: re, im [B][2][L][n] with slots a, b -> re + X^{n/2} im,
 * whose slots are a + i b. */
void oracle_restore_merge(const u64 *re, const u64 *im, u64 *out, const u64 *mods,
                          int L, int batch, int n)
{
    const size_t csz = (size_t)2 * L * n;
    u64 *sh = (u64 *)malloc(sizeof(u64) * csz);
    for (int b = 0; b < batch; ++b) {
        for (int comp = 0; comp < 2; ++comp)
            oracle_mul_monomial(im + (size_t)b * csz + (size_t)comp * L * n,
                                sh + (size_t)comp * L * n, mods, L, 1, n, n / 2);
        for (size_t at = 0; at < csz; ++at)
            out[(size_t)b * csz + at] = addmod(re[(size_t)b * csz + at], sh[at],
                                               mods[(at / n) % L]);
    }
    free(sh);
}

/* ------------------------------------------------------------------ */
/* keys, encryption, decryption (host-side utilities of the scheme)    */
/* ------------------------------------------------------------------ */

/* small signed coefficients -> NTT residues over mods[0..limbs) */
static void small_to_ntt(const i64 *v, u64 *out, const u64 *mods,
                         const ptab *tabs, int limbs, int n)
{
    #pragma omp parallel for schedule(static)
    for (int l = 0; l < limbs; ++l) {
        u64 *row = out + (size_t)l * n;
        for (int k = 0; k < n; ++k) row[k] = reduce_signed(v[k], mods[l]);
        ntt_fwd_one(row, &tabs[l], n);
    }
}

/* Switching key from s' to s (R6):  key[j][0] = -a_j s + e_j + g_j s',
 * key[j][1] = a_j over all L+K primes, NTT domain.  g_j is P on the limbs of
 * digit j and 0 elsewhere (0 on every special prime).
 * s: ternary secret coefficients [n]; sprime_ntt: s' as NTT residues
 * [L+K][n]; a: uniform NTT residues [dnum][L+K][n]; e: error coefficients
 * [dnum][n]. */
void oracle_keygen(const i64 *s, const u64 *sprime_ntt, const u64 *a,
                   const i64 *e, u64 *key, const u64 *mods, int L, int K,
                   int alpha, int n)
{
    const int dnum = digit_count(L, alpha), LK = L + K;
    ptab *tabs = ptabs_make(mods, LK, n);
    u64 *s_ntt = (u64 *)malloc(sizeof(u64) * (size_t)LK * n);
    u64 *e_ntt = (u64 *)malloc(sizeof(u64) * (size_t)LK * n);
    small_to_ntt(s, s_ntt, mods, tabs, LK, n);
    for (int j = 0; j < dnum; ++j) {
        int lo = j * alpha, hi = lo + alpha < L ? lo + alpha : L;
        small_to_ntt(e + (size_t)j * n, e_ntt, mods, tabs, LK, n);
        #pragma omp parallel for schedule(static)
        for (int t = 0; t < LK; ++t) {
            u64 q = mods[t];
            u64 gj = 0;
            if (t >= lo && t < hi) {
                gj = 1;
                for (int k = 0; k < K; ++k) gj = mulmod(gj, mods[L + k] % q, q);
            }
            for (int k = 0; k < n; ++k) {
                size_t at = (size_t)t * n + k;
                u64 av = a[(size_t)j * LK * n + at];
                u64 bv = submod(e_ntt[at], mulmod(av, s_ntt[at], q), q);
                bv = addmod(bv, mulmod(gj, sprime_ntt[at], q), q);
                key[(((size_t)j * 2 + 0) * LK) * n + at] = bv;
                key[(((size_t)j * 2 + 1) * LK) * n + at] = av;
            }
        }
    }
    free(s_ntt); free(e_ntt);
    ptabs_free(tabs, LK);
}

/* s' = phi_g(s) as NTT residues over mods[0..limbs) */
void oracle_secret_galois(const i64 *s, u64 g, u64 *out, const u64 *mods,
                          int limbs, int n)
{
    ptab *tabs = ptabs_make(mods, limbs, n);
    u64 *tmp = (u64 *)malloc(sizeof(u64) * n);
    for (int l = 0; l < limbs; ++l) {
        for (int k = 0; k < n; ++k) tmp[k] = reduce_signed(s[k], mods[l]);
        oracle_automorph_coeff(tmp, out + (size_t)l * n, mods[l], n, g);
        ntt_fwd_one(out + (size_t)l * n, &tabs[l], n);
    }
    free(tmp);
    ptabs_free(tabs, limbs);
}

/* s' = s^2 as NTT residues over mods[0..limbs) */
void oracle_secret_square(const i64 *s, u64 *out, const u64 *mods, int limbs, int n)
{
    ptab *tabs = ptabs_make(mods, limbs, n);
    small_to_ntt(s, out, mods, tabs, limbs, n);
    for (size_t at = 0; at < (size_t)limbs * n; ++at)
        out[at] = mulmod(out[at], out[at], mods[at / n]);
    ptabs_free(tabs, limbs);
}

/* Secret-key encryption: c1 = a, c0 = -a s + e + m (NTT domain, L limbs).
 * m, e: signed coefficients [n]; a: uniform NTT residues [L][n]. */
void oracle_encrypt(const i64 *m, const i64 *s, const u64 *a, const i64 *e,
                    u64 *ct /*[2][L][n]*/, const u64 *mods, int L, int n)
{
    ptab *tabs = ptabs_make(mods, L, n);
    u64 *s_ntt = (u64 *)malloc(sizeof(u64) * (size_t)L * n);
    u64 *m_ntt = (u64 *)malloc(sizeof(u64) * (size_t)L * n);
    u64 *e_ntt = (u64 *)malloc(sizeof(u64) * (size_t)L * n);
    small_to_ntt(s, s_ntt, mods, tabs, L, n);
    small_to_ntt(m, m_ntt, mods, tabs, L, n);
    small_to_ntt(e, e_ntt, mods, tabs, L, n);
    for (size_t at = 0; at < (size_t)L * n; ++at) {
        u64 q = mods[at / n];
        u64 v = submod(e_ntt[at], mulmod(a[at], s_ntt[at], q), q);
        ct[at] = addmod(v, m_ntt[at], q);
        ct[(size_t)L * n + at] = a[at];
    }
    free(s_ntt); free(m_ntt); free(e_ntt);
    ptabs_free(tabs, L);
}

/* Decryption to coefficient residues: INTT(c0 + c1 s), [L][n]. */
void oracle_decrypt(const u64 *ct, const i64 *s, u64 *out, const u64 *mods,
                    int L, int n)
{
    ptab *tabs = ptabs_make(mods, L, n);
    u64 *s_ntt = (u64 *)malloc(sizeof(u64) * (size_t)L * n);
    small_to_ntt(s, s_ntt, mods, tabs, L, n);
    for (size_t at = 0; at < (size_t)L * n; ++at) {
        u64 q = mods[at / n];
        out[at] = addmod(ct[at], mulmod(ct[(size_t)L * n + at], s_ntt[at], q), q);
    }
    #pragma omp parallel for schedule(static)
    for (int l = 0; l < L; ++l) ntt_inv_one(out + (size_t)l * n, &tabs[l], n);
    free(s_ntt);
    ptabs_free(tabs, L);
}

/* Negacyclic schoolbook product mod X^n + 1 (one limb), O(n^2). */
void oracle_negacyclic_mul(const u64 *a, const u64 *b, u64 *out, u64 q, int n)
{
    for (int k = 0; k < n; ++k) out[k] = 0;
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < n; ++j) {
            u64 p = mulmod(a[i], b[j], q);
            int k = i + j;
            if (k < n) out[k] = addmod(out[k], p, q);
            else out[k - n] = submod(out[k - n], p, q);
        }
}

/* Threads an OpenMP parallel-for of this library uses (1 without OpenMP). */
/* Thread count for the parallel loops that follow (t >= 1); for timing only. */
void oracle_set_num_threads(int t)
{
#ifdef _OPENMP
    if (t >= 1) omp_set_num_threads(t);
#else
    (void)t;
#endif
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
