// Internal declarations of libckks_b200: context layout, device modular
// arithmetic, error plumbing.  Not part of the public ABI (see include/ckks.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/ckks.h"

typedef uint64_t u64;
typedef uint32_t u32;

namespace ckks {

constexpr int kN = 2048;       // ring degree (the only one the kernels support)
constexpr int kLogN = 11;
constexpr int kMaxDigit = 64;  // alpha and K bound: sources of one basis conversion

// ---------------------------------------------------------------- per-prime constants
// 64 bytes per prime, read once per thread per job.
struct __align__(16) PrimeConst {
    u64 q;
    u64 r64, r64p;    // 2^64 mod q and its Shoup constant floor(r64 2^64 / q)
    u64 mu64;         // floor(2^64 / q)
    u64 ninv, ninvp;  // n^-1 mod q and its Shoup constant
    u64 two_q;
    u64 delta;        // 2^60 - q when that is below 2^32 (every prime of the pages' chain), else 0
};

// Device tables owned by a context (struct of device pointers, passed by value).
struct Tables {
    int L, K, alpha, dnum, LK;
    // Switching keys may be made for a longer chain of key_L >= L ciphertext
    // primes (one key set serving the contexts of every lower level): ciphertext
    // prime t sits at key row t, special prime k at key row key_L + k, and
    // each (digit, component) block holds key_LK = key_L + K rows.
    int key_L, key_LK;
    const ulonglong2 *mul_i;      // [L+K][2]: {psi^{n/2}, Shoup}, {-psi^{n/2}, Shoup} (X^{n/2} in NTT form)
    bool special;               // every prime is 2^60 - delta with delta < 2^32
    const PrimeConst *pc;       // [L+K]
    const ulonglong2 *tw_fwd;   // [L+K][n]: {psi^brv(k), Shoup}; k = 0 unused
    const ulonglong2 *tw_inv;   // [L+K][n]: {psi^-brv(k), Shoup}; k = 0 holds psi^-brv(1) n^-1
    // ModUp: source i (global ciphertext prime index) of its digit
    const ulonglong2 *up_hatinv;  // [L]: {[(Q_j/q_i)^-1]_{q_i}, Shoup}
    const u64 *up_mat;            // [dnum][alpha][L+K]: [Q_j/q_i]_t
    // ModDown
    const ulonglong2 *dn_hatinv;  // [K]: {[(P/p_k)^-1]_{p_k}, Shoup}
    const u64 *dn_mat;            // [K][L]: [P/p_k]_{q_i}
    const ulonglong2 *dn_pinv;    // [L]: {[P^-1]_{q_i}, Shoup}
    // Byte planes of the conversion matrices for the int8 tensor-core path: per target row its
    // 8 planes of 64 source bytes, targets in blocks of 128
    const uint8_t *tc_up;         // [dnum][tb_per_digit][128][8][64]
    const uint8_t *tc_dn;         // [ceil(L/128)][128][8][64]
    int tc_tb_per_digit;
    bool tc_special;              // every prime is 2^60 - delta with delta < 2^28
    // Folded byte planes for the int8 tensor-core path with the data in tensor memory
    // (conv_fold.cu), targets in blocks of 32, built on first use
    const uint8_t *fold_up;       // [dnum][fold_tb_per_digit][8][32][512]
    const uint8_t *fold_dn;       // [ceil(L/32)][8][32][512]
    int fold_tb_per_digit;
};

}  // namespace ckks

struct ckks_ctx {
    int device = 0;
    int n = ckks::kN, L = 0, K = 0, alpha = 0, dnum = 0;
    std::vector<u64> mods;  // L+K host copy
    ckks::Tables t{};
    std::vector<void *> allocations;
    // rescale constants per input level lp1: device [lp1-1] of {q_l^-1 mod q_i, Shoup}
    std::map<int, ulonglong2 *> rescale_tab;
    // modraise tables per input level l (boot.cu)
    std::map<int, void *> raise_tab;
    std::mutex mu;
    void *own_ws = nullptr;
    size_t own_ws_bytes = 0;
    int *tc_err = nullptr;  // device flag: a bounded wait of the tensor-core kernel expired
    std::atomic<int> conv_engine{CKKS_CONV_AUTO};
    // host copies of the conversion matrices, for the folded tables built on first use
    std::vector<u64> up_mat_host, dn_mat_host;
    bool fold_built = false;
    // Prime windows of the streamed rotation (built on first use, conv_fold.cu): window w covers
    // primes t0 .. t0 + n - 1, all inside digit `own`'s range, or all special primes (own = -1);
    // fold_win holds one folded block per (window, digit) for the digits that convert into it.
    struct Window {
        int t0, n, own;
    };
    std::vector<Window> windows;
    const uint8_t *fold_win = nullptr;  // [windows][dnum][blocks of 32 targets][8][32][512]
    bool win_built = false;
};

namespace ckks {

// ---------------------------------------------------------------- errors
int set_error(int code, const std::string &msg);
int cuda_status(cudaError_t e, const char *what);
#define CKKS_CHECK_LAUNCH(what)                                        \
    do {                                                               \
        cudaError_t _e = cudaGetLastError();                           \
        if (_e != cudaSuccess) return ::ckks::cuda_status(_e, what);   \
    } while (0)
#define CKKS_TRY(expr)              \
    do {                            \
        int _rc = (expr);           \
        if (_rc != CKKS_OK) return _rc; \
    } while (0)

int check_ctx(const ckks_ctx *ctx);
int check_ptr(const void *p, const char *name);
int set_device(const ckks_ctx *ctx);
// Resolves a workspace: the caller's, or the context's own grown to `bytes`.
int resolve_ws(ckks_ctx *ctx, void *ws, size_t bytes, void **out);
const ulonglong2 *rescale_table(ckks_ctx *ctx, int lp1, int *rc);

// ---------------------------------------------------------------- device arithmetic
// All primes satisfy q < 2^60, so 4q < 2^62 and lazy values never overflow.

__device__ __forceinline__ u64 mulhi(u64 a, u64 b) { return __umul64hi(a, b); }

// a * w mod q up to one extra q: result in [0, 2q) for any 64-bit a, given
// w < q and wp = floor(w 2^64 / q) (Shoup's precomputed quotient).
__device__ __forceinline__ u64 shoup_lazy(u64 a, u64 w, u64 wp, u64 q)
{
    return a * w - mulhi(a, wp) * q;
}

__device__ __forceinline__ u64 csub(u64 a, u64 m) { return a >= m ? a - m : a; }

// High half of a 64x64-bit product, approximated from three 32x32 partial
// products: the low-by-low product and the carries out of the two cross
// products are dropped, so the result is at most 2 below floor(a b / 2^64).
__device__ __forceinline__ u64 mulhi_approx(u64 a, u64 b)
{
    const u32 a0 = (u32)a, a1 = (u32)(a >> 32), b0 = (u32)b, b1 = (u32)(b >> 32);
    return (u64)a1 * b1 + __umulhi(a0, b1) + __umulhi(a1, b0);
}

// Shoup product with the approximate quotient: a w - qh q with qh at most 3
// below floor(a w / q), so the result lies in [0, 4q) for any 64-bit a.
// kSpecial: q = 2^60 - delta with delta < 2^32, so qh q = qh 2^60 - qh delta
// costs a shift and one 64x32 product instead of a full 64x64 low product.
template <bool kSpecial>
__device__ __forceinline__ u64 shoup4(u64 a, u64 w, u64 wp, u64 q, u64 delta)
{
    const u64 qh = mulhi_approx(a, wp);
    if (kSpecial) return a * w + qh * (u32)delta - (qh << 60);
    return a * w - qh * q;
}

__device__ __forceinline__ u64 shoup(u64 a, u64 w, u64 wp, u64 q)
{
    return csub(shoup_lazy(a, w, wp, q), q);
}

// x = hi 2^64 + lo (any 128-bit value) reduced mod q into [0, q).
// hi 2^64 mod q comes from Shoup on r64 = 2^64 mod q, lo from a one-step
// Barrett with mu64 = floor(2^64 / q); each part lies in [0, 2q).
__device__ __forceinline__ u64 reduce128(u64 hi, u64 lo, const PrimeConst &c)
{
    u64 a = shoup_lazy(hi, c.r64, c.r64p, c.q);
    u64 b = lo - mulhi(lo, c.mu64) * c.q;
    u64 s = a + b;
    s = csub(s, c.two_q);
    return csub(s, c.q);
}

__device__ __forceinline__ u64 mulmod(u64 a, u64 b, const PrimeConst &c)
{
    return reduce128(mulhi(a, b), a * b, c);
}

__device__ __forceinline__ u64 addmod(u64 a, u64 b, u64 q) { return csub(a + b, q); }
__device__ __forceinline__ u64 submod(u64 a, u64 b, u64 q) { return a >= b ? a - b : a + q - b; }

// 128-bit accumulator: (hi, lo) += a * b.
__device__ __forceinline__ void mac128(u64 &hi, u64 &lo, u64 a, u64 b)
{
    asm("mad.lo.cc.u64 %0, %2, %3, %0;\n\t"
        "madc.hi.u64 %1, %2, %3, %1;"
        : "+l"(lo), "+l"(hi)
        : "l"(a), "l"(b));
}

// 11-bit reversal.
__device__ __forceinline__ u32 brv11(u32 k) { return __brev(k) >> (32 - kLogN); }

// NTT-domain Galois source index: slot k of phi_g(a) reads slot k' of a with
// 2 brv(k') + 1 = g (2 brv(k) + 1) mod 2n.
__device__ __forceinline__ u32 galois_src(u32 k, u32 g)
{
    u32 e = (g * (2u * brv11(k) + 1u)) & (2u * kN - 1u);
    return brv11((e - 1u) >> 1);
}

// ---------------------------------------------------------------- host arithmetic
u64 host_mulmod(u64 a, u64 b, u64 q);
u64 host_powmod(u64 a, u64 e, u64 q);
u64 host_invmod(u64 a, u64 q);
u64 host_shoup(u64 w, u64 q);
bool host_is_prime(u64 m);
u64 host_find_psi(u64 q, int n);

}  // namespace ckks
