// Internal building blocks shared by the entry points (not part of the ABI).
#pragma once

#include <functional>

#include "common.cuh"

namespace ckks {

constexpr int kMaxKeys = 64;  // keys per hoisted launch

// Per-job key pointers and Galois elements, passed by value to kernels.
struct KeyList {
    const u64 *key[kMaxKeys];
    u32 galois[kMaxKeys];
};

// Bump allocator over a caller workspace (256-byte aligned slices).
struct Carve {
    char *base;
    size_t off = 0;
    explicit Carve(void *p) : base(static_cast<char *>(p)) {}
    template <class T>
    T *take(size_t count)
    {
        T *p = reinterpret_cast<T *>(base ? base + off : nullptr);
        off += (count * sizeof(T) + 255) & ~(size_t)255;
        return p;
    }
};

inline size_t limbs_bytes(size_t rows) { return ((rows * kN * sizeof(u64)) + 255) & ~(size_t)255; }

void parallel_for(int count, const std::function<void(int)> &fn);

// ---- int8 tensor-core basis conversion (conv_tc.cu: byte planes; conv_fold.cu: folded)
constexpr int kTcMinSources = 7;  // CKKS_CONV_AUTO: more sources (8 or more) use the tensor cores
enum ConvKind { kConvInteger = 0, kConvTensor = 1, kConvFolded = 2 };
ConvKind conv_kind(const ckks_ctx *ctx, int sources);
int launch_conv_fold_up(ckks_ctx *ctx, const u64 *y, u64 *digits, int batch, cudaStream_t s);
// whether the folded tables exist (they are built, with cudaMalloc, by the first folded conversion)
bool fold_tables_ready(const ckks_ctx *ctx);
// streamed rotation: prime windows of at most kWinMax primes (built with their folded blocks on
// first use) and the conversion of y into window w's buffer [batch][dnum][kWinMax][n]
constexpr int kWinMax = 60;
int stream_windows(ckks_ctx *ctx, const std::vector<ckks_ctx::Window> **out);
int launch_conv_fold_window(ckks_ctx *ctx, const u64 *y, u64 *buf, int batch, int w, cudaStream_t s);
int launch_conv_fold_down(ckks_ctx *ctx, const u64 *zsrc, u64 *cv, int jobs2, cudaStream_t s);
int build_tc_tables(ckks_ctx *ctx, const std::vector<u64> &up_mat, const std::vector<u64> &dn_mat);
int launch_conv_tc_up(const ckks_ctx *ctx, const u64 *y, u64 *digits, int batch, cudaStream_t s);
int launch_conv_tc_down(const ckks_ctx *ctx, const u64 *zsrc, u64 *cv, int jobs2, cudaStream_t s);
// tcgen05 int8 MMA rate (M = 128, N = n in {32, 256}, K = 32), synchronous: elapsed ms and int8 ops
int bench_mma(const ckks_ctx *ctx, int n, int blocks, int iters, double *ms, double *ops);
// launches the bounded-wait expiry self-test (asynchronous)
int selftest_wait_expiry(const ckks_ctx *ctx);

// ---- bootstrapping building blocks (boot.cu)
// conv_kernel over the Garner digits and sign rows dg[P][l+1][n] into rows l..L-1 of out[P][L][n]
int raise_conv(const Tables &T, const u64 *dg, u64 *out, const u64 *matp, int l, int P, cudaStream_t s);
void free_raise_tables(ckks_ctx *ctx);
size_t modraise_ws_bytes(const ckks_ctx *ctx, int batch, int l);
size_t conj_extract_ws_bytes(const ckks_ctx *ctx, int batch);
size_t rotate_ws_bytes(const ckks_ctx *ctx, int batch, int nkeys);
size_t rotate_streamed_ws_bytes(const ckks_ctx *ctx, int batch, int nkeys);

// ---- sizes of internal stages (bytes)
size_t modup_ws_bytes(const ckks_ctx *ctx, int batch);
size_t moddown_ws_bytes(const ckks_ctx *ctx, int jobs);
size_t rescale_ws_bytes(int batch);

// ---- stages; all asynchronous on `s`, arguments already validated.

// ModUp of `batch` polynomials, polynomial b read at in + b * in_bstride (L
// limbs, NTT domain).  If in2 != nullptr the source is the pointwise product
// in[b] * in2[b] (same stride).  digits: [batch][dnum][L+K][n].
int modup_stage(const ckks_ctx *ctx, const u64 *in, const u64 *in2, size_t in_bstride,
                u64 *digits, int batch, void *ws, cudaStream_t s);

// acc[z][2][L+K][n] for z < jobs.  Job z uses key kl.key[z / per_key] with
// Galois element kl.galois[z / per_key]; it reads digit set z % per_key when
// hoisted (digits shared by all keys) and digit set z otherwise.
int key_inner_stage(const ckks_ctx *ctx, const u64 *digits, const KeyList &kl, int per_key,
                    bool hoisted, u64 *acc, int jobs, cudaStream_t s);
// The same over a digit view: digit j of ciphertext b at prime t is read at digits + b ct_stride
// + j j_stride + (t - t_lo) n, for the primes t_lo .. t_lo + nt - 1 only (acc rows of the other
// primes are left as they are).
struct DigitView {
    size_t ct_stride, j_stride;
    int t_lo, nt;
};
int key_inner_stage(const ckks_ctx *ctx, const u64 *digits, const KeyList &kl, int per_key,
                    bool hoisted, u64 *acc, int jobs, cudaStream_t s, const DigitView &dv);

// What ModDown adds to its output after the P^-1 scaling.
//  kind 0: nothing.
//  kind 1 (rotation): component 0 of job z gets phi_g(c0) added, with
//          c0 at ct + (ct_mod ? z % ct_mod : z) * ct_bstride and g = gal[z / per].
//  kind 2 (relinearisation): job z gets the tensor terms of a[z], b[z]
//          ([.][2][L][n]): a0 b0 on component 0, a0 b1 + a1 b0 on component 1.
struct DownExtra {
    int kind = 0;
    const u64 *ct = nullptr;
    size_t ct_bstride = 0;
    int ct_mod = 0;
    int per = 1;
    u32 gal[kMaxKeys] = {0};
    const u64 *a = nullptr, *b = nullptr;
};

// ModDown of acc[jobs][2][L+K][n] into out[jobs][2][L][n].
int moddown_stage(const ckks_ctx *ctx, const u64 *acc, u64 *out, int jobs, const DownExtra &ex,
                  void *ws, cudaStream_t s);

// Rescale ct[batch][2][lp1][n] -> out[batch][2][lp1-1][n].
int rescale_stage(ckks_ctx *ctx, const u64 *ct, u64 *out, int lp1, int batch, void *ws,
                  cudaStream_t s);

}  // namespace ckks
