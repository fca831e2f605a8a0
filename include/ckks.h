/*
 * ckks.h -- C ABI of the B200 RNS-CKKS hot-path library (libckks_b200.so).
 *
 * What the library computes.  The pages describe a CPU RNS-CKKS engine with
 * ring degree n = 2048, 1024 slots, scale 2^60 and chains of 112 (layer) and
 * 2100 (bootstrapping) 60-bit primes (Kestrel FHE relay README, section 1;
 * Kestrel engine write-up, section 4.1).  Its cost sits in NTT/INTT, RNS basis
 * conversion, Galois rotation and the baby-step giant-step matmul (Kestrel
 * engine write-up, section 3 table and the boot profile in section 2 "wall 3",
 * where coeff_to_slot + slot_to_coeff take 79.1 %); a rotation is a transform
 * plus a key switch and relinearisation consumes an evaluation key
 * (EncryptedLLM GPU article, section 2.5).  This header exposes exactly those
 * operations, each as a hand-written sm_100a CUDA kernel sequence.
 *
 * Conventions (apply to every call below):
 *  - Residues are uint64 in [0, q) for the limb's prime q.  Inputs outside
 *    that range give unspecified (but memory-safe) results.
 *  - Tensors are limb-major and contiguous: [batch][component][limb][n],
 *    n = 2048 coefficients of 8 bytes (16 KiB per limb).
 *  - Primes: the context holds L ciphertext primes q_0..q_{L-1} followed by K
 *    special primes p_0..p_{K-1}; "prime index" t < L means q_t, t >= L means
 *    p_{t-L}.  Digit j of the hybrid key switch is the contiguous block
 *    q_{j alpha} .. q_{min((j+1) alpha, L) - 1}; dnum = ceil(L / alpha).
 *  - NTT domain: slot k holds a(psi^(2 brv(k) + 1)), brv = 11-bit reversal,
 *    psi = the smallest primitive 2n-th root of unity mod the limb's prime.
 *  - Every tensor pointer is DEVICE memory owned by the caller, 16-byte
 *    aligned, on the context's device.  The library never frees caller memory.
 *    Key-pointer arrays (const uint64_t *const *) are HOST arrays of device
 *    pointers.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  Outputs are valid once the stream has synchronised.
 *  - Outputs may not alias inputs unless a call says so.
 *  - `ws` is a device workspace of at least ckks_workspace_bytes(...) bytes,
 *    16-byte aligned, used only for the duration of the call's stream work.
 *    Passing NULL makes the context allocate (and keep) its own workspace;
 *    that path calls cudaMalloc and synchronises the device.  All NULL-
 *    workspace calls on one context share that one buffer, so they must be
 *    serialised: issue them on one stream from one host thread at a time.
 *  - Status: CKKS_OK (0) or a negative code.  Argument checks run on the host
 *    before any launch; a failed check launches nothing.  CUDA launch errors
 *    map to CKKS_ECUDA.  ckks_last_error() returns a thread-local message.
 *  - A context may be used from several host threads concurrently as long as
 *    their calls use distinct workspaces.
 */
#ifndef CKKS_B200_H
#define CKKS_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct ckks_ctx ckks_ctx;
typedef void *ckks_stream_t; /* cudaStream_t */

enum ckks_status {
    CKKS_OK = 0,
    CKKS_EINVAL = -1,       /* bad argument (null, size, alignment, prime) */
    CKKS_EUNSUPPORTED = -2, /* valid but outside what the kernels support */
    CKKS_ECUDA = -3,        /* a CUDA runtime call or launch failed */
    CKKS_ENOMEM = -4        /* device allocation failed */
};

/* Operation codes for ckks_workspace_bytes. */
enum ckks_op {
    CKKS_OP_MODUP = 1,
    CKKS_OP_MODDOWN = 2,
    CKKS_OP_KEYSWITCH = 3,
    CKKS_OP_ROTATE = 4,
    CKKS_OP_RESCALE = 5,
    CKKS_OP_MUL_RELIN_RESCALE = 6,
    CKKS_OP_BSGS = 7,
    CKKS_OP_ROTATE_UNHOISTED = 8,
    CKKS_OP_MODRAISE = 9,       /* aux: l, the input's prime count */
    CKKS_OP_CONJ_EXTRACT = 10,
    CKKS_OP_ROTATE_STREAMED = 11  /* aux: number of keys */
};

/* Pointwise operation codes for ckks_pointwise. */
enum ckks_pointwise_op { CKKS_PW_MUL = 0, CKKS_PW_ADD = 1, CKKS_PW_SUB = 2 };

/* ---------------------------------------------------------------- set-up */

/* Host-only.  Writes the first `count` primes q = 1 (mod 2n), 2^59 < q < 2^60,
 * scanning downward from 2^60 (largest first).  The pages ask for 60-bit
 * NTT-friendly primes (Kestrel engine write-up, section 2 "wall 2", a chain of
 * 112 of them); the scan order is this library's reading.
 * Returns CKKS_EINVAL if out is NULL, n is not a power of two in [2, 2^16]
 * or count < 0, CKKS_EUNSUPPORTED if the interval runs out of primes. */
int ckks_primes(int n, int count, uint64_t *out);

/* Creates a context on CUDA device `device`: validates the primes (each
 * prime, distinct, q = 1 mod 2n, q < 2^60), uploads NTT twiddles with Shoup
 * constants, basis-conversion matrices for ModUp/ModDown and the rescale
 * constants of the top level.  q: L host values, p: K host values.
 * Supported: n = 2048, 1 <= L <= 4096, 1 <= K <= 64, 1 <= alpha <= 64,
 * alpha <= L.  Returns CKKS_EINVAL / CKKS_EUNSUPPORTED / CKKS_ECUDA /
 * CKKS_ENOMEM with *out untouched on failure. */
int ckks_ctx_create(const uint64_t *q, int L, const uint64_t *p, int K, int alpha,
                    int n, int device, ckks_ctx **out);

/* Frees the context's device tables and its own workspace (if any).  Waits
 * for the device.  NULL is a no-op. */
void ckks_ctx_destroy(ckks_ctx *ctx);

/* Message for the last non-OK status returned on this host thread. */
const char *ckks_last_error(void);

/* Waits for the context's device and reports whether any kernel of this
 * context gave up a bounded wait since the last call: CKKS_ECUDA with a
 * message if so (the flag is then cleared), else CKKS_OK.  Only the int8
 * tensor-core basis conversion (see ckks_ctx_set_conversion) and the
 * tensor-pipe microbenchmark wait on the device; they bound every wait, and
 * if one expires the kernel stops issuing work, frees its tensor memory and
 * raises the flag, so the affected outputs must be discarded.  Also returns
 * CKKS_ECUDA for an asynchronous CUDA error on the device. */
int ckks_device_status(const ckks_ctx *ctx);

/* Failure-path self-test of the bounded device waits (no page counterpart):
 * launches, on the context's device and default stream, one kernel that waits
 * with the library's bound on a barrier nothing completes, so the wait expires
 * and the context's device flag is raised.  The next ckks_device_status then
 * returns CKKS_ECUDA and clears the flag; the context stays usable.  Takes up
 * to about a second of device time.  CKKS_EINVAL for a null context. */
int ckks_selftest_wait_expiry(const ckks_ctx *ctx);

/* Where the basis conversions of ModUp and ModDown run.  The conversion is
 * the exact product out_t = sum_s y_s [Q_j/q_s]_t (mod t), the step named
 * "RNS basis conversion" in the Kestrel engine write-up, section 3 table.
 *  CKKS_CONV_AUTO     the folded int8 tensor-core form (below) when the
 *                     conversion has 8 or more source primes (ModUp: alpha;
 *                     ModDown: K), the integer pipes otherwise (the default);
 *  CKKS_CONV_INTEGER  always the integer pipes (64x64->128-bit multiply-adds);
 *  CKKS_CONV_TENSOR   always the int8 tensor cores (byte-plane products of
 *                     both operands, 15 accumulators per output);
 *  CKKS_CONV_FOLDED   always the int8 tensor cores in the folded form: the
 *                     data's byte weights folded into the matrix modulo each
 *                     target (8 accumulators per output, the data words in
 *                     tensor memory).  Its tables (8 x 512 bytes per target
 *                     and digit) are built on the first call that uses it,
 *                     which is then synchronous; make that call before any
 *                     stream capture.
 * Every engine computes the same exact sum before the one final reduction, so
 * results are bit-identical; this is a performance switch only.  The pages
 * have no counterpart (their engine runs on CPU threads).  Takes effect for
 * calls issued after it returns; do not change it while another host thread
 * issues calls on the same context.  CKKS_EINVAL for a null context or an
 * unknown engine. */
enum { CKKS_CONV_AUTO = 0, CKKS_CONV_INTEGER = 1, CKKS_CONV_TENSOR = 2, CKKS_CONV_FOLDED = 3 };
int ckks_ctx_set_conversion(ckks_ctx *ctx, int engine);

/* Declares that the switching keys passed to this context's calls were made
 * for a chain of key_L >= L ciphertext primes q_0..q_{key_L-1} (and the same
 * special primes): layout [dnum_key][2][key_L + K][n] with dnum_key at least
 * ceil(L / alpha).  The calls then read ciphertext prime t < L at key row
 * t, special prime k at row key_L + k, and only the first ceil(L / alpha)
 * digits, which must cover the same primes as this context's digits (a
 * context below alpha primes has one digit, the start of the key's first).  A key reduced modulo a divisor of its modulus is a key for that
 * divisor, so one key set made at the top of a chain serves the context of
 * every level below it; the digits must be the same contiguous blocks of
 * alpha primes.  The default is key_L = L.  Takes effect for calls issued
 * after it returns; do not change it while another host thread issues calls
 * on the same context.  CKKS_EINVAL for a null context or key_L outside
 * [L, 4096]. */
int ckks_ctx_set_key_chain(ckks_ctx *ctx, int key_L);

/* Context parameters: writes L, K, alpha, dnum, n (any pointer may be NULL). */
int ckks_ctx_params(const ckks_ctx *ctx, int *L, int *K, int *alpha, int *dnum, int *n);

/* Bytes of workspace that `op` needs for `batch` inputs.  aux: number of keys
 * for CKKS_OP_ROTATE and CKKS_OP_ROTATE_STREAMED, input limb count (level + 1) for CKKS_OP_RESCALE,
 * bb * 1000 + gg for CKKS_OP_BSGS, ignored otherwise.  Returns 0 for an
 * unknown op or a null context. */
size_t ckks_workspace_bytes(const ckks_ctx *ctx, int op, int batch, int aux);

/* ---------------------------------------------------------------- a1/a2: NTT */

/* Forward negacyclic NTT, in place, over x[batch][limbs][n]; local limb l
 * uses prime index limb_begin + l (0 <= limb_begin, limb_begin + limbs <= L+K).
 * Natural coefficient order in, bit-reversed evaluation order out.
 * (Kestrel engine write-up, section 3 table: NTT/INTT turn the O(n^2)
 * polynomial product into O(n log n).)  batch = 0 or limbs = 0 is a no-op. */
int ckks_ntt_fwd(const ckks_ctx *ctx, uint64_t *x, int batch, int limb_begin,
                 int limbs, ckks_stream_t stream);

/* Exact inverse of ckks_ntt_fwd (includes the factor n^-1), in place. */
int ckks_ntt_inv(const ckks_ctx *ctx, uint64_t *x, int batch, int limb_begin,
                 int limbs, ckks_stream_t stream);

/* The same transforms on several tensors in one launch (a batch of
 * polynomials at several levels, such as the NTT sweep of 16 polynomials at
 * 3, 112, 512 and 2100 limbs): for g < groups, x[g] (a host array of device
 * pointers) is [batch[g]][limbs[g]][n] and its local limb l uses prime index
 * limb_begin[g] + l.  Each tensor gets exactly ckks_ntt_fwd's (or
 * ckks_ntt_inv's) result; the small tensors no longer need launches of their
 * own that leave most of the GPU idle.  Tensors must not overlap.
 * 0 <= groups <= 8; empty groups are skipped.  CKKS_EINVAL for bad ranges,
 * null or misaligned pointers; CKKS_EUNSUPPORTED past 2^30 limbs in all. */
int ckks_ntt_fwd_group(const ckks_ctx *ctx, uint64_t *const *x, const int *batch,
                       const int *limb_begin, const int *limbs, int groups,
                       ckks_stream_t stream);
int ckks_ntt_inv_group(const ckks_ctx *ctx, uint64_t *const *x, const int *batch,
                       const int *limb_begin, const int *limbs, int groups,
                       ckks_stream_t stream);

/* ---------------------------------------------------------------- a3: pointwise */

/* out = a (op) b mod q per limb, NTT domain, arrays [batch][limbs][n]
 * (limb l uses prime index limb_begin + l).  op: CKKS_PW_MUL/ADD/SUB.
 * out may alias a or b.  (ct x pt products of the diagonal method and the
 * ct x ct tensor product, EncryptedLLM GPU article, section 2.1.) */
int ckks_pointwise(const ckks_ctx *ctx, int op, const uint64_t *a, const uint64_t *b,
                   uint64_t *out, int batch, int limb_begin, int limbs,
                   ckks_stream_t stream);

/* ---------------------------------------------------------------- a4: automorphism */

/* Galois automorphism a(X) -> a(X^g) in the NTT domain, a pure index
 * permutation identical for every limb: out[.][l][k] = in[.][l][k'] with
 * 2 brv(k') + 1 = g (2 brv(k) + 1) mod 2n.  arrays [rows][n], rows = batch *
 * limbs.  galois must be odd.  out must not alias in.  (Galois rotation /
 * conjugation as slot permutation, Kestrel engine write-up, section 3.) */
int ckks_automorph(const ckks_ctx *ctx, const uint64_t *in, uint64_t *out, int batch,
                   int limbs, uint32_t galois, ckks_stream_t stream);

/* ---------------------------------------------------------------- a5-a7: key switching */

/* ModUp (hybrid key switching, approximate fast basis conversion):
 * c_ntt[batch][L][n] (NTT over q) -> digits[batch][dnum][L+K][n] (NTT over
 * q and p).  Digit j's own limbs are copies of the input; every other limb t
 * holds NTT_t( sum_{i in D_j} [c_i (Q_j/q_i)^-1]_{q_i} [Q_j/q_i]_t ).
 * (RNS basis conversion as the core of bootstrapping, Kestrel engine
 * write-up, section 3 table; basis conversion kernel, EncryptedLLM GPU
 * article, section 3.4.)  ws: CKKS_OP_MODUP bytes. */
int ckks_modup(const ckks_ctx *ctx, const uint64_t *c_ntt, uint64_t *digits, int batch,
               void *ws, ckks_stream_t stream);

/* ModUp that allocates nothing.  The paper has no counterpart: this entry point
 * exists for callers that cannot call cudaMalloc.  Examples are a host
 * framework whose caching allocator already owns the device memory under a
 * fixed budget, and a latency-critical loop that cannot absorb the device-wide
 * synchronisation that cudaMalloc/cudaFree can imply.
 * Same arguments, layouts and result as ckks_modup, without a workspace
 * argument.  Its scratch is a 32 MiB static device array inside the library,
 * which every GPU that loads the library holds until the process exits.
 * Limit: batch * L <= 2048.  Larger requests return CKKS_EUNSUPPORTED and
 * launch nothing.
 * When the context converts on the folded tensor-core engine (the automatic
 * choice from 8 primes per digit, or CKKS_CONV_FOLDED), that engine's tables
 * are built, with cudaMalloc, by the first call that converts (ckks_modup,
 * ckks_keyswitch, ckks_rotate and the other key-switching calls).  Until one
 * of them has run on the context, this entry point returns CKKS_EUNSUPPORTED
 * and launches nothing.
 * The first call on a device resolves the array's device address
 * (cudaGetSymbolAddress, once per device); make that first call before any
 * stream capture.  The address is cached for the life of the process and
 * belongs to the device's primary context as it was then: after
 * cudaDeviceReset, or anything else that tears that context down, do not
 * call this entry point again in the same process.
 * Every call shares the one array, so calls that overlap on the GPU (other
 * streams, other host threads, the same device) race: serialise them.  No
 * part of the array needs clearing between calls, because every word a call
 * reads was written earlier in the same call.  Calls no cudaMalloc, cudaFree
 * or allocating library routine. */
int ckks_modup_noalloc(const ckks_ctx *ctx, const uint64_t *c_ntt, uint64_t *digits, int batch,
                       ckks_stream_t stream);

/* Key inner product with the automorphism fused into the digit load:
 * acc[batch][2][L+K][n] with acc[b][c][t][k] = sum_j phi_g(D_j)[t][k] *
 * key[j][c][t][k] mod t.  digits [batch][dnum][L+K][n], key
 * [dnum][2][L+K][n] (component 0 = b, 1 = a).  galois = 1 means no
 * automorphism.  This is the step of a key switch that consumes the
 * evaluation key, which the EncryptedLLM GPU article (section 2.5) sizes at
 * hundreds of MB to several GB and names, with the rotation it serves, as
 * the under-rated cost of encrypted inference.  Sums over any number of
 * digits are exact (reduced once per 256 digits, or folded once per 8 when
 * every prime is 2^60 - delta with delta < 2^32).  Digit and key words must
 * be residues, below their prime.  CKKS_EINVAL for a null pointer, a pointer
 * that is not 16-byte aligned or an even galois. */
int ckks_key_inner(const ckks_ctx *ctx, const uint64_t *digits, const uint64_t *key,
                   uint32_t galois, uint64_t *acc, int batch, ckks_stream_t stream);

/* ModDown: acc[batch][2][L+K][n] -> out[batch][2][L][n],
 * out_i = (acc_i - NTT_i(sum_k [INTT(acc_{p_k}) (P/p_k)^-1]_{p_k} [P/p_k]_{q_i}))
 *         * P^-1 mod q_i.
 * The conversion from the special primes back to the q_i is the same "RNS
 * basis conversion" step that the Kestrel engine write-up (section 3
 * table) names as the core of bootstrapping, run in the other direction;
 * dividing by P ends the key switch of the EncryptedLLM GPU article
 * (section 2.5).  ws: CKKS_OP_MODDOWN bytes. */
int ckks_moddown(const ckks_ctx *ctx, const uint64_t *acc, uint64_t *out, int batch,
                 void *ws, ckks_stream_t stream);

/* KeySwitch(d) = ModDown(<ModUp(d), key>): d[batch][L][n] (NTT),
 * key[dnum][2][L+K][n], out[batch][2][L][n].  This is the key switch that
 * every rotation and every relinearisation runs (EncryptedLLM GPU article,
 * section 2.5: a rotation is a transform plus a key switch, and
 * relinearisation after a ct x ct product consumes an evaluation key); its
 * two basis conversions are the "RNS basis conversion" of the Kestrel engine
 * write-up, section 3 table.  ws: CKKS_OP_KEYSWITCH bytes. */
int ckks_keyswitch(const ckks_ctx *ctx, const uint64_t *d, const uint64_t *key,
                   uint64_t *out, int batch, void *ws, ckks_stream_t stream);

/* ---------------------------------------------------------------- a8: rotation */

/* Hoisted rotations: for every key r, out[r][b] = (phi_g(c0) + KS0, KS1)
 * with KS = ModDown(<phi_g(ModUp(c1)), keys[r]>) and g = galois[r].  ModUp
 * runs once per ciphertext and is shared by all keys.  ct[batch][2][L][n],
 * keys: host array of nkeys device pointers to [dnum][2][L+K][n], galois:
 * host array of nkeys odd elements, out[nkeys][batch][2][L][n].  (Rotation =
 * transform + key switch, EncryptedLLM GPU article, section 2.5.)
 * ws: ckks_workspace_bytes(CKKS_OP_ROTATE, batch, nkeys). */
int ckks_rotate(const ckks_ctx *ctx, const uint64_t *ct, const uint64_t *const *keys,
                const uint32_t *galois, int nkeys, uint64_t *out, int batch, void *ws,
                ckks_stream_t stream);

/* a8, the other order: Rot_g(c) = (phi_g(c0) + KS_0, KS_1) with KS the key
 * switch of phi_g(c1) -- the automorphism applied before ModUp, one ModUp per
 * key (no hoisting) -- using the same Galois keys as ckks_rotate.  This is the
 * textbook order without hoisting; the pages fix neither order (Galois
 * rotation: Kestrel engine write-up, section 3 table; rotation = transform +
 * key switch: EncryptedLLM GPU article, section 2.5).  Its low bits differ
 * from ckks_rotate's (the approximate ModUp does not commute with phi_g);
 * both decrypt to the rotated slots.
 * Arguments, layouts and errors as ckks_rotate; ws:
 * ckks_workspace_bytes(CKKS_OP_ROTATE_UNHOISTED, batch, 0). */
int ckks_rotate_unhoisted(const ckks_ctx *ctx, const uint64_t *ct, const uint64_t *const *keys,
                          const uint32_t *galois, int nkeys, uint64_t *out, int batch, void *ws,
                          ckks_stream_t stream);

/* a8 with ModUp, NTT and the key inner product fused by streaming: the same
 * hoisted rotations as ckks_rotate, word for word, without the extended
 * digits [batch][dnum][L+K][n] ever existing as a whole (1.24 GB per
 * ciphertext at 2100 + 60 primes, alpha = 60; the boot-level rotation
 * dominates the boot: Kestrel engine write-up, section 5.3 profile).  The
 * primes are cut into windows of at most 60, each inside one digit's range
 * or inside the special primes; per window the int8 tensor-core conversion
 * (folded form) writes every digit's limbs at the window's primes into one
 * buffer of batch * dnum * 60 limbs (the window's own digit gets the input's
 * limbs), the forward NTT runs over it and the key inner product consumes
 * it; consecutive windows alternate between the caller's stream and a second
 * stream (one stream while the caller's is being captured into a graph).
 * ModDown then runs as in ckks_rotate.  The first call builds the windows'
 * conversion tables (two 128 KiB blocks of 32 targets per window and digit).
 * Arguments, layouts and errors as ckks_rotate.  Each chunk of 64 keys
 * repeats the windows' work.
 * ws: ckks_workspace_bytes(CKKS_OP_ROTATE_STREAMED, batch, nkeys). */
int ckks_rotate_streamed(const ckks_ctx *ctx, const uint64_t *ct, const uint64_t *const *keys,
                         const uint32_t *galois, int nkeys, uint64_t *out, int batch, void *ws,
                         ckks_stream_t stream);

/* ---------------------------------------------------------------- a10: rescale */

/* Rescale by the last prime of the input level: ct[batch][2][lp1][n] ->
 * out[batch][2][lp1-1][n], c'_i = (c_i - NTT_i([c]_{q_l})) q_l^-1 mod q_i with
 * l = lp1 - 1 (floor form).  2 <= lp1 <= L.  (One prime dropped per
 * multiplication, Kestrel engine write-up, section 2 "wall 2".)
 * ws: ckks_workspace_bytes(CKKS_OP_RESCALE, batch, lp1). */
int ckks_rescale(const ckks_ctx *ctx, const uint64_t *ct, uint64_t *out, int lp1,
                 int batch, void *ws, ckks_stream_t stream);

/* ---------------------------------------------------------------- a9: ct x ct */

/* Tensor product, relinearisation and rescale at the top level:
 * d0 = a0 b0, d1 = a0 b1 + a1 b0, d2 = a1 b1; (d0, d1) + KeySwitch(d2, rlk);
 * then rescale by q_{L-1}.  a, b [batch][2][L][n], rlk [dnum][2][L+K][n],
 * out [batch][2][L-1][n].  (Relinearisation after ct x ct multiply,
 * EncryptedLLM GPU article, section 2.5.)  Requires L >= 2.
 * ws: CKKS_OP_MUL_RELIN_RESCALE bytes. */
int ckks_mul_relin_rescale(const ckks_ctx *ctx, const uint64_t *a, const uint64_t *b,
                           const uint64_t *rlk, uint64_t *out, int batch, void *ws,
                           ckks_stream_t stream);

/* ---------------------------------------------------------------- a11: BSGS */

/* Baby-step giant-step diagonal matrix-vector product (the engine's matmul2
 * with BB = GG = 32, Kestrel engine write-up, sections 3 and 4.4):
 * y = Rescale( sum_{g<gg} Rot_{bb g}( sum_{b<bb} diags[g][b] * Rot_b(x) ) ),
 * Rot_r with Galois element 5^r mod 2n, baby rotations sharing one ModUp.
 * x [batch][2][L][n], diags [gg][bb][L][n] (plaintexts in the NTT domain),
 * baby_keys: bb-1 host pointers (rotation b = 1..bb-1), giant_keys: gg-1
 * host pointers (rotation bb g, g = 1..gg-1), y [batch][2][L-1][n].
 * Requires L >= 2, bb >= 1, gg >= 1.  Ciphertext, diagonal and key words must be
 * residues, below their prime (the inner sums of up to 64 products below 2^120
 * are then exact in 128 bits).
 * ws: ckks_workspace_bytes(CKKS_OP_BSGS, batch, bb * 1000 + gg). */
int ckks_bsgs_lintrans(const ckks_ctx *ctx, const uint64_t *x, const uint64_t *diags,
                       const uint64_t *const *baby_keys, const uint64_t *const *giant_keys,
                       int bb, int gg, uint64_t *y, int batch, void *ws,
                       ckks_stream_t stream);

/* The same transform for a matrix whose nonzero diagonals sit at the offsets
 * stride (t0 + bb g + b), g < gg, b < bb (a group of butterfly stages of a
 * factored coeff_to_slot / slot_to_coeff):
 *   y = Rescale( sum_g Rot_{G_g}( sum_b diags[g][b] * Rot_{stride b}(x) ) ),
 *   G_g = stride (t0 + bb g) mod n/2,
 * with diags[g][b] = Encode(rot_{-G_g}(diag_{G_g + stride b})) (zeros where
 * the diagonal is absent).  baby_keys[b-1] rotates by stride b (Galois
 * 5^{stride b}); giant_keys has gg entries, giant_keys[g] rotating by G_g
 * (it may be NULL where G_g = 0, which is not rotated).  stride = 1, t0 = 0
 * is ckks_bsgs_lintrans.  Limits as ckks_bsgs_lintrans, plus stride >= 1,
 * stride (bb - 1) < n/2, |t0| <= n/2.
 * ws: ckks_workspace_bytes(CKKS_OP_BSGS, batch, bb * 1000 + gg). */
int ckks_bsgs_lintrans_plan(const ckks_ctx *ctx, const uint64_t *x, const uint64_t *diags,
                            const uint64_t *const *baby_keys, const uint64_t *const *giant_keys,
                            int stride, int t0, int bb, int gg, uint64_t *y, int batch, void *ws,
                            ckks_stream_t stream);

/* ---- building blocks of the bootstrapping refresh (Kestrel engine write-up,
 * the boot profile in section 5.3; the forms are the textbook ones, as the
 * oracle reads them). */

/* out[p][l][k] = a[p][l][k] op k[l] over [batch][limbs][n]; k is a DEVICE
 * array of `limbs` residues, k[l] in [0, q) of prime limb_begin + l (a
 * constant polynomial's NTT is the constant).  op: CKKS_PW_MUL/ADD/SUB.
 * out may alias a.  Limit: batch <= 65535. */
int ckks_pointwise_scalar(const ckks_ctx *ctx, int op, const uint64_t *a, const uint64_t *k,
                          uint64_t *out, int batch, int limb_begin, int limbs,
                          ckks_stream_t stream);

/* In place on ct[batch][2][L][n]: component 0 of every ciphertext gets k[l]
 * added at limb l (k: DEVICE array of L residues), i.e. every slot gets the
 * constant whose scaled value k encodes. */
int ckks_add_const_c0(const ckks_ctx *ctx, uint64_t *ct, const uint64_t *k, int batch,
                      ckks_stream_t stream);

/* out = X^{n/2} in over [batch][limbs][n] (NTT domain, limb l with prime
 * limb_begin + l): every slot times i.  In the NTT domain this is the
 * pointwise product by psi^{n/2} on the first n/2 evaluation slots and by
 * -psi^{n/2} on the others.  out may alias in. */
int ckks_mul_i(const ckks_ctx *ctx, const uint64_t *in, uint64_t *out, int batch, int limb_begin,
               int limbs, ckks_stream_t stream);

/* conj_extract: ct[batch][2][L][n] with slots w -> re, im [batch][2][L][n]
 * with slots 2 Re w and 2 Im w (same scale): re = ct + conj(ct),
 * im = X^{n/2} (conj(ct) - ct), conj being the hoisted rotation by the
 * Galois element 2n - 1 with conj_key ([dnum][2][L+K][n], or the layout
 * ckks_ctx_set_key_chain declares).  Limit: batch <= 32767.
 * ws: ckks_workspace_bytes(CKKS_OP_CONJ_EXTRACT, batch, 0). */
int ckks_conj_extract(const ckks_ctx *ctx, const uint64_t *ct, const uint64_t *conj_key, uint64_t *re,
                      uint64_t *im, int batch, void *ws, ckks_stream_t stream);

/* restore_merge: re, im [batch][2][L][n] with slots a, b -> out = re +
 * X^{n/2} im, slots a + i b. */
int ckks_restore_merge(const ckks_ctx *ctx, const uint64_t *re, const uint64_t *im, uint64_t *out,
                       int batch, ckks_stream_t stream);

/* modraise: in[batch][2][l][n] over q_0..q_{l-1} (NTT domain) ->
 * out[batch][2][L][n] over the context's L primes.  Each coefficient is read
 * as its centred integer X in (-Q/2, Q/2], Q = q_0 ... q_{l-1}, and reduced
 * modulo every q_t (exact: Garner's mixed-radix digits, then a conversion
 * whose sign row subtracts Q where X > (Q-1)/2).  Limbs below l are copied.
 * Limits: 1 <= l <= min(L, 63), batch <= 32767.  Tables for each l are built
 * on first use and kept by the context.
 * ws: ckks_workspace_bytes(CKKS_OP_MODRAISE, batch, l). */
int ckks_modraise(const ckks_ctx *ctx, const uint64_t *in, int l, uint64_t *out, int batch, void *ws,
                  ckks_stream_t stream);

/* ---------------------------------------------------------------- measurement */

/* Integer-pipe microbenchmarks on the context's device (no page counterpart:
 * they give the roofline denominators).  Each runs `iters` dependency-free
 * iterations in every thread of a grid of `blocks` x 256 threads and writes
 * the elapsed milliseconds (CUDA events) to *ms and the operation count to
 * *ops.  kind 0: 64-bit Shoup modular multiply; kind 1: 64x64->128
 * multiply-accumulate; kind 2: 64x64 high-half multiply; kind 5: the
 * forward NTT's own butterfly (Shoup product with the three-partial-product
 * quotient, the cheap quotient-times-q for 2^60 - delta primes when every
 * prime of the context has that form, and the lazy add/sub; *ops counts
 * butterflies, one modular product each); kind 6: the key inner product's
 * split form without its loads (each iteration runs 8 words per chain, 8
 * chains: a word split into 30-bit halves once and multiplied into the
 * three-sum accumulators of two key words with the Karatsuba middle product,
 * the sums folded every 8 words; *ops counts 60 x 60-bit products; only for
 * contexts whose primes are all 2^60 - delta, else CKKS_EUNSUPPORTED;
 * iters <= 2^26).
 * Tensor-pipe kinds (one issuing thread per CTA of 128 threads, `iters`
 * back-to-back int8 tcgen05.mma of M = 128, K = 32; *ops counts 2 M N K per
 * MMA): kind 3: N = 256 (the dense int8 rate); kind 4: N = 32 (the basis
 * conversion's tile).  blocks <= 148 * 64.  Synchronous. */
int ckks_bench_intpipe(const ckks_ctx *ctx, int kind, int blocks, int iters, double *ms,
                       double *ops);

#ifdef __cplusplus
}
#endif

#endif /* CKKS_B200_H */
