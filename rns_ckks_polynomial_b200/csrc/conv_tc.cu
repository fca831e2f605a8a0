// RNS basis conversion on the int8 tensor cores (tcgen05.mma, kind::i8).
//
// The conversion out[t][c] = (sum_s M[t][s] y[s][c]) mod q_t is a dense integer contraction:
// targets x sources times sources x coefficients, with 60-bit operands.  It is computed exactly by
// splitting both operands into bytes: M = sum_u M_u 2^(8u), y = sum_v y_v 2^(8v), u, v < 8, so that
//     sum_s M y = sum_{d=0}^{14} 2^(8d) P_d,   P_d = sum_{u+v=d} sum_s M_u[t][s] y_v[s][c].
// Each P_d is an unsigned 8-bit matrix product with at most 8 * 64 * 255^2 < 2^25 per entry, so it
// fits an int32 tensor-memory accumulator.  One CTA owns 128 targets (the MMA's M); for each tile of
// 16 coefficients it stages the y bytes in shared memory, one thread issues the 64 plane pairs x 1 or
// 2 K-steps of 32 sources as tcgen05.mma into 15 accumulators (240 TMEM columns), and the four warps
// read their 32 TMEM lanes back, rebuild the exact 128-bit sum and reduce it once mod q_t.
// 256 threads: every thread stages 4 sources of one coefficient per tile, with the next tile's loads
// issued before the wait for the current tile's products; warps w and w + 4 share TMEM lane quadrant
// w and split its 16 columns in the epilogue.
//
// Operand layout in shared memory: K-major, no swizzle, 8-row x 16-byte core matrices; the K-direction
// core-matrix stride (LBO) is 128 bytes and the 8-row-group stride (SBO) 512 bytes, for a K extent of
// 64 sources (a digit or the special basis holds at most 64 primes).  The M byte planes are built on the
// host at context creation in exactly this layout; the y planes are packed by the threads per tile.
//
// Every wait on the MMA-completion mbarrier is bounded: on expiry the kernel records an error flag,
// stops issuing and frees its tensor memory, and the host reports CKKS_ECUDA.
#include "internal.cuh"

namespace ckks {
namespace {

constexpr int kTM = 128, kTN = 16, kKP = 64, kPlanes = 8;
constexpr int kAPlane = kTM * kKP;           // 8192 bytes per A byte plane
constexpr int kBPlane = kTN * kKP;           // 1024 bytes per B byte plane
constexpr int kSmemB = kPlanes * kAPlane;    // B planes follow the A planes
constexpr int kSmemBar = kSmemB + kPlanes * kBPlane;
constexpr int kSmemBytes = 100 * 1024;       // two CTAs per SM, 256 TMEM columns each
constexpr int kTmemCols = 256;

__host__ __device__ __forceinline__ int cm_off(int row, int k)
{
    return (row >> 3) * 512 + (k >> 4) * 128 + (row & 7) * 16 + (k & 15);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Shared-memory matrix descriptor: start address >> 4, LBO 128 B, SBO 512 B, descriptor version 1,
// no swizzle.
__device__ __forceinline__ u64 smem_desc(uint32_t addr)
{
    return (u64)((addr >> 4) & 0x3FFF) | ((u64)(128 >> 4) << 16) | ((u64)(512 >> 4) << 32) | (1ull << 46);
}

// Instruction descriptor: int32 accumulate, unsigned 8-bit A and B, both K-major, N = 16, M = 128.
constexpr uint32_t kIdesc = (2u << 4) | ((uint32_t)(kTN >> 3) << 17) | ((uint32_t)(kTM >> 4) << 24);

__device__ __forceinline__ void mma_u8(uint32_t tmem_d, u64 adesc, u64 bdesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
        :: "r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0));
}

// Bounded wait for the given phase parity of an mbarrier.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity)
{
    for (int i = 0; i < (1 << 18); ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(done) : "r"(bar), "r"(parity) : "memory");
        if (done) return true;
    }
    return false;
}

// (lo, hi) += p 2^SH for a 32-bit p.
template <int SH>
__device__ __forceinline__ void add_shifted(u64 &lo, u64 &hi, uint32_t p)
{
    if constexpr (SH == 0) {
        asm("add.cc.u64 %0, %0, %2;\n\taddc.u64 %1, %1, 0;" : "+l"(lo), "+l"(hi) : "l"((u64)p));
    } else if constexpr (SH < 64) {
        u64 h = 0;
        if constexpr (SH > 32) h = (u64)p >> (64 - SH);
        asm("add.cc.u64 %0, %0, %2;\n\taddc.u64 %1, %1, %3;" : "+l"(lo), "+l"(hi) : "l"((u64)p << SH), "l"(h));
    } else {
        hi += (u64)p << (SH - 64);
    }
}

// Four output columns (CG*4 .. CG*4+3) of this thread's row: load the 15 partial products of each,
// rebuild sum_d P_d 2^(8d) in 128 bits and reduce mod the row's prime.
template <int CG>
__device__ __forceinline__ void epilogue4(uint32_t taddr, u64 *row_out, const PrimeConst &p, bool valid)
{
    uint32_t r[15][4];
#pragma unroll
    for (int d = 0; d < 15; ++d)
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(r[d][0]), "=r"(r[d][1]), "=r"(r[d][2]), "=r"(r[d][3])
                     : "r"(taddr + d * kTN + CG * 4));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
    u64 lo[4] = {0, 0, 0, 0}, hi[4] = {0, 0, 0, 0};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        add_shifted<0>(lo[c], hi[c], r[0][c]);
        add_shifted<8>(lo[c], hi[c], r[1][c]);
        add_shifted<16>(lo[c], hi[c], r[2][c]);
        add_shifted<24>(lo[c], hi[c], r[3][c]);
        add_shifted<32>(lo[c], hi[c], r[4][c]);
        add_shifted<40>(lo[c], hi[c], r[5][c]);
        add_shifted<48>(lo[c], hi[c], r[6][c]);
        add_shifted<56>(lo[c], hi[c], r[7][c]);
        add_shifted<64>(lo[c], hi[c], r[8][c]);
        add_shifted<72>(lo[c], hi[c], r[9][c]);
        add_shifted<80>(lo[c], hi[c], r[10][c]);
        add_shifted<88>(lo[c], hi[c], r[11][c]);
        add_shifted<96>(lo[c], hi[c], r[12][c]);
        add_shifted<104>(lo[c], hi[c], r[13][c]);
        add_shifted<112>(lo[c], hi[c], r[14][c]);
    }
    if (valid) {
        ulonglong2 *o = reinterpret_cast<ulonglong2 *>(row_out + CG * 4);
        o[0] = make_ulonglong2(reduce128(hi[0], lo[0], p), reduce128(hi[1], lo[1], p));
        o[1] = make_ulonglong2(reduce128(hi[2], lo[2], p), reduce128(hi[3], lo[3], p));
    }
}

// Job geometry of one launch (kind 0: ModUp over (ciphertext, digit); kind 1: ModDown over
// (job, component)).
struct TcJobs {
    int kind;
    const u64 *y;         // sources, coefficient form
    u64 *out;             // digits (ModUp) or conversion output (ModDown)
    const uint8_t *apl;   // A byte planes
    int L, LK, alpha, dnum, K, tb_per_digit;
    __device__ __forceinline__ void geometry(int z, int &S, int &T, int &lo, const u64 *&ybase,
                                             const uint8_t *&abase) const
    {
        if (kind == 0) {
            const int b = z / dnum, jd = z - b * dnum;
            lo = jd * alpha;
            S = min(alpha, L - lo);
            T = LK - S;
            ybase = y + ((size_t)b * L + lo) * kN;
            abase = apl + (size_t)jd * tb_per_digit * kPlanes * kAPlane;
        } else {
            lo = 0;
            S = K;
            T = L;
            ybase = y + (size_t)z * K * kN;
            abase = apl;
        }
    }
    __device__ __forceinline__ int prime(int ti, int lo, int S) const
    {
        return kind == 0 ? (ti < lo ? ti : ti + S) : ti;
    }
    __device__ __forceinline__ u64 *row(int z, int t) const
    {
        return kind == 0 ? out + ((size_t)z * LK + t) * kN : out + ((size_t)z * L + t) * kN;
    }
};

constexpr int kThreads = 256;

// Byte planes of 4 sources (s0 .. s0+3) of one coefficient into every B plane.
__device__ __forceinline__ void stage4(uint8_t *bplanes, const u64 *vals, int n, int s0)
{
#pragma unroll
    for (int v = 0; v < kPlanes; ++v) {
        uint32_t w = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) w |= (uint32_t)((vals[i] >> (8 * v)) & 0xff) << (8 * i);
        *reinterpret_cast<uint32_t *>(bplanes + v * kBPlane + cm_off(n, s0)) = w;
    }
}

__global__ void __launch_bounds__(kThreads, 2) conv_tc_kernel(TcJobs jobs, const PrimeConst *__restrict__ pc,
                                                               int *err)
{
    extern __shared__ __align__(1024) uint8_t sm[];
    const int tid = threadIdx.x, warp = tid >> 5, tb = blockIdx.x, z = blockIdx.y;
    int S, T, lo;
    const u64 *ybase;
    const uint8_t *abase;
    jobs.geometry(z, S, T, lo, ybase, abase);
    if (tb * kTM >= T) return;  // uniform per CTA
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + kSmemBar);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + kSmemBar + 8);
    {
        const uint4 *src = reinterpret_cast<const uint4 *>(abase + (size_t)tb * kPlanes * kAPlane);
        uint4 *dst = reinterpret_cast<uint4 *>(sm);
        for (int i = tid; i < kPlanes * kAPlane / 16; i += kThreads) dst[i] = src[i];
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(tslot)), "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" :: "r"(smem_u32(bar)));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // staging task of this thread: coefficient n of the tile, sources s0 .. s0+3
    const int n = tid & 15, s0 = (tid >> 4) * 4;
    const u64 *ysrc = ybase + (size_t)s0 * kN + n;
    u64 pre[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) pre[i] = s0 + i < S ? __ldg(ysrc + (size_t)i * kN) : 0;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tslot;
    const u64 adesc0 = smem_desc(smem_u32(sm)), bdesc0 = smem_desc(smem_u32(sm + kSmemB));
    const bool two_k = S > 32;
    const int quad = warp & 3, row = quad * 32 + (tid & 31);
    const int ti = tb * kTM + row;
    const bool valid = ti < T;
    const int t = valid ? jobs.prime(ti, lo, S) : 0;
    const PrimeConst p = pc[t];
    u64 *row_out = jobs.row(z, t);
    const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16);
    const bool high_cols = warp >= 4;
    uint32_t parity = 0;
    bool ok = true;
    for (int c0 = 0; c0 < kN && ok; c0 += kTN) {
        stage4(sm + kSmemB, pre, n, s0);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
        if (tid == 0) {
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
            for (int u = 0; u < kPlanes; ++u)
#pragma unroll
                for (int v = 0; v < kPlanes; ++v) {
                    const int d = u + v;
                    const uint32_t acc = (u == (d > 7 ? d - 7 : 0)) ? 0u : 1u;  // first write of P_d overwrites
                    const u64 ad = adesc0 + ((u * kAPlane) >> 4), bd = bdesc0 + ((v * kBPlane) >> 4);
                    mma_u8(tmem + d * kTN, ad, bd, acc);
                    if (two_k) mma_u8(tmem + d * kTN, ad + (256 >> 4), bd + (256 >> 4), 1u);
                }
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                         :: "r"(smem_u32(bar)) : "memory");
        }
        // next tile's sources, in flight while the products are formed
        if (c0 + kTN < kN) {
#pragma unroll
            for (int i = 0; i < 4; ++i) pre[i] = s0 + i < S ? __ldg(ysrc + (size_t)i * kN + c0 + kTN) : 0;
        }
        ok = mbar_wait(smem_u32(bar), parity);
        parity ^= 1;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        if (ok) {
            u64 *o = row_out + c0;
            if (high_cols) {
                epilogue4<2>(taddr, o, p, valid);
                epilogue4<3>(taddr, o, p, valid);
            } else {
                epilogue4<0>(taddr, o, p, valid);
                epilogue4<1>(taddr, o, p, valid);
            }
        } else if (tid == 0) {
            atomicExch(err, 1);
        }
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncthreads();
    }
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(kTmemCols));
}

// Host: byte planes of a (targets x sources) matrix given by `at(ti, s)`, one block of 128 targets
// after another, in the shared-memory core-matrix layout.
template <class F>
void build_planes(std::vector<uint8_t> &dst, size_t base, int T, int S, F at)
{
    const int tbs = (T + kTM - 1) / kTM;
    for (int tb = 0; tb < tbs; ++tb)
        for (int r = 0; r < kTM; ++r) {
            const int ti = tb * kTM + r;
            for (int s = 0; s < kKP; ++s) {
                const u64 m = (ti < T && s < S) ? at(ti, s) : 0;
                for (int u = 0; u < kPlanes; ++u)
                    dst[base + ((size_t)tb * kPlanes + u) * kAPlane + cm_off(r, s)] = (uint8_t)(m >> (8 * u));
            }
        }
}

}  // namespace

bool conv_on_tensor(const ckks_ctx *ctx, int sources)
{
    switch (ctx->conv_engine.load(std::memory_order_relaxed)) {
    case CKKS_CONV_INTEGER: return false;
    case CKKS_CONV_TENSOR: return true;
    default: return sources > kTcMinSources;
    }
}

int build_tc_tables(ckks_ctx *ctx, const std::vector<u64> &up_mat, const std::vector<u64> &dn_mat)
{
    Tables &T = ctx->t;
    const int L = ctx->L, K = ctx->K, LK = L + K, alpha = ctx->alpha, dnum = ctx->dnum;
    T.tc_up = nullptr;
    T.tc_dn = nullptr;
    T.tc_tb_per_digit = (LK - 1 + kTM - 1) / kTM;
    {
        const size_t per_digit = (size_t)T.tc_tb_per_digit * kPlanes * kAPlane;
        std::vector<uint8_t> h(per_digit * dnum, 0);
        for (int j = 0; j < dnum; ++j) {
            const int lo = j * alpha, S = std::min(alpha, L - lo);
            build_planes(h, per_digit * j, LK - S, S, [&](int ti, int s) {
                const int t = ti < lo ? ti : ti + S;
                return up_mat[((size_t)j * alpha + s) * LK + t];
            });
        }
        void *d = nullptr;
        if (cudaMalloc(&d, h.size()) != cudaSuccess) {
            cudaGetLastError();
            return set_error(CKKS_ENOMEM, "tensor-core table allocation failed");
        }
        ctx->allocations.push_back(d);
        cudaError_t e = cudaMemcpy(d, h.data(), h.size(), cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_status(e, "cudaMemcpy(tensor-core tables)");
        T.tc_up = static_cast<const uint8_t *>(d);
    }
    {
        const size_t bytes = (size_t)((L + kTM - 1) / kTM) * kPlanes * kAPlane;
        std::vector<uint8_t> h(bytes, 0);
        build_planes(h, 0, L, K, [&](int ti, int s) { return dn_mat[(size_t)s * L + ti]; });
        void *d = nullptr;
        if (cudaMalloc(&d, h.size()) != cudaSuccess) {
            cudaGetLastError();
            return set_error(CKKS_ENOMEM, "tensor-core table allocation failed");
        }
        ctx->allocations.push_back(d);
        cudaError_t e = cudaMemcpy(d, h.data(), h.size(), cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_status(e, "cudaMemcpy(tensor-core tables)");
        T.tc_dn = static_cast<const uint8_t *>(d);
    }
    cudaError_t e = cudaMalloc(&ctx->tc_err, sizeof(int));
    if (e != cudaSuccess) {
        cudaGetLastError();
        return set_error(CKKS_ENOMEM, "flag allocation failed");
    }
    ctx->allocations.push_back(ctx->tc_err);
    e = cudaMemset(ctx->tc_err, 0, sizeof(int));
    if (e != cudaSuccess) return cuda_status(e, "cudaMemset(flag)");
    e = cudaFuncSetAttribute(conv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return cuda_status(e, "cudaFuncSetAttribute(conv_tc_kernel)");
    return CKKS_OK;
}

int launch_conv_tc_up(const ckks_ctx *ctx, const u64 *y, u64 *digits, int batch, cudaStream_t s)
{
    const Tables &T = ctx->t;
    TcJobs j{0, y, digits, T.tc_up, T.L, T.LK, T.alpha, T.dnum, T.K, T.tc_tb_per_digit};
    dim3 grid(T.tc_tb_per_digit, batch * T.dnum);
    conv_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(j, T.pc, ctx->tc_err);
    CKKS_CHECK_LAUNCH("conv_tc_kernel");
    return CKKS_OK;
}

int launch_conv_tc_down(const ckks_ctx *ctx, const u64 *zsrc, u64 *cv, int jobs2, cudaStream_t s)
{
    const Tables &T = ctx->t;
    TcJobs j{1, zsrc, cv, T.tc_dn, T.L, T.LK, T.alpha, T.dnum, T.K, 0};
    dim3 grid((T.L + kTM - 1) / kTM, jobs2);
    conv_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(j, T.pc, ctx->tc_err);
    CKKS_CHECK_LAUNCH("conv_tc_kernel");
    return CKKS_OK;
}

}  // namespace ckks
