// ModUp for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc. Typical cases:
//  - a host framework whose own caching allocator already holds the device's memory under a fixed
//    budget, where an allocation behind its back would fail or break its accounting;
//  - a latency-critical loop that cannot absorb the device-wide synchronisation that cudaMalloc and
//    cudaFree can imply.
// ckks_modup_noalloc gives those callers ModUp with no allocation at all. Its only scratch (the
// [batch][L][n] coefficient form of the input, written by the first transform and read by the basis
// conversion) lives in the file-scope device array below. The array is part of the library image, so
// every GPU that loads the library holds its 32 MiB until the process exits.
#include <mutex>

#include "internal.cuh"

namespace {

constexpr size_t kScratchLimbs = 2048;  // 2048 limbs x 16 KiB = 32 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) u64 g_modup_scratch[kScratchLimbs * ckks::kN];

std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of the scratch array on `device` (which must be current). The array's name in host
// code is only a host-side stand-in, so the address comes from cudaGetSymbolAddress. It is resolved
// once per device and cached.
int scratch_address(int device, void **out)
{
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[device]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_modup_scratch);
        if (e != cudaSuccess) return ckks::cuda_status(e, "cudaGetSymbolAddress(modup scratch)");
        g_scratch_addr[device] = p;
    }
    *out = g_scratch_addr[device];
    return CKKS_OK;
}

}  // namespace

using namespace ckks;

extern "C" int ckks_modup_noalloc(const ckks_ctx *ctx, const uint64_t *c_ntt, uint64_t *digits,
                                  int batch, ckks_stream_t stream)
{
    CKKS_TRY(check_ctx(ctx));
    if (batch < 0) return set_error(CKKS_EINVAL, "negative batch");
    if ((size_t)batch * ctx->L > kScratchLimbs)
        return set_error(CKKS_EUNSUPPORTED,
                         "ckks_modup_noalloc: batch * L exceeds the 2048-limb (32 MiB) static scratch");
    if (batch == 0) return CKKS_OK;
    CKKS_TRY(check_ptr(c_ntt, "c_ntt"));
    CKKS_TRY(check_ptr(digits, "digits"));
    if (ctx->device < 0 || ctx->device >= kMaxDevices)
        return set_error(CKKS_EUNSUPPORTED, "device index above 63");
    // the folded conversion builds its tables on first use, which allocates: refuse until they exist
    if (conv_kind(ctx, ctx->alpha) == kConvFolded && !fold_tables_ready(ctx))
        return set_error(CKKS_EUNSUPPORTED,
                         "ckks_modup_noalloc: the folded conversion tables are not built yet (make one "
                         "converting call, e.g. ckks_modup, on this context first)");
    CKKS_TRY(set_device(ctx));
    void *scratch = nullptr;
    CKKS_TRY(scratch_address(ctx->device, &scratch));
    // The first stage writes every scratch word that the later stages read, so nothing needs clearing.
    return modup_stage(ctx, c_ntt, nullptr, (size_t)ctx->L * kN, digits, batch, scratch,
                       (cudaStream_t)stream);
}
