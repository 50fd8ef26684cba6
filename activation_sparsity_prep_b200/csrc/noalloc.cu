// noalloc.cu -- sharq_prepare_noalloc: the preparation operator with its
// scratch memory in a fixed device array instead of a caller-supplied
// workspace.
//
// Some callers cannot allocate device memory at the point where they run the
// prepare: code enqueued while a stream is being captured into a CUDA graph
// (an allocation there breaks or invalidates the capture), plugin and
// runtime hooks whose host framework owns every byte of device memory and
// forbids allocations inside its execute callback, and latency-critical
// serving loops that cannot afford the implicit device-wide synchronisation
// of cudaMalloc/cudaFree.  For them this entry point takes only the inputs
// and outputs; the scratch (tensor-wide maxima, grid barrier, per-row RMS
// factors) lives in the file-scope array below.  The array is part of the
// loaded library: every GPU that loads the library holds it until the
// process exits.
#include "../../include/sharq.h"
#include "common.cuh"
#include "sharq_internal.h"

#include <mutex>

namespace {

// 64 header bytes + 4 bytes per row.
constexpr size_t kScratchBytes = 64 + 4 * (size_t)SHARQ_NOALLOC_MAX_ROWS;

static __device__ __align__(256) uint8_t g_prepare_scratch[kScratchBytes];

// Device address of g_prepare_scratch, looked up once per device with that
// device current.  In host code the array's name is only a host-side
// stand-in; the kernel must be given this address.
void* scratch_address(cudaError_t* err) {
    static std::mutex mu;
    static void* addr[64] = {nullptr};
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess) return nullptr;
    if (dev < 0 || dev >= 64) { *err = cudaErrorInvalidDevice; return nullptr; }
    std::lock_guard<std::mutex> g(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        *err = cudaGetSymbolAddress(&p, g_prepare_scratch);
        if (*err != cudaSuccess) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" SHARQ_API sharq_status sharq_prepare_noalloc(const void* X_bf16, const void* gamma_bf16,
                                                        float eps, const sharq_prepared* out,
                                                        void* stream) {
    if (!out) return SHARQ_ERR_INVALID_ARG;
    const sharq_prepared& o = *out;
    if (o.bb_meta) return SHARQ_ERR_UNSUPPORTED;   // the compressed pair backbone is not offered here
    if (o.M < 0 || o.M > SHARQ_NOALLOC_MAX_ROWS) return SHARQ_ERR_INVALID_ARG;   // beyond the fixed scratch
    if (!(o.fmt == SHARQ_NVFP4 || o.fmt == SHARQ_MXFP4) || o.K <= 0 || o.K % 256 != 0)
        return SHARQ_ERR_INVALID_ARG;
    if (!(o.m == 2 || o.m == 4 || o.m == 8) || o.n < 1 || o.n > o.m) return SHARQ_ERR_INVALID_ARG;
    if (o.residual_scale != SHARQ_RESIDUAL_OWN && o.residual_scale != SHARQ_RESIDUAL_SHARED)
        return SHARQ_ERR_INVALID_ARG;
    if (!(eps >= 0.0f) || !(eps < 1e30f)) return SHARQ_ERR_INVALID_ARG;
    if (!o.bb_tscale || !o.rs_tscale) return SHARQ_ERR_INVALID_ARG;
    if (o.M > 0 && (!X_bf16 || !o.bb_codes || !o.bb_scales || !o.rs_codes || !o.rs_scales))
        return SHARQ_ERR_INVALID_ARG;
    if (!aligned16(X_bf16) || !aligned16(gamma_bf16) || !aligned16(o.bb_codes) ||
        !aligned16(o.bb_scales) || !aligned16(o.rs_codes) || !aligned16(o.rs_scales) ||
        !aligned16(o.mask) || ((uintptr_t)o.bb_tscale & 3u) || ((uintptr_t)o.rs_tscale & 3u))
        return SHARQ_ERR_INVALID_ARG;
    cudaError_t err = cudaSuccess;
    void* scratch = scratch_address(&err);
    if (!scratch) return SHARQ_ERR_CUDA;
    sharq::PrepareLaunch p{};
    p.X = X_bf16; p.gamma = gamma_bf16; p.eps = eps; p.M = o.M; p.K = o.K; p.n = o.n; p.m = o.m;
    p.fmt = o.fmt; p.weight = false; p.residual_shared = o.residual_scale == SHARQ_RESIDUAL_SHARED;
    p.bb_codes = o.bb_codes; p.bb_scales = o.bb_scales; p.bb_tscale = o.bb_tscale;
    p.rs_codes = o.rs_codes; p.rs_scales = o.rs_scales; p.rs_tscale = o.rs_tscale;
    p.mask = o.mask;
    p.ws = scratch;   // its 64-byte header is cleared by the launch before the kernel runs
    cudaError_t e = sharq::launch_prepare(p, static_cast<cudaStream_t>(stream), sharq::device_sm_count());
    return e == cudaSuccess ? SHARQ_OK : SHARQ_ERR_CUDA;
}
