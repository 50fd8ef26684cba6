// abi.cu -- extern "C" entry points of libsharq (declared in include/sharq.h).
//
// Argument validation happens here, on the host, before anything is
// enqueued; the kernels themselves live in prepare.cu and linear.cu.
#include "../../include/sharq.h"
#include "common.cuh"
#include "sharq_internal.h"

#include <mutex>

namespace sharq {

int device_sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    static std::mutex mu;
    static int cache[64] = {0};
    std::lock_guard<std::mutex> g(mu);
    if (dev < 64 && cache[dev]) return cache[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (dev < 64) cache[dev] = n;
    return n;
}

}  // namespace sharq

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_fmt(int fmt) { return fmt == SHARQ_NVFP4 || fmt == SHARQ_MXFP4; }

bool valid_shape(int64_t rows, int K) { return rows >= 0 && K > 0 && K % 256 == 0; }

sharq_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return SHARQ_OK;
    if (e == cudaErrorNotSupported) return SHARQ_ERR_UNSUPPORTED;
    return SHARQ_ERR_CUDA;
}

int block_size(int fmt) { return fmt == SHARQ_NVFP4 ? 16 : 32; }

}  // namespace

extern "C" {

const char* sharq_status_string(int status) {
    switch (status) {
        case SHARQ_OK: return "ok";
        case SHARQ_ERR_INVALID_ARG: return "invalid argument";
        case SHARQ_ERR_UNSUPPORTED: return "unsupported configuration";
        case SHARQ_ERR_CUDA: return "CUDA error";
        case SHARQ_ERR_TIMEOUT: return "device wait timed out";
        default: return "unknown status";
    }
}

size_t sharq_scale_bytes(int64_t rows, int K, int fmt) {
    if (!valid_fmt(fmt) || !valid_shape(rows, K)) return 0;
    int64_t rpad = (rows + 127) / 128 * 128;
    return (size_t)(rpad * (K / block_size(fmt)));
}

size_t sharq_pair_meta_bytes(int64_t rows, int K) {
    if (!valid_shape(rows, K)) return 0;
    return (size_t)((rows + 127) / 128 * 128) * (size_t)(K / 16);
}

size_t sharq_prepare_workspace_bytes(int64_t M, int K, int fmt) {
    if (!valid_fmt(fmt) || !valid_shape(M, K)) return 0;
    return sharq::prepare_ws_bytes(M);
}

sharq_status sharq_quantize_weight(const void* W_bf16, const sharq_weight* out, void* ws,
                                   size_t ws_bytes, void* stream) {
    if (!out || !W_bf16 || !ws) return SHARQ_ERR_INVALID_ARG;
    if (!valid_fmt(out->fmt) || !valid_shape(out->N, out->K) || out->N % 128 != 0 || out->N == 0)
        return SHARQ_ERR_INVALID_ARG;
    if (!out->codes || !out->scales || !out->tensor_scale) return SHARQ_ERR_INVALID_ARG;
    if (!aligned16(W_bf16) || !aligned16(out->codes) || !aligned16(out->scales) || !aligned16(ws) ||
        ((uintptr_t)out->tensor_scale & 3u))
        return SHARQ_ERR_INVALID_ARG;
    if (ws_bytes < sharq::prepare_ws_bytes(out->N)) return SHARQ_ERR_INVALID_ARG;
    sharq::PrepareLaunch p{};
    p.X = W_bf16; p.gamma = nullptr; p.eps = 0.f; p.M = out->N; p.K = out->K;
    p.n = 8; p.m = 8; p.fmt = out->fmt; p.weight = true;
    p.bb_codes = out->codes; p.bb_scales = out->scales; p.bb_tscale = out->tensor_scale;
    p.ws = ws;
    return cuda_status(sharq::launch_prepare(p, static_cast<cudaStream_t>(stream),
                                             sharq::device_sm_count()));
}

static sharq_status prepare_common(const void* X_bf16, const void* gamma_bf16, const void* beta_bf16,
                                   bool layernorm, float eps, const sharq_prepared* out, void* ws,
                                   size_t ws_bytes, void* stream, const float* amax = nullptr,
                                   unsigned long long wait_ns = 0, int skip_block = -1) {
    if (!out || !ws) return SHARQ_ERR_INVALID_ARG;
    if (layernorm && out->M > 0 && !gamma_bf16) return SHARQ_ERR_INVALID_ARG;
    if (!aligned16(beta_bf16)) return SHARQ_ERR_INVALID_ARG;
    const sharq_prepared& o = *out;
    if (!valid_fmt(o.fmt) || !valid_shape(o.M, o.K)) return SHARQ_ERR_INVALID_ARG;
    if (!(o.m == 2 || o.m == 4 || o.m == 8) || o.n < 1 || o.n > o.m) return SHARQ_ERR_INVALID_ARG;
    if (o.residual_scale != SHARQ_RESIDUAL_OWN && o.residual_scale != SHARQ_RESIDUAL_SHARED)
        return SHARQ_ERR_INVALID_ARG;
    if (!(eps >= 0.0f) || !(eps < 1e30f)) return SHARQ_ERR_INVALID_ARG;
    if (!o.bb_tscale || !o.rs_tscale) return SHARQ_ERR_INVALID_ARG;
    if (o.M > 0 && (!X_bf16 || !o.bb_codes || !o.bb_scales || !o.rs_codes || !o.rs_scales))
        return SHARQ_ERR_INVALID_ARG;
    if (!aligned16(X_bf16) || !aligned16(gamma_bf16) || !aligned16(o.bb_codes) ||
        !aligned16(o.bb_scales) || !aligned16(o.rs_codes) || !aligned16(o.rs_scales) ||
        !aligned16(o.mask) || !aligned16(ws) || ((uintptr_t)o.bb_tscale & 3u) ||
        ((uintptr_t)o.rs_tscale & 3u))
        return SHARQ_ERR_INVALID_ARG;
    if (ws_bytes < sharq::prepare_ws_bytes(o.M)) return SHARQ_ERR_INVALID_ARG;
    if (o.bb_meta) {
        // pair-granular 4:8 backbone: MXFP4, RMSNorm or no norm, the norm computed here
        if (o.fmt != SHARQ_MXFP4 || o.n != 4 || o.m != 8) return SHARQ_ERR_INVALID_ARG;
        if (!aligned16(o.bb_meta)) return SHARQ_ERR_INVALID_ARG;
        if (layernorm || amax || skip_block >= 0) return SHARQ_ERR_UNSUPPORTED;
    }
    sharq::PrepareLaunch p{};
    p.X = X_bf16; p.gamma = gamma_bf16; p.eps = eps; p.M = o.M; p.K = o.K; p.n = o.n; p.m = o.m;
    p.bb_meta = o.bb_meta;
    p.beta = layernorm ? beta_bf16 : nullptr; p.layernorm = layernorm;
    p.fmt = o.fmt; p.weight = false; p.residual_shared = o.residual_scale == SHARQ_RESIDUAL_SHARED;
    p.bb_codes = o.bb_codes; p.bb_scales = o.bb_scales; p.bb_tscale = o.bb_tscale;
    p.rs_codes = o.rs_codes; p.rs_scales = o.rs_scales; p.rs_tscale = o.rs_tscale;
    p.mask = o.mask; p.ws = ws; p.amax = amax;
    p.wait_ns = wait_ns; p.skip_block = skip_block;
    return cuda_status(sharq::launch_prepare(p, static_cast<cudaStream_t>(stream),
                                             sharq::device_sm_count()));
}

sharq_status sharq_prepare(const void* X_bf16, const void* gamma_bf16, float eps,
                           const sharq_prepared* out, void* ws, size_t ws_bytes, void* stream) {
    return prepare_common(X_bf16, gamma_bf16, nullptr, false, eps, out, ws, ws_bytes, stream);
}

sharq_status sharq_prepare_layernorm(const void* X_bf16, const void* gamma_bf16, const void* beta_bf16,
                                     float eps, const sharq_prepared* out, void* ws, size_t ws_bytes,
                                     void* stream) {
    return prepare_common(X_bf16, gamma_bf16, beta_bf16, true, eps, out, ws, ws_bytes, stream);
}

sharq_status sharq_prepare_amax(const void* X_bf16, const float* amax, const sharq_prepared* out,
                                void* ws, size_t ws_bytes, void* stream) {
    if (!amax || ((uintptr_t)amax & 3u)) return SHARQ_ERR_INVALID_ARG;
    return prepare_common(X_bf16, nullptr, nullptr, false, 0.0f, out, ws, ws_bytes, stream, amax);
}

static sharq_status check_linear_args(const sharq_prepared* x, const sharq_weight* w, void* Y) {
    if (!x || !w || (!Y && x->M > 0)) return SHARQ_ERR_INVALID_ARG;
    if (!valid_fmt(x->fmt) || x->fmt != w->fmt) return SHARQ_ERR_INVALID_ARG;
    if (x->residual_scale != SHARQ_RESIDUAL_OWN && x->residual_scale != SHARQ_RESIDUAL_SHARED)
        return SHARQ_ERR_INVALID_ARG;
    if (!valid_shape(x->M, x->K) || x->K != w->K) return SHARQ_ERR_INVALID_ARG;
    if (w->N <= 0 || w->N % 128 != 0) return SHARQ_ERR_INVALID_ARG;
    if (!x->bb_tscale || !x->rs_tscale || !w->codes || !w->scales || !w->tensor_scale)
        return SHARQ_ERR_INVALID_ARG;
    if (x->M > 0 && (!x->bb_codes || !x->bb_scales || !x->rs_codes || !x->rs_scales))
        return SHARQ_ERR_INVALID_ARG;
    if (!aligned16(x->bb_codes) || !aligned16(x->bb_scales) || !aligned16(x->rs_codes) ||
        !aligned16(x->rs_scales) || !aligned16(w->codes) || !aligned16(w->scales) || !aligned16(Y))
        return SHARQ_ERR_INVALID_ARG;
    if (x->bb_meta && (x->fmt != SHARQ_MXFP4 || !aligned16(x->bb_meta))) return SHARQ_ERR_INVALID_ARG;
    return SHARQ_OK;
}

sharq_status sharq_linear(const sharq_prepared* x, const sharq_weight* w, void* Y, int y_is_fp32,
                          void* stream) {
    sharq_status st = check_linear_args(x, w, Y);
    if (st != SHARQ_OK) return st;
    if (x->M == 0) return SHARQ_OK;
    sharq::LinearLaunch p{};
    p.bb_codes = x->bb_codes; p.bb_scales = x->bb_scales; p.bb_tscale = x->bb_tscale;
    p.bb_meta = x->bb_meta;
    p.rs_codes = x->rs_codes; p.rs_scales = x->rs_scales; p.rs_tscale = x->rs_tscale;
    p.w_codes = w->codes; p.w_scales = w->scales; p.w_tscale = w->tensor_scale;
    p.M = x->M; p.N = w->N; p.K = x->K; p.fmt = x->fmt; p.Y = Y; p.y_fp32 = y_is_fp32 ? 1 : 0;
    p.one_acc = x->fmt == SHARQ_MXFP4 || x->residual_scale == SHARQ_RESIDUAL_SHARED;
    return cuda_status(sharq::launch_linear(p, static_cast<cudaStream_t>(stream),
                                            sharq::device_sm_count()));
}

sharq_status sharq_linear_swiglu(const sharq_prepared* x, const sharq_weight* w, void* H,
                                 float* h_amax, void* stream) {
    sharq_status st = check_linear_args(x, w, H);
    if (st != SHARQ_OK) return st;
    if (!h_amax || ((uintptr_t)h_amax & 3u)) return SHARQ_ERR_INVALID_ARG;
    if (x->bb_meta) return SHARQ_ERR_UNSUPPORTED;
    if (x->M == 0)
        return cuda_status(cudaMemsetAsync(h_amax, 0, sizeof(float), static_cast<cudaStream_t>(stream)));
    sharq::LinearLaunch p{};
    p.bb_codes = x->bb_codes; p.bb_scales = x->bb_scales; p.bb_tscale = x->bb_tscale;
    p.rs_codes = x->rs_codes; p.rs_scales = x->rs_scales; p.rs_tscale = x->rs_tscale;
    p.w_codes = w->codes; p.w_scales = w->scales; p.w_tscale = w->tensor_scale;
    p.M = x->M; p.N = w->N; p.K = x->K; p.fmt = x->fmt; p.Y = H; p.y_fp32 = 0;
    p.one_acc = x->fmt == SHARQ_MXFP4 || x->residual_scale == SHARQ_RESIDUAL_SHARED;
    p.swiglu = true; p.amax = h_amax;
    return cuda_status(sharq::launch_linear(p, static_cast<cudaStream_t>(stream),
                                            sharq::device_sm_count()));
}

size_t sharq_moe_workspace_bytes(int64_t T, int E, int K, int fmt) {
    if (!valid_fmt(fmt) || !valid_shape(T, K) || E <= 0) return 0;
    return sharq::moe_ws_bytes(T, E, K, fmt);
}

static sharq_status moe_common(const sharq_prepared* x, const int32_t* row_index,
                               const int32_t* expert_offsets, int E, int64_t T, const sharq_weight* w,
                               void* Y, int y_is_fp32, float* h_amax, void* ws, size_t ws_bytes,
                               void* stream) {
    if (!x || !w) return SHARQ_ERR_INVALID_ARG;
    if (!expert_offsets || E <= 0 || T < 0 || (!row_index && T != x->M)) return SHARQ_ERR_INVALID_ARG;
    if (x->bb_meta) return SHARQ_ERR_UNSUPPORTED;
    if (E > 256) return SHARQ_ERR_UNSUPPORTED;
    if (T > 0 && (!Y || !ws)) return SHARQ_ERR_INVALID_ARG;
    if (!valid_fmt(x->fmt) || x->fmt != w->fmt || !valid_shape(x->M, x->K) || x->K != w->K)
        return SHARQ_ERR_INVALID_ARG;
    if (x->residual_scale != SHARQ_RESIDUAL_OWN && x->residual_scale != SHARQ_RESIDUAL_SHARED)
        return SHARQ_ERR_INVALID_ARG;
    if (w->N <= 0 || w->N % 128 != 0 || !w->codes || !w->scales || !w->tensor_scale)
        return SHARQ_ERR_INVALID_ARG;
    if (!x->bb_tscale || !x->rs_tscale) return SHARQ_ERR_INVALID_ARG;
    if (x->M > 0 && (!x->bb_codes || !x->bb_scales || !x->rs_codes || !x->rs_scales))
        return SHARQ_ERR_INVALID_ARG;
    if (!aligned16(x->bb_codes) || !aligned16(x->bb_scales) || !aligned16(x->rs_codes) ||
        !aligned16(x->rs_scales) || !aligned16(w->codes) || !aligned16(w->scales) || !aligned16(Y) ||
        !aligned16(ws) || ((uintptr_t)row_index & 3u) || ((uintptr_t)expert_offsets & 3u) ||
        ((uintptr_t)h_amax & 3u))
        return SHARQ_ERR_INVALID_ARG;
    if (ws_bytes < sharq::moe_ws_bytes(T, E, x->K, x->fmt)) return SHARQ_ERR_INVALID_ARG;
    if (T == 0) {
        if (!h_amax) return SHARQ_OK;
        return cuda_status(cudaMemsetAsync(h_amax, 0, sizeof(float), static_cast<cudaStream_t>(stream)));
    }
    sharq::LinearLaunch p{};
    p.bb_codes = x->bb_codes; p.bb_scales = x->bb_scales; p.bb_tscale = x->bb_tscale;
    p.rs_codes = x->rs_codes; p.rs_scales = x->rs_scales; p.rs_tscale = x->rs_tscale;
    p.w_codes = w->codes; p.w_scales = w->scales; p.w_tscale = w->tensor_scale;
    p.M = x->M; p.N = w->N; p.K = x->K; p.fmt = x->fmt; p.Y = Y; p.y_fp32 = y_is_fp32 ? 1 : 0;
    p.one_acc = x->fmt == SHARQ_MXFP4 || x->residual_scale == SHARQ_RESIDUAL_SHARED;
    p.row_index = row_index; p.offsets = expert_offsets; p.E = E; p.T = T; p.ws = ws;
    p.swiglu = h_amax != nullptr; p.amax = h_amax;
    return cuda_status(sharq::launch_moe_linear(p, static_cast<cudaStream_t>(stream),
                                                sharq::device_sm_count()));
}

sharq_status sharq_moe_linear(const sharq_prepared* x, const int32_t* row_index,
                              const int32_t* expert_offsets, int E, int64_t T,
                              const sharq_weight* w, void* Y, int y_is_fp32, void* ws,
                              size_t ws_bytes, void* stream) {
    return moe_common(x, row_index, expert_offsets, E, T, w, Y, y_is_fp32, nullptr, ws, ws_bytes, stream);
}

sharq_status sharq_moe_linear_swiglu(const sharq_prepared* x, const int32_t* row_index,
                                     const int32_t* expert_offsets, int E, int64_t T,
                                     const sharq_weight* w, void* H, float* h_amax, void* ws,
                                     size_t ws_bytes, void* stream) {
    if (!h_amax) return SHARQ_ERR_INVALID_ARG;
    return moe_common(x, row_index, expert_offsets, E, T, w, H, 0, h_amax, ws, ws_bytes, stream);
}

sharq_status sharq_selftest_wait_timeout(void* ws, int64_t limit_us, void* stream) {
    if (!ws || ((uintptr_t)ws & 3u) || limit_us < 1000 || limit_us > 1000000)
        return SHARQ_ERR_INVALID_ARG;
    return cuda_status(sharq::launch_wait_selftest(static_cast<uint32_t*>(ws),
                                                   (unsigned long long)limit_us * 1000ull,
                                                   static_cast<cudaStream_t>(stream)));
}

sharq_status sharq_selftest_prepare_timeout(const void* X_bf16, const sharq_prepared* out, void* ws,
                                            size_t ws_bytes, int64_t limit_us, void* stream) {
    if (!out || out->fmt != SHARQ_NVFP4 || out->residual_scale != SHARQ_RESIDUAL_OWN || out->M < 1 ||
        limit_us < 1000 || limit_us > 1000000)
        return SHARQ_ERR_INVALID_ARG;
    return prepare_common(X_bf16, nullptr, nullptr, false, 0.0f, out, ws, ws_bytes, stream, nullptr,
                          (unsigned long long)limit_us * 1000ull, 0);
}

sharq_status sharq_last_device_status(void* stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return SHARQ_ERR_CUDA;
    unsigned v = sharq::take_status_prepare() | sharq::take_status_linear() |
                 sharq::take_status_selftest();
    if (v & sharq::kStatusReadFailed) return SHARQ_ERR_CUDA;
    if (v & (sharq::kStatusGridTimeout | sharq::kStatusMbarTimeout)) return SHARQ_ERR_TIMEOUT;
    if (v) return SHARQ_ERR_CUDA;
    return SHARQ_OK;
}

}  // extern "C"
