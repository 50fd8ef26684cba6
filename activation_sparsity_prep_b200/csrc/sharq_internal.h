// sharq_internal.h -- host-side launch interfaces between the C ABI layer
// and the kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <algorithm>

namespace sharq {

struct PrepareLaunch {
    const void* X;
    const void* gamma;
    const void* beta;     // LayerNorm bias, may be null
    bool layernorm;       // LayerNorm (needs gamma) instead of RMSNorm
    float eps;
    int64_t M;
    int K, n, m, fmt;
    bool weight;          // quantise a whole weight tensor (keep-all, no residual)
    bool residual_shared; // NVFP4 residual quantised with the backbone's tensor scale
    const float* amax;    // no-norm prepare with A_b = max |X| given by the producer, or null
    void* bb_codes;
    void* bb_scales;
    float* bb_tscale;
    void* rs_codes;
    void* rs_scales;
    float* rs_tscale;
    void* mask;
    void* ws;
    void* bb_meta = nullptr;          // pair-granular 4:8 backbone: bb_codes compressed, metadata here
    unsigned long long wait_ns = 0;   // limit of each grid-barrier wait (0: the default, ~1 s)
    int skip_block = -1;              // self-test only: this block never arrives at a barrier
    bool spec_off = false;            // NVFP4 own scale: always run phase 3 (for measurements)
};

size_t prepare_ws_bytes(int64_t M);
cudaError_t launch_prepare(const PrepareLaunch& p, cudaStream_t s, int sms);
// Failure-path self-test (selftest.cu): the library's bounded grid barrier
// with one block that never arrives, and its bounded mbarrier wait on a
// phase that never completes, each bounded by limit_ns.
cudaError_t launch_wait_selftest(uint32_t* counter, unsigned long long limit_ns, cudaStream_t s);

struct LinearLaunch {
    const void* bb_codes;     // compressed [M, K/4] when bb_meta is set
    const void* bb_scales;
    const float* bb_tscale;
    const void* bb_meta;      // pair metadata atoms of a compressed backbone, or null
    const void* rs_codes;
    const void* rs_scales;
    const float* rs_tscale;
    const void* w_codes;      // expert 0 for the grouped form
    const void* w_scales;
    const float* w_tscale;
    int64_t M;                // rows of the prepared operands
    int N, K, fmt;
    void* Y;
    int y_fp32;
    bool one_acc;             // G_b == G_r: both paths into one accumulator
    bool swiglu;              // epilogue emits silu(gate) * up, [M, N/2] bf16, and max |H|
    float* amax;              // swiglu: max |H| (device fp32)
    // grouped form
    const int32_t* row_index; // may be null
    const int32_t* offsets;   // null for the plain linear
    int E;
    int64_t T;
    void* ws;                 // grouped form: gathered operands
};

// Rows of the gathered, per-expert 128-aligned activation operands.
inline int64_t moe_padded_rows(int64_t T, int E) { return (T + 128 * (int64_t)E + 127) / 128 * 128; }
size_t moe_ws_bytes(int64_t T, int E, int K, int fmt);

cudaError_t launch_linear(const LinearLaunch& p, cudaStream_t s, int sms);
cudaError_t launch_moe_linear(const LinearLaunch& p, cudaStream_t s, int sms);

int device_sm_count();

// Read and clear the device status words of each kernel file.
unsigned take_status_prepare();
unsigned take_status_linear();
unsigned take_status_selftest();

}  // namespace sharq
