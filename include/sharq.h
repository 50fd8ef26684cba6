/*
 * sharq.h -- C ABI of the B200 (sm_100a) SharQ hot path.
 *
 * SharQ (SharQ: Bridging Activation Sparsity and FP4 Quantization for LLM
 * Inference, arXiv 2606.26587, Abstract) splits each linear layer's input
 * online into an outlier-dominated N:M-sparse backbone and a dense residual
 * taken against the *dequantised* backbone, quantises both to FP4, and runs
 * a sparse FP4 GEMM on the backbone plus a dense FP4 GEMM on the residual,
 * both reading one shared FP4 weight payload with per-path scale views.  A
 * fused preparation operator absorbs normalisation, mask generation and
 * residual construction.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The
 *     library allocates nothing and keeps no reference after a call returns.
 *   - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *     stream.  Work is enqueued asynchronously; no call synchronises except
 *     sharq_last_device_status().
 *   - Pointers must be 16-byte aligned.  K % 256 == 0, N % 128 == 0, M >= 0.
 *   - A violated precondition returns SHARQ_ERR_INVALID_ARG (or
 *     SHARQ_ERR_UNSUPPORTED for a valid but unimplemented choice) before any
 *     work is enqueued.  A failed launch returns SHARQ_ERR_CUDA.  A bounded
 *     device-side wait that gives up (about one second) records a timeout in
 *     a device status word that sharq_last_device_status() reports.
 *   - Inputs must be finite.  Non-finite inputs are outside the contract.
 *
 * Data layouts (all row-major unless stated)
 *   bf16 tensors           raw bfloat16, [rows, K]
 *   FP4 codes              uint8 [rows, K/2]; E2M1 element 2j in bits 3:0 and
 *                          element 2j+1 in bits 7:4 of byte j
 *   block scales           "MMA-ready" atoms: rows are padded to a multiple
 *                          of 128 and the scale matrix [rows_pad, K/B] (B =
 *                          16 for NVFP4 with E4M3 codes, 32 for MXFP4 with
 *                          E8M0 codes) is stored as 512-byte atoms of 128 rows
 *                          x 4 scales.  Scale (r, s) lives at byte
 *                            ((r/128) * (K/B/4) + s/4) * 512
 *                            + (r%32) * 16 + ((r%128)/32) * 4 + s%4.
 *                          sharq_scale_bytes() gives the buffer size.
 *   tensor scale           one fp32 decode scale G (NVFP4: amax / 2688; it
 *                          is 1.0 for MXFP4 and for an all-zero tensor)
 *   mask (optional)        uint8 [M, K/8]; bit t of byte j set when element
 *                          8j+t is in the backbone
 */
#ifndef SHARQ_H
#define SHARQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SHARQ_API __attribute__((visibility("default")))
#else
#define SHARQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SHARQ_OK = 0,
    SHARQ_ERR_INVALID_ARG = 1,
    SHARQ_ERR_UNSUPPORTED = 2,
    SHARQ_ERR_CUDA = 3,
    SHARQ_ERR_TIMEOUT = 4
} sharq_status;

typedef enum {
    SHARQ_NVFP4 = 0,   /* E2M1 codes, E4M3 scale per 16 elements, fp32 tensor scale */
    SHARQ_MXFP4 = 1    /* E2M1 codes, E8M0 scale per 32 elements, no tensor scale   */
} sharq_format;

/* Tensor scale of the residual (NVFP4).  The abstract gives every FP4
 * tensor its own scaling without saying whether the residual shares the
 * backbone's; OWN (its own amax) is the plain reading and the default.
 * SHARED quantises the residual against the backbone's tensor amax, so
 * G_r = G_b: the preparation needs one tensor-wide reduction fewer and the
 * linear accumulates both paths in one accumulator.  MXFP4 has no tensor
 * scale, so the setting changes nothing there. */
typedef enum {
    SHARQ_RESIDUAL_OWN = 0,
    SHARQ_RESIDUAL_SHARED = 1
} sharq_residual_scale;

/* One FP4 weight payload shared by both GEMM paths (Abstract: a single FP4
 * weight payload with path-specific scale views).  Both paths use the same
 * codes and the same MMA-ready scale atoms, which is the layout the block-
 * scaled MMA reads for either path, so one scale copy serves as both views.
 * For a stacked (grouped) weight: codes [E, N, K/2], scales E consecutive
 * buffers of sharq_scale_bytes(N, K, fmt) bytes, tensor_scale [E]. */
typedef struct {
    void*  codes;
    void*  scales;
    float* tensor_scale;
    int    N, K;
    int    fmt;          /* sharq_format */
} sharq_weight;

/* Output of the preparation operator: the backbone and residual operands. */
typedef struct {
    void*  bb_codes;     /* [M, K/2]                                        */
    void*  bb_scales;    /* sharq_scale_bytes(M, K, fmt) bytes              */
    float* bb_tscale;    /* [1] backbone decode scale G_b                   */
    void*  rs_codes;     /* [M, K/2]                                        */
    void*  rs_scales;    /* sharq_scale_bytes(M, K, fmt) bytes              */
    float* rs_tscale;    /* [1] residual decode scale G_r                   */
    void*  mask;         /* optional [M, K/8] bitmask, NULL to skip         */
    int    M, K, n, m;
    int    fmt;          /* sharq_format */
    int    residual_scale;   /* sharq_residual_scale (0 = OWN)              */
    void*  bb_meta;      /* NULL: the backbone is zero-filled codes [M, K/2]
                            under the element-wise n:m mask.  Non-NULL: the
                            pair-granular 4:8 backbone of the FP4 sparse
                            MMA (MXFP4 only, n = 4, m = 8): in every aligned
                            group of 8 elements the two pairs of largest
                            pair magnitude max(|y_2i|, |y_2i+1|) are kept
                            (ties: lower pair index); bb_codes then holds
                            the kept pairs' code bytes in order, [M, K/4],
                            and bb_meta their pair indices,
                            sharq_pair_meta_bytes(M, K) bytes (layout
                            below).                                         */
} sharq_prepared;

/* Pair metadata of a compressed backbone (bb_meta): per group of 8
 * elements a nibble with the lower kept pair's index in bits 1:0 and the
 * higher one's in bits 3:2; group 2j of a row's 256-element K block in the
 * low nibble of byte j.  Stored in MMA-ready atoms of 128 rows x 256
 * elements (16 bytes per row, row r at byte 16 * (r % 128)), atom
 * (k-block kb, row block rb) at byte (kb * rows_pad / 128 + rb) * 2048,
 * rows padded to a multiple of 128 (padding rows hold 0x44: pairs 0 and 1
 * of zero codes). */
SHARQ_API size_t sharq_pair_meta_bytes(int64_t rows, int K);

/* Human-readable name of a status code (static string). */
SHARQ_API const char* sharq_status_string(int status);

/* Bytes of one MMA-ready block-scale buffer for `rows` x K (rows padded to
 * 128).  Returns 0 for invalid arguments. */
SHARQ_API size_t sharq_scale_bytes(int64_t rows, int K, int fmt);

/* Workspace the preparation operator needs (tensor-wide maxima, a grid
 * barrier and two fp32 per row).  Caller-owned device memory; its content on
 * entry does not matter.  Calls that share a workspace must not overlap. */
SHARQ_API size_t sharq_prepare_workspace_bytes(int64_t M, int K, int fmt);

/* Offline weight quantisation (once per layer; Abstract: shared FP4 weight
 * payload).  W bf16 [N, K] -> out->codes, out->scales, out->tensor_scale,
 * with NVFP4 scales from the tensor-wide amax (G = amax / 2688, block scale
 * E4M3(amax_block * 2688 / (6 * amax))) or MXFP4 scales (E8M0 exponent
 * floor(log2 amax_block) - 2).  `out->N, K, fmt` must be filled in by the
 * caller.  ws: sharq_prepare_workspace_bytes(N, K, fmt) bytes. */
SHARQ_API sharq_status sharq_quantize_weight(const void* W_bf16, const sharq_weight* out,
                                   void* ws, size_t ws_bytes, void* stream);

/* Fused preparation operator (Abstract: one operator absorbing layer
 * normalisation, mask generation and residual construction).  For X bf16
 * [M, K]:
 *   y   = RMSNorm(X) * gamma per row (fp32, fixed reduction order), or y = X
 *         when gamma is NULL;
 *   keep: in every aligned group of m along K the n entries of largest |y|
 *         (lower index first on ties);
 *   backbone B = keep ? y : 0, quantised to FP4 with its own tensor scale;
 *   residual r = y - dequant(Q(B)), quantised to FP4 with its own tensor
 *         scale (out->residual_scale = SHARQ_RESIDUAL_OWN) or the
 *         backbone's (SHARQ_RESIDUAL_SHARED).
 * Fills the buffers named in *out (out->M, K, n, m, fmt must match the
 * arguments).  Supported: m in {2, 4, 8}, 1 <= n <= m.  ws:
 * sharq_prepare_workspace_bytes(M, K, fmt) bytes. */
SHARQ_API sharq_status sharq_prepare(const void* X_bf16, const void* gamma_bf16, float eps,
                           const sharq_prepared* out, void* ws, size_t ws_bytes,
                           void* stream);

/* The preparation operator with LayerNorm in front (the mean-subtracting
 * norm of DiT and vision layers; the pages evaluate vision-language and
 * video models alongside LLMs but do not define the norm's arithmetic):
 *   mu  = sum(x) / K and var = sum((x - mu)^2) / K, each summed in the same
 *         fixed order as the RMS sum (32 lanes, 8-element chunk c to lane
 *         c mod 32, element order within a lane, xor butterfly 16..1);
 *   y   = fl(fl(fl(x - mu) * rstd) * gamma) [+ beta], rstd = 1/sqrt(var+eps);
 * then the mask, backbone and residual exactly as sharq_prepare.  gamma bf16
 * [K] is required (SHARQ_ERR_INVALID_ARG when NULL and M > 0); beta bf16
 * [K] may be NULL (no bias; adding a zero bias would turn -0 into +0).
 * Same buffers, preconditions and workspace as sharq_prepare. */
SHARQ_API sharq_status sharq_prepare_layernorm(const void* X_bf16, const void* gamma_bf16,
                                               const void* beta_bf16, float eps,
                                               const sharq_prepared* out, void* ws, size_t ws_bytes,
                                               void* stream);

/* Two-path FP4 linear (Abstract: a sparse FP4 GEMM on the backbone and a
 * dense FP4 GEMM on the residual, one shared weight payload):
 *   Y[i,j] = G_w * (G_b * S_b[i,j] + G_r * S_r[i,j]),
 *   S_p = sum_k val(p)[i,k] s(p)[i,k/B] * val(w)[j,k] s(w)[j,k/B].
 * Both products accumulate in fp32 tensor memory from one weight tile per
 * k-step, in two accumulators; when G_b = G_r by construction (MXFP4, whose
 * tensor scales sharq_prepare writes as 1, or SHARQ_RESIDUAL_SHARED) in one,
 * Y = G_w * G_b * (S_b + S_r), and rs_tscale is not read.  Y is bf16
 * [M, N] (y_is_fp32 = 0) or fp32 [M, N]. */
SHARQ_API sharq_status sharq_linear(const sharq_prepared* x, const sharq_weight* w,
                          void* Y, int y_is_fp32, void* stream);

/* Producer-fused MLP (the preparation operator of the Abstract, moved in
 * front of the down projection's producer).  For a SwiGLU MLP the down
 * projection's input is H = silu(x W_g^T) * (x W_u^T) (Shazeer, "GLU Variants
 * Improve Transformer", 2020).  sharq_linear_swiglu runs the two-path linear
 * of the gate+up projection and applies the gate in its epilogue:
 *   w   holds 2I rows, interleaved per 128: rows 128t .. 128t+63 are gate
 *       rows 64t .. 64t+63, rows 128t+64 .. 128t+127 the up rows with the
 *       same indices (w->N = 2I, a multiple of 128);
 *   g,u = the fp32 values sharq_linear would round to bf16 for those rows;
 *   H[i, 64t+j] = bf16_rne(fl(silu(g) * u)), silu(g) = g / (1 + e^-g) in
 *       fp32 with the fast exponential and divide: relative error within
 *       (5 + 1.2 |g|) 2^-23 for g > -87 (0 below, where |silu| < 1e-36);
 *       H is bf16 [M, I] (16-byte aligned, device);
 *   *h_amax = max |H| over the whole tensor (fp32 holding a bf16 value;
 *       device pointer, 4-byte aligned, written by this call; 0 for M = 0).
 * Like sharq_linear, M <= 64 runs the weight-streaming decode form (the
 * gate and up rows of a feature meet through shared memory), larger M the
 * row-tiled kernel.  Errors as sharq_linear; NULL h_amax is
 * SHARQ_ERR_INVALID_ARG. */
SHARQ_API sharq_status sharq_linear_swiglu(const sharq_prepared* x, const sharq_weight* w, void* H,
                                           float* h_amax, void* stream);

/* The preparation operator for a no-norm input whose producer has already
 * taken A = max |X| (sharq_linear_swiglu's h_amax): identical outputs to
 * sharq_prepare(X, NULL, ...) whenever *amax == max |X|, without the pass
 * that computes it.  The backbone's block maxima are those of X (the largest
 * entry of every group is always kept), so A is also the backbone's amax.
 * With SHARQ_RESIDUAL_SHARED the NVFP4 prepare is then a single pass without
 * a grid barrier.  amax: device fp32, 4-byte aligned, not NULL; a value
 * above max |X| is accepted (coarser scales), one below it saturates codes.
 * MXFP4 has no tensor scale and does not read it.  Buffers, workspace and
 * errors as sharq_prepare. */
SHARQ_API sharq_status sharq_prepare_amax(const void* X_bf16, const float* amax,
                                          const sharq_prepared* out, void* ws, size_t ws_bytes,
                                          void* stream);

/* Grouped (mixture-of-experts) form of sharq_linear (the pages evaluate the
 * method on a mixture-of-experts model; each expert is a SharQ linear):
 * dispatched row t (0 <= t < T) reads prepared row row_index[t] (row_index
 * NULL: row t, which needs T == x->M) and is multiplied by expert e's
 * weight when offsets[e] <= t < offsets[e+1]:
 *   Y[t,j] = G_w[e] * (G_b * S_b[t,j] + G_r * S_r[t,j]).
 * expert_offsets is a DEVICE int32 array [E+1], offsets[0] = 0, offsets[E]
 * = T, non-decreasing; row_index is a DEVICE int32 array [T] of rows < x->M.
 * w holds E stacked weights (see sharq_weight), 1 <= E <= 256.  The
 * activation tensor scales are those of the whole prepare call.  Y is [T, N]
 * in dispatch order.  The call first gathers each expert's rows into ws
 * (sharq_moe_workspace_bytes(T, E, K, fmt) bytes, caller-owned, content on
 * entry irrelevant), padded to 128-row groups, then runs one persistent
 * grouped GEMM over all experts. */
SHARQ_API size_t sharq_moe_workspace_bytes(int64_t T, int E, int K, int fmt);

SHARQ_API sharq_status sharq_moe_linear(const sharq_prepared* x, const int32_t* row_index,
                                        const int32_t* expert_offsets, int E, int64_t T,
                                        const sharq_weight* w, void* Y, int y_is_fp32,
                                        void* ws, size_t ws_bytes, void* stream);

/* Grouped form of sharq_linear_swiglu (SwiGLU experts, e.g. the pages'
 * mixture-of-experts model): every expert's gate+up weight is interleaved as
 * for sharq_linear_swiglu (w holds E stacked [2I, K] weights, w->N = 2I), and
 * row t of H is silu(gate) * up of dispatched row t through its own expert's
 * weight, with the column pairing of sharq_linear_swiglu; H is bf16 [T, I]
 * in dispatch order, the down projection's input in that order.
 * *h_amax = max |H| over all T rows (0 for T = 0).  Arguments, workspace
 * and errors as sharq_moe_linear; NULL h_amax is SHARQ_ERR_INVALID_ARG. */
SHARQ_API sharq_status sharq_moe_linear_swiglu(const sharq_prepared* x, const int32_t* row_index,
                                               const int32_t* expert_offsets, int E, int64_t T,
                                               const sharq_weight* w, void* H, float* h_amax,
                                               void* ws, size_t ws_bytes, void* stream);

/* Largest M that sharq_prepare_noalloc() accepts (its fixed scratch array
 * holds 64 bytes plus 4 bytes per row: 1 MiB + 64 bytes in all). */
#define SHARQ_NOALLOC_MAX_ROWS 262144

/* sharq_prepare without a workspace argument, for callers that cannot
 * allocate device memory where they run it: work enqueued during CUDA graph
 * stream capture, plugin or runtime callbacks whose host framework owns all
 * device memory, and serving loops that cannot pay for the device-wide
 * synchronisation of cudaMalloc/cudaFree.  The paper has no counterpart;
 * this is a deployment variant of the preparation operator above, with the
 * same arguments (minus ws) and bit-identical outputs.
 *   - Scratch lives in a fixed array inside the library (64 + 4 * M bytes,
 *     at most SHARQ_NOALLOC_MAX_ROWS rows).  Every GPU that loads the library
 *     holds that array until the process exits.
 *   - M > SHARQ_NOALLOC_MAX_ROWS returns SHARQ_ERR_INVALID_ARG.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls share the one array: calls that overlap on the GPU (other
 *     streams, other host threads) race on it.  Each call clears the part
 *     that must start at zero.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
SHARQ_API sharq_status sharq_prepare_noalloc(const void* X_bf16, const void* gamma_bf16, float eps,
                                             const sharq_prepared* out, void* stream);

/* Self-test of the failure path (for test suites): runs the library's own
 * bounded waits into their limit -- its grid barrier over a small grid whose
 * last block never arrives, then its mbarrier wait on a phase that nothing
 * completes.  Each wait gives up after limit_us microseconds (1000 ..
 * 1000000), records a timeout in the device status word and returns, so the
 * next sharq_last_device_status() reports SHARQ_ERR_TIMEOUT and the context
 * stays usable.  ws: device memory of at least 4 bytes (4-byte aligned),
 * overwritten.  Nothing faults or hangs. */
SHARQ_API sharq_status sharq_selftest_wait_timeout(void* ws, int64_t limit_us, void* stream);

/* Self-test of the failure path inside the preparation operator itself
 * (for test suites): runs sharq_prepare(X, NULL, ...) -- NVFP4, no norm, own
 * residual scale, so the launch has its two grid barriers -- with block 0
 * never arriving at them and every barrier wait limited to limit_us
 * microseconds (1000 .. 1000000).  The other blocks' waits give up, record
 * a timeout in the device status word and the kernel runs to its end, so
 * the next sharq_last_device_status() reports SHARQ_ERR_TIMEOUT; the
 * outputs of this call are unspecified and nothing faults or hangs.
 * Arguments as sharq_prepare; out->fmt must be SHARQ_NVFP4 and
 * out->residual_scale SHARQ_RESIDUAL_OWN, out->M >= 1. */
SHARQ_API sharq_status sharq_selftest_prepare_timeout(const void* X_bf16, const sharq_prepared* out,
                                                      void* ws, size_t ws_bytes, int64_t limit_us,
                                                      void* stream);

/* Synchronises `stream`, then reads and clears the device status word:
 * SHARQ_OK, SHARQ_ERR_TIMEOUT if a bounded device wait gave up since the
 * last call, or SHARQ_ERR_CUDA if the stream itself reports an error. */
SHARQ_API sharq_status sharq_last_device_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SHARQ_H */
