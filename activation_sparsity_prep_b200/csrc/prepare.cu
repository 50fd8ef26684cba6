// prepare.cu -- fused SharQ preparation operator and weight quantiser.
//
// SharQ paper, Abstract: one operator absorbs layer normalisation, the
// input-adaptive N:M mask, the FP4 backbone, and the residual taken against
// the *dequantised* backbone.  The NVFP4 tensor scales make this a chain of
// three tensor-wide dependencies:
//   phase 1  rinv per row (RMSNorm; LayerNorm: mean and rstd) and
//            A_b = max|y|                                 -> grid barrier
//   phase 2  mask, backbone codes/scales with G_b, residual r,
//            A_r = max|r|                                 -> grid barrier
//   phase 3  residual codes/scales with G_r
// One persistent cooperative launch runs the three phases.  In phase 1 each
// warp owns whole rows, lane l reading the 16-byte chunks l, l+32, ... of a
// row, which is also the fixed fp32 reduction order of the RMS sum; without
// a norm, phase 1 is a plain maximum over the whole tensor, spread over every
// lane.  Phases 2 and 3 spread (row, 256-element segment) items over every
// warp.  MXFP4 has no tensor scale, so its backbone and residual are produced
// in one pass (after the RMS barrier when there is a norm).  When the
// producer of X has already taken A_b = max |X| (a no-norm input, e.g. the
// SwiGLU epilogue of the gate+up linear), phase 1 and its barrier are
// skipped: with the shared residual scale the whole prepare is then one
// barrier-free pass.
//
// Every floating-point step is one correctly rounded fp32 operation
// (__fmul_rn / __fadd_rn / __fdiv_rn / __fsqrt_rn, no contraction), so the
// codes and scales are bit-identical to a plain sequential CPU evaluation.
#include "common.cuh"
#include "sharq_internal.h"

#include <cuda_fp16.h>

#include <atomic>

namespace sharq {

unsigned take_status_prepare() { return take_tu_status(); }

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

struct PrepArgs {
    const uint16_t* X;       // [M, K] bf16
    const uint16_t* gamma;   // [K] bf16 or null
    const uint16_t* beta;    // [K] bf16 or null (LayerNorm bias)
    float eps;
    int64_t M;
    int K;
    int n;
    uint8_t* bb_codes;
    uint8_t* bb_scales;
    float* bb_tscale;
    uint8_t* rs_codes;       // null in weight mode
    uint8_t* rs_scales;
    float* rs_tscale;
    uint8_t* mask;           // optional
    uint32_t* ws;            // [0] amax_b bits, [1] amax_r bits, [2] barrier, then rinv[M], mu[M]
    const float* amax_in;    // GIVEN: A_b = max |X| from the producer
};

__device__ __forceinline__ float* ws_rinv(uint32_t* ws) {
    return reinterpret_cast<float*>(ws + 16);
}

// Byte offset of scale (row, s) in the MMA-ready atom layout.
__device__ __forceinline__ int64_t sf_off(int64_t row, int s, int nsf) {
    return ((row >> 7) * (int64_t)(nsf >> 2) + (s >> 2)) * 512 + (row & 31) * 16 +
           ((row >> 5) & 3) * 4 + (s & 3);
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float x[8]) {
    x[0] = __uint_as_float(v.x << 16); x[1] = __uint_as_float(v.x & 0xFFFF0000u);
    x[2] = __uint_as_float(v.y << 16); x[3] = __uint_as_float(v.y & 0xFFFF0000u);
    x[4] = __uint_as_float(v.z << 16); x[5] = __uint_as_float(v.z & 0xFFFF0000u);
    x[6] = __uint_as_float(v.w << 16); x[7] = __uint_as_float(v.w & 0xFFFF0000u);
}

// y = fl(fl(x * rinv) * gamma) for one chunk, or y = x without gamma.
template <bool HAS_GAMMA>
__device__ __forceinline__ void load_y(const PrepArgs& a, int64_t row, int c, float rinv,
                                       float y[8]) {
    uint4 v = ld_nc_v4(a.X + row * a.K + (int64_t)c * 8);
    unpack_bf16x8(v, y);
    if (HAS_GAMMA) {
        float g[8];
        unpack_bf16x8(ld_nc_v4(a.gamma + (int64_t)c * 8), g);
#pragma unroll
        for (int t = 0; t < 8; ++t) y[t] = __fmul_rn(__fmul_rn(y[t], rinv), g[t]);
    }
}

// Top-n of every aligned group of MG inside the 8-element chunk; ties go to
// the lower index.  Bit t set = element t kept.
template <int MG>
__device__ __forceinline__ uint32_t topn_bits(const float y[8], int n) {
    uint32_t bits = 0;
#pragma unroll
    for (int g = 0; g < 8; g += MG) {
#pragma unroll
        for (int i = 0; i < MG; ++i) {
            float fi = fabsf(y[g + i]);
            int rank = 0;
#pragma unroll
            for (int j = 0; j < MG; ++j) {
                if (j == i) continue;
                float fj = fabsf(y[g + j]);
                rank += (j < i) ? (fj >= fi) : (fj > fi);
            }
            bits |= (uint32_t)(rank < n) << (g + i);
        }
    }
    return bits;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ float amax8(const float v[8]) {
    float m0 = max3(fabsf(v[0]), fabsf(v[1]), fabsf(v[2]));
    float m1 = max3(fabsf(v[3]), fabsf(v[4]), fabsf(v[5]));
    return max3(m0, m1, fmaxf(fabsf(v[6]), fabsf(v[7])));
}

// 2^p as fp32 for -127 <= p <= 127 (2^-127 is subnormal).
__device__ __forceinline__ float pow2f(int p) {
    return p >= -126 ? __uint_as_float((uint32_t)(p + 127) << 23) : __uint_as_float(0x00400000u);
}

// MX shared-scale code: floor(log2 amax) - 2 + 127 clamped to [0, 254]; 0
// for zero.  floor(log2) of a normal float is its biased exponent - 127 and
// every subnormal clamps to 0.
__device__ __forceinline__ uint32_t mx_code(float amax) {
    int ef = (int)((__float_as_uint(amax) >> 23) & 0xFF);
    return (uint32_t)max(ef - 2, 0);
}

// Dequantised values of 8 packed codes: fl(fl(val * s) * g).  val * s is
// exact in fp32; g is the decode tensor scale (1 for MXFP4).
__device__ __forceinline__ void dequant8(uint32_t codes, float s, float g, float d[8]) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        uint32_t h2 = cvt_e2m1x2_to_f16x2((codes >> (8 * p)) & 0xFF);
        float2 f = __half22float2(*reinterpret_cast<__half2*>(&h2));
        d[2 * p] = __fmul_rn(__fmul_rn(f.x, s), g);
        d[2 * p + 1] = __fmul_rn(__fmul_rn(f.y, s), g);
    }
}

// Bounded grid-wide barrier for a cooperative launch (all blocks resident).
__device__ __forceinline__ void grid_barrier(uint32_t* counter, unsigned target) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(counter, 1u);
        unsigned long long t0 = globaltimer();
        while (ld_acquire_gpu(counter) < target) {
            if (globaltimer() - t0 > kWaitLimitNs) {
                record_status(kStatusGridTimeout);
                break;
            }
            __nanosleep(64);
        }
        __threadfence();
    }
    __syncthreads();
}

__device__ __forceinline__ void block_amax_to_global(float v, uint32_t* dst, float* red) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) red[w] = v;
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = 0.0f;
        for (int i = 0; i < kWarps; ++i) m = fmaxf(m, red[i]);
        if (m > 0.0f) atomicMax(dst, __float_as_uint(m));   // non-negative floats order as uints
    }
    __syncthreads();
}

// NVFP4 tensor-scale chain: G_enc = 2688 / A, G_dec = A / 2688 (1 when A = 0),
// K1 = G_enc / 6; inv[e] = G_enc / val(e) (0 for e = 0).
struct NvScale {
    float genc, gdec, k1;
};

__device__ __forceinline__ NvScale nv_scale(float A) {
    NvScale s;
    s.genc = 1.0f; s.gdec = 1.0f;
    if (A != 0.0f) { s.genc = __fdiv_rn(2688.0f, A); s.gdec = __fdiv_rn(A, 2688.0f); }
    s.k1 = __fdiv_rn(s.genc, 6.0f);
    return s;
}

__device__ __forceinline__ void fill_inv_table(float* tab, float genc) {
    for (int e = threadIdx.x; e < 128; e += blockDim.x)
        tab[e] = (e == 0) ? 0.0f : __fdiv_rn(genc, e4m3_to_f32((uint32_t)e));
    __syncthreads();
}

// ------------------------------------------------------------------------
// Phases 2 and 3 give each lane one whole scale block (16 elements for
// NVFP4, 32 for MXFP4) of the flattened [M, K/BS] block array.  A warp's 32
// blocks are 32*BS consecutive elements of X, so its loads stay coalesced;
// the block maximum needs no shuffle, and a lane stores its codes with one
// 8- or 16-byte store and its scale with one byte store.  Neither phase has
// an ordering constraint (block-local arithmetic plus an exact maximum).
// ------------------------------------------------------------------------

// Walk the blocks b = start, start + stride, ... as (row, column) pairs
// without a division per step.
struct BlockCursor {
    int64_t row;
    int cb;
    int dr, dc, nbr;
    __device__ __forceinline__ void init(int64_t start, int64_t stride, int nb_row) {
        nbr = nb_row;
        row = start / nb_row;
        cb = (int)(start - row * nb_row);
        dr = (int)(stride / nb_row);
        dc = (int)(stride - (int64_t)dr * nb_row);
    }
    __device__ __forceinline__ void next() {
        cb += dc;
        row += dr;
        if (cb >= nbr) { cb -= nbr; ++row; }
    }
};

// Element i of a group of four is kept when it beats at least two of the
// other three (a beats b: |a| > |b|, or equal and a has the lower index).
__device__ __forceinline__ uint32_t keep_2of4(const float* y) {
    const float a0 = fabsf(y[0]), a1 = fabsf(y[1]), a2 = fabsf(y[2]), a3 = fabsf(y[3]);
    const bool b01 = a0 >= a1, b02 = a0 >= a2, b03 = a0 >= a3;
    const bool b12 = a1 >= a2, b13 = a1 >= a3, b23 = a2 >= a3;
    const bool k0 = (b01 & b02) | (b01 & b03) | (b02 & b03);
    const bool k1 = (!b01 & b12) | (!b01 & b13) | (b12 & b13);
    const bool k2 = (!b02 & !b12) | (!b02 & b23) | (!b12 & b23);
    const bool k3 = (!b03 & !b13) | (!b03 & !b23) | (!b13 & !b23);
    return (uint32_t)k0 | ((uint32_t)k1 << 1) | ((uint32_t)k2 << 2) | ((uint32_t)k3 << 3);
}

// Keep bits of E consecutive elements (E a multiple of 8).
template <int E, int MG, bool NM24>
__device__ __forceinline__ uint32_t keep_bits(const float* y, int n) {
    uint32_t k = 0;
#pragma unroll
    for (int g = 0; g < E; g += (NM24 ? 4 : 8)) {
        if (NM24) k |= keep_2of4(y + g) << g;
        else      k |= topn_bits<MG>(y + g, n) << g;
    }
    return k;
}

template <int E>
__device__ __forceinline__ float amaxE(const float* v) {
    float m = amax8(v);
#pragma unroll
    for (int g = 8; g < E; g += 8) m = fmaxf(m, amax8(v + g));
    return m;
}

template <int FMT, bool HAS_GAMMA, bool LN>
struct LaneBlock {
    static constexpr int E = FMT == 0 ? 16 : 32;   // elements per lane = one scale block
    static constexpr int NV = E / 8;                // 16-byte chunks
    uint4 x[NV];
    uint4 g[NV];
    uint4 b[LN ? NV : 1];
    float rinv, mu;

    __device__ __forceinline__ void load(const PrepArgs& a, int64_t row, int cb, const float* rinv_ws) {
        const uint16_t* xp = a.X + row * a.K + (int64_t)cb * E;
#pragma unroll
        for (int v = 0; v < NV; ++v) x[v] = ld_nc_v4(xp + 8 * v);
        if (HAS_GAMMA) {
#pragma unroll
            for (int v = 0; v < NV; ++v) g[v] = ld_nc_v4(a.gamma + (int64_t)cb * E + 8 * v);
            rinv = rinv_ws[row];
        }
        if (LN) {
            mu = rinv_ws[a.M + row];          // the LayerNorm means follow the M reciprocals
            if (a.beta) {
#pragma unroll
                for (int v = 0; v < NV; ++v) b[v] = ld_nc_v4(a.beta + (int64_t)cb * E + 8 * v);
            }
        }
    }

    // RMSNorm: fl(fl(x * rinv) * g).  LayerNorm: fl(fl(fl(x - mu) * rstd) * g),
    // then + beta when there is a bias.
    __device__ __forceinline__ void y(float* out, bool has_beta) const {
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            unpack_bf16x8(x[v], out + 8 * v);
            if (HAS_GAMMA) {
                float gg[8];
                unpack_bf16x8(g[v], gg);
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    const float xv = LN ? __fsub_rn(out[8 * v + t], mu) : out[8 * v + t];
                    out[8 * v + t] = __fmul_rn(__fmul_rn(xv, rinv), gg[t]);
                }
                if (LN && has_beta) {
                    float bb[8];
                    unpack_bf16x8(b[v], bb);
#pragma unroll
                    for (int t = 0; t < 8; ++t) out[8 * v + t] = __fadd_rn(out[8 * v + t], bb[t]);
                }
            }
        }
    }
};

// ------------------------------------------------------------------------
// The kernel.  FMT: 0 NVFP4, 1 MXFP4.  WEIGHT: quantise the whole tensor
// once (keep-all, no norm, no residual).  NM24: the 2-of-4 mask.  RS: the
// residual takes the backbone's tensor scale (NVFP4), so it is finished in
// phase 2 with the backbone's reciprocal table and phase 3 does not exist.
// GIVEN: no norm, A_b read from a.amax_in, no phase 1.
// ------------------------------------------------------------------------
template <int FMT, bool HAS_GAMMA, int MG, bool WEIGHT, bool NM24, bool RS, bool LN, bool GIVEN>
__global__ void __launch_bounds__(kThreads, 2)
prepare_kernel(PrepArgs a) {
    __shared__ float s_inv[128];
    __shared__ float s_red[kWarps];
    using LB = LaneBlock<FMT, HAS_GAMMA, LN>;
    static_assert(!LN || HAS_GAMMA, "LayerNorm takes gamma");
    static_assert(!GIVEN || (FMT == 0 && !HAS_GAMMA && !WEIGHT), "a given amax: NVFP4, no norm");
    const bool has_beta = LN && a.beta != nullptr;
    constexpr int E = LB::E;

    const int lane = threadIdx.x & 31;
    const int64_t gwarp = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * kWarps;
    const int K = a.K;
    const int nchunk = K / 8;
    constexpr int BS = (FMT == 0) ? 16 : 32;
    const int nsf = K / BS;
    const int64_t M = a.M;
    const int64_t Mpad = (M + 127) / 128 * 128;
    float* rinv_ws = ws_rinv(a.ws);

    // ---------------- phase 1: rinv per row, A_b = max |y| ----------------
    float amax = 0.0f;
    if (FMT == 0 && !HAS_GAMMA && !GIVEN) {
        // y = x, and A_b = max |x| needs no row structure: lane i of the
        // grid reads chunks i, i + L, ..., i + 15L (L = lanes in the grid),
        // sixteen loads in flight, then the next 16L chunks.  The magnitude
        // order of bf16 values is the integer order of their bits with the
        // sign cleared.
        const int64_t nch = M * (int64_t)nchunk;
        const int64_t L = nwarps * 32;
        uint32_t m2 = 0;
        for (int64_t c0 = gwarp * 32 + lane; c0 < nch; c0 += 16 * L) {
            uint4 v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u)
                if (c0 + u * L < nch) v[u] = ld_nc_v4(a.X + (c0 + u * L) * 8);
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                if (c0 + u * L < nch) {
                    m2 = __vmaxu2(m2, v[u].x & 0x7FFF7FFFu);
                    m2 = __vmaxu2(m2, v[u].y & 0x7FFF7FFFu);
                    m2 = __vmaxu2(m2, v[u].z & 0x7FFF7FFFu);
                    m2 = __vmaxu2(m2, v[u].w & 0x7FFF7FFFu);
                }
            }
        }
        amax = fmaxf(__uint_as_float(m2 << 16), __uint_as_float(m2 & 0xFFFF0000u));
    } else if (HAS_GAMMA) {
        // One warp per row.  rinv: lane l adds f(x) over chunks l, l+32, ...
        // element by element in k order, then the xor butterfly -- the fixed
        // reduction order.  Then (NVFP4) the row's max |y|.  Eight chunk
        // loads in flight per lane (four per operand for LayerNorm's max).
        for (int64_t row = gwarp; row < M; row += nwarps) {
            const uint16_t* xr = a.X + row * K;
            auto row_sum = [&](auto f) {
                float acc = 0.0f;
                for (int c0 = lane; c0 < nchunk; c0 += 256) {
                    uint4 v[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        if (c0 + 32 * u < nchunk) v[u] = ld_nc_v4(xr + (int64_t)(c0 + 32 * u) * 8);
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        if (c0 + 32 * u < nchunk) {
                            float x[8];
                            unpack_bf16x8(v[u], x);
#pragma unroll
                            for (int t = 0; t < 8; ++t) acc = __fadd_rn(acc, f(x[t]));
                        }
                    }
                }
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1)
                    acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, o));
                return acc;
            };
            float rinv, mu = 0.0f;
            if (LN) {
                // LayerNorm: mean, then the centred squares (two passes)
                mu = __fdiv_rn(row_sum([](float x) { return x; }), (float)K);
                const float var = __fdiv_rn(row_sum([mu](float x) {
                    const float d = __fsub_rn(x, mu);
                    return __fmul_rn(d, d);
                }), (float)K);
                rinv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(var, a.eps)));
                if (lane == 0) { rinv_ws[row] = rinv; rinv_ws[M + row] = mu; }
            } else {
                const float ms = __fdiv_rn(row_sum([](float x) { return __fmul_rn(x, x); }), (float)K);
                rinv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, a.eps)));
                if (lane == 0) rinv_ws[row] = rinv;
            }
            if (FMT == 0) {
                constexpr int D = LN ? 4 : 8;   // LayerNorm also streams beta
                for (int c0 = lane; c0 < nchunk; c0 += 32 * D) {
                    uint4 v[D], g[D], bt[LN ? D : 1];
#pragma unroll
                    for (int u = 0; u < D; ++u) {
                        if (c0 + 32 * u < nchunk) {
                            v[u] = ld_nc_v4(xr + (int64_t)(c0 + 32 * u) * 8);
                            g[u] = ld_nc_v4(a.gamma + (int64_t)(c0 + 32 * u) * 8);
                            if (LN && has_beta) bt[u] = ld_nc_v4(a.beta + (int64_t)(c0 + 32 * u) * 8);
                        }
                    }
#pragma unroll
                    for (int u = 0; u < D; ++u) {
                        if (c0 + 32 * u < nchunk) {
                            float y[8], gg[8];
                            unpack_bf16x8(v[u], y);
                            unpack_bf16x8(g[u], gg);
#pragma unroll
                            for (int t = 0; t < 8; ++t) {
                                const float xv = LN ? __fsub_rn(y[t], mu) : y[t];
                                y[t] = __fmul_rn(__fmul_rn(xv, rinv), gg[t]);
                            }
                            if (LN && has_beta) {
                                float bb[8];
                                unpack_bf16x8(bt[u], bb);
#pragma unroll
                                for (int t = 0; t < 8; ++t) y[t] = __fadd_rn(y[t], bb[t]);
                            }
                            amax = fmaxf(amax, amax8(y));
                        }
                    }
                }
            }
        }
    }

    if (FMT == 0 && !GIVEN) {
        block_amax_to_global(amax, &a.ws[0], s_red);
        grid_barrier(&a.ws[2], gridDim.x);
    } else if (HAS_GAMMA) {
        grid_barrier(&a.ws[2], gridDim.x);   // rinv of every row visible to every warp
    }

    // ------- phase 2: mask, backbone, residual amax (and MXFP4 residual) -------
    NvScale sb{1.0f, 1.0f, 1.0f};
    if (FMT == 0) {
        sb = nv_scale(GIVEN ? *a.amax_in : __uint_as_float(ld_acquire_gpu(&a.ws[0])));
        fill_inv_table(s_inv, sb.genc);
        if (blockIdx.x == 0 && threadIdx.x == 0) {
            *a.bb_tscale = sb.gdec;
            if (RS) *a.rs_tscale = sb.gdec;
        }
    } else {
        if (blockIdx.x == 0 && threadIdx.x == 0) {
            *a.bb_tscale = 1.0f;
            if (!WEIGHT) *a.rs_tscale = 1.0f;
        }
    }

    // padding rows of the scale atoms carry zero scales
    {
        const int words = nsf / 4;
        const int64_t npad = (Mpad - M) * words;
        for (int64_t i = gwarp * 32 + lane; i < npad; i += nwarps * 32) {
            const int64_t row = M + i / words;
            const int s4 = (int)(i % words);
            *reinterpret_cast<uint32_t*>(a.bb_scales + sf_off(row, s4 * 4, nsf)) = 0u;
            if (!WEIGHT) *reinterpret_cast<uint32_t*>(a.rs_scales + sf_off(row, s4 * 4, nsf)) = 0u;
        }
    }

    const int nb_row = K / E;
    float ramax = 0.0f;
    {
        BlockCursor cur;
        cur.init(gwarp * 32 + lane, nwarps * 32, nb_row);
        LB lb;
        if (cur.row < M) lb.load(a, cur.row, cur.cb, rinv_ws);
        while (cur.row < M) {
            BlockCursor nxt = cur;
            nxt.next();
            LB ln;
            if (nxt.row < M) ln.load(a, nxt.row, nxt.cb, rinv_ws);   // prefetch

            const int64_t row = cur.row;
            const int cb = cur.cb;
            float y[E];
            lb.y(y, has_beta);
            // the backbone's block max is the block max of y: the largest
            // entry of every group is always kept
            const float bm = amaxE<E>(y);
            uint32_t ecode;
            float inv, sdec;
            if (FMT == 0) {
                ecode = cvt_e4m3(__fmul_rn(bm, sb.k1));
                inv = s_inv[ecode];
                sdec = e4m3_to_f32(ecode);
            } else {
                ecode = mx_code(bm);
                inv = pow2f(127 - (int)ecode);
                sdec = pow2f((int)ecode - 127);
            }
            const uint32_t keep = WEIGHT ? 0xFFFFFFFFu : keep_bits<E, MG, NM24>(y, a.n);
            uint32_t codes[E / 8];
#pragma unroll
            for (int v = 0; v < E / 8; ++v) {
                float t8[8];
#pragma unroll
                for (int t = 0; t < 8; ++t)
                    t8[t] = ((keep >> (8 * v + t)) & 1u) ? __fmul_rn(y[8 * v + t], inv) : 0.0f;
                codes[v] = cvt_e2m1x8(t8);
            }
            uint8_t* cp = a.bb_codes + row * (K / 2) + (int64_t)cb * (E / 2);
            if (E == 16) *reinterpret_cast<uint2*>(cp) = make_uint2(codes[0], codes[1]);
            else         *reinterpret_cast<uint4*>(cp) = make_uint4(codes[0], codes[1], codes[2], codes[3]);
            a.bb_scales[sf_off(row, cb, nsf)] = (uint8_t)ecode;
            if (!WEIGHT && a.mask) {
                uint8_t* mp = a.mask + row * (K / 8) + (int64_t)cb * (E / 8);
                if (E == 16) *reinterpret_cast<uint16_t*>(mp) = (uint16_t)keep;
                else         *reinterpret_cast<uint32_t*>(mp) = keep;
            }

            if (!WEIGHT) {
                // residual r = y - dequant(backbone), in place in y
#pragma unroll
                for (int v = 0; v < E / 8; ++v) {
                    float d[8];
                    dequant8(codes[v], sdec, sb.gdec, d);
#pragma unroll
                    for (int t = 0; t < 8; ++t) y[8 * v + t] = __fsub_rn(y[8 * v + t], d[t]);
                }
                if (FMT == 0 && RS) {
                    // the residual's block scale against the backbone's G
                    const uint32_t er = cvt_e4m3(__fmul_rn(amaxE<E>(y), sb.k1));
                    const float inv_r = s_inv[er];
                    uint32_t rc[E / 8];
#pragma unroll
                    for (int v = 0; v < E / 8; ++v) {
                        float t8[8];
#pragma unroll
                        for (int t = 0; t < 8; ++t) t8[t] = __fmul_rn(y[8 * v + t], inv_r);
                        rc[v] = cvt_e2m1x8(t8);
                    }
                    *reinterpret_cast<uint2*>(a.rs_codes + row * (K / 2) + (int64_t)cb * 8) = make_uint2(rc[0], rc[1]);
                    a.rs_scales[sf_off(row, cb, nsf)] = (uint8_t)er;
                } else if (FMT == 0) {
                    ramax = fmaxf(ramax, amaxE<E>(y));
                } else {
                    // MXFP4: the residual needs no tensor-wide scale; finish it here.
                    const uint32_t rcode = mx_code(amaxE<E>(y));
                    const float rs = pow2f(127 - (int)rcode);
                    uint32_t rc[E / 8];
#pragma unroll
                    for (int v = 0; v < E / 8; ++v) {
                        float t8[8];
#pragma unroll
                        for (int t = 0; t < 8; ++t) t8[t] = __fmul_rn(y[8 * v + t], rs);
                        rc[v] = cvt_e2m1x8(t8);
                    }
                    *reinterpret_cast<uint4*>(a.rs_codes + row * (K / 2) + (int64_t)cb * (E / 2)) =
                        make_uint4(rc[0], rc[1], rc[2], rc[3]);
                    a.rs_scales[sf_off(row, cb, nsf)] = (uint8_t)rcode;
                }
            }
            cur = nxt;
            lb = ln;
        }
    }
    if (FMT == 1 || WEIGHT || RS) return;

    block_amax_to_global(ramax, &a.ws[1], s_red);
    grid_barrier(&a.ws[2], (GIVEN ? 1u : 2u) * gridDim.x);   // counts on from phase 1's

    // ---------------- phase 3: residual codes with G_r ----------------
    NvScale sr = nv_scale(__uint_as_float(ld_acquire_gpu(&a.ws[1])));
    __syncthreads();                       // everyone done reading the backbone table
    fill_inv_table(s_inv, sr.genc);
    if (blockIdx.x == 0 && threadIdx.x == 0) *a.rs_tscale = sr.gdec;
    {
        BlockCursor cur;
        cur.init(gwarp * 32 + lane, nwarps * 32, nb_row);
        LB lb;
        uint2 bc = make_uint2(0, 0);
        uint32_t bs = 0;
        if (cur.row < M) {
            lb.load(a, cur.row, cur.cb, rinv_ws);
            bc = *reinterpret_cast<const uint2*>(a.bb_codes + cur.row * (K / 2) + (int64_t)cur.cb * 8);
            bs = a.bb_scales[sf_off(cur.row, cur.cb, nsf)];
        }
        while (cur.row < M) {
            BlockCursor nxt = cur;
            nxt.next();
            LB ln;
            uint2 nbc = make_uint2(0, 0);
            uint32_t nbs = 0;
            if (nxt.row < M) {
                ln.load(a, nxt.row, nxt.cb, rinv_ws);
                nbc = *reinterpret_cast<const uint2*>(a.bb_codes + nxt.row * (K / 2) + (int64_t)nxt.cb * 8);
                nbs = a.bb_scales[sf_off(nxt.row, nxt.cb, nsf)];
            }
            const int64_t row = cur.row;
            const int cb = cur.cb;
            float y[16];
            lb.y(y, has_beta);
            const float sdec = e4m3_to_f32(bs);
            float d[8];
            dequant8(bc.x, sdec, sb.gdec, d);
#pragma unroll
            for (int t = 0; t < 8; ++t) y[t] = __fsub_rn(y[t], d[t]);
            dequant8(bc.y, sdec, sb.gdec, d);
#pragma unroll
            for (int t = 0; t < 8; ++t) y[8 + t] = __fsub_rn(y[8 + t], d[t]);   // y := r
            const uint32_t er = cvt_e4m3(__fmul_rn(amaxE<16>(y), sr.k1));
            const float inv = s_inv[er];
            float t8[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) t8[t] = __fmul_rn(y[t], inv);
            const uint32_t c0 = cvt_e2m1x8(t8);
#pragma unroll
            for (int t = 0; t < 8; ++t) t8[t] = __fmul_rn(y[8 + t], inv);
            const uint32_t c1 = cvt_e2m1x8(t8);
            *reinterpret_cast<uint2*>(a.rs_codes + row * (K / 2) + (int64_t)cb * 8) = make_uint2(c0, c1);
            a.rs_scales[sf_off(row, cb, nsf)] = (uint8_t)er;
            cur = nxt;
            lb = ln;
            bc = nbc;
            bs = nbs;
        }
    }
}

template <int FMT, bool HAS_GAMMA, int MG, bool WEIGHT, bool NM24, bool RS = false, bool LN = false,
          bool GIVEN = false>
cudaError_t launch_one(const PrepArgs& a, cudaStream_t s, int max_blocks) {
    auto kfn = prepare_kernel<FMT, HAS_GAMMA, MG, WEIGHT, NM24, RS, LN, GIVEN>;
    // same for every device of one architecture; a repeated query is harmless
    static std::atomic<int> cached{0};
    int blocks_per_sm = cached.load(std::memory_order_relaxed);
    if (blocks_per_sm == 0) {
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks_per_sm, kfn, kThreads, 0);
        if (e != cudaSuccess) return e;
        cached.store(blocks_per_sm, std::memory_order_relaxed);
    }
    // Enough warps for one row each in phase 1 and about four 32-block
    // groups each in phases 2 and 3, capped at what is resident.
    int64_t Mpad = (a.M + 127) / 128 * 128;
    int64_t groups = a.M * (int64_t)(a.K / (FMT == 0 ? 16 : 32)) / 32;
    int64_t want = std::max((Mpad + kWarps - 1) / kWarps, (groups + 4 * kWarps - 1) / (4 * kWarps));
    int64_t cap = (int64_t)blocks_per_sm * max_blocks;
    int grid = (int)std::max<int64_t>(1, std::min<int64_t>(want, cap));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;   // grid barriers: all blocks co-resident
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    // any grid barrier needs co-residency: after phase 1 (a norm, or an NVFP4
    // amax taken here) or before phase 3 (NVFP4 with its own residual scale)
    const bool barrier = HAS_GAMMA || (FMT == 0 && !GIVEN) || (FMT == 0 && !WEIGHT && !RS);
    cfg.numAttrs = barrier ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kfn, a);
}

template <int FMT, bool HAS_GAMMA, bool WEIGHT, bool RS = false, bool LN = false, bool GIVEN = false>
cudaError_t launch_m(const PrepArgs& a, int m, cudaStream_t s, int sms) {
    switch (m) {
        case 2: return launch_one<FMT, HAS_GAMMA, 2, WEIGHT, false, RS, LN, GIVEN>(a, s, sms);
        case 4: return a.n == 2 ? launch_one<FMT, HAS_GAMMA, 4, WEIGHT, true, RS, LN, GIVEN>(a, s, sms)
                                : launch_one<FMT, HAS_GAMMA, 4, WEIGHT, false, RS, LN, GIVEN>(a, s, sms);
        default: return launch_one<FMT, HAS_GAMMA, 8, WEIGHT, false, RS, LN, GIVEN>(a, s, sms);
    }
}

}  // namespace

size_t prepare_ws_bytes(int64_t M) {
    size_t b = 64 + (size_t)(M > 0 ? M : 0) * 8;
    return (b + 255) / 256 * 256;
}

cudaError_t launch_prepare(const PrepareLaunch& p, cudaStream_t s, int sms) {
    PrepArgs a;
    a.X = static_cast<const uint16_t*>(p.X);
    a.gamma = static_cast<const uint16_t*>(p.gamma);
    a.beta = static_cast<const uint16_t*>(p.beta);
    a.eps = p.eps;
    a.M = p.M;
    a.K = p.K;
    a.n = p.n;
    a.bb_codes = static_cast<uint8_t*>(p.bb_codes);
    a.bb_scales = static_cast<uint8_t*>(p.bb_scales);
    a.bb_tscale = p.bb_tscale;
    a.rs_codes = static_cast<uint8_t*>(p.rs_codes);
    a.rs_scales = static_cast<uint8_t*>(p.rs_scales);
    a.rs_tscale = p.rs_tscale;
    a.mask = static_cast<uint8_t*>(p.mask);
    a.ws = static_cast<uint32_t*>(p.ws);
    a.amax_in = p.amax;
    const bool g = p.gamma != nullptr;
    // the workspace header (maxima, barrier counter) starts at zero, unless
    // the launch uses none of it: MXFP4 without a norm, or a given amax with
    // the shared residual scale (one pass, no barrier)
    const bool no_ws = (p.fmt == 1 && !g) || (p.fmt == 0 && p.amax && p.residual_shared && !p.weight);
    if (!no_ws) {
        cudaError_t e = cudaMemsetAsync(p.ws, 0, 64, s);
        if (e != cudaSuccess) return e;
    }
    if (p.weight) {
        return p.fmt == 0 ? launch_one<0, false, 8, true, false>(a, s, sms)
                          : launch_one<1, false, 8, true, false>(a, s, sms);
    }
    if (p.layernorm) {
        if (p.fmt == 1) return launch_m<1, true, false, false, true>(a, p.m, s, sms);
        return p.residual_shared ? launch_m<0, true, false, true, true>(a, p.m, s, sms)
                                 : launch_m<0, true, false, false, true>(a, p.m, s, sms);
    }
    if (p.fmt == 0 && p.amax) {   // no norm, A_b from the producer
        return p.residual_shared ? launch_m<0, false, false, true, false, true>(a, p.m, s, sms)
                                 : launch_m<0, false, false, false, false, true>(a, p.m, s, sms);
    }
    if (p.fmt == 0 && p.residual_shared)
        return g ? launch_m<0, true, false, true>(a, p.m, s, sms) : launch_m<0, false, false, true>(a, p.m, s, sms);
    if (p.fmt == 0) return g ? launch_m<0, true, false>(a, p.m, s, sms) : launch_m<0, false, false>(a, p.m, s, sms);
    return g ? launch_m<1, true, false>(a, p.m, s, sms) : launch_m<1, false, false>(a, p.m, s, sms);
}

}  // namespace sharq
