// prepare.cu -- fused SharQ preparation operator and weight quantiser.
//
// SharQ paper, Abstract: one operator absorbs layer normalisation, the
// input-adaptive N:M mask, the FP4 backbone, and the residual taken against
// the *dequantised* backbone.  The NVFP4 tensor scales make this a chain of
// three tensor-wide dependencies:
//   phase 1  rinv per row (RMSNorm) and A_b = max|y|      -> grid barrier
//   phase 2  mask, backbone codes/scales with G_b, residual r,
//            A_r = max|r|                                 -> grid barrier
//   phase 3  residual codes/scales with G_r
// One persistent cooperative launch runs the three phases; each warp owns
// whole rows, lane l reading the 16-byte chunks l, l+32, ... of a row, which
// is also the fixed fp32 reduction order of the RMS sum.  MXFP4 has no
// tensor scale, so its backbone and residual are produced in one pass with
// no barrier.
//
// Every floating-point step is one correctly rounded fp32 operation
// (__fmul_rn / __fadd_rn / __fdiv_rn / __fsqrt_rn, no contraction), so the
// codes and scales are bit-identical to a plain sequential CPU evaluation.
#include "common.cuh"
#include "sharq_internal.h"

#include <cuda_fp16.h>

namespace sharq {

unsigned take_status_prepare() { return take_tu_status(); }

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

struct PrepArgs {
    const uint16_t* X;       // [M, K] bf16
    const uint16_t* gamma;   // [K] bf16 or null
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
    uint32_t* ws;            // [0] amax_b bits, [1] amax_r bits, [2] barrier, then rinv[M]
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

__device__ __forceinline__ float amax8(const float v[8]) {
    float m = 0.0f;
#pragma unroll
    for (int t = 0; t < 8; ++t) m = fmaxf(m, fabsf(v[t]));
    return m;
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

// Gather 4 consecutive block-scale bytes into one word at lane `lead` of each
// group of `stride*4` lanes: word = v(lead) | v(lead+stride)<<8 | ...
__device__ __forceinline__ uint32_t gather4(uint32_t v, int lane, int stride) {
    int lead = lane & ~(4 * stride - 1);
    uint32_t w = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) w |= __shfl_sync(0xffffffffu, v, lead + q * stride) << (8 * q);
    return w;
}

// ------------------------------------------------------------------------
// The kernel.  FMT: 0 NVFP4, 1 MXFP4.  WEIGHT: quantise the whole tensor
// once (keep-all, no norm, no residual).
// ------------------------------------------------------------------------
template <int FMT, bool HAS_GAMMA, int MG, bool WEIGHT>
__global__ void __launch_bounds__(kThreads)
prepare_kernel(PrepArgs a) {
    __shared__ float s_inv[128];
    __shared__ float s_red[kWarps];

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
    if (HAS_GAMMA || FMT == 0) {
        for (int64_t row = gwarp; row < M; row += nwarps) {
            float rinv = 1.0f;
            if (HAS_GAMMA) {
                float acc = 0.0f;
                for (int c = lane; c < nchunk; c += 32) {
                    float x[8];
                    unpack_bf16x8(ld_nc_v4(a.X + row * K + (int64_t)c * 8), x);
#pragma unroll
                    for (int t = 0; t < 8; ++t) acc = __fadd_rn(acc, __fmul_rn(x[t], x[t]));
                }
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1)
                    acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, o));
                float ms = __fdiv_rn(acc, (float)K);
                rinv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, a.eps)));
                if (lane == 0) rinv_ws[row] = rinv;
            }
            if (FMT == 0) {
                for (int c = lane; c < nchunk; c += 32) {
                    float y[8];
                    load_y<HAS_GAMMA>(a, row, c, rinv, y);
                    amax = fmaxf(amax, amax8(y));
                }
            }
        }
    }

    if (FMT == 0) {
        block_amax_to_global(amax, &a.ws[0], s_red);
        grid_barrier(&a.ws[2], gridDim.x);
    } else if (HAS_GAMMA) {
        __syncthreads();
        if (threadIdx.x == 0) __threadfence();
    }

    // ------- phase 2: mask, backbone, residual amax (and MXFP4 residual) -------
    NvScale sb{1.0f, 1.0f, 1.0f};
    if (FMT == 0) {
        sb = nv_scale(__uint_as_float(ld_acquire_gpu(&a.ws[0])));
        fill_inv_table(s_inv, sb.genc);
        if (blockIdx.x == 0 && threadIdx.x == 0) *a.bb_tscale = sb.gdec;
    } else {
        if (blockIdx.x == 0 && threadIdx.x == 0) {
            *a.bb_tscale = 1.0f;
            if (!WEIGHT) *a.rs_tscale = 1.0f;
        }
    }

    float ramax = 0.0f;
    for (int64_t row = gwarp; row < Mpad; row += nwarps) {
        if (row >= M) {   // padding rows of the scale atoms carry zero scales
            for (int s4 = lane; s4 < nsf / 4; s4 += 32) {
                *reinterpret_cast<uint32_t*>(a.bb_scales + sf_off(row, s4 * 4, nsf)) = 0u;
                if (!WEIGHT)
                    *reinterpret_cast<uint32_t*>(a.rs_scales + sf_off(row, s4 * 4, nsf)) = 0u;
            }
            continue;
        }
        const float rinv = HAS_GAMMA ? rinv_ws[row] : 1.0f;
        for (int c = lane; c < nchunk; c += 32) {
            float y[8];
            load_y<HAS_GAMMA>(a, row, c, rinv, y);
            uint32_t keep = WEIGHT ? 0xFFu : topn_bits<MG>(y, a.n);
            float B[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) B[t] = ((keep >> t) & 1u) ? y[t] : 0.0f;
            float bm = amax8(B);
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
            if (FMT == 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));

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
            float t8[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) t8[t] = __fmul_rn(B[t], inv);
            uint32_t codes = cvt_e2m1x8(t8);
            *reinterpret_cast<uint32_t*>(a.bb_codes + row * (K / 2) + (int64_t)c * 4) = codes;
            if (a.mask && !WEIGHT) a.mask[row * (K / 8) + c] = (uint8_t)keep;

            const int stride = (FMT == 0) ? 2 : 4;
            uint32_t word = gather4(ecode, lane, stride);
            if ((lane & (4 * stride - 1)) == 0)
                *reinterpret_cast<uint32_t*>(a.bb_scales + sf_off(row, (c * 8) / BS, nsf)) = word;

            if (!WEIGHT) {
                float d[8], r[8];
                dequant8(codes, sdec, sb.gdec, d);
#pragma unroll
                for (int t = 0; t < 8; ++t) r[t] = __fsub_rn(y[t], d[t]);
                if (FMT == 0) {
                    ramax = fmaxf(ramax, amax8(r));
                } else {
                    // MXFP4: the residual needs no tensor-wide scale; finish it here.
                    float rm = amax8(r);
                    rm = fmaxf(rm, __shfl_xor_sync(0xffffffffu, rm, 1));
                    rm = fmaxf(rm, __shfl_xor_sync(0xffffffffu, rm, 2));
                    uint32_t rc = mx_code(rm);
                    float rinvs = pow2f(127 - (int)rc);
#pragma unroll
                    for (int t = 0; t < 8; ++t) r[t] = __fmul_rn(r[t], rinvs);
                    *reinterpret_cast<uint32_t*>(a.rs_codes + row * (K / 2) + (int64_t)c * 4) =
                        cvt_e2m1x8(r);
                    uint32_t rw = gather4(rc, lane, 4);
                    if ((lane & 15) == 0)
                        *reinterpret_cast<uint32_t*>(a.rs_scales + sf_off(row, (c * 8) / 32, nsf)) = rw;
                }
            }
        }
    }
    if (FMT == 1 || WEIGHT) return;

    block_amax_to_global(ramax, &a.ws[1], s_red);
    grid_barrier(&a.ws[2], 2u * gridDim.x);

    // ---------------- phase 3: residual codes with G_r ----------------
    NvScale sr = nv_scale(__uint_as_float(ld_acquire_gpu(&a.ws[1])));
    __syncthreads();                       // everyone done reading the backbone table
    fill_inv_table(s_inv, sr.genc);
    if (blockIdx.x == 0 && threadIdx.x == 0) *a.rs_tscale = sr.gdec;
    for (int64_t row = gwarp; row < M; row += nwarps) {
        const float rinv = HAS_GAMMA ? rinv_ws[row] : 1.0f;
        for (int c = lane; c < nchunk; c += 32) {
            float y[8];
            load_y<HAS_GAMMA>(a, row, c, rinv, y);
            // backbone dequant from the codes and scale written in phase 2
            uint32_t codes = *reinterpret_cast<const uint32_t*>(a.bb_codes + row * (K / 2) + (int64_t)c * 4);
            uint32_t eb = a.bb_scales[sf_off(row, c / 2, nsf)];
            float d[8], r[8];
            dequant8(codes, e4m3_to_f32(eb), sb.gdec, d);
#pragma unroll
            for (int t = 0; t < 8; ++t) r[t] = __fsub_rn(y[t], d[t]);
            float rm = amax8(r);
            rm = fmaxf(rm, __shfl_xor_sync(0xffffffffu, rm, 1));
            uint32_t er = cvt_e4m3(__fmul_rn(rm, sr.k1));
            float inv = s_inv[er];
#pragma unroll
            for (int t = 0; t < 8; ++t) r[t] = __fmul_rn(r[t], inv);
            *reinterpret_cast<uint32_t*>(a.rs_codes + row * (K / 2) + (int64_t)c * 4) = cvt_e2m1x8(r);
            uint32_t word = gather4(er, lane, 2);
            if ((lane & 7) == 0)
                *reinterpret_cast<uint32_t*>(a.rs_scales + sf_off(row, c / 2, nsf)) = word;
        }
    }
}

template <int FMT, bool HAS_GAMMA, int MG, bool WEIGHT>
cudaError_t launch_one(const PrepArgs& a, cudaStream_t s, int max_blocks) {
    auto kfn = prepare_kernel<FMT, HAS_GAMMA, MG, WEIGHT>;
    static int blocks_per_sm = 0;          // same for every device of one architecture
    if (blocks_per_sm == 0) {
        int b = 0;
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kfn, kThreads, 0);
        if (e != cudaSuccess) return e;
        blocks_per_sm = b;
    }
    int64_t Mpad = (a.M + 127) / 128 * 128;
    int64_t want = (Mpad + kWarps - 1) / kWarps;
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
    cfg.numAttrs = (FMT == 0) ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kfn, a);
}

template <int FMT, bool HAS_GAMMA, bool WEIGHT>
cudaError_t launch_m(const PrepArgs& a, int m, cudaStream_t s, int sms) {
    switch (m) {
        case 2: return launch_one<FMT, HAS_GAMMA, 2, WEIGHT>(a, s, sms);
        case 4: return launch_one<FMT, HAS_GAMMA, 4, WEIGHT>(a, s, sms);
        default: return launch_one<FMT, HAS_GAMMA, 8, WEIGHT>(a, s, sms);
    }
}

}  // namespace

size_t prepare_ws_bytes(int64_t M) {
    size_t b = 64 + (size_t)(M > 0 ? M : 0) * 4;
    return (b + 255) / 256 * 256;
}

cudaError_t launch_prepare(const PrepareLaunch& p, cudaStream_t s, int sms) {
    PrepArgs a;
    a.X = static_cast<const uint16_t*>(p.X);
    a.gamma = static_cast<const uint16_t*>(p.gamma);
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
    cudaError_t e = cudaMemsetAsync(p.ws, 0, 64, s);
    if (e != cudaSuccess) return e;
    const bool g = p.gamma != nullptr;
    if (p.weight) {
        return p.fmt == 0 ? launch_one<0, false, 8, true>(a, s, sms)
                          : launch_one<1, false, 8, true>(a, s, sms);
    }
    if (p.fmt == 0) return g ? launch_m<0, true, false>(a, p.m, s, sms) : launch_m<0, false, false>(a, p.m, s, sms);
    return g ? launch_m<1, true, false>(a, p.m, s, sms) : launch_m<1, false, false>(a, p.m, s, sms);
}

}  // namespace sharq
