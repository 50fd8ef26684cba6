// linear.cu -- two-path block-scaled FP4 linear on tcgen05 tensor cores.
//
// SharQ paper, Abstract: a sparse FP4 GEMM runs on the backbone, a dense FP4
// GEMM on the residual, and both read one FP4 weight payload with per-path
// scale views.  Here both paths share every weight tile: per k-step one TMA
// load brings the weight tile, the backbone tile and the residual tile (plus
// their E4M3/E8M0 scale atoms) into shared memory, and one thread issues two
// block-scaled MMAs into two fp32 accumulators in tensor memory:
//   acc_b += A_b x W^T,   acc_r += A_r x W^T.
// The epilogue reads both accumulators back and writes
//   Y = G_w * (G_b * acc_b + G_r * acc_r)
// as bf16 (or fp32).  The backbone runs as a dense MMA over zero-filled codes:
// the FP4 sparse MMA carries one scale per 32 logical elements, which cannot
// express NVFP4's per-16 backbone scales.
//
// CTA layout (192 threads): warp 0 = TMA producer, warp 1 = TMEM allocator
// and MMA issuer, warps 2..5 = epilogue (one TMEM lane quarter each).
// Tile 128 x 128 x 256 (K in elements), 4-stage mbarrier pipeline.
#include "common.cuh"
#include "sharq_internal.h"

#include <cuda.h>
#include <cuda_bf16.h>

namespace sharq {
namespace {

constexpr int BM = 128, BN = 128, BK = 256;   // BK in FP4 elements = 128 bytes per row
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr uint32_t kTileBytes = BM * (BK / 2);  // 16 KiB per operand tile
constexpr uint32_t kTmemCols = 512;

template <int FMT>
struct Cfg {
    static constexpr int BS = FMT == 0 ? 16 : 32;                 // elements per scale
    static constexpr int kAtoms = BK / BS / 4;                    // scale atoms per operand per stage
    static constexpr uint32_t kSfBytes = kAtoms * 512;
    static constexpr int kStepsPerAtom = 4 * BS / 64;             // MMA k-steps (K=64) per atom
    static constexpr uint32_t kStageBytes = 3 * kTileBytes + 3 * kSfBytes;
    static constexpr uint32_t kStageStride = (kStageBytes + 1023) / 1024 * 1024;
    // Instruction descriptor: E2M1 A and B (format 1), K-major, N>>3 at bit
    // 17, scale format (0 E4M3, 1 E8M0) at bit 23, M>>4 at bit 24.
    static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                       ((uint32_t)FMT << 23) | ((uint32_t)(BM >> 4) << 24);
};

struct alignas(8) Barriers {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t acc_full;
    uint32_t tmem_base;
};

// sf_id selects the byte inside each 32-bit scale column (two E8M0 scales
// per MMA k-step for MXFP4): it goes into the instruction descriptor's
// A/B scale-factor ID fields (bits 29-30 and 4-5) and into the top two bits
// of the tensor-memory scale addresses.
template <int FMT>
__device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t sfa,
                                    uint32_t sfb, uint32_t acc, uint32_t sf_id) {
    const uint32_t idesc = Cfg<FMT>::kIdesc | (sf_id << 29) | (sf_id << 4);
    const uint32_t hi = sf_id << 30;
    if (FMT == 0) tc_mma_nvf4(d, a, b, idesc, sfa | hi, sfb | hi, acc);
    else          tc_mma_mxf4(d, a, b, idesc, sfa | hi, sfb | hi, acc);
}

struct EpiArgs {
    const float* bb_tscale;
    const float* rs_tscale;
    const float* w_tscale;
    void* Y;
    int64_t M;
    int N;
    int y_fp32;
};

template <int FMT>
__global__ void __launch_bounds__(kThreads, 1)
linear_kernel(const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_r,
              const __grid_constant__ CUtensorMap tm_w, const uint8_t* __restrict__ sf_b,
              const uint8_t* __restrict__ sf_r, const uint8_t* __restrict__ sf_w, int K,
              EpiArgs ep) {
    using C = Cfg<FMT>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Barriers* bars = reinterpret_cast<Barriers*>(smem + kStages * C::kStageStride);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mt = blockIdx.x, nt = blockIdx.y;
    const int nk = K / BK;
    const int nsf = K / C::BS;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) { mbar_init(&bars->full[s], 1); mbar_init(&bars->empty[s], 1); }
        mbar_init(&bars->acc_full, 1);
        fence_barrier_init();
    }
    if (warp == 1) { tmem_alloc(&bars->tmem_base, kTmemCols); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const uint32_t t_acc_b = tmem, t_acc_r = tmem + BN;
    const uint32_t t_sfa_b = tmem + 2 * BN;
    const uint32_t t_sfa_r = t_sfa_b + 4 * C::kAtoms;
    const uint32_t t_sfb = t_sfa_r + 4 * C::kAtoms;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tm_b); prefetch_tmap(&tm_r); prefetch_tmap(&tm_w);
            const uint8_t* gb = sf_b + (int64_t)mt * (nsf / 4) * 512;
            const uint8_t* gr = sf_r + (int64_t)mt * (nsf / 4) * 512;
            const uint8_t* gw = sf_w + (int64_t)nt * (nsf / 4) * 512;
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % kStages;
                if (kb >= kStages && !mbar_wait(&bars->empty[s], ((kb / kStages) - 1) & 1)) break;
                uint8_t* st = smem + s * C::kStageStride;
                mbar_arrive_expect_tx(&bars->full[s], C::kStageBytes);
                tma_load_2d(st, &tm_b, &bars->full[s], kb * (BK / 2), mt * BM);
                tma_load_2d(st + kTileBytes, &tm_r, &bars->full[s], kb * (BK / 2), mt * BM);
                tma_load_2d(st + 2 * kTileBytes, &tm_w, &bars->full[s], kb * (BK / 2), nt * BN);
                const int64_t sfo = (int64_t)kb * C::kAtoms * 512;
                bulk_load(st + 3 * kTileBytes, gb + sfo, C::kSfBytes, &bars->full[s]);
                bulk_load(st + 3 * kTileBytes + C::kSfBytes, gr + sfo, C::kSfBytes, &bars->full[s]);
                bulk_load(st + 3 * kTileBytes + 2 * C::kSfBytes, gw + sfo, C::kSfBytes, &bars->full[s]);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            bool ok = true;
            for (int kb = 0; kb < nk && ok; ++kb) {
                const int s = kb % kStages;
                if (!mbar_wait(&bars->full[s], (kb / kStages) & 1)) { ok = false; break; }
                tc_fence_after();
                uint8_t* st = smem + s * C::kStageStride;
                const uint32_t a_b = smem_u32(st), a_r = smem_u32(st + kTileBytes);
                const uint32_t a_w = smem_u32(st + 2 * kTileBytes);
                const uint32_t s_b = smem_u32(st + 3 * kTileBytes);
                const uint32_t s_r = s_b + C::kSfBytes, s_w = s_b + 2 * C::kSfBytes;
#pragma unroll
                for (int at = 0; at < C::kAtoms; ++at) {
                    tc_cp_32x128b_warpx4(t_sfa_b + 4 * at, sdesc_sf_atom(s_b + 512 * at));
                    tc_cp_32x128b_warpx4(t_sfa_r + 4 * at, sdesc_sf_atom(s_r + 512 * at));
                    tc_cp_32x128b_warpx4(t_sfb + 4 * at, sdesc_sf_atom(s_w + 512 * at));
                }
#pragma unroll
                for (int j = 0; j < BK / 64; ++j) {
                    const int at = j / C::kStepsPerAtom;
                    const uint32_t sf_id = (uint32_t)(j % C::kStepsPerAtom) * (4 / C::kStepsPerAtom);
                    const uint32_t col = 4 * at;
                    const uint64_t db = sdesc_sw128(a_w + 32 * j);
                    const uint32_t acc = (kb | j) ? 1u : 0u;
                    mma<FMT>(t_acc_b, sdesc_sw128(a_b + 32 * j), db, t_sfa_b + col, t_sfb + col,
                             acc, sf_id);
                    mma<FMT>(t_acc_r, sdesc_sw128(a_r + 32 * j), db, t_sfa_r + col, t_sfb + col,
                             acc, sf_id);
                }
                tc_commit(&bars->empty[s]);
            }
            tc_commit(&bars->acc_full);
        }
    } else {
        // Epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 = rows of the tile.
        const int q = warp & 3;
        const int64_t row = (int64_t)mt * BM + q * 32 + lane;
        const bool ok = mbar_wait(&bars->acc_full, 0);
        tc_fence_after();
        if (ok) {
            const float gw = *ep.w_tscale;
            const float gb = *ep.bb_tscale * gw, gr = *ep.rs_tscale * gw;
            const uint32_t lane_off = (uint32_t)(q * 32) << 16;
#pragma unroll 1
            for (int cc = 0; cc < BN / 32; ++cc) {
                uint32_t vb[32], vr[32];
                tmem_ld_32x32b_x32(t_acc_b + lane_off + cc * 32, vb);
                tmem_ld_32x32b_x32(t_acc_r + lane_off + cc * 32, vr);
                tmem_ld_wait();
                if (row < ep.M) {
                    const int64_t col0 = (int64_t)nt * BN + cc * 32;
                    if (ep.y_fp32) {
                        float* y = static_cast<float*>(ep.Y) + row * ep.N + col0;
#pragma unroll
                        for (int i = 0; i < 32; i += 4) {
                            float4 o;
                            o.x = gb * __uint_as_float(vb[i + 0]) + gr * __uint_as_float(vr[i + 0]);
                            o.y = gb * __uint_as_float(vb[i + 1]) + gr * __uint_as_float(vr[i + 1]);
                            o.z = gb * __uint_as_float(vb[i + 2]) + gr * __uint_as_float(vr[i + 2]);
                            o.w = gb * __uint_as_float(vb[i + 3]) + gr * __uint_as_float(vr[i + 3]);
                            *reinterpret_cast<float4*>(y + i) = o;
                        }
                    } else {
                        __nv_bfloat16* y = static_cast<__nv_bfloat16*>(ep.Y) + row * ep.N + col0;
#pragma unroll
                        for (int i = 0; i < 32; i += 8) {
                            uint32_t w[4];
#pragma unroll
                            for (int h = 0; h < 4; ++h) {
                                float lo = gb * __uint_as_float(vb[i + 2 * h]) + gr * __uint_as_float(vr[i + 2 * h]);
                                float hi = gb * __uint_as_float(vb[i + 2 * h + 1]) + gr * __uint_as_float(vr[i + 2 * h + 1]);
                                __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
                                w[h] = *reinterpret_cast<uint32_t*>(&p);
                            }
                            *reinterpret_cast<uint4*>(y + i) = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, kTmemCols); }
}

// ------------------------------------------------------------------ host --

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2-D uint8 map over a [rows, row_bytes] code matrix, box 128 bytes x box_rows,
// 128-byte swizzle; rows past the end read as zero.
bool make_code_map(CUtensorMap* m, const void* base, int64_t rows, int64_t row_bytes, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int FMT>
cudaError_t launch_linear_t(const LinearLaunch& p, cudaStream_t s) {
    using C = Cfg<FMT>;
    CUtensorMap tb, tr, tw;
    if (!make_code_map(&tb, p.bb_codes, p.M, p.K / 2, BM) ||
        !make_code_map(&tr, p.rs_codes, p.M, p.K / 2, BM) ||
        !make_code_map(&tw, p.w_codes, p.N, p.K / 2, BN))
        return cudaErrorInvalidValue;
    const size_t smem = kStages * C::kStageStride + sizeof(Barriers) + 1024;
    auto kfn = linear_kernel<FMT>;
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_set[dev] = true;
    }
    EpiArgs ep{p.bb_tscale, p.rs_tscale, p.w_tscale, p.Y, p.M, p.N, p.y_fp32};
    dim3 grid((unsigned)((p.M + BM - 1) / BM), (unsigned)(p.N / BN));
    kfn<<<grid, kThreads, smem, s>>>(tb, tr, tw, static_cast<const uint8_t*>(p.bb_scales),
                                     static_cast<const uint8_t*>(p.rs_scales),
                                     static_cast<const uint8_t*>(p.w_scales), p.K, ep);
    return cudaGetLastError();
}

}  // namespace

unsigned take_status_linear() { return take_tu_status(); }

cudaError_t launch_linear(const LinearLaunch& p, cudaStream_t s, int /*sms*/) {
    if (p.M == 0) return cudaSuccess;
    return p.fmt == 0 ? launch_linear_t<0>(p, s) : launch_linear_t<1>(p, s);
}

cudaError_t launch_moe_linear(const LinearLaunch&, cudaStream_t, int) {
    return cudaErrorNotSupported;
}

}  // namespace sharq
