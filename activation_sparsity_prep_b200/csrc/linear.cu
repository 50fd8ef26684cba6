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
// as bf16 (or fp32).  The SwiGLU form (the gate+up projection of an MLP,
// its weight rows interleaved 64 gate / 64 up per 128-row tile) writes
// H = silu(gate) * up instead, half as many bf16 columns, and the maximum of
// |H|: the next prepare's backbone amax, so that prepare skips its own pass
// over H.  When the two tensor scales are equal by construction (MXFP4, or
// a residual quantised against the backbone's tensor scale) both MMAs
// accumulate into one accumulator, Y = G_w * G_b * acc, and the two
// tensor-memory accumulators serve as a double buffer instead: the next
// tile's MMAs run while the epilogue drains the previous one.  An element
// n:m backbone runs as a dense MMA over zero-filled codes: the FP4 sparse
// MMA carries one scale per 32 logical elements, which cannot express
// NVFP4's per-16 backbone scales, and its metadata selects whole pairs.  The
// pair-granular 4:8 MXFP4 backbone, stored compressed, runs on the sparse
// MMA (tcgen05.mma.sp) instead (SPB).
//
// CTA layout (320 threads): warp 0 = TMA producer, warp 1 = TMEM allocator
// and MMA issuer, warps 2..5 = epilogue (one TMEM lane quarter each),
// warps 6..9 = scale warps (block scales from shared into tensor memory).
// Tile 128 x 128 x 256 (K in elements), 4-stage mbarrier pipeline; one
// persistent CTA per SM walks the output tiles.
#include "common.cuh"
#include "sharq_internal.h"

#include <cuda.h>
#include <cuda_bf16.h>

#include <atomic>

namespace sharq {
namespace {

constexpr int BM = 128, BN = 128, BK = 256;   // BK in FP4 elements = 128 bytes per row
constexpr int kStages = 4;
constexpr int kThreads = 320;
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

// Stage of the sparse-backbone form (MXFP4, pair-granular 4:8 backbone):
// the backbone tile holds only the kept pairs, 64 bytes per row (64-byte
// swizzle), followed by the residual and weight tiles, the three scale
// groups and the 128-row x 16-byte pair-metadata atom of the k-step.
struct SpStage {
    static constexpr uint32_t kBc = 0;                         // compressed backbone, 8 KiB
    static constexpr uint32_t kRs = BM * (BK / 4);             // residual tile, 16 KiB
    static constexpr uint32_t kW = kRs + kTileBytes;            // weight tile, 16 KiB
    static constexpr uint32_t kSf = kW + kTileBytes;            // 3 x 1 KiB of E8M0 scale atoms
    static constexpr uint32_t kSfBytes = Cfg<1>::kSfBytes;
    static constexpr uint32_t kMeta = kSf + 3 * kSfBytes;       // 2 KiB of pair indices
    static constexpr uint32_t kMetaBytes = BM * 16;
    static constexpr uint32_t kBytes = kMeta + kMetaBytes;
    static constexpr uint32_t kStride = (kBytes + 1023) / 1024 * 1024;
    // sparse MMA: E2M1 A and B, E8M0 scales per 32 logical elements
    // (block16 of stored elements), sparse flag, N and M as the dense form
    static constexpr uint32_t kIdesc = (1u << 2) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                       (1u << 23) | ((uint32_t)(BM >> 4) << 24);
};
static_assert(SpStage::kStride % 1024 == 0 && SpStage::kRs % 1024 == 0 && SpStage::kW % 1024 == 0,
              "swizzled tiles start on 1 KiB boundaries");

// Stage of the 256-wide tile (one accumulator, 256 output columns per MMA):
// the backbone tile (zero-filled 16 KiB, or the compressed pairs' 8 KiB),
// the residual tile, a 256-row weight tile (32 KiB), the scale atoms of the
// backbone rows, the residual rows and the weight's rows 0..127 and
// 128..255, and (SPB) the pair-metadata atom.
constexpr int BNW = 256;
constexpr int kStagesW = 3;
template <int FMT, bool SPB>
struct WideStage {
    static constexpr uint32_t kRs = SPB ? BM * (BK / 4) : kTileBytes;
    static constexpr uint32_t kW = kRs + kTileBytes;
    static constexpr uint32_t kSf = kW + 2 * kTileBytes;          // = the operand tiles' bytes
    static constexpr uint32_t kSfBytes = Cfg<FMT>::kSfBytes;
    static constexpr uint32_t kMeta = kSf + 4 * kSfBytes;
    static constexpr uint32_t kBytes = kMeta + (SPB ? BM * 16 : 0);
    static constexpr uint32_t kStride = (kBytes + 1023) / 1024 * 1024;
    static_assert(kRs % 1024 == 0 && kW % 1024 == 0, "swizzled tiles start on 1 KiB boundaries");
};

struct alignas(8) Barriers {
    uint64_t full[kStages];       // the stage's operand tiles have landed
    uint64_t sfl[kStages];        // the stage's scale atoms (and pair indices) have landed
    uint64_t empty[kStages];      // MMAs done (tcgen05.commit) + scale warps done reading
    uint64_t sf_full[kStages];    // scale factors of the stage are in tensor memory
    uint64_t acc_full[2];   // MMAs of a tile done (tcgen05.commit), per accumulator buffer
    uint64_t acc_empty[2];  // epilogue has drained that buffer (4 warps)
    uint32_t tmem_base;
};

// sf_id selects the byte inside each 32-bit scale column (two E8M0 scales
// per MMA k-step for MXFP4): it goes into the instruction descriptor's
// A/B scale-factor ID fields (bits 29-30 and 4-5) and into the top two bits
// of the tensor-memory scale addresses.
// N at bits 17..22 of an instruction descriptor (N >> 3)
constexpr uint32_t with_n(uint32_t idesc, int n) {
    return (idesc & ~(0x3Fu << 17)) | ((uint32_t)(n >> 3) << 17);
}

template <int FMT, int TN = BN>
__device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t sfa,
                                    uint32_t sfb, uint32_t acc, uint32_t sf_id) {
    const uint32_t idesc = with_n(Cfg<FMT>::kIdesc, TN) | (sf_id << 29) | (sf_id << 4);
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
    uint32_t* amax;    // SwiGLU form: max |H| as fp32 bits (zeroed before the launch)
};

// silu(g) = g / (1 + e^-g) in fp32 with the fast exponential and divide
// (relative error within (5 + 1.2 |g|) 2^-23 while 1 + e^-g < 2^126, i.e.
// g > -87; below that the quotient is 0, against a true |silu| < 1e-36).
// The correctly rounded forms cost about 6 % of the gate+up linear's time.
__device__ __forceinline__ float silu_f32(float g) {
    return __fdividef(g, 1.0f + __expf(-g));
}

// One output tile of the (plain or grouped) problem.
struct TileInfo {
    int64_t a_row;     // first row of the activation tiles (multiple of 128)
    int64_t w_row;     // first row of the weight tile in the (stacked) weight
    int64_t w_sf;      // byte offset of the weight tile's first scale atom
    int64_t y_row;     // first output row
    int rows;          // valid output rows in this tile (<= 128)
    int col;           // first output column
    int e;             // expert (0 for the plain linear)
};

constexpr int kMaxExperts = 256;    // keeps the scheduler's shared memory at 3 KiB

// Tile scheduler.  Plain linear: the CTAs working at one time walk
// neighbouring tiles of the fast dimension, so they share the slow
// dimension's operand tiles, and the fast dimension's operand rows (all of
// them) stay resident in L2 while the other operand streams from HBM about
// once.  m fastest keeps the activations resident, n fastest the weight;
// the launch keeps the smaller of the two resident (with the larger one
// resident-but-too-big, it would stream from HBM once per wave of tiles).  Grouped linear: expert-major,
// then n, then m, so one expert's weight and activation rows stay hot in L2
// while its tiles run; rows of expert e sit at a 128-aligned padded offset
// of the gathered operands.
struct Sched {
    int mt_count, nt_count;    // plain: m-tiles, n-tiles
    int64_t M;
    int nsf;                   // scales per row
    int grouped;
    const int32_t* offsets;    // grouped: dispatch offsets [E+1] (device)
    int E;
    int64_t w_sf_stride;       // grouped: bytes of one expert's scale buffer
    int N;
    int n_fast;                // plain: n-tiles fastest instead of m-tiles
    int bn;                    // plain: output columns per tile (128, or 256 for the wide tile)
};

struct SchedTables {
    int off[kMaxExperts + 1];    // dispatch offsets
    int poff[kMaxExperts + 1];   // padded row offsets (128-aligned)
    int tpre[kMaxExperts + 1];   // tile prefix
};

// Grouped form: the scheduler tables and one 1 KiB epilogue staging buffer
// per epilogue warp.  Plain form (no tables): one 2 KiB staging buffer per
// epilogue warp over the same bytes.
union SchedSmem {
    struct {
        SchedTables t;
        alignas(16) uint8_t stage[4][1024];
    } g;
    uint8_t stage2[4][2048];
};

__device__ __forceinline__ int ceil128(int x) { return (x + 127) >> 7; }

// Exclusive prefix sums of the per-expert padded rows and tiles, by warp 0.
__device__ void sched_prepare(const Sched& sc, SchedSmem* sm) {
    if (!sc.grouped) return;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x < 32) {
        int carry_p = 0, carry_t = 0;
        for (int base = 0; base < sc.E; base += 32) {
            const int e = base + lane;
            int cnt = 0;
            if (e < sc.E) {
                const int o0 = sc.offsets[e], o1 = sc.offsets[e + 1];
                sm->g.t.off[e] = o0;
                cnt = o1 - o0;
            }
            int pr = ceil128(cnt) * 128, tl = ceil128(cnt) * sc.nt_count;
            int ip = pr, it = tl;                      // inclusive warp scans
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int vp = __shfl_up_sync(0xffffffffu, ip, o), vt = __shfl_up_sync(0xffffffffu, it, o);
                if (lane >= o) { ip += vp; it += vt; }
            }
            if (e < sc.E) { sm->g.t.poff[e] = carry_p + ip - pr; sm->g.t.tpre[e] = carry_t + it - tl; }
            carry_p += __shfl_sync(0xffffffffu, ip, 31);
            carry_t += __shfl_sync(0xffffffffu, it, 31);
        }
        if (lane == 0) {
            sm->g.t.off[sc.E] = sc.offsets[sc.E];
            sm->g.t.poff[sc.E] = carry_p;
            sm->g.t.tpre[sc.E] = carry_t;
        }
    }
}

__device__ __forceinline__ int sched_count(const Sched& sc, const SchedSmem* sm) {
    return sc.grouped ? sm->g.t.tpre[sc.E] : sc.mt_count * sc.nt_count;
}

__device__ __forceinline__ TileInfo sched_tile(const Sched& sc, const SchedSmem* sm, int t) {
    TileInfo ti;
    if (!sc.grouped) {
        int nt, mt;
        if (sc.n_fast) { mt = t / sc.nt_count; nt = t - mt * sc.nt_count; }
        else           { nt = t / sc.mt_count; mt = t - nt * sc.mt_count; }
        ti.a_row = (int64_t)mt * 128;
        ti.w_row = (int64_t)nt * sc.bn;
        ti.w_sf = (int64_t)nt * (sc.bn / 128) * (sc.nsf / 4) * 512;
        ti.y_row = ti.a_row;
        ti.rows = (int)(sc.M - ti.a_row < 128 ? sc.M - ti.a_row : 128);
        ti.col = nt * sc.bn;
        ti.e = 0;
        return ti;
    }
    int lo = 0, hi = sc.E;                          // largest e with tpre[e] <= t
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (sm->g.t.tpre[mid] <= t) lo = mid; else hi = mid;
    }
    const int e = lo;
    const int cnt = sm->g.t.off[e + 1] - sm->g.t.off[e];
    const int mtn = ceil128(cnt);
    const int local = t - sm->g.t.tpre[e];
    const int nt = local / mtn, mt = local - nt * mtn;
    ti.a_row = sm->g.t.poff[e] + (int64_t)mt * 128;
    ti.w_row = (int64_t)e * sc.N + (int64_t)nt * 128;
    ti.w_sf = (int64_t)e * sc.w_sf_stride + (int64_t)nt * (sc.nsf / 4) * 512;
    ti.y_row = sm->g.t.off[e] + (int64_t)mt * 128;
    ti.rows = min(128, cnt - mt * 128);
    ti.col = nt * 128;
    ti.e = e;
    return ti;
}

// Persistent kernel: CTA c computes tiles c, c + G, c + 2G, ...  The TMA
// producer runs ahead across tile boundaries through a kStages ring; the MMA
// thread waits only until the epilogue has copied the previous tile's two
// accumulators out of tensor memory, so the epilogue's global stores overlap
// the next tile's MMAs.
// SPB: the backbone is the compressed pair-granular 4:8 form (MXFP4 only):
// per k-step two sparse MMAs (128 logical K each, pair indices in tensor
// memory) on the backbone and four dense MMAs on the residual, all into one
// accumulator and all on the same weight tile.
// WIDE (one accumulator only): 128 x 256 output tiles.  Every MMA is 256
// columns wide, so per unit of MMA work a k-step moves a third fewer operand
// and scale bytes; the 256-column accumulator fills half of tensor memory,
// so it is not double-buffered (the next tile's MMAs wait for the drain),
// and the ring has three stages.  In tensor memory the weight's scales for
// a 256-row tile take 8 columns per scale atom along K: the atom of rows
// 0..127 in the first four, that of rows 128..255 in the next four (one
// column per 32-row group, as for 128 rows).
template <int FMT, bool ONE, bool SW, bool SPB, bool WIDE = false>
__global__ void __launch_bounds__(kThreads, 1)
linear_kernel(const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_r,
              const __grid_constant__ CUtensorMap tm_w, const uint8_t* __restrict__ sf_b,
              const uint8_t* __restrict__ sf_r, const uint8_t* __restrict__ sf_w,
              const uint8_t* __restrict__ meta, int K, EpiArgs ep, Sched sc) {
    using C = Cfg<FMT>;
    using WS = WideStage<FMT, SPB>;
    static_assert(!SPB || (FMT == 1 && ONE && !SW), "sparse backbone: MXFP4, one accumulator");
    static_assert(!WIDE || (ONE && !SW), "wide tile: one accumulator, plain epilogue");
    constexpr int TBN = WIDE ? BNW : BN;                  // output columns per tile
    constexpr int NST = WIDE ? kStagesW : kStages;        // pipeline stages
    constexpr bool DBUF = ONE && !WIDE;                   // double-buffered accumulator
    constexpr uint32_t kAccCols = WIDE ? BNW : 2 * BN;
    constexpr uint32_t kStride = WIDE ? WS::kStride : SPB ? SpStage::kStride : C::kStageStride;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Barriers* bars = reinterpret_cast<Barriers*>(smem + NST * kStride);
    // 128-byte aligned: the staging buffers take 16-byte vector stores
    SchedSmem* ssm = reinterpret_cast<SchedSmem*>(
        (reinterpret_cast<uintptr_t>(bars) + sizeof(Barriers) + 127) & ~uintptr_t(127));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = K / BK;
    const int nsf = K / C::BS;
    sched_prepare(sc, ssm);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->sfl[s], 1);
            mbar_init(&bars->empty[s], 1 + 4);
            mbar_init(&bars->sf_full[s], 4);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->acc_full[b], 1);
            mbar_init(&bars->acc_empty[b], 4);
        }
        fence_barrier_init();
    }
    if (warp == 1) { tmem_alloc(&bars->tmem_base, kTmemCols); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const int ntiles = sched_count(sc, ssm);
    const uint32_t tmem = bars->tmem_base;
    const uint32_t t_acc_b = tmem, t_acc_r = tmem + BN;
    // Scale factors: one tensor-memory buffer per pipeline stage, written by
    // the four scale warps (warps 6..9) with tcgen05.st, each into its own
    // 32-lane quarter -- which also gives the replication across quarters
    // that the block-scaled MMA reads.  Copying them with tcgen05.cp would
    // put 3 * kAtoms copies per stage into the MMA issue stream, where they
    // do not overlap the MMAs.
    // Per stage: the backbone's and the residual's scales (4 columns per
    // atom each), the weight's (4, or 8 for the wide tile), the pair indices.
    constexpr uint32_t kSfbAtomCols = WIDE ? 8 : 4;
    constexpr uint32_t kScaleCols = (8 + kSfbAtomCols) * C::kAtoms;
    constexpr uint32_t kSfColsPerStage = kScaleCols + (SPB ? 4 : 0);   // + the pair indices
    static_assert(kAccCols + NST * kSfColsPerStage <= kTmemCols, "tensor memory budget");

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tm_b); prefetch_tmap(&tm_r); prefetch_tmap(&tm_w);
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
                const TileInfo ti = sched_tile(sc, ssm, tile);
                const uint8_t* gb = sf_b + (ti.a_row >> 7) * (nsf / 4) * 512;
                const uint8_t* gr = sf_r + (ti.a_row >> 7) * (nsf / 4) * 512;
                const uint8_t* gw = sf_w + ti.w_sf;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const uint32_t s = it % NST;
                    if (it >= (uint32_t)NST && !mbar_wait(&bars->empty[s], ((it / NST) - 1) & 1)) { ok = false; break; }
                    uint8_t* st = smem + s * kStride;
                    const int64_t sfo = (int64_t)kb * C::kAtoms * 512;
                    // The scale bytes come first, on their own barrier, so the
                    // scale warps stage them into tensor memory while the
                    // operand tiles are still arriving.
                    if constexpr (WIDE) {
                        mbar_arrive_expect_tx(&bars->sfl[s], WS::kBytes - WS::kSf);
                        bulk_load(st + WS::kSf, gb + sfo, WS::kSfBytes, &bars->sfl[s]);
                        bulk_load(st + WS::kSf + WS::kSfBytes, gr + sfo, WS::kSfBytes, &bars->sfl[s]);
                        // the weight's rows 0..127 and 128..255: consecutive row blocks
                        bulk_load(st + WS::kSf + 2 * WS::kSfBytes, gw + sfo, WS::kSfBytes, &bars->sfl[s]);
                        bulk_load(st + WS::kSf + 3 * WS::kSfBytes, gw + (int64_t)(nsf / 4) * 512 + sfo,
                                  WS::kSfBytes, &bars->sfl[s]);
                        if constexpr (SPB) {
                            const int64_t mpad = (sc.M + 127) / 128 * 128;
                            bulk_load(st + WS::kMeta, meta + ((int64_t)kb * (mpad >> 7) + (ti.a_row >> 7)) * 2048,
                                      BM * 16, &bars->sfl[s]);
                        }
                        mbar_arrive_expect_tx(&bars->full[s], WS::kSf);
                        tma_load_2d(st, &tm_b, &bars->full[s], kb * (SPB ? BK / 4 : BK / 2), (int)ti.a_row);
                        tma_load_2d(st + WS::kRs, &tm_r, &bars->full[s], kb * (BK / 2), (int)ti.a_row);
                        tma_load_2d(st + WS::kW, &tm_w, &bars->full[s], kb * (BK / 2), (int)ti.w_row);
                    } else if constexpr (SPB) {
                        using P = SpStage;
                        mbar_arrive_expect_tx(&bars->sfl[s], P::kBytes - P::kSf);
                        bulk_load(st + P::kSf, gb + sfo, P::kSfBytes, &bars->sfl[s]);
                        bulk_load(st + P::kSf + P::kSfBytes, gr + sfo, P::kSfBytes, &bars->sfl[s]);
                        bulk_load(st + P::kSf + 2 * P::kSfBytes, gw + sfo, P::kSfBytes, &bars->sfl[s]);
                        // metadata atom (k-step kb, row block a_row / 128)
                        const int64_t mpad = (sc.M + 127) / 128 * 128;
                        bulk_load(st + P::kMeta, meta + ((int64_t)kb * (mpad >> 7) + (ti.a_row >> 7)) * 2048,
                                  P::kMetaBytes, &bars->sfl[s]);
                        mbar_arrive_expect_tx(&bars->full[s], P::kSf);
                        tma_load_2d(st + P::kBc, &tm_b, &bars->full[s], kb * (BK / 4), (int)ti.a_row);
                        tma_load_2d(st + P::kRs, &tm_r, &bars->full[s], kb * (BK / 2), (int)ti.a_row);
                        tma_load_2d(st + P::kW, &tm_w, &bars->full[s], kb * (BK / 2), (int)ti.w_row);
                    } else {
                        mbar_arrive_expect_tx(&bars->sfl[s], 3 * C::kSfBytes);
                        bulk_load(st + 3 * kTileBytes, gb + sfo, C::kSfBytes, &bars->sfl[s]);
                        bulk_load(st + 3 * kTileBytes + C::kSfBytes, gr + sfo, C::kSfBytes, &bars->sfl[s]);
                        bulk_load(st + 3 * kTileBytes + 2 * C::kSfBytes, gw + sfo, C::kSfBytes, &bars->sfl[s]);
                        mbar_arrive_expect_tx(&bars->full[s], 3 * kTileBytes);
                        tma_load_2d(st, &tm_b, &bars->full[s], kb * (BK / 2), (int)ti.a_row);
                        tma_load_2d(st + kTileBytes, &tm_r, &bars->full[s], kb * (BK / 2), (int)ti.a_row);
                        tma_load_2d(st + 2 * kTileBytes, &tm_w, &bars->full[s], kb * (BK / 2), (int)ti.w_row);
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            uint32_t it = 0, tc = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++tc) {
                // the epilogue must have drained this buffer's previous tile
                const uint32_t buf = DBUF ? (tc & 1u) : 0u;
                const uint32_t use = DBUF ? (tc >> 1) : tc;
                if (use > 0 && !mbar_wait(&bars->acc_empty[buf], (use - 1) & 1)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_b = ONE ? tmem + buf * BN : t_acc_b;
                const uint32_t d_r = ONE ? d_b : t_acc_r;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const uint32_t s = it % NST;
                    if (!mbar_wait(&bars->full[s], (it / NST) & 1)) { ok = false; break; }
                    if (!mbar_wait(&bars->sf_full[s], (it / NST) & 1)) { ok = false; break; }
                    tc_fence_after();
                    uint8_t* st = smem + s * kStride;
                    const uint32_t t_sfa_b = tmem + kAccCols + s * kSfColsPerStage;
                    const uint32_t t_sfa_r = t_sfa_b + 4 * C::kAtoms;
                    const uint32_t t_sfb = t_sfa_r + 4 * C::kAtoms;
                    if constexpr (SPB) {
                        using P = SpStage;
                        const uint32_t a_bc = smem_u32(st + P::kBc);
                        const uint32_t a_r = smem_u32(st + (WIDE ? WS::kRs : P::kRs));
                        const uint32_t a_w = smem_u32(st + (WIDE ? WS::kW : P::kW));
                        const uint32_t t_meta = t_sfa_b + kScaleCols;
                        // backbone: two sparse MMAs of 128 logical K (32 stored
                        // bytes of A, 64 bytes of B per row; scale atom h holds
                        // their four scales per row; two metadata columns each)
#pragma unroll
                        for (int h = 0; h < 2; ++h)
                            tc_mma_sp_nvf4(d_b, sdesc_sw64(a_bc + 32 * h), sdesc_sw128(a_w + 64 * h),
                                           t_meta + 2 * h, with_n(P::kIdesc, TBN), t_sfa_b + 4 * h,
                                           t_sfb + kSfbAtomCols * h, (kb | h) ? 1u : 0u);
                        // residual: four dense MMAs of 64 K on the same weight tile
#pragma unroll
                        for (int j = 0; j < BK / 64; ++j) {
                            const uint32_t sf_id = (uint32_t)(j % C::kStepsPerAtom) * (4 / C::kStepsPerAtom);
                            mma<FMT, TBN>(d_r, sdesc_sw128(a_r + 32 * j), sdesc_sw128(a_w + 32 * j),
                                          t_sfa_r + 4 * (j / C::kStepsPerAtom),
                                          t_sfb + kSfbAtomCols * (j / C::kStepsPerAtom), 1u, sf_id);
                        }
                        tc_commit(&bars->empty[s]);
                        continue;
                    }
                    const uint32_t a_b = smem_u32(st), a_r = smem_u32(st + (WIDE ? WS::kRs : kTileBytes));
                    const uint32_t a_w = smem_u32(st + (WIDE ? WS::kW : 2 * kTileBytes));
#pragma unroll
                    for (int j = 0; j < BK / 64; ++j) {
                        const int at = j / C::kStepsPerAtom;
                        const uint32_t sf_id = (uint32_t)(j % C::kStepsPerAtom) * (4 / C::kStepsPerAtom);
                        const uint32_t col = 4 * at, colb = kSfbAtomCols * at;
                        const uint64_t db = sdesc_sw128(a_w + 32 * j);
                        const uint32_t acc = (kb | j) ? 1u : 0u;
                        mma<FMT, TBN>(d_b, sdesc_sw128(a_b + 32 * j), db, t_sfa_b + col, t_sfb + colb,
                                      acc, sf_id);
                        mma<FMT, TBN>(d_r, sdesc_sw128(a_r + 32 * j), db, t_sfa_r + col, t_sfb + colb,
                                      ONE ? 1u : acc, sf_id);
                    }
                    tc_commit(&bars->empty[s]);
                }
                tc_commit(&bars->acc_full[buf]);
            }
        }
    } else if (warp >= 6) {
        // Scale warps: warp w writes lane quarter w%4; lane l copies row l of
        // every 32-row x 16-byte scale atom of the stage into 4 columns.
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        uint32_t it = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
            for (int kb = 0; kb < nk; ++kb, ++it) {
                const uint32_t s = it % NST;
                if (!mbar_wait(&bars->sfl[s], (it / NST) & 1)) { ok = false; break; }
                const uint8_t* sf = smem + s * kStride + (WIDE ? WS::kSf : SPB ? SpStage::kSf : 3 * kTileBytes);
                const uint32_t tcol = tmem + kAccCols + s * kSfColsPerStage + lane_off;
                if constexpr (SPB) {
                    // pair indices: tensor-memory lane r holds row r's 16 bytes
                    // of the stage in K order (four columns)
                    const uint8_t* mt = smem + s * kStride + (WIDE ? WS::kMeta : SpStage::kMeta);
                    tmem_st_32x32b_x4(tcol + kScaleCols, ld_shared_v4(mt + 16 * ((warp & 3) * 32 + lane)));
                }
                if constexpr (WIDE) {
                    // the weight's 256 rows: per atom along K, the row block
                    // 0..127 then 128..255, 8 consecutive columns
                    uint4 v[2 * C::kAtoms];
#pragma unroll
                    for (int at = 0; at < C::kAtoms; ++at) {
                        v[2 * at] = ld_shared_v4(sf + 2 * C::kSfBytes + 512 * at + 16 * lane);
                        v[2 * at + 1] = ld_shared_v4(sf + 3 * C::kSfBytes + 512 * at + 16 * lane);
                    }
                    const uint32_t tb = tcol + 2 * 4 * C::kAtoms;
#pragma unroll
                    for (int h = 0; h < C::kAtoms / 2; ++h) {
                        const uint4 w4[4] = {v[4 * h], v[4 * h + 1], v[4 * h + 2], v[4 * h + 3]};
                        tmem_st_32x32b_x16(tb + 16 * h, w4);
                    }
                }
                // one store per operand: its kAtoms atoms are 4 * kAtoms
                // consecutive columns
#pragma unroll
                for (int o = 0; o < (WIDE ? 2 : 3); ++o) {
                    uint4 v[C::kAtoms];
#pragma unroll
                    for (int at = 0; at < C::kAtoms; ++at)
                        v[at] = ld_shared_v4(sf + o * C::kSfBytes + 512 * at + 16 * lane);
                    if constexpr (C::kAtoms == 4) tmem_st_32x32b_x16(tcol + o * 4 * C::kAtoms, v);
                    else                          tmem_st_32x32b_x8(tcol + o * 4 * C::kAtoms, v);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) { mbar_arrive(&bars->sf_full[s]); mbar_arrive(&bars->empty[s]); }
            }
        }
    } else {
        // Epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 = rows of the tile.
        const int q = warp & 3;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const float gbb = *ep.bb_tscale, grr = *ep.rs_tscale;
        uint32_t hmax = 0;      // SwiGLU: running max of |H| as two bf16 magnitudes
        uint32_t tc = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tc) {
            const TileInfo ti = sched_tile(sc, ssm, tile);
            const float gwv = ep.w_tscale[ti.e];
            const float gb = gbb * gwv, gr = grr * gwv;
            const int r_local = q * 32 + lane;
            const int64_t row = ti.y_row + r_local;
            const bool row_ok = r_local < ti.rows;
            const uint32_t buf = DBUF ? (tc & 1u) : 0u;
            const uint32_t use = DBUF ? (tc >> 1) : tc;
            const bool ok = mbar_wait(&bars->acc_full[buf], use & 1);
            tc_fence_after();
            if (!ok) break;
            const uint32_t src_b = ONE ? tmem + buf * BN : t_acc_b;
            const int64_t col0 = ti.col;
            if (!SW && ep.y_fp32) {
#pragma unroll 1
                for (int cc = 0; cc < TBN / 32; ++cc) {
                    uint32_t vb[32], vr[32];
                    tmem_ld_32x32b_x32(src_b + lane_off + cc * 32, vb);
                    if (!ONE) tmem_ld_32x32b_x32(t_acc_r + lane_off + cc * 32, vr);
                    tmem_ld_wait();
                    if (row_ok) {
                        float* y = static_cast<float*>(ep.Y) + row * ep.N + col0 + cc * 32;
#pragma unroll
                        for (int i = 0; i < 32; i += 4) {
                            float o[4];
#pragma unroll
                            for (int u = 0; u < 4; ++u)
                                o[u] = ONE ? gb * __uint_as_float(vb[i + u])
                                           : gb * __uint_as_float(vb[i + u]) + gr * __uint_as_float(vr[i + u]);
                            *reinterpret_cast<float4*>(y + i) = make_float4(o[0], o[1], o[2], o[3]);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->acc_empty[buf]);
            } else {
                // drain the accumulators into packed bf16x2 registers (64 for
                // Y, 32 for H), hand the tensor memory back, then store
                constexpr int kOutCols = SW ? BN / 2 : TBN;
                uint32_t out[kOutCols / 2];
                if constexpr (SW) {
                    // columns j and 64 + j of the tile: gate and up of feature j,
                    // 32 features at a time.  The tensor memory goes back after
                    // the second drain, so the next tile's MMAs run under the
                    // second half of the SwiGLU arithmetic; draining all 128
                    // values first would spill registers (slower on both the
                    // dense and the grouped launch).
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        float gv[32], uv[32];
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            uint32_t vb[32], vr[32];
                            const uint32_t c = half * (BN / 2) + cc * 32;
                            tmem_ld_32x32b_x32(src_b + lane_off + c, vb);
                            if (!ONE) tmem_ld_32x32b_x32(t_acc_r + lane_off + c, vr);
                            tmem_ld_wait();
                            float* dst = half ? uv : gv;
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                dst[i] = ONE ? gb * __uint_as_float(vb[i])
                                             : gb * __uint_as_float(vb[i]) + gr * __uint_as_float(vr[i]);
                        }
                        if (cc == 1) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&bars->acc_empty[buf]);
                        }
#pragma unroll
                        for (int h = 0; h < 16; ++h) {
                            const float h0 = __fmul_rn(silu_f32(gv[2 * h]), uv[2 * h]);
                            const float h1 = __fmul_rn(silu_f32(gv[2 * h + 1]), uv[2 * h + 1]);
                            __nv_bfloat162 p2 = __floats2bfloat162_rn(h0, h1);
                            const uint32_t bits = *reinterpret_cast<uint32_t*>(&p2);
                            out[cc * 16 + h] = bits;
                            if (row_ok) hmax = __vmaxu2(hmax, bits & 0x7FFF7FFFu);
                        }
                    }
                } else {
#pragma unroll
                    for (int cc = 0; cc < TBN / 32; ++cc) {
                        uint32_t vb[32], vr[32];
                        tmem_ld_32x32b_x32(src_b + lane_off + cc * 32, vb);
                        if (!ONE) tmem_ld_32x32b_x32(t_acc_r + lane_off + cc * 32, vr);
                        tmem_ld_wait();
#pragma unroll
                        for (int h = 0; h < 16; ++h) {
                            float lo = ONE ? gb * __uint_as_float(vb[2 * h])
                                           : gb * __uint_as_float(vb[2 * h]) + gr * __uint_as_float(vr[2 * h]);
                            float hi = ONE ? gb * __uint_as_float(vb[2 * h + 1])
                                           : gb * __uint_as_float(vb[2 * h + 1]) + gr * __uint_as_float(vr[2 * h + 1]);
                            __nv_bfloat162 p2 = __floats2bfloat162_rn(lo, hi);
                            out[cc * 16 + h] = *reinterpret_cast<uint32_t*>(&p2);
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->acc_empty[buf]);
                }
                // Stage the tile in shared memory so that every store
                // instruction writes whole 32-byte sectors of several rows
                // instead of 32 rows x 16 bytes.  Rows past ti.rows (the
                // matrix end, or the next expert's rows in the grouped form)
                // are not written.
                const int64_t wrow0 = ti.y_row + q * 32;
                __nv_bfloat16* yb = static_cast<__nv_bfloat16*>(ep.Y);
                const int64_t ldy = SW ? ep.N / 2 : ep.N;     // H has N/2 columns
                const int64_t ycol = SW ? col0 / 2 : col0;
                if (sc.grouped) {
                    // 32 rows x 16 columns at a time: 16 rows x 32 bytes per store
                    uint8_t* stg = ssm->g.stage[q];
#pragma unroll
                    for (int hc = 0; hc < kOutCols / 16; ++hc) {
#pragma unroll
                        for (int p = 0; p < 2; ++p)
                            *reinterpret_cast<uint4*>(stg + lane * 32 + 16 * (p ^ ((lane >> 2) & 1))) =
                                make_uint4(out[hc * 8 + 4 * p], out[hc * 8 + 4 * p + 1],
                                           out[hc * 8 + 4 * p + 2], out[hc * 8 + 4 * p + 3]);
                        __syncwarp();
#pragma unroll
                        for (int st = 0; st < 2; ++st) {
                            const int r = 16 * st + (lane >> 1), p = lane & 1;
                            const uint4 v = *reinterpret_cast<const uint4*>(stg + r * 32 + 16 * (p ^ ((r >> 2) & 1)));
                            if (q * 32 + r < ti.rows)
                                *reinterpret_cast<uint4*>(yb + (wrow0 + r) * ldy + ycol + hc * 16 + p * 8) = v;
                        }
                        __syncwarp();
                    }
                } else {
                    // 32 rows x 32 columns at a time: 8 rows x 64 bytes per store
                    uint8_t* stg = ssm->stage2[q];
#pragma unroll
                    for (int cc = 0; cc < kOutCols / 32; ++cc) {
#pragma unroll
                        for (int p = 0; p < 4; ++p)
                            *reinterpret_cast<uint4*>(stg + lane * 64 + 16 * (p ^ (lane & 3))) =
                                make_uint4(out[cc * 16 + 4 * p], out[cc * 16 + 4 * p + 1],
                                           out[cc * 16 + 4 * p + 2], out[cc * 16 + 4 * p + 3]);
                        __syncwarp();
#pragma unroll
                        for (int st8 = 0; st8 < 4; ++st8) {
                            const int r = 8 * st8 + (lane >> 2), p = lane & 3;
                            const uint4 v = *reinterpret_cast<const uint4*>(stg + r * 64 + 16 * (p ^ (r & 3)));
                            if (q * 32 + r < ti.rows)
                                *reinterpret_cast<uint4*>(yb + (wrow0 + r) * ldy + ycol + cc * 32 + p * 8) = v;
                        }
                        __syncwarp();
                    }
                }
            }
        }
        if (SW) {
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) hmax = __vmaxu2(hmax, __shfl_xor_sync(0xffffffffu, hmax, o));
            // the larger of the two bf16 magnitudes, as fp32 bits (non-negative
            // floats order as unsigned integers)
            const uint32_t m = max(hmax << 16, hmax & 0xFFFF0000u);
            if (lane == 0 && m) atomicMax(ep.amax, m);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, kTmemCols); }
}

// ------------------------------------------------------------------------
// Decode form (M <= 64 rows).  With few rows a 128-row activation tile is
// almost all padding and a 128 x 128 MMA spends most of its work on it.
// Here the operands swap roles: the weight tile (128 output columns) is the
// MMA's M side and the NT activation rows its N side, so every MMA does
// 128 x NT x 64 of useful work and the kernel streams the weight.  Both
// paths still share each weight tile (two MMAs, A = W, B = backbone or
// residual; the activation scale atoms serve as the B-side scales, whose
// first NT rows the MMA reads).  The accumulators hold Y^T; the epilogue
// writes them transposed.  Warp roles as in linear_kernel.
// When there are fewer output tiles than SMs, a cluster of `split` CTAs
// shares each tile, CTA rank r taking the r-th contiguous range of K
// steps; each drains its partial (already scaled by the tensor scales)
// into its shared memory and rank 0 sums the partials in rank order over
// distributed shared memory before storing Y.
// SwiGLU form (SW): with the interleaved gate+up weight, tensor-memory lanes
// 0..63 of a tile are the gate rows and lanes 64..127 the up rows of the
// same 64 features, i.e. epilogue warps 0-1 hold gates and 2-3 ups.  The
// gate warps leave their values in a shared-memory slot ([NT][64] fp32,
// two bounded mbarriers: full after the gate warps wrote it, empty after
// the up warps read it), and the up warps write H = silu(gate) * up and
// the running max |H|.
// ------------------------------------------------------------------------
template <int FMT, int NT>
struct DecCfg {
    using C = Cfg<FMT>;
    static constexpr uint32_t kActBytes = NT * (BK / 2);          // one activation tile
    static constexpr uint32_t kStageBytes = kTileBytes + 2 * kActBytes + 3 * C::kSfBytes;
    static constexpr uint32_t kStageStride = (kStageBytes + 1023) / 1024 * 1024;
    static constexpr int kStagesRaw = (200 * 1024) / (int)kStageStride;
    static constexpr int S = kStagesRaw > 8 ? 8 : kStagesRaw;
    static constexpr uint32_t kSfCols = 3 * 4 * C::kAtoms;         // per stage
    static constexpr uint32_t kAccCols = 4 * NT;                   // two buffers x two paths
    static_assert(kAccCols + S * kSfCols <= kTmemCols, "tensor memory budget");
    // E2M1 A and B, K-major, N = NT, M = 128 (see Cfg::kIdesc)
    static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(NT >> 3) << 17) |
                                       ((uint32_t)FMT << 23) | ((uint32_t)(BM >> 4) << 24);
};

template <int S>
struct alignas(8) DecBarriers {
    uint64_t full[S];
    uint64_t empty[S];        // MMAs done + scale warps done reading
    uint64_t sf_full[S];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t xg_full;         // SwiGLU: the gate warps wrote the gate values of a tile
    uint64_t xg_empty;        // SwiGLU: the up warps consumed them
    uint32_t tmem_base;
};

template <int FMT>
__device__ __forceinline__ void mma_id(uint32_t idesc0, uint32_t d, uint64_t a, uint64_t b,
                                       uint32_t sfa, uint32_t sfb, uint32_t acc, uint32_t sf_id) {
    const uint32_t idesc = idesc0 | (sf_id << 29) | (sf_id << 4);
    const uint32_t hi = sf_id << 30;
    if (FMT == 0) tc_mma_nvf4(d, a, b, idesc, sfa | hi, sfb | hi, acc);
    else          tc_mma_mxf4(d, a, b, idesc, sfa | hi, sfb | hi, acc);
}

template <int FMT, bool ONE, int NT, bool SW = false>
__global__ void __launch_bounds__(kThreads, 1)
decode_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_b,
              const __grid_constant__ CUtensorMap tm_r, const uint8_t* __restrict__ sf_w,
              const uint8_t* __restrict__ sf_b, const uint8_t* __restrict__ sf_r, int K,
              EpiArgs ep, int ntiles, int split) {
    using C = Cfg<FMT>;
    using D = DecCfg<FMT, NT>;
    constexpr int S = D::S;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    DecBarriers<S>* bars = reinterpret_cast<DecBarriers<S>*>(smem + S * D::kStageStride);
    // SwiGLU: gate values of one tile, [NT tokens][64 features], after the barriers
    float* xg = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(bars) + sizeof(DecBarriers<S>) + 15) & ~uintptr_t(15));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = K / BK;
    const int nsf = K / C::BS;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1 + 4);
            mbar_init(&bars->sf_full[s], 4);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->acc_full[b], 1);
            mbar_init(&bars->acc_empty[b], 4);
        }
        mbar_init(&bars->xg_full, 2);
        mbar_init(&bars->xg_empty, 2);
        fence_barrier_init();
    }
    if (warp == 1) { tmem_alloc(&bars->tmem_base, kTmemCols); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const uint32_t t_sf0 = tmem + D::kAccCols;
    // split > 1: one tile per cluster, this CTA's range of k-steps
    const int krank = split > 1 ? (int)cluster_ctarank() : 0;
    const int k0 = nk * krank / split, k1 = nk * (krank + 1) / split;
    const int tile0 = blockIdx.x / split, tstride = gridDim.x / split;
    float* partial = reinterpret_cast<float*>(smem);           // [NT][BM], stage memory reused

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tm_w); prefetch_tmap(&tm_b); prefetch_tmap(&tm_r);
            uint32_t it = 0;
            bool ok = true;
            for (int tile = tile0; tile < ntiles && ok; tile += tstride) {
                const uint8_t* gw = sf_w + (int64_t)tile * (nsf / 4) * 512;
                for (int kb = k0; kb < k1; ++kb, ++it) {
                    const uint32_t s = it % S;
                    if (it >= (uint32_t)S && !mbar_wait(&bars->empty[s], ((it / S) - 1) & 1)) { ok = false; break; }
                    uint8_t* st = smem + s * D::kStageStride;
                    mbar_arrive_expect_tx(&bars->full[s], D::kStageBytes);
                    tma_load_2d(st, &tm_w, &bars->full[s], kb * (BK / 2), tile * BM);
                    tma_load_2d(st + kTileBytes, &tm_b, &bars->full[s], kb * (BK / 2), 0);
                    tma_load_2d(st + kTileBytes + D::kActBytes, &tm_r, &bars->full[s], kb * (BK / 2), 0);
                    const int64_t sfo = (int64_t)kb * C::kAtoms * 512;
                    uint8_t* sfs = st + kTileBytes + 2 * D::kActBytes;
                    bulk_load(sfs, gw + sfo, C::kSfBytes, &bars->full[s]);
                    bulk_load(sfs + C::kSfBytes, sf_b + sfo, C::kSfBytes, &bars->full[s]);
                    bulk_load(sfs + 2 * C::kSfBytes, sf_r + sfo, C::kSfBytes, &bars->full[s]);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            uint32_t it = 0, tc = 0;
            bool ok = true;
            for (int tile = tile0; tile < ntiles && ok; tile += tstride, ++tc) {
                const uint32_t buf = tc & 1u, use = tc >> 1;
                if (use > 0 && !mbar_wait(&bars->acc_empty[buf], (use - 1) & 1)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_b = tmem + buf * 2 * NT;
                const uint32_t d_r = ONE ? d_b : d_b + NT;
                for (int kb = k0; kb < k1; ++kb, ++it) {
                    const uint32_t s = it % S;
                    if (!mbar_wait(&bars->full[s], (it / S) & 1)) { ok = false; break; }
                    if (!mbar_wait(&bars->sf_full[s], (it / S) & 1)) { ok = false; break; }
                    tc_fence_after();
                    uint8_t* st = smem + s * D::kStageStride;
                    const uint32_t a_w = smem_u32(st), a_b = smem_u32(st + kTileBytes);
                    const uint32_t a_r = smem_u32(st + kTileBytes + D::kActBytes);
                    const uint32_t t_sfw = t_sf0 + s * D::kSfCols;
                    const uint32_t t_sfb = t_sfw + 4 * C::kAtoms, t_sfr = t_sfb + 4 * C::kAtoms;
#pragma unroll
                    for (int j = 0; j < BK / 64; ++j) {
                        const int at = j / C::kStepsPerAtom;
                        const uint32_t sf_id = (uint32_t)(j % C::kStepsPerAtom) * (4 / C::kStepsPerAtom);
                        const uint32_t col = 4 * at;
                        const uint64_t dw = sdesc_sw128(a_w + 32 * j);
                        const uint32_t acc = (kb > k0 || j) ? 1u : 0u;
                        mma_id<FMT>(D::kIdesc, d_b, dw, sdesc_sw128(a_b + 32 * j), t_sfw + col, t_sfb + col,
                                    acc, sf_id);
                        mma_id<FMT>(D::kIdesc, d_r, dw, sdesc_sw128(a_r + 32 * j), t_sfw + col, t_sfr + col,
                                    ONE ? 1u : acc, sf_id);
                    }
                    tc_commit(&bars->empty[s]);
                }
                tc_commit(&bars->acc_full[buf]);
            }
        }
    } else if (warp >= 6) {
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        uint32_t it = 0;
        bool ok = true;
        for (int tile = tile0; tile < ntiles && ok; tile += tstride) {
            for (int kb = k0; kb < k1; ++kb, ++it) {
                const uint32_t s = it % S;
                if (!mbar_wait(&bars->full[s], (it / S) & 1)) { ok = false; break; }
                const uint8_t* sf = smem + s * D::kStageStride + kTileBytes + 2 * D::kActBytes;
                const uint32_t tcol = t_sf0 + s * D::kSfCols + lane_off;
#pragma unroll
                for (int o = 0; o < 3; ++o) {
                    uint4 v[C::kAtoms];
#pragma unroll
                    for (int at = 0; at < C::kAtoms; ++at)
                        v[at] = ld_shared_v4(sf + o * C::kSfBytes + 512 * at + 16 * lane);
                    if constexpr (C::kAtoms == 4) tmem_st_32x32b_x16(tcol + o * 4 * C::kAtoms, v);
                    else                          tmem_st_32x32b_x8(tcol + o * 4 * C::kAtoms, v);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) { mbar_arrive(&bars->sf_full[s]); mbar_arrive(&bars->empty[s]); }
            }
        }
    } else {
        // Epilogue: warp w reads TMEM lanes 32*(w%4).. = output columns of the
        // tile; each thread holds its column's NT rows.
        const int q = warp & 3;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const float gwv = ep.w_tscale[0];
        const float gb = *ep.bb_tscale * gwv, gr = *ep.rs_tscale * gwv;
        const int rows = (int)(ep.M < NT ? ep.M : NT);
        uint32_t tc = 0;
        uint32_t hmax = 0;
        for (int tile = tile0; tile < ntiles; tile += tstride, ++tc) {
            const uint32_t buf = tc & 1u, use = tc >> 1;
            const bool ok = mbar_wait(&bars->acc_full[buf], use & 1);
            tc_fence_after();
            if (!ok) break;
            if (SW && split == 1) {
                // lanes 0..63 of the tile hold gate rows (warps q = 0, 1), lanes
                // 64..127 the up rows of the same features (q = 2, 3)
                const uint32_t src = tmem + buf * 2 * NT + lane_off;
                float v[NT];
#pragma unroll
                for (int c0 = 0; c0 < NT; c0 += 16) {
                    uint32_t vb[16], vr[16];
                    tmem_ld_32x32b_x16(src + c0, vb);
                    if (!ONE) tmem_ld_32x32b_x16(src + NT + c0, vr);
                    tmem_ld_wait();
#pragma unroll
                    for (int t = 0; t < 16; ++t)
                        v[c0 + t] = ONE ? gb * __uint_as_float(vb[t])
                                        : gb * __uint_as_float(vb[t]) + gr * __uint_as_float(vr[t]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->acc_empty[buf]);
                const int j = (q & 1) * 32 + lane;              // feature within the tile
                bool good = true;
                if (q < 2) {
                    if (tc > 0) good = mbar_wait(&bars->xg_empty, (tc - 1) & 1);
                    if (good) {
#pragma unroll
                        for (int t = 0; t < NT; ++t) xg[t * 64 + j] = v[t];
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->xg_full);
                } else {
                    good = mbar_wait(&bars->xg_full, tc & 1);
                    if (good) {
                        const int64_t hcol = (int64_t)tile * (BM / 2) + j;
#pragma unroll
                        for (int t = 0; t < NT; ++t) {
                            if (t < rows) {
                                const float h = __fmul_rn(silu_f32(xg[t * 64 + j]), v[t]);
                                const __nv_bfloat16 hb = __float2bfloat16_rn(h);
                                static_cast<__nv_bfloat16*>(ep.Y)[(int64_t)t * (ep.N / 2) + hcol] = hb;
                                hmax = max(hmax, (uint32_t)(*reinterpret_cast<const uint16_t*>(&hb) & 0x7FFFu));
                            }
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->xg_empty);
                }
                if (!good) break;
                continue;
            }
            const uint32_t src_b = tmem + buf * 2 * NT + lane_off;
            const int64_t col = (int64_t)tile * BM + q * 32 + lane;
            const int jl = q * 32 + lane;                     // column within the tile
#pragma unroll
            for (int c0 = 0; c0 < NT; c0 += 16) {
                uint32_t vb[16], vr[16];
                tmem_ld_32x32b_x16(src_b + c0, vb);
                if (!ONE) tmem_ld_32x32b_x16(src_b + NT + c0, vr);
                tmem_ld_wait();
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    if (c0 + t < rows) {
                        const float y = ONE ? gb * __uint_as_float(vb[t])
                                            : gb * __uint_as_float(vb[t]) + gr * __uint_as_float(vr[t]);
                        if (split > 1) {
                            partial[(c0 + t) * BM + jl] = y;
                        } else {
                            const int64_t idx = (int64_t)(c0 + t) * ep.N + col;
                            if (ep.y_fp32) static_cast<float*>(ep.Y)[idx] = y;
                            else           static_cast<__nv_bfloat16*>(ep.Y)[idx] = __float2bfloat16_rn(y);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->acc_empty[buf]);
        }
        if (SW && split == 1 && q >= 2) {
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) hmax = max(hmax, __shfl_xor_sync(0xffffffffu, hmax, o));
            if (lane == 0 && hmax) atomicMax(ep.amax, hmax << 16);
        }
    }
    if (split > 1) {
        // every CTA's partial is in its shared memory; rank 0 adds them in
        // rank order and stores Y, then the peers may exit
        cluster_sync_all();
        if (SW && krank == 0 && warp >= 2 && warp < 6) {
            // gate warps sum their columns and leave them in xg, then the up
            // warps sum theirs and write H = silu(gate) * up
            const int q = warp & 3;
            const int jl = q * 32 + lane, j = (q & 1) * 32 + lane;
            const int rows = (int)(ep.M < NT ? ep.M : NT);
            bool good = true;
            if (q >= 2) good = mbar_wait(&bars->xg_full, 0);
            uint32_t hmax = 0;
            for (int t0 = 0; t0 < rows && good; t0 += 16) {
                float y[16], v[16];
#pragma unroll
                for (int t = 0; t < 16; ++t) y[t] = partial[(t0 + t) * BM + jl];
                for (int r = 1; r < split; ++r) {
#pragma unroll
                    for (int t = 0; t < 16; ++t) v[t] = ld_shared_cluster_f32(&partial[(t0 + t) * BM + jl], (uint32_t)r);
#pragma unroll
                    for (int t = 0; t < 16; ++t) y[t] += v[t];
                }
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    if (q < 2) {
                        xg[(t0 + t) * 64 + j] = y[t];
                    } else if (t0 + t < rows) {
                        const float h = __fmul_rn(silu_f32(xg[(t0 + t) * 64 + j]), y[t]);
                        const __nv_bfloat16 hb = __float2bfloat16_rn(h);
                        static_cast<__nv_bfloat16*>(ep.Y)[(int64_t)(t0 + t) * (ep.N / 2) + (int64_t)tile0 * (BM / 2) + j] = hb;
                        hmax = max(hmax, (uint32_t)(*reinterpret_cast<const uint16_t*>(&hb) & 0x7FFFu));
                    }
                }
            }
            __syncwarp();
            if (q < 2 && lane == 0) mbar_arrive(&bars->xg_full);
            if (q >= 2) {
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) hmax = max(hmax, __shfl_xor_sync(0xffffffffu, hmax, o));
                if (lane == 0 && hmax) atomicMax(ep.amax, hmax << 16);
            }
        } else if (krank == 0 && warp >= 2 && warp < 6) {
            const int jl = (warp & 3) * 32 + lane;
            const int64_t col = (int64_t)tile0 * BM + jl;
            const int rows = (int)(ep.M < NT ? ep.M : NT);
            for (int t0 = 0; t0 < rows; t0 += 16) {
                // 16 rows at a time: each rank's 16 loads are issued together
                float y[16], v[16];
#pragma unroll
                for (int t = 0; t < 16; ++t) y[t] = partial[(t0 + t) * BM + jl];
                for (int r = 1; r < split; ++r) {
#pragma unroll
                    for (int t = 0; t < 16; ++t) v[t] = ld_shared_cluster_f32(&partial[(t0 + t) * BM + jl], (uint32_t)r);
#pragma unroll
                    for (int t = 0; t < 16; ++t) y[t] += v[t];
                }
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    if (t0 + t < rows) {
                        const int64_t idx = (int64_t)(t0 + t) * ep.N + col;
                        if (ep.y_fp32) static_cast<float*>(ep.Y)[idx] = y[t];
                        else           static_cast<__nv_bfloat16*>(ep.Y)[idx] = __float2bfloat16_rn(y[t]);
                    }
                }
            }
        }
        cluster_sync_all();
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

// Looked up once (thread-safe static initialisation).
EncodeTiledFn encode_fn() {
    static const EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(p);
        return static_cast<EncodeTiledFn>(nullptr);
    }();
    return fn;
}

// Per-device "attribute already set" flags; setting an attribute twice is
// harmless, so concurrent first calls only need the flag itself to be atomic.
template <class Fn>
cudaError_t set_smem_once(std::atomic<bool> (&done)[64], Fn kernel, size_t bytes) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess && dev < 64) done[dev].store(true, std::memory_order_release);
    return e;
}

// 2-D uint8 map over a [rows, row_bytes] code matrix, box box_bytes x
// box_rows with the swizzle of that row length (128 bytes: 128-byte
// swizzle; 64 bytes: 64-byte swizzle); rows past the end read as zero.
bool make_code_map(CUtensorMap* m, const void* base, int64_t rows, int64_t row_bytes, int box_rows,
                   int box_bytes = 128) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {(cuuint32_t)box_bytes, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE,
              box_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int FMT, bool SPB = false, bool WIDE = false>
size_t linear_smem_bytes() {
    const size_t stride = WIDE ? WideStage<FMT, SPB>::kStride : SPB ? SpStage::kStride : Cfg<FMT>::kStageStride;
    return (WIDE ? kStagesW : kStages) * stride + sizeof(Barriers) + 128 + sizeof(SchedSmem) + 1024;
}

template <int FMT, bool ONE, bool SW, bool SPB = false, bool WIDE = false>
cudaError_t ensure_smem_attr() {
    static std::atomic<bool> done[64];
    return set_smem_once(done, linear_kernel<FMT, ONE, SW, SPB, WIDE>, linear_smem_bytes<FMT, SPB, WIDE>());
}

// A_rows: rows of the activation operands (gathered and padded for the
// grouped form); W_rows: rows of the (stacked) weight.
template <int FMT, bool ONE, bool SW, bool SPB = false, bool WIDE = false>
cudaError_t launch_gemm_t(const void* bb_codes, const void* bb_scales, const void* rs_codes,
                        const void* rs_scales, int64_t A_rows, const LinearLaunch& p, int64_t W_rows,
                        const Sched& sc, int max_tiles, cudaStream_t s, int sms) {
    CUtensorMap tb, tr, tw;
    // the compressed backbone has K/4 bytes a row: 64 bytes a k-step
    if (!make_code_map(&tb, bb_codes, A_rows, SPB ? p.K / 4 : p.K / 2, BM, SPB ? 64 : 128) ||
        !make_code_map(&tr, rs_codes, A_rows, p.K / 2, BM) ||
        !make_code_map(&tw, p.w_codes, W_rows, p.K / 2, WIDE ? BNW : BN))
        return cudaErrorInvalidValue;
    cudaError_t e = ensure_smem_attr<FMT, ONE, SW, SPB, WIDE>();
    if (e != cudaSuccess) return e;
    EpiArgs ep{p.bb_tscale, p.rs_tscale, p.w_tscale, p.Y, p.M, p.N, p.y_fp32,
               reinterpret_cast<uint32_t*>(p.amax)};
    if (SW) {
        e = cudaMemsetAsync(p.amax, 0, sizeof(float), s);
        if (e != cudaSuccess) return e;
    }
    const int grid = std::max(1, std::min(max_tiles, std::max(1, sms)));
    linear_kernel<FMT, ONE, SW, SPB, WIDE><<<grid, kThreads, linear_smem_bytes<FMT, SPB, WIDE>(), s>>>(
        tb, tr, tw, static_cast<const uint8_t*>(bb_scales), static_cast<const uint8_t*>(rs_scales),
        static_cast<const uint8_t*>(p.w_scales), static_cast<const uint8_t*>(p.bb_meta), p.K, ep, sc);
    return cudaGetLastError();
}

template <int FMT>
cudaError_t launch_gemm(const void* bb_codes, const void* bb_scales, const void* rs_codes,
                        const void* rs_scales, int64_t A_rows, const LinearLaunch& p, int64_t W_rows,
                        const Sched& sc, int max_tiles, cudaStream_t s, int sms) {
    if (p.swiglu)
        return p.one_acc ? launch_gemm_t<FMT, true, true>(bb_codes, bb_scales, rs_codes, rs_scales, A_rows,
                                                          p, W_rows, sc, max_tiles, s, sms)
                         : launch_gemm_t<FMT, false, true>(bb_codes, bb_scales, rs_codes, rs_scales, A_rows,
                                                           p, W_rows, sc, max_tiles, s, sms);
    return p.one_acc ? launch_gemm_t<FMT, true, false>(bb_codes, bb_scales, rs_codes, rs_scales, A_rows, p,
                                                      W_rows, sc, max_tiles, s, sms)
                     : launch_gemm_t<FMT, false, false>(bb_codes, bb_scales, rs_codes, rs_scales, A_rows, p,
                                                       W_rows, sc, max_tiles, s, sms);
}

template <int FMT, bool ONE, int NT, bool SW = false>
cudaError_t launch_decode_t(const LinearLaunch& p, cudaStream_t s, int sms) {
    using D = DecCfg<FMT, NT>;
    CUtensorMap tb, tr, tw;
    if (!make_code_map(&tw, p.w_codes, p.N, p.K / 2, BM) ||
        !make_code_map(&tb, p.bb_codes, p.M, p.K / 2, NT) ||
        !make_code_map(&tr, p.rs_codes, p.M, p.K / 2, NT))
        return cudaErrorInvalidValue;
    const size_t smem = D::S * D::kStageStride + sizeof(DecBarriers<D::S>) + 16 + (SW ? NT * 64 * 4 : 0) + 1024;
    static std::atomic<bool> done[64];
    if (cudaError_t e = set_smem_once(done, decode_kernel<FMT, ONE, NT, SW>, smem); e != cudaSuccess) return e;
    EpiArgs ep{p.bb_tscale, p.rs_tscale, p.w_tscale, p.Y, p.M, p.N, p.y_fp32, reinterpret_cast<uint32_t*>(p.amax)};
    if (SW) {
        cudaError_t e = cudaMemsetAsync(p.amax, 0, sizeof(float), s);
        if (e != cudaSuccess) return e;
    }
    const int ntiles = p.N / BN;
    const int nk = p.K / BK;
    // fewer tiles than SMs: clusters of `split` CTAs share a tile along K,
    // each keeping at least 8 k-steps (shorter ranges do not pay for the
    // cluster's setup and reduction)
    int split = std::max(1, std::min(std::min(8, nk / 8), std::max(1, sms) / ntiles));
    const int grid = split > 1 ? ntiles * split : std::max(1, std::min(ntiles, std::max(1, sms)));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = split > 1 ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, decode_kernel<FMT, ONE, NT, SW>, tw, tb, tr,
                              static_cast<const uint8_t*>(p.w_scales),
                              static_cast<const uint8_t*>(p.bb_scales),
                              static_cast<const uint8_t*>(p.rs_scales), p.K, ep, ntiles, split);
}

template <int FMT, int NT>
cudaError_t launch_decode_nt(const LinearLaunch& p, cudaStream_t s, int sms) {
    if (p.swiglu)
        return p.one_acc ? launch_decode_t<FMT, true, NT, true>(p, s, sms)
                         : launch_decode_t<FMT, false, NT, true>(p, s, sms);
    return p.one_acc ? launch_decode_t<FMT, true, NT>(p, s, sms) : launch_decode_t<FMT, false, NT>(p, s, sms);
}

// Plain tile walk: n fastest when the activation operands (both paths'
// codes and scales) outweigh the weight's, so the smaller operand is the
// L2-resident one.
inline int walk_n_fast(const LinearLaunch& p) {
    const double sfb = p.fmt == 0 ? 1.0 / 16 : 1.0 / 32;
    const double a_bytes = (double)p.M * p.K * 2.0 * (0.5 + sfb);
    const double w_bytes = (double)p.N * p.K * (0.5 + sfb);
    return a_bytes > w_bytes ? 1 : 0;
}

// The 256-wide tile (one accumulator only) moves a third fewer operand and
// scale bytes per unit of MMA work, but has one accumulator buffer and half
// as many tiles: it is taken where its last wave over the SMs is not much
// emptier than the 128-wide tile's.
inline bool use_wide(const LinearLaunch& p, int sms) {
    if (!p.one_acc || p.swiglu || p.N % BNW != 0) return false;
    const int64_t g = std::max(1, sms);
    const int64_t mt = (p.M + BM - 1) / BM;
    auto fill = [g](int64_t tiles) { return (double)tiles / (double)(((tiles + g - 1) / g) * g); };
    return fill(mt * (p.N / BNW)) * 1.1 >= fill(mt * (p.N / BN));
}

inline Sched plain_sched(const LinearLaunch& p, int bn, int nsf) {
    Sched sc{};
    sc.mt_count = (int)((p.M + BM - 1) / BM);
    sc.nt_count = p.N / bn;
    sc.M = p.M;
    sc.nsf = nsf;
    sc.grouped = 0;
    sc.N = p.N;
    sc.n_fast = walk_n_fast(p);
    sc.bn = bn;
    return sc;
}

template <int FMT>
cudaError_t launch_linear_t(const LinearLaunch& p, cudaStream_t s, int sms) {
    const int nsf = p.K / Cfg<FMT>::BS;
    if (p.bb_meta) {
        // compressed pair-granular backbone: the row-tiled kernel with the
        // sparse MMA (the swapped decode form would need the backbone as B)
        if (FMT != 1 || !p.one_acc || p.swiglu) return cudaErrorNotSupported;
        if (use_wide(p, sms)) {
            const Sched sc = plain_sched(p, BNW, nsf);
            return launch_gemm_t<1, true, false, true, true>(p.bb_codes, p.bb_scales, p.rs_codes, p.rs_scales,
                                                             p.M, p, p.N, sc, sc.mt_count * sc.nt_count, s, sms);
        }
        const Sched sc = plain_sched(p, BN, nsf);
        return launch_gemm_t<1, true, false, true>(p.bb_codes, p.bb_scales, p.rs_codes, p.rs_scales, p.M, p,
                                                   p.N, sc, sc.mt_count * sc.nt_count, s, sms);
    }
    // few rows: the swapped (weight-streaming) form
    if (p.M <= 16) return launch_decode_nt<FMT, 16>(p, s, sms);
    if (p.M <= 32) return launch_decode_nt<FMT, 32>(p, s, sms);
    if (p.M <= 64) return launch_decode_nt<FMT, 64>(p, s, sms);
    if (use_wide(p, sms)) {
        const Sched sc = plain_sched(p, BNW, nsf);
        return launch_gemm_t<FMT, true, false, false, true>(p.bb_codes, p.bb_scales, p.rs_codes, p.rs_scales,
                                                            p.M, p, p.N, sc, sc.mt_count * sc.nt_count, s, sms);
    }
    const Sched sc = plain_sched(p, BN, nsf);
    return launch_gemm<FMT>(p.bb_codes, p.bb_scales, p.rs_codes, p.rs_scales, p.M, p, p.N, sc,
                            sc.mt_count * sc.nt_count, s, sms);
}

// ------------------------------------------------------------ grouped ----
// Gather: dispatched row t of expert e (offsets[e] <= t < offsets[e+1])
// reads prepared row row_index[t] (or t) and is written to padded row
// poff[e] + (t - offsets[e]) of the workspace operands: both code rows and
// both rows of scale atoms (4-byte words of four scales).
template <int FMT>
__global__ void __launch_bounds__(256)
moe_gather_kernel(const uint8_t* __restrict__ bb_codes, const uint8_t* __restrict__ bb_scales,
                  const uint8_t* __restrict__ rs_codes, const uint8_t* __restrict__ rs_scales,
                  const int32_t* __restrict__ row_index, Sched sc, int K, int64_t T,
                  uint8_t* __restrict__ gb_codes, uint8_t* __restrict__ gb_scales,
                  uint8_t* __restrict__ gr_codes, uint8_t* __restrict__ gr_scales) {
    __shared__ SchedSmem ssm;
    sched_prepare(sc, &ssm);
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * 8;
    const int row_bytes = K / 2;
    const int words = sc.nsf / 4;
    for (int64_t t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); t < T; t += warps) {
        int lo = 0, hi = sc.E;                      // expert of row t
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (ssm.g.t.off[mid] <= t) lo = mid; else hi = mid;
        }
        const int64_t src = row_index ? (int64_t)row_index[t] : t;
        const int64_t dst = ssm.g.t.poff[lo] + (t - ssm.g.t.off[lo]);
        const uint4* sb = reinterpret_cast<const uint4*>(bb_codes + src * row_bytes);
        const uint4* sr = reinterpret_cast<const uint4*>(rs_codes + src * row_bytes);
        uint4* db = reinterpret_cast<uint4*>(gb_codes + dst * row_bytes);
        uint4* dr = reinterpret_cast<uint4*>(gr_codes + dst * row_bytes);
        for (int i = lane; i < row_bytes / 16; i += 32) { db[i] = sb[i]; dr[i] = sr[i]; }
        const int64_t so = (src >> 7) * words * 512 + (src & 31) * 16 + ((src >> 5) & 3) * 4;
        const int64_t d0 = (dst >> 7) * words * 512 + (dst & 31) * 16 + ((dst >> 5) & 3) * 4;
        for (int w = lane; w < words; w += 32) {
            *reinterpret_cast<uint32_t*>(gb_scales + d0 + w * 512) =
                *reinterpret_cast<const uint32_t*>(bb_scales + so + w * 512);
            *reinterpret_cast<uint32_t*>(gr_scales + d0 + w * 512) =
                *reinterpret_cast<const uint32_t*>(rs_scales + so + w * 512);
        }
    }
}

template <int FMT>
cudaError_t launch_moe_t(const LinearLaunch& p, cudaStream_t s, int sms) {
    constexpr int BS = Cfg<FMT>::BS;
    const int nsf = p.K / BS;
    const int64_t rows_max = moe_padded_rows(p.T, p.E);
    uint8_t* ws = static_cast<uint8_t*>(p.ws);
    uint8_t* gb_codes = ws;
    uint8_t* gr_codes = gb_codes + rows_max * (p.K / 2);
    uint8_t* gb_scales = gr_codes + rows_max * (p.K / 2);
    uint8_t* gr_scales = gb_scales + rows_max * nsf;
    Sched sc{};
    sc.nt_count = p.N / BN;
    sc.M = p.T;
    sc.nsf = nsf;
    sc.grouped = 1;
    sc.offsets = p.offsets;
    sc.E = p.E;
    sc.w_sf_stride = (int64_t)((p.N + 127) / 128 * 128) * nsf;
    sc.N = p.N;
    if (p.T > 0) {
        const int gblocks = (int)std::min<int64_t>((p.T + 7) / 8, (int64_t)sms * 8);
        moe_gather_kernel<FMT><<<std::max(1, gblocks), 256, 0, s>>>(
            static_cast<const uint8_t*>(p.bb_codes), static_cast<const uint8_t*>(p.bb_scales),
            static_cast<const uint8_t*>(p.rs_codes), static_cast<const uint8_t*>(p.rs_scales),
            p.row_index, sc, p.K, p.T, gb_codes, gb_scales, gr_codes, gr_scales);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const int max_tiles = (int)((p.T + 127) / 128 + p.E) * sc.nt_count;
    LinearLaunch q = p;
    q.M = p.T;
    return launch_gemm<FMT>(gb_codes, gb_scales, gr_codes, gr_scales, rows_max, q,
                            (int64_t)p.E * p.N, sc, max_tiles, s, sms);
}

}  // namespace

unsigned take_status_linear() { return take_tu_status(); }

cudaError_t launch_linear(const LinearLaunch& p, cudaStream_t s, int sms) {
    if (p.M == 0) return cudaSuccess;
    return p.fmt == 0 ? launch_linear_t<0>(p, s, sms) : launch_linear_t<1>(p, s, sms);
}

cudaError_t launch_moe_linear(const LinearLaunch& p, cudaStream_t s, int sms) {
    if (p.E > kMaxExperts) return cudaErrorNotSupported;
    return p.fmt == 0 ? launch_moe_t<0>(p, s, sms) : launch_moe_t<1>(p, s, sms);
}

size_t moe_ws_bytes(int64_t T, int E, int K, int fmt) {
    const int nsf = K / (fmt == 0 ? 16 : 32);
    return (size_t)moe_padded_rows(T, E) * (size_t)(K + 2 * nsf);
}

}  // namespace sharq
