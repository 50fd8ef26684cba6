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
// With the residual's own tensor scale, phase 1 also takes P, the largest
// |y| the mask prunes (the residual of a pruned entry is y itself, so
// A_r >= P), and phase 2 already quantises the residual against P; when
// the residual's maximum turns out to be P exactly, those are the final
// codes and phase 3 is skipped.
// One persistent cooperative launch runs the three phases.  In phase 1 each
// warp owns whole rows, lane l reading the 16-byte chunks l, l+32, ... of a
// row, which is also the fixed fp32 reduction order of the RMS sum; without
// a norm, phase 1 is a plain maximum over the whole tensor, spread over every
// lane.  Phases 2 and 3 give each lane whole scale blocks.  MXFP4 has no
// tensor scale, so its backbone and residual are produced in one pass (after
// the RMS barrier when there is a norm).  When the producer of X has already
// taken A_b = max |X| (a no-norm input, e.g. the SwiGLU epilogue of the
// gate+up linear), phase 1 and its barrier are skipped: with the shared
// residual scale the whole prepare is then one barrier-free pass.
//
// Every floating-point step is one correctly rounded fp32 operation, so the
// codes and scales are bit-identical to a plain sequential CPU evaluation.
// The multiplications run as packed pairs (__fmul2_rn: per component the
// same rounding as __fmul_rn) on the FMA pipe; additions and subtractions
// stay scalar (a packed add after a packed multiply can be fused into one
// rounding).  The integer and compare pipe, which bounds this kernel, is
// kept for the mask, the maxima and the packing.  gamma (and beta) are converted to fp32
// once per CTA into shared memory.
#include "common.cuh"
#include "sharq_internal.h"

#include <cuda_fp16.h>

#include <atomic>

namespace sharq {

unsigned take_status_prepare() { return take_tu_status(); }

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
// gamma / beta are staged in shared memory as fp32 up to this many bytes
// (two CTAs per SM still fit); longer rows read them from global memory.
constexpr int kMaxStagedBytes = 96 * 1024;
// MXFP4 RMSNorm rows of up to 32 * kRowChunks 16-byte chunks (K <= 4096)
// are loaded into registers whole in phase 1.
constexpr int kRowChunks = 16;

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
    uint32_t* ws;            // [0] amax_b bits, [1] amax_r bits, [2] barrier, [5] phase-2 guess
                             // failed, [6] max pruned |y| bits; from word 16: rinv[M], mu[M]
    const float* amax_in;    // GIVEN: A_b = max |X| from the producer
    uint8_t* bb_meta;        // PAIRS: pair metadata atoms (bb_codes then holds the kept pairs)
    int staged;              // gamma (and beta) are in shared memory as fp32
    int spec;                // NVFP4 own residual scale: quantise the residual in phase 2 against
                             // the largest pruned |y| (see phase 2)
    unsigned long long wait_ns;   // limit of each grid-barrier wait
    int skip_block;          // self-test only: this block never arrives at a barrier (-1: none)
};

__device__ __forceinline__ float* ws_rinv(uint32_t* ws) {
    return reinterpret_cast<float*>(ws + 16);
}

// Byte offset of scale (row, s) in the MMA-ready atom layout.
__device__ __forceinline__ int64_t sf_off(int64_t row, int s, int nsf) {
    return ((row >> 7) * (int64_t)(nsf >> 2) + (s >> 2)) * 512 + (row & 31) * 16 +
           ((row >> 5) & 3) * 4 + (s & 3);
}

// Two bf16 (low half = first element) -> two exact fp32.
__device__ __forceinline__ float2 bf16x2_f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float2 x[4]) {
    x[0] = bf16x2_f2(v.x); x[1] = bf16x2_f2(v.y); x[2] = bf16x2_f2(v.z); x[3] = bf16x2_f2(v.w);
}

__device__ __forceinline__ float2 f2(float v) { return make_float2(v, v); }

// Packed pair multiply: per component one correctly rounded fp32 product,
// the same bits as __fmul_rn.  There is no packed addition here on purpose:
// a packed add that consumes a packed product may be fused with it into one
// fused multiply-add (a single rounding) even when both are written with an
// explicit rounding mode, which changes the residual's bits.  Every addition
// and subtraction below is a scalar __fadd_rn / __fsub_rn, which is never
// fused.
__device__ __forceinline__ float2 mul2_rn(float2 a, float2 b) { return __fmul2_rn(a, b); }

// fl(a - b) per component (scalar, never fused).
__device__ __forceinline__ float2 sub2_rn(float2 a, float2 b) {
    return make_float2(__fsub_rn(a.x, b.x), __fsub_rn(a.y, b.y));
}

// fl(a + b) per component (scalar, never fused).
__device__ __forceinline__ float2 add2_rn(float2 a, float2 b) {
    return make_float2(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y));
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

__device__ __forceinline__ float max3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// max |v| over N >= 3 values, three at a time.
template <int N>
__device__ __forceinline__ float amax_n(const float* v) {
    float m = max3f(fabsf(v[0]), fabsf(v[1]), fabsf(v[2]));
#pragma unroll
    for (int i = 3; i + 1 < N; i += 2) m = max3f(m, fabsf(v[i]), fabsf(v[i + 1]));
    if ((N - 3) % 2) m = fmaxf(m, fabsf(v[N - 1]));
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

// Eight packed E2M1 codes -> four exact half2 pairs (element 2p low).
__device__ __forceinline__ void e2m1x8_to_h2(uint32_t codes, __half2 h[4]) {
    uint32_t r[4];
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(codes));
#pragma unroll
    for (int p = 0; p < 4; ++p) h[p] = *reinterpret_cast<__half2*>(&r[p]);
}

// An E4M3 scale code -> its exact value as f16 in both halves.
__device__ __forceinline__ __half2 e4m3_h2(uint32_t code) {
    uint32_t r;
    const uint16_t two = (uint16_t)(code | (code << 8));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(two));
    return *reinterpret_cast<__half2*>(&r);
}

// Dequantised values of 8 packed NVFP4 codes: fl(fl(val * e) * G).  val * e
// is exact in f16 (at least 0.5 * 2^-9 = 2^-10, a normal half, and at most
// 6 * 448, with at most 6 significant bits), so the only rounding is that of
// the multiplication by the tensor scale, as in the definition.
__device__ __forceinline__ void dequant8_nv(uint32_t codes, __half2 e2, float2 g, float2 d[4]) {
    __half2 h[4];
    e2m1x8_to_h2(codes, h);
#pragma unroll
    for (int p = 0; p < 4; ++p) d[p] = mul2_rn(__half22float2(__hmul2(h[p], e2)), g);
}

// Dequantised values of 8 packed MXFP4 codes: fl(val * 2^(c-127)).
__device__ __forceinline__ void dequant8_mx(uint32_t codes, float2 sc, float2 d[4]) {
    __half2 h[4];
    e2m1x8_to_h2(codes, h);
#pragma unroll
    for (int p = 0; p < 4; ++p) d[p] = mul2_rn(__half22float2(h[p]), sc);
}

// E2M1 codes of 8 values (pairs), element 2p in the low nibble of byte p.
__device__ __forceinline__ uint32_t cvt_e2m1x8_f2(const float2 v[4]) {
    return cvt_e2m1x8(reinterpret_cast<const float*>(v));
}

// Keep bits of 8 elements (bit t = element t) -> 0xF in nibble t: the AND
// mask that clears the codes of pruned elements (code 0x0, +0).
__device__ __forceinline__ uint32_t nibble_mask8(uint32_t k) {
    uint32_t x = k & 0xFFu;
    x = (x | (x << 12)) & 0x000F000Fu;
    x = (x | (x << 6)) & 0x03030303u;
    x = (x | (x << 3)) & 0x11111111u;
    return x * 0xFu;
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
// Work distribution of phases 2 and 3 over the flattened [M, K/E] scale
// blocks: lane l of global warp w starts at block 32w + l and steps by the
// number of lanes in the grid, so a warp's 32 blocks are always 32 * E
// consecutive elements (coalesced loads, one 8- or 16-byte code store per
// lane).  REV walks the same sequence from the far end of X: phase 2 starts
// on the rows phase 1 read last, which are still in L2 when X is larger
// than L2, and phase 3 (forwards) starts on the rows phase 2 read last.
// (Measured alternatives, slower: each warp taking runs of 512 consecutive
// blocks, and runs handed out from one atomic counter -- one counter
// serialises at about 10^8 atomics per second.)
template <bool REV>
struct BlockCursor {
    int64_t row;           // this lane's block (only meaningful while valid())
    int cb, nbr, dr, dc;
    int i;                 // steps taken (the same in every lane)
    int64_t sfo;           // byte offset of the block's scale, sf_off(row, cb, nbr)
    int64_t wpos, wstride, total, nrows;
    __device__ __forceinline__ void init(int64_t gw, int64_t nw, int64_t tot, int nb_row, int lane) {
        nbr = nb_row; i = 0; total = tot; nrows = tot / nb_row;
        wpos = gw * 32;                       // lane 0's position in the walk
        wstride = nw * 32;
        const int64_t j = wpos + lane;
        const int64_t b = REV ? tot - 1 - j : j;
        row = b >= 0 ? b / nb_row : -1;
        cb = (int)(b - row * nb_row);
        dr = (int)(wstride / nb_row);
        dc = (int)(wstride - (int64_t)dr * nb_row);
        sfo = sf_off(row, cb, nb_row);
    }
    __device__ __forceinline__ bool live() const { return wpos < total; }   // the same in every lane
    __device__ __forceinline__ bool valid() const { return row >= 0 && row < nrows; }
    __device__ __forceinline__ void next() {
        ++i;
        wpos += wstride;
        if (REV) { cb -= dc; row -= dr; if (cb < 0) { cb += nbr; --row; } }
        else     { cb += dc; row += dr; if (cb >= nbr) { cb -= nbr; ++row; } }
        sfo = sf_off(row, cb, nbr);
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

template <uint32_t LUT>
__device__ __forceinline__ uint32_t lop3t(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, %4;" : "=r"(d) : "r"(a), "r"(b), "r"(c), "n"(LUT));
    return d;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// The 2-of-4 mask of 8 elements as the AND mask of their packed codes (0xF
// in nibble t when element t is kept).  Each comparison |a| >= |b| is the
// sign of the exact difference fl(|a| - |b|) (no rounding can turn a
// nonzero difference into zero or flip its sign; equal magnitudes give +0),
// taken on the FMA pipe; the four keep decisions of a group are majority
// functions of three such signs, one lop3 each (element i is kept when it
// beats at least two of the other three; a tie goes to the lower index):
//   k0 = maj(a0>=a1, a0>=a2, a0>=a3)   k1 = maj(a1>a0, a1>=a2, a1>=a3)
//   k2 = maj(a2>a0, a2>a1, a2>=a3)     k3 = maj(a3>a0, a3>a1, a3>a2).
// The keep bit is bit 31 of k_i; byte permutes with sign replication turn
// those bits into byte masks, and one lop3 merges the even and odd elements
// into nibbles.
__device__ __forceinline__ uint32_t keep24_nibbles8(const float* y) {
    uint32_t k[8];
#pragma unroll
    for (int g = 0; g < 8; g += 4) {
        const float a0 = fabsf(y[g]), a1 = fabsf(y[g + 1]), a2 = fabsf(y[g + 2]), a3 = fabsf(y[g + 3]);
        const uint32_t d01 = __float_as_uint(__fsub_rn(a0, a1)), d02 = __float_as_uint(__fsub_rn(a0, a2));
        const uint32_t d03 = __float_as_uint(__fsub_rn(a0, a3)), d12 = __float_as_uint(__fsub_rn(a1, a2));
        const uint32_t d13 = __float_as_uint(__fsub_rn(a1, a3)), d23 = __float_as_uint(__fsub_rn(a2, a3));
        // sign bit set = the first operand is smaller
        k[g] = lop3t<0x17>(d01, d02, d03);        // maj(~s01, ~s02, ~s03)
        k[g + 1] = lop3t<0x71>(d01, d12, d13);    // maj(s01, ~s12, ~s13)
        k[g + 2] = lop3t<0xD4>(d02, d12, d23);    // maj(s02, s12, ~s23)
        k[g + 3] = lop3t<0xE8>(d03, d13, d23);    // maj(s03, s13, s23)
    }
    // sign-replicated byte 3 of each word: 0xFF when kept
    const uint32_t e01 = prmt(k[0], k[2], 0x00FBu), e23 = prmt(k[4], k[6], 0xFB00u);
    const uint32_t o01 = prmt(k[1], k[3], 0x00FBu), o23 = prmt(k[5], k[7], 0xFB00u);
    const uint32_t ev = prmt(e01, e23, 0x7610u), od = prmt(o01, o23, 0x7610u);
    return lop3t<0xE4>(ev, od, 0x0F0F0F0Fu);      // (ev & 0x0F..) | (od & 0xF0..)
}

// The pair-granular 4:8 mask of 8 elements: the two of the four aligned
// pairs with the largest pair magnitude max(|y_2i|, |y_2i+1|), ties to the
// lower pair index (the same majority functions as keep24_nibbles8, on the
// pair magnitudes).  Returns the code AND mask (0xFF in byte i, the codes
// of pair i, when it is kept) and in *nib the metadata nibble: the lower
// kept pair's index in bits 1:0, the higher one's in bits 3:2.
__device__ __forceinline__ uint32_t keep_pairs_bytes8(const float* y, uint32_t* nib) {
    const float a0 = fmaxf(fabsf(y[0]), fabsf(y[1])), a1 = fmaxf(fabsf(y[2]), fabsf(y[3]));
    const float a2 = fmaxf(fabsf(y[4]), fabsf(y[5])), a3 = fmaxf(fabsf(y[6]), fabsf(y[7]));
    const uint32_t d01 = __float_as_uint(__fsub_rn(a0, a1)), d02 = __float_as_uint(__fsub_rn(a0, a2));
    const uint32_t d03 = __float_as_uint(__fsub_rn(a0, a3)), d12 = __float_as_uint(__fsub_rn(a1, a2));
    const uint32_t d13 = __float_as_uint(__fsub_rn(a1, a3)), d23 = __float_as_uint(__fsub_rn(a2, a3));
    const uint32_t k0 = lop3t<0x17>(d01, d02, d03), k1 = lop3t<0x71>(d01, d12, d13);
    const uint32_t k2 = lop3t<0xD4>(d02, d12, d23), k3 = lop3t<0xE8>(d03, d13, d23);
    const uint32_t m = prmt(prmt(k0, k1, 0x00FBu), prmt(k2, k3, 0xFB00u), 0x7610u);
    // the four keep bits (bit i = pair i), then the nibble of the two kept
    // indices: 0b0011 -> 0x4, 0b0101 -> 0x8, 0b0110 -> 0x9, 0b1001 -> 0xC,
    // 0b1010 -> 0xD, 0b1100 -> 0xE
    const uint32_t k4 = ((m & 0x01010101u) * 0x01020408u) >> 24;
    constexpr unsigned long long kLut = (0x4ull << 12) | (0x8ull << 20) | (0x9ull << 24) |
                                        (0xCull << 36) | (0xDull << 40) | (0xEull << 48);
    *nib = (uint32_t)(kLut >> (4 * k4)) & 0xFu;
    return m;
}

// Keep bits (bit t = element t) of a code AND mask (0xF in nibble t).
__device__ __forceinline__ uint32_t nibbles_to_bits8(uint32_t m) {
    uint32_t b = 0;
#pragma unroll
    for (int t = 0; t < 8; ++t) b |= ((m >> (4 * t)) & 1u) << t;
    return b;
}

// The second smallest of four magnitudes: the larger of the two pruned ones
// under the 2-of-4 mask (ties prune equal values, so the value is the same
// whichever index is pruned).
__device__ __forceinline__ float second_smallest4(const float* y) {
    const float a = fabsf(y[0]), b = fabsf(y[1]), c = fabsf(y[2]), d = fabsf(y[3]);
    return fminf(fmaxf(fminf(a, b), fminf(c, d)), fminf(fmaxf(a, b), fmaxf(c, d)));
}

// max |y| over the entries of an aligned 8-element chunk that the mask prunes.
template <int MG, bool NM24>
__device__ __forceinline__ float pruned_max8(const float* y, int n) {
    if (NM24) return fmaxf(second_smallest4(y), second_smallest4(y + 4));
    const uint32_t k = keep_bits<8, MG, NM24>(y, n);
    float m = 0.0f;
#pragma unroll
    for (int t = 0; t < 8; ++t) m = fmaxf(m, ((k >> t) & 1u) ? 0.0f : fabsf(y[t]));
    return m;
}

// gamma / beta of elements [c0, c0 + 2P) as fp32 pairs: from the shared
// fp32 copy, or converted from global bf16.
template <int P>
__device__ __forceinline__ void load_vec2(const float* sv, const uint16_t* gv, bool staged, int c0,
                                          float2 out[P]) {
    if (staged) {
        const float4* s4 = reinterpret_cast<const float4*>(sv + c0);
#pragma unroll
        for (int p = 0; p < P; p += 2) {
            const float4 v = s4[p / 2];
            out[p] = make_float2(v.x, v.y);
            out[p + 1] = make_float2(v.z, v.w);
        }
    } else {
#pragma unroll
        for (int p = 0; p < P; p += 4) unpack_bf16x8(ld_nc_v4(gv + c0 + 2 * p), out + p);
    }
}

template <int FMT, bool HAS_GAMMA, bool LN>
struct LaneBlock {
    static constexpr int E = FMT == 0 ? 16 : 32;   // elements per lane = one scale block
    static constexpr int NV = E / 8;                // 16-byte chunks
    uint4 x[NV];
    float rinv, mu;

    __device__ __forceinline__ void load(const PrepArgs& a, int64_t row, int cb, const float* rinv_ws) {
        const uint16_t* xp = a.X + row * a.K + (int64_t)cb * E;
#pragma unroll
        for (int v = 0; v < NV; ++v) x[v] = ld_nc_v4(xp + 8 * v);
        if (HAS_GAMMA) rinv = rinv_ws[row];
        if (LN) mu = rinv_ws[a.M + row];          // the LayerNorm means follow the M reciprocals
    }

    // RMSNorm: fl(fl(x * rinv) * g).  LayerNorm: fl(fl(fl(x - mu) * rstd) * g),
    // then + beta when there is a bias.  Without a norm y = x.
    __device__ __forceinline__ void y(float2* out, int cb, const PrepArgs& a, const float* sg,
                                      const float* sb, bool has_beta) const {
#pragma unroll
        for (int v = 0; v < NV; ++v) unpack_bf16x8(x[v], out + 4 * v);
        if (HAS_GAMMA) {
            float2 g[E / 2];
            load_vec2<E / 2>(sg, a.gamma, a.staged, cb * E, g);
            const float2 r2 = f2(rinv), mu2 = f2(mu);
#pragma unroll
            for (int p = 0; p < E / 2; ++p) {
                float2 t = LN ? sub2_rn(out[p], mu2) : out[p];
                out[p] = mul2_rn(mul2_rn(t, r2), g[p]);
            }
            if (LN && has_beta) {
                float2 b[E / 2];
                load_vec2<E / 2>(sb, a.beta, a.staged, cb * E, b);
#pragma unroll
                for (int p = 0; p < E / 2; ++p) out[p] = add2_rn(out[p], b[p]);
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
template <int FMT, bool HAS_GAMMA, int MG, bool WEIGHT, bool NM24, bool RS, bool LN, bool GIVEN,
          bool PAIRS>
__global__ void __launch_bounds__(kThreads, 2)
prepare_kernel(PrepArgs a) {
    __shared__ float s_inv[128];
    __shared__ float s_inv_p[128];    // SPEC: reciprocal table of the residual's guessed scale
    __shared__ float s_red[kWarps];
    __shared__ unsigned s_spec_sent;  // SPEC: this CTA has met a residual block above P
    extern __shared__ __align__(16) float s_vec[];     // gamma [K] (then beta [K]) as fp32
    using LB = LaneBlock<FMT, HAS_GAMMA, LN>;
    static_assert(!LN || HAS_GAMMA, "LayerNorm takes gamma");
    static_assert(!GIVEN || (FMT == 0 && !HAS_GAMMA && !WEIGHT), "a given amax: NVFP4, no norm");
    static_assert(!PAIRS || (FMT == 1 && !WEIGHT && !LN), "pair backbone: MXFP4 activations");
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
    const bool skip = (int)blockIdx.x == a.skip_block;
    // NVFP4 with its own residual scale: phase 1 also takes P = max |y| over
    // the pruned entries, and phase 2 quantises the residual against P (see
    // the end of phase 2).
    constexpr bool SPEC = FMT == 0 && !WEIGHT && !RS && !GIVEN;
    const bool spec = SPEC && a.spec;
    float* s_gamma = s_vec;
    float* s_beta = s_vec + K;
    if (threadIdx.x == 0) s_spec_sent = 0u;    // read only after phase 1's block reductions

    if (HAS_GAMMA && a.staged) {
        for (int i = threadIdx.x; i < K / 2; i += kThreads) {
            const float2 g = bf16x2_f2(reinterpret_cast<const uint32_t*>(a.gamma)[i]);
            s_gamma[2 * i] = g.x; s_gamma[2 * i + 1] = g.y;
            if (has_beta) {
                const float2 b = bf16x2_f2(reinterpret_cast<const uint32_t*>(a.beta)[i]);
                s_beta[2 * i] = b.x; s_beta[2 * i + 1] = b.y;
            }
        }
        __syncthreads();
    }

    // ---------------- phase 1: rinv per row, A_b = max |y| ----------------
    float amax = 0.0f;
    float pmax = 0.0f;     // SPEC: max |y| over the pruned entries
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
                    if (spec) {
                        // chunks start at multiples of 8 elements, so the
                        // mask's aligned groups lie inside one chunk
                        float2 x2[4];
                        unpack_bf16x8(v[u], x2);
                        pmax = fmaxf(pmax, pruned_max8<MG, NM24>(reinterpret_cast<const float*>(x2), a.n));
                    }
                }
            }
        }
        amax = fmaxf(__uint_as_float(m2 << 16), __uint_as_float(m2 & 0xFFFF0000u));
    } else if (HAS_GAMMA) {
        // One warp per row.  rinv: lane l adds f(x) over chunks l, l+32, ...
        // element by element in k order, then the xor butterfly -- the fixed
        // reduction order.  Then (NVFP4) the row's max |y|.  Eight chunk
        // loads in flight per lane.
        for (int64_t row = gwarp; row < M; row += nwarps) {
            const uint16_t* xr = a.X + row * K;
            if constexpr (!LN && FMT == 1) {
                if (nchunk <= 32 * kRowChunks) {
                    // MXFP4 takes only rinv here: the whole row's chunk loads
                    // in flight at once, then the same reduction order as
                    // below.  (For NVFP4, which also takes max |y| here, the
                    // register-held row costs spills and is slower than the
                    // second pass over the row through L1.)
                    uint4 v[kRowChunks];
#pragma unroll
                    for (int u = 0; u < kRowChunks; ++u)
                        if (lane + 32 * u < nchunk) v[u] = ld_nc_v4(xr + (int64_t)(lane + 32 * u) * 8);
                    float acc = 0.0f;
#pragma unroll
                    for (int u = 0; u < kRowChunks; ++u) {
                        if (lane + 32 * u < nchunk) {
                            float2 x[4];
                            unpack_bf16x8(v[u], x);
#pragma unroll
                            for (int t = 0; t < 4; ++t) {
                                acc = __fadd_rn(acc, __fmul_rn(x[t].x, x[t].x));
                                acc = __fadd_rn(acc, __fmul_rn(x[t].y, x[t].y));
                            }
                        }
                    }
#pragma unroll
                    for (int o = 16; o >= 1; o >>= 1)
                        acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, o));
                    const float rinv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(acc, (float)K), a.eps)));
                    if (lane == 0) rinv_ws[row] = rinv;
                    continue;
                }
            }
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
                            float2 x[4];
                            unpack_bf16x8(v[u], x);
#pragma unroll
                            for (int t = 0; t < 4; ++t) {
                                acc = __fadd_rn(acc, f(x[t].x));
                                acc = __fadd_rn(acc, f(x[t].y));
                            }
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
                const float2 r2 = f2(rinv), mu2 = f2(mu);
                constexpr int D = LN ? 4 : 8;   // LayerNorm also reads beta
                for (int c0 = lane; c0 < nchunk; c0 += 32 * D) {
                    uint4 v[D];
#pragma unroll
                    for (int u = 0; u < D; ++u)
                        if (c0 + 32 * u < nchunk) v[u] = ld_nc_v4(xr + (int64_t)(c0 + 32 * u) * 8);
#pragma unroll
                    for (int u = 0; u < D; ++u) {
                        if (c0 + 32 * u < nchunk) {
                            const int c = c0 + 32 * u;
                            float2 y[4], g[4];
                            unpack_bf16x8(v[u], y);
                            load_vec2<4>(s_gamma, a.gamma, a.staged, c * 8, g);
#pragma unroll
                            for (int t = 0; t < 4; ++t) {
                                const float2 xv = LN ? sub2_rn(y[t], mu2) : y[t];
                                y[t] = mul2_rn(mul2_rn(xv, r2), g[t]);
                            }
                            if (LN && has_beta) {
                                float2 b[4];
                                load_vec2<4>(s_beta, a.beta, a.staged, c * 8, b);
#pragma unroll
                                for (int t = 0; t < 4; ++t) y[t] = add2_rn(y[t], b[t]);
                            }
                            amax = fmaxf(amax, amax_n<8>(reinterpret_cast<const float*>(y)));
                            if (spec) pmax = fmaxf(pmax, pruned_max8<MG, NM24>(reinterpret_cast<const float*>(y), a.n));
                        }
                    }
                }
            }
        }
    }

    if (FMT == 0 && !GIVEN) {
        block_amax_to_global(amax, &a.ws[0], s_red);
        if (spec) block_amax_to_global(pmax, &a.ws[6], s_red);
        grid_barrier(&a.ws[2], gridDim.x, a.wait_ns, skip);
    } else if (HAS_GAMMA) {
        grid_barrier(&a.ws[2], gridDim.x, a.wait_ns, skip);   // rinv of every row visible to every warp
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
    // (fewer than 128 rows: one warp a row, its lanes across the row's
    // scale words; no division)
    {
        const int words = nsf / 4;
        const int prow = (int)(Mpad - M);
        for (int r = (int)gwarp; r < prow; r += (int)nwarps) {
            const int64_t row = M + r;
            for (int s4 = lane; s4 < words; s4 += 32) {
                *reinterpret_cast<uint32_t*>(a.bb_scales + sf_off(row, s4 * 4, nsf)) = 0u;
                if (!WEIGHT) *reinterpret_cast<uint32_t*>(a.rs_scales + sf_off(row, s4 * 4, nsf)) = 0u;
            }
        }
        if (PAIRS) {
            // padding rows of the metadata atoms: pairs 0 and 1 (of zero codes)
            const int kblk = K / 256;
            for (int r = (int)gwarp; r < prow; r += (int)nwarps) {
                const int64_t row = M + r;
                for (int kb = lane; kb < kblk; kb += 32)
                    *reinterpret_cast<uint4*>(a.bb_meta + ((int64_t)kb * (Mpad >> 7) + (row >> 7)) * 2048 +
                                              (row & 127) * 16) =
                        make_uint4(0x44444444u, 0x44444444u, 0x44444444u, 0x44444444u);
            }
        }
    }

    const int nb_row = K / E;
    const float2 gb2 = f2(sb.gdec);
    NvScale sp{1.0f, 1.0f, 1.0f};
    uint32_t pbits = 0;
    if (spec) {
        pbits = ld_acquire_gpu(&a.ws[6]);
        sp = nv_scale(__uint_as_float(pbits));
        fill_inv_table(s_inv_p, sp.genc);
        if (blockIdx.x == 0 && threadIdx.x == 0) *a.rs_tscale = sp.gdec;
    }
    const bool guess = spec;
    bool spec_on = guess;      // this lane still writes residual codes against P
    float ramax = 0.0f;
    {
        BlockCursor<true> cur;
        cur.init(gwarp, nwarps, M * nb_row, nb_row, lane);
        LB lb;
        if (cur.live() && cur.valid()) lb.load(a, cur.row, cur.cb, rinv_ws);
        while (cur.live()) {
            if (guess && (cur.i & 3) == 0) {
                // Once any lane anywhere has met a residual block above P the
                // guess is wrong and phase 3 will run: stop writing residual
                // codes.  One global flag write per CTA; each warp reads the
                // flag every fourth block, each lane its CTA's flag every block.
                uint32_t f = 0;
                if (lane == 0) f = ld_acquire_gpu(&a.ws[5]);
                if (__shfl_sync(0xffffffffu, f, 0)) spec_on = false;
            }
            if (spec_on && *reinterpret_cast<volatile unsigned*>(&s_spec_sent)) spec_on = false;
            BlockCursor<true> nxt = cur;
            nxt.next();
            LB ln;
            if (nxt.live() && nxt.valid()) ln.load(a, nxt.row, nxt.cb, rinv_ws);   // prefetch
            if (cur.valid()) {
            const int64_t row = cur.row;
            const int cb = cur.cb;
            float2 y2[E / 2];
            lb.y(y2, cb, a, s_gamma, s_beta, has_beta);
            const float* y = reinterpret_cast<const float*>(y2);
            // the backbone's block max is the block max of y: the largest
            // entry of every group is always kept
            const float bm = amax_n<E>(y);
            uint32_t ecode;
            float inv;
            if (FMT == 0) {
                ecode = cvt_e4m3(__fmul_rn(bm, sb.k1));
                inv = s_inv[ecode];
            } else {
                ecode = mx_code(bm);
                inv = pow2f(127 - (int)ecode);
            }
            // the mask as one code AND mask (0xF per kept element) per 8 elements
            uint32_t kmask[E / 8];
            uint32_t pnib[E / 8];          // PAIRS: metadata nibble of each group of 8
#pragma unroll
            for (int v = 0; v < E / 8; ++v) {
                if (WEIGHT)     kmask[v] = 0xFFFFFFFFu;
                else if (PAIRS) kmask[v] = keep_pairs_bytes8(y + 8 * v, &pnib[v]);
                else if (NM24)  kmask[v] = keep24_nibbles8(y + 8 * v);
                else            kmask[v] = nibble_mask8(keep_bits<8, MG, NM24>(y + 8 * v, a.n));
            }
            uint32_t codes[E / 8];
            const float2 inv2 = f2(inv);
#pragma unroll
            for (int v = 0; v < E / 8; ++v) {
                float2 q[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) q[p] = mul2_rn(y2[4 * v + p], inv2);
                codes[v] = cvt_e2m1x8_f2(q) & kmask[v];   // pruned: code 0 (+0)
            }
            if constexpr (PAIRS) {
                // the kept pairs' code bytes in order (8 bytes for the 32
                // elements), and the four metadata nibbles into the atom
                uint32_t kept[4];
#pragma unroll
                for (int v = 0; v < 4; ++v)
                    kept[v] = prmt(codes[v], 0u, (pnib[v] & 3u) | ((pnib[v] >> 2) << 4) | 0x4400u);
                *reinterpret_cast<uint2*>(a.bb_codes + row * (K / 4) + (int64_t)cb * 8) =
                    make_uint2(kept[0] | (kept[1] << 16), kept[2] | (kept[3] << 16));
                const uint32_t nib16 = pnib[0] | (pnib[1] << 4) | (pnib[2] << 8) | (pnib[3] << 12);
                *reinterpret_cast<uint16_t*>(a.bb_meta + ((int64_t)(cb >> 3) * (Mpad >> 7) + (row >> 7)) * 2048 +
                                             (row & 127) * 16 + 2 * (cb & 7)) = (uint16_t)nib16;
            } else {
                uint8_t* cp = a.bb_codes + row * (K / 2) + (int64_t)cb * (E / 2);
                if (E == 16) *reinterpret_cast<uint2*>(cp) = make_uint2(codes[0], codes[1]);
                else         *reinterpret_cast<uint4*>(cp) = make_uint4(codes[0], codes[1], codes[2], codes[3]);
            }
            a.bb_scales[cur.sfo] = (uint8_t)ecode;
            if (!WEIGHT && a.mask) {
                uint8_t* mp = a.mask + row * (K / 8) + (int64_t)cb * (E / 8);
#pragma unroll
                for (int v = 0; v < E / 8; ++v) mp[v] = (uint8_t)nibbles_to_bits8(kmask[v]);
            }

            if (!WEIGHT) {
                // residual r = y - dequant(backbone), in place in y2
                const __half2 eh = e4m3_h2(FMT == 0 ? ecode : 0u);
                const float2 sd2 = f2(pow2f((int)ecode - 127));
#pragma unroll
                for (int v = 0; v < E / 8; ++v) {
                    float2 d[4];
                    if (FMT == 0) dequant8_nv(codes[v], eh, gb2, d);
                    else          dequant8_mx(codes[v], sd2, d);
#pragma unroll
                    for (int p = 0; p < 4; ++p) y2[4 * v + p] = sub2_rn(y2[4 * v + p], d[p]);
                }
                const float rbm = amax_n<E>(y);
                if (FMT == 0 && RS) {
                    // the residual's block scale against the backbone's G
                    const uint32_t er = cvt_e4m3(__fmul_rn(rbm, sb.k1));
                    const float2 ir2 = f2(s_inv[er]);
                    uint32_t rc[E / 8];
#pragma unroll
                    for (int v = 0; v < E / 8; ++v) {
                        float2 q[4];
#pragma unroll
                        for (int p = 0; p < 4; ++p) q[p] = mul2_rn(y2[4 * v + p], ir2);
                        rc[v] = cvt_e2m1x8_f2(q);
                    }
                    *reinterpret_cast<uint2*>(a.rs_codes + row * (K / 2) + (int64_t)cb * 8) = make_uint2(rc[0], rc[1]);
                    a.rs_scales[cur.sfo] = (uint8_t)er;
                } else if (FMT == 0) {
                    ramax = fmaxf(ramax, rbm);
                    if (spec_on) {
                        if (__float_as_uint(rbm) > pbits) {   // A_r > P: phase 3 will run
                            if (atomicExch(&s_spec_sent, 1u) == 0u) atomicOr(&a.ws[5], 1u);
                            spec_on = false;
                        } else {
                            const uint32_t er = cvt_e4m3(__fmul_rn(rbm, sp.k1));
                            const float2 ir2 = f2(s_inv_p[er]);
                            uint32_t rc[2];
#pragma unroll
                            for (int v = 0; v < 2; ++v) {
                                float2 q[4];
#pragma unroll
                                for (int p = 0; p < 4; ++p) q[p] = mul2_rn(y2[4 * v + p], ir2);
                                rc[v] = cvt_e2m1x8_f2(q);
                            }
                            *reinterpret_cast<uint2*>(a.rs_codes + row * (K / 2) + (int64_t)cb * 8) = make_uint2(rc[0], rc[1]);
                            a.rs_scales[cur.sfo] = (uint8_t)er;
                        }
                    }
                } else {
                    // MXFP4: the residual needs no tensor-wide scale; finish it here.
                    const uint32_t rcode = mx_code(rbm);
                    const float2 rs2 = f2(pow2f(127 - (int)rcode));
                    uint32_t rc[E / 8];
#pragma unroll
                    for (int v = 0; v < E / 8; ++v) {
                        float2 q[4];
#pragma unroll
                        for (int p = 0; p < 4; ++p) q[p] = mul2_rn(y2[4 * v + p], rs2);
                        rc[v] = cvt_e2m1x8_f2(q);
                    }
                    *reinterpret_cast<uint4*>(a.rs_codes + row * (K / 2) + (int64_t)cb * (E / 2)) =
                        make_uint4(rc[0], rc[1], rc[2], rc[3]);
                    a.rs_scales[cur.sfo] = (uint8_t)rcode;
                }
            }
            }   // valid
            cur = nxt;
            lb = ln;
        }
    }
    if constexpr (FMT == 0 && !WEIGHT && !RS) {

    block_amax_to_global(ramax, &a.ws[1], s_red);
    grid_barrier(&a.ws[2], (GIVEN ? 1u : 2u) * gridDim.x, a.wait_ns, skip);   // counts on from phase 1's

    // The residual's tensor max is A_r = max(P, Q): P = max |y| over the
    // pruned entries (whose residual is y itself) and Q = max |y - D_b| over
    // the kept ones.  Phase 1 took P; phase 2, which is the first to know Q,
    // already quantised every residual block against P.  When A_r == P those
    // codes, scales and G_r are the final ones and phase 3 is not needed.
    const uint32_t arbits = ld_acquire_gpu(&a.ws[1]);
    if (guess && arbits == pbits) return;
    // ---------------- phase 3: residual codes with G_r ----------------
    NvScale sr = nv_scale(__uint_as_float(arbits));
    __syncthreads();                       // everyone done reading the backbone table
    fill_inv_table(s_inv, sr.genc);
    if (blockIdx.x == 0 && threadIdx.x == 0) *a.rs_tscale = sr.gdec;
    {
        BlockCursor<false> cur;
        cur.init(gwarp, nwarps, M * nb_row, nb_row, lane);
        LB lb;
        uint2 bc = make_uint2(0, 0);
        uint32_t bs = 0;
        if (cur.live() && cur.valid()) {
            lb.load(a, cur.row, cur.cb, rinv_ws);
            bc = *reinterpret_cast<const uint2*>(a.bb_codes + cur.row * (K / 2) + (int64_t)cur.cb * 8);
            bs = a.bb_scales[cur.sfo];
        }
        while (cur.live()) {
            BlockCursor<false> nxt = cur;
            nxt.next();
            LB ln;
            uint2 nbc = make_uint2(0, 0);
            uint32_t nbs = 0;
            if (nxt.live() && nxt.valid()) {
                ln.load(a, nxt.row, nxt.cb, rinv_ws);
                nbc = *reinterpret_cast<const uint2*>(a.bb_codes + nxt.row * (K / 2) + (int64_t)nxt.cb * 8);
                nbs = a.bb_scales[nxt.sfo];
            }
            if (cur.valid()) {
            const int64_t row = cur.row;
            const int cb = cur.cb;
            float2 y2[8];
            lb.y(y2, cb, a, s_gamma, s_beta, has_beta);
            const __half2 eh = e4m3_h2(bs);
            float2 d[4];
            dequant8_nv(bc.x, eh, gb2, d);
#pragma unroll
            for (int p = 0; p < 4; ++p) y2[p] = sub2_rn(y2[p], d[p]);
            dequant8_nv(bc.y, eh, gb2, d);
#pragma unroll
            for (int p = 0; p < 4; ++p) y2[4 + p] = sub2_rn(y2[4 + p], d[p]);   // y2 := r
            const uint32_t er = cvt_e4m3(__fmul_rn(amax_n<16>(reinterpret_cast<const float*>(y2)), sr.k1));
            const float2 inv2 = f2(s_inv[er]);
            float2 q[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) q[p] = mul2_rn(y2[p], inv2);
            const uint32_t c0 = cvt_e2m1x8_f2(q);
#pragma unroll
            for (int p = 0; p < 4; ++p) q[p] = mul2_rn(y2[4 + p], inv2);
            const uint32_t c1 = cvt_e2m1x8_f2(q);
            *reinterpret_cast<uint2*>(a.rs_codes + row * (K / 2) + (int64_t)cb * 8) = make_uint2(c0, c1);
            a.rs_scales[cur.sfo] = (uint8_t)er;
            }   // valid
            cur = nxt;
            lb = ln;
            bc = nbc;
            bs = nbs;
        }
    }
    }   // phase 3
}

template <int FMT, bool HAS_GAMMA, int MG, bool WEIGHT, bool NM24, bool RS = false, bool LN = false,
          bool GIVEN = false, bool PAIRS = false>
cudaError_t launch_one(const PrepArgs& a, cudaStream_t s, int max_blocks) {
    auto kfn = prepare_kernel<FMT, HAS_GAMMA, MG, WEIGHT, NM24, RS, LN, GIVEN, PAIRS>;
    const size_t smem = a.staged ? (size_t)a.K * 4 * (LN && a.beta ? 2 : 1) : 0;
    // Resident blocks per SM at this shared-memory size (the cooperative
    // grid must not exceed it); the same for every device of one
    // architecture, so cache the answer per size class.
    static std::atomic<int> cached[4];
    const int cls = smem == 0 ? 0 : smem <= 32 * 1024 ? 1 : smem <= 64 * 1024 ? 2 : 3;
    const size_t cls_bytes[4] = {0, 32 * 1024, 64 * 1024, (size_t)kMaxStagedBytes};
    int blocks_per_sm = cached[cls].load(std::memory_order_relaxed);
    if (blocks_per_sm == 0) {
        if (cls_bytes[cls] > 48 * 1024) {
            cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)kMaxStagedBytes);
            if (e != cudaSuccess) return e;
        }
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks_per_sm, kfn, kThreads,
                                                                      cls_bytes[cls]);
        if (e != cudaSuccess) return e;
        if (blocks_per_sm < 1) return cudaErrorInvalidConfiguration;
        cached[cls].store(blocks_per_sm, std::memory_order_relaxed);
    }
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kMaxStagedBytes);
        if (e != cudaSuccess) return e;
    }
    // Enough warps for one row each in phase 1 and about four 32-block
    // groups each in phases 2 and 3, capped at what is resident.
    int64_t Mpad = (a.M + 127) / 128 * 128;
    int64_t groups = a.M * (int64_t)(a.K / (FMT == 0 ? 16 : 32)) / 32;
    int64_t want = std::max((Mpad + kWarps - 1) / kWarps, (groups + 4 * kWarps - 1) / (4 * kWarps));
    int64_t cap = (int64_t)blocks_per_sm * max_blocks;
    int grid = (int)std::max<int64_t>(1, std::min(want, cap));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
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
    a.bb_meta = static_cast<uint8_t*>(p.bb_meta);
    const bool g = p.gamma != nullptr;
    const size_t vec_bytes = (size_t)p.K * 4 * (p.layernorm && p.beta ? 2 : 1);
    a.staged = g && vec_bytes <= (size_t)kMaxStagedBytes;
    a.spec = p.spec_off ? 0 : 1;
    a.wait_ns = p.wait_ns ? p.wait_ns : kWaitLimitNs;
    a.skip_block = p.skip_block;
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
    if (p.bb_meta) {              // pair-granular 4:8 backbone, MXFP4
        return g ? launch_one<1, true, 8, false, false, false, false, false, true>(a, s, sms)
                 : launch_one<1, false, 8, false, false, false, false, false, true>(a, s, sms);
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
