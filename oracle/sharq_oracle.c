/*
 * sharq_oracle.c -- plain, slow CPU reference for the SharQ hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA path and never calls it.
 *
 * What it follows (SharQ: Bridging Activation Sparsity and FP4 Quantization
 * for LLM Inference, arXiv 2606.26587, Abstract):
 *   - an input-adaptive N:M mask picks an outlier-dominated sparse backbone
 *     of the (normalised) activation tensor;
 *   - the backbone is quantised to FP4;
 *   - the dense residual is taken against the *dequantised* backbone and is
 *     quantised to FP4 as well;
 *   - layer normalisation, mask generation and residual construction form one
 *     preparation operator;
 *   - formats: NVFP4 (main) and MXFP4.
 * The pages define none of the formats or scale recipes; those follow the
 * public OCP specifications (OCP 8-bit Floating Point Specification, E4M3;
 * OCP Microscaling Formats (MX) v1.0, E2M1 elements and E8M0 scales) and
 * NVIDIA's published NVFP4 recipe (16-element blocks, E4M3 block scale, FP32
 * tensor scale equal to amax / (6 * 448)).
 *
 * Arithmetic: every float operation below is one IEEE-754 binary32 operation
 * with round-to-nearest-even.  Build with -O2 -ffp-contract=off and without
 * -ffast-math so the compiler neither fuses nor reorders anything.
 *
 * Parity status of each function is listed in its comment.  "pinned" means a
 * test checks it against something other than itself (closed forms,
 * brute-force search, a library cast, invariants fixed by the mathematics).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_NVFP4 0
#define ORC_MXFP4 1

/* ------------------------------------------------------------------------ */
/* E2M1 (OCP MX v1.0, FP4 element): 1 sign, 2 exponent (bias 1), 1 mantissa. */
/* Magnitudes by code 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6.  No inf / NaN.       */
/* Pinned: exhaustive brute-force nearest search and ml_dtypes cast.         */
/* ------------------------------------------------------------------------ */

static const float E2M1_MAG[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

float orc_e2m1_decode(uint8_t code) {
    float v = E2M1_MAG[code & 7];
    return (code & 8) ? -v : v;
}

/* Round to nearest E2M1 value, ties to the even code (mantissa bit 0),
 * saturating to +-6.  The sign of the input is kept, also when the result is
 * zero (so -0.1 -> 0x8).  The boundaries are the midpoints of the grid; a
 * midpoint goes to the neighbour whose code is even. */
uint8_t orc_e2m1_encode(float v) {
    uint8_t sign = signbit(v) ? 8 : 0;
    float a = fabsf(v);
    uint8_t c;
    if (a <= 0.25f)      c = 0;   /* tie 0.25 -> 0 (code 0 even)   */
    else if (a < 0.75f)  c = 1;   /* tie 0.75 -> 1.0 (code 2)      */
    else if (a <= 1.25f) c = 2;   /* tie 1.25 -> 1.0 (code 2)      */
    else if (a < 1.75f)  c = 3;   /* tie 1.75 -> 2.0 (code 4)      */
    else if (a <= 2.5f)  c = 4;   /* tie 2.5  -> 2.0 (code 4)      */
    else if (a < 3.5f)   c = 5;   /* tie 3.5  -> 4.0 (code 6)      */
    else if (a <= 5.0f)  c = 6;   /* tie 5.0  -> 4.0 (code 6)      */
    else                 c = 7;   /* (5, inf) -> 6 (satfinite)     */
    return (uint8_t)(sign | c);
}

void orc_e2m1_encode_array(const float* v, uint8_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_encode(v[i]);
}

/* ------------------------------------------------------------------------ */
/* E4M3 (OCP FP8, "E4M3FN"): bias 7, subnormals m * 2^-9, max 448, no inf,  */
/* 0x7F / 0xFF are NaN.  Encode: round to nearest even, saturate to 448.    */
/* Pinned: all 256 codes decoded against the closed form, exhaustive        */
/* brute-force nearest search on the scale domain, ml_dtypes cast.          */
/* ------------------------------------------------------------------------ */

float orc_e4m3_decode(uint8_t code) {
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    float v;
    if (e == 15 && m == 7) v = NAN;
    else if (e == 0) v = ldexpf((float)m, -9);
    else v = ldexpf(1.0f + (float)m / 8.0f, e - 7);
    return s ? -v : v;
}

uint8_t orc_e4m3_encode(float v) {
    uint8_t sign = signbit(v) ? 0x80 : 0;
    float a = fabsf(v);
    if (a >= 448.0f) return (uint8_t)(sign | 0x7E);          /* satfinite */
    if (a < ldexpf(1.0f, -6)) {                               /* subnormal range */
        float q = rintf(a * 512.0f);                          /* exact scaling, RNE */
        return (uint8_t)(sign | (uint8_t)q);                  /* q == 8 is the min normal 0x08 */
    }
    int E;
    frexpf(a, &E);                                            /* a = f * 2^E, f in [0.5,1) */
    int e = E - 1;                                            /* a in [2^e, 2^(e+1)) */
    float frac = ldexpf(a, -e) - 1.0f;                        /* exact, in [0,1) */
    int m = (int)rintf(frac * 8.0f);                          /* RNE on 3 mantissa bits */
    if (m == 8) { m = 0; e += 1; }
    int be = e + 7;
    if (be > 15 || (be == 15 && m == 7)) return (uint8_t)(sign | 0x7E);
    return (uint8_t)(sign | (be << 3) | m);
}

void orc_e4m3_encode_array(const float* v, uint8_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(v[i]);
}

void orc_e4m3_decode_array(const uint8_t* c, float* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_decode(c[i]);
}

/* ------------------------------------------------------------------------ */
/* E8M0 (OCP MX v1.0 shared scale): code c means 2^(c-127), c = 255 is NaN. */
/* MX scale choice for a 32-block with amax b: floor(log2 b) - emax(E2M1)   */
/* where emax(E2M1) = 2, biased by 127 and clamped to [0, 254]; b = 0 gives */
/* code 0.  Pinned: closed-form exponent checks and grid identity.          */
/* ------------------------------------------------------------------------ */

float orc_e8m0_decode(uint8_t c) { return ldexpf(1.0f, (int)c - 127); }

uint8_t orc_mx_scale_code(float amax) {
    if (amax == 0.0f) return 0;
    int E;
    frexpf(amax, &E);               /* exact floor(log2 amax) = E - 1, subnormals included */
    int c = (E - 1) - 2 + 127;
    if (c < 0) c = 0;
    if (c > 254) c = 254;
    return (uint8_t)c;
}

/* ------------------------------------------------------------------------ */
/* RMSNorm in the fixed reduction order (fp32):                              */
/*   sq_k = x_k*x_k; 32 virtual lanes, chunk c = elements [8c, 8c+8) belongs */
/*   to lane c mod 32 and is added element by element in k order; the lanes  */
/*   are then combined by an xor butterfly over offsets 16, 8, 4, 2, 1;      */
/*   ms = S / K; rinv = 1 / sqrt(ms + eps); y_k = (x_k * rinv) * gamma_k.    */
/* The pages say only that normalisation is fused into the preparation       */
/* operator (Abstract); RMSNorm and the order are this library's reading.    */
/* Pinned: constant-row closed form, fp64 agreement, a lane-order probe     */
/* that only this order predicts, and bit equality with an exact-rational   */
/* model of IEEE binary32 round-to-nearest-even evaluated in this order.    */
/* ------------------------------------------------------------------------ */

float orc_rms_rinv(const uint16_t* x_bf16, int K, float eps) {
    float lane[32];
    for (int l = 0; l < 32; ++l) lane[l] = 0.0f;
    int nchunks = K / 8;
    for (int c = 0; c < nchunks; ++c) {
        int l = c % 32;
        for (int t = 0; t < 8; ++t) {
            uint32_t u = (uint32_t)x_bf16[8 * c + t] << 16;
            float xv; memcpy(&xv, &u, 4);
            float sq = xv * xv;
            lane[l] = lane[l] + sq;
        }
    }
    for (int o = 16; o >= 1; o >>= 1) {
        float nxt[32];
        for (int l = 0; l < 32; ++l) nxt[l] = lane[l] + lane[l ^ o];
        memcpy(lane, nxt, sizeof(lane));
    }
    float S = lane[0];
    float ms = S / (float)K;
    float den = sqrtf(ms + eps);
    return 1.0f / den;
}

static inline float bf16f(uint16_t b) {
    uint32_t u = (uint32_t)b << 16; float f; memcpy(&f, &u, 4); return f;
}

/* ------------------------------------------------------------------------ */
/* LayerNorm statistics (the mean-subtracting norm of DiT and vision         */
/* layers, which the pages name among the evaluated models; the reading of   */
/* its precision is this library's):                                         */
/*   S1 = sum x_k and S2 = sum (x_k - mu)^2, each in the canonical order of  */
/*   the RMS sum above (32 lanes, chunk c to lane c mod 32, element order    */
/*   inside a lane, xor butterfly 16..1);                                    */
/*   mu = S1 / K;  d_k = x_k - mu;  var = S2 / K;                            */
/*   rstd = 1 / sqrt(var + eps);  y_k = (d_k * rstd) * gamma_k [+ beta_k].   */
/* Two passes (mean, then centred squares): the textbook stable form.        */
/* Pinned: constant row (y = beta exactly), a +-a row against its closed     */
/* form, a lane-order probe on S1, and bit equality of mu, rstd and y with  */
/* an exact-rational IEEE binary32 model evaluated in this order.           */
/* ------------------------------------------------------------------------ */

static float canonical_sum(const float* v, int K) {
    float lane[32];
    for (int l = 0; l < 32; ++l) lane[l] = 0.0f;
    for (int c = 0; c < K / 8; ++c)
        for (int t = 0; t < 8; ++t) lane[c % 32] = lane[c % 32] + v[8 * c + t];
    for (int o = 16; o >= 1; o >>= 1) {
        float nxt[32];
        for (int l = 0; l < 32; ++l) nxt[l] = lane[l] + lane[l ^ o];
        memcpy(lane, nxt, sizeof(lane));
    }
    return lane[0];
}

/* mu and rstd of one row; returns -1 if K is not a multiple of 8 or too big */
int orc_ln_stats(const uint16_t* x_bf16, int K, float eps, float* mu_out, float* rstd_out) {
    if (K <= 0 || K % 8 != 0 || K > (1 << 20)) return -1;
    float* v = (float*)malloc(sizeof(float) * (size_t)K);
    if (!v) return -1;
    for (int k = 0; k < K; ++k) v[k] = bf16f(x_bf16[k]);
    float mu = canonical_sum(v, K) / (float)K;
    for (int k = 0; k < K; ++k) {
        float d = v[k] - mu;
        v[k] = d * d;
    }
    float var = canonical_sum(v, K) / (float)K;
    float den = sqrtf(var + eps);
    *mu_out = mu;
    *rstd_out = 1.0f / den;
    free(v);
    return 0;
}

void orc_normalize_ln(const uint16_t* X, const uint16_t* gamma, const uint16_t* beta, float eps,
                      int64_t M, int K, float* y) {
    for (int64_t i = 0; i < M; ++i) {
        const uint16_t* xr = X + i * (int64_t)K;
        float* yr = y + i * (int64_t)K;
        float mu = 0.0f, rstd = 1.0f;
        orc_ln_stats(xr, K, eps, &mu, &rstd);
        for (int k = 0; k < K; ++k) {
            float d = bf16f(xr[k]) - mu;
            float t = (d * rstd) * bf16f(gamma[k]);
            yr[k] = beta ? t + bf16f(beta[k]) : t;
        }
    }
}

/* y = RMSNorm(x) * gamma per row, or y = x when gamma is NULL. */
void orc_normalize(const uint16_t* X, const uint16_t* gamma, float eps,
                   int64_t M, int K, float* y) {
    for (int64_t i = 0; i < M; ++i) {
        const uint16_t* xr = X + i * (int64_t)K;
        float* yr = y + i * (int64_t)K;
        if (!gamma) {
            for (int k = 0; k < K; ++k) yr[k] = bf16f(xr[k]);
            continue;
        }
        float rinv = orc_rms_rinv(xr, K, eps);
        for (int k = 0; k < K; ++k) {
            float t = bf16f(xr[k]) * rinv;
            yr[k] = t * bf16f(gamma[k]);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Input-adaptive N:M mask (Abstract: the mask extracts an outlier-dominated */
/* backbone).  Reading: inside every aligned group of m along K keep the n   */
/* entries of largest |y|; on equal |y| the lower index ranks higher.        */
/* Pinned: exactly n kept per group, brute-force stable sort, group max kept.*/
/* ------------------------------------------------------------------------ */

void orc_mask(const float* y, int64_t M, int K, int n, int m, uint8_t* keep) {
    for (int64_t i = 0; i < M; ++i) {
        for (int g = 0; g < K; g += m) {
            const float* yg = y + i * (int64_t)K + g;
            for (int a = 0; a < m; ++a) {
                int rank = 0;
                for (int b = 0; b < m; ++b) {
                    if (b == a) continue;
                    float fa = fabsf(yg[a]), fb = fabsf(yg[b]);
                    if (fb > fa || (fb == fa && b < a)) ++rank;
                }
                keep[i * (int64_t)K + g + a] = (uint8_t)(rank < n);
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Block quantisers.  T is one tensor [R, K]; the tensor scale (NVFP4) is    */
/* taken over the whole tensor.  Outputs in canonical row-major layouts:     */
/*   codes [R, K/2]   E2M1 pairs, element 2j in bits 3:0, 2j+1 in bits 7:4   */
/*   scales [R, K/B]  one byte per block (E4M3 for B = 16, E8M0 for B = 32)  */
/*   gdec             decode tensor scale (1.0 for MXFP4)                    */
/*   D [R, K]         dequantised values (optional)                          */
/* ------------------------------------------------------------------------ */

/* NVFP4: A = max|T|; G_enc = 2688/A, G_dec = A/2688 (both 1 when A = 0),
 * 2688 = 6 * 448; K1 = G_enc/6; per 16-block e = E4M3(b*K1);
 * inv = G_enc/e (0 when e = 0); q = E2M1(T*inv); D = (val(q)*e)*G_dec. */
float orc_tensor_amax(const float* T, int64_t n) {
    float A = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(T[i]);
        if (a > A) A = a;
    }
    return A;
}

/* The same quantiser with the tensor amax A given by the caller instead of
 * taken over T (the shared-scale residual below uses the backbone's A). */
void orc_quant_nvfp4_amax(const float* T, int64_t R, int K, float A,
                          uint8_t* codes, uint8_t* scales, float* gdec_out, float* D);

void orc_quant_nvfp4(const float* T, int64_t R, int K,
                     uint8_t* codes, uint8_t* scales, float* gdec_out, float* D) {
    orc_quant_nvfp4_amax(T, R, K, orc_tensor_amax(T, R * (int64_t)K), codes, scales, gdec_out, D);
}

void orc_quant_nvfp4_amax(const float* T, int64_t R, int K, float A,
                          uint8_t* codes, uint8_t* scales, float* gdec_out, float* D) {
    float genc = 1.0f, gdec = 1.0f;
    if (A != 0.0f) { genc = 2688.0f / A; gdec = A / 2688.0f; }
    float k1 = genc / 6.0f;
    int nb = K / 16;
    memset(codes, 0, (size_t)(R * (int64_t)(K / 2)));
    for (int64_t i = 0; i < R; ++i) {
        const float* t = T + i * (int64_t)K;
        for (int blk = 0; blk < nb; ++blk) {
            float b = 0.0f;
            for (int j = 0; j < 16; ++j) {
                float a = fabsf(t[blk * 16 + j]);
                if (a > b) b = a;
            }
            uint8_t e = orc_e4m3_encode(b * k1);
            float ev = orc_e4m3_decode(e);
            float inv = (ev == 0.0f) ? 0.0f : genc / ev;
            scales[i * nb + blk] = e;
            for (int j = 0; j < 16; ++j) {
                int k = blk * 16 + j;
                uint8_t q = orc_e2m1_encode(t[k] * inv);
                uint8_t* byte = codes + i * (int64_t)(K / 2) + k / 2;
                *byte |= (uint8_t)((k & 1) ? (q << 4) : q);
                if (D) {
                    float p = orc_e2m1_decode(q) * ev;       /* exact */
                    D[i * (int64_t)K + k] = p * gdec;
                }
            }
        }
    }
    *gdec_out = gdec;
}

/* MXFP4: per 32-block c = mx_scale_code(b); q = E2M1(T * 2^(127-c));
 * D = val(q) * 2^(c-127).  No tensor scale (reported as 1.0). */
void orc_quant_mxfp4(const float* T, int64_t R, int K,
                     uint8_t* codes, uint8_t* scales, float* gdec_out, float* D) {
    int nb = K / 32;
    memset(codes, 0, (size_t)(R * (int64_t)(K / 2)));
    for (int64_t i = 0; i < R; ++i) {
        const float* t = T + i * (int64_t)K;
        for (int blk = 0; blk < nb; ++blk) {
            float b = 0.0f;
            for (int j = 0; j < 32; ++j) {
                float a = fabsf(t[blk * 32 + j]);
                if (a > b) b = a;
            }
            uint8_t c = orc_mx_scale_code(b);
            float enc = ldexpf(1.0f, 127 - (int)c);
            float dec = ldexpf(1.0f, (int)c - 127);
            scales[i * nb + blk] = c;
            for (int j = 0; j < 32; ++j) {
                int k = blk * 32 + j;
                uint8_t q = orc_e2m1_encode(t[k] * enc);
                uint8_t* byte = codes + i * (int64_t)(K / 2) + k / 2;
                *byte |= (uint8_t)((k & 1) ? (q << 4) : q);
                if (D) D[i * (int64_t)K + k] = orc_e2m1_decode(q) * dec;
            }
        }
    }
    *gdec_out = 1.0f;
}

static void quant(int fmt, const float* T, int64_t R, int K,
                  uint8_t* codes, uint8_t* scales, float* g, float* D) {
    if (fmt == ORC_NVFP4) orc_quant_nvfp4(T, R, K, codes, scales, g, D);
    else                  orc_quant_mxfp4(T, R, K, codes, scales, g, D);
}

/* ------------------------------------------------------------------------ */
/* Preparation operator (Abstract: norm + mask + backbone FP4 + residual     */
/* against the dequantised backbone + residual FP4, one operator):           */
/*   y = norm(x) (RMSNorm with gamma, none without, or LayerNorm with gamma  */
/*       and an optional beta); keep = mask(y); B = keep ? y : +0;           */
/*   (codes_b, scales_b, G_b, D_b) = Q(B); r = y - D_b;                      */
/*   (codes_r, scales_r, G_r) = Q(r)   -- residual has its own tensor scale, */
/*   or, with residual_shared (NVFP4), the backbone's: Q(r) is taken with    */
/*   A = max|B| in place of max|r|, so G_r = G_b (a variant the pages leave  */
/*   open: the abstract names one tensor scale per FP4 tensor or none).      */
/* mask_bits [M, K/8] (bit t of byte j = element 8j+t kept) is optional, as  */
/* are the y / r outputs used by invariant tests.                            */
/* Returns 0, or -1 on a bad argument or allocation failure.                 */
/* ------------------------------------------------------------------------ */

int orc_prepare(const uint16_t* X, const uint16_t* gamma, const uint16_t* beta, int layernorm,
                float eps, int64_t M, int K, int n, int m, int fmt, int residual_shared,
                uint8_t* mask_bits,
                uint8_t* bb_codes, uint8_t* bb_scales, float* bb_g,
                uint8_t* rs_codes, uint8_t* rs_scales, float* rs_g,
                float* y_out, float* r_out) {
    if (K <= 0 || m <= 0 || n < 0 || n > m || K % m != 0 || K % 32 != 0) return -1;
    if (layernorm && !gamma) return -1;
    int64_t E = M * (int64_t)K;
    float* y = y_out ? y_out : (float*)malloc(sizeof(float) * (size_t)(E ? E : 1));
    float* B = (float*)malloc(sizeof(float) * (size_t)(E ? E : 1));
    float* D = (float*)malloc(sizeof(float) * (size_t)(E ? E : 1));
    uint8_t* keep = (uint8_t*)malloc((size_t)(E ? E : 1));
    if (!y || !B || !D || !keep) { free(B); free(D); free(keep); if (!y_out) free(y); return -1; }

    if (layernorm) orc_normalize_ln(X, gamma, beta, eps, M, K, y);
    else           orc_normalize(X, gamma, eps, M, K, y);
    orc_mask(y, M, K, n, m, keep);
    for (int64_t i = 0; i < E; ++i) B[i] = keep[i] ? y[i] : 0.0f;
    const float A_b = orc_tensor_amax(B, E);
    quant(fmt, B, M, K, bb_codes, bb_scales, bb_g, D);
    float* r = B;                                /* reuse: B is no longer needed */
    for (int64_t i = 0; i < E; ++i) r[i] = y[i] - D[i];
    if (residual_shared && fmt == ORC_NVFP4) orc_quant_nvfp4_amax(r, M, K, A_b, rs_codes, rs_scales, rs_g, NULL);
    else                                     quant(fmt, r, M, K, rs_codes, rs_scales, rs_g, NULL);
    if (r_out) memcpy(r_out, r, sizeof(float) * (size_t)E);
    if (mask_bits) {
        for (int64_t i = 0; i < M; ++i)
            for (int j = 0; j < K / 8; ++j) {
                uint8_t v = 0;
                for (int t = 0; t < 8; ++t)
                    v |= (uint8_t)(keep[i * (int64_t)K + 8 * j + t] << t);
                mask_bits[i * (int64_t)(K / 8) + j] = v;
            }
    }
    free(B); free(D); free(keep);
    if (!y_out) free(y);
    return 0;
}

/* Weight payload: one quantisation of the whole [N, K] weight; the two GEMM
 * paths read the same codes and scales (Abstract: one shared FP4 weight
 * payload). */
int orc_quantize_weight(const uint16_t* W, int64_t N, int K, int fmt,
                        uint8_t* codes, uint8_t* scales, float* g) {
    int64_t E = N * (int64_t)K;
    float* w = (float*)malloc(sizeof(float) * (size_t)(E ? E : 1));
    if (!w) return -1;
    for (int64_t i = 0; i < E; ++i) w[i] = bf16f(W[i]);
    quant(fmt, w, N, K, codes, scales, g, NULL);
    free(w);
    return 0;
}

/* Block-scaled values without the tensor scale, in fp64 (val(q) * e is exact):
 * the operands the GEMM reference multiplies. */
void orc_dequant_blocks_f64(const uint8_t* codes, const uint8_t* scales, int fmt,
                            int64_t R, int K, double* out) {
    int bs = (fmt == ORC_NVFP4) ? 16 : 32;
    int nb = K / bs;
    for (int64_t i = 0; i < R; ++i)
        for (int k = 0; k < K; ++k) {
            uint8_t byte = codes[i * (int64_t)(K / 2) + k / 2];
            uint8_t q = (k & 1) ? (byte >> 4) : (byte & 15);
            uint8_t s = scales[i * nb + k / bs];
            double e = (fmt == ORC_NVFP4) ? (double)orc_e4m3_decode(s)
                                          : (double)orc_e8m0_decode(s);
            out[i * (int64_t)K + k] = (double)orc_e2m1_decode(q) * e;
        }
}
