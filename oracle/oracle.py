"""Python face of the C oracle (test infrastructure only).

Builds ``sharq_oracle.c`` with gcc into ``oracle/_build/liboracle.so`` on
first use, wraps it with ctypes and adds the fp64 GEMM reference.  Nothing
here imports the CUDA package; the inputs come from the seeded generators in
``activation_sparsity_prep_b200.workloads``.

Layouts returned (canonical, row-major):
  mask      uint8 [M, K/8]   bit t of byte j = element 8j+t kept
  codes     uint8 [R, K/2]   E2M1 pairs, even element in the low nibble
  scales    uint8 [R, K/B]   E4M3 (NVFP4, B=16) or E8M0 (MXFP4, B=32) codes
  tscale    float32          decode tensor scale (1.0 for MXFP4)
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sharq_oracle.c")
_LIB = os.path.join(_HERE, "_build", "liboracle.so")
_lock = threading.Lock()
_lib = None

NVFP4, MXFP4 = 0, 1
FMT = {"nvfp4": NVFP4, "mxfp4": MXFP4}
BLOCK = {NVFP4: 16, MXFP4: 32}

GCC_FLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
             "-Wall", "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    """Compile the oracle library (idempotent).  Returns its path."""
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", *GCC_FLAGS, "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i64, i32, f32 = ctypes.c_int64, ctypes.c_int, ctypes.c_float
            L.orc_e2m1_encode_array.argtypes = [P, P, i64]
            L.orc_e4m3_encode_array.argtypes = [P, P, i64]
            L.orc_e4m3_decode_array.argtypes = [P, P, i64]
            L.orc_e2m1_decode.argtypes = [ctypes.c_uint8]
            L.orc_e2m1_decode.restype = f32
            L.orc_e8m0_decode.argtypes = [ctypes.c_uint8]
            L.orc_e8m0_decode.restype = f32
            L.orc_mx_scale_code.argtypes = [f32]
            L.orc_mx_scale_code.restype = ctypes.c_uint8
            L.orc_rms_rinv.argtypes = [P, i32, f32]
            L.orc_rms_rinv.restype = f32
            L.orc_normalize.argtypes = [P, P, f32, i64, i32, P]
            L.orc_mask.argtypes = [P, i64, i32, i32, i32, P]
            L.orc_quant_nvfp4.argtypes = [P, i64, i32, P, P, P, P]
            L.orc_quant_mxfp4.argtypes = [P, i64, i32, P, P, P, P]
            L.orc_quant_nvfp4_amax.argtypes = [P, i64, i32, f32, P, P, P, P]
            L.orc_tensor_amax.argtypes = [P, i64]
            L.orc_tensor_amax.restype = f32
            L.orc_prepare.argtypes = [P, P, P, i32, f32, i64, i32, i32, i32, i32, i32,
                                      P, P, P, P, P, P, P, P, P]
            L.orc_ln_stats.argtypes = [P, i32, f32, P, P]
            L.orc_ln_stats.restype = i32
            L.orc_normalize_ln.argtypes = [P, P, P, f32, i64, i32, P]
            L.orc_prepare.restype = i32
            L.orc_quantize_weight.argtypes = [P, i64, i32, i32, P, P, P]
            L.orc_quantize_weight.restype = i32
            L.orc_dequant_blocks_f64.argtypes = [P, P, i32, i64, i32, P]
            _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _fmt(fmt) -> int:
    return FMT[fmt] if isinstance(fmt, str) else int(fmt)


# ---------------------------------------------------------------- formats --

def e2m1_encode(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().orc_e2m1_encode_array(_p(v), _p(out), v.size)
    return out


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    tab = np.array([lib().orc_e2m1_decode(c) for c in range(16)], dtype=np.float32)
    return tab[np.asarray(codes) & 15]


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().orc_e4m3_encode_array(_p(v), _p(out), v.size)
    return out


def e4m3_decode(c: np.ndarray) -> np.ndarray:
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float32)
    lib().orc_e4m3_decode_array(_p(c), _p(out), c.size)
    return out


def e8m0_decode(c: np.ndarray) -> np.ndarray:
    tab = np.array([lib().orc_e8m0_decode(i) for i in range(256)], dtype=np.float32)
    return tab[np.asarray(c, dtype=np.uint8)]


def mx_scale_code(amax: float) -> int:
    return int(lib().orc_mx_scale_code(float(amax)))


# ------------------------------------------------------------------- steps --

def rms_rinv(x_row_bf16: np.ndarray, eps: float) -> np.float32:
    x = np.ascontiguousarray(x_row_bf16, dtype=np.uint16)
    return np.float32(lib().orc_rms_rinv(_p(x), x.size, eps))


def normalize(X: np.ndarray, gamma: Optional[np.ndarray], eps: float) -> np.ndarray:
    X = np.ascontiguousarray(X, dtype=np.uint16)
    M, K = X.shape
    g = None if gamma is None else np.ascontiguousarray(gamma, dtype=np.uint16)
    y = np.empty((M, K), dtype=np.float32)
    lib().orc_normalize(_p(X), _p(g), eps, M, K, _p(y))
    return y


def mask(y: np.ndarray, n: int, m: int) -> np.ndarray:
    """0/1 keep flags per element, [M, K] uint8."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    M, K = y.shape
    keep = np.empty((M, K), dtype=np.uint8)
    lib().orc_mask(_p(y), M, K, n, m, _p(keep))
    return keep


@dataclass
class Quantized:
    codes: np.ndarray
    scales: np.ndarray
    tscale: np.float32
    fmt: int
    D: Optional[np.ndarray] = None


def quantize(T: np.ndarray, fmt="nvfp4", want_D: bool = False) -> Quantized:
    fmt = _fmt(fmt)
    T = np.ascontiguousarray(T, dtype=np.float32)
    R, K = T.shape
    codes = np.empty((R, K // 2), dtype=np.uint8)
    scales = np.empty((R, K // BLOCK[fmt]), dtype=np.uint8)
    g = np.zeros(1, dtype=np.float32)
    D = np.empty((R, K), dtype=np.float32) if want_D else None
    fn = lib().orc_quant_nvfp4 if fmt == NVFP4 else lib().orc_quant_mxfp4
    fn(_p(T), R, K, _p(codes), _p(scales), _p(g), _p(D))
    return Quantized(codes, scales, g[0], fmt, D)


@dataclass
class Prepared:
    mask: np.ndarray
    bb: Quantized
    rs: Quantized
    n: int
    m: int
    fmt: int
    y: Optional[np.ndarray] = None
    r: Optional[np.ndarray] = None


RESIDUAL_SCALES = {"own": 0, "shared": 1}


def ln_stats(x: np.ndarray, eps: float = 1e-6):
    """(mu, rstd) of one bf16 row under the LayerNorm reading."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    mu = np.zeros(1, dtype=np.float32)
    rs = np.zeros(1, dtype=np.float32)
    if lib().orc_ln_stats(_p(x), x.shape[-1], eps, _p(mu), _p(rs)) != 0:
        raise ValueError("bad row")
    return mu[0], rs[0]


def normalize_ln(X: np.ndarray, gamma: np.ndarray, beta: Optional[np.ndarray], eps: float = 1e-6):
    X = np.ascontiguousarray(X, dtype=np.uint16)
    M, K = X.shape
    y = np.empty((M, K), dtype=np.float32)
    b = None if beta is None else np.ascontiguousarray(beta, dtype=np.uint16)
    lib().orc_normalize_ln(_p(X), _p(np.ascontiguousarray(gamma, dtype=np.uint16)), _p(b), eps, M, K, _p(y))
    return y


def prepare(X: np.ndarray, gamma: Optional[np.ndarray], eps: float = 1e-6,
            n: int = 2, m: int = 4, fmt="nvfp4", keep_intermediates: bool = False,
            residual_scale: str = "own", norm: str = "rms",
            beta: Optional[np.ndarray] = None) -> Prepared:
    """The preparation operator on a whole tensor X [M, K] (bf16 bits).

    residual_scale "own": the residual is quantised with its own tensor
    scale (the plain reading of the abstract); "shared": with the backbone's
    (NVFP4 only; MXFP4 has no tensor scale, so both settings agree).
    norm "rms": RMSNorm with gamma (no norm when gamma is None); "layernorm":
    LayerNorm with gamma and an optional beta."""
    fmt = _fmt(fmt)
    X = np.ascontiguousarray(X, dtype=np.uint16)
    M, K = X.shape
    g = None if gamma is None else np.ascontiguousarray(gamma, dtype=np.uint16)
    B = BLOCK[fmt]
    mk = np.empty((M, K // 8), dtype=np.uint8)
    bc = np.empty((M, K // 2), dtype=np.uint8)
    bs = np.empty((M, K // B), dtype=np.uint8)
    rc = np.empty((M, K // 2), dtype=np.uint8)
    rsc = np.empty((M, K // B), dtype=np.uint8)
    bg = np.zeros(1, dtype=np.float32)
    rg = np.zeros(1, dtype=np.float32)
    y = np.empty((M, K), dtype=np.float32) if keep_intermediates else None
    r = np.empty((M, K), dtype=np.float32) if keep_intermediates else None
    if norm not in ("rms", "layernorm"):
        raise ValueError(norm)
    b = None if beta is None else np.ascontiguousarray(beta, dtype=np.uint16)
    rc_ = lib().orc_prepare(_p(X), _p(g), _p(b), int(norm == "layernorm"), eps, M, K, n, m, fmt,
                            RESIDUAL_SCALES[residual_scale], _p(mk),
                            _p(bc), _p(bs), _p(bg), _p(rc), _p(rsc), _p(rg),
                            _p(y), _p(r))
    if rc_ != 0:
        raise ValueError("oracle prepare rejected its arguments")
    return Prepared(mk, Quantized(bc, bs, bg[0], fmt), Quantized(rc, rsc, rg[0], fmt),
                    n, m, fmt, y, r)


def quantize_weight(W: np.ndarray, fmt="nvfp4") -> Quantized:
    fmt = _fmt(fmt)
    W = np.ascontiguousarray(W, dtype=np.uint16)
    N, K = W.shape
    codes = np.empty((N, K // 2), dtype=np.uint8)
    scales = np.empty((N, K // BLOCK[fmt]), dtype=np.uint8)
    g = np.zeros(1, dtype=np.float32)
    if lib().orc_quantize_weight(_p(W), N, K, fmt, _p(codes), _p(scales), _p(g)) != 0:
        raise MemoryError("oracle weight quantisation failed")
    return Quantized(codes, scales, g[0], fmt)


def dequant_blocks(q: Quantized, rows: Optional[np.ndarray] = None) -> np.ndarray:
    """val(code) * block scale in fp64 (no tensor scale), [R, K]."""
    codes, scales = q.codes, q.scales
    if rows is not None:
        codes, scales = codes[rows], scales[rows]
    codes = np.ascontiguousarray(codes)
    scales = np.ascontiguousarray(scales)
    R, K2 = codes.shape
    out = np.empty((R, 2 * K2), dtype=np.float64)
    lib().orc_dequant_blocks_f64(_p(codes), _p(scales), q.fmt, R, 2 * K2, _p(out))
    return out


# --------------------------------------------------------------- GEMM ref --

def linear(prep: Prepared, w: Quantized, rows: Optional[np.ndarray] = None,
           cols: Optional[np.ndarray] = None) -> np.ndarray:
    """Two-path FP4 linear in fp64 (Abstract: a sparse FP4 GEMM on the
    backbone plus a dense FP4 GEMM on the residual, one shared weight):
        S_b = Db @ Dw^T,  S_r = Dr @ Dw^T  (block-scaled values, fp64)
        Y   = G_w * (G_b * S_b + G_r * S_r)
    ``rows``/``cols`` restrict the output to a sample."""
    Db = dequant_blocks(prep.bb, rows)
    Dr = dequant_blocks(prep.rs, rows)
    wq = w if cols is None else Quantized(w.codes[cols], w.scales[cols], w.tscale, w.fmt)
    Dw = dequant_blocks(wq)
    Sb = Db @ Dw.T
    Sr = Dr @ Dw.T
    return float(w.tscale) * (float(prep.bb.tscale) * Sb + float(prep.rs.tscale) * Sr)


def linear_abs(prep: Prepared, w: Quantized, rows: Optional[np.ndarray] = None) -> np.ndarray:
    """G_w * (G_b |Db| |Dw|^T + G_r |Dr| |Dw|^T) in fp64: the magnitude sum
    that bounds the rounding error of any fp32 accumulation of the linear
    (recursive summation: |error| <= gamma_n * sum |a_k b_k|)."""
    Db = np.abs(dequant_blocks(prep.bb, rows))
    Dr = np.abs(dequant_blocks(prep.rs, rows))
    Dw = np.abs(dequant_blocks(w))
    return float(w.tscale) * (float(prep.bb.tscale) * (Db @ Dw.T) + float(prep.rs.tscale) * (Dr @ Dw.T))


def gather_rows(prep: Prepared, row_index: np.ndarray) -> Prepared:
    """The prepared rows a grouped linear reads, in dispatch order (tensor
    scales stay those of the whole prepare call)."""
    ri = np.asarray(row_index)
    return Prepared(prep.mask[ri],
                    Quantized(prep.bb.codes[ri], prep.bb.scales[ri], prep.bb.tscale, prep.fmt),
                    Quantized(prep.rs.codes[ri], prep.rs.scales[ri], prep.rs.tscale, prep.fmt),
                    prep.n, prep.m, prep.fmt)


def moe_linear(prep: Prepared, row_index: np.ndarray, offsets: np.ndarray,
               experts: list, rows: Optional[np.ndarray] = None) -> np.ndarray:
    """Grouped form: dispatched row t (token row_index[t]) of group e is
    multiplied by expert e's weight.  Returns Y [T, N] (or the sampled rows,
    given as dispatch positions)."""
    T = len(row_index)
    N = experts[0].codes.shape[0]
    sel = np.arange(T) if rows is None else np.asarray(rows)
    Y = np.zeros((len(sel), N), dtype=np.float64)
    grp = np.searchsorted(np.asarray(offsets), sel, side="right") - 1
    gp = gather_rows(prep, np.asarray(row_index)[sel])
    for e in np.unique(grp):
        idx = np.nonzero(grp == e)[0]
        sub = Prepared(gp.mask[idx], Quantized(gp.bb.codes[idx], gp.bb.scales[idx], gp.bb.tscale, gp.fmt),
                       Quantized(gp.rs.codes[idx], gp.rs.scales[idx], gp.rs.tscale, gp.fmt),
                       gp.n, gp.m, gp.fmt)
        Y[idx] = linear(sub, experts[int(e)])
    return Y


# ----------------------------------------- pair-granular 4:8 backbone ----
# The FP4 sparse tensor-core MMA takes its sparse operand as kept PAIRS of
# FP4 elements: two of the four aligned pairs of every eight elements, with
# a 2-bit pair index each.  An input-adaptive mask of that shape (SharQ
# paper, Abstract: the N:M mask is chosen per input) keeps, in every aligned
# group of eight, the two pairs of largest magnitude.  Reading: a pair's
# magnitude is max(|y_2i|, |y_2i+1|), so the pair holding the group's largest
# entry is always kept (the backbone's block maxima stay those of y); ties go
# to the lower pair index.  The backbone format is MXFP4, whose per-32
# scales the sparse MMA can carry (NVFP4's per-16 scales it cannot).

def mask_pairs(y: np.ndarray) -> np.ndarray:
    """0/1 keep flags [M, K] of the pair-granular 4:8 mask of y [M, K]."""
    y = np.asarray(y, dtype=np.float32)
    M, K = y.shape
    if K % 8:
        raise ValueError("K must be a multiple of 8")
    mag = np.abs(y).reshape(M, K // 8, 4, 2).max(axis=3)          # [M, G, 4] pair magnitudes
    keep_pair = np.zeros((M, K // 8, 4), dtype=np.uint8)
    for i in range(4):
        beaten_by = np.zeros((M, K // 8), dtype=np.int32)
        for j in range(4):
            if j == i:
                continue
            # j outranks i: larger magnitude, or equal and a lower index
            beaten_by += (mag[:, :, j] > mag[:, :, i]) | ((mag[:, :, j] == mag[:, :, i]) & (j < i))
        keep_pair[:, :, i] = beaten_by < 2
    return np.repeat(keep_pair, 2, axis=2).reshape(M, K)


def compress_pairs(codes: np.ndarray, keep: np.ndarray):
    """Zero-filled packed E2M1 codes [M, K/2] and their pair mask -> (kept
    codes [M, K/4]: the two kept pairs of every group of eight in order, one
    byte per pair; pair indices [M, K/16]: per group of eight a nibble with
    the lower kept pair's 2-bit index in bits 1:0 and the higher one's in
    bits 3:2, group 2j in the low nibble of byte j -- the row-major
    metadata the FP4 sparse MMA reads, 4 bits per 8 logical elements)."""
    codes = np.asarray(codes, dtype=np.uint8)
    M, K2 = codes.shape
    K = 2 * K2
    kp = np.asarray(keep, dtype=np.int32).reshape(M, K // 8, 4, 2)[:, :, :, 0]   # [M, G, 4]
    if not np.all(kp.sum(axis=2) == 2):
        raise ValueError("every group of eight must keep exactly two pairs")
    pairs = codes.reshape(M, K // 8, 4)                            # one byte = one pair
    idx = np.argsort(-kp, axis=2, kind="stable")[:, :, :2]         # kept pair indices, ascending
    idx = np.sort(idx, axis=2)
    kept = np.take_along_axis(pairs, idx, axis=2).reshape(M, K // 4)
    nib = (idx[:, :, 0] | (idx[:, :, 1] << 2)).astype(np.uint8)          # [M, K/8]
    meta = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)          # [M, K/16]
    return kept.astype(np.uint8), meta


def decompress_pairs(kept: np.ndarray, meta: np.ndarray) -> np.ndarray:
    """Inverse of compress_pairs: the zero-filled packed codes [M, K/2]."""
    kept = np.asarray(kept, dtype=np.uint8)
    meta = np.asarray(meta, dtype=np.uint8)
    M = meta.shape[0]
    nib = np.stack([meta & 0xF, meta >> 4], axis=2).reshape(M, -1)        # [M, K/8]
    G = nib.shape[1]
    out = np.zeros((M, G, 4), dtype=np.uint8)
    k2 = kept.reshape(M, G, 2)
    for slot in range(2):
        idx = (nib >> (2 * slot)) & 3
        np.put_along_axis(out, idx[:, :, None].astype(np.int64), k2[:, :, slot:slot + 1], axis=2)
    return out.reshape(M, G * 4)


def prepare_pairs(X: np.ndarray, gamma: Optional[np.ndarray], eps: float = 1e-6):
    """The preparation operator with the pair-granular 4:8 mask and an MXFP4
    backbone: y = RMSNorm(X) * gamma (or X), keep = mask_pairs(y), the
    backbone B = keep ? y : 0 quantised to MXFP4 (its zero-filled codes and
    their compressed form), and the residual y - dequant(B) quantised to
    MXFP4.  Returns (Prepared with the zero-filled backbone, kept codes,
    pair indices)."""
    y = normalize(X, gamma, eps)
    keep = mask_pairs(y)
    B = np.where(keep == 1, y, np.float32(0.0)).astype(np.float32)
    bq = quantize(B, "mxfp4", want_D=True)
    r = (y - bq.D).astype(np.float32)                               # one fp32 subtraction each
    rq = quantize(r, "mxfp4")
    M, K = y.shape
    mbits = np.packbits(keep.reshape(M, K // 8, 8), axis=2, bitorder="little").reshape(M, K // 8)
    kept, meta = compress_pairs(bq.codes, keep)
    bq.D = None
    return Prepared(mbits, bq, rq, 4, 8, MXFP4, y, r), kept, meta


# ------------------------------------------------ producer-fused MLP ----
# SharQ paper, Abstract: the preparation is one operator in front of each
# FP4 linear.  For a SwiGLU MLP the down projection's input is
# silu(gate) * up, both halves of the gate+up linear; the fused form computes
# it in that linear's epilogue.  SwiGLU itself is the standard gated unit
# (Shazeer, "GLU Variants Improve Transformer", 2020): silu(x W_g) * (x W_u).

GATE_UP_BLOCK = 64


def interleave_gate_up(W_gate: np.ndarray, W_up: np.ndarray) -> np.ndarray:
    """[I, K] gate and up weights -> the [2I, K] layout of the fused linear:
    rows 128t .. 128t+63 are gate rows 64t .. 64t+63 and rows
    128t+64 .. 128t+127 the up rows with the same indices, so that every
    128-row output tile holds 64 gate columns and their 64 up columns."""
    I, K = W_gate.shape
    if W_up.shape != (I, K) or I % GATE_UP_BLOCK:
        raise ValueError("gate and up must both be [I, K] with I a multiple of 64")
    out = np.empty((2 * I, K), dtype=W_gate.dtype)
    for t in range(I // GATE_UP_BLOCK):
        out[128 * t:128 * t + 64] = W_gate[64 * t:64 * t + 64]
        out[128 * t + 64:128 * t + 128] = W_up[64 * t:64 * t + 64]
    return out


def silu(x) -> np.ndarray:
    """x * sigmoid(x) = x / (1 + e^-x) in fp64 (e^-x overflows to inf for
    x < -709, giving -0)."""
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-x))


def _deinterleave(Y: np.ndarray):
    """Columns of a [R, 2I] gate+up output -> (gate [R, I], up [R, I])."""
    R, N = Y.shape
    t = np.arange(N // 2) // GATE_UP_BLOCK
    j = np.arange(N // 2) % GATE_UP_BLOCK
    return Y[:, 128 * t + j], Y[:, 128 * t + 64 + j]


def swiglu_linear(prep: Prepared, w: Quantized, rows: Optional[np.ndarray] = None) -> np.ndarray:
    """The two-path linear over the interleaved gate+up weight followed by
    the SwiGLU gate, in fp64: H[:, 64t + j] = silu(Y[:, 128t + j]) *
    Y[:, 128t + 64 + j].  Returns [R, I]."""
    g, u = _deinterleave(linear(prep, w, rows))
    return silu(g) * u


def swiglu_parts(prep: Prepared, w: Quantized, rows: Optional[np.ndarray] = None):
    """(gate, up, |gate| bound, |up| bound) of the fused linear in fp64: the
    two halves of the linear and their magnitude sums (linear_abs), from
    which a test derives the rounding bound of an fp32 evaluation."""
    g, u = _deinterleave(linear(prep, w, rows))
    ga, ua = _deinterleave(linear_abs(prep, w, rows))
    return g, u, ga, ua


def moe_swiglu_parts(prep: Prepared, row_index: np.ndarray, offsets: np.ndarray, experts: list):
    """Grouped form of swiglu_parts: (gate, up, |gate| bound, |up| bound) of
    every dispatched row through its own expert's interleaved gate+up weight,
    [T, I] each, in dispatch order."""
    T = len(row_index)
    grp = np.searchsorted(np.asarray(offsets), np.arange(T), side="right") - 1
    I = experts[0].codes.shape[0] // 2
    out = [np.zeros((T, I)) for _ in range(4)]
    for e in np.unique(grp):
        idx = np.nonzero(grp == e)[0]
        parts = swiglu_parts(gather_rows(prep, np.asarray(row_index)[idx]), experts[int(e)])
        for o, p in zip(out, parts):
            o[idx] = p
    return tuple(out)


def moe_swiglu_linear(prep: Prepared, row_index: np.ndarray, offsets: np.ndarray,
                      experts: list) -> np.ndarray:
    """silu(gate) * up of every dispatched row through its own expert, fp64,
    [T, I] in dispatch order."""
    g, u, _, _ = moe_swiglu_parts(prep, row_index, offsets, experts)
    return silu(g) * u


def bf16_rne_from_f64(Y: np.ndarray) -> np.ndarray:
    """RNE(Y64) to bf16 bits, the reference for the bf16 output (fp64 -> bf16
    in one rounding, done exactly through the neighbouring bf16 values)."""
    Y = np.asarray(Y, dtype=np.float64)
    f = Y.astype(np.float32)                    # may round; fix below
    u = f.view(np.uint32).astype(np.uint64)
    lo = (u >> np.uint64(16)) << np.uint64(16)  # truncation toward zero in magnitude
    hi = lo + np.uint64(1 << 16)
    lo32 = lo.astype(np.uint32).view(np.float32).astype(np.float64)
    hi32 = hi.astype(np.uint32).view(np.float32).astype(np.float64)
    dlo = np.abs(Y - lo32)
    dhi = np.abs(hi32 - Y)
    lo_b = (lo >> np.uint64(16)).astype(np.uint16)
    hi_b = (hi >> np.uint64(16)).astype(np.uint16)
    pick_hi = (dhi < dlo) | ((dhi == dlo) & ((lo_b & 1) == 1))
    return np.where(pick_hi, hi_b, lo_b).astype(np.uint16)


__all__ = [n for n in dir() if not n.startswith("_")]
