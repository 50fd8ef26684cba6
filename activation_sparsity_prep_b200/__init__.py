"""SharQ hot path on B200 (sm_100a): Python binding of libsharq.

Thin ctypes marshalling over the C ABI declared in ``include/sharq.h``.
PyTorch supplies device memory and the current CUDA stream; every step of
the computation runs in the library's CUDA kernels.  There is no CPU
fallback: without the compiled library every call raises.

SharQ paper, Abstract: a fused preparation operator (normalisation, an
input-adaptive N:M mask, an FP4 backbone and an FP4 residual taken against
the dequantised backbone) feeds a sparse FP4 GEMM and a dense FP4 GEMM that
share one FP4 weight payload.  For a SwiGLU MLP the gate+up linear can apply
the gate in its epilogue (linear_swiglu / moe_linear_swiglu) and hand max |H|
to the down projection's prepare (prepare_amax), which then skips its own
amax pass.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass
from typing import Optional

__all__ = [
    "NVFP4", "MXFP4", "SharqError", "load_sharq_ops", "scale_bytes", "pair_meta_bytes",
    "prepare_workspace_bytes", "Weight", "Prepared", "quantize_weight",
    "prepare", "prepare_layernorm", "prepare_amax", "prepare_noalloc", "linear",
    "linear_swiglu", "interleave_gate_up", "moe_linear", "moe_linear_swiglu",
    "moe_workspace_bytes", "selftest_wait_timeout", "selftest_prepare_timeout", "last_device_status",
]

NVFP4, MXFP4 = 0, 1
_FMT = {"nvfp4": NVFP4, "mxfp4": MXFP4}
_BLOCK = {NVFP4: 16, MXFP4: 32}

_STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration",
           3: "CUDA error", 4: "device wait timed out"}


class SharqError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {_STATUS.get(status, status)} (status {status})")
        self.status = status


class _Weight(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("tensor_scale", ctypes.c_void_p), ("N", ctypes.c_int),
                ("K", ctypes.c_int), ("fmt", ctypes.c_int)]


class _Prepared(ctypes.Structure):
    _fields_ = [("bb_codes", ctypes.c_void_p), ("bb_scales", ctypes.c_void_p),
                ("bb_tscale", ctypes.c_void_p), ("rs_codes", ctypes.c_void_p),
                ("rs_scales", ctypes.c_void_p), ("rs_tscale", ctypes.c_void_p),
                ("mask", ctypes.c_void_p), ("M", ctypes.c_int), ("K", ctypes.c_int),
                ("n", ctypes.c_int), ("m", ctypes.c_int), ("fmt", ctypes.c_int),
                ("residual_scale", ctypes.c_int), ("bb_meta", ctypes.c_void_p)]


_lib = None
_lock = threading.Lock()
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsharq.so")


def load_sharq_ops(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load libsharq.so (building it with nvcc when it is missing or older
    than its sources).  Raises if the library cannot be produced."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if build_if_missing:
            from . import build as _build
            if not _build.up_to_date():
                _build.build()
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libsharq.so not found at {LIB_PATH}; run "
                              "python -m activation_sparsity_prep_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        L.sharq_status_string.argtypes = [I]
        L.sharq_status_string.restype = ctypes.c_char_p
        L.sharq_scale_bytes.argtypes = [I64, I, I]
        L.sharq_scale_bytes.restype = SZ
        L.sharq_prepare_workspace_bytes.argtypes = [I64, I, I]
        L.sharq_prepare_workspace_bytes.restype = SZ
        L.sharq_pair_meta_bytes.argtypes = [I64, I]
        L.sharq_pair_meta_bytes.restype = SZ
        L.sharq_quantize_weight.argtypes = [P, ctypes.POINTER(_Weight), P, SZ, P]
        L.sharq_quantize_weight.restype = I
        L.sharq_prepare.argtypes = [P, P, ctypes.c_float, ctypes.POINTER(_Prepared), P, SZ, P]
        L.sharq_prepare.restype = I
        L.sharq_prepare_layernorm.argtypes = [P, P, P, ctypes.c_float, ctypes.POINTER(_Prepared), P, SZ, P]
        L.sharq_prepare_layernorm.restype = I
        L.sharq_linear.argtypes = [ctypes.POINTER(_Prepared), ctypes.POINTER(_Weight), P, I, P]
        L.sharq_linear.restype = I
        L.sharq_linear_swiglu.argtypes = [ctypes.POINTER(_Prepared), ctypes.POINTER(_Weight), P, P, P]
        L.sharq_linear_swiglu.restype = I
        L.sharq_prepare_amax.argtypes = [P, P, ctypes.POINTER(_Prepared), P, SZ, P]
        L.sharq_prepare_amax.restype = I
        L.sharq_moe_workspace_bytes.argtypes = [I64, I, I, I]
        L.sharq_moe_workspace_bytes.restype = SZ
        L.sharq_moe_linear.argtypes = [ctypes.POINTER(_Prepared), P, P, I, I64,
                                       ctypes.POINTER(_Weight), P, I, P, SZ, P]
        L.sharq_moe_linear.restype = I
        L.sharq_moe_linear_swiglu.argtypes = [ctypes.POINTER(_Prepared), P, P, I, I64,
                                              ctypes.POINTER(_Weight), P, P, P, SZ, P]
        L.sharq_moe_linear_swiglu.restype = I
        L.sharq_prepare_noalloc.argtypes = [P, P, ctypes.c_float, ctypes.POINTER(_Prepared), P]
        L.sharq_prepare_noalloc.restype = I
        L.sharq_selftest_wait_timeout.argtypes = [P, I64, P]
        L.sharq_selftest_wait_timeout.restype = I
        L.sharq_selftest_prepare_timeout.argtypes = [P, ctypes.POINTER(_Prepared), P, SZ, I64, P]
        L.sharq_selftest_prepare_timeout.restype = I
        L.sharq_last_device_status.argtypes = [P]
        L.sharq_last_device_status.restype = I
        _lib = L
        return L


def _fmt(fmt) -> int:
    return _FMT[fmt] if isinstance(fmt, str) else int(fmt)


_RESIDUAL = {"own": 0, "shared": 1}


def _residual(rs) -> int:
    return _RESIDUAL[rs] if isinstance(rs, str) else int(rs)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _check(fn: str, st: int):
    if st != 0:
        raise SharqError(fn, st)



# ------------------------------------------------------- argument checks --
# The C ABI sees raw pointers only, so a tensor of the wrong shape, dtype or
# device would be read or written past its end on the GPU.  Every wrapper
# checks its tensors here first and raises ValueError.

def _need(cond: bool, msg: str):
    if not cond:
        raise ValueError(msg)


def _check_tensor(name: str, t, shape, dtype, device=None):
    """t must be a contiguous tensor of exactly `shape` and `dtype` on
    `device` (when given)."""
    _need(t is not None, f"{name} is required")
    _need(tuple(t.shape) == tuple(shape), f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    _need(t.dtype == dtype, f"{name} has dtype {t.dtype}, expected {dtype}")
    _need(t.is_contiguous(), f"{name} must be contiguous")
    if device is not None:
        _need(t.device == device, f"{name} is on {t.device}, expected {device}")


def _check_min(name: str, t, numel: int, dtype, device):
    """A flat buffer of at least `numel` elements of `dtype` on `device`."""
    _need(t is not None, f"{name} is required")
    _need(t.dtype == dtype, f"{name} has dtype {t.dtype}, expected {dtype}")
    _need(t.is_contiguous(), f"{name} must be contiguous")
    _need(t.numel() >= numel, f"{name} holds {t.numel()} elements, needs {numel}")
    _need(t.device == device, f"{name} is on {t.device}, expected {device}")


def _check_input(X, gamma=None, beta=None):
    """X bf16 [M, K] on a CUDA device; gamma / beta bf16 [K] beside it."""
    import torch
    _need(X is not None and X.dim() == 2, "X must be a 2-D tensor [M, K]")
    _need(X.is_cuda, "X must be a CUDA tensor")
    _check_tensor("X", X, X.shape, torch.bfloat16)
    K = X.shape[1]
    for nm, v in (("gamma", gamma), ("beta", beta)):
        if v is not None:
            _check_tensor(nm, v, (K,), torch.bfloat16, X.device)


def _check_prepared(p: "Prepared", M: int, K: int, fmt: int, device):
    """A caller-given Prepared must describe [M, K] in `fmt` with buffers
    large enough for it, on `device`."""
    import torch
    _need((p.M, p.K, p.fmt) == (M, K, fmt),
          f"out describes M={p.M}, K={p.K}, fmt={p.fmt}; the call needs M={M}, K={K}, fmt={fmt}")
    _check_prepared_buffers(p, device)


def _check_prepared_buffers(p: "Prepared", device=None):
    import torch
    dev = device if device is not None else p.bb_codes.device
    sb = scale_bytes(p.M, p.K, p.fmt)
    u8 = torch.uint8
    _check_min("bb_codes", p.bb_codes, p.M * p.K // (4 if p.bb_meta is not None else 2), u8, dev)
    if p.bb_meta is not None:
        _check_min("bb_meta", p.bb_meta, pair_meta_bytes(p.M, p.K), u8, dev)
    _check_min("rs_codes", p.rs_codes, p.M * p.K // 2, u8, dev)
    _check_min("bb_scales", p.bb_scales, sb, u8, dev)
    _check_min("rs_scales", p.rs_scales, sb, u8, dev)
    _check_min("bb_tscale", p.bb_tscale, 1, torch.float32, dev)
    _check_min("rs_tscale", p.rs_tscale, 1, torch.float32, dev)
    if p.mask is not None:
        _check_min("mask", p.mask, p.M * p.K // 8, u8, dev)
    return dev


def _check_weight(w: "Weight", K: int, fmt: int, device, E: int = 1):
    import torch
    _need(w.K == K, f"weight K={w.K} does not match the activations' K={K}")
    _need(w.fmt == fmt, f"weight format {w.fmt} does not match the activations' {fmt}")
    _check_min("weight codes", w.codes, E * w.N * K // 2, torch.uint8, device)
    _check_min("weight scales", w.scales, E * scale_bytes(w.N, K, fmt), torch.uint8, device)
    _check_min("weight tensor_scale", w.tensor_scale, E, torch.float32, device)


def _check_output(name: str, Y, shape, dtype, device):
    _check_tensor(name, Y, shape, dtype, device)


def scale_bytes(rows: int, K: int, fmt="nvfp4") -> int:
    return int(load_sharq_ops().sharq_scale_bytes(rows, K, _fmt(fmt)))


def pair_meta_bytes(M: int, K: int) -> int:
    """Bytes of the pair metadata of a compressed (pair-granular 4:8) backbone."""
    return int(load_sharq_ops().sharq_pair_meta_bytes(M, K))


def prepare_workspace_bytes(M: int, K: int, fmt="nvfp4") -> int:
    return int(load_sharq_ops().sharq_prepare_workspace_bytes(M, K, _fmt(fmt)))


@dataclass
class Weight:
    """Shared FP4 weight payload (device tensors)."""
    codes: "object"          # uint8 [N, K/2] (or [E, N, K/2])
    scales: "object"         # uint8 MMA-ready atoms
    tensor_scale: "object"   # fp32 [1] (or [E])
    N: int
    K: int
    fmt: int
    E: int = 1

    def _c(self) -> _Weight:
        return _Weight(_ptr(self.codes), _ptr(self.scales), _ptr(self.tensor_scale),
                       self.N, self.K, self.fmt)

    @staticmethod
    def empty(N: int, K: int, fmt="nvfp4", device="cuda", E: int = 1) -> "Weight":
        import torch
        f = _fmt(fmt)
        sb = scale_bytes(N, K, f)
        shape = (N, K // 2) if E == 1 else (E, N, K // 2)
        return Weight(torch.empty(shape, dtype=torch.uint8, device=device),
                      torch.empty((E * sb,), dtype=torch.uint8, device=device),
                      torch.empty((E,), dtype=torch.float32, device=device), N, K, f, E)


@dataclass
class Prepared:
    """Backbone and residual FP4 operands produced by prepare()."""
    bb_codes: "object"
    bb_scales: "object"
    bb_tscale: "object"
    rs_codes: "object"
    rs_scales: "object"
    rs_tscale: "object"
    mask: "object"
    M: int
    K: int
    n: int
    m: int
    fmt: int
    residual_scale: int = 0      # 0 own, 1 shared with the backbone (NVFP4)
    bb_meta: "object" = None     # pair metadata: the backbone is the compressed pair-granular 4:8 form

    def _c(self) -> _Prepared:
        return _Prepared(_ptr(self.bb_codes), _ptr(self.bb_scales), _ptr(self.bb_tscale),
                         _ptr(self.rs_codes), _ptr(self.rs_scales), _ptr(self.rs_tscale),
                         _ptr(self.mask), self.M, self.K, self.n, self.m, self.fmt,
                         self.residual_scale, _ptr(self.bb_meta))

    @staticmethod
    def empty(M: int, K: int, n: int = 2, m: int = 4, fmt="nvfp4", want_mask: bool = False,
              device="cuda", residual_scale="own", pairs: bool = False) -> "Prepared":
        """pairs: the pair-granular 4:8 backbone of the FP4 sparse MMA (MXFP4):
        bb_codes holds the kept pairs [M, K/4] and bb_meta their indices."""
        import torch
        f = _fmt(fmt)
        if pairs:
            _need(f == MXFP4, "the pair-granular backbone is MXFP4")
            n, m = 4, 8
        sb = scale_bytes(M, K, f)
        u8 = dict(dtype=torch.uint8, device=device)
        return Prepared(torch.empty((M, K // 4 if pairs else K // 2), **u8), torch.empty((sb,), **u8),
                        torch.empty((1,), dtype=torch.float32, device=device),
                        torch.empty((M, K // 2), **u8), torch.empty((sb,), **u8),
                        torch.empty((1,), dtype=torch.float32, device=device),
                        torch.empty((M, K // 8), **u8) if want_mask else None,
                        M, K, n, m, f, _residual(residual_scale),
                        torch.empty((pair_meta_bytes(M, K),), **u8) if pairs else None)


def _workspace(M: int, K: int, fmt: int, ws=None, device="cuda"):
    import torch
    need = prepare_workspace_bytes(M, K, fmt)
    if ws is None or ws.numel() < need:
        ws = torch.empty((max(need, 256),), dtype=torch.uint8, device=device)
    return ws


def quantize_weight(W, fmt="nvfp4", out: Optional[Weight] = None, ws=None, stream=None) -> Weight:
    """W: bf16 [N, K] device tensor -> shared FP4 payload."""
    L = load_sharq_ops()
    _check_input(W)
    N, K = W.shape
    f = _fmt(fmt)
    if out is not None:
        _need((out.N, out.K, out.fmt) == (N, K, f), "out does not describe W's shape and format")
        _check_weight(out, K, f, W.device)
    w = out if out is not None else Weight.empty(N, K, f, device=W.device)
    ws = _workspace(N, K, f, ws, W.device)
    cw = w._c()
    _check("sharq_quantize_weight",
           L.sharq_quantize_weight(W.data_ptr(), ctypes.byref(cw), ws.data_ptr(), ws.numel(),
                                   _stream(stream)))
    return w


def prepare(X, gamma=None, eps: float = 1e-6, n: int = 2, m: int = 4, fmt="nvfp4",
            want_mask: bool = False, out: Optional[Prepared] = None, ws=None,
            stream=None, residual_scale="own", pairs: bool = False) -> Prepared:
    """X: bf16 [M, K] device tensor; gamma: bf16 [K] or None (no norm).
    residual_scale: "own" or "shared" (ignored when ``out`` is given: the
    output's own setting applies).  pairs: the pair-granular 4:8 backbone
    (MXFP4; n and m are then 4 and 8), compressed for the sparse MMA."""
    if pairs:
        fmt, n, m = "mxfp4", 4, 8
    L = load_sharq_ops()
    _check_input(X, gamma)
    M, K = X.shape
    f = _fmt(fmt)
    if out is not None:
        _check_prepared(out, M, K, f, X.device)
    p = out if out is not None else Prepared.empty(M, K, n, m, f, want_mask, device=X.device,
                                                   residual_scale=residual_scale, pairs=pairs)
    ws = _workspace(M, K, f, ws, X.device)
    cp = p._c()
    _check("sharq_prepare",
           L.sharq_prepare(X.data_ptr(), _ptr(gamma), float(eps), ctypes.byref(cp),
                           ws.data_ptr(), ws.numel(), _stream(stream)))
    return p


def prepare_layernorm(X, gamma, beta=None, eps: float = 1e-6, n: int = 2, m: int = 4,
                      fmt="nvfp4", want_mask: bool = False, out: Optional[Prepared] = None,
                      ws=None, stream=None, residual_scale="own") -> Prepared:
    """prepare() with LayerNorm (gamma required, beta optional) instead of
    RMSNorm in front of the mask."""
    L = load_sharq_ops()
    _check_input(X, gamma, beta)
    M, K = X.shape
    f = _fmt(fmt)
    if out is not None:
        _check_prepared(out, M, K, f, X.device)
    p = out if out is not None else Prepared.empty(M, K, n, m, f, want_mask, device=X.device,
                                                   residual_scale=residual_scale)
    ws = _workspace(M, K, f, ws, X.device)
    cp = p._c()
    _check("sharq_prepare_layernorm",
           L.sharq_prepare_layernorm(X.data_ptr(), _ptr(gamma), _ptr(beta), float(eps),
                                     ctypes.byref(cp), ws.data_ptr(), ws.numel(), _stream(stream)))
    return p


NOALLOC_MAX_ROWS = 262144


def prepare_noalloc(X, gamma=None, eps: float = 1e-6, out: Optional[Prepared] = None,
                    n: int = 2, m: int = 4, fmt="nvfp4", stream=None) -> Prepared:
    """prepare() through the entry point that allocates no device memory
    (fixed in-library scratch, M <= NOALLOC_MAX_ROWS).  The output buffers
    are the caller's: pass ``out`` when the caller cannot allocate either."""
    L = load_sharq_ops()
    _check_input(X, gamma)
    M, K = X.shape
    f = _fmt(fmt)
    if out is not None:
        _check_prepared(out, M, K, f, X.device)
    p = out if out is not None else Prepared.empty(M, K, n, m, f, device=X.device)
    cp = p._c()
    _check("sharq_prepare_noalloc",
           L.sharq_prepare_noalloc(X.data_ptr(), _ptr(gamma), float(eps), ctypes.byref(cp),
                                   _stream(stream)))
    return p


def linear(x: Prepared, w: Weight, out_fp32: bool = False, out=None, stream=None):
    """Two-path FP4 linear: Y = G_w (G_b A_b W^T + G_r A_r W^T)."""
    import torch
    L = load_sharq_ops()
    dev = _check_prepared_buffers(x)
    _check_weight(w, x.K, x.fmt, dev)
    dt = torch.float32 if out_fp32 else torch.bfloat16
    if out is not None:
        _check_output("out", out, (x.M, w.N), dt, dev)
    Y = out if out is not None else torch.empty((x.M, w.N), dtype=dt, device=dev)
    cx, cw = x._c(), w._c()
    _check("sharq_linear", L.sharq_linear(ctypes.byref(cx), ctypes.byref(cw), Y.data_ptr(),
                                          1 if out_fp32 else 0, _stream(stream)))
    return Y


def interleave_gate_up(W_gate, W_up):
    """[I, K] gate and up weights (bf16 tensors) -> the [2I, K] layout that
    linear_swiglu expects: per 128 rows, 64 gate rows then the 64 up rows with
    the same indices.  An offline layout step of the weight, done once."""
    import torch
    I, K = W_gate.shape
    if tuple(W_up.shape) != (I, K) or I % 64:
        raise ValueError("gate and up must both be [I, K] with I a multiple of 64")
    return torch.stack((W_gate.reshape(I // 64, 64, K), W_up.reshape(I // 64, 64, K)), 1).reshape(2 * I, K)


def linear_swiglu(x: Prepared, w: Weight, out=None, amax=None, stream=None):
    """Gate+up linear with the SwiGLU epilogue: returns (H bf16 [M, w.N/2],
    amax fp32 [1] = max |H|), for w quantised from interleave_gate_up(...)."""
    import torch
    L = load_sharq_ops()
    dev = _check_prepared_buffers(x)
    _check_weight(w, x.K, x.fmt, dev)
    if out is not None:
        _check_output("out", out, (x.M, w.N // 2), torch.bfloat16, dev)
    if amax is not None:
        _check_output("amax", amax, (1,), torch.float32, dev)
    H = out if out is not None else torch.empty((x.M, w.N // 2), dtype=torch.bfloat16, device=dev)
    a = amax if amax is not None else torch.empty((1,), dtype=torch.float32, device=dev)
    cx, cw = x._c(), w._c()
    _check("sharq_linear_swiglu", L.sharq_linear_swiglu(ctypes.byref(cx), ctypes.byref(cw), H.data_ptr(),
                                                        a.data_ptr(), _stream(stream)))
    return H, a


def prepare_amax(X, amax, n: int = 2, m: int = 4, fmt="nvfp4", want_mask: bool = False,
                 out: Optional[Prepared] = None, ws=None, stream=None, residual_scale="own") -> Prepared:
    """prepare() of a no-norm input whose max |X| the producer has already
    taken (amax: fp32 [1] device tensor, e.g. from linear_swiglu)."""
    L = load_sharq_ops()
    _check_input(X)
    M, K = X.shape
    f = _fmt(fmt)
    if out is not None:
        _check_prepared(out, M, K, f, X.device)
    p = out if out is not None else Prepared.empty(M, K, n, m, f, want_mask, device=X.device,
                                                   residual_scale=residual_scale)
    import torch
    _check_tensor("amax", amax, (1,), torch.float32, X.device)
    ws = _workspace(M, K, f, ws, X.device)
    cp = p._c()
    _check("sharq_prepare_amax",
           L.sharq_prepare_amax(X.data_ptr(), amax.data_ptr(), ctypes.byref(cp), ws.data_ptr(),
                                ws.numel(), _stream(stream)))
    return p


def _check_grouped(x: Prepared, row_index, offsets, w: Weight, T: int):
    """Shapes of the grouped form's index arrays and stacked weight; returns
    the device."""
    import torch
    dev = _check_prepared_buffers(x)
    _need(offsets is not None and offsets.dim() == 1 and offsets.numel() >= 2,
          "offsets must be an int32 [E+1] tensor with E >= 1")
    E = int(offsets.numel()) - 1
    _check_tensor("offsets", offsets, (E + 1,), torch.int32, dev)
    if row_index is not None:
        _check_tensor("row_index", row_index, (T,), torch.int32, dev)
    else:
        _need(T == x.M, f"without row_index the dispatched rows are the prepared rows: T={T}, M={x.M}")
    _need(w.E == E, f"the weight stacks {w.E} experts, offsets describe {E}")
    _check_weight(w, x.K, x.fmt, dev, E)
    return dev


def moe_workspace_bytes(T: int, E: int, K: int, fmt="nvfp4") -> int:
    return int(load_sharq_ops().sharq_moe_workspace_bytes(T, E, K, _fmt(fmt)))


def moe_linear(x: Prepared, row_index, offsets, w: Weight, out_fp32: bool = False, out=None,
               ws=None, T: Optional[int] = None, stream=None):
    """Grouped two-path linear.  row_index: int32 [T] device tensor (or None:
    dispatched row t is prepared row t); offsets: int32 [E+1] device tensor;
    w: E stacked expert weights (Weight.empty(..., E=E))."""
    import torch
    L = load_sharq_ops()
    if T is None:
        T = int(row_index.numel()) if row_index is not None else x.M
    E = int(offsets.numel()) - 1
    dt = torch.float32 if out_fp32 else torch.bfloat16
    dev = _check_grouped(x, row_index, offsets, w, T)
    if out is not None:
        _check_output("out", out, (T, w.N), dt, dev)
    Y = out if out is not None else torch.empty((T, w.N), dtype=dt, device=dev)
    need = moe_workspace_bytes(T, E, x.K, x.fmt)
    if ws is None or ws.numel() < need:
        ws = torch.empty((max(need, 256),), dtype=torch.uint8, device=dev)
    cx, cw = x._c(), w._c()
    _check("sharq_moe_linear",
           L.sharq_moe_linear(ctypes.byref(cx), _ptr(row_index), offsets.data_ptr(), E, T,
                              ctypes.byref(cw), Y.data_ptr(), 1 if out_fp32 else 0,
                              ws.data_ptr(), ws.numel(), _stream(stream)))
    return Y


def moe_linear_swiglu(x: Prepared, row_index, offsets, w: Weight, out=None, amax=None, ws=None,
                      T: Optional[int] = None, stream=None):
    """Grouped gate+up linear with the SwiGLU epilogue over E stacked
    interleaved expert weights: returns (H bf16 [T, w.N/2] in dispatch order,
    amax fp32 [1] = max |H|)."""
    import torch
    L = load_sharq_ops()
    if T is None:
        T = int(row_index.numel()) if row_index is not None else x.M
    E = int(offsets.numel()) - 1
    dev = _check_grouped(x, row_index, offsets, w, T)
    if out is not None:
        _check_output("out", out, (T, w.N // 2), torch.bfloat16, dev)
    if amax is not None:
        _check_output("amax", amax, (1,), torch.float32, dev)
    H = out if out is not None else torch.empty((T, w.N // 2), dtype=torch.bfloat16, device=dev)
    a = amax if amax is not None else torch.empty((1,), dtype=torch.float32, device=dev)
    need = moe_workspace_bytes(T, E, x.K, x.fmt)
    if ws is None or ws.numel() < need:
        ws = torch.empty((max(need, 256),), dtype=torch.uint8, device=dev)
    cx, cw = x._c(), w._c()
    _check("sharq_moe_linear_swiglu",
           L.sharq_moe_linear_swiglu(ctypes.byref(cx), _ptr(row_index), offsets.data_ptr(), E, T,
                                     ctypes.byref(cw), H.data_ptr(), a.data_ptr(), ws.data_ptr(),
                                     ws.numel(), _stream(stream)))
    return H, a


def selftest_wait_timeout(limit_us: int = 10000, stream=None) -> None:
    """Run the bounded-wait self-test: a grid wait that one block never
    joins gives up after limit_us and records a timeout, which the next
    last_device_status() reports (SHARQ_ERR_TIMEOUT = 4)."""
    import torch
    L = load_sharq_ops()
    ws = torch.zeros((16,), dtype=torch.uint8, device="cuda")
    _check("sharq_selftest_wait_timeout", L.sharq_selftest_wait_timeout(ws.data_ptr(), int(limit_us),
                                                                        _stream(stream)))


def selftest_prepare_timeout(X, limit_us: int = 10000, stream=None) -> Prepared:
    """Run the real NVFP4 prepare of X (no norm, own residual scale) with one
    block that never arrives at its grid barriers and each barrier wait
    limited to limit_us: the waits give up and record a timeout, which the
    next last_device_status() reports.  The returned outputs are unspecified."""
    L = load_sharq_ops()
    _check_input(X)
    M, K = X.shape
    p = Prepared.empty(M, K, device=X.device)
    ws = _workspace(M, K, NVFP4, None, X.device)
    cp = p._c()
    _check("sharq_selftest_prepare_timeout",
           L.sharq_selftest_prepare_timeout(X.data_ptr(), ctypes.byref(cp), ws.data_ptr(), ws.numel(),
                                            int(limit_us), _stream(stream)))
    return p


def last_device_status(stream=None) -> int:
    """Synchronise and return (then clear) the device status word."""
    return int(load_sharq_ops().sharq_last_device_status(_stream(stream)))
