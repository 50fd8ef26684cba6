"""Guard bytes around every buffer a kernel writes: a stand-in for a memory
checker, which these tests do not run.

Each output and workspace of a call is placed in the middle of a larger
device buffer whose first and last 4 KiB (and the payload itself) are filled
with the byte 0xA5 beforehand.  After the call (1) both guard regions must
still hold the pattern, so nothing was written past either end of the
buffer, and (2) the payload must equal, byte for byte, what the same call
writes into buffers the binding allocates itself, so every byte the call
owns was written (none still holds the poison).  The shapes are odd on
purpose: row counts that are not multiples of 128 (or of the decode tile),
and both the row-tiled and the weight-streaming forms of the linear."""
import numpy as np
import pytest
import torch

import activation_sparsity_prep_b200 as sq
from activation_sparsity_prep_b200 import workloads as wl
from tests.sharq_testlib import to_dev

pytestmark = pytest.mark.gpu

GUARD = 4096        # bytes of pattern on each side; keeps the payload 256-byte aligned
PATTERN = 0xA5
U8, F32, BF16 = torch.uint8, torch.float32, torch.bfloat16


class Guarded:
    """A payload of `numel` elements of `dtype` inside a pattern-filled buffer."""

    def __init__(self, numel, dtype, shape=None):
        self.nbytes = numel * torch.empty(0, dtype=dtype).element_size()
        self.raw = torch.full((2 * GUARD + self.nbytes,), PATTERN, dtype=U8, device="cuda")
        t = self.raw[GUARD:GUARD + self.nbytes].view(dtype)
        self.t = t.view(shape) if shape is not None else t

    def intact(self) -> bool:
        return bool((self.raw[:GUARD] == PATTERN).all()) and \
            bool((self.raw[GUARD + self.nbytes:] == PATTERN).all())


def same_bytes(a, b) -> bool:
    return torch.equal(a.reshape(-1).view(U8), b.reshape(-1).view(U8))


def check(guarded: dict, ref: dict):
    """Guards intact; payloads equal to the reference call's outputs (a
    workspace, which has no reference, only has its guards checked)."""
    torch.cuda.synchronize()
    assert sq.last_device_status() == 0
    for name, g in guarded.items():
        assert g.intact(), f"{name}: bytes written outside the buffer"
        if name in ref:
            assert same_bytes(g.t, ref[name]), f"{name}: differs from the same call into plain buffers"


def guarded_prepared(M, K, n, m, fmt, want_mask=False, rs="own", pairs=False):
    f = sq._FMT[fmt]
    sb = sq.scale_bytes(M, K, f)
    G = {"bb_codes": Guarded(M * K // (4 if pairs else 2), U8), "bb_scales": Guarded(sb, U8),
         "bb_tscale": Guarded(1, F32), "rs_codes": Guarded(M * K // 2, U8),
         "rs_scales": Guarded(sb, U8), "rs_tscale": Guarded(1, F32)}
    if want_mask:
        G["mask"] = Guarded(M * K // 8, U8)
    if pairs:
        G["bb_meta"] = Guarded(sq.pair_meta_bytes(M, K), U8)
    P = sq.Prepared(G["bb_codes"].t, G["bb_scales"].t, G["bb_tscale"].t, G["rs_codes"].t,
                    G["rs_scales"].t, G["rs_tscale"].t, G["mask"].t if want_mask else None,
                    M, K, n, m, f, sq._residual(rs), G["bb_meta"].t if pairs else None)
    return P, G


def prepared_outputs(P) -> dict:
    d = {k: getattr(P, k) for k in ("bb_codes", "bb_scales", "bb_tscale", "rs_codes",
                                    "rs_scales", "rs_tscale", "mask", "bb_meta")}
    return {k: v for k, v in d.items() if v is not None}


def guarded_weight(N, K, fmt, E=1):
    f = sq._FMT[fmt]
    sb = sq.scale_bytes(N, K, f)
    G = {"codes": Guarded(E * N * K // 2, U8, (N, K // 2) if E == 1 else (E, N, K // 2)),
         "scales": Guarded(E * sb, U8), "tensor_scale": Guarded(E, F32)}
    return sq.Weight(G["codes"].t, G["scales"].t, G["tensor_scale"].t, N, K, f, E), G


def quantized(Wbits, fmt):
    """Weight quantised into guarded buffers (weight, its workspace), checked
    against the binding's own allocation."""
    N, K = Wbits.shape
    W = to_dev(Wbits)
    ref = sq.quantize_weight(W, fmt)
    w, G = guarded_weight(N, K, fmt)
    ws = Guarded(sq.prepare_workspace_bytes(N, K, fmt), U8)
    sq.quantize_weight(W, fmt, out=w, ws=ws.t)
    check({**G, "ws": ws}, {"codes": ref.codes, "scales": ref.scales, "tensor_scale": ref.tensor_scale})
    return w


PREPARE_CASES = [
    # M, K, gamma, n, m, fmt, residual scale, pairs
    (1, 256, True, 2, 4, "nvfp4", "own", False),
    (17, 4096, False, 2, 4, "nvfp4", "own", False),      # decode form with cluster split-K
    (129, 1024, True, 2, 4, "nvfp4", "shared", False),
    (300, 512, True, 2, 4, "mxfp4", "own", False),
    (33, 512, False, 1, 4, "nvfp4", "own", False),
    (65, 512, True, 4, 8, "mxfp4", "own", True),
]


@pytest.mark.parametrize("M,K,gamma,n,m,fmt,rs,pairs", PREPARE_CASES)
def test_prepare_and_linear_stay_inside_their_buffers(M, K, gamma, n, m, fmt, rs, pairs):
    X = to_dev(wl.activation("laplace_outlier", 61, M, M, K))
    g = to_dev(wl.gamma_random(61, 0, K)) if gamma else None
    ref = sq.prepare(X, g, wl.EPS, n, m, fmt, want_mask=not pairs, residual_scale=rs, pairs=pairs)
    P, G = guarded_prepared(M, K, n, m, "mxfp4" if pairs else fmt, not pairs, rs, pairs)
    ws = Guarded(sq.prepare_workspace_bytes(M, K, fmt), U8)
    sq.prepare(X, g, wl.EPS, n, m, fmt, out=P, ws=ws.t, pairs=pairs)
    check({**G, "ws": ws}, prepared_outputs(ref))

    N = 384
    w = quantized(wl.weight(61, 1, N, K), "mxfp4" if pairs else fmt)
    for fp32 in (False, True):
        Yref = sq.linear(ref, w, out_fp32=fp32)
        Y = Guarded(M * N, F32 if fp32 else BF16, (M, N))
        sq.linear(P, w, out_fp32=fp32, out=Y.t)
        check({"Y": Y}, {"Y": Yref})


def test_wide_tile_linear_stays_inside_its_buffer():
    """Enough 256-wide output tiles to fill whole waves of the SMs, so the
    one-accumulator launch takes the 128 x 256 tile."""
    M, K, N = 200, 256, 37888
    X = to_dev(wl.activation("laplace_outlier", 66, 0, M, K))
    P = sq.prepare(X, to_dev(wl.gamma_ones(K)), wl.EPS, 2, 4, "mxfp4")
    w = quantized(wl.weight(66, 1, N, K), "mxfp4")
    Yref = sq.linear(P, w)
    Y = Guarded(M * N, BF16, (M, N))
    sq.linear(P, w, out=Y.t)
    check({"Y": Y}, {"Y": Yref})


@pytest.mark.parametrize("with_beta,fmt", [(True, "nvfp4"), (False, "mxfp4")])
def test_layernorm_prepare_stays_inside_its_buffers(with_beta, fmt):
    M, K = 33, 256
    X = to_dev(wl.activation("laplace_outlier", 62, 0, M, K))
    g = to_dev(wl.gamma_random(62, 0, K))
    b = to_dev(wl.beta_random(62, 0, K)) if with_beta else None
    ref = sq.prepare_layernorm(X, g, b, wl.EPS, 2, 4, fmt, want_mask=True)
    P, G = guarded_prepared(M, K, 2, 4, fmt, True)
    ws = Guarded(sq.prepare_workspace_bytes(M, K, fmt), U8)
    sq.prepare_layernorm(X, g, b, wl.EPS, 2, 4, fmt, out=P, ws=ws.t)
    check({**G, "ws": ws}, prepared_outputs(ref))


@pytest.mark.parametrize("M", [16, 130])
def test_swiglu_linear_and_amax_prepare_stay_inside_their_buffers(M):
    K, I = 512, 256
    X = to_dev(wl.activation("laplace_outlier", 63, 0, M, K))
    Wi = sq.interleave_gate_up(to_dev(wl.weight(63, 1, I, K)), to_dev(wl.weight(63, 2, I, K)))
    w = sq.quantize_weight(Wi, "nvfp4")
    P = sq.prepare(X, to_dev(wl.gamma_ones(K)), wl.EPS)
    Href, aref = sq.linear_swiglu(P, w)
    H, a = Guarded(M * I, BF16, (M, I)), Guarded(1, F32)
    sq.linear_swiglu(P, w, out=H.t, amax=a.t)
    check({"H": H, "amax": a}, {"H": Href, "amax": aref})

    ref = sq.prepare_amax(Href, aref, want_mask=True)
    Pd, G = guarded_prepared(M, I, 2, 4, "nvfp4", True)
    ws = Guarded(sq.prepare_workspace_bytes(M, I, "nvfp4"), U8)
    sq.prepare_amax(Href, aref, out=Pd, ws=ws.t)
    check({**G, "ws": ws}, prepared_outputs(ref))


def stacked(E, N, K, fmt, cfg, swiglu=False):
    w = sq.Weight.empty(N, K, fmt, E=E)
    sb = sq.scale_bytes(N, K, fmt)
    for e in range(E):
        if swiglu:
            W = sq.interleave_gate_up(to_dev(wl.weight(cfg, 10 + e, N // 2, K)),
                                      to_dev(wl.weight(cfg, 20 + e, N // 2, K)))
        else:
            W = to_dev(wl.weight(cfg, 100 + e, N, K))
        we = sq.Weight(w.codes[e], w.scales[e * sb:(e + 1) * sb], w.tensor_scale[e:e + 1], N, K, w.fmt)
        sq.quantize_weight(W, fmt, out=we)
    return w


@pytest.mark.parametrize("swiglu", [False, True])
def test_grouped_linear_stays_inside_its_buffers(swiglu):
    T_tok, E, K, N = 70, 5, 256, 256
    ex = np.zeros((T_tok, 2), dtype=np.int32)
    ex[:, 1] = 3
    ex[:5, 1] = 4                                   # experts 1 and 2 empty, 4 nearly so
    ri, off = wl.group_by_expert(ex, E)
    T = len(ri)
    X = to_dev(wl.activation("laplace_outlier", 64, 0, T_tok, K))
    P = sq.prepare(X, to_dev(wl.gamma_ones(K)), wl.EPS)
    w = stacked(E, N, K, "nvfp4", 64, swiglu)
    ri_d, off_d = torch.from_numpy(ri).cuda(), torch.from_numpy(off).cuda()
    ws = Guarded(sq.moe_workspace_bytes(T, E, K, "nvfp4"), U8)
    if swiglu:
        Href, aref = sq.moe_linear_swiglu(P, ri_d, off_d, w)
        H, a = Guarded(T * (N // 2), BF16, (T, N // 2)), Guarded(1, F32)
        sq.moe_linear_swiglu(P, ri_d, off_d, w, out=H.t, amax=a.t, ws=ws.t)
        check({"H": H, "amax": a, "ws": ws}, {"H": Href, "amax": aref})
    else:
        Yref = sq.moe_linear(P, ri_d, off_d, w)
        Y = Guarded(T * N, BF16, (T, N))
        sq.moe_linear(P, ri_d, off_d, w, out=Y.t, ws=ws.t)
        check({"Y": Y, "ws": ws}, {"Y": Yref})


def test_noalloc_prepare_stays_inside_its_buffers():
    M, K = 77, 512
    X = to_dev(wl.activation("laplace_outlier", 65, 0, M, K))
    g = to_dev(wl.gamma_ones(K))
    ref = sq.prepare(X, g, wl.EPS, want_mask=True)
    P, G = guarded_prepared(M, K, 2, 4, "nvfp4", True)
    sq.prepare_noalloc(X, g, wl.EPS, out=P)
    check(G, prepared_outputs(ref))
