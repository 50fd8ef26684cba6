"""GPU parity of the producer-fused MLP path: the gate+up linear with the
SwiGLU epilogue (H = silu(gate) * up and max |H|) and the prepare that takes
its amax from that producer.

H tolerance, element by element, against the fp64 oracle h = silu(g) u:
  |H - h| <= ulp_bf16(h) + B,
  B = (1.1 E_g + c |s|) (|u| + E_u) + (|s| + 1.1 E_g) E_u + 2 eps |h|,
with E_g, E_u the fp32 accumulation bounds of the two linear halves (gamma A,
as in the linear tests), s = silu(g), eps = 2^-23 and c = (5 + 1.2 |g|) eps:
|silu'| <= 1.1, and the kernel's fp32 silu (fast exponential: 2 + 1.173 |x|
ulp; one add; fast divide: 2 ulp) is within c of silu relative to it.
Elements beyond one ulp of RNE(h) are counted and must stay rare."""
import numpy as np
import pytest
import torch

import activation_sparsity_prep_b200 as sq
from activation_sparsity_prep_b200 import workloads as wl
import oracle
from tests.sharq_testlib import atoms_to_canonical, to_dev, to_np
from tests.test_linear_parity import bf16_ordered, bf16_ulp, upload_prepared, upload_weight

pytestmark = pytest.mark.gpu

EPS23 = 2.0 ** -23


def bf16_value(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def check_h(H, R, Rw, K, one_acc, rows=None):
    """H (device bf16) against the oracle's SwiGLU of the same operands."""
    got = to_np(H)
    if rows is not None:
        got = got[rows]
    return check_h_parts(got, *oracle.swiglu_parts(R, Rw, rows), K, one_acc)


def check_h_parts(got, g, u, ga, ua, K, one_acc):
    """H bits against h = silu(g) u, with the bounds of g and u."""
    h = oracle.silu(g) * u
    gamma = ((2 if one_acc else 1) * K / 64 + 2) * EPS23
    Eg, Eu = gamma * ga + 2.0 ** -126, gamma * ua + 2.0 ** -126
    s = np.abs(oracle.silu(g))
    c = (5.0 + 1.2 * np.abs(g)) * EPS23
    B = ((1.1 * Eg + c * s) * (np.abs(u) + Eu) + (s + 1.1 * Eg) * Eu
         + 2 * EPS23 * np.abs(h))
    gv = bf16_value(got)
    err = np.abs(gv - h)
    ok = err <= bf16_ulp(h) + B
    assert np.all(ok), f"{int((~ok).sum())} elements beyond the bound; worst ratio " \
                       f"{(err / (bf16_ulp(h) + B)).max():.2f}"
    strict = np.abs(bf16_ordered(got) - bf16_ordered(oracle.bf16_rne_from_f64(h))) <= 1
    frac = 1.0 - strict.mean()
    print(f"{int((~strict).sum())} of {strict.size} elements beyond 1 ulp of RNE(h)")
    assert frac < 1e-3
    return got


def check_amax(H, amax):
    got = to_np(H)
    want = np.max(np.abs(bf16_value(got))) if got.size else 0.0
    assert float(to_np(amax)[0]) == want


SWIGLU_SHAPES = [
    # M, I, K, fmt, residual scale
    (16, 64, 256, "nvfp4", "own"),       # one 128-column tile (decode form)
    (1, 128, 256, "nvfp4", "own"),       # decode form, two tiles
    (64, 192, 512, "nvfp4", "own"),      # decode form, the largest token tile
    (16, 256, 4096, "nvfp4", "own"),     # decode form, 4 tiles x 2-CTA split-K clusters
    (32, 512, 8192, "mxfp4", "own"),     # decode form, 8 tiles x 4-CTA split-K clusters
    (20, 256, 4096, "nvfp4", "shared"),  # decode form, split-K, one accumulator
    (129, 256, 1024, "nvfp4", "own"),
    (300, 320, 2048, "nvfp4", "own"),
    (200, 192, 1024, "mxfp4", "own"),
    (129, 256, 1024, "nvfp4", "shared"),
]


@pytest.mark.parametrize("M,I,K,fmt,rs", SWIGLU_SHAPES)
def test_linear_swiglu_matches_oracle(M, I, K, fmt, rs):
    X = wl.activation("laplace_outlier", 41, M + I, M, K)
    Wi = oracle.interleave_gate_up(wl.weight(41, 1, I, K), wl.weight(41, 2, I, K))
    R = oracle.prepare(X, wl.gamma_ones(K), 1e-6, 2, 4, fmt, residual_scale=rs)
    Rw = oracle.quantize_weight(Wi, fmt)
    P = upload_prepared(R, M, K, fmt)
    P.residual_scale = sq._residual(rs)
    w = upload_weight(Rw, 2 * I, K, fmt)
    H, amax = sq.linear_swiglu(P, w)
    torch.cuda.synchronize()
    assert sq.last_device_status() == 0
    assert H.shape == (M, I)
    check_h(H, R, Rw, K, one_acc=fmt == "mxfp4" or rs == "shared")
    check_amax(H, amax)


def test_linear_swiglu_empty_input_zeroes_amax():
    K, I = 256, 64
    P = sq.Prepared.empty(0, K)
    w = sq.Weight.empty(2 * I, K)
    amax = torch.full((1,), 7.0, device="cuda")
    H, a = sq.linear_swiglu(P, w, amax=amax)
    torch.cuda.synchronize()
    assert H.shape == (0, I) and float(a.item()) == 0.0


def compare_prepared(P, R, M, K, fmt):
    assert np.array_equal(to_np(P.bb_codes), R.bb.codes), "backbone codes"
    assert np.array_equal(to_np(P.rs_codes), R.rs.codes), "residual codes"
    assert np.array_equal(atoms_to_canonical(to_np(P.bb_scales), M, K, fmt), R.bb.scales), "backbone scales"
    assert np.array_equal(atoms_to_canonical(to_np(P.rs_scales), M, K, fmt), R.rs.scales), "residual scales"
    assert to_np(P.bb_tscale).view(np.uint32)[0] == np.float32(R.bb.tscale).view(np.uint32)
    assert to_np(P.rs_tscale).view(np.uint32)[0] == np.float32(R.rs.tscale).view(np.uint32)
    if P.mask is not None:
        assert np.array_equal(to_np(P.mask), R.mask), "mask"


AMAX_CASES = [
    # M, K, dist, n, m, fmt, residual scale
    (16, 256, "normal_outlier", 2, 4, "nvfp4", "own"),
    (1, 4096, "laplace_outlier", 2, 4, "nvfp4", "own"),
    (129, 2048, "student_t", 1, 4, "nvfp4", "own"),
    (300, 512, "laplace_outlier", 4, 8, "nvfp4", "own"),
    (700, 3584, "student_t", 2, 4, "nvfp4", "shared"),
    (3, 768, "laplace_outlier", 1, 2, "nvfp4", "shared"),
    (129, 1024, "laplace_outlier", 2, 4, "mxfp4", "own"),
]


@pytest.mark.parametrize("M,K,dist,n,m,fmt,rs", AMAX_CASES)
def test_prepare_amax_bit_exact(M, K, dist, n, m, fmt, rs):
    """With amax = max |X| (the definition, taken on the host) the outputs
    equal the oracle's no-norm prepare bit for bit."""
    X = wl.activation(dist, 43, M + K, M, K)
    amax = np.max(np.abs(bf16_value(X))).astype(np.float32)
    P = sq.prepare_amax(to_dev(X), torch.tensor([amax], device="cuda"), n, m, fmt, want_mask=True,
                        residual_scale=rs)
    torch.cuda.synchronize()
    assert sq.last_device_status() == 0
    compare_prepared(P, oracle.prepare(X, None, 1e-6, n, m, fmt, residual_scale=rs), M, K, fmt)


@pytest.mark.parametrize("fmt,rs", [("nvfp4", "own"), ("nvfp4", "shared"), ("mxfp4", "own")])
def test_fused_mlp_chain(fmt, rs):
    """prepare -> gate+up with the SwiGLU epilogue -> prepare from the
    producer's amax -> down: H and its amax against the oracle, and the
    down prepare bit-identical to the plain prepare of the same H."""
    M, K, I, Nd = 257, 512, 512, 256       # I is the down projection's K: a multiple of 256
    X = wl.activation("laplace_outlier", 44, 0, M, K)
    g = wl.gamma_ones(K)
    Wi = oracle.interleave_gate_up(wl.weight(44, 1, I, K), wl.weight(44, 2, I, K))
    Wd = wl.weight(44, 3, Nd, I)
    P = sq.prepare(to_dev(X), to_dev(g), 1e-6, 2, 4, fmt, residual_scale=rs)
    w = sq.quantize_weight(to_dev(Wi), fmt)
    wd = sq.quantize_weight(to_dev(Wd), fmt)
    H, amax = sq.linear_swiglu(P, w)
    Pd = sq.prepare_amax(H, amax, 2, 4, fmt, want_mask=True, residual_scale=rs)
    Pref = sq.prepare(H, None, 1e-6, 2, 4, fmt, want_mask=True, residual_scale=rs)
    Y = sq.linear(Pd, wd)
    Yref = sq.linear(Pref, wd)
    torch.cuda.synchronize()
    assert sq.last_device_status() == 0
    R = oracle.prepare(X, g, 1e-6, 2, 4, fmt, residual_scale=rs)
    check_h(H, R, oracle.quantize_weight(Wi, fmt), K, one_acc=fmt == "mxfp4" or rs == "shared")
    check_amax(H, amax)
    for f in ("bb_codes", "bb_scales", "bb_tscale", "rs_codes", "rs_scales", "rs_tscale", "mask"):
        assert torch.equal(getattr(Pd, f), getattr(Pref, f)), f
    assert torch.equal(Y, Yref)


def test_fused_mlp_full_size_llama_prefill():
    """The Llama-8B gate+up projection at M = 2048 with the SwiGLU epilogue:
    48 sampled rows x all 14336 features against the oracle, the amax over
    the whole H, and the down prepare from that amax bit-identical to the
    plain prepare of H."""
    W = wl.WORKLOADS["llama8b"]
    L = next(l for l in W.linears if l.name == "gate_up")
    M, I = 2048, L.N // 2
    d = wl.linear_inputs(W, L, M)
    Wi = oracle.interleave_gate_up(d["W"][:I], d["W"][I:])
    P = sq.prepare(to_dev(d["X"]), to_dev(d["gamma"]), wl.EPS, 2, 4, "nvfp4")
    w = sq.quantize_weight(to_dev(Wi), "nvfp4")
    H, amax = sq.linear_swiglu(P, w)
    Pd = sq.prepare_amax(H, amax)
    Pref = sq.prepare(H, None)
    torch.cuda.synchronize()
    assert sq.last_device_status() == 0
    check_amax(H, amax)
    for f in ("bb_codes", "bb_scales", "bb_tscale", "rs_codes", "rs_scales", "rs_tscale"):
        assert torch.equal(getattr(Pd, f), getattr(Pref, f)), f
    del Pd, Pref, w
    R = oracle.prepare(d["X"], d["gamma"], wl.EPS, 2, 4, "nvfp4")
    rows = np.sort(np.random.default_rng(7).choice(M, 48, replace=False))
    check_h(H, R, oracle.quantize_weight(Wi, "nvfp4"), L.K, one_acc=False, rows=rows)


def stacked_swiglu_weights(cfg, E, I, K, fmt):
    Wis = [oracle.interleave_gate_up(wl.weight(cfg, 10 + e, I, K), wl.weight(cfg, 20 + e, I, K))
           for e in range(E)]
    w = sq.Weight.empty(2 * I, K, fmt, E=E)
    sb = sq.scale_bytes(2 * I, K, fmt)
    for e, Wi in enumerate(Wis):
        we = sq.Weight(w.codes[e], w.scales[e * sb:(e + 1) * sb], w.tensor_scale[e:e + 1], 2 * I, K, w.fmt)
        sq.quantize_weight(to_dev(Wi), fmt, out=we)
    return Wis, w


MOE_CASES = [
    # tokens, experts, top-k, K, I, fmt, residual scale, routing
    (200, 3, 2, 512, 128, "nvfp4", "own", "uniform"),
    (70, 5, 2, 256, 64, "nvfp4", "own", "uneven"),       # experts 1, 2 (and most of 4) empty
    (96, 4, 2, 256, 192, "mxfp4", "own", "uniform"),
    (200, 3, 2, 512, 128, "nvfp4", "shared", "uniform"),
]


@pytest.mark.parametrize("T_tok,E,topk,K,I,fmt,rs,route", MOE_CASES)
def test_moe_linear_swiglu_matches_oracle(T_tok, E, topk, K, I, fmt, rs, route):
    X = wl.activation("laplace_outlier", 45, 0, T_tok, K)
    g = wl.gamma_ones(K)
    if route == "uneven":
        ex = np.zeros((T_tok, 2), dtype=np.int32)
        ex[:, 1] = 3
        ex[:5, 1] = 4
    else:
        ex = wl.routing(45, T_tok, E, topk)
    ri, off = wl.group_by_expert(ex.astype(np.int32), E)
    Wis, w = stacked_swiglu_weights(45, E, I, K, fmt)
    P = sq.prepare(to_dev(X), to_dev(g), wl.EPS, 2, 4, fmt, residual_scale=rs)
    H, amax = sq.moe_linear_swiglu(P, torch.from_numpy(ri).cuda(), torch.from_numpy(off).cuda(), w)
    torch.cuda.synchronize()
    assert sq.last_device_status() == 0
    assert H.shape == (len(ri), I)
    R = oracle.prepare(X, g, wl.EPS, 2, 4, fmt, residual_scale=rs)
    Rws = [oracle.quantize_weight(Wi, fmt) for Wi in Wis]
    check_h_parts(to_np(H), *oracle.moe_swiglu_parts(R, ri, off, Rws), K,
                  one_acc=fmt == "mxfp4" or rs == "shared")
    check_amax(H, amax)


def test_fused_moe_layer_full_size():
    """The Qwen3-30B-A3B-shaped expert layer with the SwiGLU epilogue on the
    grouped gate+up: H of 4 sampled experts against the oracle, the amax
    over all 32768 dispatched rows, and the down prepare from that amax
    bit-identical to the plain prepare of H."""
    W = wl.WORKLOADS["qwen3moe"]
    L = W.linears[0]
    T, E, topk = W.moe["T"], W.moe["E"], W.moe["topk"]
    I = L.N // 2
    ri, off = wl.group_by_expert(wl.routing(W.cfg, T, E, topk), E)
    X = wl.activation(W.dist, W.cfg, L.index, T, L.K)
    g = wl.gamma_ones(L.K)
    Wis = {}
    w = sq.Weight.empty(L.N, L.K, "nvfp4", E=E)
    sb = sq.scale_bytes(L.N, L.K, "nvfp4")
    sampled = (0, 37, 64, 127)
    for e in range(E):
        Wb = wl.weight(W.cfg * 1000, 100 + e, L.N, L.K)
        Wi = oracle.interleave_gate_up(Wb[:I], Wb[I:])
        if e in sampled:
            Wis[e] = Wi
        we = sq.Weight(w.codes[e], w.scales[e * sb:(e + 1) * sb], w.tensor_scale[e:e + 1], L.N, L.K, w.fmt)
        sq.quantize_weight(to_dev(Wi), "nvfp4", out=we)
    P = sq.prepare(to_dev(X), to_dev(g), wl.EPS)
    H, amax = sq.moe_linear_swiglu(P, torch.from_numpy(ri).cuda(), torch.from_numpy(off).cuda(), w)
    Pd = sq.prepare_amax(H, amax)
    Pref = sq.prepare(H, None)
    torch.cuda.synchronize()
    assert sq.last_device_status() == 0
    check_amax(H, amax)
    for f in ("bb_codes", "bb_scales", "bb_tscale", "rs_codes", "rs_scales", "rs_tscale"):
        assert torch.equal(getattr(Pd, f), getattr(Pref, f)), f
    R = oracle.prepare(X, g, wl.EPS)
    got = to_np(H)
    for e in sampled:
        idx = np.arange(off[e], off[e + 1])
        if len(idx) == 0:
            continue
        parts = oracle.swiglu_parts(oracle.gather_rows(R, ri[idx]), oracle.quantize_weight(Wis[e]))
        check_h_parts(got[idx], *parts, L.K, one_acc=False)
