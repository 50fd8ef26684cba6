"""Pins of the oracle's producer-fused MLP functions (CPU only).

SwiGLU is the standard gated unit silu(x W_g) * (x W_u) (Shazeer, "GLU
Variants Improve Transformer", 2020); the SharQ paper (Abstract) places the
preparation in front of every FP4 linear, so the down projection's input is
that product.  The pins check the oracle against an independent closed form
of the sigmoid, a hand-placed interleave, and a brute-force evaluation with
the gate/up pairing written out index by index.
"""
import math

import numpy as np
import pytest

import oracle
from activation_sparsity_prep_b200 import workloads as wl


def sigmoid_tanh(x: float) -> float:
    """sigmoid(x) through other closed forms than the oracle's 1 / (1 + e^-x):
    (1 + tanh(x / 2)) / 2 for x >= 0 and e^x / (1 + e^x) below zero (where
    1 + tanh would cancel)."""
    if x >= 0:
        return 0.5 * (1.0 + math.tanh(0.5 * x))
    e = math.exp(x)
    return e / (1.0 + e)


def test_silu_matches_tanh_form():
    xs = np.concatenate([np.linspace(-30, 30, 2001), [-1e-300, 1e-300, 1e-8, -1e-8, 700.0]])
    got = oracle.silu(xs)
    want = np.array([x * sigmoid_tanh(x) for x in xs])
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-300)


def test_silu_special_values():
    assert oracle.silu(0.0) == 0.0
    assert oracle.silu(50.0) == 50.0                    # e^-50 is below half an ulp of 1
    v = oracle.silu(-800.0)                             # e^800 overflows: -800 / inf
    assert v == 0.0 and np.signbit(v)
    # silu(x) - silu(-x) = x (sigmoid(x) + sigmoid(-x) = 1)
    for x in (0.25, 1.0, 3.5, 17.0):
        assert abs(oracle.silu(x) - oracle.silu(-x) - x) <= 1e-15 * max(1.0, x)


def test_interleave_places_rows():
    I, K = 128, 256
    Wg = np.arange(I * K, dtype=np.uint16).reshape(I, K)
    Wu = (np.arange(I * K, dtype=np.uint32) + 40000).astype(np.uint16).reshape(I, K)
    W = oracle.interleave_gate_up(Wg, Wu)
    assert W.shape == (2 * I, K)
    assert np.array_equal(W[0], Wg[0]) and np.array_equal(W[63], Wg[63])
    assert np.array_equal(W[64], Wu[0]) and np.array_equal(W[127], Wu[63])
    assert np.array_equal(W[128], Wg[64]) and np.array_equal(W[191], Wg[127])
    assert np.array_equal(W[192], Wu[64]) and np.array_equal(W[255], Wu[127])
    with pytest.raises(ValueError):
        oracle.interleave_gate_up(Wg[:96], Wu[:96])


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_swiglu_linear_brute_force(fmt):
    M, K, I = 3, 256, 128
    X = wl.activation("laplace_outlier", 91, 0, M, K)
    P = oracle.prepare(X, None, 1e-6, 2, 4, fmt)
    Wg = wl.weight(91, 1, I, K)
    Wu = wl.weight(91, 2, I, K)
    Wq = oracle.quantize_weight(oracle.interleave_gate_up(Wg, Wu), fmt)
    H = oracle.swiglu_linear(P, Wq)
    assert H.shape == (M, I)
    Db = oracle.dequant_blocks(P.bb)
    Dr = oracle.dequant_blocks(P.rs)
    Dw = oracle.dequant_blocks(Wq)
    gw, gb, gr = float(Wq.tscale), float(P.bb.tscale), float(P.rs.tscale)

    def y(mrow, wrow):
        sb = sum(Db[mrow, k] * Dw[wrow, k] for k in range(K))
        sr = sum(Dr[mrow, k] * Dw[wrow, k] for k in range(K))
        return gw * (gb * sb + gr * sr)

    worst = 0.0
    for mrow in range(M):
        for j in range(I):
            gate_row = (j // 64) * 128 + (j % 64)
            yg, yu = y(mrow, gate_row), y(mrow, gate_row + 64)
            want = yg * sigmoid_tanh(yg) * yu
            worst = max(worst, abs(H[mrow, j] - want) / max(abs(want), 1e-30))
            if j in (5, 70):
                # the planted swap (gate and up exchanged) must be visible
                swapped = yu * sigmoid_tanh(yu) * yg
                assert abs(swapped - want) > 1e-6 * abs(want)
    assert worst < 1e-9


def test_swiglu_parts_bound_the_linear():
    M, K, I = 4, 512, 64
    X = wl.activation("laplace_outlier", 92, 0, M, K)
    P = oracle.prepare(X, None, 1e-6, 2, 4, "nvfp4")
    Wq = oracle.quantize_weight(oracle.interleave_gate_up(wl.weight(92, 1, I, K), wl.weight(92, 2, I, K)))
    g, u, ga, ua = oracle.swiglu_parts(P, Wq)
    assert np.all(ga >= np.abs(g)) and np.all(ua >= np.abs(u))
    np.testing.assert_array_equal(oracle.silu(g) * u, oracle.swiglu_linear(P, Wq))


def test_moe_swiglu_is_the_per_expert_loop():
    """The grouped oracle equals a loop of the plain SwiGLU linear over
    dispatched rows, each through its own expert."""
    T_tok, E, K, I = 12, 3, 256, 64
    X = wl.activation("laplace_outlier", 93, 0, T_tok, K)
    P = oracle.prepare(X, None, 1e-6, 2, 4, "nvfp4")
    ex = wl.routing(93, T_tok, E, 2)
    ri, off = wl.group_by_expert(ex.astype(np.int32), E)
    Wq = [oracle.quantize_weight(oracle.interleave_gate_up(wl.weight(93, 10 + e, I, K),
                                                           wl.weight(93, 20 + e, I, K))) for e in range(E)]
    H = oracle.moe_swiglu_linear(P, ri, off, Wq)
    for t in range(len(ri)):
        e = int(np.searchsorted(off, t, side="right") - 1)
        want = oracle.swiglu_linear(oracle.gather_rows(P, ri[t:t + 1]), Wq[e])[0]
        np.testing.assert_array_equal(H[t], want)


def test_moe_swiglu_parts_are_the_per_row_parts():
    """All four grouped parts (gate, up and their magnitude-sum bounds, which
    set the grouped SwiGLU test's tolerance) equal the plain parts of each
    dispatched row through its own expert."""
    T_tok, E, K, I = 10, 4, 256, 64
    X = wl.activation("laplace_outlier", 94, 0, T_tok, K)
    P = oracle.prepare(X, wl.gamma_ones(K), 1e-6, 2, 4, "nvfp4")
    ex = np.zeros((T_tok, 2), dtype=np.int32)
    ex[:, 1] = 3
    ex[:4, 0] = 1                                   # expert 2 empty
    ri, off = wl.group_by_expert(ex, E)
    Wq = [oracle.quantize_weight(oracle.interleave_gate_up(wl.weight(94, 10 + e, I, K),
                                                           wl.weight(94, 20 + e, I, K))) for e in range(E)]
    parts = oracle.moe_swiglu_parts(P, ri, off, Wq)
    for t in range(len(ri)):
        e = int(np.searchsorted(off, t, side="right") - 1)
        want = oracle.swiglu_parts(oracle.gather_rows(P, ri[t:t + 1]), Wq[e])
        for got, w in zip(parts, want):
            np.testing.assert_array_equal(got[t], w[0])
