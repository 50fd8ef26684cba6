"""GPU parity at decode-sized M on the Llama-3.1-8B-shaped linears, every
row of every output checked against the fp64 oracle.

M <= 64 runs the swapped (weight-streaming) decode linear.  At these shapes
it reaches the paths the small parity cases do not:
* gate+up (N = 28672): 224 output tiles on 148 SMs, so each persistent CTA
  walks several tiles, carrying its pipeline stage counter and both
  tensor-memory accumulator buffers from one tile to the next;
* qkv, o and down (N = 6144 / 4096): fewer tiles than SMs, so clusters of
  CTAs split each tile along K and add their partials in rank order.
M = 128 runs the row-tiled kernel with one (full) 128-row tile.
The prepare of each input is also compared bit for bit.  Tolerances are
those of tests/test_linear_parity.py."""
import numpy as np
import pytest
import torch

import activation_sparsity_prep_b200 as sq
from activation_sparsity_prep_b200 import workloads as wl
import oracle
from tests.sharq_testlib import to_dev
from tests.test_linear_parity import check
from tests.test_mlp_fused_parity import check_amax, check_h, compare_prepared

pytestmark = pytest.mark.gpu

LLAMA = wl.WORKLOADS["llama8b"]
_weights = {}


def _weight(lin, fmt):
    """(oracle weight, device weight) of one Llama linear, quantised once."""
    key = (lin, fmt)
    if key not in _weights:
        L = LLAMA.linears[lin]
        Wb = wl.weight(LLAMA.cfg, L.index, L.N, L.K)
        _weights.clear()                       # keep one full-size weight alive at a time
        _weights[key] = (oracle.quantize_weight(Wb, fmt), sq.quantize_weight(to_dev(Wb), fmt))
    return _weights[key]


def _run(lin, M, fmt="nvfp4", residual="own"):
    L = LLAMA.linears[lin]
    X = wl.activation(LLAMA.dist, LLAMA.cfg, L.index, M, L.K)
    g = wl.gamma_ones(L.K) if L.norm else None
    Rw, w = _weight(lin, fmt)
    P = sq.prepare(to_dev(X), None if g is None else to_dev(g), wl.EPS, 2, 4, fmt, want_mask=True,
                   residual_scale=residual)
    Y32 = sq.linear(P, w, out_fp32=True)
    Ybf = sq.linear(P, w)
    torch.cuda.synchronize()
    assert sq.last_device_status() == 0
    R = oracle.prepare(X, g, wl.EPS, 2, 4, fmt, residual_scale=residual)
    compare_prepared(P, R, M, L.K, fmt)
    one = fmt == "mxfp4" or residual == "shared"
    check(Y32, Ybf, oracle.linear(R, Rw), oracle.linear_abs(R, Rw), L.K, one_acc=one)


@pytest.mark.parametrize("M", [1, 16, 128])
@pytest.mark.parametrize("lin", range(4), ids=[L.name for L in LLAMA.linears])
def test_llama_decode_every_row(M, lin):
    _run(lin, M)


@pytest.mark.parametrize("M,fmt,residual", [(1, "nvfp4", "shared"), (16, "nvfp4", "shared"),
                                            (64, "nvfp4", "own"), (1, "mxfp4", "own"),
                                            (16, "mxfp4", "own"), (64, "mxfp4", "own")])
def test_decode_more_tiles_than_sms(M, fmt, residual):
    """gate+up (224 tiles): the persistent multi-tile loop in both formats,
    with one accumulator (MXFP4, shared scale) or two (own scale)."""
    _run(2, M, fmt, residual)


@pytest.mark.parametrize("M", [17, 64])
def test_decode_cluster_split_qkv(M):
    """qkv (48 tiles, split-K clusters) at M = 17 (a 32-row token tile,
    ragged) and M = 64 (the largest decode tile)."""
    _run(0, M)


def test_swiglu_llama_gate_up_decode():
    """The SwiGLU epilogue at M = 16 on the Llama gate+up shape (K = 4096,
    2 x 14336 interleaved rows): every row of H against the oracle."""
    L = LLAMA.linears[2]
    M, I = 16, L.N // 2
    X = wl.activation(LLAMA.dist, LLAMA.cfg, L.index, M, L.K)
    Wb = wl.weight(LLAMA.cfg, L.index, L.N, L.K)
    Wi = oracle.interleave_gate_up(Wb[:I], Wb[I:])
    _weights.clear()
    Rw = oracle.quantize_weight(Wi)
    w = sq.quantize_weight(to_dev(Wi))
    g = wl.gamma_ones(L.K)
    P = sq.prepare(to_dev(X), to_dev(g), wl.EPS)
    H, amax = sq.linear_swiglu(P, w)
    torch.cuda.synchronize()
    assert sq.last_device_status() == 0
    R = oracle.prepare(X, g, wl.EPS)
    check_h(H, R, Rw, L.K, one_acc=False)
    check_amax(H, amax)
