"""GPU parity of the grouped (mixture-of-experts) two-path linear against the
fp64 oracle's per-expert loop, with the same tolerances as the plain linear
(relative Frobenius <= 1e-5 on fp32, summation-bound element check, bf16
within one ulp outside cancellation points)."""
import numpy as np
import pytest
import torch

import activation_sparsity_prep_b200 as sq
from activation_sparsity_prep_b200 import workloads as wl
import oracle
from tests.sharq_testlib import to_dev, to_np
from tests.test_linear_parity import check

pytestmark = pytest.mark.gpu


def stacked_weights(cfg, E, N, K, fmt="nvfp4"):
    Ws = [wl.weight(cfg, 100 + e, N, K) for e in range(E)]
    w = sq.Weight.empty(N, K, fmt, E=E)
    sb = sq.scale_bytes(N, K, fmt)
    for e, W in enumerate(Ws):
        we = sq.Weight(w.codes[e], w.scales[e * sb:(e + 1) * sb], w.tensor_scale[e:e + 1], N, K, w.fmt)
        sq.quantize_weight(to_dev(W), fmt, out=we)
    return Ws, w


def dispatch(experts, E):
    ri, off = wl.group_by_expert(experts.astype(np.int32), E)
    return ri, off


def run_case(T_tok, E, topk, K, N, experts=None, fmt="nvfp4", seed=51, residual_scale="own"):
    X = wl.activation("laplace_outlier", seed, 0, T_tok, K)
    g = wl.gamma_ones(K)
    if experts is None:
        experts = wl.routing(seed, T_tok, E, topk)
    ri, off = dispatch(experts, E)
    Ws, w = stacked_weights(seed, E, N, K, fmt)
    P = sq.prepare(to_dev(X), to_dev(g), wl.EPS, 2, 4, fmt, residual_scale=residual_scale)
    ri_d = torch.from_numpy(ri).cuda()
    off_d = torch.from_numpy(off).cuda()
    Y32 = sq.moe_linear(P, ri_d, off_d, w, out_fp32=True)
    Ybf = sq.moe_linear(P, ri_d, off_d, w)
    torch.cuda.synchronize()
    assert sq.last_device_status() == 0
    R = oracle.prepare(X, g, wl.EPS, 2, 4, fmt, residual_scale=residual_scale)
    Rws = [oracle.quantize_weight(W, fmt) for W in Ws]
    Y64 = oracle.moe_linear(R, ri, off, Rws)
    # the summation bound of every dispatched row, from its own expert
    A = np.zeros_like(Y64)
    grp = np.searchsorted(off, np.arange(len(ri)), side="right") - 1
    for e in range(E):
        idx = np.nonzero(grp == e)[0]
        if len(idx):
            A[idx] = oracle.linear_abs(oracle.gather_rows(R, ri[idx]), Rws[e])
    return check(Y32, Ybf, Y64, A, K, one_acc=fmt == "mxfp4" or residual_scale == "shared")


def test_moe_small_uniform_routing():
    run_case(T_tok=200, E=3, topk=2, K=256, N=256)   # ~133 rows per expert: two m-tiles each


def test_moe_uneven_and_empty_experts():
    T = 70
    ex = np.zeros((T, 2), dtype=np.int32)
    ex[:, 0] = 0                       # expert 0 gets every token (70 rows)
    ex[:, 1] = 3                       # expert 3 too; experts 1, 2, 4 stay empty
    ex[:5, 1] = 4                      # expert 4 gets five rows
    run_case(T_tok=T, E=5, topk=2, K=512, N=384, experts=ex)


def test_moe_mxfp4():
    run_case(T_tok=96, E=4, topk=2, K=256, N=128, fmt="mxfp4")


def test_moe_shared_residual_scale():
    run_case(T_tok=200, E=3, topk=2, K=512, N=256, residual_scale="shared")


def test_moe_single_expert_equals_linear():
    M, K, N = 300, 512, 256
    X = wl.activation("laplace_outlier", 52, 0, M, K)
    P = sq.prepare(to_dev(X), to_dev(wl.gamma_ones(K)), wl.EPS)
    w = sq.quantize_weight(to_dev(wl.weight(52, 0, N, K)))
    off = torch.tensor([0, M], dtype=torch.int32, device="cuda")
    Yl = sq.linear(P, w, out_fp32=True)
    Ym = sq.moe_linear(P, None, off, w, out_fp32=True)
    ri = torch.arange(M, dtype=torch.int32, device="cuda")
    Yg = sq.moe_linear(P, ri, off, w, out_fp32=True)
    torch.cuda.synchronize()
    assert torch.equal(Yl, Ym) and torch.equal(Yl, Yg)


def test_moe_row_index_none_reads_rows_in_order():
    """row_index = NULL: the prepared operand is already in dispatch order
    (e.g. the down projection's input); the result equals the gathered form."""
    T_tok, E, topk, K, N = 64, 4, 2, 256, 128
    X = wl.activation("laplace_outlier", 53, 0, T_tok, K)
    ri, off = dispatch(wl.routing(53, T_tok, E, topk), E)
    Ws, w = stacked_weights(53, E, N, K)
    P = sq.prepare(to_dev(X), None, wl.EPS)
    Xd = X[ri]                                       # rows in dispatch order
    Pd = sq.prepare(to_dev(Xd), None, wl.EPS)        # same tensor scales: every row appears
    off_d = torch.from_numpy(off).cuda()
    Y1 = sq.moe_linear(P, torch.from_numpy(ri).cuda(), off_d, w, out_fp32=True)
    Y2 = sq.moe_linear(Pd, None, off_d, w, out_fp32=True)
    torch.cuda.synchronize()
    assert torch.equal(P.bb_tscale, Pd.bb_tscale)
    assert torch.equal(Y1, Y2)


@pytest.mark.parametrize("lin", [0, 1])
def test_moe_full_size_qwen3_layer_sampled(lin):
    """Qwen3-30B-A3B-shaped expert layer: 4096 tokens, 128 experts, top-8
    (32768 dispatched rows); gate+up (K 2048, N 1536) reads the token rows
    through row_index, down (K 768, N 2048) reads rows in dispatch order.
    Rows of four sampled experts are checked against the oracle."""
    Wl = wl.WORKLOADS["qwen3moe"]
    L = Wl.linears[lin]
    T, E, topk = Wl.moe["T"], Wl.moe["E"], Wl.moe["topk"]
    ex = wl.routing(Wl.cfg, T, E, topk)
    ri, off = dispatch(ex, E)
    Ws, w = stacked_weights(Wl.cfg * 1000 + lin, E, L.N, L.K)
    off_d = torch.from_numpy(off).cuda()
    if lin == 0:
        X = wl.activation(Wl.dist, Wl.cfg, L.index, T, L.K)
        g = wl.gamma_ones(L.K)
        P = sq.prepare(to_dev(X), to_dev(g), wl.EPS)
        Y32 = sq.moe_linear(P, torch.from_numpy(ri).cuda(), off_d, w, out_fp32=True)
        Ybf = sq.moe_linear(P, torch.from_numpy(ri).cuda(), off_d, w)
        R = oracle.prepare(X, g, wl.EPS)
        rows_src = ri
    else:
        X = wl.activation(Wl.dist, Wl.cfg, L.index, T * topk, L.K)   # already in dispatch order
        P = sq.prepare(to_dev(X), None, wl.EPS)
        Y32 = sq.moe_linear(P, None, off_d, w, out_fp32=True)
        Ybf = sq.moe_linear(P, None, off_d, w)
        R = oracle.prepare(X, None, wl.EPS)
        rows_src = np.arange(T * topk, dtype=np.int32)
    torch.cuda.synchronize()
    assert sq.last_device_status() == 0
    Y32n, Ybfn = to_np(Y32), to_np(Ybf)
    for e in (0, 37, 64, 127):
        idx = np.arange(off[e], off[e + 1])
        Rw = oracle.quantize_weight(Ws[e])
        sub = oracle.gather_rows(R, rows_src[idx])
        check(torch.from_numpy(Y32n[idx]), torch.from_numpy(Ybfn[idx].view(np.int16)).view(torch.bfloat16),
              oracle.linear(sub, Rw), oracle.linear_abs(sub, Rw), L.K)
