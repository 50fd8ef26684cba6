"""GPU parity at the benchmark's full sizes, through the calls bench.py times:
every prepare output compared bit for bit with the oracle on the whole
tensor, and 48 seeded rows x all N of each linear against the fp64 oracle.
Qwen2.5-7B-shaped linears at M = 4096, the format/mask sweep at M = 16384
and the LayerNorm DiT block at M = 8192 (the Llama M = 2048 linears and the
grouped Qwen3 layer are covered in the per-kernel test files)."""
import numpy as np
import pytest
import torch

import activation_sparsity_prep_b200 as sq
from activation_sparsity_prep_b200 import workloads as wl
import oracle
from tests.sharq_testlib import atoms_to_canonical, to_dev, to_np
from tests.test_linear_parity import check

pytestmark = pytest.mark.gpu


def _run(W, L, M, fmt="nvfp4", n=2, m=4, residual="own"):
    d = wl.linear_inputs(W, L, M)
    g = None if d["gamma"] is None else to_dev(d["gamma"])
    if d["norm"] == "layernorm":
        P = sq.prepare_layernorm(to_dev(d["X"]), g, to_dev(d["beta"]), wl.EPS, n, m, fmt,
                                 residual_scale=residual)
    else:
        P = sq.prepare(to_dev(d["X"]), g, wl.EPS, n, m, fmt, residual_scale=residual)
    w = sq.quantize_weight(to_dev(d["W"]), fmt)
    Y32 = sq.linear(P, w, out_fp32=True)
    Ybf = sq.linear(P, w)
    torch.cuda.synchronize()
    assert sq.last_device_status() == 0
    R = oracle.prepare(d["X"], d["gamma"], wl.EPS, n, m, fmt, residual_scale=residual,
                       norm=d["norm"], beta=d["beta"])
    assert np.array_equal(to_np(P.bb_codes), R.bb.codes), "backbone codes"
    assert np.array_equal(to_np(P.rs_codes), R.rs.codes), "residual codes"
    assert np.array_equal(atoms_to_canonical(to_np(P.bb_scales), M, L.K, fmt), R.bb.scales)
    assert np.array_equal(atoms_to_canonical(to_np(P.rs_scales), M, L.K, fmt), R.rs.scales)
    assert to_np(P.bb_tscale).view(np.uint32)[0] == np.float32(R.bb.tscale).view(np.uint32)
    assert to_np(P.rs_tscale).view(np.uint32)[0] == np.float32(R.rs.tscale).view(np.uint32)
    del P
    Rw = oracle.quantize_weight(d["W"], fmt)
    rows = np.sort(np.random.default_rng(L.index + M).choice(M, 48, replace=False))
    one = fmt == "mxfp4" or residual == "shared"
    check(Y32, Ybf, oracle.linear(R, Rw, rows=rows), oracle.linear_abs(R, Rw, rows=rows), L.K,
          rows=rows, one_acc=one)


@pytest.mark.parametrize("lin", range(3))
def test_qwen7b_prefill(lin):
    W = wl.WORKLOADS["qwen7b"]
    _run(W, W.linears[lin], 4096)


@pytest.mark.parametrize("fmt,nm", [(f, nm) for f in ("nvfp4", "mxfp4") for nm in ((2, 4), (1, 4), (4, 8))])
def test_sweep(fmt, nm):
    W = wl.WORKLOADS["sweep"]
    _run(W, W.linears[0], 16384, fmt, *nm)


def test_sweep_shared_residual_scale():
    W = wl.WORKLOADS["sweep"]
    _run(W, W.linears[0], 16384, residual="shared")


@pytest.mark.parametrize("lin", range(4))
def test_wan_dit_layernorm_block(lin):
    W = wl.WORKLOADS["wan_dit"]
    _run(W, W.linears[lin], 8192)
