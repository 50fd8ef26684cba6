"""GPU parity of the pair-granular 4:8 backbone (the operand of the FP4
sparse tensor-core MMA) against the oracle's prepare_pairs: in every aligned
group of eight the two pairs of largest pair magnitude are kept, the MXFP4
backbone is stored compressed (kept pairs' code bytes in order) with 2-bit
pair indices, and the residual is taken against the dequantised backbone.
Everything is compared bit for bit: compressed codes, metadata (through the
atom layout of include/sharq.h), scales, residual codes and scales, tensor
scales and the exported element mask."""
import numpy as np
import pytest
import torch

import activation_sparsity_prep_b200 as sq
from activation_sparsity_prep_b200 import workloads as wl
import oracle
from tests.sharq_testlib import (atom_index, atoms_to_canonical, meta_atom_index,
                                 meta_atoms_to_canonical, to_dev, to_np)

pytestmark = pytest.mark.gpu

CASES = [
    # M, K, dist, gamma
    (16, 256, "normal_outlier", "ones"),
    (1, 512, "laplace_outlier", None),
    (129, 1024, "laplace_outlier", "ones"),
    (33, 768, "student_t", "random"),
    (300, 2048, "laplace_outlier", None),
    (1024, 4096, "laplace_outlier", "ones"),
]


def _gamma(kind, K):
    if kind == "ones":
        return wl.gamma_ones(K)
    if kind == "random":
        return wl.gamma_random(72, 0, K)
    return None


def compare_pairs(P, R, kept, meta, M, K):
    assert np.array_equal(to_np(P.bb_codes), kept), "compressed backbone codes"
    mb = to_np(P.bb_meta)
    assert np.array_equal(meta_atoms_to_canonical(mb, M, K), meta), "pair metadata"
    Mp = (M + 127) // 128 * 128
    if Mp > M:                                   # padding rows: pairs 0 and 1
        pad = np.ones(mb.size, bool)
        pad[meta_atom_index(M, K).reshape(-1)] = False
        assert np.all(mb[pad] == 0x44)
    assert np.array_equal(atoms_to_canonical(to_np(P.bb_scales), M, K, "mxfp4"), R.bb.scales), "backbone scales"
    assert np.array_equal(to_np(P.rs_codes), R.rs.codes), "residual codes"
    assert np.array_equal(atoms_to_canonical(to_np(P.rs_scales), M, K, "mxfp4"), R.rs.scales), "residual scales"
    assert float(to_np(P.bb_tscale)[0]) == 1.0 and float(to_np(P.rs_tscale)[0]) == 1.0
    assert np.array_equal(to_np(P.mask), R.mask), "element mask"


@pytest.mark.parametrize("M,K,dist,gk", CASES)
def test_prepare_pairs_bit_exact(M, K, dist, gk):
    X = wl.activation(dist, 71, M + K, M, K)
    g = _gamma(gk, K)
    P = sq.prepare(to_dev(X), None if g is None else to_dev(g), 1e-6, pairs=True, want_mask=True)
    torch.cuda.synchronize()
    assert sq.last_device_status() == 0
    R, kept, meta = oracle.prepare_pairs(X, g, 1e-6)
    compare_pairs(P, R, kept, meta, M, K)


def test_prepare_pairs_full_size_sweep_input():
    """The format sweep's input (16384 x 4096, RMSNorm) in the pair form."""
    W = wl.WORKLOADS["sweep"]
    L = W.linears[0]
    M = 16384
    X = wl.activation(W.dist, W.cfg, L.index, M, L.K)
    g = wl.gamma_ones(L.K)
    P = sq.prepare(to_dev(X), to_dev(g), wl.EPS, pairs=True, want_mask=True)
    torch.cuda.synchronize()
    assert sq.last_device_status() == 0
    R, kept, meta = oracle.prepare_pairs(X, g, wl.EPS)
    compare_pairs(P, R, kept, meta, M, L.K)


def test_pair_backbone_is_rejected_where_it_is_not_offered():
    """NVFP4, LayerNorm, a producer's amax and the allocation-free entry
    point do not take a compressed backbone."""
    X = to_dev(wl.activation("laplace_outlier", 73, 0, 8, 256))
    P = sq.Prepared.empty(8, 256, fmt="mxfp4", pairs=True)
    L = sq.load_sharq_ops()
    ws = torch.empty(4096, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    import ctypes
    bad = P._c()
    bad.fmt = 0
    assert L.sharq_prepare(X.data_ptr(), None, ctypes.c_float(1e-6), ctypes.byref(bad), ws.data_ptr(),
                           ws.numel(), stream) == 1
    c = P._c()
    g = to_dev(wl.gamma_ones(256))
    assert L.sharq_prepare_layernorm(X.data_ptr(), g.data_ptr(), None, ctypes.c_float(1e-6), ctypes.byref(c),
                                     ws.data_ptr(), ws.numel(), stream) == 2
    assert L.sharq_prepare_noalloc(X.data_ptr(), None, ctypes.c_float(1e-6), ctypes.byref(c), stream) == 2


# ---------------------------------------------------------------------------
# The two-path linear with the sparse tensor-core MMA on the compressed
# backbone (tcgen05.mma.sp, pair indices in tensor memory) and the dense MMA
# on the residual, one accumulator (MXFP4), against the fp64 oracle of the
# same operands (the backbone decompressed to zero-filled codes).
# ---------------------------------------------------------------------------

LINEAR_CASES = [
    # M, N, K
    (16, 256, 256),
    (1, 128, 512),
    (129, 384, 1024),
    (300, 512, 2048),
    (2048, 1024, 4096),
    (1000, 4608, 2048),     # the 256-wide tile, ragged M
]


@pytest.mark.parametrize("M,N,K", LINEAR_CASES)
def test_linear_sparse_backbone_matches_oracle(M, N, K):
    from tests.test_linear_parity import check
    X = wl.activation("laplace_outlier", 74, M + N, M, K)
    W = wl.weight(74, N + K, N, K)
    g = wl.gamma_ones(K)
    P = sq.prepare(to_dev(X), to_dev(g), 1e-6, pairs=True)
    w = sq.quantize_weight(to_dev(W), "mxfp4")
    Y32 = sq.linear(P, w, out_fp32=True)
    Ybf = sq.linear(P, w)
    torch.cuda.synchronize()
    assert sq.last_device_status() == 0
    R, kept, meta = oracle.prepare_pairs(X, g, 1e-6)
    assert np.array_equal(to_np(P.bb_codes), kept) and np.array_equal(
        meta_atoms_to_canonical(to_np(P.bb_meta), M, K), meta)
    Rw = oracle.quantize_weight(W, "mxfp4")
    rows = None if M <= 512 else np.sort(np.random.default_rng(M).choice(M, 48, replace=False))
    check(Y32, Ybf, oracle.linear(R, Rw, rows=rows), oracle.linear_abs(R, Rw, rows=rows), K,
          rows=rows, one_acc=True)
