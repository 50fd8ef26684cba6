"""GPU parity of the fused prepare kernel and the weight quantiser against
the CPU oracle: masks, packed E2M1 codes, E4M3/E8M0 block scales and the fp32
tensor scales must match bit for bit."""
import numpy as np
import pytest
import torch

import activation_sparsity_prep_b200 as sq
from activation_sparsity_prep_b200 import workloads as wl
import oracle
from tests.sharq_testlib import atoms_to_canonical, to_dev, to_np

pytestmark = pytest.mark.gpu


def _gamma(kind, cfg, K):
    if kind == "ones":
        return wl.gamma_ones(K)
    if kind == "random":
        return wl.gamma_random(cfg, 0, K)
    return None


def run_and_compare(X, g, n, m, fmt, eps=1e-6, residual_scale="own"):
    M, K = X.shape
    P = sq.prepare(to_dev(X), None if g is None else to_dev(g), eps, n, m, fmt, want_mask=True,
                   residual_scale=residual_scale)
    torch.cuda.synchronize()
    assert sq.last_device_status() == 0
    R = oracle.prepare(X, g, eps, n, m, fmt, residual_scale=residual_scale)
    assert np.array_equal(to_np(P.mask), R.mask), "mask"
    assert np.array_equal(to_np(P.bb_codes), R.bb.codes), "backbone codes"
    assert np.array_equal(to_np(P.rs_codes), R.rs.codes), "residual codes"
    bs = to_np(P.bb_scales)
    rs = to_np(P.rs_scales)
    assert np.array_equal(atoms_to_canonical(bs, M, K, fmt), R.bb.scales), "backbone scales"
    assert np.array_equal(atoms_to_canonical(rs, M, K, fmt), R.rs.scales), "residual scales"
    assert to_np(P.bb_tscale).view(np.uint32)[0] == np.float32(R.bb.tscale).view(np.uint32)
    assert to_np(P.rs_tscale).view(np.uint32)[0] == np.float32(R.rs.tscale).view(np.uint32)
    # scale-atom padding rows are zero
    Mp = (M + 127) // 128 * 128
    if Mp > M:
        pad = np.ones(Mp, bool)
        pad[:M] = False
        from tests.sharq_testlib import atom_index
        idx = atom_index(Mp, K, fmt)[pad]
        assert np.all(bs[idx] == 0) and np.all(rs[idx] == 0)
    return P, R


CASES = [
    # M, K, dist, gamma, n, m, fmt
    (16, 256, "normal_outlier", "ones", 2, 4, "nvfp4"),        # the tiny single-linear case
    (1, 4096, "laplace_outlier", "ones", 2, 4, "nvfp4"),
    (3, 768, "laplace_outlier", None, 2, 4, "nvfp4"),
    (17, 1024, "student_t", "random", 2, 4, "nvfp4"),
    (129, 2048, "laplace_outlier", "ones", 1, 4, "nvfp4"),
    (300, 512, "student_t", "ones", 4, 8, "nvfp4"),
    (64, 256, "normal_outlier", "random", 1, 2, "nvfp4"),
    (40, 768, "laplace_outlier", None, 3, 4, "nvfp4"),
    (16, 256, "normal_outlier", "ones", 2, 4, "mxfp4"),
    (129, 1024, "laplace_outlier", "ones", 1, 4, "mxfp4"),
    (33, 768, "student_t", None, 4, 8, "mxfp4"),
    (200, 4096, "laplace_outlier", "random", 2, 4, "mxfp4"),
    # several hundred rows: many CTAs per phase, ragged last CTA
    (1024, 4096, "laplace_outlier", "ones", 2, 4, "mxfp4"),
    (600, 4096, "student_t", None, 1, 4, "nvfp4"),
    (700, 3584, "student_t", "random", 4, 8, "nvfp4"),
]


@pytest.mark.parametrize("M,K,dist,gk,n,m,fmt", CASES)
def test_prepare_bit_exact(M, K, dist, gk, n, m, fmt):
    X = wl.activation(dist, 21, M + K, M, K)
    run_and_compare(X, _gamma(gk, 21, K), n, m, fmt)


SHARED_CASES = [
    # M, K, dist, gamma, n, m
    (16, 256, "normal_outlier", "ones", 2, 4),
    (3, 768, "laplace_outlier", None, 2, 4),
    (129, 2048, "student_t", "random", 1, 4),
    (300, 512, "laplace_outlier", "ones", 4, 8),
    (700, 3584, "student_t", None, 2, 4),
]


@pytest.mark.parametrize("M,K,dist,gk,n,m", SHARED_CASES)
def test_prepare_shared_residual_scale_bit_exact(M, K, dist, gk, n, m):
    X = wl.activation(dist, 24, M + K, M, K)
    P, R = run_and_compare(X, _gamma(gk, 24, K), n, m, "nvfp4", residual_scale="shared")
    assert torch.equal(P.rs_tscale, P.bb_tscale)


LN_CASES = [
    # M, K, dist, beta, n, m, fmt, residual
    (16, 256, "normal_outlier", True, 2, 4, "nvfp4", "own"),
    (3, 768, "laplace_outlier", False, 2, 4, "nvfp4", "own"),
    (129, 5120, "laplace_outlier", True, 2, 4, "nvfp4", "own"),
    (300, 1024, "student_t", True, 1, 4, "nvfp4", "shared"),
    (64, 2048, "laplace_outlier", True, 4, 8, "mxfp4", "own"),
    (600, 4096, "student_t", False, 2, 4, "mxfp4", "own"),
]


@pytest.mark.parametrize("M,K,dist,hb,n,m,fmt,rs", LN_CASES)
def test_prepare_layernorm_bit_exact(M, K, dist, hb, n, m, fmt, rs):
    X = wl.activation(dist, 25, M + K, M, K)
    g = wl.gamma_random(25, 0, K)
    b = wl.beta_random(25, 0, K) if hb else None
    P = sq.prepare_layernorm(to_dev(X), to_dev(g), None if b is None else to_dev(b), 1e-6, n, m, fmt,
                             want_mask=True, residual_scale=rs)
    torch.cuda.synchronize()
    assert sq.last_device_status() == 0
    R = oracle.prepare(X, g, 1e-6, n, m, fmt, residual_scale=rs, norm="layernorm", beta=b)
    assert np.array_equal(to_np(P.mask), R.mask), "mask"
    assert np.array_equal(to_np(P.bb_codes), R.bb.codes), "backbone codes"
    assert np.array_equal(to_np(P.rs_codes), R.rs.codes), "residual codes"
    assert np.array_equal(atoms_to_canonical(to_np(P.bb_scales), M, K, fmt), R.bb.scales)
    assert np.array_equal(atoms_to_canonical(to_np(P.rs_scales), M, K, fmt), R.rs.scales)
    assert to_np(P.bb_tscale).view(np.uint32)[0] == np.float32(R.bb.tscale).view(np.uint32)
    assert to_np(P.rs_tscale).view(np.uint32)[0] == np.float32(R.rs.tscale).view(np.uint32)


# Long rows: gamma (and beta) no longer fit the kernel's 96 KiB shared-memory
# stage and are read from global memory (RMSNorm K > 24576, LayerNorm with a
# bias K > 12288), and MXFP4 RMSNorm rows past the 4096 elements it holds in
# registers take the chunked path.
LONG_K_CASES = [
    # M, K, norm, beta, fmt, residual
    (5, 32768, "rms", False, "nvfp4", "own"),
    (3, 32768, "rms", False, "mxfp4", "own"),
    (9, 8192, "rms", False, "mxfp4", "own"),
    (4, 32768, "rms", False, "nvfp4", "shared"),
    (7, 16384, "layernorm", True, "nvfp4", "own"),
    (6, 32768, "layernorm", False, "mxfp4", "own"),
]


@pytest.mark.parametrize("M,K,norm,hb,fmt,rs", LONG_K_CASES)
def test_prepare_long_rows_bit_exact(M, K, norm, hb, fmt, rs):
    X = wl.activation("laplace_outlier", 27, M + K, M, K)
    g = wl.gamma_random(27, 0, K)
    if norm == "rms":
        run_and_compare(X, g, 2, 4, fmt, residual_scale=rs)
        return
    b = wl.beta_random(27, 0, K) if hb else None
    P = sq.prepare_layernorm(to_dev(X), to_dev(g), None if b is None else to_dev(b), 1e-6, 2, 4, fmt,
                             want_mask=True, residual_scale=rs)
    torch.cuda.synchronize()
    assert sq.last_device_status() == 0
    R = oracle.prepare(X, g, 1e-6, 2, 4, fmt, residual_scale=rs, norm="layernorm", beta=b)
    assert np.array_equal(to_np(P.mask), R.mask), "mask"
    assert np.array_equal(to_np(P.bb_codes), R.bb.codes), "backbone codes"
    assert np.array_equal(to_np(P.rs_codes), R.rs.codes), "residual codes"
    assert np.array_equal(atoms_to_canonical(to_np(P.bb_scales), M, K, fmt), R.bb.scales)
    assert np.array_equal(atoms_to_canonical(to_np(P.rs_scales), M, K, fmt), R.rs.scales)
    assert to_np(P.bb_tscale).view(np.uint32)[0] == np.float32(R.bb.tscale).view(np.uint32)
    assert to_np(P.rs_tscale).view(np.uint32)[0] == np.float32(R.rs.tscale).view(np.uint32)


def test_prepare_layernorm_constant_rows_give_beta():
    """Constant rows normalise to exactly beta: the backbone and residual
    are those of the tensor [beta; beta; ...] with no norm."""
    K = 512
    b = wl.beta_random(26, 0, K)
    X = np.repeat(wl.f32_to_bf16_bits(np.full((1, K), 2.5, np.float32)), 8, axis=0)
    P = sq.prepare_layernorm(to_dev(X), to_dev(wl.gamma_random(26, 0, K)), to_dev(b))
    Q = sq.prepare(to_dev(np.repeat(b[None], 8, axis=0)), None)
    torch.cuda.synchronize()
    assert torch.equal(P.bb_codes, Q.bb_codes) and torch.equal(P.rs_codes, Q.rs_codes)
    assert torch.equal(P.bb_scales, Q.bb_scales) and torch.equal(P.rs_tscale, Q.rs_tscale)


def test_prepare_special_values():
    """Rows of zeros, -0, exact ties inside groups, a constant row, values at
    E2M1/E4M3 rounding boundaries and one huge outlier."""
    K = 512
    rows = []
    rows.append(np.zeros(K))
    rows.append(-np.zeros(K))
    t = np.tile([1.0, -1.0, 1.0, 0.5], K // 4)
    rows.append(t)
    rows.append(np.full(K, 3.25))
    rows.append(np.linspace(-6, 6, K))
    r = np.random.default_rng(0).standard_normal(K)
    r[7] = 3.0e4
    rows.append(r)
    X = wl.f32_to_bf16_bits(np.array(rows, dtype=np.float32))
    for g in (None, wl.gamma_ones(K)):
        for fmt in ("nvfp4", "mxfp4"):
            run_and_compare(X, g, 2, 4, fmt)


def test_prepare_all_zero_tensor_has_unit_scales():
    X = np.zeros((5, 256), dtype=np.uint16)
    P, R = run_and_compare(X, None, 2, 4, "nvfp4")
    assert float(to_np(P.bb_tscale)[0]) == 1.0 and float(to_np(P.rs_tscale)[0]) == 1.0


def test_prepare_empty_input():
    X = np.zeros((0, 256), dtype=np.uint16)
    P = sq.prepare(torch.empty((0, 256), dtype=torch.bfloat16, device="cuda"), None)
    torch.cuda.synchronize()
    assert float(P.bb_tscale.cpu()[0]) == 1.0 and float(P.rs_tscale.cpu()[0]) == 1.0


def test_prepare_repeated_calls_reuse_workspace():
    X = wl.activation("laplace_outlier", 22, 0, 64, 1024)
    ws = torch.empty(sq.prepare_workspace_bytes(64, 1024), dtype=torch.uint8, device="cuda")
    outs = [sq.prepare(to_dev(X), to_dev(wl.gamma_ones(1024)), ws=ws) for _ in range(3)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o.rs_codes, outs[0].rs_codes) and torch.equal(o.bb_scales, outs[0].bb_scales)
        assert torch.equal(o.rs_tscale, outs[0].rs_tscale)


@pytest.mark.parametrize("N,K,fmt", [(256, 256, "nvfp4"), (384, 4096, "nvfp4"),
                                     (128, 768, "mxfp4"), (1536, 2048, "nvfp4")])
def test_quantize_weight_bit_exact(N, K, fmt):
    W = wl.weight(23, N, N, K)
    w = sq.quantize_weight(to_dev(W), fmt)
    torch.cuda.synchronize()
    R = oracle.quantize_weight(W, fmt)
    assert np.array_equal(to_np(w.codes), R.codes)
    assert np.array_equal(atoms_to_canonical(to_np(w.scales), N, K, fmt), R.scales)
    assert to_np(w.tensor_scale).view(np.uint32)[0] == np.float32(R.tscale).view(np.uint32)


@pytest.mark.parametrize("lin", range(4))
def test_prepare_full_size_llama_prefill(lin):
    """Whole tensors at the benchmark's size (M = 2048, Llama-3.1-8B-shaped
    linears): every output compared."""
    W = wl.WORKLOADS["llama8b"]
    L = W.linears[lin]
    X = wl.activation(W.dist, W.cfg, L.index, 2048, L.K)
    run_and_compare(X, wl.gamma_ones(L.K) if L.norm else None, 2, 4, "nvfp4")
