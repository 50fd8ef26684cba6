"""Pins of the oracle's LayerNorm reading (mean-subtracting norm for DiT and
vision layers): closed forms, a summation-order probe and the preparation
invariants with LayerNorm in front."""
import numpy as np
import pytest

import oracle
from activation_sparsity_prep_b200 import workloads as wl


def _bf16(a):
    return wl.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def _f(b):
    return wl.bf16_bits_to_f32(b)


@pytest.mark.parametrize("c,K", [(1.5, 256), (-40.0, 1024), (0.0078125, 4096)])
def test_constant_row_gives_beta_exactly(c, K):
    """x = c everywhere: the mean is c exactly, every centred value is 0, so
    y = (0 * rstd) * gamma + beta = beta bit for bit (and a zero with the
    sign of gamma without a bias)."""
    x = _bf16(np.full((1, K), c))
    g = wl.gamma_random(71, 0, K)
    b = _bf16(np.random.default_rng(71).standard_normal(K))
    mu, _ = oracle.ln_stats(x[0])
    assert mu == np.float32(c)
    y = oracle.normalize_ln(x, g, b)
    assert np.array_equal(y[0], _f(b)[0] if _f(b).ndim == 2 else _f(b))
    y0 = oracle.normalize_ln(x, g, None)
    assert np.all(y0 == 0) and np.array_equal(np.signbit(y0[0]), np.signbit(_f(g)))


@pytest.mark.parametrize("a", [3.0, 0.25, 17.5])
def test_plus_minus_row_closed_form(a):
    """Alternating +a, -a: mean 0 exactly, variance a^2 exactly, so
    y_k = +-a * gamma_k / sqrt(a^2 + eps) up to the rounding of three
    operations."""
    K = 512
    x = np.tile([a, -a], K // 2)
    g = wl.gamma_random(72, 0, K)
    y = oracle.normalize_ln(_bf16(x[None]), g, None)[0].astype(np.float64)
    want = x * _f(g).astype(np.float64) / np.sqrt(a * a + 1e-6)
    ulp = np.spacing(np.abs(want).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(y - want) <= 3 * ulp)


def test_mean_uses_the_stated_lane_order():
    """x_0 = 2^24 and eight ones in chunk 1 (lane 1): lane 1 sums to 8, the
    butterfly adds it to 2^24 in one step (2^24 + 8 is exact), so the mean
    over K = 256 is 65536.03125.  A sequential sum drops every +1 (2^24 + 1
    rounds to even) and gives exactly 65536."""
    x = np.zeros(256)
    x[0] = 2.0 ** 24
    x[8:16] = 1.0
    mu, _ = oracle.ln_stats(_bf16(x))
    assert mu == np.float32(65536.03125)


def test_stats_match_fp64():
    X = wl.activation("laplace_outlier", 73, 0, 16, 4096)
    x64 = _f(X).astype(np.float64)
    for i in range(16):
        mu, rstd = oracle.ln_stats(X[i])
        m64 = x64[i].mean()
        r64 = 1.0 / np.sqrt(((x64[i] - m64) ** 2).mean() + 1e-6)
        assert abs(mu - m64) <= 1e-5 * np.abs(x64[i]).max()
        assert abs(rstd - r64) <= 1e-5 * r64


@pytest.mark.parametrize("fmt,rs", [("nvfp4", "own"), ("nvfp4", "shared"), ("mxfp4", "own")])
def test_prepare_invariants_under_layernorm(fmt, rs):
    """With LayerNorm in front: exactly n kept per group, the group maximum
    kept, and the Sterbenz reconstruction D_b + r == y bit for bit."""
    K = 1024
    X = wl.activation("student_t", 74, 0, 24, K)
    g, b = wl.gamma_random(74, 0, K), wl.gamma_random(74, 1, K)
    P = oracle.prepare(X, g, 1e-6, 2, 4, fmt, keep_intermediates=True, residual_scale=rs,
                       norm="layernorm", beta=b)
    assert np.array_equal(P.y, oracle.normalize_ln(X, g, b))
    keep = np.unpackbits(P.mask, axis=1, bitorder="little").astype(bool)
    assert np.all(keep.reshape(24, K // 4, 4).sum(axis=2) == 2)
    yg = np.abs(P.y).reshape(24, K // 4, 4)
    kept_max = np.where(keep.reshape(24, K // 4, 4), yg, -1).max(axis=2)
    assert np.array_equal(kept_max, yg.max(axis=2))
    Db = oracle.dequant_blocks(P.bb) * np.float64(P.bb.tscale)
    assert np.array_equal((Db.astype(np.float32) + P.r).astype(np.float32), P.y)
