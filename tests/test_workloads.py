"""The seeded synthetic inputs: both the CUDA path and the oracle read these
arrays, so their structure is what the parity and bench numbers stand on.
Checked here: bf16 rounding to nearest even, determinism and independence
of the seeds, the outlier structure of each activation distribution (whole
columns, their count and factor range), the per-token scales of the
heavy-tailed rows, the weight spread, and the routing / dispatch helpers of
the grouped linear."""
from fractions import Fraction

import numpy as np
import pytest

from activation_sparsity_prep_b200 import workloads as wl


def test_bf16_rounding_is_nearest_even():
    rng = np.random.default_rng(3)
    f = (rng.standard_normal(3000) * 10.0 ** rng.integers(-30, 30, 3000)).astype(np.float32)
    # exact halfway cases: a bf16 value plus half its spacing, both parities
    b = rng.integers(0x0080, 0x7F00, 200).astype(np.uint32)
    half = ((b << np.uint32(16)) | np.uint32(0x8000)).view(np.float32)
    f = np.concatenate([f, half, -half])
    got = wl.f32_to_bf16_bits(f)
    for v, g in zip(f, got):
        q = Fraction(float(v))
        top = int(np.array([v], dtype=np.float32).view(np.uint32)[0] >> np.uint32(16))
        cands = [c for c in (top, top + 1) if (c & 0x7F80) != 0x7F80]
        val = lambda c: Fraction(float((np.uint32(c) << np.uint32(16)).view(np.float32)))
        best = min(cands, key=lambda c: (abs(val(c) - q), c & 1))
        assert int(g) == best, (float(v), hex(int(g)), hex(best))


def test_generators_are_seeded_and_distinct():
    a = wl.activation("laplace_outlier", 2, 0, 8, 512)
    assert np.array_equal(a, wl.activation("laplace_outlier", 2, 0, 8, 512))
    assert not np.array_equal(a, wl.activation("laplace_outlier", 2, 1, 8, 512))   # another linear
    assert not np.array_equal(a, wl.activation("laplace_outlier", 3, 0, 8, 512))   # another config
    w = wl.weight(2, 0, 64, 512)
    assert np.array_equal(w, wl.weight(2, 0, 64, 512))
    assert not np.array_equal(w, wl.weight(2, 1, 64, 512))


def _column_median_abs(X):
    return np.median(np.abs(wl.bf16_bits_to_f32(X)), axis=0)


@pytest.mark.parametrize("K", [4096, 14336])
def test_laplace_outliers_are_whole_columns(K):
    """round(0.005 K) columns scaled by factors in [20, 100]; the rest
    Laplace(0, 1), whose median |x| is ln 2."""
    X = wl.activation("laplace_outlier", 2, 0, 512, K)
    med = _column_median_abs(X)
    out = med > 8.0
    assert int(out.sum()) == int(round(0.005 * K))
    assert abs(np.median(med[~out]) - np.log(2)) < 0.02
    ratio = med[out] / np.log(2)
    assert ratio.min() > 20 * 0.8 and ratio.max() < 100 * 1.2
    # the same channels in every row: each outlier column is large in most rows
    x = np.abs(wl.bf16_bits_to_f32(X))
    assert np.all((x[:, out] > 2.0).mean(axis=0) > 0.8)


def test_normal_outliers():
    X = wl.activation("normal_outlier", 1, 0, 256, 256)
    med = _column_median_abs(X)
    out = med > 8.0
    assert int(out.sum()) == 4
    base = np.median(med[~out])                     # median |N(0,1)| = 0.674
    assert abs(base - 0.674) < 0.03
    assert np.allclose(med[out] / base, 50.0, rtol=0.25)


def test_student_t_rows_carry_per_token_scales():
    """t(3) entries times s ~ LogNormal(0, 0.5) per row: heavy tails inside a
    row, and log row scales spread with standard deviation about 0.5."""
    X = wl.bf16_bits_to_f32(wl.activation("student_t", 3, 0, 400, 3584)).astype(np.float64)
    med = np.median(np.abs(X), axis=1)               # median |t(3)| = 0.765 times s
    assert abs(np.std(np.log(med)) - 0.5) < 0.06
    z = X / med[:, None]
    kurt = np.mean(z ** 4) / np.mean(z ** 2) ** 2
    assert kurt > 6.0                               # a normal row would give 3
    assert np.all(np.abs(np.median(X, axis=1)) < 0.2 * med)


def test_weight_spread_and_chunk_independence():
    W = wl.bf16_bits_to_f32(wl.weight(5, 1, 3000, 512)).astype(np.float64)
    assert abs(W.std() - 0.02) < 0.0005 and abs(W.mean()) < 0.0005
    # drawn in 2048-row chunks from one stream: a shorter weight is a prefix
    assert np.array_equal(wl.weight(5, 1, 2048, 512), wl.weight(5, 1, 3000, 512)[:2048])


def test_routing_is_distinct_and_uniform():
    T, E, k = 4096, 128, 8
    ex = wl.routing(4, T, E, k)
    assert ex.shape == (T, k) and ex.dtype == np.int32
    assert all(len(set(r)) == k for r in ex)
    counts = np.bincount(ex.reshape(-1), minlength=E)
    mean = T * k / E                                 # 256 rows per expert
    assert counts.min() > mean - 6 * np.sqrt(mean) and counts.max() < mean + 6 * np.sqrt(mean)


def test_group_by_expert_is_a_grouped_permutation():
    ex = wl.routing(9, 100, 6, 3)
    ri, off = wl.group_by_expert(ex, 6)
    assert off[0] == 0 and off[-1] == 300 and np.all(np.diff(off) >= 0)
    for e in range(6):
        rows = ri[off[e]:off[e + 1]]
        assert np.all(np.diff(rows) > 0)             # tokens ascending, each once per expert
        assert set(rows.tolist()) == set(np.nonzero((ex == e).any(axis=1))[0].tolist())
    # every (token, expert) pair appears exactly once
    pairs = sorted((int(t), e) for e in range(6) for t in ri[off[e]:off[e + 1]])
    assert pairs == sorted((t, int(e)) for t in range(100) for e in ex[t])
