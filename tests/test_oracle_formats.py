"""Pins of the oracle's format encoders/decoders against things other than
themselves: the OCP specification tables (tests/golden), brute-force nearest
search with ties to even, and the ml_dtypes library casts."""
import os

import ml_dtypes
import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _read_table(name):
    rows = []
    for line in open(os.path.join(GOLD, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        c, v = line.split()
        rows.append((int(c, 16), float(v)))
    return rows


def _near(points, span, rng, n_random=200_000):
    """float32 inputs: every value within +-span ulps of each point, plus a
    wide random sample of finite floats, plus special values."""
    out = []
    for p in points:
        b = np.float32(p).view(np.int32).astype(np.int64)
        ints = np.arange(max(0, b - span), b + span + 1, dtype=np.int64)
        out.append(ints.astype(np.int32).view(np.float32))
    u = rng.integers(0, 0x7F800000, size=n_random, dtype=np.int64).astype(np.int32)
    out.append(u.view(np.float32))
    out.append(np.array([0.0, np.finfo(np.float32).max, np.finfo(np.float32).tiny,
                         1e-45, 6.0, 448.0, 480.0, 1e30], dtype=np.float32))
    v = np.concatenate(out)
    return np.concatenate([v, -v])


def _nearest_ties_even(v, grid_vals, grid_codes):
    """Brute force: nearest grid value by exact fp64 distance; on a tie the
    neighbour with the even code wins."""
    v64 = np.abs(v.astype(np.float64))[:, None]
    d = np.abs(v64 - grid_vals[None, :].astype(np.float64))
    dmin = d.min(axis=1, keepdims=True)
    cand = d == dmin
    even = (grid_codes[None, :] & 1) == 0
    has_even = (cand & even).any(axis=1)
    idx_even = np.argmax(cand & even, axis=1)
    idx_any = np.argmax(cand, axis=1)
    idx = np.where(has_even, idx_even, idx_any)
    return grid_codes[idx]


# ------------------------------------------------------------------- E2M1 --

def test_e2m1_decode_matches_spec_table():
    for code, val in _read_table("e2m1_grid.txt"):
        got = oracle.e2m1_decode(np.array([code]))[0]
        assert got == val and np.signbit(got) == np.signbit(val), (code, got, val)


def test_e2m1_encode_bruteforce_nearest_even():
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float32)
    codes = np.arange(8, dtype=np.uint8)
    pts = list(mags) + [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    v = _near(pts, 4096, np.random.default_rng(0))
    got = oracle.e2m1_encode(v)
    # distances stay exact in fp64 once |v| is clipped to 8 (all of (6, inf) has 6 nearest)
    mag = _nearest_ties_even(np.minimum(np.abs(v), 8.0).astype(np.float32), mags, codes)
    want = mag | np.where(np.signbit(v), 8, 0).astype(np.uint8)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (v[bad[:5]], got[bad[:5]], want[bad[:5]])


def test_e2m1_encode_matches_ml_dtypes_in_range():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.uniform(-6, 6, 500_000).astype(np.float32),
                        np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -5.0],
                                 dtype=np.float32)])
    ref = v.astype(ml_dtypes.float4_e2m1fn).astype(np.float32)
    got = oracle.e2m1_decode(oracle.e2m1_encode(v))
    assert np.array_equal(got, ref)


# ------------------------------------------------------------------- E4M3 --

def _e4m3_all_finite_nonneg():
    c = np.arange(0, 0x7F, dtype=np.uint8)          # 0x00..0x7E
    return c, oracle.e4m3_decode(c)


def test_e4m3_decode_spec_table_and_ml_dtypes():
    for code, val in _read_table("e4m3_selected.txt"):
        got = oracle.e4m3_decode(np.array([code], dtype=np.uint8))[0]
        if np.isnan(val):
            assert np.isnan(got)
        else:
            assert got == val and np.signbit(got) == np.signbit(val), (hex(code), got, val)
    allc = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(allc)
    ref = allc.view(ml_dtypes.float8_e4m3fn).astype(np.float32)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert np.array_equal(np.signbit(ours[ok]), np.signbit(ref[ok]))


def test_e4m3_encode_bruteforce_nearest_even():
    codes, vals = _e4m3_all_finite_nonneg()
    mids = (vals[:-1].astype(np.float64) + vals[1:]) / 2
    v = _near(list(vals) + list(mids.astype(np.float32)) + [464.0], 2048,
              np.random.default_rng(2))
    got = oracle.e4m3_encode(v)
    mag = _nearest_ties_even(np.minimum(np.abs(v), 448.0).astype(np.float32), vals, codes)
    want = mag | np.where(np.signbit(v), 0x80, 0).astype(np.uint8)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (v[bad[:5]], got[bad[:5]], want[bad[:5]])


def test_e4m3_encode_matches_ml_dtypes_in_range():
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.uniform(0, 448, 300_000), 2.0 ** rng.uniform(-12, 8.8, 300_000)]
                       ).astype(np.float32)
    v = v[v <= 448]
    ref = v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(oracle.e4m3_encode(v), ref)


# ------------------------------------------------------------------- E8M0 --

def test_e8m0_decode_matches_ml_dtypes():
    c = np.arange(255, dtype=np.uint8)
    ref = c.view(ml_dtypes.float8_e8m0fnu).astype(np.float32)
    assert np.array_equal(oracle.e8m0_decode(c), ref)


def test_mx_scale_maps_block_max_into_4_8():
    """OCP MX: shared exponent = floor(log2 amax) - emax(E2M1), emax = 2, so
    amax / scale lies in [4, 8) whenever no clamping happens."""
    rng = np.random.default_rng(4)
    b = np.concatenate([2.0 ** rng.uniform(-120, 120, 20000),
                        2.0 ** np.arange(-120, 121, dtype=np.float64)]).astype(np.float32)
    for x in b:
        c = oracle.mx_scale_code(x)
        s = float(oracle.e8m0_decode(np.array([c]))[0])
        assert 4.0 <= float(x) / s < 8.0, (x, c)
    assert oracle.mx_scale_code(0.0) == 0
    assert oracle.mx_scale_code(np.float32(1e-45)) == 0          # clamped low
    assert oracle.mx_scale_code(np.finfo(np.float32).max) == 127 - 2 + 127
