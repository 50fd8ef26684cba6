"""Pins of the oracle's pair-granular 4:8 backbone (the shape the FP4 sparse
MMA takes: two kept pairs of every eight elements), CPU only.

Reading pinned here: a pair's magnitude is max(|y_2i|, |y_2i+1|), the two
largest pairs of every aligned group of eight are kept, ties go to the lower
pair index; the backbone is MXFP4 with its per-32 E8M0 scales."""
import itertools

import numpy as np
import pytest

import oracle
from activation_sparsity_prep_b200 import workloads as wl


def brute_mask(y):
    """Keep flags by enumerating, per group, the six choices of two pairs and
    taking the lexicographically best one under (magnitude desc, index asc)."""
    M, K = y.shape
    out = np.zeros((M, K), dtype=np.uint8)
    for r in range(M):
        for g in range(K // 8):
            mags = [max(abs(float(y[r, 8 * g + 2 * p])), abs(float(y[r, 8 * g + 2 * p + 1]))) for p in range(4)]
            ranked = sorted(range(4), key=lambda p: (-mags[p], p))
            best = None
            for choice in itertools.combinations(range(4), 2):
                key = sorted(ranked.index(p) for p in choice)
                if best is None or key < best[0]:
                    best = (key, choice)
            for p in best[1]:
                out[r, 8 * g + 2 * p] = out[r, 8 * g + 2 * p + 1] = 1
    return out


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_mask_pairs_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((3, 64)).astype(np.float32)
    assert np.array_equal(oracle.mask_pairs(y), brute_mask(y))


def test_mask_pairs_ties_go_to_the_lower_pair():
    y = np.array([[1, 0, 0, 1, 1, -1, 0.5, 0.5]], dtype=np.float32)   # pair magnitudes 1, 1, 1, 0.5
    assert oracle.mask_pairs(y).tolist() == [[1, 1, 1, 1, 0, 0, 0, 0]]
    rng = np.random.default_rng(7)
    y = rng.choice(np.array([0, 1, -1, 2], dtype=np.float32), size=(4, 128))   # many ties
    assert np.array_equal(oracle.mask_pairs(y), brute_mask(y))


def test_mask_pairs_invariants():
    X = wl.activation("laplace_outlier", 71, 0, 8, 512)
    y = oracle.normalize(X, wl.gamma_ones(512), 1e-6)
    keep = oracle.mask_pairs(y)
    g = keep.reshape(8, 64, 4, 2)
    assert np.all(g[..., 0] == g[..., 1])                              # whole pairs
    assert np.all(g[..., 0].sum(axis=2) == 2)                          # two of four pairs
    grp = np.abs(y).reshape(8, 64, 8)
    top = np.argmax(grp, axis=2)
    assert np.all(np.take_along_axis(keep.reshape(8, 64, 8), top[..., None], axis=2) == 1)   # group max kept


def test_compress_round_trip_and_layout():
    X = wl.activation("student_t", 72, 0, 5, 256)
    P, kept, meta = oracle.prepare_pairs(X, None)
    assert kept.shape == (5, 64) and meta.shape == (5, 16)
    assert np.array_equal(oracle.decompress_pairs(kept, meta), P.bb.codes)
    for nib in (meta & 0xF, meta >> 4):
        lo, hi = nib & 3, nib >> 2
        assert np.all(lo < hi) and np.all(hi < 4)
    # hand-made groups: pairs 1 and 3 kept, then pairs 0 and 2
    codes = np.array([[0x00, 0x21, 0x00, 0x9F, 0x7A, 0x00, 0x05, 0x00]], dtype=np.uint8)
    keep = np.array([[0, 0, 1, 1, 0, 0, 1, 1, 1, 1, 0, 0, 1, 1, 0, 0]], dtype=np.uint8)
    k, m = oracle.compress_pairs(codes, keep)
    assert k.tolist() == [[0x21, 0x9F, 0x7A, 0x05]]
    assert m.tolist() == [[(1 | (3 << 2)) | ((0 | (2 << 2)) << 4)]]


def test_prepare_pairs_reconstructs_and_shares_block_scales():
    """y = D_b + r exactly (E2M1 rounding keeps D_b within a factor two of y,
    so the subtraction is exact), pruned codes are zero, and the block scales
    equal those of the plain 2:4 MXFP4 prepare: both masks keep every group's
    largest entry, so both backbones have y's block maxima."""
    X = wl.activation("laplace_outlier", 73, 0, 6, 1024)
    g = wl.gamma_random(73, 0, 1024)
    P, kept, meta = oracle.prepare_pairs(X, g)
    Db = oracle.dequant_blocks(P.bb).astype(np.float32)
    assert np.array_equal((Db + P.r).astype(np.float32), P.y)
    keep = np.unpackbits(P.mask, axis=1, bitorder="little")
    nib = np.stack([P.bb.codes & 0xF, P.bb.codes >> 4], axis=2).reshape(6, 1024)
    assert np.all(nib[keep == 0] == 0)
    R24 = oracle.prepare(X, g, 1e-6, 2, 4, "mxfp4")
    assert np.array_equal(P.bb.scales, R24.bb.scales)
