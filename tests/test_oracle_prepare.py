"""Pins of the oracle's preparation steps and GEMM reference against the
mathematics: closed forms, invariants, grid identities and brute force.  Each
test is chosen so that a plausible slip in the oracle (a dropped factor, a
wrong index, swapped nibbles, the unquantised backbone used for the residual)
fails at least one of them."""
import numpy as np
import pytest

import oracle
from activation_sparsity_prep_b200 import workloads as wl

F32 = np.float32


def _bf16(a):
    return wl.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


# -------------------------------------------------------------- RMSNorm ----

@pytest.mark.parametrize("c", [1.0, -3.5, 0.0078125, 96.0])
@pytest.mark.parametrize("K", [256, 768, 4096])
def test_rmsnorm_constant_row_closed_form(c, K):
    x = _bf16(np.full((1, K), c))
    cv = float(wl.bf16_bits_to_f32(x)[0, 0])
    y = oracle.normalize(x, wl.gamma_ones(K), 1e-6)
    want = cv / np.sqrt(cv * cv + 1e-6)
    ulp = np.spacing(np.float32(abs(want)))
    assert np.all(np.abs(y.astype(np.float64) - want) <= 2 * ulp)


def test_rmsnorm_matches_fp64_and_applies_gamma():
    X = wl.activation("laplace_outlier", 9, 0, 8, 4096)
    g = wl.gamma_random(9, 0, 4096)
    y = oracle.normalize(X, g, 1e-6)
    x64 = wl.bf16_bits_to_f32(X).astype(np.float64)
    g64 = wl.bf16_bits_to_f32(g).astype(np.float64)
    y64 = x64 / np.sqrt((x64 ** 2).mean(axis=1, keepdims=True) + 1e-6) * g64
    rel = np.abs(y - y64) / np.maximum(np.abs(y64), 1e-30)
    assert rel.max() < 2e-6
    # gamma = NULL means no normalisation at all
    assert np.array_equal(oracle.normalize(X, None, 1e-6), wl.bf16_bits_to_f32(X))


def test_rms_sum_uses_the_stated_lane_order():
    """x_0 = 2^14 (square 2^28, ulp 32) and two chunks of 1.25 (squares
    1.5625) in chunks 1 and 3.  Strided chunk-to-lane assignment puts the
    chunks in lanes 1 and 3 (12.5 each); the butterfly joins lanes 1 and 3
    (25) before they meet lane 0, and 2^28 + 25 rounds to 2^28 + 32.  A
    sequential sum, contiguous lanes or a linear lane sum all lose the small
    terms one at a time and give 2^28."""
    K = 512
    x = np.zeros(K, dtype=np.float32)
    x[0] = 2.0 ** 14
    x[8:16] = 1.25
    x[24:32] = 1.25
    S_expect = np.float32(2.0 ** 28 + 32)
    ms = np.float32(S_expect / np.float32(K))
    rinv = np.float32(1) / np.sqrt(np.float32(ms + np.float32(1e-6)))
    S_seq = np.float32(2.0 ** 28)
    rinv_seq = np.float32(1) / np.sqrt(np.float32(np.float32(S_seq / np.float32(K)) + np.float32(1e-6)))
    assert rinv != rinv_seq
    got = oracle.rms_rinv(_bf16(x), 1e-6)
    assert got == rinv


# ------------------------------------------------------------------ mask ---

@pytest.mark.parametrize("n,m", [(2, 4), (1, 4), (4, 8), (3, 4), (1, 8)])
def test_mask_exact_n_per_group_and_bruteforce_sort(n, m):
    rng = np.random.default_rng(5)
    y = rng.standard_normal((7, 64)).astype(np.float32)
    y[:, ::3] = np.round(y[:, ::3])          # plenty of ties
    y[0, :8] = 0.0
    y[1, :4] = [-0.0, 0.0, -0.0, 0.0]
    keep = oracle.mask(y, n, m)
    g = keep.reshape(7, -1, m)
    assert np.all(g.sum(axis=2) == n)
    for i in range(7):
        for s in range(0, 64, m):
            a = np.abs(y[i, s:s + m])
            order = np.argsort(-a, kind="stable")          # ties -> lower index first
            want = np.zeros(m, dtype=np.uint8)
            want[order[:n]] = 1
            assert np.array_equal(keep[i, s:s + m], want)
            assert a[keep[i, s:s + m] == 1].max() == a.max()


# ---------------------------------------------------------- quantisers -----

def _grid_tensor_nvfp4(rng, R, K, j, sparse24=False):
    """T on the NVFP4 grid: T = val * e0 * 2^j with one element equal to
    6 * 448 * 2^j so that the tensor amax is exactly 2688 * 2^j.  With
    ``sparse24`` positions 2 and 3 of every group of 4 are zero and each
    block's amax element sits at a kept position."""
    vals = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    e4 = oracle.e4m3_decode(np.arange(0x08, 0x7F, dtype=np.uint8)).astype(np.float64)
    T = np.zeros((R, K))
    kept = np.array([p for p in range(16) if (not sparse24) or p % 4 < 2])
    for i in range(R):
        for b in range(K // 16):
            e0 = rng.choice(e4)
            v = rng.choice(vals, 16) * rng.choice([-1, 1], 16)
            if sparse24:
                v[np.arange(16) % 4 >= 2] = 0.0
            v[rng.choice(kept)] = 6.0 * rng.choice([-1, 1])    # block amax = 6 e0
            T[i, b * 16:(b + 1) * 16] = v * e0 * 2.0 ** j
    T[0, :16] = 0
    T[0, 1] = 6 * 448 * 2.0 ** j
    return T.astype(np.float32)


@pytest.mark.parametrize("j", [-12, 0, 5])
def test_nvfp4_identity_on_grid(j):
    rng = np.random.default_rng(100 + j)
    T = _grid_tensor_nvfp4(rng, 5, 128, j)
    q = oracle.quantize(T, "nvfp4", want_D=True)
    assert q.tscale == F32(2.0 ** j)
    assert np.array_equal(q.D, T)
    # codes decode to the right elements: even k in the low nibble
    lo = q.codes & 15
    hi = q.codes >> 4
    dec = np.empty_like(T)
    dec[:, 0::2] = oracle.e2m1_decode(lo)
    dec[:, 1::2] = oracle.e2m1_decode(hi)
    sc = np.repeat(oracle.e4m3_decode(q.scales), 16, axis=1)
    assert np.array_equal((dec * sc * q.tscale).astype(np.float32), T)


def test_mxfp4_identity_on_grid():
    rng = np.random.default_rng(7)
    vals = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    R, K = 3, 128
    T = np.zeros((R, K))
    for i in range(R):
        for b in range(K // 32):
            s = 2.0 ** rng.integers(-20, 20)
            v = rng.choice(vals, 32) * rng.choice([-1, 1], 32)
            v[rng.integers(32)] = rng.choice([4.0, 6.0])        # amax in {4,6} * s
            T[i, b * 32:(b + 1) * 32] = v * s
    T = T.astype(np.float32)
    q = oracle.quantize(T, "mxfp4", want_D=True)
    assert q.tscale == 1.0
    assert np.array_equal(q.D, T)


def test_nvfp4_scale_and_code_bounds():
    """Away from the grid: the block scale is the E4M3 rounding of
    amax_block * G_enc / 6, and each code is the nearest E2M1 value of
    T * G_enc / e (checked with independent float64 arithmetic)."""
    X = wl.activation("laplace_outlier", 11, 0, 4, 512)
    T = wl.bf16_bits_to_f32(X)
    q = oracle.quantize(T, "nvfp4", want_D=True)
    A = np.abs(T).max().astype(np.float64)
    assert abs(float(q.tscale) * 2688 - A) <= A * 2 ** -23
    genc = 2688.0 / A
    e = oracle.e4m3_decode(q.scales).astype(np.float64)
    bmax = np.abs(T).reshape(4, -1, 16).max(axis=2).astype(np.float64)
    target = bmax * genc / 6
    # e is one of the two E4M3 neighbours of the target and the nearer one
    allv = oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8)).astype(np.float64)
    for t, ev in zip(target.ravel(), e.ravel()):
        assert abs(ev - t) <= np.abs(allv - t).min() * (1 + 1e-6) + 1e-12
    dec = np.empty(T.shape)
    dec[:, 0::2] = oracle.e2m1_decode(q.codes & 15)
    dec[:, 1::2] = oracle.e2m1_decode(q.codes >> 4)
    x = T.astype(np.float64) * genc / np.repeat(e, 16, axis=1)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    ok = np.abs(np.abs(dec) - np.minimum(np.abs(x), 6.0)) <= \
        np.min(np.abs(np.minimum(np.abs(x), 6.0)[..., None] - grid), axis=-1) + 1e-6
    assert ok.all()


# ------------------------------------------------------------- prepare -----

@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
@pytest.mark.parametrize("n,m", [(2, 4), (1, 4), (4, 8)])
def test_prepare_reconstruction_exact(fmt, n, m):
    """y == fl(D_b + r) bitwise: the residual is taken against the
    dequantised backbone and the subtraction is exact (Sterbenz)."""
    X = wl.activation("laplace_outlier", 12, 0, 6, 1024)
    P = oracle.prepare(X, wl.gamma_ones(1024), 1e-6, n, m, fmt, keep_intermediates=True)
    blk = 16 if fmt == "nvfp4" else 32
    dec = np.empty(P.y.shape, dtype=np.float32)
    dec[:, 0::2] = oracle.e2m1_decode(P.bb.codes & 15)
    dec[:, 1::2] = oracle.e2m1_decode(P.bb.codes >> 4)
    sc = (oracle.e4m3_decode(P.bb.scales) if fmt == "nvfp4"
          else oracle.e8m0_decode(P.bb.scales))
    Db = (dec * np.repeat(sc, blk, axis=1)).astype(np.float32) * np.float32(P.bb.tscale)
    assert np.array_equal((Db + P.r).astype(np.float32), P.y)
    # pruned positions carry code 0 and their residual is y itself
    keep = np.unpackbits(P.mask, axis=1, bitorder="little").astype(bool)
    assert np.all(np.where(keep, True, (dec == 0) & ~np.signbit(dec)))
    assert np.array_equal(P.r[~keep], P.y[~keep])
    assert np.all(keep.reshape(6, -1, m).sum(axis=2) == n)
    # the residual is not the unquantised complement: kept entries differ
    assert np.any(P.r[keep] != 0)


def test_prepare_on_grid_sparse_input_has_zero_residual():
    """Input already on the NVFP4 grid with <= n nonzeros per group: the
    backbone holds it exactly, so the residual is zero (tensor scale 1)."""
    rng = np.random.default_rng(13)
    T = _grid_tensor_nvfp4(rng, 4, 256, 0, sparse24=True)
    X = _bf16(T)
    assert np.array_equal(wl.bf16_bits_to_f32(X), T)
    P = oracle.prepare(X, None, 1e-6, 2, 4, "nvfp4")
    assert np.all(P.rs.codes == 0) and P.rs.tscale == 1.0
    assert P.bb.tscale == 1.0


def test_prepare_commutes_with_row_gather():
    X = wl.activation("laplace_outlier", 14, 0, 9, 512)
    P = oracle.prepare(X, wl.gamma_ones(512), 1e-6)
    idx = np.array([3, 3, 0, 8, 1, 1, 1, 5, 2, 4, 6, 7])
    Q = oracle.prepare(X[idx], wl.gamma_ones(512), 1e-6)
    assert Q.bb.tscale == P.bb.tscale and Q.rs.tscale == P.rs.tscale
    for a, b in [(Q.bb.codes, P.bb.codes), (Q.bb.scales, P.bb.scales),
                 (Q.rs.codes, P.rs.codes), (Q.rs.scales, P.rs.scales), (Q.mask, P.mask)]:
        assert np.array_equal(a, b[idx])


# ---------------------------------------------------------------- GEMM -----

def test_linear_bruteforce_tiny():
    X = wl.activation("normal_outlier", 1, 0, 3, 64)
    W = wl.weight(1, 0, 5, 64)
    P = oracle.prepare(X, wl.gamma_ones(64), 1e-6)
    Wq = oracle.quantize_weight(W)
    Y = oracle.linear(P, Wq)

    def val(codes, scales, i, k):
        byte = int(codes[i, k // 2])
        c = byte & 15 if k % 2 == 0 else byte >> 4
        mag = [0, .5, 1, 1.5, 2, 3, 4, 6][c & 7] * (-1 if c & 8 else 1)
        return mag * float(oracle.e4m3_decode(np.array([scales[i, k // 16]]))[0])

    for i in range(3):
        for j in range(5):
            sb = sr = 0.0
            for k in range(64):
                w = val(Wq.codes, Wq.scales, j, k)
                sb += val(P.bb.codes, P.bb.scales, i, k) * w
                sr += val(P.rs.codes, P.rs.scales, i, k) * w
            want = float(Wq.tscale) * (float(P.bb.tscale) * sb + float(P.rs.tscale) * sr)
            assert abs(Y[i, j] - want) <= 1e-12 * max(1.0, abs(want))


def test_linear_on_grid_equals_plain_matmul():
    """X on the grid with r = 0 and W on the grid: the two-path linear is the
    plain fp64 product of the original values."""
    rng = np.random.default_rng(15)
    T = _grid_tensor_nvfp4(rng, 6, 256, -4, sparse24=True)
    W = _grid_tensor_nvfp4(rng, 16, 256, -9)
    P = oracle.prepare(_bf16(T), None, 1e-6, 2, 4, "nvfp4")
    Wq = oracle.quantize_weight(_bf16(W))
    Y = oracle.linear(P, Wq)
    ref = T.astype(np.float64) @ W.astype(np.float64).T
    assert np.allclose(Y, ref, rtol=1e-13, atol=1e-13 * np.abs(ref).max())


def test_linear_dense_residual_compensates():
    """The two-path result is closer to the unquantised product than the
    backbone path alone (the residual path carries mask loss and backbone
    quantisation error)."""
    X = wl.activation("laplace_outlier", 16, 0, 32, 1024)
    W = wl.weight(16, 0, 64, 1024)
    P = oracle.prepare(X, wl.gamma_ones(1024), 1e-6, keep_intermediates=True)
    Wq = oracle.quantize_weight(W)
    Y = oracle.linear(P, Wq)
    Dw = oracle.dequant_blocks(Wq) * float(Wq.tscale)
    exact = P.y.astype(np.float64) @ Dw.T
    bb_only = float(Wq.tscale) * float(P.bb.tscale) * (oracle.dequant_blocks(P.bb) @ oracle.dequant_blocks(Wq).T)
    assert np.linalg.norm(Y - exact) < 0.5 * np.linalg.norm(bb_only - exact)


def test_bf16_rne_reference():
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, -(1.0 + 2 ** -8), 1e-40, 3.0e38,
                  1.00390625 + 1e-12], dtype=np.float64)
    got = wl.bf16_bits_to_f32(oracle.bf16_rne_from_f64(v)).astype(np.float64)
    want = [1.0, 1.0, 1.0 + 2 ** -7, -1.0, None, None, 1.0078125]
    assert got[0] == want[0] and got[1] == want[1] and got[2] == want[2] and got[3] == want[3]
    assert got[6] == want[6]


def test_moe_reduces_to_per_expert_linear():
    X = wl.activation("laplace_outlier", 17, 0, 10, 256)
    P = oracle.prepare(X, wl.gamma_ones(256), 1e-6)
    experts = [oracle.quantize_weight(wl.weight(17, e, 32, 256)) for e in range(3)]
    ex = np.array([[0, 2], [1, 2], [0, 1], [2, 0], [1, 0], [0, 2], [2, 1], [0, 1], [1, 2], [2, 0]])
    ri, off = wl.group_by_expert(ex.astype(np.int32), 3)
    Y = oracle.moe_linear(P, ri, off, experts)
    for t in range(len(ri)):
        e = int(np.searchsorted(off, t, side="right") - 1)
        want = oracle.linear(oracle.gather_rows(P, ri[t:t + 1]), experts[e])[0]
        assert np.array_equal(Y[t], want)


# ---------------------------------------------------------------------------
# Residual quantised with the backbone's tensor scale ("shared" variant).
# ---------------------------------------------------------------------------

def _row32(vals):
    x = np.zeros((1, 32), dtype=np.float32)
    for k, v in vals.items():
        x[0, k] = v
    return wl.f32_to_bf16_bits(x)


def test_shared_residual_scale_worked_example():
    """One row, K = 32, no norm, 2:4, NVFP4; worked by hand.

    Backbone: element 0 = 2688 (with element 1 = 0 kept beside it; every
    all-zero group keeps its first two slots), and the
    group [768, 384, 384, 0] at elements 16..19 keeps 768 and the first 384.
    A_b = 2688, so G_enc = 1, G_dec = 1, K1 = fl(1/6); block 0 gets
    E4M3(fl(2688 K1)) = 448 (0x7E) and block 1 E4M3(fl(768 K1) = 128) = 0x70;
    every kept value is exactly on its grid, so the residual is zero except
    r[18] = 384 (the pruned 384).
    Own residual scale: A_r = 384, G_enc = 7, K1 = fl(7/6) and
    fl(384 fl(7/6)) is 448 - 2^-16, a tie that rounds to even 448: block
    scale 0x7E, G_r = fl(384/2688) = fl(1/7).
    Shared: A = A_b = 2688, fl(384 fl(1/6)) = 64: block scale 0x68 (64),
    G_r = 1.  Either way r[18] / scale-product is exactly 6 -> code 7."""
    X = _row32({0: 2688.0, 16: 768.0, 17: 384.0, 18: 384.0})
    own = oracle.prepare(X, None, 1e-6, 2, 4, "nvfp4", residual_scale="own")
    sh = oracle.prepare(X, None, 1e-6, 2, 4, "nvfp4", residual_scale="shared")
    for P in (own, sh):
        # every group keeps its first two slots here (all-zero groups too)
        assert list(P.mask[0]) == [0x33] * 4
        assert list(P.bb.scales[0]) == [0x7E, 0x70]
        assert float(P.bb.tscale) == 1.0
        rc = P.rs.codes[0]
        assert rc[9] == 0x07 and np.count_nonzero(rc) == 1             # element 18: code 7 (6.0)
        assert P.rs.scales[0, 0] == 0
    assert own.rs.scales[0, 1] == 0x7E
    assert np.float32(own.rs.tscale) == np.float32(384.0) / np.float32(2688.0)
    assert sh.rs.scales[0, 1] == 0x68
    assert float(sh.rs.tscale) == 1.0


def test_shared_equals_own_when_a_pruned_entry_ties_the_max():
    """If a pruned element's |y| equals the tensor maximum, max|r| = max|B|,
    so the two settings must give the same residual bit for bit."""
    X = wl.activation("laplace_outlier", 61, 0, 8, 256).copy()
    big = wl.f32_to_bf16_bits(np.array([[3000.0]], dtype=np.float32))[0, 0]
    X[3, 40:43] = big            # group 40..43: two of the three equal maxima are kept
    X[3, 43] = 0
    own = oracle.prepare(X, None, 1e-6, 2, 4, "nvfp4", residual_scale="own")
    sh = oracle.prepare(X, None, 1e-6, 2, 4, "nvfp4", residual_scale="shared")
    assert np.array_equal(own.rs.codes, sh.rs.codes)
    assert np.array_equal(own.rs.scales, sh.rs.scales)
    assert np.float32(own.rs.tscale) == np.float32(sh.rs.tscale)


def test_shared_residual_tensor_scale_is_the_backbones():
    X = wl.activation("laplace_outlier", 62, 0, 33, 512)
    for g in (None, wl.gamma_ones(512)):
        sh = oracle.prepare(X, g, 1e-6, 2, 4, "nvfp4", residual_scale="shared")
        own = oracle.prepare(X, g, 1e-6, 2, 4, "nvfp4", residual_scale="own")
        assert np.float32(sh.rs.tscale).view(np.uint32) == np.float32(sh.bb.tscale).view(np.uint32)
        assert np.array_equal(sh.bb.codes, own.bb.codes) and np.array_equal(sh.mask, own.mask)
        assert not np.array_equal(sh.rs.scales, own.rs.scales)     # a real difference on real data
    # MXFP4 has no tensor scale: the setting changes nothing
    a = oracle.prepare(X, None, 1e-6, 2, 4, "mxfp4", residual_scale="own")
    b = oracle.prepare(X, None, 1e-6, 2, 4, "mxfp4", residual_scale="shared")
    assert np.array_equal(a.rs.codes, b.rs.codes) and np.array_equal(a.rs.scales, b.rs.scales)


def _val_e2m1_bruteforce(codes, i, k):
    """Decoded E2M1 element k of row i, from the nibble layout and the format
    table written out here (not the oracle's decoder)."""
    byte = int(codes[i, k // 2])
    c = byte & 15 if k % 2 == 0 else byte >> 4
    return [0, .5, 1, 1.5, 2, 3, 4, 6][c & 7] * (-1.0 if c & 8 else 1.0)


def _scale_bruteforce(scales, fmt, i, k):
    """Block scale of element k of row i: E4M3 per 16 (bias 7, subnormals
    m * 2^-9) or E8M0 per 32 (2^(c - 127)), from the bit fields."""
    if fmt == "nvfp4":
        c = int(scales[i, k // 16])
        e, m = (c >> 3) & 15, c & 7
        return m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
    return 2.0 ** (int(scales[i, k // 32]) - 127)


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
@pytest.mark.parametrize("residual", ["own", "shared"])
def test_linear_abs_bruteforce_tiny(fmt, residual):
    """linear_abs sets the width of the GPU parity tolerance, so it is pinned
    from both sides: it must EQUAL the magnitude sum
    G_w (G_b sum_k |b_ik w_jk| + G_r sum_k |r_ik w_jk|), evaluated here index
    by index with its own decoder.  A tensor scale applied twice, a missing
    absolute value or a swapped operand would all change it."""
    X = wl.activation("laplace_outlier", 2, 7, 3, 128)
    W = wl.weight(2, 7, 5, 128)
    P = oracle.prepare(X, wl.gamma_ones(128), 1e-6, 2, 4, fmt, residual_scale=residual)
    Wq = oracle.quantize_weight(W, fmt)
    A = oracle.linear_abs(P, Wq)
    Y = oracle.linear(P, Wq)
    assert A.shape == (3, 5)
    for i in range(3):
        for j in range(5):
            ab = ar = yb = yr = 0.0
            for k in range(128):
                w = _val_e2m1_bruteforce(Wq.codes, j, k) * _scale_bruteforce(Wq.scales, fmt, j, k)
                b = _val_e2m1_bruteforce(P.bb.codes, i, k) * _scale_bruteforce(P.bb.scales, fmt, i, k)
                r = _val_e2m1_bruteforce(P.rs.codes, i, k) * _scale_bruteforce(P.rs.scales, fmt, i, k)
                ab += abs(b * w)
                ar += abs(r * w)
                yb += b * w
                yr += r * w
            gw, gb, gr = float(Wq.tscale), float(P.bb.tscale), float(P.rs.tscale)
            want = gw * (gb * ab + gr * ar)
            assert abs(A[i, j] - want) <= 1e-12 * want
            # the bound holds the signed result and is not slack by a constant
            assert abs(Y[i, j]) <= A[i, j] * (1 + 1e-12)
            assert abs(Y[i, j] - gw * (gb * yb + gr * yr)) <= 1e-12 * want
    # both paths contribute (neither half of the sum was dropped)
    assert np.abs(P.rs.codes & 0x77).sum() > 0 and np.abs(P.bb.codes & 0x77).sum() > 0


def _pruned_and_kept_residual_max(X, g, n=2, m=4):
    y = oracle.normalize(X, g, 1e-6)
    keep = oracle.mask(y, n, m).astype(bool)
    R = oracle.prepare(X, g, 1e-6, n, m, "nvfp4")
    D = (oracle.dequant_blocks(R.bb).astype(np.float32) * np.float32(R.bb.tscale))
    r = (y - D).astype(np.float32)
    P = np.abs(np.where(keep, np.float32(0), y)).max()
    Q = np.abs(np.where(keep, r, np.float32(0))).max()
    return P, Q, R


@pytest.mark.parametrize("dist,gk", [("student_t", None), ("student_t", "ones"),
                                     ("laplace_outlier", None), ("laplace_outlier", "ones")])
def test_residual_tensor_max_is_pruned_or_kept_max(dist, gk):
    """The residual of a pruned entry is y itself and that of a kept entry is
    y - dequant(backbone), so A_r = max(P, Q) with P the largest pruned |y|
    and Q the largest kept |y - D|.  The GPU prepare takes P in its first
    pass and guesses A_r = P; these inputs (the parity cases' distributions)
    cover both outcomes: P wins for Student-t activations, the kept
    outliers' quantisation error wins for outlier-channel ones."""
    X = wl.activation(dist, 21, 5, 128, 4096)
    g = None if gk is None else wl.gamma_ones(4096)
    P, Q, R = _pruned_and_kept_residual_max(X, g)
    A_r = np.float32(max(P, Q))
    assert np.float32(R.rs.tscale) == (np.float32(1) if A_r == 0 else np.float32(A_r / np.float32(2688)))
    if dist == "student_t":
        assert P >= Q
    else:
        assert Q > P


def test_bf16_rne_reference_against_exact_rounding():
    """RNE(Y64) to bf16 against a brute-force nearest-even choice on exact
    rationals, on random values and on values a hair off bf16 midpoints
    (where a rounding through fp32 first would land on the midpoint and
    then tie the wrong way)."""
    from fractions import Fraction
    rng = np.random.default_rng(5)
    base = rng.standard_normal(400) * 10.0 ** rng.integers(-6, 6, 400)
    mids = []
    for b in rng.integers(0x3000, 0x4F00, 200).astype(np.uint32):
        lo = float((b << np.uint32(16)).view(np.float32))
        hi = float(((b + np.uint32(1)) << np.uint32(16)).view(np.float32))
        mid = (lo + hi) / 2
        for d in (-1e-13, 1e-13, 0.0):
            mids += [mid * (1 + d), -mid * (1 + d)]
    Y = np.concatenate([base, np.array(mids)])
    got = oracle.bf16_rne_from_f64(Y)
    for y, g in zip(Y, got):
        q = Fraction(float(y))
        b32 = np.array([y], dtype=np.float32).view(np.uint32)[0] >> np.uint32(16)
        cands = [int(b32) + k for k in (-2, -1, 0, 1, 2) if 0 <= int(b32) + k < 0xFFFF]
        def val(c):
            return Fraction(float((np.uint32(c) << np.uint32(16)).view(np.float32)))
        cands = [c for c in cands if np.isfinite(float(val(c)))]
        best = min(cands, key=lambda c: (abs(val(c) - q), c & 1))
        assert int(g) == best, (y, hex(int(g)), hex(best))
