"""Pins of the oracle's fp32 normalisation arithmetic against an exact model
of IEEE-754 binary32: every operation is carried out on exact rationals and
rounded to nearest-even, written here from the definition of the format (24
significant bits, normal exponents down to -126, subnormals below), with no
use of the oracle's C code or of the CPU's fp32 unit.  Together with the
fixed reduction order (32 lanes, chunk c to lane c mod 32, element order in
a lane, xor butterfly 16..1) this fixes the RMSNorm and LayerNorm statistics
bit for bit, so a compiler that contracted, reordered or widened any step of
the oracle would fail here."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from activation_sparsity_prep_b200 import workloads as wl

TWO = Fraction(2)


def rne32(q: Fraction) -> Fraction:
    """The binary32 value nearest to q, ties to the even significand."""
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()      # 2^e <= a < 2^(e+2)
    if TWO ** e > a:
        e -= 1
    if TWO ** (e + 1) <= a:
        e += 1
    e = max(e, -126)                                               # subnormal spacing below
    ulp = TWO ** (e - 23)
    t = a / ulp
    n = t.numerator // t.denominator
    rem = t - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    assert n * ulp < TWO ** 128, "overflow is outside these pins"
    return sign * n * ulp


def f32_neighbours(v: Fraction):
    f = np.float32(float(v))
    assert Fraction(float(f)) == v
    lo = np.nextafter(f, np.float32(-np.inf), dtype=np.float32)
    hi = np.nextafter(f, np.float32(np.inf), dtype=np.float32)
    return Fraction(float(lo)), Fraction(float(hi))


def sqrt32(q: Fraction) -> Fraction:
    """Correctly rounded binary32 square root of q >= 0: the candidate from
    a double sqrt, moved until q lies between the squared midpoints to its
    neighbours (ties to even)."""
    assert q >= 0
    if q == 0:
        return Fraction(0)
    c = rne32(Fraction(float(np.sqrt(float(q)))))
    for _ in range(4):
        lo, hi = f32_neighbours(c)
        m_lo, m_hi = (lo + c) / 2, (c + hi) / 2
        if m_lo * m_lo > q:
            c = lo
        elif m_hi * m_hi < q:
            c = hi
        else:
            even = (int(np.float32(float(c)).view(np.uint32)) & 1) == 0
            if m_hi * m_hi == q and not even:
                c = hi
            elif m_lo * m_lo == q and not even:
                c = lo
            return c
    raise AssertionError("sqrt candidate did not settle")


def bf16(b) -> Fraction:
    return Fraction(float((np.uint32(b) << np.uint32(16)).view(np.float32)))


def f32(v) -> Fraction:
    return Fraction(float(np.float32(v)))


def canonical_sum(vals):
    lane = [Fraction(0)] * 32
    for c in range(len(vals) // 8):
        for t in range(8):
            lane[c % 32] = rne32(lane[c % 32] + vals[8 * c + t])
    o = 16
    while o >= 1:
        lane = [rne32(lane[l] + lane[l ^ o]) for l in range(32)]
        o >>= 1
    assert len(set(lane)) == 1          # every lane holds the same sum
    return lane[0]


def model_rinv(xb, eps):
    x = [bf16(b) for b in xb]
    S = canonical_sum([rne32(v * v) for v in x])
    ms = rne32(S / len(x))
    return rne32(1 / sqrt32(rne32(ms + f32(eps))))


def model_ln(xb, eps):
    x = [bf16(b) for b in xb]
    mu = rne32(canonical_sum(x) / len(x))
    d = [rne32(v - mu) for v in x]
    var = rne32(canonical_sum([rne32(v * v) for v in d]) / len(x))
    return mu, rne32(1 / sqrt32(rne32(var + f32(eps))))


ROWS = [("laplace_outlier", 256), ("student_t", 512), ("normal_outlier", 1024), ("laplace_outlier", 768)]


def test_model_rounding_against_known_values():
    # the model itself, on values whose rounding is known by hand
    assert rne32(Fraction(1) + TWO ** -24) == 1                       # tie: even (1.0)
    assert rne32(Fraction(1) + 3 * TWO ** -24) == 1 + TWO ** -22      # tie: up to even
    assert rne32(Fraction(1, 3)) == Fraction(float(np.float32(1 / 3)))
    assert rne32(TWO ** -149 * Fraction(3, 2)) == TWO ** -148         # subnormal tie to even
    assert sqrt32(Fraction(2)) == Fraction(float(np.float32(np.sqrt(np.float32(2)))))
    assert sqrt32(Fraction(9, 4)) == Fraction(3, 2)


@pytest.mark.parametrize("dist,K", ROWS)
def test_rms_rinv_is_the_exact_fp32_model(dist, K):
    X = wl.activation(dist, 95, K, 3, K)
    for row in X:
        got = Fraction(float(oracle.rms_rinv(row, 1e-6)))
        assert got == model_rinv(row, 1e-6)


@pytest.mark.parametrize("dist,K", ROWS)
def test_layernorm_stats_are_the_exact_fp32_model(dist, K):
    X = wl.activation(dist, 96, K, 2, K)
    for row in X:
        mu, rstd = oracle.ln_stats(row, 1e-6)
        wmu, wrstd = model_ln(row, 1e-6)
        assert Fraction(float(mu)) == wmu and Fraction(float(rstd)) == wrstd


def test_rmsnorm_outputs_are_the_exact_fp32_model():
    K = 256
    X = wl.activation("laplace_outlier", 97, 0, 2, K)
    g = wl.gamma_random(97, 0, K)
    y = oracle.normalize(X, g, 1e-6)
    for i, row in enumerate(X):
        r = model_rinv(row, 1e-6)
        want = [rne32(rne32(bf16(x) * r) * bf16(gk)) for x, gk in zip(row, g)]
        assert [Fraction(float(v)) for v in y[i]] == want


@pytest.mark.parametrize("with_beta", [False, True])
def test_layernorm_outputs_are_the_exact_fp32_model(with_beta):
    """y = fl(fl(fl(x - mu) * rstd) * gamma), then fl(. + beta) only when a
    bias is given, on the model's own mu and rstd."""
    K = 256
    X = wl.activation("student_t", 98, 0, 2, K)
    g = wl.gamma_random(98, 0, K)
    b = wl.beta_random(98, 0, K) if with_beta else None
    y = oracle.normalize_ln(X, g, b, 1e-6)
    for i, row in enumerate(X):
        mu, rstd = model_ln(row, 1e-6)
        want = [rne32(rne32(rne32(bf16(x) - mu) * rstd) * bf16(gk)) for x, gk in zip(row, g)]
        if with_beta:
            want = [rne32(w + bf16(bk)) for w, bk in zip(want, b)]
        assert [Fraction(float(v)) for v in y[i]] == want


def test_the_model_sees_a_different_order():
    """A plain left-to-right sum (a plausible mistake) gives other bits than
    the oracle on at least one of these rows, so the pins above constrain
    the order and not only the values."""
    differs = False
    for dist, K in ROWS:
        for row in wl.activation(dist, 95, K, 3, K):
            x = [bf16(b) for b in row]
            S = Fraction(0)
            for v in x:
                S = rne32(S + rne32(v * v))
            seq = rne32(1 / sqrt32(rne32(rne32(S / K) + f32(1e-6))))
            differs |= seq != Fraction(float(oracle.rms_rinv(row, 1e-6)))
    assert differs


# ------------------------------------------------ the NVFP4 / MXFP4 chains --
# The FP4 grids, written from the formats: E2M1 magnitudes of codes 0..7 and
# E4M3 (bias 7, 3 mantissa bits, subnormal spacing 2^-9, largest 448).

E2M1 = [Fraction(v) for v in ("0", "1/2", "1", "3/2", "2", "3", "4", "6")]
E4M3 = ([Fraction(m, 8) * TWO ** -6 for m in range(8)]
        + [(1 + Fraction(m, 8)) * TWO ** (e - 7) for e in range(1, 16) for m in range(8)])[:127]


def nearest_even(grid, v: Fraction) -> int:
    """Index (= code) of the grid value nearest to v >= 0, ties to the even
    code, values past the top saturating."""
    if v >= grid[-1]:
        return len(grid) - 1
    best = min(range(len(grid)), key=lambda c: (abs(grid[c] - v), c & 1))
    return best


def e2m1_code(v: Fraction, negative: bool) -> int:
    return nearest_even(E2M1, abs(v)) | (8 if negative else 0)


def keep_top2(vals):
    order = sorted(range(4), key=lambda i: (-abs(vals[i]), i))
    return {order[0], order[1]}


def model_nvfp4(Y, A):
    """Codes, block-scale codes and decode scale of Y (rows of exact values,
    already masked) under the reading: G_enc = fl(2688 / A), k1 = fl(G_enc /
    6), block code = E4M3(fl(amax_block * k1)), inv = fl(G_enc / e4m3(code)),
    element code = E2M1(fl(y * inv)), G_dec = fl(A / 2688)."""
    genc = rne32(Fraction(2688) / A) if A else Fraction(1)
    gdec = rne32(A / Fraction(2688)) if A else Fraction(1)
    k1 = rne32(genc / 6)
    codes, scales = [], []
    for row in Y:
        rc, rs = [], []
        for b0 in range(0, len(row), 16):
            blk = row[b0:b0 + 16]
            e = nearest_even(E4M3, rne32(max(abs(v) for v in blk) * k1))
            inv = rne32(genc / E4M3[e]) if e else Fraction(0)
            rs.append(e)
            rc += [e2m1_code(rne32(v * inv), v < 0) for v in blk]
        codes.append(rc)
        scales.append(rs)
    return codes, scales, gdec


def pack(codes_row):
    return [codes_row[2 * j] | (codes_row[2 * j + 1] << 4) for j in range(len(codes_row) // 2)]


def test_nvfp4_prepare_chain_is_the_exact_model():
    """Backbone and residual of a no-norm 2:4 prepare, every fp32 step
    through the exact model, against the oracle's bytes."""
    M, K = 2, 256
    X = wl.activation("laplace_outlier", 98, 0, M, K)
    R = oracle.prepare(X, None, 1e-6, 2, 4, "nvfp4")
    x = [[bf16(b) for b in row] for row in X]
    B = []
    for row in x:
        out = []
        for g0 in range(0, K, 4):
            kp = keep_top2(row[g0:g0 + 4])
            out += [row[g0 + i] if i in kp else Fraction(0) for i in range(4)]
        B.append(out)
    A_b = max(abs(v) for row in x for v in row)
    bc, bs, bgdec = model_nvfp4(B, A_b)
    assert [pack(r) for r in bc] == R.bb.codes.tolist()
    assert bs == R.bb.scales.tolist()
    assert Fraction(float(R.bb.tscale)) == bgdec
    # residual r = y - fl(fl(val * s) * G_dec), then its own chain
    res = []
    for i, row in enumerate(x):
        rr = []
        for k, v in enumerate(row):
            c = bc[i][k]
            d = rne32(rne32((-1 if c & 8 else 1) * E2M1[c & 7] * E4M3[bs[i][k // 16]]) * bgdec)
            rr.append(rne32(v - d))
        res.append(rr)
    A_r = max(abs(v) for row in res for v in row)
    rcodes, rscales, rgdec = model_nvfp4(res, A_r)
    assert [pack(r) for r in rcodes] == R.rs.codes.tolist()
    assert rscales == R.rs.scales.tolist()
    assert Fraction(float(R.rs.tscale)) == rgdec


def test_mxfp4_prepare_chain_is_the_exact_model():
    """MXFP4 backbone: block exponent floor(log2 amax) - 2 (biased 127),
    element code E2M1(y * 2^-(e-127)), no tensor scale."""
    M, K = 2, 256
    X = wl.activation("student_t", 99, 0, M, K)
    R = oracle.prepare(X, None, 1e-6, 2, 4, "mxfp4")
    for i, row in enumerate(X):
        x = [bf16(b) for b in row]
        out_codes, out_scales = [], []
        for b0 in range(0, K, 32):
            blk = x[b0:b0 + 32]
            kept = []
            for g0 in range(0, 32, 4):
                kp = keep_top2(blk[g0:g0 + 4])
                kept += [blk[g0 + j] if j in kp else Fraction(0) for j in range(4)]
            amax = max(abs(v) for v in kept)
            e = 0
            if amax:
                fl = amax.numerator.bit_length() - amax.denominator.bit_length()
                if TWO ** fl > amax:
                    fl -= 1
                e = max(fl - 2 + 127, 0)
            out_scales.append(e)
            out_codes += [e2m1_code(v * TWO ** (127 - e), v < 0) for v in kept]
        assert pack(out_codes) == R.bb.codes[i].tolist()
        assert out_scales == R.bb.scales[i].tolist()
    assert float(R.bb.tscale) == 1.0


def model_mxfp4(Y):
    """Element codes and E8M0 block exponents of rows of exact values:
    exponent floor(log2 amax) - 2 + 127 (clamped at 0; 0 for an all-zero
    block), element code E2M1(v * 2^(127 - e)) -- a power-of-two scaling,
    exact -- and the dequantised values val(code) * 2^(e - 127)."""
    codes, scales, deq = [], [], []
    for row in Y:
        rc, rs, rd = [], [], []
        for b0 in range(0, len(row), 32):
            blk = row[b0:b0 + 32]
            amax = max(abs(v) for v in blk)
            e = 0
            if amax:
                fl = amax.numerator.bit_length() - amax.denominator.bit_length()
                if TWO ** fl > amax:
                    fl -= 1
                e = max(fl - 2 + 127, 0)
            rs.append(e)
            for v in blk:
                c = e2m1_code(v * TWO ** (127 - e), v < 0)
                rc.append(c)
                rd.append((-1 if c & 8 else 1) * E2M1[c & 7] * TWO ** (e - 127))
        codes.append(rc)
        scales.append(rs)
        deq.append(rd)
    return codes, scales, deq


def test_mxfp4_residual_chain_is_the_exact_model():
    """MXFP4 residual: r = fl(y - D_b) with D_b the exact dequantised
    backbone, then r's own MXFP4 codes and exponents."""
    M, K = 3, 256
    X = wl.activation("laplace_outlier", 100, 0, M, K)
    R = oracle.prepare(X, None, 1e-6, 2, 4, "mxfp4")
    x = [[bf16(b) for b in row] for row in X]
    B = []
    for row in x:
        out = []
        for g0 in range(0, K, 4):
            kp = keep_top2(row[g0:g0 + 4])
            out += [row[g0 + i] if i in kp else Fraction(0) for i in range(4)]
        B.append(out)
    bc, bs, bd = model_mxfp4(B)
    assert [pack(r) for r in bc] == R.bb.codes.tolist() and bs == R.bb.scales.tolist()
    res = [[rne32(v - d) for v, d in zip(row, drow)] for row, drow in zip(x, bd)]
    rc, rs, _ = model_mxfp4(res)
    assert [pack(r) for r in rc] == R.rs.codes.tolist()
    assert rs == R.rs.scales.tolist()
    assert float(R.rs.tscale) == 1.0


def test_nvfp4_shared_residual_chain_is_the_exact_model():
    """Shared residual scale: the residual's quantiser takes the backbone's
    tensor maximum A_b, so its G_enc, k1 and G_dec are the backbone's."""
    M, K = 2, 256
    X = wl.activation("student_t", 101, 0, M, K)
    R = oracle.prepare(X, None, 1e-6, 2, 4, "nvfp4", residual_scale="shared")
    x = [[bf16(b) for b in row] for row in X]
    B = []
    for row in x:
        out = []
        for g0 in range(0, K, 4):
            kp = keep_top2(row[g0:g0 + 4])
            out += [row[g0 + i] if i in kp else Fraction(0) for i in range(4)]
        B.append(out)
    A_b = max(abs(v) for row in x for v in row)
    bc, bs, bgdec = model_nvfp4(B, A_b)
    assert [pack(r) for r in bc] == R.bb.codes.tolist()
    res = []
    for i, row in enumerate(x):
        rr = []
        for k, v in enumerate(row):
            c = bc[i][k]
            d = rne32(rne32((-1 if c & 8 else 1) * E2M1[c & 7] * E4M3[bs[i][k // 16]]) * bgdec)
            rr.append(rne32(v - d))
        res.append(rr)
    rcodes, rscales, rgdec = model_nvfp4(res, A_b)
    assert [pack(r) for r in rcodes] == R.rs.codes.tolist()
    assert rscales == R.rs.scales.tolist()
    assert Fraction(float(R.rs.tscale)) == rgdec == bgdec


def test_pair_prepare_chain_is_the_exact_model():
    """Pair-granular 4:8 prepare with RMSNorm: y on the exact model, pair
    magnitude max(|y_2i|, |y_2i+1|), the two strongest of four pairs kept
    (ties to the lower pair), MXFP4 backbone and residual, and the
    compressed form: the kept pairs' code bytes in order and one nibble per
    group of eight (lower kept pair index in bits 1:0), group 2j in the low
    nibble of byte j."""
    M, K = 2, 256
    X = wl.activation("laplace_outlier", 102, 0, M, K)
    g = wl.gamma_random(102, 0, K)
    P, kept, meta = oracle.prepare_pairs(X, g, 1e-6)
    ys, B, nibs = [], [], []
    for row in X:
        r = model_rinv(row, 1e-6)
        y = [rne32(rne32(bf16(xv) * r) * bf16(gk)) for xv, gk in zip(row, g)]
        ys.append(y)
        out, rn = [], []
        for g0 in range(0, K, 8):
            mag = [max(abs(y[g0 + 2 * p]), abs(y[g0 + 2 * p + 1])) for p in range(4)]
            order = sorted(range(4), key=lambda p: (-mag[p], p))
            lo, hi = sorted(order[:2])
            rn.append(lo | (hi << 2))
            out += [y[g0 + i] if i // 2 in (lo, hi) else Fraction(0) for i in range(8)]
        B.append(out)
        nibs.append(rn)
    bc, bs, bd = model_mxfp4(B)
    assert [pack(r) for r in bc] == P.bb.codes.tolist() and bs == P.bb.scales.tolist()
    for i in range(M):
        packed = pack(bc[i])
        want_kept = []
        for gi, nb in enumerate(nibs[i]):
            want_kept += [packed[4 * gi + (nb & 3)], packed[4 * gi + (nb >> 2)]]
        assert want_kept == kept[i].tolist()
        want_meta = [nibs[i][2 * j] | (nibs[i][2 * j + 1] << 4) for j in range(K // 16)]
        assert want_meta == meta[i].tolist()
    res = [[rne32(v - d) for v, d in zip(row, drow)] for row, drow in zip(ys, bd)]
    rc, rs, _ = model_mxfp4(res)
    assert [pack(r) for r in rc] == P.rs.codes.tolist() and rs == P.rs.scales.tolist()
