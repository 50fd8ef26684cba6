"""CPU-side checks of the C ABI: the library builds and loads, exports every
symbol include/sharq.h declares, and rejects bad arguments on the host
before touching a device."""
import ctypes
import os
import re

import numpy as np
import pytest

import activation_sparsity_prep_b200 as sq
from tests.sharq_testlib import atom_index

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "sharq.h")).read()
    return re.findall(r"SHARQ_API\s+[\w\s\*]+?\b(sharq_\w+)\s*\(", src)


def test_library_exports_every_declared_symbol():
    L = sq.load_sharq_ops()
    names = _declared()
    assert len(names) >= 8
    for n in names:
        assert hasattr(L, n), n


def test_scale_and_workspace_sizes():
    assert sq.scale_bytes(16, 256, "nvfp4") == 128 * 16
    assert sq.scale_bytes(129, 4096, "nvfp4") == 256 * 256
    assert sq.scale_bytes(128, 4096, "mxfp4") == 128 * 128
    assert sq.scale_bytes(16, 100, "nvfp4") == 0          # K % 256 != 0
    assert sq.prepare_workspace_bytes(1000, 4096) >= 64 + 8 * 1000
    assert sq.scale_bytes(0, 256) == 0


def test_atom_layout_is_a_permutation():
    idx = atom_index(256, 1024, "nvfp4")
    assert np.array_equal(np.sort(idx.ravel()), np.arange(256 * 64))


def _fake_prepared(M=16, K=256, n=2, m=4, fmt=0, p=0x1000, rs=0):
    return sq._Prepared(p, p, p, p, p, p, None, M, K, n, m, fmt, rs)


@pytest.mark.parametrize("kw", [dict(K=100), dict(m=3), dict(n=0), dict(n=5), dict(fmt=7),
                                dict(M=-1), dict(p=0x1001), dict(rs=2), dict(rs=-1)])
def test_prepare_rejects_bad_arguments_on_host(kw):
    L = sq.load_sharq_ops()
    cp = _fake_prepared(**kw)
    st = L.sharq_prepare(0x1000, None, 1e-6, ctypes.byref(cp), 0x1000, 1 << 20, None)
    assert st == 1


def test_prepare_rejects_small_workspace_and_bad_eps():
    L = sq.load_sharq_ops()
    cp = _fake_prepared()
    assert L.sharq_prepare(0x1000, None, 1e-6, ctypes.byref(cp), 0x1000, 8, None) == 1
    assert L.sharq_prepare(0x1000, None, float("nan"), ctypes.byref(cp), 0x1000, 1 << 20, None) == 1
    assert L.sharq_prepare(0x1000, None, 1e-6, None, 0x1000, 1 << 20, None) == 1


def test_linear_rejects_mismatched_operands():
    L = sq.load_sharq_ops()
    cp = _fake_prepared()
    w = sq._Weight(0x1000, 0x1000, 0x1000, 256, 512, 0)          # K mismatch
    assert L.sharq_linear(ctypes.byref(cp), ctypes.byref(w), 0x1000, 0, None) == 1
    w = sq._Weight(0x1000, 0x1000, 0x1000, 200, 256, 0)          # N % 128
    assert L.sharq_linear(ctypes.byref(cp), ctypes.byref(w), 0x1000, 0, None) == 1
    w = sq._Weight(0x1000, 0x1000, 0x1000, 256, 256, 1)          # format mismatch
    assert L.sharq_linear(ctypes.byref(cp), ctypes.byref(w), 0x1000, 0, None) == 1
    w = sq._Weight(0x1000, 0x1000, 0x1000, 256, 256, 0)
    assert L.sharq_linear(ctypes.byref(cp), ctypes.byref(w), 0x1008, 0, None) == 1   # misaligned Y
    ws = sq.moe_workspace_bytes(16, 4, 256)
    assert ws >= (16 + 4 * 128) * (256 + 32)
    assert L.sharq_moe_linear(ctypes.byref(cp), None, None, 4, 16, ctypes.byref(w), 0x1000, 0,
                              0x1000, ws, None) == 1                       # no offsets
    assert L.sharq_moe_linear(ctypes.byref(cp), None, 0x1000, 4, 17, ctypes.byref(w), 0x1000, 0,
                              0x1000, ws, None) == 1                       # T != M without row_index
    assert L.sharq_moe_linear(ctypes.byref(cp), None, 0x1000, 4, 16, ctypes.byref(w), 0x1000, 0,
                              0x1000, ws - 1, None) == 1                   # workspace too small
    assert L.sharq_moe_linear(ctypes.byref(cp), None, 0x1000, 300, 16, ctypes.byref(w), 0x1000, 0,
                              0x1000, 1 << 30, None) == 2                  # too many experts


def test_status_strings():
    L = sq.load_sharq_ops()
    assert L.sharq_status_string(0) == b"ok"
    assert L.sharq_status_string(4) == b"device wait timed out"


def test_unknown_residual_scale_is_rejected_everywhere():
    L = sq.load_sharq_ops()
    cp = _fake_prepared(rs=3)
    w = sq._Weight(0x1000, 0x1000, 0x1000, 256, 256, 0)
    assert L.sharq_linear(ctypes.byref(cp), ctypes.byref(w), 0x1000, 0, None) == 1
    ws = sq.moe_workspace_bytes(16, 4, 256)
    assert L.sharq_moe_linear(ctypes.byref(cp), None, 0x1000, 4, 16, ctypes.byref(w), 0x1000, 0,
                              0x1000, ws, None) == 1
    assert L.sharq_prepare_noalloc(0x1000, None, 1e-6, ctypes.byref(cp), None) == 1


def test_layernorm_prepare_needs_gamma_and_aligned_beta():
    L = sq.load_sharq_ops()
    cp = _fake_prepared()
    assert L.sharq_prepare_layernorm(0x1000, None, None, 1e-6, ctypes.byref(cp), 0x1000, 1 << 20, None) == 1
    assert L.sharq_prepare_layernorm(0x1000, 0x1000, 0x1004, 1e-6, ctypes.byref(cp), 0x1000, 1 << 20, None) == 1
    assert sq.prepare_workspace_bytes(1000, 4096) >= 64 + 8 * 1000      # mean and rstd per row


def test_workload_inputs_carry_the_norm_kind():
    from activation_sparsity_prep_b200 import workloads as wl
    W = wl.WORKLOADS["wan_dit"]
    d = wl.linear_inputs(W, W.linears[0], 4)
    assert d["norm"] == "layernorm" and d["beta"].shape == (5120,) and d["gamma"].shape == (5120,)
    d = wl.linear_inputs(W, W.linears[1], 4)
    assert d["norm"] == "rms" and d["gamma"] is None and d["beta"] is None


def test_swiglu_linear_rejects_bad_arguments_on_host():
    L = sq.load_sharq_ops()
    cp = _fake_prepared()
    w = sq._Weight(0x1000, 0x1000, 0x1000, 256, 256, 0)
    assert L.sharq_linear_swiglu(ctypes.byref(cp), ctypes.byref(w), 0x1000, None, None) == 1     # no amax
    assert L.sharq_linear_swiglu(ctypes.byref(cp), ctypes.byref(w), 0x1000, 0x1002, None) == 1   # misaligned amax
    assert L.sharq_linear_swiglu(ctypes.byref(cp), ctypes.byref(w), 0x1008, 0x1000, None) == 1   # misaligned H
    w = sq._Weight(0x1000, 0x1000, 0x1000, 192, 256, 0)                                           # N % 128
    assert L.sharq_linear_swiglu(ctypes.byref(cp), ctypes.byref(w), 0x1000, 0x1000, None) == 1
    cp = _fake_prepared(rs=2)
    w = sq._Weight(0x1000, 0x1000, 0x1000, 256, 256, 0)
    assert L.sharq_linear_swiglu(ctypes.byref(cp), ctypes.byref(w), 0x1000, 0x1000, None) == 1


@pytest.mark.parametrize("kw", [dict(K=100), dict(m=3), dict(n=0), dict(fmt=7), dict(p=0x1001), dict(rs=2)])
def test_prepare_amax_rejects_bad_arguments_on_host(kw):
    L = sq.load_sharq_ops()
    cp = _fake_prepared(**kw)
    assert L.sharq_prepare_amax(0x1000, 0x1000, ctypes.byref(cp), 0x1000, 1 << 20, None) == 1


def test_prepare_amax_needs_an_aligned_amax():
    L = sq.load_sharq_ops()
    cp = _fake_prepared()
    assert L.sharq_prepare_amax(0x1000, None, ctypes.byref(cp), 0x1000, 1 << 20, None) == 1
    assert L.sharq_prepare_amax(0x1000, 0x1001, ctypes.byref(cp), 0x1000, 1 << 20, None) == 1
    assert L.sharq_prepare_amax(0x1000, 0x1000, ctypes.byref(cp), 0x1000, 8, None) == 1          # workspace


def test_interleave_helper_matches_the_oracle_layout():
    import torch

    import oracle
    from activation_sparsity_prep_b200 import workloads as wl
    Wg, Wu = wl.weight(5, 1, 192, 256), wl.weight(5, 2, 192, 256)
    got = sq.interleave_gate_up(torch.from_numpy(Wg.view(np.int16)), torch.from_numpy(Wu.view(np.int16)))
    assert np.array_equal(got.numpy().view(np.uint16), oracle.interleave_gate_up(Wg, Wu))
    with pytest.raises(ValueError):
        sq.interleave_gate_up(torch.zeros(96, 256), torch.zeros(96, 256))


def test_moe_swiglu_needs_an_amax():
    L = sq.load_sharq_ops()
    cp = _fake_prepared()
    w = sq._Weight(0x1000, 0x1000, 0x1000, 256, 256, 0)
    ws = sq.moe_workspace_bytes(16, 4, 256)
    assert L.sharq_moe_linear_swiglu(ctypes.byref(cp), None, 0x1000, 4, 16, ctypes.byref(w), 0x1000,
                                     None, 0x1000, ws, None) == 1
    assert L.sharq_moe_linear_swiglu(ctypes.byref(cp), None, 0x1000, 4, 16, ctypes.byref(w), 0x1000,
                                     0x1001, 0x1000, ws, None) == 1
    assert L.sharq_moe_linear_swiglu(ctypes.byref(cp), None, 0x1000, 4, 16, ctypes.byref(w), 0x1000,
                                     0x1000, 0x1000, ws - 1, None) == 1


def test_public_api_names_resolve():
    for n in sq.__all__:
        assert hasattr(sq, n), n


def test_wait_selftest_rejects_bad_arguments_on_host():
    L = sq.load_sharq_ops()
    assert L.sharq_selftest_wait_timeout(None, 10000, None) == 1
    assert L.sharq_selftest_wait_timeout(0x1002, 10000, None) == 1      # misaligned
    assert L.sharq_selftest_wait_timeout(0x1000, 10, None) == 1         # below 1 ms
    assert L.sharq_selftest_wait_timeout(0x1000, 5_000_000, None) == 1  # above 1 s


def test_prepare_timeout_selftest_rejects_bad_arguments_on_host():
    L = sq.load_sharq_ops()
    cp = _fake_prepared()
    ok = L.sharq_selftest_prepare_timeout(ctypes.c_void_p(0x1000), ctypes.byref(cp), ctypes.c_void_p(0x1000),
                                          1 << 20, 10, None)
    assert ok == 1                                                          # limit below 1 ms
    cp.fmt = 1
    assert L.sharq_selftest_prepare_timeout(ctypes.c_void_p(0x1000), ctypes.byref(cp), ctypes.c_void_p(0x1000),
                                            1 << 20, 10000, None) == 1      # MXFP4 has no grid barriers here
    cp.fmt = 0
    cp.residual_scale = 1
    assert L.sharq_selftest_prepare_timeout(ctypes.c_void_p(0x1000), ctypes.byref(cp), ctypes.c_void_p(0x1000),
                                            1 << 20, 10000, None) == 1      # shared scale: one barrier only
