"""sharq_prepare_noalloc: the prepare entry point for callers that cannot
allocate device memory (graph-capture regions, framework-owned memory, hot
serving loops).  Its scratch is a fixed array inside the library, so the
test calls it through the C ABI twice in a row -- the second call runs on
the scratch contents the first one left -- and compares every output with
the workspace entry point sharq_prepare, bit for bit (the prepare parity
tolerance).  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import activation_sparsity_prep_b200 as sq
from activation_sparsity_prep_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _outputs(P):
    return [P.bb_codes, P.bb_scales, P.bb_tscale, P.rs_codes, P.rs_scales, P.rs_tscale, P.mask]


@pytest.mark.parametrize("M,K,gamma,fmt,rs", [(300, 4096, True, "nvfp4", "own"), (17, 768, False, "nvfp4", "own"),
                                              (129, 1024, True, "mxfp4", "own"),
                                              (200, 2048, True, "nvfp4", "shared")])
def test_noalloc_matches_workspace_entry_point_on_two_calls(M, K, gamma, fmt, rs):
    L = sq.load_sharq_ops()
    X = torch.from_numpy(wl.activation("laplace_outlier", 41, M, M, K)).view(torch.bfloat16).cuda()
    g = torch.from_numpy(wl.gamma_ones(K)).view(torch.bfloat16).cuda() if gamma else None
    ref = sq.prepare(X, g, wl.EPS, 2, 4, fmt, want_mask=True, residual_scale=rs)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        out = sq.Prepared.empty(M, K, 2, 4, fmt, want_mask=True, residual_scale=rs)
        for t in _outputs(out):
            t.fill_(0xA5 if t.dtype == torch.uint8 else 7.0)      # poison
        c = out._c()
        st = L.sharq_prepare_noalloc(ctypes.c_void_p(X.data_ptr()),
                                     None if g is None else ctypes.c_void_p(g.data_ptr()),
                                     ctypes.c_float(wl.EPS), ctypes.byref(c), stream)
        assert st == 0, f"call {call}: status {st}"
        torch.cuda.synchronize()
        assert sq.last_device_status() == 0
        for a, b in zip(_outputs(out), _outputs(ref)):
            assert torch.equal(a, b), f"call {call} differs from sharq_prepare"


def test_noalloc_rejects_rows_beyond_its_scratch():
    L = sq.load_sharq_ops()
    M = sq.NOALLOC_MAX_ROWS + 1
    c = sq._Prepared(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, None, M, 256, 2, 4, 0)
    assert L.sharq_prepare_noalloc(ctypes.c_void_p(0x1000), None, ctypes.c_float(1e-6),
                                   ctypes.byref(c), None) == 1
