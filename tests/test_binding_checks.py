"""The Python binding checks every tensor's shape, dtype, layout and device
before it hands raw pointers to the C ABI (which cannot see shapes): a
mismatch raises ValueError and enqueues nothing."""
import pytest
import torch

import activation_sparsity_prep_b200 as sq


def test_host_tensors_and_wrong_dtypes_are_rejected_on_cpu():
    with pytest.raises(ValueError, match="CUDA"):
        sq.prepare(torch.zeros((4, 256), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="2-D"):
        sq.prepare(torch.zeros((256,), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="CUDA"):
        sq.quantize_weight(torch.zeros((128, 256), dtype=torch.float32))


gpu = pytest.mark.gpu


@gpu
def test_input_checks_on_the_device():
    dev = torch.device("cuda")
    X = torch.zeros((8, 256), dtype=torch.bfloat16, device=dev)
    with pytest.raises(ValueError, match="dtype"):
        sq.prepare(X.float())
    with pytest.raises(ValueError, match="contiguous"):
        sq.prepare(torch.zeros((256, 8), dtype=torch.bfloat16, device=dev).t())
    with pytest.raises(ValueError, match="gamma"):
        sq.prepare(X, torch.ones((128,), dtype=torch.bfloat16, device=dev))
    with pytest.raises(ValueError, match="beta"):
        sq.prepare_layernorm(X, torch.ones((256,), dtype=torch.bfloat16, device=dev),
                             torch.ones((255,), dtype=torch.bfloat16, device=dev))
    with pytest.raises(ValueError, match="out describes"):
        sq.prepare(X, out=sq.Prepared.empty(16, 256))
    with pytest.raises(ValueError, match="amax"):
        sq.prepare_amax(X, torch.zeros((2,), dtype=torch.float32, device=dev))
    with pytest.raises(ValueError, match="out describes"):
        sq.prepare_noalloc(X, out=sq.Prepared.empty(8, 512))


@gpu
def test_linear_checks_on_the_device():
    dev = torch.device("cuda")
    P = sq.Prepared.empty(8, 256)
    w = sq.Weight.empty(128, 256)
    with pytest.raises(ValueError, match="out"):
        sq.linear(P, w, out=torch.empty((8, 256), dtype=torch.bfloat16, device=dev))
    with pytest.raises(ValueError, match="dtype"):
        sq.linear(P, w, out_fp32=True, out=torch.empty((8, 128), dtype=torch.bfloat16, device=dev))
    with pytest.raises(ValueError, match="K="):
        sq.linear(P, sq.Weight.empty(128, 512))
    with pytest.raises(ValueError, match="format"):
        sq.linear(P, sq.Weight.empty(128, 256, "mxfp4"))
    short = sq.Prepared.empty(8, 256)
    short.bb_codes = short.bb_codes[:4]
    with pytest.raises(ValueError, match="bb_codes"):
        sq.linear(short, w)
    with pytest.raises(ValueError, match="out"):
        sq.linear_swiglu(P, w, out=torch.empty((8, 128), dtype=torch.bfloat16, device=dev))
    off = torch.tensor([0, 4, 8], dtype=torch.int32, device=dev)
    with pytest.raises(ValueError, match="experts"):
        sq.moe_linear(P, None, off, w)                       # 1 stacked weight, 2 experts
    w2 = sq.Weight.empty(128, 256, E=2)
    with pytest.raises(ValueError, match="row_index"):
        sq.moe_linear(P, torch.zeros((5,), dtype=torch.int64, device=dev), off, w2, T=5)
    with pytest.raises(ValueError, match="offsets"):
        sq.moe_linear(P, None, off.long(), w2)
