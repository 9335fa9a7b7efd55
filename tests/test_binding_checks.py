"""The Python binding's own checks (weight_only_additive_b200/layer.py), on CPU
tensors: the kernels read and write exactly the sizes that (M, B, g, K, N, batch)
imply, so a tensor of another shape or dtype is rejected before any call reaches
the library."""
import numpy as np
import pytest
import torch

from weight_only_additive_b200 import layer as L
from weight_only_additive_b200 import synth


def _weights(M=2, B=8, g=8, K=64, N=16, **override):
    ld = synth.make_layer(M, B, g, K, N, seed=3, with_bias=True)
    raw = ld.codes.view(np.int16) if ld.codes.dtype == np.uint16 else ld.codes
    fields = dict(codes=torch.from_numpy(np.ascontiguousarray(raw)), codebooks=torch.from_numpy(ld.codebooks),
                  scales=torch.from_numpy(ld.scales), bias=torch.from_numpy(ld.bias), M=M, B=B, g=g)
    fields.update(override)
    return L.AqlmWeights(**fields)


@pytest.mark.parametrize("M,B,g", [(2, 8, 8), (1, 16, 8), (4, 8, 16), (2, 16, 16)])
def test_well_formed_weights_are_accepted(M, B, g):
    w = _weights(M, B, g)
    assert (w.N, w.K) == (16, 64)
    if B == 16:  # uint16 codes are taken as well as their int16 view
        _weights(M, B, g, codes=w.codes.view(torch.uint16))


def test_malformed_weights_are_rejected():
    w = _weights()
    with pytest.raises(TypeError):
        _weights(codes=w.codes.to(torch.int16))                  # B = 8 codes are bytes
    with pytest.raises(TypeError):
        _weights(M=1, B=16, codes=w.codes[:, :, :1].contiguous())  # B = 16 codes are 16-bit
    with pytest.raises(ValueError):
        _weights(codes=w.codes[:, :, :1].contiguous())           # M = 2 needs two codes per group
    with pytest.raises(ValueError):
        _weights(codes=w.codes.transpose(0, 1))                  # not contiguous
    with pytest.raises(ValueError):
        _weights(codebooks=w.codebooks[:, :128].contiguous())    # 2^B entries per codebook
    with pytest.raises(ValueError):
        _weights(codebooks=w.codebooks[:1].contiguous())         # M codebooks
    with pytest.raises(TypeError):
        _weights(codebooks=w.codebooks.float())
    with pytest.raises(ValueError):
        _weights(scales=w.scales[:8].contiguous())               # one scale per output row
    with pytest.raises(ValueError):
        _weights(bias=w.bias[:8].contiguous())
    _weights(bias=None)                                          # no bias is fine


def test_calls_need_cuda_weights():
    w = _weights()
    with pytest.raises(ValueError):
        L.matmul(torch.zeros((1, 64), dtype=torch.float16), w)
