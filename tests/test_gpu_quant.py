"""MXFP8 quantiser (1x32 ue8m0 scales, e4m3 codes) bit-exact against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_persistent_b200 import quantize_mxfp8
from tests._support import bits_to_bf16

pytestmark = pytest.mark.gpu


def _special_rows():
    rows = np.zeros((6, 64), np.float32)
    rows[1, :32] = 448.0 * 2.0 ** -3          # amax exactly 448 * 2^e
    rows[1, 32:] = np.linspace(-57, 57, 32)   # just above 448 * 2^-3
    rows[2, :] = 1e-30                        # tiny
    rows[3, :] = np.linspace(-3e38, 3e38, 64)
    rows[4, ::2] = 1.0
    rows[4, 1::2] = -1.75
    rows[5, :] = 2.0 ** -133                  # bf16 subnormal
    return rows


@pytest.mark.parametrize("shape", [(6, 64), (1000, 7168), (37, 2048)])
def test_quantize_matches_oracle(shape):
    g = torch.Generator().manual_seed(shape[0])
    x = torch.randn(shape, generator=g) * torch.exp2(torch.randint(-20, 20, (shape[0], 1), generator=g).float())
    if shape == (6, 64):
        x = torch.from_numpy(_special_rows())
    xb = x.to(torch.bfloat16)
    bits = xb.view(torch.int16).numpy().view(np.uint16)
    q, s = quantize_mxfp8(xb.cuda())
    torch.cuda.synchronize()
    oq, os_ = oracle.mx_quantize(bits)
    assert np.array_equal(s.cpu().numpy(), os_)
    assert np.array_equal(q.cpu().numpy(), oq)


@pytest.mark.parametrize("shape", [(256, 512), (384, 7168)])
def test_weight_quantize_packs_the_same_scales(shape):
    """moe_quantize_mxfp8_weights: the same codes as the oracle, and the oracle's scales
    at the packed weight-scale offsets (every byte of the packed buffer written once)."""
    from mixture_experts_layer_persistent_b200 import quantize_mxfp8_weights
    from tests._support import packed_scale_offsets
    g = torch.Generator().manual_seed(shape[1])
    x = torch.randn(shape, generator=g) * torch.exp2(torch.randint(-20, 20, (shape[0], 1), generator=g).float())
    xb = x.to(torch.bfloat16)
    bits = xb.view(torch.int16).numpy().view(np.uint16)
    q, s = quantize_mxfp8_weights(xb.cuda())
    torch.cuda.synchronize()
    oq, os_ = oracle.mx_quantize(bits)
    assert np.array_equal(q.cpu().numpy(), oq)
    at = packed_scale_offsets(np.arange(shape[0]), shape[1] // 32, shape[0])
    assert np.array_equal(np.sort(at.ravel()), np.arange(s.numel()))
    assert np.array_equal(s.cpu().numpy()[at], os_)


@pytest.mark.parametrize("shape", [(2, 256, 192), (3, 512, 384)])
def test_transposed_weight_quantize_matches_oracle(shape):
    """moe_quantize_mxfp8_weights_t: codes [batch, C, R] and packed scales equal the
    oracle's quantisation of each transposed matrix (rows of src[b]^T along R),
    byte for byte, on rows of very different magnitudes (so the blocks down a
    column hold values far apart)."""
    from mixture_experts_layer_persistent_b200 import quantize_mxfp8_weights_t
    from tests._support import packed_scale_offsets
    batch, R, C = shape
    g = torch.Generator().manual_seed(R + C)
    x = torch.randn(shape, generator=g) * torch.exp2(torch.randint(-20, 20, (batch, R, 1), generator=g).float())
    xb = x.to(torch.bfloat16)
    q, s = quantize_mxfp8_weights_t(xb.cuda())
    torch.cuda.synchronize()
    bits = xb.view(torch.int16).numpy().view(np.uint16)
    t_bits = np.ascontiguousarray(bits.transpose(0, 2, 1)).reshape(batch * C, R)
    oq, os_ = oracle.mx_quantize(t_bits)
    assert np.array_equal(q.cpu().numpy().reshape(batch * C, R), oq)
    at = packed_scale_offsets(np.arange(batch * C), R // 32, batch * C)
    assert np.array_equal(np.sort(at.ravel()), np.arange(s.numel()))
    assert np.array_equal(s.cpu().numpy()[at], os_)


@pytest.mark.parametrize("shape", [(2, 256, 512), (3, 384, 768)])
def test_both_copies_in_one_pass(shape):
    """moe_quantize_mxfp8_weights_both: byte for byte the outputs of
    moe_quantize_mxfp8_weights and moe_quantize_mxfp8_weights_t, and in place."""
    from mixture_experts_layer_persistent_b200 import (quantize_mxfp8_weights, quantize_mxfp8_weights_both,
                                                       quantize_mxfp8_weights_t)
    g = torch.Generator().manual_seed(shape[2])
    x = torch.randn(shape, generator=g) * torch.exp2(torch.randint(-20, 20, (shape[0], shape[1], 1), generator=g).float())
    xb = x.to(torch.bfloat16).cuda()
    q, s, qt, st = quantize_mxfp8_weights_both(xb)
    q1, s1 = quantize_mxfp8_weights(xb)
    qt1, st1 = quantize_mxfp8_weights_t(xb)
    out = tuple(torch.full_like(t, 0x5A) for t in (q, s, qt, st))
    quantize_mxfp8_weights_both(xb, out)
    torch.cuda.synchronize()
    for a, b in ((q, q1), (s, s1), (qt, qt1), (st, st1)):
        assert torch.equal(a.view(-1), b.view(-1))
    for a, b in zip(out, (q, s, qt, st)):
        assert torch.equal(a, b)
