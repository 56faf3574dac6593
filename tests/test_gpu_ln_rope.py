"""Fused LayerNorm + adaLN + NVFP4 (kl_ln_modulate_quantize_nvfp4) and the
RoPE table (kl_rope_table) vs the oracle."""

import numpy as np
import pytest
import torch

import diffusion_transformer_image_nvfp4_b200 as kl
from oracle import block, codecs, nvfp4
from synth import normal_bf16
from tests.helpers import f32_bits, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,cols,seed", [(48, 128, 0), (320, 512, 1), (4608, 3072, 2)])
def test_ln_modulate_quantize(rows, cols, seed):
    x = normal_bf16((rows, cols), seed)
    shift = normal_bf16((cols,), seed + 100, 0.1)
    scale = normal_bf16((cols,), seed + 200, 0.1)
    q, m = kl.ln_modulate_quantize_nvfp4(x.cuda(), shift.cuda(), scale.cuda(), export_m=True)
    torch.cuda.synchronize()
    m_gpu = to_np(m)
    m_ref = block.modulate(x.float().numpy(), shift.float().numpy(), scale.float().numpy())
    # fp32 statistics vs fp64: the bf16 result may differ by one ulp on a few elements
    diff = np.abs(m_gpu - m_ref)
    ulp = np.abs(m_ref) * 2.0 ** -7 + 2.0 ** -133
    assert np.all(diff <= ulp)
    assert np.mean(diff == 0) > 0.995
    # the codes are exactly the NVFP4 encoding of the kernel's own bf16 m
    c, s, g = nvfp4.quantize(m_gpu)
    assert f32_bits(to_np(q.gs)[0]) == f32_bits(g)
    np.testing.assert_array_equal(to_np(kl.scales_mma_to_linear(q.scales, rows, cols)), s)
    np.testing.assert_array_equal(to_np(q.codes), c)


def test_ln_constant_rows_and_scale_minus_one():
    # scale = -1 gives m = shift for every row, whatever x
    x = normal_bf16((130, 256), 3)
    shift = normal_bf16((256,), 4, 0.1)
    scale = torch.full((256,), -1.0, dtype=torch.bfloat16)
    _, m = kl.ln_modulate_quantize_nvfp4(x.cuda(), shift.cuda(), scale.cuda(), export_m=True)
    np.testing.assert_array_equal(to_np(m), np.broadcast_to(shift.float().numpy(), (130, 256)))


@pytest.mark.parametrize("lay", [(64, 16, 16, 0), (512, 64, 64, 1), (7, 3, 5, 2)])
def test_rope_table(lay):
    cs = to_np(kl.rope_table(*lay))
    phi = block.rope_angles(block.TokenLayout(*lay))
    np.testing.assert_allclose(cs[..., 0], np.cos(phi), rtol=0, atol=2e-7)
    np.testing.assert_allclose(cs[..., 1], np.sin(phi), rtol=0, atol=2e-7)
