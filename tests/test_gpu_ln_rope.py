"""Fused LayerNorm + adaLN + NVFP4 (kl_ln_modulate_quantize_nvfp4) and the
RoPE table (kl_rope_table) vs the oracle."""

import numpy as np
import pytest
import torch

import diffusion_transformer_image_nvfp4_b200 as kl
from oracle import block, codecs, nvfp4
from synth import normal_bf16
from tests.helpers import to_np

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
    # fp32 statistics vs fp64: m = LN(x)(1+scale)+shift is O(1) before the bf16
    # rounding, so fp32 leaves ~2^-22 absolute noise; the bf16 result may move
    # by one bf16 ulp on a few elements
    diff = np.abs(m_gpu - m_ref)
    assert np.all(diff <= np.abs(m_ref) * 2.0 ** -7 + 2.0 ** -16)
    assert np.mean(diff == 0) > 0.995
    # the fused encoder gives exactly what the standalone quantiser gives for
    # the kernel's own bf16 m (GPU against GPU; the standalone quantiser is
    # the one pinned bit-exact to the oracle on seeded inputs)
    q2 = kl.quantize_nvfp4(m)
    torch.cuda.synchronize()
    assert to_np(q.gs)[0].tobytes() == to_np(q2.gs)[0].tobytes()
    np.testing.assert_array_equal(to_np(q.scales), to_np(q2.scales))
    np.testing.assert_array_equal(to_np(q.codes), to_np(q2.codes))
    # and the scales it writes decode to the oracle's encoding of its reference m
    # within one global-scale rounding: compare decoded magnitudes loosely
    c, s, g = nvfp4.quantize(m_ref)
    assert abs(float(to_np(q.gs)[0]) / float(g) - 1) <= 2.0 ** -7


def test_ln_constant_rows_and_scale_minus_one():
    # scale = -1 gives m = shift for every row, whatever x
    x = normal_bf16((130, 256), 3)
    shift = normal_bf16((256,), 4, 0.1)
    scale = torch.full((256,), -1.0, dtype=torch.bfloat16)
    _, m = kl.ln_modulate_quantize_nvfp4(x.cuda(), shift.cuda(), scale.cuda(), export_m=True)
    np.testing.assert_array_equal(to_np(m), np.broadcast_to(shift.float().numpy(), (130, 256)))


@pytest.mark.parametrize("lay", [(64, 16, 16, 0), (512, 64, 64, 1), (7, 3, 5, 2)])
def test_rope_table(lay):
    cs16 = to_np(kl.rope_table(*lay))  # [16, T, 4, 2]: groups of 4 pairs
    cs = cs16.transpose(1, 0, 2, 3).reshape(cs16.shape[1], 64, 2)
    phi = block.rope_angles(block.TokenLayout(*lay))
    np.testing.assert_allclose(cs[..., 0], np.cos(phi), rtol=0, atol=2e-7)
    np.testing.assert_allclose(cs[..., 1], np.sin(phi), rtol=0, atol=2e-7)
