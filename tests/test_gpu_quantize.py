"""NVFP4 quantiser (kl_quantize_nvfp4) vs the oracle: codes, scales and the
global scale must match bit for bit."""

import numpy as np
import pytest
import torch

import diffusion_transformer_image_nvfp4_b200 as kl
from oracle import nvfp4
from synth import normal_bf16
from tests.helpers import f32_bits, swiglu_perm, to_np

pytestmark = pytest.mark.gpu


def _check(x_bf16, layout="linear", gs=None, perm=False):
    x = x_bf16.contiguous()
    q = kl.quantize_nvfp4(x.cuda(), layout=layout, global_scale=gs, swiglu_interleave=perm)
    torch.cuda.synchronize()
    xn = x.float().numpy()
    if perm:
        xn = xn[swiglu_perm(xn.shape[0])]
    c, s, g = nvfp4.quantize(xn, gs=gs)
    assert f32_bits(to_np(q.gs)[0]) == f32_bits(g), (to_np(q.gs)[0], g)
    got_s = to_np(q.scales) if layout == "linear" else to_np(kl.scales_mma_to_linear(q.scales, *x.shape))
    np.testing.assert_array_equal(got_s, s)
    np.testing.assert_array_equal(to_np(q.codes), c)
    if layout == "mma":  # padding rows of the MMA layout hold scale 0
        R, C = x.shape
        total = to_np(q.scales).size
        assert total == ((R + 127) // 128) * 128 * (C // 16)
        assert int(to_np(q.scales).astype(np.int64).sum()) == int(s.astype(np.int64).sum())
    return q


@pytest.mark.parametrize("shape,seed,std", [((1, 16), 0, 1.0), ((3, 48), 1, 1.0), ((128, 512), 2, 1.0),
                                            ((333, 3072), 3, 1.0), ((1000, 1536), 4, 0.02), ((77, 64), 5, 300.0)])
def test_linear_layout_bit_exact(shape, seed, std):
    _check(normal_bf16(shape, seed, std), "linear")


@pytest.mark.parametrize("shape,seed", [((128, 64), 0), ((320, 512), 1), ((130, 3072), 2), ((4608, 3072), 3)])
def test_mma_layout_bit_exact(shape, seed):
    _check(normal_bf16(shape, seed), "mma")


def test_full_size_weight_bit_exact():
    # the largest weight of the 1024^2 block: W1 [2F, D] = [18432, 3072], N(0, 0.02)
    _check(normal_bf16((18432, 3072), 11, 0.02), "mma", perm=True)


def test_swiglu_interleave():
    _check(normal_bf16((768, 128), 12, 0.02), "mma", perm=True)


def test_given_global_scale():
    x = normal_bf16((64, 256), 13)
    _check(x, "linear", gs=np.float32(2.0 ** -7))
    _check(x, "mma", gs=np.float32(0.013))


def _adversarial():
    rows = []
    # exact E2M1 midpoints times a power-of-two block scale (see the oracle pins)
    blk0 = np.zeros(16, np.float32)
    blk0[0] = 2.625
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0, 0.0],
                    np.float32) * np.float32(0.25)
    rows.append(np.concatenate([blk0, mids, -mids, np.zeros(16, np.float32)]))
    # +-0, equal values, a single nonzero element, the amax element
    r = np.zeros(64, np.float32)
    r[16:32] = 0.75
    r[33] = -1.5
    r[48:64] = -0.0
    r[63] = 2.625
    rows.append(r)
    # a block 2^-120 smaller and one tiny negative in a normal block
    r = np.linspace(-2, 2, 64).astype(np.float32)
    r[0:16] *= np.float32(2.0 ** -120)
    r[20] = np.float32(-1e-6)
    rows.append(r)
    x = torch.from_numpy(np.stack(rows)).to(torch.bfloat16)
    return x


def test_adversarial_rows():
    x = _adversarial()
    _check(x, "linear")
    _check(x, "mma")


def test_extreme_magnitudes():
    big = (normal_bf16((8, 64), 14).float() * 2.0 ** 120).to(torch.bfloat16)
    _check(big, "linear")
    small = (normal_bf16((8, 64), 15).float() * 2.0 ** -125).to(torch.bfloat16)  # bf16 subnormals
    _check(small, "linear")
    _check(torch.zeros((4, 32), dtype=torch.bfloat16), "linear")
