"""tcgen05 NVFP4 GEMM (kl_gemm_nvfp4_fused) vs the oracle's fp64 GEMM of the
same NVFP4 operands, and its fused epilogues vs the oracle's definitions."""

import numpy as np
import pytest
import torch

import diffusion_transformer_image_nvfp4_b200 as kl
from oracle import block, codecs, nvfp4
from synth import normal_bf16
from tests.helpers import rel_l2, swiglu_perm, to_np

pytestmark = pytest.mark.gpu


def _operands(M, N, K, seed, w_std=0.02, perm=False):
    a = normal_bf16((M, K), seed)
    w = normal_bf16((N, K), seed + 1, w_std)
    A = kl.quantize_nvfp4(a.cuda())
    W = kl.quantize_nvfp4(w.cuda(), swiglu_interleave=perm)
    return a, w, A, W


def _ref(a, w, rows=None):
    an = a.float().numpy() if rows is None else a.float().numpy()
    qa = nvfp4.quantize(an)
    qw = nvfp4.quantize(w.float().numpy())
    A = nvfp4.dequantize(*qa)
    if rows is not None:
        A = A[rows]
    return A @ nvfp4.dequantize(*qw).T


def _bound(a, w, rows=None):
    """|sum| error scale: sum_k |a_k w_k| per output (fp32 accumulation error ~ K * 2^-24 of this)."""
    qa = nvfp4.quantize(a.float().numpy())
    qw = nvfp4.quantize(w.float().numpy())
    A = np.abs(nvfp4.dequantize(*qa))
    if rows is not None:
        A = A[rows]
    return A @ np.abs(nvfp4.dequantize(*qw)).T


# N = 384 and 128 run the 128-wide tiles (two TMEM accumulators), the others
# the 256-wide tiles; K = 64 / 320 end on a partial 256-wide K tile
@pytest.mark.parametrize("M,N,K", [(128, 128, 64), (128, 256, 256), (200, 384, 320), (1, 128, 512),
                                   (320, 1536, 512), (333, 512, 1536), (1000, 3072, 768)])
def test_gemm_f32_matches_oracle(M, N, K):
    a, w, A, W = _operands(M, N, K, seed=M + N + K)
    out = kl.gemm_nvfp4_fused(A, W, out_dtype=torch.float32)
    torch.cuda.synchronize()
    got = to_np(out)
    ref = _ref(a, w)
    bound = _bound(a, w)
    assert np.all(np.abs(got - ref) <= 1e-5 * bound + 1e-30)
    assert rel_l2(got, ref) <= 1e-5


@pytest.mark.parametrize("M,N,K", [(4608, 9216, 3072), (8704, 3072, 9216)])
def test_gemm_full_size_sampled_rows(M, N, K):
    # the QKV projection of the 1024^2 T2I block and the MLP down projection of
    # the I2I block, checked on sampled rows (the oracle decodes all of W)
    a, w, A, W = _operands(M, N, K, seed=M)
    out = kl.gemm_nvfp4_fused(A, W, out_dtype=torch.float32)
    rows = np.unique(np.concatenate([np.arange(0, M, 97), [M - 1]]))
    got = to_np(out)[rows]
    ref = _ref(a, w, rows)
    assert rel_l2(got, ref) <= 1e-5
    assert np.all(np.abs(got - ref) <= 1e-5 * _bound(a, w, rows) + 1e-30)


def test_bf16_output_and_single_block_operand():
    # an A with one nonzero 16-block picks that block of every W row
    M, N, K = 130, 256, 512
    a = torch.zeros((M, K), dtype=torch.bfloat16)
    a[129, 32:48] = 1.5
    w = normal_bf16((N, K), 21, 0.02)
    A, W = kl.quantize_nvfp4(a.cuda()), kl.quantize_nvfp4(w.cuda())
    got = to_np(kl.gemm_nvfp4_fused(A, W))
    ref = codecs.bf16_round(_ref(a, w))
    assert np.all(got[:129] == 0)
    # row 129 sums 16 products per output: a cancelling sum can leave fp32
    # accumulation noise where the fp64 sum is ~0, hence the absolute term
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2 ** -7 + 1e-5 * _bound(a, w))


def test_gated_residual_epilogue():
    M, N, K = 333, 512, 768
    a, w, A, W = _operands(M, N, K, seed=31)
    x = normal_bf16((M, N), 32)
    gate = normal_bf16((N,), 33, 0.1)
    got = to_np(kl.gemm_nvfp4_fused(A, W, "gated_residual", gate=gate.cuda(), residual=x.cuda()))
    ref = codecs.bf16_round(x.float().numpy() + gate.float().numpy()[None, :] * _ref(a, w))
    d = np.abs(got - ref)
    assert np.all(d <= np.abs(ref) * 2 ** -7 + 1e-6)
    assert np.mean(d == 0) > 0.99


@pytest.mark.parametrize("lay,H", [((16, 4, 4, 1), 1), ((64, 16, 16, 0), 4), ((37, 8, 8, 1), 2)])
def test_qkv_rope_epilogue(lay, H):
    layout = block.TokenLayout(*lay)
    T, D = layout.n_tokens, 128 * H
    a, w, A, W = _operands(T, 3 * D, D, seed=41 + H, w_std=0.05)
    cs = kl.rope_table(*lay)
    amax = torch.zeros(3 * H, dtype=torch.float32, device="cuda")
    got = to_np(kl.gemm_nvfp4_fused(A, W, "qkv_rope", rope_cs=cs, amax=amax))
    c = _ref(a, w)
    phi = block.rope_angles(layout)
    q = block.apply_rope(c[:, :D].reshape(T, H, 128), phi).reshape(T, D)
    k = block.apply_rope(c[:, D:2 * D].reshape(T, H, 128), phi).reshape(T, D)
    ref = codecs.bf16_round(np.concatenate([q, k, c[:, 2 * D:]], axis=1))
    d = np.abs(got - ref)
    assert np.all(d <= np.abs(ref) * 2 ** -7 + 1e-5 * np.abs(ref).max())
    assert np.mean(d == 0) > 0.98
    want_amax = np.abs(got).reshape(T, 3, H, 128).max(axis=(0, 3)).reshape(-1)
    np.testing.assert_array_equal(to_np(amax), want_amax.astype(np.float32))


def test_swiglu_epilogue():
    M, F, K = 300, 384, 512
    a = normal_bf16((M, K), 51)
    w1 = normal_bf16((2 * F, K), 52, 0.05)
    A = kl.quantize_nvfp4(a.cuda())
    W = kl.quantize_nvfp4(w1.cuda(), swiglu_interleave=True)
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    got = to_np(kl.gemm_nvfp4_fused(A, W, "swiglu", amax=amax))
    gu = _ref(a, w1)
    ref = codecs.bf16_round(block.silu(gu[:, :F]) * gu[:, F:])
    d = np.abs(got - ref)
    assert np.all(d <= np.abs(ref) * 2 ** -6 + 1e-5 * np.abs(ref).max())
    assert np.mean(d == 0) > 0.97
    assert to_np(amax)[0] == np.abs(got).max()


TILES = ["1cta_128x128", "1cta_128x256", "2sm_256x128", "2sm_256x256"]


@pytest.mark.parametrize("tile", TILES)
@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (200, 384, 320), (1, 128, 512), (333, 512, 1536),
                                   (1000, 3072, 768), (257, 768, 64)])
def test_gemm_tile_variants_match_oracle(tile, M, N, K):
    # every forced output-tile variant, including 2-SM pair tiles over a
    # ragged last pair (M = 257, 333, 1000) and a single-row M
    a, w, A, W = _operands(M, N, K, seed=7 * M + N + K)
    if tile.endswith("x256") and N % 256:
        with pytest.raises(kl.KLError, match="UNSUPPORTED_SHAPE"):
            kl.gemm_nvfp4_fused(A, W, out_dtype=torch.float32, tile=tile)
        return
    got = to_np(kl.gemm_nvfp4_fused(A, W, out_dtype=torch.float32, tile=tile))
    ref = _ref(a, w)
    assert np.all(np.abs(got - ref) <= 1e-5 * _bound(a, w) + 1e-30)
    assert rel_l2(got, ref) <= 1e-5


def test_gemm_tile_variants_bit_identical_with_epilogues():
    # the tile variants accumulate every output over the same 64-wide K steps
    # in the same order, so all four give the same bits, epilogues included
    M, N, K = 333, 1536, 768
    a, w, A, W = _operands(M, N, K, seed=91)
    Wp = kl.quantize_nvfp4(w.cuda(), swiglu_interleave=True)
    x = normal_bf16((M, N), 92).cuda()
    gate = normal_bf16((N,), 93, 0.1).cuda()
    lay = (13, 16, 20, 0)  # 13 + 320 = 333 tokens
    cs = kl.rope_table(*lay)
    outs = {}
    for tile in TILES:
        amax_q = torch.zeros(3 * (N // 384), dtype=torch.float32, device="cuda")
        amax_s = torch.zeros(1, dtype=torch.float32, device="cuda")
        outs[tile] = [
            to_np(kl.gemm_nvfp4_fused(A, W, out_dtype=torch.float32, tile=tile)),
            to_np(kl.gemm_nvfp4_fused(A, W, "gated_residual", gate=gate, residual=x, tile=tile)),
            to_np(kl.gemm_nvfp4_fused(A, W, "qkv_rope", rope_cs=cs, amax=amax_q, tile=tile)),
            to_np(kl.gemm_nvfp4_fused(A, Wp, "swiglu", amax=amax_s, tile=tile)),
            to_np(amax_q), to_np(amax_s),
        ]
    for tile in TILES[1:]:
        for got, want in zip(outs[tile], outs[TILES[0]]):
            np.testing.assert_array_equal(got, want)
