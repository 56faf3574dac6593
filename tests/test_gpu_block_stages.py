"""The joint block stage by stage against the oracle.

The block (kl_joint_block_forward) is first shown to be exactly the
composition of the library's stage entry points (ulysses.UlyssesBlock on one
rank runs LN + adaLN, the QKV GEMM with RoPE, the FP8 cast, attention, the
NVFP4 encodes, the output and MLP GEMMs one call at a time, and keeps every
intermediate): the two outputs are equal bit for bit.  Each stage is then
compared with the oracle's function for that stage applied to the GPU's own
previous intermediate, at the bars of the stage's unit tests:

* LayerNorm + adaLN m: one bf16 ulp (fp32 statistics against fp64);
* every NVFP4 encode (m1, O, m2, h) and the FP8 cast: bit-exact;
* GEMM epilogues (QKV + RoPE, gated residuals, SwiGLU): one bf16 ulp plus
  fp32 accumulation noise, nearly all elements equal; the gated branches
  themselves (x1 - x, out - x1, each with the oracle's own bf16 rounding of
  the sum) within 5e-3 relative L2, so a branch that is off by a few percent
  fails even though the residual dominates the output;
* attention: 5e-3 relative L2 against the oracle's FP8 flash pass on the same
  E4M3 operands (BF16: 1e-2 against fp64 softmax attention on the same bf16
  operands).

A stage that feeds on the GPU's previous output cannot hide behind a
legitimately different NVFP4 encoding upstream (a one-ulp amax difference
that moves a global scale), which is what loosens the end-to-end bars.  Rows
are sampled on the large workloads (every row on the tiny one); each sample
also holds the row with the largest |value| of each encoded tensor, so the
oracle derives the same per-tensor scale from the sample.
"""

import numpy as np
import pytest
import torch

import diffusion_transformer_image_nvfp4_b200 as kl
from diffusion_transformer_image_nvfp4_b200 import ulysses
from oracle import block, codecs, nvfp4
from synth import MOD_NAMES, WORKLOADS, block_inputs
from tests.helpers import rel_l2, to_np

pytestmark = pytest.mark.gpu

LOG2E = float(np.log2(np.e))


def _within_ulp(got, ref, noise, frac_equal, rel=2.0 ** -7):
    d = np.abs(got - ref)
    bad = d > np.abs(ref) * rel + noise
    assert not bad.any(), (int(bad.sum()), float(d[bad].max()))
    assert np.mean(d == 0) >= frac_equal, float(np.mean(d == 0))


def _nvfp4_np(triple, rows, cols):
    codes, scales, gs = triple
    lin = kl.scales_mma_to_linear(scales, rows, cols)
    return to_np(codes), to_np(lin), np.float32(to_np(gs)[0])


def _check_encode(x_gpu, enc_gpu, S):
    """NVFP4 of the GPU's bf16 tensor on rows S (which hold its largest |x|):
    bit-exact codes, scales and global scale."""
    codes, scales, gs = nvfp4.quantize(x_gpu[S])
    np.testing.assert_array_equal(enc_gpu[0][S], codes)
    np.testing.assert_array_equal(enc_gpu[1][S], scales)
    assert np.float32(gs).tobytes() == enc_gpu[2].tobytes()


def _with_argmax(S, *tensors):
    extra = [int(np.argmax(np.abs(t).max(axis=1))) for t in tensors]
    return np.unique(np.concatenate([S, extra]))


@pytest.mark.parametrize("name", ["tiny", "t2i_1024", "i2i_1024", "multiref_1024"])
def test_block_stages_against_the_oracle(name):
    wl = WORKLOADS[name]
    T, D, H, F = wl.n_tokens, wl.hidden, wl.heads, wl.mlp_hidden
    inp = block_inputs(name)
    dev = {k: v.cuda() for k, v in inp.items()}
    W = kl.prepare_block_weights(dev["wqkv"], dev["wo"], dev["w1"], dev["w2"])
    cs = kl.rope_table(wl.n_text, wl.grid_h, wl.grid_w, wl.n_ref)
    mod_d = {n: dev[n] for n in MOD_NAMES}
    ref_out = kl.joint_block_forward(W, dev["x"], mod_d, cs, H, F, attn=wl.attn).clone()
    tr = {}
    blk = ulysses.UlyssesBlock(W, T, D, H, F, wl.attn)
    out_d = blk.forward(dev["x"], mod_d, ulysses.local_rope(cs, 0, T), trace=tr)
    torch.cuda.synchronize()
    assert kl.device_status() == "KL_OK"
    # the traced composition is the block
    assert torch.equal(out_d, ref_out)

    x = inp["x"].float().numpy()
    mod = {n: inp[n].float().numpy() for n in MOD_NAMES}
    g = {k: to_np(v) for k, v in tr.items() if not isinstance(v, tuple)}
    if name == "tiny":
        S = np.arange(T)
    else:
        rng = np.random.default_rng(7)
        seg = [0, wl.n_text] + [wl.n_text + (k + 1) * wl.grid_h * wl.grid_w for k in range(wl.n_ref + 1)]
        S = np.unique(np.concatenate([rng.choice(T, 384, replace=False), seg[:-1], np.array(seg[1:]) - 1]))
    out = to_np(out_d)
    wq = {n: nvfp4.quantize(inp[n].float().numpy()) for n in ("wqkv", "wo", "w1", "w2")}

    # 1. LN1 + adaLN -> m1, NVFP4
    m1 = g["m1"]
    _within_ulp(m1[S], block.modulate(x[S], mod["shift1"], mod["scale1"]), 2.0 ** -16, 0.995)
    a1 = _nvfp4_np(tr["a1"], T, D)
    S1 = _with_argmax(S, m1)
    _check_encode(m1, a1, S1)

    # 2. QKV GEMM + RoPE (oracle GEMM on the GPU's m1 encoding), per-head amax
    qkv = g["qkv"]
    c = block.gemm_nvfp4((a1[0][S], a1[1][S], a1[2]), wq["wqkv"])
    phi = block.rope_angles(block.TokenLayout(wl.n_text, wl.grid_h, wl.grid_w, wl.n_ref))[S]
    q = block.apply_rope(c[:, :D].reshape(-1, H, 128), phi).reshape(-1, D)
    k = block.apply_rope(c[:, D:2 * D].reshape(-1, H, 128), phi).reshape(-1, D)
    ref = codecs.bf16_round(np.concatenate([q, k, c[:, 2 * D:]], axis=1))
    _within_ulp(qkv[S], ref, 1e-5 * np.abs(ref).max(), 0.98)
    np.testing.assert_array_equal(g["qkv_amax"], np.abs(qkv).reshape(T, 3, H, 128).max(axis=(0, 3)).reshape(-1))

    # 3-4. FP8 cast (bit-exact) and attention on the GPU's own operands
    qkv3 = qkv.reshape(T, 3 * H, 128)
    if wl.attn == "fp8":
        amax_rows = [int(np.argmax(np.abs(qkv3[:, j]).max(axis=1))) for j in range(3 * H)]
        S8 = np.unique(np.concatenate([S, amax_rows]))
        vals, scales = block.fp8_encode_heads(qkv3[S8])
        b8 = g["qkv8"].reshape(T, 3 * H, 128)
        np.testing.assert_array_equal(codecs.e4m3_decode(b8[S8]), vals)
        np.testing.assert_array_equal(g["sc8"], scales)
        sq, sk, sv = scales[:H], scales[H:2 * H], scales[2 * H:]
        o_emu = np.empty((len(S), H, 128))
        o_exact = np.empty((len(S), H, 128))
        for h in range(H):
            qh, kh, vh = (codecs.e4m3_decode(b8[:, j]) for j in (h, H + h, 2 * H + h))
            cc = LOG2E / np.sqrt(128.0) * float(sq[h]) * float(sk[h])
            acc, l = block.fp8_flash_rows(qh[S], kh, vh, cc)
            o_emu[:, h] = acc * float(sv[h]) / (16.0 * l[:, None])
            o_exact[:, h] = block.attention((qh * sq[h])[:, None], (kh * sk[h])[:, None], (vh * sv[h])[:, None],
                                            rows=S)[0][:, 0]
        o_gpu = g["o"].reshape(T, H, 128)[S]
        assert rel_l2(o_gpu, o_emu) <= 5e-3
        assert rel_l2(o_gpu, o_exact) <= 8e-2
    else:
        o_ref, _ = block.attention(qkv3[:, :H], qkv3[:, H:2 * H], qkv3[:, 2 * H:], rows=S)
        assert rel_l2(g["o"].reshape(T, H, 128)[S], o_ref) <= 1e-2

    # 5. NVFP4 of O (bit-exact on the GPU's O)
    o = g["o"]
    oq = _nvfp4_np(tr["oq"], T, D)
    _check_encode(o, oq, _with_argmax(S, o))

    # 6. out-projection + gated residual on the GPU's O encoding
    acc1 = block.gemm_nvfp4((oq[0][S], oq[1][S], oq[2]), wq["wo"])
    x1_ref = codecs.bf16_round(x[S] + mod["gate1"][None, :] * acc1)
    x1 = g["x1"]
    _within_ulp(x1[S], x1_ref, 1e-5 * np.abs(x1_ref).max(), 0.99)
    assert rel_l2(x1[S] - x[S], x1_ref - x[S]) <= 5e-3

    # 7. LN2 + adaLN -> m2, NVFP4
    m2 = g["m2"]
    _within_ulp(m2[S], block.modulate(x1[S], mod["shift2"], mod["scale2"]), 2.0 ** -16, 0.995)
    a2 = _nvfp4_np(tr["a2"], T, D)
    _check_encode(m2, a2, _with_argmax(S, m2))

    # 8. MLP-up + SwiGLU on the GPU's m2 encoding (W1 in the oracle's row order)
    gu = block.gemm_nvfp4((a2[0][S], a2[1][S], a2[2]), wq["w1"])
    h_ref = codecs.bf16_round(block.silu(gu[:, :F]) * gu[:, F:])
    h = g["h"]
    _within_ulp(h[S], h_ref, 1e-5 * np.abs(h_ref).max(), 0.97, rel=2.0 ** -6)

    # 9. NVFP4 of h (bit-exact on the GPU's h)
    hq = _nvfp4_np(tr["hq"], T, F)
    _check_encode(h, hq, _with_argmax(S, h))

    # 10. MLP-down + gated residual on the GPU's h encoding
    acc2 = block.gemm_nvfp4((hq[0][S], hq[1][S], hq[2]), wq["w2"])
    out_ref = codecs.bf16_round(x1[S] + mod["gate2"][None, :] * acc2)
    _within_ulp(out[S], out_ref, 1e-5 * np.abs(out_ref).max(), 0.99)
    assert rel_l2(out[S] - x1[S], out_ref - x1[S]) <= 5e-3
