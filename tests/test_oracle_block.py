"""Pins for the oracle's block pieces: LayerNorm/adaLN, RoPE, GEMM, attention,
SiLU, and the whole block (closed forms, invariants, library routines, brute
force)."""

import math
import os

import numpy as np
import pytest
import torch

from oracle import block, codecs, nvfp4
from synth import WORKLOADS, block_inputs, normal_bf16

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.txt")


def _facts():
    out = {}
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if line:
            k, v = line.split()
            out[k] = int(v)
    return out


# ---------------------------------------------------------------- token counts
def test_token_counts_match_pages():
    f = _facts()
    assert block.image_tokens(1024, 1024, f["vae_downsample"], f["patch"]) == f["tokens_per_1024_image"]
    assert block.image_tokens(256, 256) == 256
    t2i, i2i = WORKLOADS["t2i_1024"], WORKLOADS["i2i_1024"]
    assert t2i.hidden == f["hidden_width"]
    assert t2i.n_tokens == 512 + f["tokens_per_1024_image"]
    assert i2i.n_tokens - t2i.n_tokens == f["tokens_per_1024_reference"]
    assert WORKLOADS["multiref_1024"].n_tokens == 512 + 5 * 4096 == 20992
    assert WORKLOADS["multiref_21504"].n_tokens == 21504
    assert WORKLOADS["multiref_1024"].n_ref <= f["max_references"]
    lay = block.TokenLayout(512, 64, 64, 1)
    assert lay.n_tokens == i2i.n_tokens


# ----------------------------------------------------------------- LayerNorm
def test_layernorm_matches_torch():
    x = normal_bf16((33, 512), 1, 3.0).double()
    ref = torch.nn.functional.layer_norm(x, (512,), eps=1e-6).numpy()
    np.testing.assert_allclose(block.layernorm(x.numpy()), ref, rtol=1e-12, atol=1e-12)


def test_modulate_scale_minus_one_gives_shift():
    x = normal_bf16((7, 256), 2).float().numpy()
    shift = normal_bf16((256,), 3, 0.1).float().numpy()
    m = block.modulate(x, shift, -np.ones(256, np.float32))
    np.testing.assert_array_equal(m, np.broadcast_to(shift, m.shape))


# ---------------------------------------------------------------------- RoPE
def test_rope_position_zero_is_identity():
    lay = block.TokenLayout(3, 2, 2, 1)
    phi = block.rope_angles(lay)
    assert np.all(phi[0] == 0)                       # text token 0
    assert np.all(phi[lay.n_text] == 0)              # image (f, r, c) = (0, 0, 0)
    x = np.random.default_rng(0).standard_normal((lay.n_tokens, 2, 128))
    y = block.apply_rope(x, phi)
    np.testing.assert_array_equal(y[0], x[0])


def test_rope_matches_complex_rotation_and_keeps_norms():
    lay = block.TokenLayout(5, 3, 4, 2)
    phi = block.rope_angles(lay)
    x = np.random.default_rng(1).standard_normal((lay.n_tokens, 3, 128))
    y = block.apply_rope(x, phi)
    z = (x[..., 0::2] + 1j * x[..., 1::2]) * np.exp(1j * phi)[:, None, :]
    np.testing.assert_allclose(y[..., 0::2], z.real, rtol=0, atol=1e-12)
    np.testing.assert_allclose(y[..., 1::2], z.imag, rtol=0, atol=1e-12)
    n0 = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    n1 = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    np.testing.assert_allclose(n0, n1, rtol=1e-12)


def test_rope_relative_positions():
    # <R(p) q, R(p') k> depends only on p - p' (per axis): text tokens 2 and 5
    # vs 0 and 3, and image tokens shifted by the same (dr, dc)
    lay = block.TokenLayout(8, 6, 6, 1)
    phi = block.rope_angles(lay)
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 1, 128))
    k = rng.standard_normal((1, 1, 128))

    def dot(i, j):
        return float(np.sum(block.apply_rope(q, phi[i:i + 1]) * block.apply_rope(k, phi[j:j + 1])))

    assert dot(2, 5) == pytest.approx(dot(0, 3), rel=1e-12, abs=1e-12)
    t0 = lay.n_text

    def img(f, r, c):
        return t0 + f * lay.n_image + r * lay.grid_w + c

    assert dot(img(0, 1, 2), img(0, 3, 5)) == pytest.approx(dot(img(0, 2, 0), img(0, 4, 3)), rel=1e-10)
    # reference frame offset: same (r, c) on frames 0 and 1 differ only by f
    assert dot(img(0, 2, 2), img(1, 2, 2)) == pytest.approx(dot(img(0, 4, 1), img(1, 4, 1)), rel=1e-10)


def test_rope_angle_structure():
    lay = block.TokenLayout(4, 3, 5, 2)
    phi = block.rope_angles(lay)
    # text token i, pair 0 turns by exactly i; frequencies are geometric
    np.testing.assert_array_equal(phi[:4, 0], np.arange(4.0))
    ratio = phi[3, 1:] / phi[3, :-1]
    np.testing.assert_allclose(ratio, ratio[0], rtol=1e-12)
    np.testing.assert_allclose(ratio[0], 10000.0 ** (-1 / 64), rtol=1e-12)
    # first pair of each axial section turns by the axis position
    t = lay.n_text + 2 * lay.n_image + 1 * lay.grid_w + 3          # f=2, r=1, c=3
    assert (phi[t, 0], phi[t, 16], phi[t, 40]) == (2.0, 1.0, 3.0)
    # the last pair of the f / r sections uses the section's own dim
    np.testing.assert_allclose(phi[t, 15], 2.0 * 10000.0 ** (-30 / 32), rtol=1e-12)
    np.testing.assert_allclose(phi[t, 39], 1.0 * 10000.0 ** (-46 / 48), rtol=1e-12)


# ---------------------------------------------------------------------- GEMM
def test_gemm_matches_library_matmul():
    a = nvfp4.quantize(normal_bf16((40, 128), 4).float().numpy())
    w = nvfp4.quantize(normal_bf16((24, 128), 5, 0.02).float().numpy())
    ref = torch.from_numpy(nvfp4.dequantize(*a)) @ torch.from_numpy(nvfp4.dequantize(*w)).T
    np.testing.assert_allclose(block.gemm_nvfp4(a, w), ref.numpy(), rtol=1e-13, atol=1e-15)


def test_gemm_single_block_selects_weight_columns():
    # A with a single nonzero block (k in [16, 32)) of value c * S picks out
    # that block of every W row: C[m, n] = gA*gW * sum_{k in blk} a_k w[n, k]
    x = np.zeros((2, 64), np.float32)
    x[1, 16:32] = np.float32(1.5)
    a = nvfp4.quantize(x)
    w = nvfp4.quantize(normal_bf16((8, 64), 6).float().numpy())
    c = block.gemm_nvfp4(a, w)
    W = nvfp4.dequantize(*w)
    av = nvfp4.dequantize(*a)[1, 16]
    assert np.all(c[0] == 0)
    np.testing.assert_allclose(c[1], av * W[:, 16:32].sum(axis=1), rtol=1e-14)


# ----------------------------------------------------------------- attention
def test_attention_matches_torch_sdpa():
    rng = np.random.default_rng(7)
    q, k, v = (rng.standard_normal((50, 3, 128)) for _ in range(3))
    o, psum = block.attention(q, k, v, chunk=16)
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(t).permute(1, 0, 2) for t in (q, k, v)))
    np.testing.assert_allclose(o, ref.permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(psum, 1.0, atol=1e-12)


def test_attention_identical_values_and_single_token():
    rng = np.random.default_rng(8)
    q, k = rng.standard_normal((40, 2, 128)) * 5, rng.standard_normal((40, 2, 128)) * 5
    v = np.broadcast_to(rng.standard_normal((1, 2, 128)), (40, 2, 128))
    o, _ = block.attention(q, k, v)
    np.testing.assert_allclose(o, v, rtol=1e-13)
    o1, _ = block.attention(q[:1], k[:1], v[:1])
    np.testing.assert_allclose(o1, v[:1], rtol=1e-15)


def test_silu_matches_torch():
    g = np.linspace(-30, 30, 1001)
    np.testing.assert_allclose(block.silu(g), torch.nn.functional.silu(torch.from_numpy(g)).numpy(), rtol=1e-14)


# --------------------------------------------------------------------- block
def _micro_inputs(n_text=4, gh=2, gw=2, n_ref=1, D=128, F=384, seed=9):
    T = n_text + (1 + n_ref) * gh * gw
    g = torch.Generator().manual_seed(seed)

    def r(*s, std=1.0):
        return (torch.randn(*s, generator=g) * std).to(torch.bfloat16).float().numpy()

    x = r(T, D)
    mod = {n: r(D, std=0.1) for n in ("shift1", "scale1", "gate1", "shift2", "scale2", "gate2")}
    w = dict(wqkv=r(3 * D, D, std=0.02), wo=r(D, D, std=0.02), w1=r(2 * F, D, std=0.02), w2=r(D, F, std=0.02))
    return x, mod, w, block.TokenLayout(n_text, gh, gw, n_ref)


def test_block_zero_gates_is_identity():
    x, mod, w, lay = _micro_inputs()
    mod["gate1"] = np.zeros_like(mod["gate1"])
    mod["gate2"] = np.zeros_like(mod["gate2"])
    out = block.block_forward(x, mod, w, lay, 1)
    np.testing.assert_array_equal(out, x)


def test_block_constant_modulation_gives_uniform_attention_output():
    # scale1 = -1 makes every modulated token equal to shift1, so every v row
    # is the same and attention returns that row for every query
    x, mod, w, lay = _micro_inputs()
    mod["scale1"] = -np.ones_like(mod["scale1"])
    _, inter = block.block_forward(x, mod, w, lay, 1, keep=True)
    v = inter["v"].reshape(lay.n_tokens, -1)
    assert np.all(v == v[0])
    np.testing.assert_array_equal(inter["o"], np.broadcast_to(v[0], inter["o"].shape))


def _naive_block(x, mod, w, lay, H):
    """Every step as explicit loops over output elements (brute force)."""
    T, D = x.shape
    d = 128
    wq = {n: nvfp4.quantize(w[n]) for n in w}
    wdec = {n: nvfp4.dequantize(*wq[n]) for n in wq}
    F = wdec["w2"].shape[1]

    def ln_mod(xx, sh, sc):
        out = np.zeros_like(xx)
        for t in range(T):
            mu = math.fsum(xx[t]) / D
            var = math.fsum((float(v) - mu) ** 2 for v in xx[t]) / D
            for j in range(D):
                out[t, j] = ((xx[t, j] - mu) / math.sqrt(var + 1e-6)) * (1 + sh[1][j]) + sh[0][j]
        return codecs.bf16_round(out)

    def mm(a, wname):
        A = nvfp4.dequantize(*nvfp4.quantize(a))
        W = wdec[wname]
        out = np.zeros((A.shape[0], W.shape[0]))
        for i in range(A.shape[0]):
            for n in range(W.shape[0]):
                out[i, n] = math.fsum(A[i, kk] * W[n, kk] for kk in range(A.shape[1]))
        return out

    def angle(t, j):
        if t < lay.n_text:
            return t * 10000.0 ** (-2 * j / 128)
        s = t - lay.n_text
        f, rc = divmod(s, lay.grid_h * lay.grid_w)
        r, c = divmod(rc, lay.grid_w)
        if j < 16:
            return f * 10000.0 ** (-2 * j / 32)
        if j < 40:
            return r * 10000.0 ** (-2 * (j - 16) / 48)
        return c * 10000.0 ** (-2 * (j - 40) / 48)

    m1 = ln_mod(x, (mod["shift1"], mod["scale1"]), None)
    qkv = mm(m1, "wqkv")
    q = np.zeros((T, H, d)); k = np.zeros((T, H, d)); v = np.zeros((T, H, d))
    for t in range(T):
        for h in range(H):
            for j in range(64):
                ph = angle(t, j)
                cs, sn = math.cos(ph), math.sin(ph)
                for dst, off in ((q, 0), (k, D)):
                    a = qkv[t, off + 128 * h + 2 * j]
                    b = qkv[t, off + 128 * h + 2 * j + 1]
                    dst[t, h, 2 * j] = a * cs - b * sn
                    dst[t, h, 2 * j + 1] = a * sn + b * cs
            v[t, h] = qkv[t, 2 * D + 128 * h: 2 * D + 128 * h + 128]
    q, k, v = codecs.bf16_round(q), codecs.bf16_round(k), codecs.bf16_round(v)
    o = np.zeros((T, D))
    for h in range(H):
        for t in range(T):
            s = [math.fsum(q[t, h, i] * k[u, h, i] for i in range(d)) / math.sqrt(d) for u in range(T)]
            mx = max(s)
            e = [math.exp(si - mx) for si in s]
            z = math.fsum(e)
            for i in range(d):
                o[t, 128 * h + i] = math.fsum(e[u] * v[u, h, i] for u in range(T)) / z
    o = codecs.bf16_round(o)
    att = mm(o, "wo")
    x1 = codecs.bf16_round(x + mod["gate1"][None, :] * att)
    m2 = ln_mod(x1, (mod["shift2"], mod["scale2"]), None)
    gu = mm(m2, "w1")
    hh = np.zeros((T, F))
    for t in range(T):
        for j in range(F):
            g_ = gu[t, j]
            hh[t, j] = g_ / (1 + math.exp(-g_)) * gu[t, F + j]
    hh = codecs.bf16_round(hh)
    return codecs.bf16_round(x1 + mod["gate2"][None, :] * mm(hh, "w2"))


@pytest.mark.slow
def test_block_brute_force_micro():
    x, mod, w, lay = _micro_inputs()
    want = _naive_block(x, mod, w, lay, 1)
    got = block.block_forward(x, mod, w, lay, 1)
    # identical definitions; only summation order differs, which can move a
    # bf16 rounding by one ulp somewhere
    diff = np.abs(got - want)
    ulp = np.abs(want) * 2.0**-7 + 1e-30
    assert np.all(diff <= ulp)
    assert np.mean(diff == 0) > 0.99


def test_block_runs_on_tiny_workload():
    inp = {k: v.float().numpy() for k, v in block_inputs("micro").items()}
    wl = WORKLOADS["micro"]
    lay = block.TokenLayout(wl.n_text, wl.grid_h, wl.grid_w, wl.n_ref)
    mod = {k: inp[k] for k in ("shift1", "scale1", "gate1", "shift2", "scale2", "gate2")}
    out, inter = block.block_forward(inp["x"], mod, inp, lay, wl.heads, keep=True)
    assert out.shape == (wl.n_tokens, wl.hidden) and np.isfinite(out).all()
    # branch deltas are non-trivial
    assert np.abs(inter["x1"] - inp["x"]).max() > 0


def test_fp8_emulation_uniform_scores_give_mean_of_quantised_values():
    # q = 0 makes every score 0, every p exactly 1 (p * 16 = 16 is an E4M3
    # value), so O is the plain mean of the E4M3-decoded v, over any tiling
    rng = np.random.default_rng(12)
    T, H = 300, 2
    q = np.zeros((T, H, 128))
    k = rng.standard_normal((T, H, 128))
    v = rng.standard_normal((T, H, 128)).astype(np.float32)
    o = block.attention_fp8_emulated(q, k, v)
    v8, sv = block.fp8_encode_heads(v)
    want = (v8 * sv[None, :, None]).mean(axis=0)
    np.testing.assert_allclose(o, np.broadcast_to(want, o.shape), rtol=1e-12, atol=1e-15)
    o2 = block.attention_fp8_emulated(q, k, v, tile=64)
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-15)


def test_fp8_emulation_close_to_exact_and_rows_subset():
    rng = np.random.default_rng(13)
    q, k, v = (rng.standard_normal((260, 2, 128)) for _ in range(3))
    exact, _ = block.attention(q, k, v)
    emu = block.attention_fp8_emulated(q, k, v)
    err = np.linalg.norm(emu - exact) / np.linalg.norm(exact)
    assert 0.0 < err < 0.08
    rows = np.array([0, 5, 259])
    np.testing.assert_allclose(block.attention_fp8_emulated(q, k, v, rows=rows), emu[rows], rtol=1e-13)
    s, inv = block.fp8_head_scales(v)
    np.testing.assert_allclose(s * inv, 1.0, rtol=1e-6)


def _integer_score_case(seed, R=24, tiles=(0, 6, 9, 15, 13), tile=128, T=600):
    """E4M3-valued q8 [R, d], k8 [T, d], v8 [T, d] whose scores q8 . k8 are
    small integers: key j of tile i scores base_i - u_j + a_r * b_j with
    u_j in [0, 9] (0 at the tile's first key and at its key 64, so 64-key
    tiles have the same maxima), a_r in {-1, 0, 1}, b_j in {0, 1}.  With
    c = 1 every p = 2^(t - m) is then a power of two; the tile maxima rise
    by more than 4 at tiles 1 and 3, so the running maximum moves there."""
    rng = np.random.default_rng(seed)
    d = 128
    s = np.empty(T)
    for i, base in enumerate(tiles):
        j0, j1 = i * tile, min(T, (i + 1) * tile)
        u = rng.integers(0, 10, j1 - j0).astype(np.float64)
        u[0] = 0.0
        if j1 - j0 > 64:
            u[64] = 0.0
        s[j0:j1] = base - u
    a = rng.integers(-1, 2, R).astype(np.float64)
    b = rng.integers(0, 2, T).astype(np.float64)
    q8 = np.zeros((R, d))
    q8[:, 0] = 1.0
    q8[:, 1] = a
    k8 = np.zeros((T, d))
    k8[:, 0] = s
    k8[:, 1] = b
    v8 = codecs.e4m3_round(rng.standard_normal((T, d)) * 8.0)
    t = q8 @ k8.T
    assert np.array_equal(t, np.round(t)) and np.abs(k8).max() <= 16   # integers, exact in E4M3
    return q8, k8, v8, t


def _softmax2(t, v8):
    """sum_j 2^t_j v_j / sum_j 2^t_j in fp64 (the softmax in base 2)."""
    w = np.exp2(t - t.max(axis=1, keepdims=True))
    return (w @ v8) / w.sum(axis=1, keepdims=True)


@pytest.mark.parametrize("tau,tile", [(4.0, 128), (0.0, 128), (4.0, 64), (0.0, 64)])
def test_fp8_flash_rescale_is_exact_on_power_of_two_probabilities(tau, tile):
    # Every p * 16 is a power of two in [2^-9, 256], so E4M3 holds it exactly,
    # and the tile-by-tile pass must equal the plain softmax over the same
    # operands up to fp64 rounding -- through every move of the running
    # maximum (tiles 1 and 3 always move it; tau = 0 moves it whenever a tile
    # maximum rises).  A rescale of acc or l that is dropped, applied twice or
    # given the wrong sign breaks this by a factor of 2^5 or more.
    q8, k8, v8, t = _integer_score_case(21)
    acc, l = block.fp8_flash_rows(q8, k8, v8, 1.0, tile=tile, p_scale=16.0, tau=tau)
    np.testing.assert_allclose(acc / (16.0 * l[:, None]), _softmax2(t, v8), rtol=1e-12, atol=1e-12)
    # l itself is the sum of 2^(t - m_final), m_final the last reference maximum
    m_final = t[:, 384:512].max(axis=1)   # set at tile 3, never moved after it
    np.testing.assert_allclose(l, np.exp2(t - m_final[:, None]).sum(axis=1), rtol=1e-13)


def test_fp8_flash_visits_only_the_listed_tiles_in_order():
    # the same exact case restricted to a list of key tiles: equal to the
    # softmax over those tiles' keys (ascending lists, as the sparse path uses)
    q8, k8, v8, t = _integer_score_case(22)
    for tiles in ([0, 1, 3], [1, 2, 3, 4], [0, 3, 4], [3]):
        cols = np.concatenate([np.arange(j * 128, min(600, (j + 1) * 128)) for j in tiles])
        acc, l = block.fp8_flash_rows(q8, k8, v8, 1.0, key_tiles=tiles)
        np.testing.assert_allclose(acc / (16.0 * l[:, None]), _softmax2(t[:, cols], v8[cols]), rtol=1e-12,
                                   atol=1e-12)


def test_fp8_flash_rounds_p_for_the_product_but_sums_the_unrounded_p():
    # Two keys whose log2 scores are 0 and log2(1.1): the tile maximum is
    # log2(1.1), so p = (1/1.1, 1) and p * 16 = (14.545..., 16).  E4M3 has
    # steps of 1 on [8, 16): 14.545... rounds to 15 and 16 stays.  The product
    # uses the rounded values, the row sum the unrounded ones:
    # O = (15 v0 + 16 v1) / (16 * (1/1.1 + 1)).
    d = 128
    q8 = np.zeros((1, d))
    q8[0, 0] = 1.0
    k8 = np.zeros((2, d))
    k8[1, 0] = 1.0
    v8 = np.zeros((2, d))
    v8[0, 0] = 1.0
    v8[1, 1] = 2.0
    acc, l = block.fp8_flash_rows(q8, k8, v8, math.log2(1.1))
    np.testing.assert_allclose(l, [1.0 / 1.1 + 1.0], rtol=1e-15)
    want = np.zeros(d)
    want[0] = 15.0 / (16.0 * (1.0 / 1.1 + 1.0))
    want[1] = 32.0 / (16.0 * (1.0 / 1.1 + 1.0))
    np.testing.assert_allclose(acc[0] / (16.0 * l[0]), want, rtol=1e-14, atol=1e-15)
