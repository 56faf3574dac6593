"""Joint transformer block forward, plain fp64 reading (TEST INFRASTRUCTURE ONLY).

What the pages fix:
* [P2] "FLUX.3 Image Klein Brings 2-Second AI Image Generation to Diffusers",
  §Summary, and [P4] "Welcome FLUX.3 Image Klein in Diffusers",
  §Architecture and Technical Deep Dive / Two-Stage Processing: after the
  per-mode blocks, text, noisy-image and reference tokens are concatenated and
  processed by joint blocks whose attention runs over all of them.
* [P4] §The VAE and Tokenization: 8x VAE and 2x2 patches, so a 1024x1024
  image is a 64x64 grid of 4,096 tokens; [P2] §Summary: each 1024x1024
  reference adds 4,096 tokens.
* [P1] "Optimizing FLUX 3 Image Klein inference on NVIDIA Blackwell GPUs",
  §How it works: NVFP4 weights and activations; GEMMs with fused SwiGLU and
  rotary position embeddings; FP8 query/key/value attention.

Readings (the pages are silent; each is the plainest choice consistent with
the above):
* token order [text; noisy image (row-major grid); ref 1; ...; ref R];
  attention is full and unmasked;
* LayerNorm over the hidden dim, biased variance, eps 1e-6, no affine; adaLN
  modulation m = LN(x) * (1 + scale) + shift with one (shift, scale, gate)
  triple per branch shared by all tokens; m is stored as bf16;
* QKV projection: columns [0, D) are q, [D, 2D) k, [2D, 3D) v; head h is
  columns [128h, 128h + 128) of each; no bias; no QK-norm;
* RoPE (theta 10000) rotates interleaved pairs (2j, 2j+1):
  (a, b) -> (a cos phi - b sin phi, a sin phi + b cos phi).  Text token i:
  phi_j = i * theta^(-2j/128) over all 64 pairs.  Image-family tokens carry
  (f, r, c) and split the 64 pairs into axial sections of 16 / 24 / 24 pairs
  with phi = p_axis * theta^(-2u/d_axis) (u the pair index inside the section,
  d_axis = 32 / 48 / 48).  The noisy image has f = 0; reference k has f = k on
  its own grid ("offset by a frame index");
* gated residuals x1 = x + gate1 * attn_out, out = x1 + gate2 * mlp_out,
  each stored as bf16;
* MLP: W1 rows [0, F) are the gate projection g, rows [F, 2F) the up
  projection u; h = silu(g) * u with silu(g) = g / (1 + exp(-g)); h stored as
  bf16 then NVFP4-encoded for the down projection.
Parity with the real model (section split, pairing, wiring) is unpinned; the
functions are pinned to closed forms, invariants and library routines.
"""

from dataclasses import dataclass

import numpy as np

from . import nvfp4
from .codecs import bf16_round, e4m3_round

ROPE_THETA = 10000.0
HEAD_DIM = 128
LN_EPS = 1e-6
AXIS_PAIRS = (16, 24, 24)          # pairs per axial section (f, r, c)


@dataclass(frozen=True)
class TokenLayout:
    """Segments of the joint sequence: L text tokens, a gh x gw noisy-image
    grid, and R reference images on grids of the same size."""

    n_text: int
    grid_h: int
    grid_w: int
    n_ref: int = 0

    @property
    def n_image(self):
        return self.grid_h * self.grid_w

    @property
    def n_tokens(self):
        return self.n_text + (1 + self.n_ref) * self.n_image


def image_tokens(pixels_h, pixels_w, vae_factor=8, patch=2):
    """Tokens per image: the VAE divides each side by 8 and 2x2 latent patches
    become one token ([P4] §The VAE and Tokenization)."""
    gh = pixels_h // vae_factor // patch
    gw = pixels_w // vae_factor // patch
    return gh * gw


# ---------------------------------------------------------------------------
# RoPE
# ---------------------------------------------------------------------------
def rope_angles(layout):
    """Angles phi [T, 64] (fp64) for every token and rotation pair."""
    T = layout.n_tokens
    phi = np.zeros((T, HEAD_DIM // 2), dtype=np.float64)
    # text: 1D over all 64 pairs
    j = np.arange(HEAD_DIM // 2, dtype=np.float64)
    inv_freq_1d = ROPE_THETA ** (-2.0 * j / HEAD_DIM)
    pos_text = np.arange(layout.n_text, dtype=np.float64)
    phi[: layout.n_text] = pos_text[:, None] * inv_freq_1d[None, :]
    # image-family tokens: (f, r, c) axial sections
    n_img = layout.n_image
    rows = np.repeat(np.arange(layout.grid_h, dtype=np.float64), layout.grid_w)
    cols = np.tile(np.arange(layout.grid_w, dtype=np.float64), layout.grid_h)
    for k in range(layout.n_ref + 1):
        t0 = layout.n_text + k * n_img
        axes = (np.full(n_img, float(k)), rows, cols)
        p0 = 0
        for pos, npairs in zip(axes, AXIS_PAIRS):
            u = np.arange(npairs, dtype=np.float64)
            inv_freq = ROPE_THETA ** (-2.0 * u / (2 * npairs))
            phi[t0 : t0 + n_img, p0 : p0 + npairs] = pos[:, None] * inv_freq[None, :]
            p0 += npairs
    return phi


def apply_rope(x, phi):
    """Rotate interleaved pairs of x [T, H, 128] by phi [T, 64] (fp64)."""
    x = np.asarray(x, dtype=np.float64)
    a = x[..., 0::2]
    b = x[..., 1::2]
    c = np.cos(phi)[:, None, :]
    s = np.sin(phi)[:, None, :]
    out = np.empty_like(x)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


# ---------------------------------------------------------------------------
# LayerNorm + adaLN modulation
# ---------------------------------------------------------------------------
def layernorm(x, eps=LN_EPS):
    """(x - mean) / sqrt(var + eps) over the last axis, biased variance, fp64."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps)


def modulate(x, shift, scale):
    """adaLN: bf16(LN(x) * (1 + scale) + shift), evaluated in fp64."""
    y = layernorm(x) * (1.0 + np.asarray(scale, np.float64)) + np.asarray(shift, np.float64)
    return bf16_round(y)


# ---------------------------------------------------------------------------
# NVFP4 GEMM
# ---------------------------------------------------------------------------
def gemm_nvfp4(a, w):
    """C[m, n] = gA * gW * sum_k dec(A)[m, k] * dec(W)[n, k] in fp64.

    ``a`` and ``w`` are (codes, scales, gs) triples from ``nvfp4.quantize``;
    both operands are K-major ("TN": y = x W^T).  Every product of decoded
    values is exact in fp64; only the summation rounds.
    """
    A = nvfp4.dequantize(*a)
    W = nvfp4.dequantize(*w)
    return A @ W.T


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------
def attention(q, k, v, rows=None, chunk=1024):
    """softmax(q k^T / sqrt(d)) v per head, fp64, max-subtracted.

    q, k, v: [T, H, d].  ``rows`` optionally restricts the query rows
    computed.  Returns (O [len(rows), H, d], row sums of the normalised
    probabilities [len(rows), H]) -- the latter are 1 up to rounding.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    T, H, d = q.shape
    rows = np.arange(T) if rows is None else np.asarray(rows)
    out = np.empty((len(rows), H, d), dtype=np.float64)
    psum = np.empty((len(rows), H), dtype=np.float64)
    scale = 1.0 / np.sqrt(d)
    for h in range(H):
        kh = k[:, h, :]
        vh = v[:, h, :]
        for r0 in range(0, len(rows), chunk):
            rr = rows[r0 : r0 + chunk]
            s = (q[rr, h, :] @ kh.T) * scale
            s -= s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)
            out[r0 : r0 + len(rr), h, :] = p @ vh
            psum[r0 : r0 + len(rr), h] = p.sum(axis=1)
    return out, psum


def fp8_head_scales(x):
    """Per-head E4M3 decode scale s_h = amax_h / 448 and encode multiplier
    448 / amax_h (both fp32; 1 and 1 when amax_h is 0) of x [T, H, d]."""
    amax = np.max(np.abs(np.asarray(x, np.float32)), axis=(0, 2)).astype(np.float32)
    nz = amax > 0
    safe = np.where(nz, amax, np.float32(1.0))
    s = np.where(nz, (safe / np.float32(448.0)).astype(np.float32), np.float32(1.0)).astype(np.float32)
    inv = np.where(nz, (np.float32(448.0) / safe).astype(np.float32), np.float32(1.0)).astype(np.float32)
    return s, inv


def fp8_encode_heads(x):
    """E4M3 values (decoded, unscaled) of x * (448 / amax_h), and the decode
    scales s_h: x is approximated by e4m3 * s_h."""
    s, inv = fp8_head_scales(x)
    y = (np.asarray(x, np.float32) * inv[None, :, None]).astype(np.float32)
    return e4m3_round(y), s


def fp8_flash_rows(q8, k8, v8, c, key_tiles=None, tile=128, p_scale=16.0, tau=4.0, return_m=False):
    """One head's flash-style pass over E4M3 operands (a reading; see below).

    q8 [R, d], k8 [T, d], v8 [T, d]: decoded E4M3 values (unscaled); c: the
    factor that turns q8 . k8 into log2 units of the softmax argument;
    key_tiles: the tiles of ``tile`` keys to visit, in order (default: all).
    Returns (acc, l) with O = acc / (p_scale * l) times the V decode scale;
    with ``return_m`` also the final reference maximum m, so that l * 2^m is
    the visited keys' softmax mass sum 2^t.

    Steps, per visited tile: t = (q8 . k8) * c for its keys; the row's
    reference maximum m (initially -inf) is moved to the tile maximum only
    when that exceeds m by more than ``tau``, and then acc and l are first
    multiplied by 2^(m_old - m_new); p = 2^(t - m), so p <= 2^tau;
    acc += e4m3(p * p_scale) . v8 and l += sum of the unrounded p.  Visiting
    keys a tile at a time with a running maximum is the flash-attention
    scheme; moving the maximum only past a threshold is the conditional
    rescale of the Blackwell flash-attention design (the normalisation is
    unchanged: rescaling by any common reference gives the same softmax).
    Its effect here is where P is rounded: with p_scale = 16 and tau = 4,
    p * p_scale <= 256 stays inside E4M3's range (448).
    """
    q8 = np.asarray(q8, np.float64)
    k8 = np.asarray(k8, np.float64)
    v8 = np.asarray(v8, np.float64)
    R, d = q8.shape
    T = k8.shape[0]
    if key_tiles is None:
        key_tiles = range(-(-T // tile))
    m = np.full(R, -np.inf)
    l = np.zeros(R)
    acc = np.zeros((R, v8.shape[1]))
    for j in key_tiles:
        j0 = j * tile
        t = (q8 @ k8[j0:j0 + tile].T) * c
        mx = t.max(axis=1)
        move = mx > m + tau
        alpha = np.where(move, np.exp2(np.where(move, m - mx, 0.0)), 1.0)
        acc *= alpha[:, None]
        l *= alpha
        m = np.where(move, mx, m)
        p = np.exp2(t - m[:, None])
        l += p.sum(axis=1)
        acc += e4m3_round(p * p_scale) @ v8[j0:j0 + tile]
    return (acc, l, m) if return_m else (acc, l)


def attention_fp8_emulated(q, k, v, tile=128, p_scale=16.0, tau=4.0, rows=None):
    """FP8 joint attention, flash-style (a reading; the pages name FP8 Q/K/V
    attention but not its arithmetic).

    Q, K and V are rounded to E4M3 after scaling each head by 448 / amax
    (``fp8_encode_heads``); the softmax argument in log2 units is
    t = (q8 . k8) * sq * sk * log2(e) / sqrt(d); ``fp8_flash_rows`` visits all
    key tiles in order; O = acc * s_v / (p_scale * l).  Everything else fp64.
    ``rows`` optionally restricts the query rows (scales still use all rows).
    """
    q8, sq = fp8_encode_heads(q)
    k8, sk = fp8_encode_heads(k)
    v8, sv = fp8_encode_heads(v)
    T, H, d = q8.shape
    if rows is not None:
        q8 = q8[np.asarray(rows)]
    R = q8.shape[0]
    out = np.empty((R, H, d), dtype=np.float64)
    for h in range(H):
        c = np.log2(np.e) / np.sqrt(d) * float(sq[h]) * float(sk[h])
        acc, l = fp8_flash_rows(q8[:, h, :], k8[:, h, :], v8[:, h, :], c, tile=tile, p_scale=p_scale, tau=tau)
        out[:, h, :] = acc * float(sv[h]) / (p_scale * l[:, None])
    return out


# ---------------------------------------------------------------------------
# The joint block
# ---------------------------------------------------------------------------
def silu(g):
    g = np.asarray(g, np.float64)
    return g / (1.0 + np.exp(-g))


def block_forward(x, mod, weights, layout, n_heads, attn="exact", keep=False):
    """Forward pass of one joint transformer block.

    x        : [T, D] bf16 values (as float32)
    mod      : dict with bf16 vectors shift1, scale1, gate1, shift2, scale2, gate2 [D]
    weights  : dict with bf16 matrices wqkv [3D, D], wo [D, D], w1 [2F, D], w2 [D, F]
               (each NVFP4-encoded here with its own global scale), or already
               encoded (codes, scales, gs) triples
    layout   : TokenLayout (T must equal layout.n_tokens)
    attn     : "exact" (fp64 attention on the bf16 q, k, v) or "fp8"
               (``attention_fp8_emulated``, a diagnostic)

    Returns the bf16 block output [T, D] (float32), and with ``keep`` a dict of
    intermediates.
    """
    x = np.asarray(x, np.float32)
    T, D = x.shape
    if T != layout.n_tokens:
        raise ValueError("x rows do not match the token layout")
    H = n_heads
    d = D // H
    if d != HEAD_DIM:
        raise ValueError("head dim must be 128")

    def enc(w):
        return w if isinstance(w, tuple) else nvfp4.quantize(w)

    wqkv, wo, w1, w2 = (enc(weights[n]) for n in ("wqkv", "wo", "w1", "w2"))
    F = w2[0].shape[1] * 2

    # branch 1: attention
    m1 = modulate(x, mod["shift1"], mod["scale1"])
    a1 = nvfp4.quantize(m1)
    qkv = gemm_nvfp4(a1, wqkv)
    phi = rope_angles(layout)
    q = apply_rope(qkv[:, 0:D].reshape(T, H, d), phi)
    k = apply_rope(qkv[:, D : 2 * D].reshape(T, H, d), phi)
    v = qkv[:, 2 * D : 3 * D].reshape(T, H, d)
    q, k, v = bf16_round(q), bf16_round(k), bf16_round(v)
    if attn == "exact":
        o, _ = attention(q, k, v)
    elif attn == "fp8":
        o = attention_fp8_emulated(q, k, v)
    else:
        raise ValueError("attn must be 'exact' or 'fp8'")
    o = bf16_round(o.reshape(T, D))
    oq = nvfp4.quantize(o)
    x1 = bf16_round(x + np.asarray(mod["gate1"], np.float64) * gemm_nvfp4(oq, wo))

    # branch 2: SwiGLU MLP
    m2 = modulate(x1, mod["shift2"], mod["scale2"])
    a2 = nvfp4.quantize(m2)
    gu = gemm_nvfp4(a2, w1)
    h = bf16_round(silu(gu[:, :F]) * gu[:, F:])
    hq = nvfp4.quantize(h)
    out = bf16_round(x1 + np.asarray(mod["gate2"], np.float64) * gemm_nvfp4(hq, w2))
    if not keep:
        return out
    inter = dict(m1=m1, a1=a1, q=q, k=k, v=v, o=o, x1=x1, m2=m2, a2=a2, h=h, out=out)
    return out, inter
