"""One Euler step of the synthetic DiT, plain fp64 reading (TEST
INFRASTRUCTURE ONLY: imported by tests/, never by the library).

What the pages fix: [P2] "FLUX.3 Image Klein Brings 2-Second AI Image
Generation to Diffusers", Summary -- each stream first goes through its own
(per-mode) blocks, then the concatenated sequence through joint blocks;
[P4] "Welcome FLUX.3 Image Klein in Diffusers", The VAE and Tokenization --
2x2 patches of the latent become the image tokens; Two-Stage Processing.
Flow matching integrates the velocity from noise (t = 1) to the image (t = 0)
in Euler steps.

Readings (the pages stop at the block structure; the same readings as the
library's kl_dit_step):
* patch features p[t][k] = latent[y][x][c] with t = (y//2)*gw + x//2 and
  k = 4c + 2(y%2) + (x%2), rounded to bf16; no bias, no norm;
* image tokens = bf16(NVFP4(p) . NVFP4(w_in)^T); the text conditioning
  [n_text, D] is placed in front of them every step;
* per-mode block i = the joint block applied to the text rows alone (text
  RoPE layout) and to the image rows alone (image layout), each with its own
  weights and modulation;
* joint block i on [text; image];
* v = NVFP4(bf16(LN(image rows)(1 + scale_f) + shift_f)) . NVFP4(w_out)^T;
* Euler: latent <- fl32(latent + fl32(dt * fl32(v))) (the library keeps the
  latent and v in fp32).
"""

import numpy as np

from . import nvfp4
from .block import TokenLayout, block_forward, gemm_nvfp4, modulate
from .codecs import bf16_round

MOD_ORDER = ("shift1", "scale1", "gate1", "shift2", "scale2", "gate2")


def patchify(latent):
    """[2gh, 2gw, C] -> [gh*gw, 4C] (t = ty*gw + tx, k = 4c + 2dy + dx)."""
    h2, w2, c = latent.shape
    gh, gw = h2 // 2, w2 // 2
    p = np.asarray(latent).reshape(gh, 2, gw, 2, c)  # [ty, dy, tx, dx, c]
    return p.transpose(0, 2, 4, 1, 3).reshape(gh * gw, 4 * c)


def unpatchify(v, gh, gw, c):
    """Inverse of patchify: [gh*gw, 4C] -> [2gh, 2gw, C]."""
    p = np.asarray(v).reshape(gh, gw, c, 2, 2)  # [ty, tx, c, dy, dx]
    return p.transpose(0, 3, 1, 4, 2).reshape(2 * gh, 2 * gw, c)


def euler(latent, v_patches, dt, gh, gw, c):
    """latent + dt * v in fp32, one rounding per operation."""
    lat = np.asarray(latent, np.float32)
    v = unpatchify(np.asarray(v_patches, np.float32), gh, gw, c)
    return (lat + (np.float32(dt) * v).astype(np.float32)).astype(np.float32)


def _embed(latent, text, weights, shape):
    """[text; image tokens] (bf16 values, float32 [T, D])."""
    p = bf16_round(patchify(np.asarray(latent, np.float64)))
    img = bf16_round(gemm_nvfp4(nvfp4.quantize(p), nvfp4.quantize(weights["w_in"])))
    return np.concatenate([np.asarray(text, np.float64), img]).astype(np.float32)


def _n_blocks(weights):
    return len(weights["mode_text"]) + len(weights["joint"])


def _block(tok, i, weights, mods, shape, attn):
    """Block i of the stack (per-mode blocks first, then the joint blocks)."""
    nt, gh, gw, H = shape["n_text"], shape["grid_h"], shape["grid_w"], shape["H"]

    def mod_dict(v6):
        return {n: v6[j] for j, n in enumerate(MOD_ORDER)}

    n_mode = len(weights["mode_text"])
    if i < n_mode:
        lay_t, lay_i = TokenLayout(nt, 0, 0, 0), TokenLayout(0, gh, gw, 0)
        t_out = block_forward(tok[:nt], mod_dict(mods["mode"][i][0]), weights["mode_text"][i], lay_t, H, attn)
        i_out = block_forward(tok[nt:], mod_dict(mods["mode"][i][1]), weights["mode_image"][i], lay_i, H, attn)
        return np.concatenate([t_out, i_out]).astype(np.float32)
    j = i - n_mode
    return block_forward(tok, mod_dict(mods["joint"][j]), weights["joint"][j], TokenLayout(nt, gh, gw, 0), H, attn)


def _head(tok, weights, mods, shape):
    """Final LN + adaLN of the image rows, NVFP4, output projection (fp64)."""
    return gemm_nvfp4(nvfp4.quantize(head_input(tok, mods, shape)), nvfp4.quantize(weights["w_out"]))


def velocity(latent, text, weights, mods, shape, attn="exact"):
    """The velocity per patch [gh*gw, 4C] (fp64) of one DiT evaluation.

    weights: dict w_in [D, 4C], w_out [4C, D] (bf16 values), mode_text,
    mode_image, joint (lists of block weight dicts, see block_forward);
    mods: dict mode [n_mode, 2, 6, D], joint [n_joint, 6, D], final [2, D]
    (bf16 values, kl_block_io order shift1, scale1, gate1, shift2, scale2,
    gate2); shape: dict n_text, grid_h, grid_w, channels, H.
    """
    return _head(stack_tokens(latent, text, weights, mods, shape, attn), weights, mods, shape)


def stack_tokens(latent, text, weights, mods, shape, attn="exact"):
    """The token sequence [T, D] (bf16 values) after the last block of the
    stack: the head's input (arguments as for ``velocity``)."""
    tok = _embed(latent, text, weights, shape)
    for i in range(_n_blocks(weights)):
        tok = _block(tok, i, weights, mods, shape, attn)
    return tok


def head_input(tok, mods, shape):
    """bf16(LN(image rows)(1 + scale_f) + shift_f): what the head encodes to
    NVFP4 before the output projection."""
    return modulate(np.asarray(tok)[shape["n_text"]:], mods["final"][0], mods["final"][1])


# ---------------------------------------------------------------- Cache-DiT
# [P1] "Optimizing FLUX 3 Image Klein inference on NVIDIA Blackwell GPUs", How
# it works: Cache-DiT watches a residual difference between denoising steps
# and, while it stays under a threshold, reuses cached transformer outputs in
# place of recomputing them (What you can do: residual_diff_threshold 0.24).
# The pages name no more than that; the readings here:
# * the probe is the first block of the stack (the first per-mode pair, or the
#   first joint block when there are none); it runs every step, and its
#   residual is r = probe output - probe input over all [T, D] entries;
# * the residual difference is the relative L1 change
#   sum |r - r_ref| / sum |r_ref| against r_ref, the probe residual of the
#   last step that ran every block (so slow drift accumulates until it forces
#   a recompute); 0/0 reads as 0 and x/0 (x > 0) as +inf;
# * a step with no reference yet (the first of a generation) runs every block;
# * a step that runs every block stores R = final tokens - probe output and
#   makes r its reference; a step with diff < threshold skips the remaining
#   blocks and takes final tokens = bf16(probe output + R).


def residual_diff(r, r_ref):
    """Relative L1 change of the probe residual: sum|r - r_ref| / sum|r_ref|."""
    num = float(np.abs(np.asarray(r, np.float64) - np.asarray(r_ref, np.float64)).sum())
    den = float(np.abs(np.asarray(r_ref, np.float64)).sum())
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return num / den


def velocity_cached(latent, text, weights, mods, shape, cache, threshold, attn="exact"):
    """velocity() with Cache-DiT step caching.  ``cache`` is a dict, empty at
    the first step of a generation, updated in place: r_ref, R (fp64 [T, D]),
    and for the step just taken diff (+inf without a reference), hit (bool)
    and hits (count over the generation)."""
    if _n_blocks(weights) < 1:
        raise ValueError("step caching needs at least one block")
    tok = _embed(latent, text, weights, shape)
    f = _block(tok, 0, weights, mods, shape, attn)
    r = f.astype(np.float64) - tok.astype(np.float64)
    has_ref = "r_ref" in cache
    diff = residual_diff(r, cache["r_ref"]) if has_ref else float("inf")
    hit = has_ref and diff < threshold
    if hit:
        final = bf16_round(f.astype(np.float64) + cache["R"])
    else:
        final = f
        for i in range(1, _n_blocks(weights)):
            final = _block(final, i, weights, mods, shape, attn)
        cache["R"] = final.astype(np.float64) - f.astype(np.float64)
        cache["r_ref"] = r
    cache["diff"], cache["hit"] = diff, hit
    cache["hits"] = cache.get("hits", 0) + int(hit)
    return _head(final, weights, mods, shape)


def dit_step(latent, text, weights, mods, shape, dt, attn="exact", cache=None, threshold=0.0):
    """latent after one Euler step (fp32 [2gh, 2gw, C]); with a ``cache``
    dict, the Cache-DiT step (velocity_cached) at ``threshold``."""
    if cache is None:
        v = velocity(latent, text, weights, mods, shape, attn)
    else:
        v = velocity_cached(latent, text, weights, mods, shape, cache, threshold, attn)
    return euler(latent, v, dt, shape["grid_h"], shape["grid_w"], shape["channels"])


def timesteps(n_steps, shift=1.0):
    """Flow-matching timesteps from t = 1 (noise) to t = 0: t_i = 1 - i/n,
    mapped by the time shift s * t / (1 + (s - 1) * t) (s = 1: linear).  The
    shift keeps the endpoints, is monotone and spends more steps at high
    noise for s > 1 (the pages name a shift of 6.93 for the distilled
    schedule: "black-forest-labs/flux-3-image-klein", Behavior and
    constraints)."""
    out = []
    for i in range(n_steps + 1):
        t = 1.0 - i / n_steps
        out.append(shift * t / (1.0 + (shift - 1.0) * t))
    return out
