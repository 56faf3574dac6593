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


def velocity(latent, text, weights, mods, shape, attn="exact"):
    """The velocity per patch [gh*gw, 4C] (fp64) of one DiT evaluation.

    weights: dict w_in [D, 4C], w_out [4C, D] (bf16 values), mode_text,
    mode_image, joint (lists of block weight dicts, see block_forward);
    mods: dict mode [n_mode, 2, 6, D], joint [n_joint, 6, D], final [2, D]
    (bf16 values, kl_block_io order shift1, scale1, gate1, shift2, scale2,
    gate2); shape: dict n_text, grid_h, grid_w, channels, H.
    """
    nt, gh, gw, H = shape["n_text"], shape["grid_h"], shape["grid_w"], shape["H"]
    p = bf16_round(patchify(np.asarray(latent, np.float64)))
    img = bf16_round(gemm_nvfp4(nvfp4.quantize(p), nvfp4.quantize(weights["w_in"])))
    tok = np.concatenate([np.asarray(text, np.float64), img]).astype(np.float32)
    lay_t, lay_i, lay_j = TokenLayout(nt, 0, 0, 0), TokenLayout(0, gh, gw, 0), TokenLayout(nt, gh, gw, 0)

    def mod_dict(v6):
        return {n: v6[i] for i, n in enumerate(MOD_ORDER)}

    for i in range(len(weights["mode_text"])):
        t_out = block_forward(tok[:nt], mod_dict(mods["mode"][i][0]), weights["mode_text"][i], lay_t, H, attn)
        i_out = block_forward(tok[nt:], mod_dict(mods["mode"][i][1]), weights["mode_image"][i], lay_i, H, attn)
        tok = np.concatenate([t_out, i_out]).astype(np.float32)
    for i in range(len(weights["joint"])):
        tok = block_forward(tok, mod_dict(mods["joint"][i]), weights["joint"][i], lay_j, H, attn)
    m = modulate(tok[nt:], mods["final"][0], mods["final"][1])
    return gemm_nvfp4(nvfp4.quantize(m), nvfp4.quantize(weights["w_out"]))


def dit_step(latent, text, weights, mods, shape, dt, attn="exact"):
    """latent after one Euler step (fp32 [2gh, 2gw, C])."""
    v = velocity(latent, text, weights, mods, shape, attn)
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
