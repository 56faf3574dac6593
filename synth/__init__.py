"""Seeded synthetic inputs shared by the oracle and the CUDA path.

This package holds shapes and random draws only -- none of the block's
arithmetic (no quantisation, normalisation, RoPE, attention or GEMM).  Both
``oracle`` and the tests/bench feed the CUDA library from the same tensors made
here, so the two sides see identical bytes.

Workloads (token counts from [P4] "Welcome FLUX.3 Image Klein in Diffusers",
§The VAE and Tokenization -- 8x VAE, 2x2 patches, 1024x1024 -> 64x64 = 4,096
tokens -- and [P2] "FLUX.3 Image Klein Brings 2-Second AI Image Generation to
Diffusers", §Summary -- each 1024x1024 reference adds 4,096 tokens; hidden
width 3072 from [P4] §The Qwen3-VL Text Encoder):

=============  ======  ======  ====  ===  =====  =====  =========
name           text    grid    refs  D    heads  F      attention
=============  ======  ======  ====  ===  =====  =====  =========
micro          16      4x4     1     128  1      384    bf16
tiny           64      16x16   0     512  4      1536   bf16
t2i_1024       512     64x64   0     3072 24     9216   fp8
i2i_1024       512     64x64   1     3072 24     9216   fp8
multiref_1024  512     64x64   4     3072 24     9216   fp8
multiref_21504 1024    64x64   4     3072 24     9216   fp8
=============  ======  ======  ====  ===  =====  =====  =========

Draw recipe (fixed order, one ``torch.Generator`` seeded per workload, every
tensor ``randn`` in fp32 then cast to bf16 with round-to-nearest-even):
x ~ N(0, 1) [T, D]; shift1, scale1, gate1, shift2, scale2, gate2 ~ N(0, 0.1)
[D]; Wqkv [3D, D], Wo [D, D], W1 [2F, D], W2 [D, F] ~ N(0, 0.02).
"""

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    n_text: int
    grid_h: int
    grid_w: int
    n_ref: int
    hidden: int
    heads: int
    mlp_hidden: int
    attn: str          # "bf16" or "fp8"
    seed: int

    @property
    def n_tokens(self):
        return self.n_text + (1 + self.n_ref) * self.grid_h * self.grid_w


WORKLOADS = {
    w.name: w
    for w in [
        Workload("micro", 16, 4, 4, 1, 128, 1, 384, "bf16", 7),
        Workload("tiny", 64, 16, 16, 0, 512, 4, 1536, "bf16", 0),
        Workload("t2i_1024", 512, 64, 64, 0, 3072, 24, 9216, "fp8", 1),
        Workload("i2i_1024", 512, 64, 64, 1, 3072, 24, 9216, "fp8", 2),
        Workload("multiref_1024", 512, 64, 64, 4, 3072, 24, 9216, "fp8", 4),
        Workload("multiref_21504", 1024, 64, 64, 4, 3072, 24, 9216, "fp8", 4),
    ]
}

MOD_NAMES = ("shift1", "scale1", "gate1", "shift2", "scale2", "gate2")


def _randn(gen, shape, std):
    return (torch.randn(*shape, generator=gen, dtype=torch.float32) * std).to(torch.bfloat16)


def block_inputs(wl, with_weights=True):
    """All seeded inputs of one joint-block call, as bf16 CPU tensors."""
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    g = torch.Generator().manual_seed(wl.seed)
    T, D, F = wl.n_tokens, wl.hidden, wl.mlp_hidden
    out = {"x": _randn(g, (T, D), 1.0)}
    for n in MOD_NAMES:
        out[n] = _randn(g, (D,), 0.1)
    if with_weights:
        out["wqkv"] = _randn(g, (3 * D, D), 0.02)
        out["wo"] = _randn(g, (D, D), 0.02)
        out["w1"] = _randn(g, (2 * F, D), 0.02)
        out["w2"] = _randn(g, (D, F), 0.02)
    return out


def normal_bf16(shape, seed, std=1.0):
    """A seeded N(0, std^2) bf16 tensor (used for standalone kernel tests)."""
    g = torch.Generator().manual_seed(seed)
    return _randn(g, shape, std)


def uniform_int(shape, low, high, seed):
    """Seeded integers in [low, high) as an int64 tensor."""
    g = torch.Generator().manual_seed(seed)
    return torch.randint(low, high, shape, generator=g, dtype=torch.int64)


# ------------------------------------------------------------- DiT loop
@dataclass(frozen=True)
class DitConfig:
    """A synthetic DiT: latent [2*grid_h, 2*grid_w, channels] (2x2 patches ->
    grid_h x grid_w image tokens of 4*channels features), n_text text tokens,
    n_mode per-mode blocks then n_joint joint blocks, n_steps Euler steps."""

    name: str
    n_text: int
    grid_h: int
    grid_w: int
    channels: int
    hidden: int
    heads: int
    mlp_hidden: int
    n_mode: int
    n_joint: int
    n_steps: int
    attn: str
    seed: int


# c4: a 1024x1024 image -> 128x128x32 latent -> 64x64 tokens of 128 features,
# 512 text tokens, 5 per-mode + 28 joint blocks, 16 steps; seed 3 (config
# index - 1).  dit_tiny: the same structure at block-test sizes.  dit_wide:
# the c4 widths (3072 hidden, 24 heads, 9216 MLP, 32 latent channels, FP8
# attention) on a 256x256 image (16x16 tokens) and 64 text tokens, one
# per-mode and two joint blocks, for parity at full width.
DIT_CONFIGS = {
    c.name: c
    for c in [
        DitConfig("dit_tiny", 16, 4, 4, 32, 128, 1, 384, 1, 2, 2, "bf16", 11),
        DitConfig("dit_t2i_1024", 512, 64, 64, 32, 3072, 24, 9216, 5, 28, 16, "fp8", 3),
        DitConfig("dit_wide", 64, 16, 16, 32, 3072, 24, 9216, 1, 2, 1, "fp8", 12),
    ]
}


def dit_inputs(cfg, with_weights=True, device="cpu", mods="independent"):
    """Seeded inputs of a DiT run as CPU tensors.  Draw order: latent (fp32
    N(0,1)); text (bf16 N(0,1)); w_in [D, 4C], w_out [4C, D] (N(0,0.02));
    per-mode blocks i = 0..n_mode-1: text weights then image weights (each
    Wqkv, Wo, W1, W2 as in block_inputs); joint blocks; modulation vectors
    (N(0,0.1)): mode [n_mode, 2, 6, D], joint [n_joint, 6, D], final [2, D].
    ``mods="independent"``: drawn afresh for each of the n_steps steps
    ([n_steps, ...]); ``mods="smooth"``: two such sets m0 then m1 are drawn and
    step i takes bf16(m0 + t_i m1) with t_i = 1 - i / n_steps, a stand-in for
    modulations that a timestep embedding makes a smooth function of t.
    ``device``: where the generator and tensors live (a CUDA generator draws
    different numbers than the CPU one; the parity tests use the CPU draws)."""
    if isinstance(cfg, str):
        cfg = DIT_CONFIGS[cfg]
    g = torch.Generator(device=device).manual_seed(cfg.seed)
    D, F, C = cfg.hidden, cfg.mlp_hidden, cfg.channels

    def _randn(gen, shape, std):
        return (torch.randn(*shape, generator=gen, dtype=torch.float32, device=device) * std).to(torch.bfloat16)

    out = {"latent": torch.randn(2 * cfg.grid_h, 2 * cfg.grid_w, C, generator=g, dtype=torch.float32,
                                 device=device),
           "text": _randn(g, (cfg.n_text, D), 1.0)}

    def block_w():
        return {"wqkv": _randn(g, (3 * D, D), 0.02), "wo": _randn(g, (D, D), 0.02),
                "w1": _randn(g, (2 * F, D), 0.02), "w2": _randn(g, (D, F), 0.02)}

    if with_weights:
        out["w_in"] = _randn(g, (D, 4 * C), 0.02)
        out["w_out"] = _randn(g, (4 * C, D), 0.02)
        out["mode_text"], out["mode_image"] = [], []
        for _ in range(cfg.n_mode):
            out["mode_text"].append(block_w())
            out["mode_image"].append(block_w())
        out["joint"] = [block_w() for _ in range(cfg.n_joint)]
    shapes = {"mod_mode": (cfg.n_mode, 2, 6, D), "mod_joint": (cfg.n_joint, 6, D), "mod_final": (2, D)}
    if mods == "independent":
        for k, sh in shapes.items():
            out[k] = _randn(g, (cfg.n_steps,) + sh, 0.1)
    elif mods == "smooth":
        m0 = {k: _randn(g, sh, 0.1).float() for k, sh in shapes.items()}
        m1 = {k: _randn(g, sh, 0.1).float() for k, sh in shapes.items()}
        t = [1.0 - i / cfg.n_steps for i in range(cfg.n_steps)]
        for k in shapes:
            out[k] = torch.stack([m0[k] + ti * m1[k] for ti in t]).to(torch.bfloat16)
    else:
        raise ValueError("mods must be 'independent' or 'smooth'")
    return out


def sparse_attention_qkv(T, H, seed, lean=8.0, spread=2.0):
    """bf16 [T, 3*H*128] q | k | v with tile structure, for attention tile
    skipping: per head a random unit direction u; q = N(0, 0.25) + lean * u;
    the keys of 128-key tile j = N(0, 0.25) + a_j * u with a_j ~ U(-spread,
    spread) (one draw per head and tile); v ~ N(0, 1).  Draw order: u, q noise,
    a, k noise, v (torch CPU generator)."""
    g = torch.Generator().manual_seed(seed)
    D = H * 128
    u = torch.randn(H, 128, generator=g, dtype=torch.float64)
    u /= u.norm(dim=1, keepdim=True)
    q = 0.5 * torch.randn(T, H, 128, generator=g, dtype=torch.float64) + lean * u
    nkt = -(-T // 128)
    a = (torch.rand(nkt, H, generator=g, dtype=torch.float64) * 2 - 1) * spread
    a_rows = a.repeat_interleave(128, dim=0)[:T]
    k = 0.5 * torch.randn(T, H, 128, generator=g, dtype=torch.float64) + a_rows[:, :, None] * u
    v = torch.randn(T, H, 128, generator=g, dtype=torch.float64)
    return torch.cat([q.reshape(T, D), k.reshape(T, D), v.reshape(T, D)], dim=1).to(torch.bfloat16)
