"""kl_dit_step (one Euler step of the synthetic DiT on the block kernels) vs
the oracle's fp64 DiT step, on the tiny DiT configuration."""

import numpy as np
import pytest
import torch

import diffusion_transformer_image_nvfp4_b200 as kl
from oracle import dit
from synth import DIT_CONFIGS, dit_inputs
from tests.helpers import rel_l2, to_np

pytestmark = pytest.mark.gpu


def _gpu(cfg, d, zero_out=False):
    c = lambda t: t.cuda()
    w_out = d["w_out"] * (0 if zero_out else 1)
    blocks = lambda bl: [kl.prepare_block_weights(c(b["wqkv"]), c(b["wo"]), c(b["w1"]), c(b["w2"])) for b in bl]
    W = kl.DitWeights(kl.quantize_nvfp4(c(d["w_in"])), blocks(d["mode_text"]), blocks(d["mode_image"]),
                      blocks(d["joint"]), kl.quantize_nvfp4(c(w_out)))
    shape = kl.DitShape(cfg.n_text, cfg.grid_h, cfg.grid_w, cfg.channels, cfg.hidden, cfg.heads, cfg.mlp_hidden,
                        cfg.n_mode, cfg.n_joint, cfg.attn)
    ropes = (kl.rope_table(cfg.n_text, 0, 0), kl.rope_table(0, cfg.grid_h, cfg.grid_w),
             kl.rope_table(cfg.n_text, cfg.grid_h, cfg.grid_w))
    return W, shape, ropes


def _oracle_args(cfg, d, step, zero_out=False):
    f = lambda t: t.float().numpy()
    w = {"w_in": f(d["w_in"]), "w_out": f(d["w_out"]) * (0.0 if zero_out else 1.0),
         "mode_text": [{k: f(v) for k, v in b.items()} for b in d["mode_text"]],
         "mode_image": [{k: f(v) for k, v in b.items()} for b in d["mode_image"]],
         "joint": [{k: f(v) for k, v in b.items()} for b in d["joint"]]}
    mods = {"mode": f(d["mod_mode"][step]), "joint": f(d["mod_joint"][step]), "final": f(d["mod_final"][step])}
    shape = {"n_text": cfg.n_text, "grid_h": cfg.grid_h, "grid_w": cfg.grid_w, "channels": cfg.channels,
             "H": cfg.heads}
    return f(d["text"]), w, mods, shape


def _step(cfg, d, W, shape, ropes, lat, step, dt):
    kl.dit_step(shape, W, lat, d["text"].cuda(), d["mod_mode"][step].cuda().contiguous(),
                d["mod_joint"][step].cuda().contiguous(), d["mod_final"][step].cuda().contiguous(), *ropes, dt)


def test_dit_steps_match_oracle():
    cfg = DIT_CONFIGS["dit_tiny"]
    d = dit_inputs(cfg)
    W, shape, ropes = _gpu(cfg, d)
    ts = dit.timesteps(16)
    lat = d["latent"].cuda().contiguous()
    ref = d["latent"].numpy()
    for step in range(cfg.n_steps):
        dt = ts[step + 1] - ts[step]
        before_gpu, before_ref = to_np(lat).copy(), ref.copy()
        _step(cfg, d, W, shape, ropes, lat, step, dt)
        text, w, mods, sh = _oracle_args(cfg, d, step)
        # the velocity of this step, both sides from the same (GPU) latent
        v_ref = dit.velocity(before_gpu, text, w, mods, sh)
        v_gpu = (to_np(lat).astype(np.float64) - before_gpu) / dt
        err = rel_l2(v_gpu, dit.unpatchify(v_ref, cfg.grid_h, cfg.grid_w, cfg.channels))
        # three blocks at <= 1e-2 each (BF16 attention) plus the NVFP4 input
        # and output projections
        assert err <= 3e-2, err
        ref = dit.dit_step(before_ref, text, w, mods, sh, dt)
    # the two trajectories after the steps (oracle on its own latents)
    assert rel_l2(to_np(lat) - d["latent"].numpy(), ref - d["latent"].numpy()) <= 3e-2


def test_zero_output_projection_leaves_the_latent_bit_identical():
    cfg = DIT_CONFIGS["dit_tiny"]
    d = dit_inputs(cfg)
    W, shape, ropes = _gpu(cfg, d, zero_out=True)
    lat = d["latent"].cuda().contiguous()
    _step(cfg, d, W, shape, ropes, lat, 0, -1 / 16)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_np(lat), d["latent"].numpy())
    assert kl.device_status() == "KL_OK"


def test_dit_step_rejects_bad_shapes():
    cfg = DIT_CONFIGS["dit_tiny"]
    bad = kl.DitShape(cfg.n_text, cfg.grid_h, cfg.grid_w, 20, cfg.hidden, cfg.heads, cfg.mlp_hidden, 1, 2, "bf16")
    assert kl.dit_workspace_size(bad) == 0  # 4*channels not a multiple of 128
