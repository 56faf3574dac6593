"""kl_dit_step (one Euler step of the synthetic DiT on the block kernels) vs
the oracle's fp64 DiT step, on the tiny DiT configuration."""

import numpy as np
import pytest
import torch

import diffusion_transformer_image_nvfp4_b200 as kl
from oracle import block, dit, nvfp4
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


MOD6 = ("shift1", "scale1", "gate1", "shift2", "scale2", "gate2")


def test_full_width_fp8_dit_step_stage_by_stage():
    # The DiT step at the 1024^2 loop's widths (3072 hidden, 24 heads, 9216
    # MLP, 128 -> 3072 input projection, FP8 attention) on 64 text and 16x16
    # image tokens: one per-mode pair and two joint blocks.  Its final
    # velocity goes through an E2M1 encode of a LayerNorm, which turns any
    # upstream difference into whole-code flips, and the image tokens are
    # small (the projected patches) next to each block's branch, so a whole-
    # sequence comparison mostly measures the NVFP4 branch noise the block
    # tests bound stage by stage.  What the step adds to the blocks is checked
    # exactly instead:
    cfg = DIT_CONFIGS["dit_wide"]
    d = dit_inputs(cfg)
    W, shape, ropes = _gpu(cfg, d)
    mm, mj, mf = (d[k][0].cuda().contiguous() for k in ("mod_mode", "mod_joint", "mod_final"))
    text_d = d["text"].cuda()
    lat = d["latent"].cuda().contiguous()
    before = to_np(lat).copy()
    dt = -1.0 / 16
    text, w, mods, sh = _oracle_args(cfg, d, 0)
    Ti, D, nt = cfg.grid_h * cfg.grid_w, cfg.hidden, cfg.n_text
    # 0. the embedding (a step with no block leaves it as the head's input):
    #    patches -> NVFP4 -> input projection, the text in front; one bf16 ulp
    #    plus fp32 accumulation noise against the oracle
    shape0 = kl.DitShape(cfg.n_text, cfg.grid_h, cfg.grid_w, cfg.channels, D, cfg.heads, cfg.mlp_hidden, 0, 0,
                         cfg.attn)
    W0 = kl.DitWeights(W.w_in, [], [], [], W.w_out)
    ws0 = torch.empty(kl.dit_workspace_size(shape0), dtype=torch.uint8, device="cuda")
    kl.dit_step(shape0, W0, lat.clone(), text_d, None, None, mf, *ropes, dt, workspace=ws0)
    x0 = kl.dit_views(shape0, ws0)["tokens"].clone()
    torch.cuda.synchronize()
    ref0 = dit.stack_tokens(before, text, {**w, "mode_text": [], "mode_image": [], "joint": []}, mods, sh)
    e0 = to_np(x0)
    assert np.array_equal(e0[:nt], ref0[:nt])
    dd = np.abs(e0[nt:] - ref0[nt:])
    assert np.all(dd <= np.abs(ref0[nt:]) * 2.0 ** -7 + 1e-5 * np.abs(ref0[nt:]).max())
    assert np.mean(dd == 0) >= 0.99
    # 1. the stack is the library's joint block applied as the readings say:
    #    per-mode blocks on the text rows and on the image rows alone (own
    #    weights, modulation and RoPE layout), then joint blocks on all rows;
    #    replayed with kl_joint_block_forward, bit for bit
    ws = torch.empty(kl.dit_workspace_size(shape), dtype=torch.uint8, device="cuda")
    kl.dit_step(shape, W, lat, text_d, mm, mj, mf, *ropes, dt, workspace=ws)
    torch.cuda.synchronize()
    assert kl.device_status() == "KL_OK"
    views = kl.dit_views(shape, ws)
    md = lambda v6: {n: v6[i] for i, n in enumerate(MOD6)}
    t = x0
    for i in range(cfg.n_mode):
        tt = kl.joint_block_forward(W.mode_text[i], t[:nt].contiguous(), md(mm[i, 0]), ropes[0], cfg.heads,
                                    cfg.mlp_hidden, cfg.attn).clone()
        ti = kl.joint_block_forward(W.mode_image[i], t[nt:].contiguous(), md(mm[i, 1]), ropes[1], cfg.heads,
                                    cfg.mlp_hidden, cfg.attn).clone()
        t = torch.cat([tt, ti])
    for j in range(cfg.n_joint):
        t = kl.joint_block_forward(W.joint[j], t.contiguous(), md(mj[j]), ropes[2], cfg.heads, cfg.mlp_hidden,
                                   cfg.attn).clone()
    torch.cuda.synchronize()
    assert torch.equal(views["tokens"], t)
    tok = to_np(views["tokens"])
    for attn in ("fp8", "exact"):  # reported: the NVFP4 branch noise of three blocks, see above
        ref = dit.stack_tokens(before, text, w, mods, sh, attn=attn)
        print(f"dit_wide tokens vs oracle ({attn}): {rel_l2(tok, ref):.3e} "
              f"(text rows {rel_l2(tok[:nt], ref[:nt]):.3e}, image rows {rel_l2(tok[nt:], ref[nt:]):.3e})")
    # 2. the head's NVFP4 operand against the oracle's encode of its LN +
    #    adaLN of the GPU's tokens: m may differ by one bf16 ulp where the
    #    fp32 statistics round differently, so nearly all codes and scales
    #    agree and the global scale agrees to one bf16 rounding
    codes, scales, gs = nvfp4.quantize(dit.head_input(tok, mods, sh))
    g_codes = to_np(views["head_codes"])
    g_scales = to_np(kl.scales_mma_to_linear(views["head_scales"], Ti, D))
    g_gs = np.float32(to_np(views["head_gs"])[0])
    assert np.mean(g_codes == codes) >= 0.99
    assert np.mean(g_scales == scales) >= 0.99
    assert abs(float(g_gs) / float(gs) - 1.0) <= 2.0 ** -7
    # 3. the output projection of the GPU's operand: fp32 accumulation
    v = to_np(views["velocity"])
    v_ref = block.gemm_nvfp4((g_codes, g_scales, g_gs), nvfp4.quantize(w["w_out"]))
    assert rel_l2(v, v_ref) <= 1e-5
    # 4. the Euler update of the latent with that velocity: bit-exact
    np.testing.assert_array_equal(to_np(lat), dit.euler(before, v, dt, cfg.grid_h, cfg.grid_w, cfg.channels))
