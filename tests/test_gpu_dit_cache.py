"""kl_dit_step_cached (Cache-DiT step caching) against kl_dit_step, its own
device residuals and the oracle's cached step, eager and under CUDA graph
capture (where the skip is a conditional graph node), on the tiny DiT."""

import numpy as np
import pytest
import torch

import diffusion_transformer_image_nvfp4_b200 as kl
from oracle import dit
from synth import DIT_CONFIGS, dit_inputs
from tests.helpers import rel_l2, to_np
from tests.test_gpu_dit import _gpu, _oracle_args

pytestmark = pytest.mark.gpu

CFG = DIT_CONFIGS["dit_tiny"]


def _io(d, step):
    return (d["text"].cuda(), d["mod_mode"][step].cuda().contiguous(), d["mod_joint"][step].cuda().contiguous(),
            d["mod_final"][step].cuda().contiguous())


def _setup():
    d = dit_inputs(CFG)
    W, shape, ropes = _gpu(CFG, d)
    io = [_io(d, s) for s in range(CFG.n_steps)]
    return d, W, shape, ropes, io


def _cached(shape, W, cache, thr, lat, io_s, ropes, dt):
    kl.dit_step_cached(shape, W, cache, thr, lat, *io_s, *ropes, dt)


def test_threshold_zero_is_bit_identical_to_the_plain_step():
    d, W, shape, ropes, io = _setup()
    cache = kl.DitCache(shape)
    a = d["latent"].cuda().contiguous()
    b = a.clone()
    for step in range(CFG.n_steps):
        kl.dit_step(shape, W, a, *io[step], *ropes, -1 / 16)
        _cached(shape, W, cache, 0.0, b, io[step], ropes, -1 / 16)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(to_np(b), to_np(a))
        h = cache.header()
        assert h["hit"] == 0 and h["steps"] == step + 1
    assert cache.header()["hits"] == 0
    assert kl.device_status() == "KL_OK"


def test_repeated_input_hits_with_zero_change_and_reproduces_the_step():
    d, W, shape, ropes, io = _setup()
    cache = kl.DitCache(shape)
    x0 = d["latent"].cuda().contiguous()
    a = x0.clone()
    _cached(shape, W, cache, 1e-6, a, io[0], ropes, -1 / 16)
    h = cache.header()
    assert h["hit"] == 0 and h["has_ref"] == 1 and h["diff"] == float("inf")
    b = x0.clone()
    _cached(shape, W, cache, 1e-6, b, io[0], ropes, -1 / 16)
    h = cache.header()
    assert h["hit"] == 1 and h["diff"] == 0.0 and h["hits"] == 1
    # bf16(F + (final - F)) = final: the reused step equals the computed one
    np.testing.assert_array_equal(to_np(b), to_np(a))


def test_hit_step_matches_the_device_residuals_and_the_oracle():
    d, W, shape, ropes, io = _setup()
    cache = kl.DitCache(shape)
    lat = d["latent"].cuda().contiguous()
    ts = dit.timesteps(16)
    ref_cache = {}
    for step in range(CFG.n_steps):
        dt = ts[step + 1] - ts[step]
        before = to_np(lat).copy()
        _cached(shape, W, cache, 1e9, lat, io[step], ropes, dt)  # every step after the first reuses
        h = cache.header()
        arr = {k: v.double().cpu().numpy() for k, v in cache.arrays().items()}
        assert h["hit"] == (1 if step > 0 else 0)
        if step > 0:
            # the reduction: diff against the device's own residual buffers
            want = np.abs(arr["r_cur"] - arr["r_ref"]).sum() / np.abs(arr["r_ref"]).sum()
            assert abs(h["diff"] - want) <= 1e-5 * want, (h["diff"], want)
        text, w, mods, sh = _oracle_args(CFG, d, step)
        v_ref = dit.velocity_cached(before, text, w, mods, sh, ref_cache, 1e9)
        assert ref_cache["hit"] == bool(h["hit"])
        v_gpu = (to_np(lat).astype(np.float64) - before) / dt
        err = rel_l2(v_gpu, dit.unpatchify(v_ref, CFG.grid_h, CFG.grid_w, CFG.channels))
        assert err <= 3e-2, (step, err)
        if step > 0:
            # both sides measured a clearly non-zero change of the probe residual
            assert h["diff"] > 0 and ref_cache["diff"] > 0


@pytest.mark.parametrize("thr", [0.0, 1e9, 0.24])
def test_graph_capture_takes_the_same_decisions_as_eager(thr):
    d, W, shape, ropes, io = _setup()
    n = 3
    steps = [io[s % CFG.n_steps] for s in range(n)]
    x0 = d["latent"].cuda().contiguous()
    # eager
    cache_e = kl.DitCache(shape)
    lat_e = x0.clone()
    hits_e = []
    for s in range(n):
        _cached(shape, W, cache_e, thr, lat_e, steps[s], ropes, -1 / 16)
        hits_e.append(cache_e.header()["hit"])
    # captured: the decision is taken on the device and guards blocks 1.. with
    # a conditional node
    cache_g = kl.DitCache(shape)
    lat_g = x0.clone()
    wabi = W.abi()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for s in range(n):
            kl.dit_step_cached(shape, W, cache_g, thr, lat_g, *steps[s], *ropes, -1 / 16, w_abi=wabi)
    for _ in range(2):  # replays are independent once the cache is reset
        lat_g.copy_(x0)
        cache_g.reset()
        g.replay()
        torch.cuda.synchronize()
        h = cache_g.header()
        assert h["steps"] == n and h["hits"] == sum(hits_e), (h, hits_e)
        np.testing.assert_array_equal(to_np(lat_g), to_np(lat_e))
    if thr == 0.0:
        assert sum(hits_e) == 0
    if thr == 1e9:
        assert hits_e == [0] + [1] * (n - 1)
    del g
    assert kl.device_status() == "KL_OK"


def test_cached_step_rejects_bad_arguments():
    d, W, shape, ropes, io = _setup()
    cache = kl.DitCache(shape)
    small = kl.DitCache.__new__(kl.DitCache)
    small.shape, small.buf = shape, cache.buf[: cache.buf.numel() // 2]
    with pytest.raises(kl.KLError) as e:
        _cached(shape, W, small, 0.24, d["latent"].cuda().contiguous(), io[0], ropes, -1 / 16)
    assert e.value.status == 4  # KL_ERR_WORKSPACE
    none = kl.DitShape(CFG.n_text, CFG.grid_h, CFG.grid_w, CFG.channels, CFG.hidden, CFG.heads, CFG.mlp_hidden, 0, 0,
                       CFG.attn)
    with pytest.raises(kl.KLError):
        kl.DitCache(none)
