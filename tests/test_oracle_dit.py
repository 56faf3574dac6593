"""Pins of the oracle's DiT step (oracle/dit.py) against index brute force,
exact special cases and the Euler closed form."""

import numpy as np

from oracle import dit
from synth import DIT_CONFIGS, dit_inputs


def test_patchify_matches_the_index_map_and_inverts():
    rng = np.random.default_rng(0)
    gh, gw, c = 3, 5, 4
    lat = rng.standard_normal((2 * gh, 2 * gw, c))
    p = dit.patchify(lat)
    assert p.shape == (gh * gw, 4 * c)
    for y in range(2 * gh):
        for x in range(2 * gw):
            for ch in range(c):
                t, k = (y // 2) * gw + x // 2, 4 * ch + 2 * (y % 2) + (x % 2)
                assert p[t, k] == lat[y, x, ch]
    np.testing.assert_array_equal(dit.unpatchify(p, gh, gw, c), lat)


def test_euler_closed_form_over_linear_timesteps():
    # 16 steps of dt = -1/16 with a constant velocity: x_end = x_0 - v, exact
    # here (integers and multiples of 1/16 are exact in fp32)
    ts = dit.timesteps(16)
    assert ts[0] == 1.0 and ts[-1] == 0.0
    dts = np.diff(ts)
    assert np.all(dts == -1 / 16)
    rng = np.random.default_rng(1)
    gh, gw, c = 2, 3, 8
    x0 = rng.integers(-100, 100, (2 * gh, 2 * gw, c)).astype(np.float32)
    v_lat = rng.integers(-32, 32, (2 * gh, 2 * gw, c)).astype(np.float32)
    v = dit.patchify(v_lat)
    x = x0
    for dt in dts:
        x = dit.euler(x, v, dt, gh, gw, c)
    np.testing.assert_array_equal(x, x0 - v_lat)


def _tiny(zero_out=False, with_mode=True):
    cfg = DIT_CONFIGS["dit_tiny"]
    d = dit_inputs(cfg)
    f = lambda t: t.float().numpy()
    w = {"w_in": f(d["w_in"]), "w_out": f(d["w_out"]) * (0.0 if zero_out else 1.0),
         "mode_text": [{k: f(v) for k, v in b.items()} for b in d["mode_text"]] if with_mode else [],
         "mode_image": [{k: f(v) for k, v in b.items()} for b in d["mode_image"]] if with_mode else [],
         "joint": [{k: f(v) for k, v in b.items()} for b in d["joint"]]}
    mods = {"mode": f(d["mod_mode"][0]), "joint": f(d["mod_joint"][0]), "final": f(d["mod_final"][0])}
    shape = {"n_text": cfg.n_text, "grid_h": cfg.grid_h, "grid_w": cfg.grid_w, "channels": cfg.channels,
             "H": cfg.heads}
    return cfg, d["latent"].numpy(), f(d["text"]), w, mods, shape


def test_zero_output_projection_leaves_the_latent_unchanged():
    cfg, lat, text, w, mods, shape = _tiny(zero_out=True)
    out = dit.dit_step(lat, text, w, mods, shape, -1 / 16)
    np.testing.assert_array_equal(out, lat)


def test_velocity_is_finite_and_depends_on_the_text():
    cfg, lat, text, w, mods, shape = _tiny()
    v1 = dit.velocity(lat, text, w, mods, shape)
    v2 = dit.velocity(lat, text + 1.0, w, mods, shape)
    assert v1.shape == (cfg.grid_h * cfg.grid_w, 4 * cfg.channels)
    assert np.isfinite(v1).all()
    # the joint blocks mix text into the image tokens; the per-mode blocks alone
    # would not (checked with the joint blocks removed)
    assert np.abs(v1 - v2).max() > 0
    w_nojoint = dict(w, joint=[])
    mods_nj = dict(mods, joint=mods["joint"][:0])
    u1 = dit.velocity(lat, text, w_nojoint, mods_nj, shape)
    u2 = dit.velocity(lat, text + 1.0, w_nojoint, mods_nj, shape)
    np.testing.assert_array_equal(u1, u2)


def test_time_shift_keeps_endpoints_and_matches_its_closed_form():
    lin = dit.timesteps(16)
    sh = dit.timesteps(16, shift=6.93)
    assert sh[0] == 1.0 and sh[-1] == 0.0
    assert all(a > b for a, b in zip(sh, sh[1:]))  # strictly decreasing
    # the shift maps t to s t / (1 + (s - 1) t): at t = 1/2 that is s / (s + 1)
    assert abs(dit.timesteps(2, shift=6.93)[1] - 6.93 / 7.93) < 1e-15
    # s = 1 is the linear schedule; s > 1 keeps every step at higher noise
    assert dit.timesteps(16, shift=1.0) == lin
    assert all(a >= b for a, b in zip(sh, lin))
    # the Euler steps still integrate exactly from 1 to 0
    assert abs(sum(b - a for a, b in zip(sh, sh[1:])) + 1.0) < 1e-15
