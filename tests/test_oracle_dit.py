"""Pins of the oracle's DiT step (oracle/dit.py) against index brute force,
exact special cases and the Euler closed form."""

import numpy as np

from oracle import dit
from oracle.codecs import bf16_round
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


# ---------------------------------------------------------------- Cache-DiT


def test_residual_diff_hand_values_and_special_cases():
    # worked by hand: |1.5-1| + |-2+2| + |2-3| = 1.5 over |1| + |-2| + |3| = 6
    assert dit.residual_diff([1.5, -2.0, 2.0], [1.0, -2.0, 3.0]) == 0.25
    r_ref = np.array([[0.5, -1.0], [2.0, 0.0]])
    assert dit.residual_diff(2 * r_ref, r_ref) == 1.0   # doubled residual: 100% change
    assert dit.residual_diff(0 * r_ref, r_ref) == 1.0   # vanished residual
    assert dit.residual_diff(r_ref, r_ref) == 0.0
    assert dit.residual_diff(np.zeros(3), np.zeros(3)) == 0.0
    assert dit.residual_diff(np.ones(3), np.zeros(3)) == float("inf")


def _tiny_step_mods(step):
    cfg = DIT_CONFIGS["dit_tiny"]
    d = dit_inputs(cfg)
    f = lambda t: t.float().numpy()
    return {"mode": f(d["mod_mode"][step]), "joint": f(d["mod_joint"][step]), "final": f(d["mod_final"][step])}


def test_cache_threshold_zero_reproduces_the_plain_steps():
    cfg, lat, text, w, mods, shape = _tiny()
    cache, plain = {}, lat.copy()
    cached = lat.copy()
    for step in range(cfg.n_steps):
        m = _tiny_step_mods(step)
        plain = dit.dit_step(plain, text, w, m, shape, -1 / 16)
        cached = dit.dit_step(cached, text, w, m, shape, -1 / 16, cache=cache, threshold=0.0)
        assert not cache["hit"]
        np.testing.assert_array_equal(cached, plain)
    assert cache["hits"] == 0


def test_first_step_never_hits_and_a_repeated_input_reuses_exactly():
    cfg, lat, text, w, mods, shape = _tiny()
    cache = {}
    v0 = dit.velocity_cached(lat, text, w, mods, shape, cache, threshold=float("inf"))
    assert not cache["hit"] and cache["diff"] == float("inf")
    np.testing.assert_array_equal(v0, dit.velocity(lat, text, w, mods, shape))
    # the same input again: the probe residual is unchanged (diff 0), so the
    # step skips the remaining blocks and bf16(F + (final - F)) = final exactly
    v1 = dit.velocity_cached(lat, text, w, mods, shape, cache, threshold=1e-9)
    assert cache["hit"] and cache["diff"] == 0.0 and cache["hits"] == 1
    np.testing.assert_array_equal(v1, v0)


def test_a_hit_keeps_the_reference_and_really_skips_the_rest():
    cfg, lat, text, w, mods, shape = _tiny()
    rng = np.random.default_rng(5)
    lat_b = (lat + 0.05 * rng.standard_normal(lat.shape)).astype(np.float32)
    lat_c = (lat + 0.10 * rng.standard_normal(lat.shape)).astype(np.float32)

    def probe(x):
        tok = dit._embed(x, text, w, shape)
        f = dit._block(tok, 0, w, mods, shape, "exact")
        return tok, f, f.astype(np.float64) - tok.astype(np.float64)

    cache = {}
    dit.velocity_cached(lat, text, w, mods, shape, cache, threshold=1e9)  # miss: reference A
    _, _, r_a = probe(lat)
    v_b = dit.velocity_cached(lat_b, text, w, mods, shape, cache, threshold=1e9)  # hit
    assert cache["hit"]
    tok_b, f_b, r_b = probe(lat_b)
    assert cache["diff"] == dit.residual_diff(r_b, r_a) > 0
    # the hit's velocity is the head on bf16(F_B + R_A), not the full stack's
    full_b = dit.velocity(lat_b, text, w, mods, shape)
    assert np.abs(v_b - full_b).max() > 0
    _, f_a, _ = probe(lat)
    final_a = f_a
    for i in range(1, dit._n_blocks(w)):
        final_a = dit._block(final_a, i, w, mods, shape, "exact")
    r_rest_a = final_a.astype(np.float64) - f_a.astype(np.float64)
    reuse = bf16_round(f_b.astype(np.float64) + r_rest_a)
    np.testing.assert_array_equal(v_b, dit._head(reuse, w, mods, shape))
    # step C is measured against A (the last full step), not against B
    dit.velocity_cached(lat_c, text, w, mods, shape, cache, threshold=1e9)
    _, _, r_c = probe(lat_c)
    assert cache["diff"] == dit.residual_diff(r_c, r_a) != dit.residual_diff(r_c, r_b)
    # a threshold below the change forces the full stack again, which then
    # becomes the reference
    v_c = dit.velocity_cached(lat_c, text, w, mods, shape, cache, threshold=0.0)
    assert not cache["hit"]
    np.testing.assert_array_equal(v_c, dit.velocity(lat_c, text, w, mods, shape))
    np.testing.assert_array_equal(cache["r_ref"], r_c)


def test_smooth_modulations_are_linear_in_t_and_keep_the_other_draws():
    from synth import DitConfig
    cfg = DitConfig("smooth_probe", 16, 4, 4, 32, 128, 1, 384, 1, 2, 8, "bf16", 7)
    ind = dit_inputs(cfg, with_weights=False)
    smo = dit_inputs(cfg, with_weights=False, mods="smooth")
    np.testing.assert_array_equal(ind["latent"].numpy(), smo["latent"].numpy())
    np.testing.assert_array_equal(ind["text"].float().numpy(), smo["text"].float().numpy())
    for k in ("mod_mode", "mod_joint", "mod_final"):
        m = smo[k].double().numpy()
        assert m.shape == ind[k].shape
        # equal t steps: second differences vanish up to the three bf16
        # roundings in them (8 significant bits: each within 2^-8 of its value)
        second = m[2:] - 2 * m[1:-1] + m[:-2]
        assert np.abs(second).max() <= 4 * 2.0 ** -8 * np.abs(m).max()
        # consecutive steps move by |m1| / n_steps, far less than fresh draws
        step = np.abs(np.diff(m, axis=0)).mean()
        fresh = np.abs(np.diff(ind[k].double().numpy(), axis=0)).mean()
        assert step < 0.2 * fresh


def test_cache_probe_is_the_first_joint_block_without_per_mode_blocks():
    cfg, lat, text, w, mods, shape = _tiny(with_mode=False)
    mods = dict(mods, mode=mods["mode"][:0])
    cache = {}
    v0 = dit.velocity_cached(lat, text, w, mods, shape, cache, threshold=0.5)
    np.testing.assert_array_equal(v0, dit.velocity(lat, text, w, mods, shape))
    # the probe residual is joint block 0's: the reference equals it exactly
    tok = dit._embed(lat, text, w, shape)
    f = dit._block(tok, 0, w, mods, shape, "exact")
    np.testing.assert_array_equal(cache["r_ref"], f.astype(np.float64) - tok.astype(np.float64))
    v1 = dit.velocity_cached(lat, text, w, mods, shape, cache, threshold=0.5)
    assert cache["hit"] and cache["diff"] == 0.0
    np.testing.assert_array_equal(v1, v0)
