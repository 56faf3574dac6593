"""Pins of the Sol-Attention oracle (oracle/sparse.py): block means and the
estimated tile scores by brute force, the dense limits (tau = inf equals the
dense exact attention and the dense FP8 emulation), tau = 0 keeping only the
strongest tile, sparse attention by brute force over the kept keys, and a
far-away key tile that is skipped without changing the output."""

import numpy as np

from oracle import block, sparse


def _qkv(T, H, d, seed):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((T, H, d)) for _ in range(3)]


def test_block_means_and_scores_by_brute_force():
    T, H, d, qb, tile = 11, 2, 8, 4, 3   # ragged query block (3 rows) and key tile (2 rows)
    q, k, _ = _qkv(T, H, d, 0)
    c = np.array([0.7, 1.3])
    keep, s_hat = sparse.sol_select(q, k, c, 1.0, qb, tile)
    assert s_hat.shape == (H, 3, 4)
    for h in range(H):
        for b in range(3):
            qbar = [sum(q[r, h, x] for r in range(b * qb, min(T, (b + 1) * qb))) / len(range(b * qb, min(T, (b + 1) * qb)))
                    for x in range(d)]
            for j in range(4):
                rows = range(j * tile, min(T, (j + 1) * tile))
                kbar = [sum(k[r, h, x] for r in rows) / len(rows) for x in range(d)]
                want = c[h] * sum(a * bb for a, bb in zip(qbar, kbar))
                assert abs(s_hat[h, b, j] - want) <= 1e-12 * (1 + abs(want))
            assert keep[h, b, np.argmax(s_hat[h, b])]
            np.testing.assert_array_equal(keep[h, b], s_hat[h, b] >= s_hat[h, b].max() - 1.0)


def test_tau_limits():
    q, k, _ = _qkv(40, 3, 8, 1)
    keep, s_hat = sparse.sol_select(q, k, np.ones(3), np.inf, 8, 8)
    assert keep.all()
    keep0, _ = sparse.sol_select(q, k, np.ones(3), 0.0, 8, 8)
    np.testing.assert_array_equal(keep0, s_hat == s_hat.max(axis=2, keepdims=True))
    assert (keep0.sum(axis=2) >= 1).all()


def test_dense_limit_equals_the_dense_attention_and_fp8_emulation():
    T, H, d = 300, 2, 128   # three key tiles, the last ragged; two query blocks of 256
    q, k, v = _qkv(T, H, d, 2)
    keep = np.ones((H, 2, 3), dtype=bool)
    dense, _ = block.attention(q, k, v)
    np.testing.assert_allclose(sparse.attention_sparse_exact(q, k, v, keep, 256), dense, rtol=0, atol=1e-12)
    emu = block.attention_fp8_emulated(q, k, v)
    np.testing.assert_allclose(sparse.attention_fp8_emulated_sparse(q, k, v, keep, 256), emu, rtol=0, atol=1e-12)


def test_sparse_attention_by_brute_force_over_the_kept_keys():
    T, H, d, qb, tile = 10, 1, 4, 4, 3
    q, k, v = _qkv(T, H, d, 3)
    keep = np.array([[[True, False, True, False], [False, True, False, True], [True, True, False, False]]])
    out = sparse.attention_sparse_exact(q, k, v, keep, qb, tile)
    for r in range(T):
        b = r // qb
        cols = [c for c in range(T) if keep[0, b, c // tile]]
        s = [sum(q[r, 0, x] * k[c, 0, x] for x in range(d)) / np.sqrt(d) for c in cols]
        w = np.exp(np.array(s) - max(s))
        w /= w.sum()
        want = sum(wi * v[c, 0] for wi, c in zip(w, cols))
        np.testing.assert_allclose(out[r, 0], want, rtol=0, atol=1e-12)


def test_a_far_away_tile_is_skipped_without_changing_the_output():
    T, H, d = 384, 1, 128
    rng = np.random.default_rng(4)
    q = 0.1 * rng.standard_normal((T, H, d))
    k = 0.1 * rng.standard_normal((T, H, d))
    v = rng.standard_normal((T, H, d))
    q[:, 0, 0] += 3.0          # every query leans on direction 0
    k[128:256, 0, 0] -= 60.0   # key tile 1 points away: scores ~ -180 / sqrt(128) lower
    c = np.array([sparse.LOG2E / np.sqrt(d)])
    keep, s_hat = sparse.sol_select(q, k, c, 4.0, 128)
    assert not keep[0, :, 1].any() and keep[0, :, 0].all() and keep[0, :, 2].all()
    dense, _ = block.attention(q, k, v)
    # the skipped keys carry weights below 2^-20 of the kept ones
    np.testing.assert_allclose(sparse.attention_sparse_exact(q, k, v, keep, 128), dense, rtol=0, atol=1e-5)
    q8, k8, c8 = sparse.fp8_select_inputs(q, k)
    keep8, _ = sparse.sol_select(q8, k8, c8, 4.0, 256)
    assert not keep8[0, :, 1].any()


def test_fp8_sparse_emulation_equals_the_dense_emulation_over_the_kept_keys():
    # When every kept list holds the tile that carries each head's largest |k|
    # and |v| (tile 0 here), the per-head E4M3 scales over all tokens equal
    # those over the kept keys, so each query block's sparse pass must equal
    # the dense FP8 emulation run on just its kept keys (full 128-key tiles,
    # so the tile boundaries coincide).  This pins the per-block bookkeeping
    # of the sparse wrapper; the tile-by-tile steps themselves are pinned
    # exactly in test_oracle_block.py.
    T, H, d = 512, 2, 128
    q, k, v = _qkv(T, H, d, 5)
    k[3] *= 4.0
    v[5] *= 4.0
    keep = np.array([[[True, False, True, True], [True, True, False, False]],
                     [[True, True, True, False], [True, False, False, True]]])
    got = sparse.attention_fp8_emulated_sparse(q, k, v, keep, 256)
    for h in range(H):
        for b in range(2):
            rows = np.arange(b * 256, (b + 1) * 256)
            cols = sparse.kept_key_rows(keep[h, b], T)
            qq = np.concatenate([q[rows][:, h:h + 1], q[:, h:h + 1]])   # all rows keep the q scale unchanged
            want = block.attention_fp8_emulated(qq, k[cols][:, h:h + 1], v[cols][:, h:h + 1],
                                                 rows=np.arange(len(rows)))
            np.testing.assert_allclose(got[rows, h], want[:, 0], rtol=0, atol=1e-12)
