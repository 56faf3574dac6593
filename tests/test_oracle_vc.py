"""Pins of the VC-Attention repair oracle (oracle/vc.py): the budget limits
(0 is the FP8 reading, 1 is exact softmax attention), the exact merge of
softmax parts over a random split of the keys against a brute-force softmax,
the estimated attention shares by explicit loops, the selection (count,
order, ties) by brute force, and repair moving the output toward the exact
attention."""

import math

import numpy as np

from oracle import block, vc


def _qkv(T, H, d, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((T, H, d)) * scale for _ in range(3)]


def test_budget_zero_is_the_fp8_reading_and_one_is_exact():
    q, k, v = _qkv(300, 2, 128, 1)        # two query blocks, three key tiles (the last ragged)
    none = vc.vc_select(q, k, 0.0)
    assert not none.any()
    np.testing.assert_allclose(vc.attention_vc(q, k, v, none), block.attention_fp8_emulated(q, k, v),
                               rtol=0, atol=1e-14)
    every = vc.vc_select(q, k, 1.0)
    assert every.all()
    np.testing.assert_allclose(vc.attention_vc(q, k, v, every), block.attention(q, k, v)[0], rtol=1e-12,
                               atol=1e-13)


def test_merge_of_parts_is_the_softmax_over_their_union():
    rng = np.random.default_rng(2)
    R, N, d = 5, 37, 8
    q, k, v = rng.standard_normal((R, d)) * 3, rng.standard_normal((N, d)), rng.standard_normal((N, d))
    perm = rng.permutation(N)
    parts = [vc.exact_part(q, k, v, np.sort(perm[a:b])) for a, b in ((0, 10), (10, 11), (11, N))]
    got = vc.merge_parts(parts)
    for r in range(R):
        t = [sum(q[r, x] * k[c, x] for x in range(d)) / math.sqrt(d) for c in range(N)]
        e = [math.exp(ti - max(t)) for ti in t]
        want = [sum(e[c] * v[c, x] for c in range(N)) / sum(e) for x in range(d)]
        np.testing.assert_allclose(got[r], want, rtol=1e-12, atol=1e-13)
    # each part's (m, l) carries its mass: l * 2^m = sum 2^t, t in log2 units
    O, m, l = parts[2]
    cols = np.sort(perm[11:])
    t2 = (q @ k[cols].T) * (np.log2(np.e) / np.sqrt(d))
    np.testing.assert_allclose(l * np.exp2(m), np.exp2(t2).sum(axis=1), rtol=1e-12)


def test_attention_shares_by_explicit_loops():
    T, H, d, qb, tile = 11, 2, 4, 4, 3
    q, k, _ = _qkv(T, H, d, 3)
    w = vc.vc_weights(q, k, qb, tile)
    assert w.shape == (H, 3, 4)
    for h in range(H):
        for b in range(3):
            rq = range(b * qb, min(T, (b + 1) * qb))
            qbar = [sum(q[r, h, x] for r in rq) / len(rq) for x in range(d)]
            s = []
            for j in range(4):
                rk = range(j * tile, min(T, (j + 1) * tile))
                kbar = [sum(k[r, h, x] for r in rk) / len(rk) for x in range(d)]
                s.append(sum(a * c for a, c in zip(qbar, kbar)) / math.sqrt(d) * math.log2(math.e))
            e = [2.0 ** (si - max(s)) for si in s]
            np.testing.assert_allclose(w[h, b], [ei / sum(e) for ei in e], rtol=1e-12)


def test_selection_count_order_and_ties():
    q, k, _ = _qkv(11, 2, 4, 4)
    w = vc.vc_weights(q, k, 4, 3)                        # 3 x 4 = 12 pairs per head
    for budget, R in ((0.05, 0), (0.1, 1), (0.25, 3), (0.5, 6)):
        rep = vc.vc_select(q, k, budget, 4, 3)
        for h in range(2):
            assert rep[h].sum() == R
            if R:
                # brute force: the R largest shares
                assert w[h][rep[h]].min() >= w[h][~rep[h]].max()
    # equal shares go to the lower (b, j): three identical key tiles give
    # every pair a share of 1/3
    ke = np.tile(k[:3], (3, 1, 1))                       # 9 keys, tiles of 3
    qe = q[:9]
    rep = vc.vc_select(qe, ke, 0.25, 4, 3)
    we = vc.vc_weights(qe, ke, 4, 3)
    np.testing.assert_allclose(we, np.full_like(we, 1 / 3), rtol=1e-12)
    R = int(np.floor(0.25 * 3 * 3))
    for h in range(2):
        flat = np.flatnonzero(rep[h].reshape(-1))
        np.testing.assert_array_equal(flat, np.arange(R))


def test_repairing_the_heaviest_tiles_moves_the_output_toward_exact():
    # one key tile carries most of the attention (queries lean on a direction
    # its keys share); repairing it removes most of the FP8 error of the block
    T, H, d = 512, 1, 128
    rng = np.random.default_rng(5)
    q = 0.3 * rng.standard_normal((T, H, d))
    k = 0.3 * rng.standard_normal((T, H, d))
    v = rng.standard_normal((T, H, d))
    q[:, 0, :8] += 1.5
    k[256:384, 0, :8] += 1.5
    exact, _ = block.attention(q, k, v)
    none = vc.attention_vc(q, k, v, vc.vc_select(q, k, 0.0))
    rep = vc.vc_select(q, k, 0.25)                       # 2 blocks x 4 tiles: R = 2
    assert rep[0, :, 2].all() and rep.sum() == 2         # the heavy tile of each query block
    fixed = vc.attention_vc(q, k, v, rep)
    err = lambda a: np.linalg.norm(a - exact) / np.linalg.norm(exact)
    assert err(fixed) < 0.5 * err(none)
