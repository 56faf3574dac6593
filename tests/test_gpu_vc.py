"""VC-Attention repair on the GPU (kl_vc_select, kl_joint_attention_vc, the
block's vc_budget) against the oracle's reading (oracle/vc.py): the device's
selection equals the oracle's up to pairs whose fp32 shares lie within
rounding of the R-th largest, the merged attention over the device's own
selection is within the FP8 bar of the oracle, budget 0 is the FP8 kernel bit
for bit and budget 1 is BF16 attention over every key."""

import numpy as np
import pytest
import torch

import diffusion_transformer_image_nvfp4_b200 as kl
from oracle import block, vc
from synth import MOD_NAMES, WORKLOADS, block_inputs, normal_bf16, sparse_attention_qkv
from tests.helpers import rel_l2, to_np

pytestmark = pytest.mark.gpu


def _fp8(qkv, T, H):
    D = H * 128
    amax = qkv.float().abs().view(T, 3, H, 128).amax(dim=(0, 3)).reshape(-1).contiguous()
    x8, sc = kl.cast_fp8_per_head(qkv, amax)
    return x8, dict(sq=sc[:H], sk=sc[H:2 * H], sv=sc[2 * H:])


def _run(qkv, T, H, budget):
    D = H * 128
    x8, sc = _fp8(qkv, T, H)
    l8, l16 = kl.vc_select(qkv, qkv[:, D:], T, H, 3 * D, budget)
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    out = kl.joint_attention_vc(x8, x8[:, D:], x8[:, 2 * D:], 3 * D, sc["sq"], sc["sk"], sc["sv"], qkv, qkv[:, D:],
                                qkv[:, 2 * D:], 3 * D, T, H, l8, l16, amax=amax)
    torch.cuda.synchronize()
    assert kl.device_status() == "KL_OK"
    return x8, sc, to_np(l8), to_np(l16), to_np(out), float(amax.item())


def _repaired_from_lists(l8, l16, nkt):
    """The repaired set [H, n_qb, n_kt] the device chose, and a consistency
    check of the two lists (complements; both halves of a block agree)."""
    H, nqb, _ = l8.shape
    rep = np.zeros((H, nqb, nkt), dtype=bool)
    for h in range(H):
        for b in range(nqb):
            keep = l8[h, b, 1:1 + l8[h, b, 0]]
            fix = l16[h, 2 * b, 1:1 + l16[h, 2 * b, 0]]
            assert np.all(np.diff(keep) > 0) and np.all(np.diff(fix) > 0)
            assert sorted(np.concatenate([keep, fix]).tolist()) == list(range(nkt))
            if 2 * b + 1 < l16.shape[1]:
                np.testing.assert_array_equal(l16[h, 2 * b + 1], l16[h, 2 * b])
            rep[h, b, fix] = True
    return rep


def _check_selection(q, k, rep_dev, budget):
    w = vc.vc_weights(q, k)
    H, nqb, nkt = w.shape
    R = int(np.floor(budget * nqb * nkt))
    rep_ref = vc.vc_select(q, k, budget)
    for h in range(H):
        assert rep_dev[h].sum() == R
        diff = rep_dev[h] ^ rep_ref[h]
        if diff.any():
            wr = np.sort(w[h].reshape(-1))[::-1][R - 1]
            assert np.all(np.abs(w[h][diff] - wr) <= 1e-5 * wr + 1e-30), (h, w[h][diff], wr)


@pytest.mark.parametrize("T,H,budget,seed", [(1000, 2, 0.05, 1), (4608, 2, 0.005, 2), (300, 3, 0.3, 3)])
def test_vc_attention_matches_the_oracle_on_structured_inputs(T, H, budget, seed):
    qkv = sparse_attention_qkv(T, H, seed=seed).cuda()
    x8, sc, l8, l16, out, amax = _run(qkv, T, H, budget)
    nkt = -(-T // 128)
    rep = _repaired_from_lists(l8, l16, nkt)
    v3 = qkv.float().cpu().numpy().reshape(T, 3, H, 128)
    q, k, v = v3[:, 0], v3[:, 1], v3[:, 2]
    _check_selection(q, k, rep, budget)
    want = vc.attention_vc(q, k, v, rep).reshape(T, H * 128)
    err = rel_l2(out, want)
    print(f"vc T={T} H={H} budget={budget}: repaired {int(rep.sum())} pairs, rel L2 vs oracle {err:.2e}")
    assert err <= 5e-3
    assert amax == np.abs(out).max()


def test_budget_zero_is_the_fp8_kernel_bit_for_bit():
    T, H = 1000, 2
    qkv = normal_bf16((T, 3 * H * 128), 5).cuda()
    x8, sc, l8, l16, out, _ = _run(qkv, T, H, 0.0)
    assert (l16[:, :, 0] == 0).all()
    D = H * 128
    dense = kl.joint_attention(x8, x8[:, D:], x8[:, 2 * D:], T, H, 3 * D, "fp8", **sc)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out, to_np(dense))


def test_budget_one_is_bf16_attention_over_every_key():
    T, H = 640, 2
    qkv = normal_bf16((T, 3 * H * 128), 6).cuda()
    _, _, l8, l16, out, _ = _run(qkv, T, H, 1.0)
    assert (l8[:, :, 0] == 0).all() and (l16[:, :, 0] == 5).all()
    v3 = qkv.float().cpu().numpy().reshape(T, 3, H, 128)
    exact, _ = block.attention(v3[:, 0], v3[:, 1], v3[:, 2])
    assert rel_l2(out, exact.reshape(T, H * 128)) <= 1e-2


def test_block_with_repair_budget():
    name = "tiny"
    wl = WORKLOADS[name]
    inp = block_inputs(name)
    d = {k: v.cuda() for k, v in inp.items()}
    W = kl.prepare_block_weights(d["wqkv"], d["wo"], d["w1"], d["w2"])
    cs = kl.rope_table(wl.n_text, wl.grid_h, wl.grid_w, wl.n_ref)
    mod = {n: d[n] for n in MOD_NAMES}
    run = lambda b: to_np(kl.joint_block_forward(W, d["x"], mod, cs, wl.heads, wl.mlp_hidden, "fp8",
                                                 vc_budget=b).clone())
    dense = run(0.0)
    np.testing.assert_array_equal(run(0.0), dense)
    a, b = run(0.2), run(0.2)
    np.testing.assert_array_equal(a, b)                  # deterministic
    assert np.isfinite(a).all() and not np.array_equal(a, dense)
    with pytest.raises(kl.KLError, match="INVALID_ARG"):  # BF16 attention has nothing to repair
        kl.joint_block_forward(W, d["x"], mod, cs, wl.heads, wl.mlp_hidden, "bf16", vc_budget=0.1)
    assert kl.device_status() == "KL_OK"
