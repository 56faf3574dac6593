"""Sol-Attention tile skipping (kl_sol_select, kl_joint_attention_sparse and
the block's sol_tau) against the oracle's reading of it (oracle/sparse.py)."""

import numpy as np
import pytest
import torch

import diffusion_transformer_image_nvfp4_b200 as kl
from oracle import sparse
from oracle.codecs import e4m3_decode
from synth import WORKLOADS, block_inputs, normal_bf16, sparse_attention_qkv
from tests.helpers import rel_l2, to_np

pytestmark = pytest.mark.gpu


def _split(qkv, T, H):
    x = qkv.float().numpy().reshape(T, 3, H, 128)
    return x[:, 0], x[:, 1], x[:, 2]


def _fp8(qkv, T, H):
    g = qkv.cuda()
    q, k, v = _split(qkv, T, H)
    am = np.concatenate([np.abs(t).max(axis=(0, 2)) for t in (q, k, v)]).astype(np.float32)
    return kl.cast_fp8_per_head(g, torch.from_numpy(am).cuda())


def _lists_match(got, keep, s_hat, tau):
    """The device lists against the oracle's keep mask: counts and ascending
    indices well formed; a tile may differ only within fp32 noise of the
    threshold (the device forms means and dots in fp32)."""
    H, nqb, nkt = keep.shape
    got = got.cpu().numpy()
    for h in range(H):
        for b in range(nqb):
            cnt = got[h, b, 0]
            idx = got[h, b, 1:1 + cnt]
            assert 1 <= cnt <= nkt and np.all(np.diff(idx) > 0) and idx[0] >= 0 and idx[-1] < nkt
            mask = np.zeros(nkt, dtype=bool)
            mask[idx] = True
            thr = s_hat[h, b].max() - tau
            for j in np.flatnonzero(mask != keep[h, b]):
                assert abs(s_hat[h, b, j] - thr) <= 1e-4 * (1 + abs(thr)), (h, b, j, s_hat[h, b, j], thr)


@pytest.mark.parametrize("T,H,tau", [(1000, 2, 1.0), (4608, 3, 2.0), (300, 1, 0.5)])
def test_fp8_selection_and_sparse_attention_match_the_oracle(T, H, tau):
    qkv = sparse_attention_qkv(T, H, seed=T + H)
    D = H * 128
    q8, sc = _fp8(qkv, T, H)
    lst = kl.sol_select(q8, q8[:, D:], T, H, 3 * D, tau, "fp8", sq=sc[:H], sk=sc[H:2 * H])
    # the oracle selects from the same E4M3 values and scales
    raw = to_np(q8).reshape(T, 3, H, 128)
    qv, kv = e4m3_decode(raw[:, 0]), e4m3_decode(raw[:, 1])
    scn = to_np(sc).astype(np.float64)
    c = sparse.LOG2E / np.sqrt(128) * scn[:H] * scn[H:2 * H]
    keep, s_hat = sparse.sol_select(qv, kv, c, tau, 256)
    _lists_match(lst, keep, s_hat, tau)
    # attention over the device's own lists
    dev_keep = np.zeros_like(keep)
    ln = lst.cpu().numpy()
    for h in range(H):
        for b in range(keep.shape[1]):
            dev_keep[h, b, ln[h, b, 1:1 + ln[h, b, 0]]] = True
    assert (~dev_keep).any(), "the structured input should skip tiles"
    got = to_np(kl.joint_attention_sparse(q8, q8[:, D:], q8[:, 2 * D:], T, H, 3 * D, lst, "fp8", sq=sc[:H],
                                          sk=sc[H:2 * H], sv=sc[2 * H:])).reshape(T, H, 128)
    q, k, v = _split(qkv, T, H)
    emu = sparse.attention_fp8_emulated_sparse(q, k, v, dev_keep, 256)
    assert rel_l2(got, emu) <= 5e-3
    exact = sparse.attention_sparse_exact(q, k, v, dev_keep, 256)
    assert rel_l2(got, exact) <= 8e-2


def test_bf16_sparse_attention_matches_the_exact_masked_softmax():
    T, H, tau = 900, 2, 1.0
    qkv = sparse_attention_qkv(T, H, seed=17)
    g = qkv.cuda()
    D = H * 128
    lst = kl.sol_select(g, g[:, D:], T, H, 3 * D, tau, "bf16")
    q, k, v = _split(qkv, T, H)
    keep, s_hat = sparse.sol_select(q, k, np.full(H, sparse.LOG2E / np.sqrt(128)), tau, 128)
    _lists_match(lst, keep, s_hat, tau)
    ln = lst.cpu().numpy()
    dev_keep = np.zeros_like(keep)
    for h in range(H):
        for b in range(keep.shape[1]):
            dev_keep[h, b, ln[h, b, 1:1 + ln[h, b, 0]]] = True
    assert (~dev_keep).any()
    got = to_np(kl.joint_attention_sparse(g, g[:, D:], g[:, 2 * D:], T, H, 3 * D, lst, "bf16")).reshape(T, H, 128)
    assert rel_l2(got, sparse.attention_sparse_exact(q, k, v, dev_keep, 128)) <= 1e-2


@pytest.mark.parametrize("prec", ["fp8", "bf16"])
def test_infinite_tau_is_bit_identical_to_dense(prec):
    T, H = 1000, 2
    qkv = normal_bf16((T, 3 * H * 128), 3, 1.0)
    D = H * 128
    if prec == "fp8":
        x, sc = _fp8(qkv, T, H)
        sv = dict(sq=sc[:H], sk=sc[H:2 * H], sv=sc[2 * H:])
    else:
        x, sv = qkv.cuda(), {}
    lst = kl.sol_select(x, x[:, D:], T, H, 3 * D, float("inf"), prec, sq=sv.get("sq"), sk=sv.get("sk"))
    nkt = -(-T // 128)
    assert (lst[:, :, 0] == nkt).all()
    dense = kl.joint_attention(x, x[:, D:], x[:, 2 * D:], T, H, 3 * D, prec, **sv)
    sp = kl.joint_attention_sparse(x, x[:, D:], x[:, 2 * D:], T, H, 3 * D, lst, prec, **sv)
    torch.cuda.synchronize()
    assert torch.equal(dense, sp)


def test_block_sol_tau_dense_limit_and_skipping():
    wl = WORKLOADS["tiny"]
    d = block_inputs(wl)
    H, F = wl.heads, wl.mlp_hidden
    W = kl.prepare_block_weights(d["wqkv"].cuda(), d["wo"].cuda(), d["w1"].cuda(), d["w2"].cuda())
    x = d["x"].cuda()
    mod = {k: d[k].cuda() for k in ("shift1", "scale1", "gate1", "shift2", "scale2", "gate2")}
    rope = kl.rope_table(wl.n_text, wl.grid_h, wl.grid_w)
    dense = kl.joint_block_forward(W, x, mod, rope, H, F, wl.attn).clone()
    inf = kl.joint_block_forward(W, x, mod, rope, H, F, wl.attn, sol_tau=float("inf")).clone()
    torch.cuda.synchronize()
    assert torch.equal(dense, inf)
    # a tiny tau keeps (about) only the strongest tile of each query block
    tight = kl.joint_block_forward(W, x, mod, rope, H, F, wl.attn, sol_tau=1e-6).clone()
    torch.cuda.synchronize()
    assert torch.isfinite(tight.float()).all() and not torch.equal(dense, tight)
    assert kl.device_status() == "KL_OK"
