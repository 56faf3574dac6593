"""Ulysses sequence parallelism (ulysses.UlyssesBlock) against the unsharded
block: one rank reproduces kl_joint_block_forward bit for bit (the sharded
path uses the same kernels with the amax taken as given); with two or more
GPUs, two NCCL ranks reproduce it too (skipped on a one-GPU machine: ranks
whose collectives wait on each other never share a GPU)."""

import os
import socket
import sys
from datetime import timedelta

import pytest
import torch

import diffusion_transformer_image_nvfp4_b200 as kl
from diffusion_transformer_image_nvfp4_b200 import ulysses
from synth import WORKLOADS, block_inputs

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
NAMES = ("shift1", "scale1", "gate1", "shift2", "scale2", "gate2")


def _setup(dev):
    wl = WORKLOADS["tiny"]
    d = block_inputs(wl)
    W = kl.prepare_block_weights(*(d[k].to(dev) for k in ("wqkv", "wo", "w1", "w2")))
    mod = {k: d[k].to(dev) for k in NAMES}
    rope = kl.rope_table(wl.n_text, wl.grid_h, wl.grid_w, device=dev)
    return wl, W, d["x"].to(dev), mod, rope


@pytest.mark.parametrize("attn", ["bf16", "fp8"])
def test_one_rank_is_bit_identical_to_the_block(attn):
    wl, W, x, mod, rope = _setup(torch.device("cuda"))
    T, H, F = wl.n_tokens, wl.heads, wl.mlp_hidden
    ref = kl.joint_block_forward(W, x, mod, rope, H, F, attn).clone()
    blk = ulysses.UlyssesBlock(W, T, wl.hidden, H, F, attn)
    got = blk.forward(x, mod, ulysses.local_rope(rope, 0, T))
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
    assert kl.device_status() == "KL_OK"


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, attn, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      NCCL_NVLS_ENABLE="0")
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    dev = torch.device("cuda", rank)
    torch.cuda.set_device(dev)
    dist.init_process_group("nccl", rank=rank, world_size=world, timeout=timedelta(seconds=60),
                            device_id=dev)
    try:
        wl, W, x, mod, rope = _setup(dev)
        T, H, F = wl.n_tokens, wl.heads, wl.mlp_hidden
        ref = kl.joint_block_forward(W, x, mod, rope, H, F, attn).clone()
        blk = ulysses.UlyssesBlock(W, T, wl.hidden, H, F, attn, group=dist.group.WORLD, device=dev)
        got = blk.forward(x[blk.t0:blk.t1].contiguous(), mod, ulysses.local_rope(rope, blk.t0, blk.t1))
        torch.cuda.synchronize()
        q.put((rank, bool(torch.equal(got, ref[blk.t0:blk.t1]))))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.skipif(torch.cuda.device_count() < 2, reason="needs two GPUs (one rank per GPU)")
@pytest.mark.parametrize("attn", ["bf16", "fp8"])
def test_two_ranks_are_bit_identical_to_the_block(attn):
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, attn, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    assert sorted(q.get(timeout=10) for _ in range(2)) == [(0, True), (1, True)]


def _staged_worker(rank, world, port, name, attn, q):
    # every rank on cuda:0; collectives over gloo through host memory, so the
    # ranks' kernels never wait on one another
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    try:
        wl = WORKLOADS[name]
        d = block_inputs(wl)
        W = kl.prepare_block_weights(*(d[k].to(dev) for k in ("wqkv", "wo", "w1", "w2")))
        mod = {k: d[k].to(dev) for k in NAMES}
        rope = kl.rope_table(wl.n_text, wl.grid_h, wl.grid_w, wl.n_ref, device=dev)
        x = d["x"].to(dev)
        T, H, F = wl.n_tokens, wl.heads, wl.mlp_hidden
        ref = kl.joint_block_forward(W, x, mod, rope, H, F, attn).clone()
        blk = ulysses.UlyssesBlock(W, T, wl.hidden, H, F, attn, group=dist.group.WORLD, device=dev)
        got = blk.forward(x[blk.t0:blk.t1].contiguous(), mod, ulysses.local_rope(rope, blk.t0, blk.t1))
        torch.cuda.synchronize()
        q.put((rank, bool(torch.equal(got, ref[blk.t0:blk.t1])), kl.device_status()))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("name,attn,world", [("tiny", "bf16", 2), ("tiny", "fp8", 2), ("tiny", "fp8", 4),
                                             ("t2i_1024", "fp8", 4)])
def test_host_staged_ranks_on_one_gpu_are_bit_identical_to_the_block(name, attn, world):
    # the sharded path with world > 1 on one GPU: token shards, the head
    # all-to-alls feeding the attention kernel, and the all-reduced amaxes
    # feeding the encodes (4 ranks x 6 heads on the 4,608-token block)
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_staged_worker, args=(r, world, port, name, attn, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=600)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0] * world, codes
    got = sorted(q.get(timeout=10) for _ in range(world))
    assert got == [(r, True, "KL_OK") for r in range(world)], got
