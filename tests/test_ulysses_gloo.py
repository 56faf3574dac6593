"""The data movement of Ulysses sequence parallelism on CPU: two gloo ranks
run the same all-to-all head scatter / gather and max all-reduce helpers the
NCCL path uses, checked against slices of the unsharded tensors."""

import os
import socket
import sys
from datetime import timedelta

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    from diffusion_transformer_image_nvfp4_b200 import ulysses

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        T, H, d, parts = 12, 4, 8, 3
        g = torch.Generator().manual_seed(0)
        full = torch.randn(T, parts, H, d, generator=g)          # the unsharded q | k | v
        t0, t1 = ulysses.token_range(T, world, rank)
        hn = H // world
        results = []
        for dtype in (torch.float32, torch.bfloat16, torch.uint8):
            src = (full * 40).to(dtype) if dtype == torch.uint8 else full.to(dtype)
            mine = src[t0:t1].reshape(t1 - t0, parts * H * d).contiguous()
            heads = ulysses.scatter_heads(mine, parts, H, None if world == 1 else dist.group.WORLD)
            want = src[:, :, rank * hn:(rank + 1) * hn, :].reshape(T, parts * hn * d)
            ok_s = torch.equal(heads, want)
            # O of this rank's heads for all tokens -> this rank's tokens, all heads
            o_full = src[:, 0]                                     # [T, H, d]
            o_heads = o_full[:, rank * hn:(rank + 1) * hn, :].reshape(T, hn * d).contiguous()
            back = ulysses.gather_heads(o_heads, H, dist.group.WORLD)
            ok_g = torch.equal(back, o_full[t0:t1].reshape(t1 - t0, H * d))
            results.append((str(dtype), ok_s, ok_g))
        m = torch.tensor([float(rank), 10.0 - rank, -1.0])
        ulysses.all_max(m, dist.group.WORLD)
        q.put((rank, results, m.tolist()))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_ranks_scatter_gather_heads_and_max_reduce():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, results, m in got:
        for dtype, ok_s, ok_g in results:
            assert ok_s and ok_g, (rank, dtype, ok_s, ok_g)
        assert m == [1.0, 10.0, -1.0]


def test_token_range_and_shape_checks():
    sys.path.insert(0, ROOT)
    from diffusion_transformer_image_nvfp4_b200 import ulysses
    assert ulysses.token_range(4608, 8, 3) == (1728, 2304)
    assert [ulysses.token_range(12, 3, r) for r in range(3)] == [(0, 4), (4, 8), (8, 12)]
    with pytest.raises(ValueError):
        ulysses.token_range(10, 4, 0)
