"""Ulysses sequence parallelism for the joint block.

[P1] "Optimizing FLUX 3 Image Klein inference on NVIDIA Blackwell GPUs", How
it works: to use several GPUs, the token sequence is split between them
(Ulysses) and attention is computed in a distributed way that still sees
every token; What you can do: the degree of this split is a setting
(``ulysses_size``).

The tokens of one sequence are sharded over the N ranks of a process group
(rank r holds tokens [r T/N, (r+1) T/N)); the weights are replicated.  Every
step of the block works per token except two:

* each per-tensor NVFP4 amax (of m1, O, m2 and h) and the per-head FP8 amax of
  q, k, v is a maximum over all tokens: the ranks all-reduce it (max) before
  encoding, so every rank encodes with the scales the unsharded block uses;
* attention mixes all tokens: an all-to-all turns the sequence shards of the
  FP8 (or bf16) q, k, v into head shards (all T tokens, H/N heads per rank),
  each rank runs the attention kernel on its heads, and an all-to-all turns
  the head shards of O back into sequence shards.

Every GEMM tile variant sums in the same K order and attention works per
head, so the sharded block gives the unsharded block's output bit for bit.
The collectives are torch.distributed calls (NCCL over NVLink on GPUs; the
data-movement helpers below also run on CPU tensors over gloo); all
arithmetic is the library's kernels.  N must divide T and H.

With a gloo process group and CUDA tensors the helpers stage through host
memory (device -> CPU, the gloo collective, CPU -> device): the same bytes
move and the ranks stay independent processes whose kernels never wait on
one another, so several ranks can share one GPU (a test configuration; the
data path is NCCL).
"""

import torch
import torch.distributed as dist

from . import (NVFP4, _check, _need, _stream, gemm_nvfp4_fused, joint_attention, lib, ln_modulate_bf16,
               quantize_nvfp4)


def _world(group):
    return 1 if group is None else dist.get_world_size(group)


def _rank(group):
    return 0 if group is None else dist.get_rank(group)


def _host_staged(t, group):
    """True when a collective on t must go through host memory: a CUDA
    tensor and a gloo group (gloo moves CPU tensors)."""
    return t.is_cuda and dist.get_backend(group) == "gloo"


def _all_to_all(recv, send, group):
    if _host_staged(send, group):
        r = torch.empty(recv.shape, dtype=recv.dtype)
        dist.all_to_all_single(r, send.cpu(), group=group)
        recv.copy_(r)
    else:
        dist.all_to_all_single(recv, send, group=group)


def token_range(T, world, rank):
    """Tokens [t0, t1) of ``rank`` when T tokens are split evenly over ``world``."""
    if T % world:
        raise ValueError(f"{world} ranks do not divide {T} tokens")
    n = T // world
    return rank * n, (rank + 1) * n


def scatter_heads(x, parts, heads, group=None):
    """Sequence shard -> head shard.

    x: [T/N, parts * heads * d] (e.g. q | k | v, each heads x d wide) on every
    rank.  Returns [T, parts * (heads/N) * d]: all T tokens (rank-major, i.e.
    in sequence order) and, in each part, this rank's heads r H/N .. (r+1) H/N.
    """
    world = _world(group)
    if world == 1:
        return x
    T_loc, C = x.shape
    if heads % world or C % (parts * heads):
        raise ValueError("ranks must divide the heads, and the columns be parts x heads x d")
    d = C // (parts * heads)
    hn = heads // world
    send = x.reshape(T_loc, parts, world, hn, d).permute(2, 0, 1, 3, 4).contiguous()
    recv = torch.empty_like(send)
    _all_to_all(recv, send, group)
    return recv.reshape(world * T_loc, parts * hn * d)


def gather_heads(o, heads, group=None):
    """Head shard -> sequence shard: o [T, (heads/N) * d] of this rank's heads
    for all tokens; returns [T/N, heads * d] of this rank's tokens."""
    world = _world(group)
    if world == 1:
        return o
    T, C = o.shape
    if heads % world or T % world:
        raise ValueError("ranks must divide the heads and the tokens")
    hn = heads // world
    d = C // hn
    T_loc = T // world
    send = o.contiguous()  # [world (destination), T/N, hn, d] in row-major order
    recv = torch.empty_like(send)
    _all_to_all(recv, send, group)
    return recv.reshape(world, T_loc, hn, d).permute(1, 0, 2, 3).reshape(T_loc, heads * d)


def all_max(t, group=None):
    """In-place elementwise maximum over the ranks (identity for one rank)."""
    if _world(group) > 1:
        if _host_staged(t, group):
            h = t.cpu()
            dist.all_reduce(h, op=dist.ReduceOp.MAX, group=group)
            t.copy_(h)
        else:
            dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return t


def _keep(trace, **tensors):
    """Device copies of intermediates into ``trace`` (no-op without one)."""
    if trace is None:
        return
    for k, t in tensors.items():
        trace[k] = (t.codes.clone(), t.scales.clone(), t.gs.clone()) if isinstance(t, NVFP4) else t.clone()


class UlyssesBlock:
    """One joint block over this rank's T/N tokens of a T-token sequence.

    weights: BlockWeights (replicated); T: tokens of the whole sequence;
    attn: "fp8" or "bf16"; group: the process group the sequence is sharded
    over (None: one rank).  D % 256 == 0, D <= 4096 (the widths the block
    computes its LayerNorm through the stored m).  Buffers are allocated once,
    for T/N tokens."""

    def __init__(self, weights, T, D, H, F, attn="fp8", group=None, device=None):
        self.w, self.T, self.D, self.H, self.F, self.attn, self.group = weights, T, D, H, F, attn, group
        self.world, self.rank = _world(group), _rank(group)
        if D != 128 * H or H % self.world:
            raise ValueError("D must be 128 H and the ranks must divide the heads")
        self.t0, self.t1 = token_range(T, self.world, self.rank)
        Tl, dev = self.t1 - self.t0, device or torch.device("cuda")
        self.T_loc, self.hn = Tl, H // self.world
        L = lib()
        bf = dict(dtype=torch.bfloat16, device=dev)

        def nvfp4(rows, cols):
            return NVFP4(torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev),
                         torch.empty(L.kl_nvfp4_scales_bytes(rows, cols, 1), dtype=torch.uint8, device=dev),
                         torch.empty(1, dtype=torch.float32, device=dev), rows, cols, "mma")

        self.m = torch.empty((Tl, D), **bf)
        self.a = nvfp4(Tl, D)           # m1, then O, then m2
        self.qkv = torch.empty((Tl, 3 * D), **bf)
        self.qkv8 = torch.empty((Tl, 3 * D), dtype=torch.uint8, device=dev)
        self.sc8 = torch.empty(3 * H, dtype=torch.float32, device=dev)
        self.qkv_amax = torch.empty(3 * H, dtype=torch.float32, device=dev)
        self.o_heads = torch.empty((T, self.hn * 128), **bf)
        self.x1 = torch.empty((Tl, D), **bf)
        self.h = torch.empty((Tl, F), **bf)
        self.hq = nvfp4(Tl, F)
        # amax words, one 256-byte slot each (the quantiser's workspace form):
        # 0 m1, 1 O, 2 m2, 3 h
        self.amax = torch.empty((4, 64), dtype=torch.float32, device=dev)

    def forward(self, x, mod, rope_local, out=None, trace=None):
        """x: bf16 [T/N, D] (this rank's tokens); mod: shift1 .. gate2 bf16 [D];
        rope_local: fp32 [16, T/N, 4, 2] (the rank's token columns of the
        kl_rope_table of the whole sequence).  Returns bf16 [T/N, D].
        ``trace`` (a dict, optional): receives device copies of every
        intermediate (m1, a1, qkv, qkv_amax, qkv8, sc8, o, oq, x1, m2, a2, h,
        hq; NVFP4 ones as (codes, scales, gs)) for stage-by-stage checks."""
        _need(x, torch.bfloat16, "x")
        if x.shape != (self.T_loc, self.D):
            raise ValueError("x: expected this rank's [T/N, D] tokens")
        D, H, hn, g = self.D, self.H, self.hn, self.group
        L = lib()
        if out is None:
            out = torch.empty_like(x)
        self.amax.zero_()
        self.qkv_amax.zero_()
        # 1. LN1 + adaLN -> m1, amax over all tokens, NVFP4
        ln_modulate_bf16(x, mod["shift1"], mod["scale1"], m_out=self.m, amax_out=self.amax[0])
        all_max(self.amax, g)
        quantize_nvfp4(self.m, amax_slot=self.amax[0], out=self.a)
        _keep(trace, m1=self.m, a1=self.a)
        # 2. QKV GEMM + RoPE, per-head amax over all tokens
        gemm_nvfp4_fused(self.a, self.w.wqkv, "qkv_rope", out=self.qkv, rope_cs=rope_local, amax=self.qkv_amax)
        all_max(self.qkv_amax, g)
        _keep(trace, qkv=self.qkv, qkv_amax=self.qkv_amax)
        # 3-4. (FP8 cast,) sequence shards -> head shards, attention on this rank's heads
        h0 = self.rank * hn
        if self.attn == "fp8":
            _check(L.kl_cast_fp8_per_head(self.qkv.data_ptr(), self.T_loc, 3 * D, 3 * D, self.qkv_amax.data_ptr(),
                                          self.qkv8.data_ptr(), self.sc8.data_ptr(), _stream()),
                   "kl_cast_fp8_per_head")
            heads = scatter_heads(self.qkv8, 3, H, g)
            _keep(trace, qkv8=self.qkv8, sc8=self.sc8)
            scales = dict(sq=self.sc8[h0:h0 + hn], sk=self.sc8[H + h0:H + h0 + hn],
                          sv=self.sc8[2 * H + h0:2 * H + h0 + hn])
        else:
            heads = scatter_heads(self.qkv, 3, H, g)
            scales = {}
        w = hn * 128
        joint_attention(heads, heads[:, w:], heads[:, 2 * w:], self.T, hn, 3 * w, self.attn,
                        amax=self.amax[1], out=self.o_heads, **scales)
        o = gather_heads(self.o_heads, H, g)
        _keep(trace, o=o)
        all_max(self.amax, g)
        # 5-6. NVFP4 of O, out-projection + gated residual
        quantize_nvfp4(o.contiguous(), amax_slot=self.amax[1], out=self.a)
        _keep(trace, oq=self.a)
        gemm_nvfp4_fused(self.a, self.w.wo, "gated_residual", out=self.x1, gate=mod["gate1"], residual=x)
        _keep(trace, x1=self.x1)
        # 7. LN2 + adaLN -> m2
        ln_modulate_bf16(self.x1, mod["shift2"], mod["scale2"], m_out=self.m, amax_out=self.amax[2])
        all_max(self.amax, g)
        quantize_nvfp4(self.m, amax_slot=self.amax[2], out=self.a)
        _keep(trace, m2=self.m, a2=self.a)
        # 8-10. MLP-up + SwiGLU, NVFP4 of h, MLP-down + gated residual
        gemm_nvfp4_fused(self.a, self.w.w1, "swiglu", out=self.h, amax=self.amax[3])
        all_max(self.amax, g)
        quantize_nvfp4(self.h, amax_slot=self.amax[3], out=self.hq)
        _keep(trace, h=self.h, hq=self.hq)
        gemm_nvfp4_fused(self.hq, self.w.w2, "gated_residual", out=out, gate=mod["gate2"], residual=self.x1)
        return out


def local_rope(rope_cs, t0, t1):
    """The columns of tokens [t0, t1) of a [16, T, 4, 2] kl_rope_table, contiguous."""
    return rope_cs[:, t0:t1].contiguous()

