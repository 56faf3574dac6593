"""The whole joint block (kl_joint_block_forward) vs the oracle, from the raw
inputs: rel L2 of the bf16 block output within 1e-2 with BF16 attention, and
with FP8 attention within 3e-2 of the exact oracle and 1e-2 of the oracle's
FP8 flash pass (the block-level bars).  The residual x ~ N(0, 1) dominates the
output; the branches themselves are bounded stage by stage, each on the
GPU's own previous intermediate, in test_gpu_block_stages.py.  The
multi-reference blocks (20,992 and 21,504 tokens) compare sampled output rows
with the oracle's full-size run, stored by tests/golden/make_block_samples.py."""

import os

import numpy as np
import pytest
import torch

import diffusion_transformer_image_nvfp4_b200 as kl
from oracle import block, codecs, nvfp4
from synth import MOD_NAMES, WORKLOADS, block_inputs
from tests.helpers import rel_l2, to_np

pytestmark = pytest.mark.gpu


def _gpu_forward(name, inp=None, **over):
    wl = WORKLOADS[name]
    inp = block_inputs(name) if inp is None else inp
    inp = {**inp, **over}
    dev = {k: v.cuda() for k, v in inp.items()}
    W = kl.prepare_block_weights(dev["wqkv"], dev["wo"], dev["w1"], dev["w2"])
    cs = kl.rope_table(wl.n_text, wl.grid_h, wl.grid_w, wl.n_ref)
    out = kl.joint_block_forward(W, dev["x"], {n: dev[n] for n in MOD_NAMES}, cs, wl.heads, wl.mlp_hidden,
                                 attn=wl.attn)
    torch.cuda.synchronize()
    assert kl.device_status() == "KL_OK"
    return to_np(out), inp


def _oracle(name, inp, attn):
    wl = WORKLOADS[name]
    n = {k: v.float().numpy() for k, v in inp.items()}
    lay = block.TokenLayout(wl.n_text, wl.grid_h, wl.grid_w, wl.n_ref)
    return block.block_forward(n["x"], {k: n[k] for k in MOD_NAMES}, n, lay, wl.heads, attn=attn)


@pytest.mark.parametrize("name", ["micro", "tiny"])
def test_bf16_attention_blocks(name):
    got, inp = _gpu_forward(name)
    ref = _oracle(name, inp, "exact")
    x = inp["x"].float().numpy()
    assert rel_l2(got, ref) <= 1e-2
    print(f"{name}: out {rel_l2(got, ref):.2e}, branch out-x {rel_l2(got - x, ref - x):.2e}")


def test_zero_gates_return_the_input_exactly():
    name = "tiny"
    inp = block_inputs(name)
    z = torch.zeros_like(inp["gate1"])
    got, _ = _gpu_forward(name, inp, gate1=z, gate2=z)
    np.testing.assert_array_equal(got, inp["x"].float().numpy())


@pytest.mark.parametrize("name", ["t2i_1024", "i2i_1024"])
def test_fp8_attention_blocks_1024(name):
    got, inp = _gpu_forward(name)
    x = inp["x"].float().numpy()
    ref = _oracle(name, inp, "exact")
    assert rel_l2(got, ref) <= 3e-2
    emu = _oracle(name, inp, "fp8")
    assert rel_l2(got, emu) <= 1e-2
    print(f"{name}: out vs exact {rel_l2(got, ref):.2e}, vs fp8 {rel_l2(got, emu):.2e}; branch out-x vs exact "
          f"{rel_l2(got - x, ref - x):.2e}, vs fp8 {rel_l2(got - x, emu - x):.2e}")


GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.mark.parametrize("name", ["multiref_1024", "multiref_21504"])
def test_multiref_blocks_against_the_stored_oracle_rows(name):
    # the oracle's full-size run of this workload (both attention modes),
    # stored on a fixed sample of rows by tests/golden/make_block_samples.py
    ref = np.load(os.path.join(GOLDEN, f"block_samples_{name}.npz"))
    rows = ref["rows"]
    got, inp = _gpu_forward(name)
    assert got.shape[0] == WORKLOADS[name].n_tokens
    g = got[rows]
    exact, emu = codecs.bf16_from_bits(ref["exact"]), codecs.bf16_from_bits(ref["fp8"])
    assert rel_l2(g, exact) <= 3e-2
    assert rel_l2(g, emu) <= 1e-2
    x = inp["x"].float().numpy()[rows]
    print(f"{name}: out vs exact {rel_l2(g, exact):.2e}, vs fp8 {rel_l2(g, emu):.2e}; branch out-x vs exact "
          f"{rel_l2(g - x, exact - x):.2e}, vs fp8 {rel_l2(g - x, emu - x):.2e}")


def test_multiref_block_is_deterministic_and_zero_gates_are_the_identity():
    name = "multiref_1024"
    inp = block_inputs(name)
    a, _ = _gpu_forward(name, inp)
    b, _ = _gpu_forward(name, inp)
    assert np.isfinite(a).all()
    np.testing.assert_array_equal(a, b)
    z = torch.zeros_like(inp["gate1"])
    c, _ = _gpu_forward(name, inp, gate1=z, gate2=z)
    np.testing.assert_array_equal(c, inp["x"].float().numpy())


def test_host_buffer_entry_point_equals_the_device_one():
    # kl_joint_block_forward_host: x, modulation and out in pinned host memory,
    # copied on the stream around the same kernels -> the same bits
    name = "tiny"
    wl = WORKLOADS[name]
    inp = block_inputs(name)
    dev_out, _ = _gpu_forward(name, inp)
    d = {k: v.cuda() for k, v in inp.items()}
    W = kl.prepare_block_weights(d["wqkv"], d["wo"], d["w1"], d["w2"])
    cs = kl.rope_table(wl.n_text, wl.grid_h, wl.grid_w, wl.n_ref)
    x_h = inp["x"].pin_memory()
    mod_h = {n: inp[n].pin_memory() for n in MOD_NAMES}
    for _ in range(2):
        out_h = kl.joint_block_forward_host(W, x_h, mod_h, cs, wl.heads, wl.mlp_hidden, attn=wl.attn)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(out_h.float().numpy(), dev_out)
    assert kl.device_status() == "KL_OK"
