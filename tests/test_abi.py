"""CPU-only checks of the C ABI: the library loads, exports every function
that include/klein.h declares, and its host-side validation / size logic
answers without touching a GPU."""

import ctypes
import os
import re

import pytest

import diffusion_transformer_image_nvfp4_b200 as kl
from diffusion_transformer_image_nvfp4_b200 import build

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "klein.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b(kl_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


@pytest.fixture(scope="module")
def L():
    build.build()
    return kl.lib()


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert "kl_joint_block_forward" in names and "kl_quantize_nvfp4" in names
    assert "kl_gemm_nvfp4_fused" in names and "kl_joint_attention_fp8" in names
    for n in names:
        assert hasattr(L, n), n
    # and the binding declares a signature for each
    assert set(names) <= set(kl._SIGS)


def test_status_strings_and_version(L):
    assert L.kl_status_string(0) == b"KL_OK"
    assert L.kl_status_string(6) == b"KL_ERR_DEVICE_TIMEOUT"
    assert L.kl_status_string(99) == b"KL_ERR_UNKNOWN"
    assert L.kl_version() >= 100


def test_scale_and_workspace_sizes(L):
    assert L.kl_nvfp4_scales_bytes(320, 512, kl.KL_SCALE_LINEAR) == 320 * 32
    assert L.kl_nvfp4_scales_bytes(320, 512, kl.KL_SCALE_MMA) == 384 * 32      # padded to 128 rows
    assert L.kl_quantize_workspace_size() >= 4
    ws = L.kl_block_workspace_size(8704, 3072, 24, 9216, 0)
    T, D, F = 8704, 3072, 9216
    assert ws >= T * 3 * D * 2 + T * 3 * D + 2 * T * D * 2 + T * F * 2 + T * F // 2
    assert L.kl_block_workspace_size(8704, 3072, 24, 9216, 1) < ws            # no FP8 copy in BF16 mode
    assert L.kl_block_workspace_size(0, 3072, 24, 9216, 0) == 0
    host = L.kl_block_host_workspace_size(T, D, 24, F, 0)
    assert host >= ws + 2 * T * D * 2 + 6 * D * 2                             # + x, out, modulation
    assert L.kl_block_host_workspace_size(0, 3072, 24, 9216, 0) == 0


def test_layout_tokens(L):
    lay = kl._TokenLayout(512, 64, 64, 1)
    assert L.kl_layout_tokens(ctypes.byref(lay)) == 8704
    lay = kl._TokenLayout(512, 64, 64, 4)
    assert L.kl_layout_tokens(ctypes.byref(lay)) == 20992
    lay = kl._TokenLayout(-1, 64, 64, 0)
    assert L.kl_layout_tokens(ctypes.byref(lay)) == -1


def test_validation_rejects_bad_arguments_before_any_device_work(L):
    # null pointers
    assert L.kl_quantize_nvfp4(None, 4, 64, None, None, None, 0, None, 0, None) == 1
    fake = 1 << 20   # never dereferenced: every call below fails validation first
    # unsupported shapes
    assert L.kl_quantize_nvfp4(fake, 4, 24, fake, fake, fake, 0, fake, 256, None) == 2
    assert L.kl_quantize_nvfp4(fake, 4, 80, fake, fake, fake, kl.KL_SCALE_MMA, fake, 256, None) == 2
    assert L.kl_quantize_nvfp4(fake, 100, 64, fake, fake, fake, kl.KL_ROWS_SWIGLU_INTERLEAVE, fake, 256, None) == 2
    # misaligned input
    assert L.kl_quantize_nvfp4(fake + 2, 4, 64, fake, fake, fake, 0, fake, 256, None) == 3
    # missing workspace when gs is derived
    assert L.kl_quantize_nvfp4(fake, 4, 64, fake, fake, fake, 0, None, 0, None) == 4
    # bad flag bits
    assert L.kl_quantize_nvfp4(fake, 4, 64, fake, fake, fake, 64, fake, 256, None) == 1
    # GEMM shape and epilogue checks
    t = kl._NVFP4Tensor(fake, fake, fake)
    epi = kl._Epilogue(0, 0, fake, None, None, None, None)
    assert L.kl_gemm_nvfp4_fused(ctypes.byref(t), ctypes.byref(t), 128, 100, 64, ctypes.byref(epi), None) == 2
    assert L.kl_gemm_nvfp4_fused(ctypes.byref(t), ctypes.byref(t), 128, 128, 96, ctypes.byref(epi), None) == 2
    epi_q = kl._Epilogue(1, 0, fake, None, None, None, None)
    assert L.kl_gemm_nvfp4_fused(ctypes.byref(t), ctypes.byref(t), 128, 384, 64, ctypes.byref(epi_q), None) == 1
    epi_bad = kl._Epilogue(9, 0, fake, None, None, None, None)
    assert L.kl_gemm_nvfp4_fused(ctypes.byref(t), ctypes.byref(t), 128, 128, 64, ctypes.byref(epi_bad), None) == 1
    # attention
    assert L.kl_joint_attention_fp8(fake, fake, fake, 3072, None, None, None, 100, 24, 128, 0, fake, None, None) == 1
    assert L.kl_joint_attention_fp8(fake, fake, fake, 3072, fake, fake, fake, 100, 24, 64, 0, fake, None, None) == 2
    assert L.kl_joint_attention_fp8(fake, fake, fake, 3072, fake, fake, fake, 100, 24, 128, 7, fake, None, None) == 1
    # block: D must be 128 * H
    io = kl._BlockIO(fake, (ctypes.c_void_p * 6)(*([fake] * 6)), fake, 100, 3000, 24, 9216, 0, fake + 4096)
    w = kl._BlockWeights(t, t, t, t)
    assert L.kl_joint_block_forward(ctypes.byref(w), ctypes.byref(io), fake, 1 << 40, None) == 2
    io.D = 3072
    io.out = fake
    assert L.kl_joint_block_forward(ctypes.byref(w), ctypes.byref(io), fake, 1 << 40, None) == 1  # out aliases x
    io.out = fake + 4096
    assert L.kl_joint_block_forward(ctypes.byref(w), ctypes.byref(io), fake, 16, None) == 4     # workspace


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(kl, "_LIB", None)
    monkeypatch.setattr(kl, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        kl.lib()


def test_dit_cache_size_and_cached_step_validation(L):
    up = lambda b: (b + 255) // 256 * 256
    assert ctypes.sizeof(kl._DitCacheHeader) == 40
    sh = kl._DitShape(16, 4, 4, 32, 128, 1, 384, 1, 2, 1)
    T, D = 16 + 4 * 4, 128
    # header, then F bf16 and r_cur, r_ref, R fp32, each [T, D] at 256-byte boundaries
    assert L.kl_dit_cache_size(ctypes.byref(sh)) == 256 + up(T * D * 2) + 3 * up(T * D * 4)
    none = kl._DitShape(16, 4, 4, 32, 128, 1, 384, 0, 0, 1)
    assert L.kl_dit_cache_size(ctypes.byref(none)) == 0
    fake = 1 << 20   # never dereferenced: every call below fails validation first
    t = kl._NVFP4Tensor(fake, fake, fake)
    blocks = (kl._BlockWeights * 2)(kl._BlockWeights(t, t, t, t), kl._BlockWeights(t, t, t, t))
    bp = ctypes.cast(blocks, ctypes.POINTER(kl._BlockWeights))
    w = kl._DitWeights(t, bp, bp, bp, t)
    io = kl._DitStepIO(fake, fake, fake, fake, fake, fake, fake, fake, -0.0625)
    ws = L.kl_dit_workspace_size(ctypes.byref(sh))
    need = L.kl_dit_cache_size(ctypes.byref(sh))
    step = lambda shape, cache, nbytes: L.kl_dit_step_cached(ctypes.byref(shape), ctypes.byref(w), ctypes.byref(io),
                                                             0.24, cache, nbytes, fake, ws, None)
    assert step(sh, None, need) == 1           # no cache
    assert step(sh, fake, need - 1) == 4       # cache too small
    assert step(sh, fake + 16, need) == 3      # cache not 256-byte aligned
    assert step(none, fake, need) == 2         # no block to probe
    assert L.kl_dit_cache_reset(None, None) == 1
    assert L.kl_dit_cache_reset(fake + 8, None) == 3


def test_sol_sizes_and_validation(L):
    T, H = 4608, 24
    nqb8, nqb16, nkt = 18, 36, 36
    assert L.kl_sol_list_ints(T, H, 0) == H * nqb8 * (nkt + 1)      # FP8: 256-row query blocks
    assert L.kl_sol_list_ints(T, H, 1) == H * nqb16 * (nkt + 1)     # BF16: 128-row query blocks
    assert L.kl_sol_workspace_size(T, H, 0) == H * (nqb8 + nkt) * 128 * 4
    assert L.kl_sol_list_ints(0, H, 0) == 0 and L.kl_sol_workspace_size(T, H, 7) == 0
    fake = 1 << 20
    ws = L.kl_sol_workspace_size(T, H, 0)
    sel = lambda tau, lst=fake, wsb=ws, sq=fake: L.kl_sol_select(fake, fake, 3 * H * 128, sq, sq, T, H, 0, tau, lst,
                                                                 fake, wsb, None)
    assert sel(float("nan")) == 1 and sel(-1.0) == 1           # tau must be >= 0
    assert sel(1.0, sq=None) == 1                                # FP8 needs scales
    assert sel(1.0, lst=None) == 1
    assert sel(1.0, wsb=ws - 1) == 4
    assert sel(1.0, lst=fake + 2) == 3
    assert L.kl_sol_select(fake + 1, fake, 3 * H * 128, fake, fake, T, H, 0, 1.0, fake, fake, ws, None) == 3
    assert L.kl_sol_select(fake, fake, 3 * H * 128 + 4, fake, fake, T, H, 0, 1.0, fake, fake, ws, None) == 2
    att = lambda lst, hd=128: L.kl_joint_attention_sparse(fake, fake, fake, 3 * H * 128, fake, fake, fake, T, H, hd, 0,
                                                          lst, fake, None, None)
    assert att(None) == 1 and att(fake, hd=64) == 2 and att(fake + 1) == 3


def test_sequence_parallel_pieces_validation(L):
    fake = 1 << 20
    assert L.kl_amax_bf16(None, 64, fake, None) == 1
    assert L.kl_amax_bf16(fake, 7, fake, None) == 2          # whole 16-byte vectors only
    assert L.kl_amax_bf16(fake + 2, 64, fake, None) == 3
    ws = L.kl_ln_workspace_size(100)
    ln = lambda cols, wsb=ws, m=fake: L.kl_ln_modulate_bf16(fake, 100, cols, fake, fake, m, fake, fake, wsb, None)
    assert ln(320) == 2 and ln(1280) == 2 and ln(5120) == 2  # widths / 256 in {1, 2, 4, 8, 12, 16} only
    assert ln(512, m=None) == 1
    assert ln(512, wsb=ws - 1) == 4
    # KL_AMAX_GIVEN and KL_GLOBAL_SCALE_GIVEN exclude each other
    assert L.kl_quantize_nvfp4(fake, 4, 64, fake, fake, fake, kl.KL_AMAX_GIVEN | kl.KL_GLOBAL_SCALE_GIVEN, fake,
                               256, None) == 1
    assert L.kl_quantize_nvfp4(fake, 4, 64, fake, fake, fake, kl.KL_AMAX_GIVEN, None, 0, None) == 4


def test_selftest_limit_is_checked_before_any_device_work(L):
    assert L.kl_selftest_wait_timeout(0, None, None) == 1              # KL_ERR_INVALID_ARG
    assert L.kl_selftest_wait_timeout(2_000_000_000, None, None) == 1
    assert L.kl_selftest_wait_timeout(1_000_000, ctypes.c_void_p(2), None) == 3   # misaligned flag


def test_dit_workspace_views_lie_inside_the_workspace(L):
    sh = kl._DitShape(64, 16, 16, 32, 3072, 24, 9216, 1, 2, kl.ATTN["fp8"])
    v = kl._DitViews()
    assert L.kl_dit_workspace_views(ctypes.byref(sh), ctypes.byref(v)) == 0
    size = L.kl_dit_workspace_size(ctypes.byref(sh))
    T, Ti, D, K = 64 + 256, 256, 3072, 128
    assert v.tokens + T * D * 2 <= size and v.velocity + Ti * K * 4 <= size
    assert v.head_codes + Ti * D // 2 <= v.head_scales and v.head_gs % 4 == 0
    assert all(x % 16 == 0 for x in (v.tokens, v.head_codes, v.head_scales, v.velocity))
    # three blocks ping-pong from the first token buffer and end in the second
    sh2 = kl._DitShape(64, 16, 16, 32, 3072, 24, 9216, 1, 1, kl.ATTN["fp8"])
    v2 = kl._DitViews()
    assert L.kl_dit_workspace_views(ctypes.byref(sh2), ctypes.byref(v2)) == 0
    assert v2.tokens != v.tokens
    assert L.kl_dit_workspace_views(None, ctypes.byref(v)) == 1


def test_vc_argument_checks(L):
    fake = ctypes.c_void_p(1 << 20)
    assert L.kl_vc_workspace_size(4608, 24) > 0 and L.kl_vc_workspace_size(0, 24) == 0
    assert L.kl_vc_attention_workspace_size(4608, 24) >= 2 * 4608 * 24 * 8 + 4608 * 24 * 128 * 4
    ws = L.kl_vc_workspace_size(1000, 2)
    sel = lambda budget: L.kl_vc_select(fake, fake, 768, 1000, 2, budget, fake, fake, fake, ws, None)
    assert sel(float("nan")) == 1 and sel(-0.1) == 1 and sel(1.5) == 1          # KL_ERR_INVALID_ARG
    assert L.kl_vc_select(fake, fake, 100, 1000, 2, 0.1, fake, fake, fake, ws, None) == 2   # ld too small
    assert L.kl_vc_select(fake, fake, 768, 1000, 2, 0.1, fake, fake, fake, ws - 1, None) == 4  # workspace
