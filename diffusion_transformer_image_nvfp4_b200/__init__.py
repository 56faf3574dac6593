"""Thin Python binding of libklein.so (the NVFP4 joint-block CUDA library).

Argument marshalling only: every step of the block runs in the library's
sm_100a kernels.  Tensors are ``torch`` CUDA tensors (PyTorch supplies device
memory and the current stream); the calls mirror the C ABI in
``include/klein.h`` and keep its names (``kl_quantize_nvfp4`` ->
``quantize_nvfp4`` and so on).  There is no CPU or PyTorch fallback: if the
library is missing every call raises.
"""

import ctypes
import os
from dataclasses import dataclass

import torch

from .build import LIB_PATH

__all__ = [
    "KLError", "lib", "NVFP4", "quantize_nvfp4", "ln_modulate_quantize_nvfp4", "gemm_nvfp4_fused",
    "rope_table", "cast_fp8_per_head", "joint_attention", "BlockWeights", "prepare_block_weights",
    "DitShape", "DitWeights", "dit_step", "dit_workspace_size",
    "joint_block_forward", "block_workspace_size", "device_status", "scales_mma_to_linear",
]

KL_OK = 0
STATUS = {0: "KL_OK", 1: "KL_ERR_INVALID_ARG", 2: "KL_ERR_UNSUPPORTED_SHAPE", 3: "KL_ERR_MISALIGNED",
          4: "KL_ERR_WORKSPACE", 5: "KL_ERR_CUDA", 6: "KL_ERR_DEVICE_TIMEOUT", 7: "KL_ERR_ARCH",
          8: "KL_ERR_NONFINITE"}
KL_SCALE_LINEAR, KL_SCALE_MMA, KL_GLOBAL_SCALE_GIVEN, KL_ROWS_SWIGLU_INTERLEAVE, KL_AMAX_GIVEN = 0, 1, 2, 4, 8
EPI = {"none": 0, "qkv_rope": 1, "swiglu": 2, "gated_residual": 3}
KL_OUT_BF16, KL_OUT_F32 = 0, 1
ATTN = {"fp8": 0, "bf16": 1}


class KLError(RuntimeError):
    def __init__(self, status, where):
        msg = f"{where}: {STATUS.get(status, status)}"
        if status == 5 and _LIB is not None:
            msg += " (" + _LIB.kl_last_cuda_error().decode() + ")"
        super().__init__(msg)
        self.status = status


class _NVFP4Tensor(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("global_scale", ctypes.c_void_p)]


class _Epilogue(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("out_dtype", ctypes.c_int), ("out", ctypes.c_void_p),
                ("rope_cs", ctypes.c_void_p), ("gate", ctypes.c_void_p), ("residual", ctypes.c_void_p),
                ("amax_out", ctypes.c_void_p), ("tile", ctypes.c_int)]


class _TokenLayout(ctypes.Structure):
    _fields_ = [("n_text", ctypes.c_int64), ("grid_h", ctypes.c_int64), ("grid_w", ctypes.c_int64),
                ("n_ref", ctypes.c_int64)]


class _BlockWeights(ctypes.Structure):
    _fields_ = [("wqkv", _NVFP4Tensor), ("wo", _NVFP4Tensor), ("w1", _NVFP4Tensor), ("w2", _NVFP4Tensor)]


class _BlockIO(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("mod", ctypes.c_void_p * 6), ("rope_cs", ctypes.c_void_p),
                ("T", ctypes.c_int64), ("D", ctypes.c_int64), ("H", ctypes.c_int64), ("F", ctypes.c_int64),
                ("attn_precision", ctypes.c_int), ("out", ctypes.c_void_p),
                ("stage_events", ctypes.POINTER(ctypes.c_void_p)), ("sol_tau", ctypes.c_float),
                ("vc_budget", ctypes.c_float)]


class _DitShape(ctypes.Structure):
    _fields_ = [("n_text", ctypes.c_int64), ("grid_h", ctypes.c_int64), ("grid_w", ctypes.c_int64),
                ("channels", ctypes.c_int64), ("D", ctypes.c_int64), ("H", ctypes.c_int64), ("F", ctypes.c_int64),
                ("n_mode_blocks", ctypes.c_int), ("n_joint_blocks", ctypes.c_int), ("attn_precision", ctypes.c_int)]


class _DitWeights(ctypes.Structure):
    _fields_ = [("w_in", _NVFP4Tensor), ("mode_text", ctypes.POINTER(_BlockWeights)),
                ("mode_image", ctypes.POINTER(_BlockWeights)), ("joint", ctypes.POINTER(_BlockWeights)),
                ("w_out", _NVFP4Tensor)]


class _DitStepIO(ctypes.Structure):
    _fields_ = [("latent", ctypes.c_void_p), ("text", ctypes.c_void_p), ("mod_mode", ctypes.c_void_p),
                ("mod_joint", ctypes.c_void_p), ("mod_final", ctypes.c_void_p), ("rope_text", ctypes.c_void_p),
                ("rope_image", ctypes.c_void_p), ("rope_joint", ctypes.c_void_p), ("dt", ctypes.c_float),
                ("sol_tau", ctypes.c_float)]


class _DitViews(ctypes.Structure):
    _fields_ = [("tokens", ctypes.c_size_t), ("head_codes", ctypes.c_size_t), ("head_scales", ctypes.c_size_t),
                ("head_gs", ctypes.c_size_t), ("velocity", ctypes.c_size_t)]


class _DitCacheHeader(ctypes.Structure):
    _fields_ = [("num", ctypes.c_double), ("den", ctypes.c_double), ("diff", ctypes.c_float), ("hit", ctypes.c_int),
                ("has_ref", ctypes.c_int), ("hits", ctypes.c_int), ("steps", ctypes.c_int)]


_LIB = None
_VP, _I64, _I, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
_SIGS = {
    "kl_status_string": ([_I], ctypes.c_char_p),
    "kl_last_cuda_error": ([], ctypes.c_char_p),
    "kl_version": ([], _I),
    "kl_device_status": ([_I], _I),
    "kl_selftest_wait_timeout": ([ctypes.c_uint64, _VP, _VP], _I),
    "kl_nvfp4_scales_bytes": ([_I64, _I64, _I], _SZ),
    "kl_quantize_workspace_size": ([], _SZ),
    "kl_quantize_nvfp4": ([_VP, _I64, _I64, _VP, _VP, _VP, _I, _VP, _SZ, _VP], _I),
    "kl_ln_workspace_size": ([_I64], _SZ),
    "kl_amax_bf16": ([_VP, _I64, _VP, _VP], _I),
    "kl_ln_modulate_bf16": ([_VP, _I64, _I64, _VP, _VP, _VP, _VP, _VP, _SZ, _VP], _I),
    "kl_ln_modulate_quantize_nvfp4": ([_VP, _I64, _I64, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP], _I),
    "kl_ln_modulate_quantize_nvfp4_static": ([_VP, _I64, _I64, _VP, _VP, _VP, _VP, _VP, _VP, _VP], _I),
    "kl_gemm_nvfp4_fused": ([ctypes.POINTER(_NVFP4Tensor), ctypes.POINTER(_NVFP4Tensor), _I64, _I64, _I64,
                             ctypes.POINTER(_Epilogue), _VP], _I),
    "kl_layout_tokens": ([ctypes.POINTER(_TokenLayout)], _I64),
    "kl_rope_table": ([ctypes.POINTER(_TokenLayout), ctypes.c_float, _VP, _VP], _I),
    "kl_cast_fp8_per_head": ([_VP, _I64, _I64, _I64, _VP, _VP, _VP, _VP], _I),
    "kl_joint_attention_fp8": ([_VP, _VP, _VP, _I64, _VP, _VP, _VP, _I64, _I64, _I64, _I, _VP, _VP, _VP], _I),
    "kl_sol_list_ints": ([_I64, _I64, _I], _SZ),
    "kl_sol_workspace_size": ([_I64, _I64, _I], _SZ),
    "kl_sol_select": ([_VP, _VP, _I64, _VP, _VP, _I64, _I64, _I, ctypes.c_float, _VP, _VP, _SZ, _VP], _I),
    "kl_joint_attention_sparse": ([_VP, _VP, _VP, _I64, _VP, _VP, _VP, _I64, _I64, _I64, _I, _VP, _VP, _VP, _VP],
                                  _I),
    "kl_vc_workspace_size": ([_I64, _I64], _SZ),
    "kl_vc_select": ([_VP, _VP, _I64, _I64, _I64, ctypes.c_float, _VP, _VP, _VP, _SZ, _VP], _I),
    "kl_vc_attention_workspace_size": ([_I64, _I64], _SZ),
    "kl_joint_attention_vc": ([_VP, _VP, _VP, _I64, _VP, _VP, _VP, _VP, _VP, _VP, _I64, _I64, _I64, _I64, _VP, _VP,
                               _VP, _VP, _VP, _SZ, _VP], _I),
    "kl_block_workspace_size": ([_I64, _I64, _I64, _I64, _I], _SZ),
    "kl_joint_block_forward": ([ctypes.POINTER(_BlockWeights), ctypes.POINTER(_BlockIO), _VP, _SZ, _VP], _I),
    "kl_block_host_workspace_size": ([_I64, _I64, _I64, _I64, _I], _SZ),
    "kl_joint_block_forward_host": ([ctypes.POINTER(_BlockWeights), ctypes.POINTER(_BlockIO), _VP, _SZ, _VP], _I),
    "kl_dit_workspace_size": ([ctypes.POINTER(_DitShape)], _SZ),
    "kl_dit_workspace_views": ([ctypes.POINTER(_DitShape), ctypes.POINTER(_DitViews)], _I),
    "kl_dit_step": ([ctypes.POINTER(_DitShape), ctypes.POINTER(_DitWeights), ctypes.POINTER(_DitStepIO), _VP, _SZ,
                     _VP], _I),
    "kl_dit_cache_size": ([ctypes.POINTER(_DitShape)], _SZ),
    "kl_dit_cache_reset": ([_VP, _VP], _I),
    "kl_dit_step_cached": ([ctypes.POINTER(_DitShape), ctypes.POINTER(_DitWeights), ctypes.POINTER(_DitStepIO),
                            ctypes.c_float, _VP, _SZ, _VP, _SZ, _VP], _I),
}


def lib():
    """The loaded libklein.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m diffusion_transformer_image_nvfp4_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _LIB = L
    return _LIB


def _check(status, where):
    if status != KL_OK:
        raise KLError(status, where)


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _need(t, dtype, name):
    if not (t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor")


_WS = {}


def _workspace(nbytes, device, tag):
    key = (tag, device.index if device.index is not None else torch.cuda.current_device())
    buf = _WS.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        _WS[key] = buf
    return buf


# ---------------------------------------------------------------- NVFP4
@dataclass
class NVFP4:
    """An NVFP4 tensor: codes uint8 [R, C/2]; scales uint8 (linear [R, C/16] or
    MMA layout, padded to 128-row blocks); gs fp32 [1] decode global scale."""

    codes: torch.Tensor
    scales: torch.Tensor
    gs: torch.Tensor
    rows: int
    cols: int
    layout: str

    def abi(self):
        return _NVFP4Tensor(self.codes.data_ptr(), self.scales.data_ptr(), self.gs.data_ptr())


def quantize_nvfp4(x, layout="mma", global_scale=None, swiglu_interleave=False, amax_slot=None, out=None):
    """kl_quantize_nvfp4 on a contiguous CUDA bf16 [R, C] tensor.  ``amax_slot``
    (optional): a CUDA fp32 tensor of >= 64 elements, 16-byte aligned, whose
    first element holds the tensor's amax (KL_AMAX_GIVEN: e.g. a max reduced
    over ranks).  ``out`` (optional): an NVFP4 whose buffers are reused."""
    _need(x, torch.bfloat16, "x")
    R, C = x.shape
    L = lib()
    flags = KL_SCALE_MMA if layout == "mma" else KL_SCALE_LINEAR
    if out is not None:
        codes, scales, gs = out.codes, out.scales, out.gs
        if global_scale is not None or amax_slot is None:
            raise ValueError("out= is for the amax_slot form")
        flags |= KL_AMAX_GIVEN
        _check(L.kl_quantize_nvfp4(x.data_ptr(), R, C, codes.data_ptr(), scales.data_ptr(), gs.data_ptr(), flags,
                                   amax_slot.data_ptr(), amax_slot.numel() * 4, _stream()), "kl_quantize_nvfp4")
        return out
    codes = torch.empty((R, C // 2), dtype=torch.uint8, device=x.device)
    scales = torch.empty(L.kl_nvfp4_scales_bytes(R, C, flags & 1), dtype=torch.uint8, device=x.device)
    if amax_slot is not None:
        flags |= KL_AMAX_GIVEN
        gs = torch.empty(1, dtype=torch.float32, device=x.device)
        _check(L.kl_quantize_nvfp4(x.data_ptr(), R, C, codes.data_ptr(), scales.data_ptr(), gs.data_ptr(), flags,
                                   amax_slot.data_ptr(), amax_slot.numel() * 4, _stream()), "kl_quantize_nvfp4")
        return NVFP4(codes, scales, gs, R, C, layout)
    if global_scale is not None:
        flags |= KL_GLOBAL_SCALE_GIVEN
        gs = torch.as_tensor(global_scale, dtype=torch.float32, device=x.device).reshape(1).clone()
    else:
        gs = torch.empty(1, dtype=torch.float32, device=x.device)
    if swiglu_interleave:
        flags |= KL_ROWS_SWIGLU_INTERLEAVE
    ws = _workspace(L.kl_quantize_workspace_size(), x.device, "quant")
    _check(L.kl_quantize_nvfp4(x.data_ptr(), R, C, codes.data_ptr(), scales.data_ptr(), gs.data_ptr(), flags,
                               ws.data_ptr(), ws.numel(), _stream()), "kl_quantize_nvfp4")
    if layout != "mma":
        scales = scales.view(R, C // 16)
    return NVFP4(codes, scales, gs, R, C, layout)


def ln_modulate_quantize_nvfp4(x, shift, scale, export_m=False):
    """kl_ln_modulate_quantize_nvfp4: NVFP4 of bf16(LN(x)(1+scale)+shift)."""
    for t, n in ((x, "x"), (shift, "shift"), (scale, "scale")):
        _need(t, torch.bfloat16, n)
    R, C = x.shape
    L = lib()
    codes = torch.empty((R, C // 2), dtype=torch.uint8, device=x.device)
    scales = torch.empty(L.kl_nvfp4_scales_bytes(R, C, KL_SCALE_MMA), dtype=torch.uint8, device=x.device)
    gs = torch.empty(1, dtype=torch.float32, device=x.device)
    m = torch.empty_like(x) if export_m else None
    ws = _workspace(L.kl_ln_workspace_size(R), x.device, "ln")
    _check(L.kl_ln_modulate_quantize_nvfp4(x.data_ptr(), R, C, shift.data_ptr(), scale.data_ptr(), codes.data_ptr(),
                                           scales.data_ptr(), gs.data_ptr(), _ptr(m), ws.data_ptr(), ws.numel(),
                                           _stream()), "kl_ln_modulate_quantize_nvfp4")
    q = NVFP4(codes, scales, gs, R, C, "mma")
    return (q, m) if export_m else q


def amax_bf16(x, out=None):
    """kl_amax_bf16: max|x| of a contiguous CUDA bf16 tensor (numel % 8 == 0)."""
    _need(x, torch.bfloat16, "x")
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=x.device)
    _check(lib().kl_amax_bf16(x.data_ptr(), x.numel(), out.data_ptr(), _stream()), "kl_amax_bf16")
    return out


def ln_modulate_bf16(x, shift, scale, m_out=None, amax_out=None):
    """kl_ln_modulate_bf16: m = bf16(LN(x)(1+scale)+shift) and max|m|
    max-accumulated into amax_out (zero-filled here when not given)."""
    for t, n in ((x, "x"), (shift, "shift"), (scale, "scale")):
        _need(t, torch.bfloat16, n)
    R, C = x.shape
    L = lib()
    if m_out is None:
        m_out = torch.empty_like(x)
    if amax_out is None:
        amax_out = torch.zeros(1, dtype=torch.float32, device=x.device)
    ws = _workspace(L.kl_ln_workspace_size(R), x.device, "ln")
    _check(L.kl_ln_modulate_bf16(x.data_ptr(), R, C, shift.data_ptr(), scale.data_ptr(), m_out.data_ptr(),
                                 amax_out.data_ptr(), ws.data_ptr(), ws.numel(), _stream()), "kl_ln_modulate_bf16")
    return m_out, amax_out


def ln_modulate_quantize_nvfp4_static(x, shift, scale, export_m=False):
    """kl_ln_modulate_quantize_nvfp4_static: as ln_modulate_quantize_nvfp4, but
    the library's scratch comes from its own fixed device array (no workspace)."""
    for t, n in ((x, "x"), (shift, "shift"), (scale, "scale")):
        _need(t, torch.bfloat16, n)
    R, C = x.shape
    L = lib()
    codes = torch.empty((R, C // 2), dtype=torch.uint8, device=x.device)
    scales = torch.empty(L.kl_nvfp4_scales_bytes(R, C, KL_SCALE_MMA), dtype=torch.uint8, device=x.device)
    gs = torch.empty(1, dtype=torch.float32, device=x.device)
    m = torch.empty_like(x) if export_m else None
    _check(L.kl_ln_modulate_quantize_nvfp4_static(x.data_ptr(), R, C, shift.data_ptr(), scale.data_ptr(),
                                                  codes.data_ptr(), scales.data_ptr(), gs.data_ptr(), _ptr(m),
                                                  _stream()), "kl_ln_modulate_quantize_nvfp4_static")
    q = NVFP4(codes, scales, gs, R, C, "mma")
    return (q, m) if export_m else q


GEMM_TILES = {"auto": 0, "1cta_128x128": 1, "1cta_128x256": 2, "2sm_256x128": 3, "2sm_256x256": 4}


def gemm_nvfp4_fused(A, W, epilogue="none", out=None, out_dtype=torch.bfloat16, rope_cs=None, gate=None,
                     residual=None, amax=None, tile="auto"):
    """kl_gemm_nvfp4_fused: C = gA gW dec(A) dec(W)^T with a fused epilogue.

    tile: "auto" or one of GEMM_TILES (forces an output-tile variant)."""
    if A.layout != "mma" or W.layout != "mma" or A.cols != W.cols:
        raise ValueError("operands must share K and use the MMA scale layout")
    M, N, K = A.rows, W.rows, A.cols
    kind = EPI[epilogue]
    if out is None:
        cols = N // 2 if kind == EPI["swiglu"] else N
        out = torch.empty((M, cols), dtype=out_dtype, device=A.codes.device)
    epi = _Epilogue(kind, KL_OUT_F32 if out.dtype == torch.float32 else KL_OUT_BF16, out.data_ptr(), _ptr(rope_cs),
                    _ptr(gate), _ptr(residual), _ptr(amax), GEMM_TILES[tile])
    a, w = A.abi(), W.abi()
    _check(lib().kl_gemm_nvfp4_fused(ctypes.byref(a), ctypes.byref(w), M, N, K, ctypes.byref(epi), _stream()),
           "kl_gemm_nvfp4_fused")
    return out


def rope_table(n_text, grid_h, grid_w, n_ref=0, theta=10000.0, device="cuda"):
    """kl_rope_table: fp32 (cos, sin) [16, T, 4, 2] (groups of 4 pairs) for the joint sequence."""
    lay = _TokenLayout(n_text, grid_h, grid_w, n_ref)
    T = lib().kl_layout_tokens(ctypes.byref(lay))
    cs = torch.empty((16, T, 4, 2), dtype=torch.float32, device=device)
    _check(lib().kl_rope_table(ctypes.byref(lay), theta, cs.data_ptr(), _stream()), "kl_rope_table")
    return cs


def cast_fp8_per_head(x, amax, ncols=None, ld=None):
    """kl_cast_fp8_per_head: (E4M3 bytes like x, fp32 decode scales [ncols/128])."""
    T = x.shape[0]
    ld = x.shape[1] if ld is None else ld
    ncols = x.shape[1] if ncols is None else ncols
    out = torch.zeros(x.shape, dtype=torch.uint8, device=x.device)
    sc = torch.empty(ncols // 128, dtype=torch.float32, device=x.device)
    _check(lib().kl_cast_fp8_per_head(x.data_ptr(), T, ncols, ld, amax.data_ptr(), out.data_ptr(), sc.data_ptr(),
                                      _stream()), "kl_cast_fp8_per_head")
    return out, sc


def joint_attention(q, k, v, T, H, ld, precision="fp8", sq=None, sk=None, sv=None, amax=None, out=None):
    """kl_joint_attention_fp8 on [T, H, 128] views with row stride ld elements
    (q, k, v are tensors whose data_ptr is the first element of each)."""
    if out is None:
        out = torch.empty((T, H * 128), dtype=torch.bfloat16, device=q.device)
    _check(lib().kl_joint_attention_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), ld, _ptr(sq), _ptr(sk), _ptr(sv),
                                        T, H, 128, ATTN[precision], out.data_ptr(), _ptr(amax), _stream()),
           "kl_joint_attention_fp8")
    return out


SOL_QUERY_ROWS = {"fp8": 256, "bf16": 128}


def sol_select(q, k, T, H, ld, tau, precision="fp8", sq=None, sk=None):
    """kl_sol_select: Sol-Attention key-tile lists (int32 [H, n_qb, n_kt + 1]:
    count, then the kept tile indices in ascending order)."""
    n = lib().kl_sol_list_ints(T, H, ATTN[precision])
    nqb = -(-T // SOL_QUERY_ROWS[precision])
    nkt = -(-T // 128)
    assert n == H * nqb * (nkt + 1)
    lst = torch.zeros(n, dtype=torch.int32, device=q.device)
    need = lib().kl_sol_workspace_size(T, H, ATTN[precision])
    ws = _workspace(need, q.device, "sol")
    _check(lib().kl_sol_select(q.data_ptr(), k.data_ptr(), ld, _ptr(sq), _ptr(sk), T, H, ATTN[precision], float(tau),
                               lst.data_ptr(), ws.data_ptr(), ws.numel(), _stream()), "kl_sol_select")
    return lst.view(H, nqb, nkt + 1)


def joint_attention_sparse(q, k, v, T, H, ld, kv_list, precision="fp8", sq=None, sk=None, sv=None, amax=None,
                           out=None):
    """kl_joint_attention_sparse: joint_attention over the key tiles of
    ``kv_list`` (the layout sol_select returns)."""
    if out is None:
        out = torch.empty((T, H * 128), dtype=torch.bfloat16, device=q.device)
    _need(kv_list, torch.int32, "kv_list")
    _check(lib().kl_joint_attention_sparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), ld, _ptr(sq), _ptr(sk),
                                           _ptr(sv), T, H, 128, ATTN[precision], kv_list.data_ptr(), out.data_ptr(),
                                           _ptr(amax), _stream()), "kl_joint_attention_sparse")
    return out


def vc_select(q, k, T, H, ld, budget):
    """kl_vc_select on bf16 q, k: (list_fp8 int32 [H, ceil(T/256), n_kt + 1]
    of the tiles that are not repaired, list_bf16 int32 [H, ceil(T/128), n_kt +
    1] of the repaired ones), each row the count then ascending tile indices."""
    nkt = -(-T // 128)
    l8 = torch.zeros((H, -(-T // 256), nkt + 1), dtype=torch.int32, device=q.device)
    l16 = torch.zeros((H, -(-T // 128), nkt + 1), dtype=torch.int32, device=q.device)
    ws = _workspace(lib().kl_vc_workspace_size(T, H), q.device, "vc")
    _check(lib().kl_vc_select(q.data_ptr(), k.data_ptr(), ld, T, H, float(budget), l8.data_ptr(), l16.data_ptr(),
                              ws.data_ptr(), ws.numel(), _stream()), "kl_vc_select")
    return l8, l16


def joint_attention_vc(q8, k8, v8, ld8, sq, sk, sv, q, k, v, ld, T, H, list_fp8, list_bf16, amax=None, out=None):
    """kl_joint_attention_vc: FP8 attention (E4M3 q8, k8, v8 with per-head
    scales) with the pairs of list_bf16 computed from the bf16 q, k, v."""
    if out is None:
        out = torch.empty((T, H * 128), dtype=torch.bfloat16, device=q8.device)
    ws = _workspace(lib().kl_vc_attention_workspace_size(T, H), q8.device, "vc_att")
    _check(lib().kl_joint_attention_vc(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), ld8, sq.data_ptr(), sk.data_ptr(),
                                       sv.data_ptr(), q.data_ptr(), k.data_ptr(), v.data_ptr(), ld, T, H, 128,
                                       list_fp8.data_ptr(), list_bf16.data_ptr(), out.data_ptr(), _ptr(amax),
                                       ws.data_ptr(), ws.numel(), _stream()), "kl_joint_attention_vc")
    return out


# ---------------------------------------------------------------- block
@dataclass
class BlockWeights:
    wqkv: NVFP4
    wo: NVFP4
    w1: NVFP4   # SwiGLU-interleaved rows
    w2: NVFP4

    def abi(self):
        return _BlockWeights(self.wqkv.abi(), self.wo.abi(), self.w1.abi(), self.w2.abi())


def prepare_block_weights(wqkv, wo, w1, w2):
    """NVFP4-encode bf16 block weights (W1 rows SwiGLU-interleaved) on the GPU."""
    return BlockWeights(quantize_nvfp4(wqkv), quantize_nvfp4(wo), quantize_nvfp4(w1, swiglu_interleave=True),
                        quantize_nvfp4(w2))


def block_workspace_size(T, D, H, F, attn="fp8"):
    return lib().kl_block_workspace_size(T, D, H, F, ATTN[attn])


BLOCK_STAGES = ("ln1", "qkv_gemm", "fp8_cast", "attention", "quant_o", "out_gemm", "ln2", "mlp_up_gemm",
                "quant_h", "mlp_down_gemm")


def joint_block_forward(weights, x, mod, rope_cs, H, F, attn="fp8", out=None, workspace=None, stage_events=None,
                        sol_tau=0.0, vc_budget=0.0):
    """kl_joint_block_forward.  ``mod`` maps shift1, scale1, gate1, shift2,
    scale2, gate2 to bf16 [D] CUDA tensors.  ``stage_events`` (optional): a list
    of len(BLOCK_STAGES)+1 recorded torch.cuda.Event(enable_timing=True); the
    library re-records them around each stage on the current stream.
    ``sol_tau`` > 0: Sol-Attention tile skipping at that threshold.
    ``vc_budget`` > 0: VC-Attention repair of that fraction of the FP8 tile pairs."""
    _need(x, torch.bfloat16, "x")
    T, D = x.shape
    names = ("shift1", "scale1", "gate1", "shift2", "scale2", "gate2")
    for n in names:
        _need(mod[n], torch.bfloat16, n)
    if out is None:
        out = torch.empty_like(x)
    need = block_workspace_size(T, D, H, F, attn)
    if workspace is None:
        workspace = _workspace(need, x.device, "block")
    ev = None
    if stage_events is not None:
        if len(stage_events) != len(BLOCK_STAGES) + 1:
            raise ValueError("stage_events: need one event per stage plus one")
        ev = (ctypes.c_void_p * len(stage_events))(*[e.cuda_event for e in stage_events])
    io = _BlockIO(x.data_ptr(), (ctypes.c_void_p * 6)(*[mod[n].data_ptr() for n in names]), rope_cs.data_ptr(),
                  T, D, H, F, ATTN[attn], out.data_ptr(), ctypes.cast(ev, ctypes.POINTER(ctypes.c_void_p)),
                  float(sol_tau), float(vc_budget))
    w = weights.abi()
    _check(lib().kl_joint_block_forward(ctypes.byref(w), ctypes.byref(io), workspace.data_ptr(), workspace.numel(),
                                        _stream()), "kl_joint_block_forward")
    return out


def joint_block_forward_host(weights, x_host, mod_host, rope_cs, H, F, attn="fp8", out_host=None, workspace=None,
                             device=None):
    """kl_joint_block_forward_host: ``x_host`` and the six ``mod_host`` vectors
    are CPU bf16 tensors (pin them for asynchronous copies); the output comes
    back into ``out_host`` (a CPU bf16 tensor, allocated if None) when the
    current stream reaches the end of the call."""
    if x_host.is_cuda or x_host.dtype != torch.bfloat16 or not x_host.is_contiguous():
        raise ValueError("x_host: expected a contiguous CPU bf16 tensor")
    T, D = x_host.shape
    names = ("shift1", "scale1", "gate1", "shift2", "scale2", "gate2")
    for n in names:
        t = mod_host[n]
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{n}: expected a contiguous CPU bf16 tensor")
    if out_host is None:
        out_host = torch.empty_like(x_host, pin_memory=x_host.is_pinned())
    device = rope_cs.device if device is None else device
    need = lib().kl_block_host_workspace_size(T, D, H, F, ATTN[attn])
    if workspace is None:
        workspace = _workspace(need, device, "block_host")
    io = _BlockIO(x_host.data_ptr(), (ctypes.c_void_p * 6)(*[mod_host[n].data_ptr() for n in names]),
                  rope_cs.data_ptr(), T, D, H, F, ATTN[attn], out_host.data_ptr(), None, 0.0, 0.0)
    w = weights.abi()
    _check(lib().kl_joint_block_forward_host(ctypes.byref(w), ctypes.byref(io), workspace.data_ptr(),
                                             workspace.numel(), _stream()), "kl_joint_block_forward_host")
    return out_host


# ------------------------------------------------------------------ DiT step
@dataclass
class DitShape:
    n_text: int
    grid_h: int
    grid_w: int
    channels: int
    D: int
    H: int
    F: int
    n_mode_blocks: int
    n_joint_blocks: int
    attn: str = "fp8"

    def abi(self):
        return _DitShape(self.n_text, self.grid_h, self.grid_w, self.channels, self.D, self.H, self.F,
                         self.n_mode_blocks, self.n_joint_blocks, ATTN[self.attn])


@dataclass
class DitWeights:
    w_in: NVFP4            # [D, 4*channels]
    mode_text: list        # [n_mode_blocks] BlockWeights
    mode_image: list       # [n_mode_blocks] BlockWeights
    joint: list            # [n_joint_blocks] BlockWeights
    w_out: NVFP4           # [4*channels, D]

    def abi(self):
        def arr(blocks):
            if not blocks:
                return None
            return (_BlockWeights * len(blocks))(*[b.abi() for b in blocks])
        # keep the ctypes arrays alive with the struct
        self._arrays = (arr(self.mode_text), arr(self.mode_image), arr(self.joint))
        ptr = lambda a: ctypes.cast(a, ctypes.POINTER(_BlockWeights)) if a is not None else None
        return _DitWeights(self.w_in.abi(), ptr(self._arrays[0]), ptr(self._arrays[1]), ptr(self._arrays[2]),
                           self.w_out.abi())


def dit_workspace_size(shape):
    sh = shape.abi()
    return lib().kl_dit_workspace_size(ctypes.byref(sh))


def dit_step(shape, weights, latent, text, mod_mode, mod_joint, mod_final, rope_text, rope_image, rope_joint, dt,
             workspace=None, w_abi=None, sol_tau=0.0):
    """kl_dit_step: one Euler step, latent (fp32 [2gh, 2gw, C], CUDA) updated in
    place.  mod_mode bf16 [n_mode, 2, 6, D]; mod_joint bf16 [n_joint, 6, D];
    mod_final bf16 [2, D]; rope tables from rope_table for the text-only,
    image-only and joint layouts.  ``w_abi`` (optional): a cached
    weights.abi() (the ctypes struct), to keep host work out of loops."""
    _need(latent, torch.float32, "latent")
    _need(text, torch.bfloat16, "text")
    sh = shape.abi()
    need = lib().kl_dit_workspace_size(ctypes.byref(sh))
    if workspace is None:
        workspace = _workspace(need, latent.device, "dit")
    w = weights.abi() if w_abi is None else w_abi
    io = _DitStepIO(latent.data_ptr(), text.data_ptr(), _ptr(mod_mode), _ptr(mod_joint), mod_final.data_ptr(),
                    rope_text.data_ptr(), rope_image.data_ptr(), rope_joint.data_ptr(), float(dt), float(sol_tau))
    _check(lib().kl_dit_step(ctypes.byref(sh), ctypes.byref(w), ctypes.byref(io), workspace.data_ptr(),
                             workspace.numel(), _stream()), "kl_dit_step")
    return latent


def dit_views(shape, workspace):
    """kl_dit_workspace_views as torch views into a kl_dit_step workspace
    (uint8 CUDA tensor): tokens bf16 [T, D], head_codes uint8 [Ti, D/2],
    head_scales uint8 (KL_SCALE_MMA layout), head_gs fp32 [1], velocity fp32
    [Ti, 4C].  Valid after an uncached dit_step on that workspace."""
    sh = shape.abi()
    v = _DitViews()
    _check(lib().kl_dit_workspace_views(ctypes.byref(sh), ctypes.byref(v)), "kl_dit_workspace_views")
    Ti, T, D, K = shape.grid_h * shape.grid_w, shape.n_text + shape.grid_h * shape.grid_w, shape.D, 4 * shape.channels
    nsc = lib().kl_nvfp4_scales_bytes(Ti, D, KL_SCALE_MMA)

    def view(off, n, dtype):
        return workspace[off:off + n * torch.tensor([], dtype=dtype).element_size()].view(dtype)

    return {"tokens": view(v.tokens, T * D, torch.bfloat16).view(T, D),
            "head_codes": view(v.head_codes, Ti * D // 2, torch.uint8).view(Ti, D // 2),
            "head_scales": view(v.head_scales, nsc, torch.uint8),
            "head_gs": view(v.head_gs, 1, torch.float32),
            "velocity": view(v.velocity, Ti * K, torch.float32).view(Ti, K)}


class DitCache:
    """Device state of kl_dit_step_cached (Cache-DiT) for one generation:
    a kl_dit_cache_header followed by F bf16 [T, D], r_cur, r_ref and R fp32
    [T, D], each at a 256-byte boundary.  reset() before every generation."""

    def __init__(self, shape, device=None):
        sh = shape.abi()
        n = lib().kl_dit_cache_size(ctypes.byref(sh))
        if n == 0:
            raise KLError(2, "kl_dit_cache_size")
        self.shape = shape
        self.buf = torch.empty(n, dtype=torch.uint8, device=device or torch.device("cuda"))
        self.reset()

    def reset(self):
        _check(lib().kl_dit_cache_reset(self.buf.data_ptr(), _stream()), "kl_dit_cache_reset")

    def header(self):
        """The header as a dict (copies it to the host: synchronising)."""
        raw = bytes(self.buf[:ctypes.sizeof(_DitCacheHeader)].cpu().numpy().tobytes())
        h = _DitCacheHeader.from_buffer_copy(raw)
        return {f: getattr(h, f) for f, _ in _DitCacheHeader._fields_}

    def arrays(self):
        """Views F (bf16), r_cur, r_ref, R (fp32), each [T, D]."""
        s = self.shape
        n = (s.n_text + s.grid_h * s.grid_w) * s.D
        up = lambda b: (b + 255) // 256 * 256
        off = up(ctypes.sizeof(_DitCacheHeader))
        out = {}
        for name, dt, es in (("F", torch.bfloat16, 2), ("r_cur", torch.float32, 4), ("r_ref", torch.float32, 4),
                             ("R", torch.float32, 4)):
            out[name] = self.buf[off:off + n * es].view(dt).view(-1, s.D)
            off += up(n * es)
        return out


def dit_step_cached(shape, weights, cache, threshold, latent, text, mod_mode, mod_joint, mod_final, rope_text,
                    rope_image, rope_joint, dt, workspace=None, w_abi=None, sol_tau=0.0):
    """kl_dit_step_cached: dit_step with Cache-DiT step caching at
    ``threshold`` (the residual-difference threshold; 0 never reuses), state
    in ``cache`` (a DitCache).  Eager calls synchronise the stream once to read
    the decision; under CUDA graph capture the decision stays on the device."""
    _need(latent, torch.float32, "latent")
    _need(text, torch.bfloat16, "text")
    sh = shape.abi()
    need = lib().kl_dit_workspace_size(ctypes.byref(sh))
    if workspace is None:
        workspace = _workspace(need, latent.device, "dit")
    w = weights.abi() if w_abi is None else w_abi
    io = _DitStepIO(latent.data_ptr(), text.data_ptr(), _ptr(mod_mode), _ptr(mod_joint), mod_final.data_ptr(),
                    rope_text.data_ptr(), rope_image.data_ptr(), rope_joint.data_ptr(), float(dt), float(sol_tau))
    _check(lib().kl_dit_step_cached(ctypes.byref(sh), ctypes.byref(w), ctypes.byref(io), float(threshold),
                                    cache.buf.data_ptr(), cache.buf.numel(), workspace.data_ptr(), workspace.numel(),
                                    _stream()), "kl_dit_step_cached")
    return latent


def device_status(clear=True):
    """kl_device_status: synchronises and returns the status name."""
    return STATUS.get(lib().kl_device_status(1 if clear else 0), "?")


def selftest_wait_timeout(limit_ns, waited=None):
    """kl_selftest_wait_timeout: one warp waits on an mbarrier nothing arrives
    on, with a bounded wait of ``limit_ns``; ``waited`` (optional CUDA int32
    [1]) receives 0 when the wait gave up.  Asynchronous on the current stream."""
    if waited is not None:
        _need(waited, torch.int32, "waited")
    _check(lib().kl_selftest_wait_timeout(int(limit_ns), _ptr(waited), _stream()), "kl_selftest_wait_timeout")


def scales_mma_to_linear(scales, rows, cols):
    """Reorder a KL_SCALE_MMA scale buffer into the linear [rows, cols/16]
    layout (index arithmetic of the documented layout; no arithmetic on values)."""
    r = torch.arange(rows, device=scales.device)[:, None]
    kb = torch.arange(cols // 16, device=scales.device)[None, :]
    off = ((r // 128) * (cols // 64) + kb // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + kb % 4
    return scales.reshape(-1)[off]
