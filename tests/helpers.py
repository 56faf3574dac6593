"""Shared test helpers (comparison metrics and host-side reshaping only)."""

import numpy as np
import torch


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def to_np(t):
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu()
        if t.dtype == torch.bfloat16:
            t = t.float()
        return t.numpy()
    return np.asarray(t)


def f32_bits(x):
    return np.asarray(x, np.float32).view(np.uint32)


def swiglu_perm(rows):
    """Source row of each output row under the KL_ROWS_SWIGLU_INTERLEAVE order
    (each 128-row group = 64 gate rows then the matching 64 up rows)."""
    r = np.arange(rows)
    g, i = r // 128, r % 128
    return np.where(i < 64, g * 64 + i, rows // 2 + g * 64 + (i - 64))
