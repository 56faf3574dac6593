"""NVFP4 block-scaled encoding, plain reading (TEST INFRASTRUCTURE ONLY).

[P1] "Optimizing FLUX 3 Image Klein inference on NVIDIA Blackwell GPUs",
§How it works / §Key details: weights and activations of the diffusion
transformer are quantised to NVFP4 so the GPU "processes more data per
cycle".  The page does not define the encoding; this module fixes the
reading used by the whole library:

* elements are E2M1 (magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}, plus sign);
* every 16 consecutive elements of a row share one unsigned E4M3 scale ``sb``;
* one fp32 per-tensor decode scale ``gs``;
* decoded value = e2m1(code) * e4m3(sb) * gs.

Encoding, every operation one IEEE fp32 operation rounded to nearest even
(numpy float32 arithmetic; no FMA, no flush-to-zero, correctly rounded
division):

1. ``amax_t`` = max |x| over the tensor (exact).
2. ``gs`` = 1 if amax_t == 0 else amax_t / 2688   (2688 = 6 * 448, so that the
   largest block scale lands at the top of the E4M3 range).
3. ``d6`` = 6 * gs; ``inv`` = 1 / d6.
4. per block: ``amax_b`` = max |x_i|; ``sb`` = e4m3_rne_satfinite(amax_b * inv),
   except ``sb`` = 0 when amax_b == 0 (so 0 * inf never arises when ``inv``
   overflows for a tensor of subnormal-sized values).
5. ``S`` = e4m3(sb) * gs; if S == 0 all 16 codes are 0.
6. otherwise ``r`` = 1 / S and code_i = e2m1_rne_satfinite(x_i * r); a negative
   x_i whose magnitude rounds to 0 keeps its sign (code 0x8).
7. packing: element 2i in the low nibble of byte i, element 2i+1 in the high
   nibble.

Readings that the pages leave open and this module fixes: the stored global
scale is the *decode* scale (not 2688 / amax); the element scaling is a
multiply by the rounded reciprocal 1/S (not a divide by S); the all-zero
cases above.
"""

import numpy as np

from .codecs import e2m1_decode, e2m1_encode, e4m3_decode, e4m3_encode

BLOCK = 16
E2M1_MAX = np.float32(6.0)
E4M3_MAX = np.float32(448.0)
GS_DIVISOR = np.float32(6.0 * 448.0)        # 2688


def global_scale(x):
    """Decode global scale gs of a tensor (steps 1-2), as float32."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x))) if x.size else np.float32(0.0)
    if amax == 0:
        return np.float32(1.0)
    with np.errstate(under="ignore"):
        return np.float32(amax / GS_DIVISOR)


def quantize(x, gs=None):
    """Encode a bf16-valued array [R, C] (C % 16 == 0) to NVFP4.

    ``x`` holds bf16 values as float32 (or anything exactly convertible).
    ``gs`` optionally fixes the global decode scale (float32); by default it is
    derived from the tensor's amax (step 2).

    Returns ``(codes, scales, gs)``: codes uint8 [R, C/2] (packed pairs),
    scales uint8 [R, C/16] (unsigned E4M3, row-major "linear" layout),
    gs float32.
    """
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    if x.ndim != 2 or x.shape[1] % BLOCK:
        raise ValueError("quantize: expected [R, C] with C a multiple of 16")
    R, C = x.shape
    gs = global_scale(x) if gs is None else np.float32(gs)
    # rows are independent once gs is fixed: encode in row chunks (memory only)
    step = max(1, (1 << 20) // max(C, 1))
    if R > step:
        parts = [_quantize_rows(x[r:r + step], gs) for r in range(0, R, step)]
        return (np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts]), np.float32(gs))
    return _quantize_rows(x, gs)


def _quantize_rows(x, gs):
    """Steps 3-7 for the rows of x with the global scale gs already fixed."""
    R, C = x.shape
    with np.errstate(over="ignore", divide="ignore", under="ignore", invalid="ignore"):
        d6 = np.float32(E2M1_MAX * gs)
        inv = np.float32(np.float32(1.0) / d6)
        xb = x.reshape(R, C // BLOCK, BLOCK)
        amax_b = np.max(np.abs(xb), axis=2)                       # exact
        sv = (amax_b * inv).astype(np.float32)                    # fp32 multiply
        sb = np.where(amax_b > 0, e4m3_encode(np.where(amax_b > 0, sv, 0.0)), 0).astype(np.uint8)
        S = (e4m3_decode(sb).astype(np.float32) * gs).astype(np.float32)
        nz = S != 0
        r = np.where(nz, np.float32(1.0) / np.where(nz, S, np.float32(1.0)), np.float32(0.0)).astype(np.float32)
        y = (xb * r[:, :, None]).astype(np.float32)               # fp32 multiply
    codes = e2m1_encode(y)
    codes = np.where(nz[:, :, None], codes, 0).astype(np.uint8)
    codes = codes.reshape(R, C)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, sb, np.float32(gs)


def unpack_codes(packed):
    """Unpack [R, C/2] bytes to [R, C] 4-bit codes (low nibble first)."""
    packed = np.asarray(packed, dtype=np.uint8)
    R, half = packed.shape
    out = np.empty((R, 2 * half), dtype=np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out


def dequantize(packed, scales, gs):
    """Decoded fp64 values e2m1(code) * e4m3(sb) * gs, shape [R, C] (exact)."""
    codes = unpack_codes(packed)
    R, C = codes.shape
    vals = e2m1_decode(codes).reshape(R, C // BLOCK, BLOCK)
    sc = e4m3_decode(scales).astype(np.float64)[:, :, None]
    return (vals * sc * np.float64(gs)).reshape(R, C)
