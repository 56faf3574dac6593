"""VC-Attention repair of FP8 attention, plain fp64 reading (TEST
INFRASTRUCTURE ONLY: imported by tests/, never by the library).

What the pages fix: [P1] "Optimizing FLUX 3 Image Klein inference on NVIDIA
Blackwell GPUs", How it works -- the quantized attention takes Q, K and V in
FP8, and VC-Attention adds a repair budget that corrects quantization errors;
Key details -- a repair budget of 0.005; What you can do -- the vc_attention
switch and vc_repair_budget.

Readings (the pages give no more):
* the unit of repair is the FP8 attention's tile pair, as for Sol-Attention:
  a query block of 256 rows against a key tile of 128 keys, per head;
* a budget b repairs R = floor(b * n_qb * n_kt) of a head's n_qb * n_kt
  pairs (none when that is 0; all of them at b = 1);
* the pairs repaired are those with the largest estimated share of their
  query block's attention: with the block means qbar_b, kbar_j of the bf16 q
  and k (valid rows only), s_hat(b, j) = (qbar_b . kbar_j) log2(e)/sqrt(d)
  and w(b, j) = 2^(s_hat(b, j) - max_j') / sum_j' 2^(s_hat(b, j') - max_j');
  equal shares go to the lower (b, j) in row-major order.  The FP8 rounding
  error a tile adds to the output is about proportional to the attention mass
  it carries, so the budget goes where it removes the most error;
* a repaired pair is computed from the bf16 q, k, v, the values before the
  E4M3 cast: a query block's output is the softmax over all keys, combined
  from the FP8 pass over its other tiles (``block.fp8_flash_rows``, the FP8
  reading, with the per-head scales over all tokens) and an exact pass over
  its repaired tiles, merged exactly: O = (O_8 W_8 + O_16 W_16) / (W_8 +
  W_16), W the unnormalised softmax mass sum_keys 2^t of each part.
"""

import numpy as np

from .block import fp8_encode_heads, fp8_flash_rows
from .sparse import LOG2E, block_means


def vc_weights(q, k, q_block=256, tile=128):
    """w [H, n_qb, n_kt]: each key tile's estimated share of its query
    block's attention, from block means of the bf16 q and k."""
    qb = block_means(q, q_block)
    kb = block_means(k, tile)
    d = np.asarray(q).shape[2]
    s_hat = np.einsum("hqd,hkd->hqk", qb, kb) * (LOG2E / np.sqrt(d))
    e = np.exp2(s_hat - s_hat.max(axis=2, keepdims=True))
    return e / e.sum(axis=2, keepdims=True)


def vc_select(q, k, budget, q_block=256, tile=128):
    """repaired [H, n_qb, n_kt] (bool): per head the R = floor(budget * n_qb *
    n_kt) pairs with the largest w, ties to the lower (b, j)."""
    w = vc_weights(q, k, q_block, tile)
    H, nqb, nkt = w.shape
    R = int(np.floor(budget * nqb * nkt))
    rep = np.zeros(w.shape, dtype=bool)
    for h in range(H):
        order = np.argsort(-w[h].reshape(-1), kind="stable")   # descending, lower index first on ties
        rep[h].reshape(-1)[order[:R]] = True
    return rep


def exact_part(q, k, v, cols):
    """The exact softmax part of rows q [R, d] over keys ``cols``: (O [R, d],
    m [R], l [R]) with O normalised and l * 2^m = sum over cols of 2^t,
    t = (q . k) log2(e)/sqrt(d)."""
    q = np.asarray(q, np.float64)
    d = q.shape[1]
    t = (q @ np.asarray(k, np.float64)[cols].T) * (LOG2E / np.sqrt(d))
    m = t.max(axis=1)
    p = np.exp2(t - m[:, None])
    l = p.sum(axis=1)
    return (p @ np.asarray(v, np.float64)[cols]) / l[:, None], m, l


def merge_parts(parts):
    """Softmax of the union from parts (O, m, l) over disjoint key sets:
    O = sum_i O_i l_i 2^(m_i - M) / sum_i l_i 2^(m_i - M), M = max_i m_i."""
    M = np.max([m for _, m, _ in parts], axis=0)
    num = sum(O * (l * np.exp2(m - M))[:, None] for O, m, l in parts)
    den = sum(l * np.exp2(m - M) for _, m, l in parts)
    return num / den[:, None]


def attention_vc(q, k, v, repaired, q_block=256, tile=128, p_scale=16.0, tau=4.0):
    """FP8 joint attention with the pairs of ``repaired`` [H, n_qb, n_kt]
    computed exactly from the bf16 values; q, k, v [T, H, d]."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    q8, sq = fp8_encode_heads(q)
    k8, sk = fp8_encode_heads(k)
    v8, sv = fp8_encode_heads(v)
    T, H, d = q.shape
    out = np.empty((T, H, d))
    for h in range(H):
        c = LOG2E / np.sqrt(d) * float(sq[h]) * float(sk[h])
        for b in range(repaired.shape[1]):
            rows = np.arange(b * q_block, min((b + 1) * q_block, T))
            fix = np.flatnonzero(repaired[h, b])
            keep = np.flatnonzero(~repaired[h, b])
            parts = []
            if len(keep):
                acc, l, m = fp8_flash_rows(q8[rows, h], k8[:, h], v8[:, h], c, keep, tile=tile, p_scale=p_scale,
                                           tau=tau, return_m=True)
                parts.append((acc * float(sv[h]) / (p_scale * l[:, None]), m, l))
            if len(fix):
                cols = np.concatenate([np.arange(j * tile, min((j + 1) * tile, T)) for j in fix])
                parts.append(exact_part(q[rows, h], k[:, h], v[:, h], cols))
            out[rows, h] = merge_parts(parts)
    return out
