"""Sol-Attention tile skipping, plain fp64 reading (TEST INFRASTRUCTURE ONLY:
imported by tests/, never by the library).

What the pages fix: [P1] "Optimizing FLUX 3 Image Klein inference on NVIDIA
Blackwell GPUs", How it works -- sparse attention (Sol-Attention) leaves out
the computation of less important token pairs, chosen by a sparsity
threshold; What you can do / Key details -- a ``tau`` parameter, and a number
of initial denoising steps that stay dense (12 or 16).

Readings (the pages give nothing further; the same readings as the
library's kl_sol_select / kl_joint_attention_sparse):
* pairs are skipped a whole tile at a time: a query block (the rows one
  attention CTA owns: 256 with FP8 inputs, 128 with BF16) against a key tile
  of 128 keys, so the skipped work is whole tensor-core tiles;
* a pair's importance is estimated from the block means: s_hat = c * (qbar .
  kbar), qbar the mean of the block's query rows, kbar the mean of the tile's
  key rows (valid rows only at a ragged end), c the kernel's log2 score scale
  (log2(e)/sqrt(d), times the per-head E4M3 scales sq * sk with FP8 inputs,
  which then pools the unscaled E4M3 values);
* a key tile is kept for a query block when s_hat >= max over tiles - tau,
  i.e. its estimated softmax weight is at least 2^-tau of the strongest
  tile's; the strongest tile is always kept; tau = +inf keeps every tile;
* attention over the kept tiles is the usual softmax restricted to their
  keys (the FP8 kernel's tile-by-tile steps, visiting the kept tiles in
  ascending order).
"""

import numpy as np

from .block import attention, fp8_encode_heads, fp8_flash_rows

LOG2E = np.log2(np.e)


def block_means(x, rows_per_block):
    """Means of consecutive row blocks of x [T, H, d] -> [H, n_blocks, d]
    (the last block over its valid rows only)."""
    x = np.asarray(x, np.float64)
    T, H, d = x.shape
    nb = -(-T // rows_per_block)
    out = np.empty((H, nb, d))
    for b in range(nb):
        out[:, b, :] = x[b * rows_per_block:(b + 1) * rows_per_block].mean(axis=0)
    return out


def sol_select(q, k, c_head, tau, q_block, tile=128):
    """keep [H, n_qb, n_kt] (bool) and s_hat [H, n_qb, n_kt] (fp64).

    q, k: [T, H, d] values the scores are formed from; c_head: [H] log2 score
    scale per head; tau: the threshold in log2 units (>= 0, inf = dense)."""
    qb = block_means(q, q_block)
    kb = block_means(k, tile)
    c = np.asarray(c_head, np.float64)
    s_hat = np.einsum("hqd,hkd->hqk", qb, kb) * c[:, None, None]
    keep = s_hat >= s_hat.max(axis=2, keepdims=True) - tau
    return keep, s_hat


def kept_key_rows(keep_row, T, tile=128):
    """Key indices of the kept tiles (ascending)."""
    idx = [np.arange(j * tile, min((j + 1) * tile, T)) for j in np.flatnonzero(keep_row)]
    return np.concatenate(idx) if idx else np.zeros(0, dtype=np.int64)


def attention_sparse_exact(q, k, v, keep, q_block, tile=128):
    """fp64 softmax attention of each query block over its kept key tiles."""
    q = np.asarray(q, np.float64)
    T, H, d = q.shape
    out = np.empty((T, H, d))
    for h in range(H):
        for b in range(keep.shape[1]):
            rows = np.arange(b * q_block, min((b + 1) * q_block, T))
            cols = kept_key_rows(keep[h, b], T, tile)
            o, _ = attention(q[rows][:, h:h + 1], np.asarray(k)[cols][:, h:h + 1], np.asarray(v)[cols][:, h:h + 1])
            out[rows, h] = o[:, 0]
    return out


def attention_fp8_emulated_sparse(q, k, v, keep, q_block, tile=128, p_scale=16.0, tau=4.0):
    """The FP8 reading of ``block.attention_fp8_emulated`` (E4M3 Q/K/V with
    per-head scales over all tokens, ``block.fp8_flash_rows``) with each query
    block visiting only its kept key tiles, in ascending order."""
    q8, sq = fp8_encode_heads(q)
    k8, sk = fp8_encode_heads(k)
    v8, sv = fp8_encode_heads(v)
    T, H, d = q8.shape
    out = np.empty((T, H, d))
    for h in range(H):
        c = LOG2E / np.sqrt(d) * float(sq[h]) * float(sk[h])
        for b in range(keep.shape[1]):
            rows = np.arange(b * q_block, min((b + 1) * q_block, T))
            acc, l = fp8_flash_rows(q8[rows, h, :], k8[:, h, :], v8[:, h, :], c, np.flatnonzero(keep[h, b]),
                                    tile=tile, p_scale=p_scale, tau=tau)
            out[rows, h, :] = acc * float(sv[h]) / (p_scale * l[:, None])
    return out


def fp8_select_inputs(q, k):
    """The values and per-head scale the FP8 path selects from: the unscaled
    E4M3 values of q and k and c_h = log2(e)/sqrt(d) * sq_h * sk_h."""
    q8, sq = fp8_encode_heads(q)
    k8, sk = fp8_encode_heads(k)
    d = q8.shape[2]
    return q8, k8, LOG2E / np.sqrt(d) * sq.astype(np.float64) * sk.astype(np.float64)
