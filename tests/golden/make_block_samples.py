"""Write the oracle's expected block outputs for the multi-reference
workloads, on a fixed sample of output rows (TEST DATA GENERATOR: calls only
the oracle and the seeded input generators).

The 20,992- and 21,504-token blocks are too large to recompute with the fp64
oracle inside a GPU test run, so this script runs ``oracle.block.block_forward``
once per workload and attention mode on the full workload (every token takes
part in the attention and in every per-tensor scale) and stores the bf16 bit
patterns of the sampled rows of the output:

    python tests/golden/make_block_samples.py [workload ...]

Output: tests/golden/block_samples_<workload>.npz with
  rows   int64 [R]        the sampled token indices (ascending)
  exact  uint16 [R, D]    output rows, oracle attention "exact" (fp64 softmax)
  fp8    uint16 [R, D]    output rows, oracle attention "fp8" (E4M3 emulation)
"""

import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from oracle import block, codecs  # noqa: E402
from synth import MOD_NAMES, WORKLOADS, block_inputs  # noqa: E402

N_ROWS = 256


def sample_rows(wl, n=N_ROWS, seed=1234):
    """A fixed row sample: the first and last token of every segment (text,
    noisy image, each reference) and random tokens to make up n."""
    seg = [0, wl.n_text] + [wl.n_text + (k + 1) * wl.grid_h * wl.grid_w for k in range(wl.n_ref + 1)]
    must = set()
    for a, b in zip(seg[:-1], seg[1:]):
        must.update((a, b - 1))
    rng = np.random.default_rng(seed)
    rest = [r for r in rng.permutation(wl.n_tokens) if r not in must][: n - len(must)]
    return np.array(sorted(must | set(int(r) for r in rest)), dtype=np.int64)


def path_for(name):
    return os.path.join(HERE, f"block_samples_{name}.npz")


def main(names):
    for name in names:
        wl = WORKLOADS[name]
        inp = {k: v.float().numpy() for k, v in block_inputs(name).items()}
        lay = block.TokenLayout(wl.n_text, wl.grid_h, wl.grid_w, wl.n_ref)
        rows = sample_rows(wl)
        res = {"rows": rows}
        for attn in ("exact", "fp8"):
            out = block.block_forward(inp["x"], {k: inp[k] for k in MOD_NAMES}, inp, lay, wl.heads, attn=attn)
            res[attn] = codecs.bf16_bits(out[rows])
            print(f"{name} {attn}: done", flush=True)
        np.savez_compressed(path_for(name), **res)


if __name__ == "__main__":
    main(sys.argv[1:] or ["multiref_1024", "multiref_21504"])
