"""CPU oracle for the FLUX-3-Image-Klein-style NVFP4 joint transformer block.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA path (``diffusion_transformer_image_nvfp4_b200``) and
imports nothing from it; the two meet only in the seeded input generators of
the ``synth`` package, which hold none of the method's arithmetic.

The oracle is the plain definition of what the block computes, written for a
reader to check by eye:

* ``codecs``  -- exact E2M1 / E4M3 / bf16 rounding (round-to-nearest-even,
  satfinite), by enumerating the representable values.
* ``nvfp4``   -- the NVFP4 block-scaled encoding (16-element blocks, one
  unsigned E4M3 scale per block, one fp32 per-tensor scale) and its decode.
* ``block``   -- LayerNorm + adaLN modulation, 1D / axial RoPE, the NVFP4 GEMM
  (fp64 over decoded operands), joint softmax attention (fp64) and the whole
  joint-block forward with its gated residuals and SwiGLU MLP.

Sources.  The pages describing the method are
  [P1] "Optimizing FLUX 3 Image Klein inference on NVIDIA Blackwell GPUs"
       (sections "What happened", "How it works", "Key details");
  [P2] "FLUX.3 Image Klein Brings 2-Second AI Image Generation to Diffusers"
       (section "Summary");
  [P4] "Welcome FLUX.3 Image Klein in Diffusers"
       (section "Architecture and Technical Deep Dive": "The VAE and
       Tokenization", "Two-Stage Processing").
The pages name NVFP4 weights/activations, GEMMs with fused SwiGLU and rotary
embeddings, FP8 Q/K/V attention, and joint attention over concatenated text /
noisy-image / reference tokens, but they do not spell out the NVFP4 encoding,
the block wiring (LayerNorm, adaLN, gates) or the RoPE axes.  Every such step
below is a stated reading; each function's docstring says which.

Parity status.  Every function here is pinned by ``tests/test_oracle_*.py``
against something other than itself (library codecs, closed forms,
invariants, brute force, PyTorch fp64 routines) except where a docstring says
"parity unpinned".
"""

from . import codecs, nvfp4, block  # noqa: F401

__all__ = ["codecs", "nvfp4", "block"]
