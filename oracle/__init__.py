"""CPU oracle for the SVDQuant W4A4 linear layer (TEST INFRASTRUCTURE ONLY).

This package is the plain, slow, obviously-correct restatement of what the
layer computes, written from the Nunchaku/SVDQuant pages:

  * "Nunchaku und SVDQuant" (mind-verse.de, Nunchaku 4-bit in Diffusers):
    the main layers run with 4-bit weights and activations (W4A4);
    activation outliers are moved into the weights; the hardest part of each
    weight matrix is carried by a small 16-bit low-rank branch; the rest is
    quantised to 4 bits.
  * same page, "Native Ladefunktion": the svdq_w4a4 config block names
    precision nvfp4, group_size 16, rank 32; the awq block names int4 with
    group_size 64.
  * charmloop.ai news item, second paragraph: the low-rank down-projection
    is fused into the quantisation kernel and the up-projection into the
    4-bit compute kernel.

Every step is written out in fp64 (or in fp32 where the step is defined as
an fp32 rounding) with numpy; library primitives (matmul, SVD) serve as steps.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may
import this package.  The CUDA product path never does, and this package
never imports the product: the two share only the seeded input generators
in `synth`.

Modules:
  formats  - RNE rounding to bf16 / fp16 / E4M3 / E2M1, codecs, nibble packing
  quant    - the NVFP4 group-16 and INT4 group-64 quantisers
  svd      - truncated SVD (LAPACK for small, subspace iteration for large)
  svdq     - smoothing factor, weight preparation, activation quantisation
             with lora-down, and the fp64 forward
  qkv      - the attention prologue of the fused QKV projection (per-head
             RMS normalisation of Q and K, rotary embedding)
  awq      - the awq_w4a16 layer (INT4 group-64 weights, 16-bit activations)
  chain    - the dynamic activation tensor scale and chained layers (an
             activation between them, the next layer's amax)
"""
from . import awq, chain, formats, qkv, quant, svd, svdq  # noqa: F401
