"""Plain CPU oracle for the NVFP4 W4A4 Gated DeltaNet layer forward.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code, tables or constants with the CUDA library under
``nvfp4_w4a4_gated_quant_b200/csrc``; both sides only receive the same seeded
inputs.

Sources.  The method comes from the pages "Why Gated DeltaNet Survives 4-Bit
Quantization: NVFP4 W4A4 for the Recurrent Half of a Hybrid 27B LLM"
(franklineh.com research summary, section "Why the 'Fragile' Recurrence is
Actually Robust": NVFP4 block scaling over groups of 16) and "Anthology of the
SOTA, theory-128" (section "The account": the gated delta rule and its gate
parameterisation).  The element / scale formats (E2M1 values, one E4M3 scale
per 16 elements, one FP32 per-tensor scale) are the ones the benchmark spec
fixes for NVFP4.

Precision.  The quantizer is defined in IEEE FP32 with round-to-nearest-even,
one operation at a time (numpy float32 scalars/arrays).  Everything else is
FP64.  Where a step is a plain definition (a GEMM over dequantised operands) the
oracle is that definition, with ``numpy.matmul`` as the library primitive.

Modules
  nvfp4       E2M1 / E4M3 encode+decode, the two-level NVFP4 quantizer, dequant
  gemm        FP64 GEMM over dequantised operands, bf16 rounding of the result
  gates       decay gate log(alpha) and write strength beta
  delta_rule  sequential gated delta rule (the literal recurrence) and the
              chunked (UT / WY) form, both FP64
  layer       the four steps composed into one layer forward (optionally
              with the short convolution and the gated output norm)
  conv_norm   the short causal convolution + SiLU and the gated RMSNorm of
              the Gated DeltaNet block (outside specification)
  replay      clean vs NVFP4 trajectories of the recurrent state, the decay
              of an impulse, gate-noise and gate-error-compression arms (the
              pages' robustness measurements)

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, brute force, hand-worked examples or independent
library routines; ``layer.layer_forward`` by a hand-worked two-token layer.
Two things are "parity unpinned": the values the replay harness reports (the
pages' figures come from trained layers and real text; the harness itself is
pinned), and the composition of the layer's optional convolution and output
gate (each step is pinned; their wiring has no hand-worked example).
"""
