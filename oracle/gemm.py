"""Block-scaled FP4 GEMM over dequantised operands (oracle; test infrastructure).

Definition: Y = X_hat W_hat^T, where X_hat, W_hat are the dequantised NVFP4
operands (``oracle.nvfp4.dequantize``) and the products are summed in FP64.
This is what every W4A4 projection of the layer computes ("Why Gated DeltaNet
Survives 4-Bit Quantization", section "Performance and Efficiency Gains": all
496 linear layers, gate projections included, run with 4-bit weights and
activations).  ``numpy.matmul`` in FP64 is the library primitive for the sum.

The bf16 result is the nearest-even bf16 of the FP64 sum (one rounding).
"""
import numpy as np

from .nvfp4 import dequantize, round_bf16


def gemm_fp64(a_q, b_q):
    """a_q, b_q: dicts from ``oracle.nvfp4.quantize`` ([M,K] and [N,K]).
    Returns the FP64 product [M, N]."""
    xa = dequantize(a_q["codes"], a_q["scales"], a_q["g"])
    xb = dequantize(b_q["codes"], b_q["scales"], b_q["g"])
    return np.matmul(xa, xb.T)


def gemm_bf16(a_q, b_q):
    """The FP64 product rounded once to bf16 (returned as FP64 values)."""
    return round_bf16(gemm_fp64(a_q, b_q))
