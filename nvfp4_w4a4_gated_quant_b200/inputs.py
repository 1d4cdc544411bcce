"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module holds no arithmetic of the method: it only draws random numbers
in a fixed, documented order and rounds activations to bf16 storage.  Every
array is returned as numpy (bf16 values carried in float32 arrays, exact).

Workloads (shapes and distributions of the 27B-hybrid GDN layer the pages
describe; the pages measure on trained weights and real text, which these
synthetic draws stand in for):

  tiny      B=1, T=64, d_model=256, H=2, d=32, seed 0
  gemm      X 8192x5120 (0.1% outliers x50), W 12288x5120, seed 1
  scan      B=1, T=32768, H=16, d=128, seed 2
  layer     B=4, T=8192, d_model=5120, H=32, d=128, seed 3
  replay    12 x T=32768, H=16, d=128, seed 4

Draw order inside one generator (numpy default_rng(seed)):
  activations  x ~ N(0,1) (float32 draw), then round(0.001 * numel) outlier
               positions without replacement, those entries x50, then bf16;
  weights      q, k, v, a, b, out in that order, each N(0, 0.02) float32;
  gates        A_log ~ U(lo, hi) per head, then dt_bias (U(lo, hi) or 0);
  scan only    q, k, v ~ N(0,1) -> bf16, then a, b ~ N(0,1) float32, then
               A_log, dt_bias.
"""
import numpy as np
import torch

OUTLIER_FRACTION = 0.001
OUTLIER_GAIN = 50.0
WEIGHT_STD = 0.02


def to_bf16_values(a):
    """Round a float32 array to bf16 storage; return it as float32 values."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def activations(rng, shape, outliers=True):
    x = rng.standard_normal(shape, dtype=np.float32)
    if outliers:
        n_out = int(round(OUTLIER_FRACTION * x.size))
        if n_out:
            idx = rng.choice(x.size, n_out, replace=False)
            flat = x.reshape(-1)
            flat[idx] *= np.float32(OUTLIER_GAIN)
    return to_bf16_values(x)


def weight(rng, rows, cols):
    return (rng.standard_normal((rows, cols), dtype=np.float32) * np.float32(WEIGHT_STD)).astype(np.float32)


def layer_inputs(B, T, d_model, H, dk, dv, seed, A_range=(-2.0, 1.0), dt_range=(-1.0, 1.0)):
    """Inputs of one layer forward.  ``dt_range`` None means dt_bias = 0."""
    rng = np.random.default_rng(seed)
    x = activations(rng, (B, T, d_model))
    W = {
        "q": weight(rng, H * dk, d_model),
        "k": weight(rng, H * dk, d_model),
        "v": weight(rng, H * dv, d_model),
        "a": weight(rng, H, d_model),
        "b": weight(rng, H, d_model),
        "out": weight(rng, d_model, H * dv),
    }
    A_log = rng.uniform(A_range[0], A_range[1], H).astype(np.float32)
    if dt_range is None:
        dt_bias = np.zeros(H, np.float32)
    else:
        dt_bias = rng.uniform(dt_range[0], dt_range[1], H).astype(np.float32)
    return {"x": x, "W": W, "A_log": A_log, "dt_bias": dt_bias,
            "B": B, "T": T, "d_model": d_model, "H": H, "dk": dk, "dv": dv}


def gemm_inputs(M, N, K, seed):
    """X [M, K] bf16 with outliers (quantized on the fly), W [N, K] float32."""
    rng = np.random.default_rng(seed)
    x = activations(rng, (M, K))
    w = weight(rng, N, K)
    return {"x": x, "w": w}


def scan_inputs(B, T, H, dk, dv, seed, A_range=(-2.0, 1.0), dt_range=(-1.0, 1.0)):
    """q, k, v [B, T, H, d] bf16 N(0,1); gate pre-activations a, b [B, T, H]."""
    rng = np.random.default_rng(seed)
    q = to_bf16_values(rng.standard_normal((B, T, H, dk), dtype=np.float32))
    k = to_bf16_values(rng.standard_normal((B, T, H, dk), dtype=np.float32))
    v = to_bf16_values(rng.standard_normal((B, T, H, dv), dtype=np.float32))
    a = rng.standard_normal((B, T, H), dtype=np.float32)
    b = rng.standard_normal((B, T, H), dtype=np.float32)
    A_log = rng.uniform(A_range[0], A_range[1], H).astype(np.float32)
    dt_bias = rng.uniform(dt_range[0], dt_range[1], H).astype(np.float32)
    return {"q": q, "k": k, "v": v, "a": a, "b": b, "A_log": A_log, "dt_bias": dt_bias}


def tiny_layer():
    return layer_inputs(1, 64, 256, 2, 32, 32, seed=0, A_range=(-1.0, 1.0), dt_range=None)


def gemm_workload():
    return gemm_inputs(8192, 12288, 5120, seed=1)


def scan_workload(T=32768):
    return scan_inputs(1, T, 16, 128, 128, seed=2)


def layer_workload(B=4, T=8192):
    return layer_inputs(B, T, 5120, 32, 128, 128, seed=3)
