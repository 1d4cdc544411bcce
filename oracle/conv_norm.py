"""Short causal convolution and gated output norm of a Gated DeltaNet block
(oracle; test infrastructure).

The pages name "the convolution" only as an alternative explanation and define
neither it nor an output gate.  These two pieces follow the outside
specification of the Gated DeltaNet block (Yang, Kautz and Hatamizadeh,
"Gated Delta Networks: Improving Mamba2 with Delta Rule", ICLR 2025, the GDN
block): q, k and v each pass through a short causal depthwise convolution over
tokens followed by SiLU before q and k are L2-normalised; the recurrence's
output is RMS-normalised per head and gated by SiLU of a sixth projection
g = x W_g before the output projection.  FP64 throughout.

Readings where that specification leaves a choice:
  * kernel width 4; the window of token t holds tokens t-3 .. t, the oldest
    first (weight column j multiplies token t-3+j); tokens before the first
    one come from a carried state (the last three inputs of the previous
    call) or are zero;
  * SiLU(x) = x * sigmoid(x);
  * RMSNorm over d_v per (token, head): o / sqrt(mean(o^2) + 1e-6), times a
    learned weight gamma [d_v] shared by the heads.
"""
import numpy as np

WIDTH = 4
NORM_EPS = 1e-6


def silu(x):
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def short_conv(x, w, state=None):
    """x [B, T, C]; w [C, WIDTH]; state [B, WIDTH-1, C] or None (zeros).
    Returns (SiLU of the causal depthwise convolution [B, T, C], the new
    state: the last WIDTH-1 inputs, carried state included, [B, WIDTH-1, C])."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    B, T, C = x.shape
    if state is None:
        state = np.zeros((B, WIDTH - 1, C))
    xe = np.concatenate([np.asarray(state, dtype=np.float64), x], axis=1)     # [B, T + 3, C]
    pre = np.zeros((B, T, C))
    for j in range(WIDTH):
        pre += w[:, j][None, None, :] * xe[:, j:j + T, :]
    return silu(pre), xe[:, T:, :].copy()


def gated_rmsnorm(o, g, gamma, eps=NORM_EPS):
    """o, g [..., dv]; gamma [dv].  o / sqrt(mean(o^2) + eps) * gamma * SiLU(g)."""
    o = np.asarray(o, dtype=np.float64)
    r = 1.0 / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)
    return o * r * np.asarray(gamma, dtype=np.float64) * silu(g)
