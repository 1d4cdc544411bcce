"""Decay and write-strength gates (oracle; test infrastructure).

"Anthology of the SOTA, theory-128", section "The account": the decay is
exp(-exp(A) * softplus(a + b)) and the write strength is a sigmoid.  Reading:
the "b" inside the softplus is the per-head bias dt_bias (the benchmark spec
writes alpha_t = exp(-exp(A) softplus(a_t + dt_bias))), not the write-strength
projection; A is a per-head log-rate used as exp(A).  FP64 throughout.

softplus(x) = max(x, 0) + log1p(exp(-|x|)), which is exact algebra for
log(1 + e^x) and needs no threshold.
"""
import numpy as np


def softplus(x):
    x = np.asarray(x, dtype=np.float64)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def sigmoid(x):
    x = np.asarray(x, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-x))


def gates(a, b, A_log, dt_bias):
    """a, b: [..., H]; A_log, dt_bias: [H].  Returns (log_alpha, beta), FP64.

    log_alpha = -exp(A_log) * softplus(a + dt_bias);  beta = sigmoid(b)."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    A_log = np.asarray(A_log, dtype=np.float64)
    dt_bias = np.asarray(dt_bias, dtype=np.float64)
    log_alpha = -np.exp(A_log) * softplus(a + dt_bias)
    beta = sigmoid(b)
    return log_alpha, beta
