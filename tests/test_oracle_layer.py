"""Pin of the oracle's layer composition (``oracle.layer.layer_forward``)
against a hand-worked two-token layer (``tests/golden/layer_hand.txt``).

Every activation and weight of the example lies exactly on its NVFP4 grid, so
each quantization is lossless up to one FP32 decode-scale factor per tensor
(within 2^-24 of 1); the gates come out as alpha = 1/4, beta = 1/2 from
softplus(0) = ln 2 and sigmoid(0) = 1/2; the normalised keys and queries are
unit vectors with dyadic dot products.  The hand-derived q, k, v, o, S_T and y
are therefore exact (the 1e-6 inside the norm moves o and S_T by < 2e-6).

Steps: "Why Gated DeltaNet Survives 4-Bit Quantization", section "Performance
and Efficiency Gains" (all projections W4A4, the gates included) and
"Anthology of the SOTA, theory-128", section "The account" (gates and the
recurrence).  Every projection has a distinct weight, so feeding any two of
them to each other's place changes y; the last test checks that the pin
catches each such swap.
"""
import os

import numpy as np
import pytest

from oracle.layer import layer_forward, quantize_weights

B, T, D, H, DK, DV = 1, 2, 32, 1, 16, 16
SHAPES = {"x": (T, D), "Wq": (H * DK, D), "Wk": (H * DK, D), "Wv": (H * DV, D), "Wa": (H, D), "Wb": (H, D),
          "Wout": (D, H * DV), "S0": (DK, DV), "q": (T, H * DK), "k": (T, H * DK), "v": (T, H * DV),
          "a": (T, H), "log_alpha": (T, H), "beta": (T, H), "o": (T, H * DV), "S_T": (DK, DV), "y": (T, D)}


def _load(golden_dir):
    arrays = {n: np.zeros(s) for n, s in SHAPES.items()}
    scalars = {}
    with open(os.path.join(golden_dir, "layer_hand.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].split()
            if not line:
                continue
            if len(line) == 2:
                scalars[line[0]] = float(line[1])
            else:
                arrays[line[0]][int(line[1]), int(line[2])] = float(line[3])
    return arrays, scalars


def _inputs(g, s):
    W = {"q": g["Wq"], "k": g["Wk"], "v": g["Wv"], "a": g["Wa"], "b": g["Wb"], "out": g["Wout"]}
    W = {n: w.astype(np.float32) for n, w in W.items()}
    x = g["x"].astype(np.float32).reshape(B, T, D)
    A_log = np.array([s["A_log"]])
    dt_bias = np.array([s["dt_bias"]])
    S0 = g["S0"].reshape(B, H, DK, DV)
    return x, W, A_log, dt_bias, S0


def _rel(a, b):
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.mark.parametrize("chunked", [True, False], ids=["chunked", "sequential"])
def test_layer_matches_hand_worked_example(golden_dir, chunked):
    g, s = _load(golden_dir)
    x, W, A_log, dt_bias, S0 = _inputs(g, s)
    y, S_T, inter = layer_forward(x, quantize_weights(W), A_log, dt_bias, H, DK, DV, chunked=chunked, S0=S0)
    # q, k, v are bf16-rounded projections: exact
    np.testing.assert_array_equal(inter["q"].reshape(T, -1), g["q"])
    np.testing.assert_array_equal(inter["k"].reshape(T, -1), g["k"])
    np.testing.assert_array_equal(inter["v"].reshape(T, -1), g["v"])
    # gate pre-activations and gates: exact up to the decode-scale factors
    np.testing.assert_allclose(inter["a"].reshape(T, H), g["a"], rtol=1e-6)
    np.testing.assert_allclose(inter["b"].reshape(T, H), 0.0, atol=1e-12)
    np.testing.assert_allclose(inter["log_alpha"].reshape(T, H), g["log_alpha"], rtol=1e-6)
    np.testing.assert_allclose(inter["beta"].reshape(T, H), g["beta"], rtol=1e-12)
    # o and the final state: the normalisation's 1e-6 moves them by < 2e-6
    assert _rel(inter["o"].reshape(T, -1), g["o"]) < 1e-5
    assert _rel(S_T.reshape(DK, DV), g["S_T"]) < 1e-5
    # o rounds to bf16 onto the hand values (o_2[0] = (3/16)(1 - k1^.k2^ / (1/2))
    # is ~2.6e-7 from the norm's 1e-6, and its NVFP4 code is 0)
    np.testing.assert_allclose(inter["o_bf16"], g["o"], rtol=0, atol=1e-6)
    np.testing.assert_array_equal(inter["o_bf16"][np.abs(g["o"]) > 0], g["o"][np.abs(g["o"]) > 0])
    # y: bf16 of an exact dot product up to two decode-scale factors
    np.testing.assert_array_equal(y.reshape(T, D), g["y"])


@pytest.mark.parametrize("swap", [("q", "k"), ("k", "v"), ("q", "v"), ("a", "b")],
                         ids=["q-k", "k-v", "q-v", "a-b"])
def test_pin_catches_swapped_projections(golden_dir, swap):
    """A layer that feeds one projection in another's place (a plausible
    wiring mistake) misses the hand-worked y and S_T by far more than their
    tolerance."""
    g, s = _load(golden_dir)
    x, W, A_log, dt_bias, S0 = _inputs(g, s)
    Wq = quantize_weights(W)
    Wq[swap[0]], Wq[swap[1]] = Wq[swap[1]], Wq[swap[0]]
    y, S_T, _ = layer_forward(x, Wq, A_log, dt_bias, H, DK, DV, S0=S0)
    assert _rel(y.reshape(T, D), g["y"]) > 0.05 or _rel(S_T.reshape(DK, DV), g["S_T"]) > 0.05
    assert _rel(y.reshape(T, D), g["y"]) > 1e-3


def test_given_scales_equal_to_the_dynamic_ones_reproduce_the_example(golden_dir):
    """Static activation scales: handing the layer the encode scales its two
    activations would get dynamically (x: amax 1 -> 2688; o: amax 1.5 ->
    1792) gives the same hand-worked result; another o scale changes y."""
    g, s = _load(golden_dir)
    x, W, A_log, dt_bias, S0 = _inputs(g, s)
    Wq = quantize_weights(W)
    y, S_T, inter = layer_forward(x, Wq, A_log, dt_bias, H, DK, DV, S0=S0, x_g_enc=np.float32(2688.0),
                                  o_g_enc=np.float32(1792.0))
    np.testing.assert_array_equal(y.reshape(T, D), g["y"])
    assert inter["oq"]["g_enc"] == np.float32(1792.0) and inter["xq"]["g_enc"] == np.float32(2688.0)
    y2, _, _ = layer_forward(x, Wq, A_log, dt_bias, H, DK, DV, S0=S0, o_g_enc=np.float32(1792.0 * 3.3))
    assert _rel(y2.reshape(T, D), g["y"]) > 1e-3
