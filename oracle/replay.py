"""Replay harness: how far NVFP4 W4A4 projections move the recurrent state
(oracle; test infrastructure).

"Why Gated DeltaNet Survives 4-Bit Quantization", section "Why the 'Fragile'
Recurrence is Actually Robust": the pages compare the state of a clean
trajectory with the states of NVFP4 trajectories over long sequences (a state
error of a few tens of percent that does not grow without bound) and follow
an impulse added to the state until it has decayed.  Their numbers come from
trained layers and real text; here the same measurements run on synthetic
inputs, so the statistics themselves are parity unpinned.  The same page
applies multiplicative noise directly to the gates (alpha and beta) to show
where the recurrence is fragile; ``gate_noise_arm`` does that here.  What is
pinned (``tests/test_oracle_replay.py``) is the harness: zero error when
nothing is quantized or no noise is added, the exact permutation invariance
of the clean projections, an impulse on a write-free (beta = 0) trajectory
decaying exactly as the product of the decays, and alpha noise on such a
trajectory scaling each head's state by exactly prod (1 + sigma z) (by
prod min(1 + sigma z, 1) when the perturbed decay is capped at 1 and every
alpha is 1).  ``gate_error_compression`` (the page's account of how a
projection error shrinks through the gates) is pinned by a single perturbed
token whose gate errors are sigmoid(d) - 1/2 and the closed-form softplus
difference.

Readings where the pages are silent:
  * clean trajectory: FP64 projections of the bf16 activations with the FP32
    weights, q / k / v rounded to bf16 (the storage precision of the layer);
  * NVFP4 trajectories: a fixed random permutation P_s of the d_model axis is
    applied to x and to every weight before quantizing (x P_s (W P_s)^T =
    x W^T exactly, but the 16-element blocks change), so each seed is an
    independent realisation of the quantization error against one target;
  * state error at t: ||S^q_t - S^clean_t||_F / ||S^clean_t||_F over all
    heads; impulse: S_t <- S_t * (1 + eps z), z ~ N(0, 1) elementwise, and the
    number of tokens until ||dS|| falls to 1/e of its start, per head; the
    decay-implied horizon is the first n with prod_{s=1..n} alpha_{t+s} <= 1/e.
"""
import numpy as np

from . import nvfp4
from .delta_rule import delta_rule_chunked, delta_rule_sequential
from .gates import gates
from .gemm import gemm_fp64

PROJ = ("q", "k", "v", "a", "b")


def clean_projections(x, W):
    """x [M, d_model] (bf16 values), W dict of FP32 [out, d_model] -> dict of
    FP64 projections x W^T (q, k, v rounded to bf16)."""
    x = np.asarray(x, dtype=np.float64)
    out = {}
    for n in PROJ:
        p = x @ np.asarray(W[n], dtype=np.float64).T
        out[n] = nvfp4.round_bf16(p) if n in ("q", "k", "v") else p
    return out


def nvfp4_projections(x, W, perm=None):
    """The W4A4 projections: x and every weight permuted along d_model by
    ``perm`` (None: identity), then quantized (x dynamically, each weight with
    its own scale), FP64 GEMM over the dequantised operands, q / k / v
    rounded to bf16."""
    x = np.asarray(x, dtype=np.float32)
    if perm is not None:
        x = x[:, perm]
    xq = nvfp4.quantize(x)
    out = {}
    for n in PROJ:
        w = np.asarray(W[n], dtype=np.float32)
        if perm is not None:
            w = w[:, perm]
        p = gemm_fp64(xq, nvfp4.quantize(w))
        out[n] = nvfp4.round_bf16(p) if n in ("q", "k", "v") else p
    return out


def _scan_inputs(proj, B, T, H, dk, dv, A_log, dt_bias):
    q = proj["q"].reshape(B, T, H, dk)
    k = proj["k"].reshape(B, T, H, dk)
    v = proj["v"].reshape(B, T, H, dv)
    la, be = gates(proj["a"].reshape(B, T, H), proj["b"].reshape(B, T, H), A_log, dt_bias)
    return q, k, v, la, be


def states_at(q, k, v, la, be, checkpoints, S0=None):
    """The state after each checkpoint token count (chunked form with the
    state carried from segment to segment)."""
    out = []
    S, t_prev = S0, 0
    for t in checkpoints:
        _, S = delta_rule_chunked(q[:, t_prev:t], k[:, t_prev:t], v[:, t_prev:t], la[:, t_prev:t],
                                  be[:, t_prev:t], S0=S)
        out.append(S)
        t_prev = t
    return out


def rel_state_error(S_q, S_ref):
    return float(np.linalg.norm(S_q - S_ref) / np.linalg.norm(S_ref))


def impulse_response(q, k, v, la, be, t_imp, window, eps, rng):
    """Perturb the state after t_imp tokens and follow the difference token
    by token.  Returns (steps to 1/e per (b, h) or -1 if not reached within
    the window, decay-implied horizon per (b, h) or -1)."""
    _, S = delta_rule_chunked(q[:, :t_imp], k[:, :t_imp], v[:, :t_imp], la[:, :t_imp], be[:, :t_imp])
    S_p = S * (1.0 + eps * rng.standard_normal(S.shape))
    d0 = np.linalg.norm((S_p - S).reshape(S.shape[0], S.shape[1], -1), axis=-1)
    B, H = S.shape[:2]
    steps = -np.ones((B, H), dtype=np.int64)
    for n in range(1, window + 1):
        t = t_imp + n - 1
        sl = slice(t, t + 1)
        _, S = delta_rule_sequential(q[:, sl], k[:, sl], v[:, sl], la[:, sl], be[:, sl], S0=S)
        _, S_p = delta_rule_sequential(q[:, sl], k[:, sl], v[:, sl], la[:, sl], be[:, sl], S0=S_p)
        d = np.linalg.norm((S_p - S).reshape(B, H, -1), axis=-1)
        steps[(steps < 0) & (d <= d0 / np.e)] = n
    G = np.cumsum(la[:, t_imp:t_imp + window], axis=1)            # [B, n, H]
    hit = G <= -1.0
    horizon = np.where(hit.any(axis=1), hit.argmax(axis=1) + 1, -1)
    return steps, horizon


def replay(d, seeds, checkpoints, t_imp, window, eps=0.01, quantize=True):
    """Run the clean trajectory and one NVFP4 trajectory per seed on the
    layer inputs ``d`` (inputs.layer_inputs).  Returns the state errors per
    seed and checkpoint, their mean and max, and the impulse statistics of
    the clean trajectory."""
    B, T, D, H, dk, dv = d["B"], d["T"], d["d_model"], d["H"], d["dk"], d["dv"]
    x = d["x"].reshape(B * T, D)
    clean = _scan_inputs(clean_projections(x, d["W"]), B, T, H, dk, dv, d["A_log"], d["dt_bias"])
    S_clean = states_at(*clean, checkpoints)
    errs = []
    for s in seeds:
        perm = np.random.default_rng(s).permutation(D)
        proj = nvfp4_projections(x, d["W"], perm) if quantize else clean_projections(x[:, perm], {
            n: np.asarray(d["W"][n])[:, perm] for n in PROJ})
        S_q = states_at(*_scan_inputs(proj, B, T, H, dk, dv, d["A_log"], d["dt_bias"]), checkpoints)
        errs.append([rel_state_error(a, b) for a, b in zip(S_q, S_clean)])
    errs = np.asarray(errs)
    steps, horizon = impulse_response(*clean, t_imp, window, eps, np.random.default_rng(12345))
    return {"checkpoints": list(checkpoints), "state_error": errs, "mean": errs.mean(axis=0),
            "max": errs.max(axis=0), "impulse_steps": steps, "decay_horizon": horizon}


def gate_noise_arm(scan_in, sigma, target, seeds, checkpoints, S0=None):
    """Multiplicative gate noise on a given trajectory: every alpha_t (target
    "alpha" or "alpha_clamped") or beta_t ("beta") times (1 + sigma z),
    z ~ N(0, 1) per (token, head), seeded.  "alpha" lets a perturbed decay
    exceed 1 (the state then grows for that token); "alpha_clamped" caps it at
    1, min(alpha_t (1 + sigma z), 1), so the noise can only make the state
    forget faster or slower, never expand.  Returns the relative state error
    against the noise-free trajectory, [seeds, checkpoints]."""
    q, k, v, la, be = scan_in
    S_ref = states_at(q, k, v, la, be, checkpoints, S0=S0)
    out = []
    for s in seeds:
        z = np.random.default_rng(s).standard_normal(la.shape)
        f = 1.0 + sigma * z
        assert np.all(f > 0), "noise too large for a multiplicative perturbation"
        if target == "alpha":
            la_n, be_n = la + np.log(f), be
        elif target == "alpha_clamped":
            la_n, be_n = np.minimum(la + np.log(f), 0.0), be
        elif target == "beta":
            la_n, be_n = la, be * f
        else:
            raise ValueError(f"unknown target {target!r}")
        S_n = states_at(q, k, v, la_n, be_n, checkpoints, S0=S0)
        out.append([rel_state_error(a, b) for a, b in zip(S_n, S_ref)])
    return np.asarray(out)


def gate_error_compression(a_ref, b_ref, a_q, b_q, A_log, dt_bias):
    """How an error on the gate projections shrinks through the gates
    ("Anthology of the SOTA, theory-128", section "The account": the decay
    and write gates pass the projection through softplus / exp and a sigmoid,
    whose slopes are below 1 where the gates saturate).  Given reference and
    perturbed projections a, b ([..., H]), returns the relative Frobenius
    errors on a, on b, on 1 - alpha and on beta."""
    la_r, be_r = gates(a_ref, b_ref, A_log, dt_bias)
    la_q, be_q = gates(a_q, b_q, A_log, dt_bias)
    oma_r, oma_q = -np.expm1(la_r), -np.expm1(la_q)       # 1 - alpha, without cancellation
    return {"a": rel_state_error(a_q, a_ref), "b": rel_state_error(b_q, b_ref),
            "one_minus_alpha": rel_state_error(oma_q, oma_r), "beta": rel_state_error(be_q, be_r)}


def clean_scan_inputs(d):
    """The clean trajectory's scan inputs (q, k, v, log_alpha, beta) for the
    layer inputs ``d``."""
    B, T, D, H, dk, dv = d["B"], d["T"], d["d_model"], d["H"], d["dk"], d["dv"]
    return _scan_inputs(clean_projections(d["x"].reshape(B * T, D), d["W"]), B, T, H, dk, dv, d["A_log"],
                        d["dt_bias"])
