"""Pins of the replay harness (oracle/replay.py), CPU only.

The statistics it reports (state error of NVFP4 trajectories against a clean
one, impulse decay) have no values on the pages that synthetic inputs could
reproduce; these tests pin the harness itself: it measures zero when nothing
is quantized, the clean projections do not depend on the d_model permutation
that makes the NVFP4 realisations independent, and an impulse on a
write-free (beta = 0) trajectory decays exactly as the product of the decays.
"""
import numpy as np
import pytest

from nvfp4_w4a4_gated_quant_b200 import inputs
from oracle.replay import clean_projections, impulse_response, replay

D = dict(B=1, T=256, d_model=128, H=2, dk=32, dv=32)
CHECK = (64, 128, 256)


def _inputs():
    return inputs.layer_inputs(D["B"], D["T"], D["d_model"], D["H"], D["dk"], D["dv"], seed=40)


def test_no_quantization_means_no_state_error():
    r = replay(_inputs(), seeds=(1, 2), checkpoints=CHECK, t_imp=128, window=16, quantize=False)
    assert np.all(r["state_error"] < 1e-12)


def test_clean_projections_do_not_depend_on_the_permutation():
    d = _inputs()
    x = d["x"].reshape(-1, D["d_model"])
    perm = np.random.default_rng(7).permutation(D["d_model"])
    p0 = clean_projections(x, d["W"])
    p1 = clean_projections(x[:, perm], {n: np.asarray(d["W"][n])[:, perm] for n in ("q", "k", "v", "a", "b")})
    for n in ("a", "b"):
        np.testing.assert_allclose(p1[n], p0[n], rtol=1e-12, atol=1e-14)
    for n in ("q", "k", "v"):
        assert np.mean(p1[n] != p0[n]) < 1e-3          # bf16 rounding ties only


def test_nvfp4_realisations_are_independent_and_bounded():
    r = replay(_inputs(), seeds=(1, 2, 3), checkpoints=CHECK, t_imp=128, window=16)
    e = r["state_error"]                                # [seeds, checkpoints]
    assert e.shape == (3, len(CHECK))
    assert np.all(np.isfinite(e)) and np.all(e > 1e-4) and np.all(e < 1.0)
    assert len(set(np.round(e[:, -1], 12))) == 3        # three different realisations
    np.testing.assert_allclose(r["mean"], e.mean(axis=0))
    assert np.all(r["max"] >= r["mean"])


def test_impulse_without_writes_decays_as_the_gate_product():
    rng = np.random.default_rng(3)
    B, T, H, dk, dv = 1, 96, 3, 8, 6
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    la = rng.uniform(-0.3, -0.01, (B, T, H))
    be = np.zeros((B, T, H))
    # a nonzero state to perturb: writes before the impulse, none after it
    be[:, :32] = 0.5
    steps, horizon = impulse_response(q, k, v, la, be, t_imp=32, window=60, eps=0.01,
                                      rng=np.random.default_rng(0))
    assert np.all(horizon > 0)
    np.testing.assert_array_equal(steps, horizon)


def test_gate_noise_arm_zero_noise_and_write_free_closed_form():
    from oracle.replay import clean_scan_inputs, gate_noise_arm
    scan_in = clean_scan_inputs(_inputs())
    assert np.all(gate_noise_arm(scan_in, 0.0, "alpha", (1, 2), CHECK) == 0.0)
    assert np.all(gate_noise_arm(scan_in, 0.0, "beta", (1, 2), CHECK) == 0.0)
    # write-free trajectory from a nonzero state: S_t = prod(alpha) S_0, so
    # alpha noise scales head h's state by prod_s (1 + sigma z_s) exactly
    rng = np.random.default_rng(5)
    B, T, H, dk, dv = 1, 40, 3, 6, 4
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    la = rng.uniform(-0.2, -0.01, (B, T, H))
    be = np.zeros((B, T, H))
    S0 = rng.standard_normal((B, H, dk, dv))
    sigma = 0.01
    e = gate_noise_arm((q, k, v, la, be), sigma, "alpha", (9,), (T,), S0=S0)
    z = np.random.default_rng(9).standard_normal(la.shape)
    g = np.prod(1.0 + sigma * z, axis=1)                         # [B, H]
    n2 = np.sum(S0 ** 2, axis=(2, 3))                            # ||S0_h||^2
    G = np.exp(np.sum(la, axis=1))
    want = np.sqrt(np.sum((G * (g - 1.0)) ** 2 * n2) / np.sum(G ** 2 * n2))
    np.testing.assert_allclose(e[0, 0], want, rtol=1e-9)
    # beta noise cannot act without writes
    assert np.all(gate_noise_arm((q, k, v, la, be), sigma, "beta", (9,), (T,), S0=S0) == 0.0)


def test_clamped_alpha_arm_closed_form():
    """Capping the perturbed decay at 1: with every alpha = 1 and no writes,
    head h's state is scaled by prod_s min(1 + sigma z_s, 1); with decays far
    below 1 the cap never binds and the arm equals the unclamped one."""
    from oracle.replay import gate_noise_arm
    rng = np.random.default_rng(6)
    B, T, H, dk, dv = 1, 30, 2, 5, 4
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    be = np.zeros((B, T, H))
    S0 = rng.standard_normal((B, H, dk, dv))
    sigma = 0.02
    la = np.zeros((B, T, H))                                     # alpha = 1
    e = gate_noise_arm((q, k, v, la, be), sigma, "alpha_clamped", (4,), (T,), S0=S0)
    z = np.random.default_rng(4).standard_normal(la.shape)
    g = np.prod(np.minimum(1.0 + sigma * z, 1.0), axis=1)        # [B, H]
    n2 = np.sum(S0 ** 2, axis=(2, 3))
    want = np.sqrt(np.sum((g - 1.0) ** 2 * n2) / np.sum(n2))
    np.testing.assert_allclose(e[0, 0], want, rtol=1e-9)
    la = np.full((B, T, H), -1.0)                                # alpha = e^-1: the cap never binds
    np.testing.assert_allclose(gate_noise_arm((q, k, v, la, be), sigma, "alpha_clamped", (4,), (T,), S0=S0),
                               gate_noise_arm((q, k, v, la, be), sigma, "alpha", (4,), (T,), S0=S0), rtol=1e-12)


def test_gate_error_compression_single_token():
    """One head, two tokens, one perturbed: at a = b = 0, A_log = 0,
    dt_bias = 0 the reference gates are alpha = beta = 1/2; perturbing token 1
    by d changes beta by sigmoid(d) - 1/2 and 1 - alpha by
    (1 - e^{-softplus(d)}) - 1/2 = sigmoid(d) - 1/2 as well (exp(-softplus(x))
    = sigmoid(-x)).  Token 0 carries the reference value r."""
    from oracle.replay import gate_error_compression
    d, r = 0.3, 0.8
    a_ref = np.array([[r], [0.0]])
    b_ref = np.array([[r], [0.0]])
    a_q = np.array([[r], [d]])
    b_q = np.array([[r], [d]])
    e = gate_error_compression(a_ref, b_ref, a_q, b_q, np.zeros(1), np.zeros(1))
    sig = lambda x: 1.0 / (1.0 + np.exp(-x))
    assert e["a"] == pytest.approx(d / r) and e["b"] == pytest.approx(d / r)
    want_beta = abs(sig(d) - 0.5) / np.hypot(sig(r), 0.5)
    assert e["beta"] == pytest.approx(want_beta, rel=1e-12)
    oma_r = np.array([1.0 - sig(-r), 0.5])                       # 1 - alpha = 1 - sigmoid(-a)
    want_alpha = abs(sig(d) - 0.5) / np.linalg.norm(oma_r)
    assert e["one_minus_alpha"] == pytest.approx(want_alpha, rel=1e-12)
    # no perturbation, no error
    z = gate_error_compression(a_ref, b_ref, a_ref, b_ref, np.zeros(1), np.zeros(1))
    assert all(val == 0.0 for val in z.values())
