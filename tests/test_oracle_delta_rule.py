"""Pins for the oracle's gated delta rule (CPU only).

The recurrence is S_t = alpha_t S_{t-1} + beta_t k_t (v_t - S_{t-1}^T k_t)^T,
o_t = S_t^T q_t ("Anthology of the SOTA, theory-128", section "The account").
The pins are what that page and the algebra fix:
  * a hand-worked two-token example with d_k != d_v and a nonzero S_0
    (tests/golden/delta_rule_hand.txt; it separates the literal undecayed read
    from the decayed-read variant and catches transposes);
  * the overwrite invariant: alpha = beta = 1 and ||k|| = 1 give
    S_t^T k_t = v_t ("the write replaces whatever the state currently returns
    for key k_t with v_t");
  * beta = 0 is pure decay: S_T = prod(alpha) S_0 and
    o_t = prod_{s<=t}(alpha_s) S_0^T q_t ("the decay forgets uniformly");
  * T = 1 from S_0 = 0: S_1 = beta k v^T, o_1 = beta (k.q) v;
  * the chunked form equals the sequential scan; segment splits with the
    state carried equal one shot; a d_v slice alone equals that slice.
"""
import os

import numpy as np
import pytest

from oracle.delta_rule import delta_rule_chunked, delta_rule_sequential, l2_normalize


def _rand(rng, B, T, H, dk, dv, decay=(-1.0, 0.0)):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    la = rng.uniform(decay[0], decay[1], (B, T, H))
    be = rng.uniform(0, 1, (B, T, H))
    return q, k, v, la, be


def _hand(golden_dir):
    d = {}
    with open(os.path.join(golden_dir, "delta_rule_hand.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                key, *vals = line.split()
                d[key] = np.array([float(x) for x in vals])
    return d


@pytest.mark.parametrize("fn", [delta_rule_sequential, delta_rule_chunked])
def test_hand_worked_example(golden_dir, fn):
    d = _hand(golden_dir)
    q = np.stack([d["q1"], d["q2"]])[None, :, None, :]
    k = np.stack([d["k1"], d["k2"]])[None, :, None, :]
    v = np.stack([d["v1"], d["v2"]])[None, :, None, :]
    la = np.log(np.array([d["alpha1"][0], d["alpha2"][0]]))[None, :, None]
    be = np.array([d["beta1"][0], d["beta2"][0]])[None, :, None]
    S0 = d["S0"].reshape(1, 1, 2, 3)
    kw = {"chunk": 2} if fn is delta_rule_chunked else {}
    o, S = fn(q, k, v, la, be, S0=S0, normalize=False, **kw)
    np.testing.assert_allclose(o[0, 0, 0], d["o1"], atol=1e-14)
    np.testing.assert_allclose(o[0, 1, 0], d["o2"], atol=1e-14)
    np.testing.assert_allclose(S[0, 0].reshape(-1), d["S2"], atol=1e-14)


def test_overwrite_invariant():
    rng = np.random.default_rng(0)
    B, T, H, dk, dv = 1, 40, 2, 8, 5
    q, k, v, _, _ = _rand(rng, B, T, H, dk, dv)
    k = k / np.linalg.norm(k, axis=-1, keepdims=True)
    la = np.zeros((B, T, H))
    be = np.ones((B, T, H))
    S0 = rng.standard_normal((B, H, dk, dv))
    S = S0[0]
    # step through one token at a time and check S_t^T k_t = v_t after each
    for t in range(T):
        _, S_t = delta_rule_sequential(q[:, t:t + 1], k[:, t:t + 1], v[:, t:t + 1],
                                       la[:, t:t + 1], be[:, t:t + 1], S0=S[None], normalize=False)
        S = S_t[0]
        for h in range(H):
            np.testing.assert_allclose(S[h].T @ k[0, t, h], v[0, t, h], atol=1e-12)


def test_beta_zero_is_pure_decay():
    rng = np.random.default_rng(1)
    B, T, H, dk, dv = 2, 37, 3, 6, 4
    q, k, v, la, _ = _rand(rng, B, T, H, dk, dv)
    be = np.zeros((B, T, H))
    S0 = rng.standard_normal((B, H, dk, dv))
    for fn in (delta_rule_sequential, delta_rule_chunked):
        kw = {"chunk": 8} if fn is delta_rule_chunked else {}
        o, S = fn(q, k, v, la, be, S0=S0, **kw)
        G = np.cumsum(la, axis=1)                                       # [B, T, H]
        np.testing.assert_allclose(S, np.exp(G[:, -1])[:, :, None, None] * S0, rtol=1e-12)
        qh = l2_normalize(q)
        want = np.exp(G)[..., None] * np.einsum("bhkv,bthk->bthv", S0, qh)
        np.testing.assert_allclose(o, want, rtol=1e-11, atol=1e-14)


def test_single_token_from_zero_state():
    rng = np.random.default_rng(2)
    q, k, v, la, be = _rand(rng, 2, 1, 3, 7, 5)
    o, S = delta_rule_sequential(q, k, v, la, be)
    qh, kh = l2_normalize(q), l2_normalize(k)
    S_want = be[:, 0, :, None, None] * kh[:, 0, :, :, None] * v[:, 0, :, None, :]
    np.testing.assert_allclose(S, S_want, rtol=1e-13)
    o_want = (be[:, 0] * np.sum(kh[:, 0] * qh[:, 0], -1))[..., None] * v[:, 0]
    np.testing.assert_allclose(o[:, 0], o_want, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("T,chunk", [(1, 64), (63, 64), (64, 64), (65, 64), (200, 64), (130, 16), (77, 32)])
def test_chunked_equals_sequential(T, chunk):
    rng = np.random.default_rng(T * 7 + chunk)
    B, H, dk, dv = 2, 2, 16, 12
    q, k, v, la, be = _rand(rng, B, T, H, dk, dv, decay=(-3.0, 0.0))
    S0 = rng.standard_normal((B, H, dk, dv))
    o1, S1 = delta_rule_sequential(q, k, v, la, be, S0=S0)
    o2, S2 = delta_rule_chunked(q, k, v, la, be, S0=S0, chunk=chunk)
    scale = max(np.abs(o1).max(), 1.0)
    np.testing.assert_allclose(o2, o1, atol=1e-10 * scale, rtol=0)
    np.testing.assert_allclose(S2, S1, atol=1e-10 * max(np.abs(S1).max(), 1.0), rtol=0)


def test_chunked_strong_decay_no_overflow():
    """log alpha down to -13 per token (the synthetic gates reach that): every
    exponent in the chunk form is <= 0, so nothing overflows."""
    rng = np.random.default_rng(3)
    q, k, v, la, be = _rand(rng, 1, 150, 2, 8, 8, decay=(-13.0, 0.0))
    with np.errstate(over="raise"):
        o2, S2 = delta_rule_chunked(q, k, v, la, be)
    o1, S1 = delta_rule_sequential(q, k, v, la, be)
    np.testing.assert_allclose(o2, o1, atol=1e-10)
    np.testing.assert_allclose(S2, S1, atol=1e-10)


def test_segment_split_with_state_carry():
    rng = np.random.default_rng(4)
    q, k, v, la, be = _rand(rng, 1, 300, 2, 8, 6)
    o, S = delta_rule_chunked(q, k, v, la, be)
    o_a, S_a = delta_rule_chunked(q[:, :130], k[:, :130], v[:, :130], la[:, :130], be[:, :130])
    o_b, S_b = delta_rule_chunked(q[:, 130:], k[:, 130:], v[:, 130:], la[:, 130:], be[:, 130:], S0=S_a)
    np.testing.assert_allclose(np.concatenate([o_a, o_b], 1), o, atol=1e-12)
    np.testing.assert_allclose(S_b, S, atol=1e-12)


def test_dv_slice_independent():
    rng = np.random.default_rng(5)
    q, k, v, la, be = _rand(rng, 1, 90, 2, 8, 12)
    S0 = rng.standard_normal((1, 2, 8, 12))
    o, S = delta_rule_sequential(q, k, v, la, be, S0=S0)
    o_s, S_s = delta_rule_sequential(q, k, v[..., 4:8], la, be, S0=S0[..., 4:8])
    np.testing.assert_allclose(o_s, o[..., 4:8], atol=1e-13)
    np.testing.assert_allclose(S_s, S[..., 4:8], atol=1e-13)


# ---------------------------------------------------------- decayed read --
# The other reading of the correction term (it reads alpha_t S_{t-1}):
# S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T.

def test_decayed_read_single_step_matrix_form():
    """One step against the matrix form written out with an explicit
    identity, from a nonzero state, alpha != 1."""
    rng = np.random.default_rng(21)
    B, H, dk, dv = 2, 3, 7, 5
    q, k, v, la, be = _rand(rng, B, 1, H, dk, dv)
    S0 = rng.standard_normal((B, H, dk, dv))
    o, S = delta_rule_sequential(q, k, v, la, be, S0=S0, decayed_read=True)
    qh, kh = l2_normalize(q), l2_normalize(k)
    for b in range(B):
        for h in range(H):
            a, bt, kk = np.exp(la[b, 0, h]), be[b, 0, h], kh[b, 0, h]
            S_want = a * (np.eye(dk) - bt * np.outer(kk, kk)) @ S0[b, h] + bt * np.outer(kk, v[b, 0, h])
            np.testing.assert_allclose(S[b, h], S_want, rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(o[b, 0, h], S_want.T @ qh[b, 0, h], rtol=1e-12, atol=1e-14)


def test_decayed_read_overwrite_invariant_any_alpha():
    """With beta = 1 and a unit key the decayed-read update returns v_t for
    k_t whatever alpha_t is; the undecayed read does so only at alpha = 1."""
    rng = np.random.default_rng(22)
    B, T, H, dk, dv = 1, 12, 2, 8, 5
    q, k, v, la, _ = _rand(rng, B, T, H, dk, dv)
    k = k / np.linalg.norm(k, axis=-1, keepdims=True)
    be = np.ones((B, T, H))
    S = rng.standard_normal((B, H, dk, dv))
    for t in range(T):
        _, S = delta_rule_sequential(q[:, t:t + 1], k[:, t:t + 1], v[:, t:t + 1], la[:, t:t + 1],
                                     be[:, t:t + 1], S0=S, normalize=False, decayed_read=True)
        for h in range(H):
            np.testing.assert_allclose(S[0, h].T @ k[0, t, h], v[0, t, h], atol=1e-12)
    _, S_u = delta_rule_sequential(q[:, :1], k[:, :1], v[:, :1], la[:, :1], be[:, :1],
                                   S0=rng.standard_normal((B, H, dk, dv)), normalize=False)
    assert np.abs(S_u[0, 0].T @ k[0, 0, 0] - v[0, 0, 0]).max() > 1e-3


def test_decayed_read_equals_undecayed_at_alpha_one():
    rng = np.random.default_rng(23)
    q, k, v, _, be = _rand(rng, 2, 19, 3, 6, 4)
    la = np.zeros(be.shape)
    S0 = rng.standard_normal((2, 3, 6, 4))
    o1, S1 = delta_rule_sequential(q, k, v, la, be, S0=S0)
    o2, S2 = delta_rule_sequential(q, k, v, la, be, S0=S0, decayed_read=True)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(S1, S2)
