"""GPU parity of step 4, the chunked gated delta rule, against the FP64 oracle.

"Anthology of the SOTA, theory-128", section "The account":
S_t = alpha_t S_{t-1} + beta_t k_t (v_t - S_{t-1}^T k_t)^T, o_t = S_t^T q_t over
L2-normalised q, k.  Tolerance: 2e-3 relative Frobenius on o (FP32 output) and
on the final state, the bound stated for 32K tokens.  Both sides get the same
bf16 q / k / v and the same FP32 gates.  Shapes with d_k = 128 and d_v a
multiple of 64 run on the tcgen05 kernel by default; every such case is also
run on the mma.sync kernel (``mma_sync=True``).
"""
import numpy as np
import pytest
import torch

from nvfp4_w4a4_gated_quant_b200 import _lib, inputs
from oracle.delta_rule import delta_rule_chunked
from oracle.gates import gates as oracle_gates
from tests._helpers import bf16_cuda, f32_cuda, rel_fro, to_np

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _case(B, T, H, dk, dv, seed, with_s0=False):
    rng = np.random.default_rng(seed)
    q = inputs.to_bf16_values(rng.standard_normal((B, T, H, dk), dtype=np.float32))
    k = inputs.to_bf16_values(rng.standard_normal((B, T, H, dk), dtype=np.float32))
    v = inputs.to_bf16_values(rng.standard_normal((B, T, H, dv), dtype=np.float32))
    a = rng.standard_normal((B, T, H)).astype(np.float32)
    b = rng.standard_normal((B, T, H)).astype(np.float32)
    A = rng.uniform(-2, 1, H)
    dt = rng.uniform(-1, 1, H)
    la, be = oracle_gates(a, b, A, dt)
    la = la.astype(np.float32)
    be = be.astype(np.float32)
    S0 = (rng.standard_normal((B, H, dk, dv)) * 0.5).astype(np.float32) if with_s0 else None
    return q, k, v, la, be, S0


def _run(q, k, v, la, be, S0, o_fp32=True, mma_sync=False):
    o, S = _lib.gdn_delta_rule_fwd(bf16_cuda(q), bf16_cuda(k), bf16_cuda(v), f32_cuda(la), f32_cuda(be),
                                   S0=None if S0 is None else f32_cuda(S0), o_fp32=o_fp32, mma_sync=mma_sync)
    _lib.stream_check()
    return to_np(o).astype(np.float64), to_np(S).astype(np.float64)


@pytest.mark.parametrize("B,T,H,dk,dv,seed,s0", [
    (1, 64, 2, 128, 128, 0, False),     # one full chunk, 4 chains -> 16-column slices
    (2, 200, 3, 128, 128, 1, True),     # ragged last chunk, initial state
    (1, 1, 2, 128, 64, 2, False),       # a single token
    (1, 65, 20, 128, 128, 3, False),    # 20 chains -> 32-column slices
    (2, 130, 20, 128, 64, 4, True),     # 40 chains, dv 64
    (2, 96, 40, 128, 128, 5, False),    # 80 chains -> whole 128-column state per CTA
    (1, 160, 2, 32, 32, 6, True),       # the tiny layer's head dims
    (1, 100, 3, 64, 64, 7, False),
    (3, 300, 50, 128, 128, 8, True),    # 150 chains: more CTAs than SMs
])
@pytest.mark.parametrize("mma_sync", [False, True], ids=["tcgen05", "mma_sync"])
def test_delta_rule_matches_oracle(B, T, H, dk, dv, seed, s0, mma_sync):
    if mma_sync and dk != 128:
        pytest.skip("shape runs on the mma.sync kernel anyway")
    q, k, v, la, be, S0 = _case(B, T, H, dk, dv, seed, s0)
    o, S = _run(q, k, v, la, be, S0, mma_sync=mma_sync)
    o_ref, S_ref = delta_rule_chunked(q, k, v, la, be, S0=S0)
    assert rel_fro(o, o_ref) < TOL, rel_fro(o, o_ref)
    assert rel_fro(S, S_ref) < TOL, rel_fro(S, S_ref)


@pytest.mark.parametrize("mma_sync", [False, True], ids=["tcgen05", "mma_sync"])
def test_delta_rule_bf16_output(mma_sync):
    q, k, v, la, be, S0 = _case(1, 190, 4, 128, 128, 9)
    o, _ = _run(q, k, v, la, be, S0, o_fp32=False, mma_sync=mma_sync)
    o_ref, _ = delta_rule_chunked(q, k, v, la, be)
    # bf16 storage adds its own rounding (~1.5e-3 relative RMS) on top
    assert rel_fro(o, o_ref) < 3e-3


@pytest.mark.parametrize("mma_sync", [False, True], ids=["tcgen05", "mma_sync"])
def test_delta_rule_empty_sequence_returns_initial_state(mma_sync):
    q, k, v, la, be, S0 = _case(1, 0, 2, 128, 128, 10, True)
    o, S = _run(q, k, v, la, be, S0, mma_sync=mma_sync)
    np.testing.assert_array_equal(S, S0)


def test_delta_rule_segments_with_state_carry():
    """Two calls over [0, 150) and [150, 300) with the state carried equal
    one call over [0, 300) (checkpoint / resume of a long prefill)."""
    q, k, v, la, be, _ = _case(1, 300, 4, 128, 128, 12)
    o_all, S_all = _run(q, k, v, la, be, None)
    o1, S1 = _run(q[:, :150], k[:, :150], v[:, :150], la[:, :150], be[:, :150], None)
    o2, S2 = _run(q[:, 150:], k[:, 150:], v[:, 150:], la[:, 150:], be[:, 150:], S1.astype(np.float32))
    assert rel_fro(np.concatenate([o1, o2], 1), o_all) < 1e-3
    assert rel_fro(S2, S_all) < 1e-3


@pytest.mark.parametrize("mma_sync", [False, True], ids=["tcgen05", "mma_sync"])
def test_delta_rule_scan_workload_32k(mma_sync):
    """The scan workload: B=1, T=32768, H=16, d=128 (gates from a, b as the
    layer computes them); o and S_T within 2e-3 of the FP64 oracle."""
    d = inputs.scan_workload()
    la, be = oracle_gates(d["a"], d["b"], d["A_log"], d["dt_bias"])
    la = la.astype(np.float32)
    be = be.astype(np.float32)
    o, S = _run(d["q"], d["k"], d["v"], la, be, None, mma_sync=mma_sync)
    o_ref, S_ref = delta_rule_chunked(d["q"], d["k"], d["v"], la, be)
    e_o, e_s = rel_fro(o, o_ref), rel_fro(S, S_ref)
    print(f"scan 32K: rel_fro o {e_o:.3e}  S_T {e_s:.3e}")
    assert e_o < TOL and e_s < TOL


def test_delta_rule_strong_and_no_decay():
    """Gates at the ends of their range: alpha ~ e^-30 per token (the state
    forgets within a token) and alpha = 1 with beta = 1 (pure delta rule);
    every exponent the chunk form takes stays <= 0, so both stay finite."""
    q, k, v, _, _, S0 = _case(1, 190, 4, 128, 128, 13, True)
    for la_val, be_val in ((-30.0, 0.5), (0.0, 1.0)):
        la = np.full(q.shape[:3], la_val, np.float32)
        be = np.full(q.shape[:3], be_val, np.float32)
        o_ref, S_ref = delta_rule_chunked(q, k, v, la, be, S0=S0)
        for mma_sync in (False, True):
            o, S = _run(q, k, v, la, be, S0, mma_sync=mma_sync)
            assert np.isfinite(o).all() and np.isfinite(S).all()
            assert rel_fro(o, o_ref) < TOL and rel_fro(S, S_ref) < TOL, (la_val, mma_sync)


@pytest.mark.parametrize("mma_sync", [False, True], ids=["tcgen05", "mma_sync"])
def test_fp16_overflow_is_reported(mma_sync):
    """A value of v beyond the FP16 range of the chunk contractions
    (|beta v| >= 65520 rounds to infinity) makes the call report
    GDN_ERR_RANGE through the status word instead of returning inf / NaN
    silently; the next call on the same context is unaffected."""
    q, k, v, la, be, _ = _case(1, 100, 2, 128, 128, 11)
    v = v.copy()
    v[0, 37, 1, 5] = 2.0 ** 17
    be = np.ones_like(be)
    _lib.gdn_delta_rule_fwd(bf16_cuda(q), bf16_cuda(k), bf16_cuda(v), f32_cuda(la), f32_cuda(be), o_fp32=True,
                            mma_sync=mma_sync)
    with pytest.raises(_lib.GdnError, match="status 7"):
        _lib.stream_check()
    _lib.stream_check()      # the status word was cleared
    q, k, v, la, be, S0 = _case(1, 100, 2, 128, 128, 12)
    o, S = _run(q, k, v, la, be, S0, mma_sync=mma_sync)
    o_ref, S_ref = delta_rule_chunked(q, k, v, la, be)
    assert rel_fro(o, o_ref) < TOL and rel_fro(S, S_ref) < TOL


@pytest.mark.parametrize("T,H,o_fp32,s0", [(2000, 2, True, True), (4096, 4, False, False), (4100, 1, True, False)],
                         ids=["ragged_s0", "bf16", "one_chain_ragged"])
def test_segmented_scan_matches_oracle(T, H, o_fp32, s0):
    """Few chains on long sequences: the library cuts each sequence into
    segments (state transitions of the segments in parallel, their FP32
    composition, then every segment from its entry state).  Same tolerance as
    the unsegmented scan; the workspace query says the path is taken."""
    assert _lib.lib().gdn_delta_rule_workspace_size(1, T, H, 128, 128) > 0
    q, k, v, la, be, S0 = _case(1, T, H, 128, 128, 30 + T, with_s0=s0)
    o, S = _run(q, k, v, la, be, S0, o_fp32=o_fp32)
    o_ref, S_ref = delta_rule_chunked(q, k, v, la, be, S0=S0)
    if not o_fp32:
        from oracle.nvfp4 import round_bf16
        o_ref = round_bf16(o_ref)
    assert rel_fro(o, o_ref) < (TOL if o_fp32 else 3e-3)
    assert rel_fro(S, S_ref) < TOL


def test_segmented_scan_equals_unsegmented_within_tolerance():
    """Without a workspace the same call runs every sequence in one piece."""
    q, k, v, la, be, S0 = _case(1, 3000, 2, 128, 128, 77, with_s0=True)
    args = (bf16_cuda(q), bf16_cuda(k), bf16_cuda(v), f32_cuda(la), f32_cuda(be))
    o1, S1 = _lib.gdn_delta_rule_fwd(*args, S0=f32_cuda(S0), o_fp32=True)
    o2, S2 = _lib.gdn_delta_rule_fwd(*args, S0=f32_cuda(S0), o_fp32=True, use_workspace=False)
    _lib.stream_check()
    assert rel_fro(to_np(o1), to_np(o2)) < TOL and rel_fro(to_np(S1), to_np(S2)) < TOL


@pytest.mark.parametrize("B,T,H,o_fp32", [(1, 4100, 1, True), (1, 6000, 2, False)], ids=["fp32_o", "bf16_o"])
def test_precomputed_inverse_is_bit_identical(B, T, H, o_fp32):
    """Segmented sequences: with the full workspace a wide pre-pass computes
    every chunk's (I + L)^{-1} and its beta-weighted copy once, with the
    scan's own arithmetic (normalisation, tensor-core K K^T, L rows,
    inverse), and both passes over the segments load them; a workspace short
    of those 16 KB per chunk and head makes each pass invert on its own.
    Both must give the same bits."""
    q, k, v, la, be, S0 = _case(B, T, H, 128, 128, 91 + T, with_s0=True)
    args = (bf16_cuda(q), bf16_cuda(k), bf16_cuda(v), f32_cuda(la), f32_cuda(be))
    full = int(_lib.lib().gdn_delta_rule_workspace_size(B, T, H, 128, 128))
    img = B * ((T + 63) // 64) * H * 16384
    assert full > img
    o1, S1 = _lib.gdn_delta_rule_fwd(*args, S0=f32_cuda(S0), o_fp32=o_fp32, workspace_bytes=full)
    o2, S2 = _lib.gdn_delta_rule_fwd(*args, S0=f32_cuda(S0), o_fp32=o_fp32, workspace_bytes=full - img)
    _lib.stream_check()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    o_ref, S_ref = delta_rule_chunked(q, k, v, la, be, S0=S0)
    if not o_fp32:
        from oracle.nvfp4 import round_bf16
        o_ref = round_bf16(o_ref)
    assert rel_fro(to_np(o1), o_ref) < (TOL if o_fp32 else 3e-3) and rel_fro(to_np(S1), S_ref) < TOL
