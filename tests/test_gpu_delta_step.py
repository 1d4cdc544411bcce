"""GPU parity of the token-by-token recurrence (decode step) against the FP64
sequential oracle.

"Anthology of the SOTA, theory-128", section "The account":
S_t = alpha_t S_{t-1} + beta_t k_t (v_t - S_{t-1}^T k_t)^T, o_t = S_t^T q_t over
L2-normalised q, k; with the decayed-read flag the correction reads
alpha_t S_{t-1}.  The kernel keeps the state in FP32 registers and sums in
FP32: tolerance 1e-5 relative Frobenius on the state and on an FP32 o (a few
FP32 roundings per token over d_k = 128 terms), 5e-3 on a bf16 o against the
oracle's o rounded to bf16 (bf16 rounding alone is ~1.5e-3).
"""
import numpy as np
import pytest
import torch

from nvfp4_w4a4_gated_quant_b200 import _lib, inputs
from oracle.delta_rule import delta_rule_sequential
from oracle.gates import gates as oracle_gates
from oracle.nvfp4 import round_bf16
from tests._helpers import bf16_cuda, f32_cuda, rel_fro, to_np

pytestmark = pytest.mark.gpu
TOL = 1e-5


def _case(B, T, H, dk, dv, seed, with_s0=True):
    rng = np.random.default_rng(seed)
    q = inputs.to_bf16_values(rng.standard_normal((B, T, H, dk), dtype=np.float32))
    k = inputs.to_bf16_values(rng.standard_normal((B, T, H, dk), dtype=np.float32))
    v = inputs.to_bf16_values(rng.standard_normal((B, T, H, dv), dtype=np.float32))
    a = rng.standard_normal((B, T, H)).astype(np.float32)
    b = rng.standard_normal((B, T, H)).astype(np.float32)
    la, be = oracle_gates(a, b, rng.uniform(-2, 1, H), rng.uniform(-1, 1, H))
    S0 = (rng.standard_normal((B, H, dk, dv)) * 0.5).astype(np.float32) if with_s0 else None
    return q, k, v, la.astype(np.float32), be.astype(np.float32), S0


def _step(q, k, v, la, be, S0, decayed=False, o_fp32=True):
    o, S = _lib.gdn_delta_rule_step(bf16_cuda(q), bf16_cuda(k), bf16_cuda(v), f32_cuda(la), f32_cuda(be),
                                    S=None if S0 is None else f32_cuda(S0), o_fp32=o_fp32, decayed_read=decayed)
    _lib.stream_check()
    return to_np(o).astype(np.float64), to_np(S).astype(np.float64)


@pytest.mark.parametrize("B,T,H,dk,dv,seed,decayed", [
    (3, 1, 5, 128, 128, 0, False),
    (3, 1, 5, 128, 128, 0, True),
    (2, 7, 4, 64, 32, 1, False),
    (2, 7, 4, 64, 32, 1, True),
    (1, 3, 2, 32, 64, 2, False),
    (2, 1, 3, 128, 64, 3, True),
    (1, 40, 1, 128, 128, 4, False),
])
def test_step_matches_sequential_oracle(B, T, H, dk, dv, seed, decayed):
    q, k, v, la, be, S0 = _case(B, T, H, dk, dv, seed)
    o, S = _step(q, k, v, la, be, S0, decayed=decayed)
    o_ref, S_ref = delta_rule_sequential(q, k, v, la, be, S0=S0, decayed_read=decayed)
    assert rel_fro(S, S_ref) < TOL
    assert rel_fro(o, o_ref) < TOL


@pytest.mark.parametrize("dk,dv,decayed", [(128, 128, False), (64, 32, True)])
def test_step_element_aligned_state(dk, dv, decayed):
    """A state buffer aligned to its element but not to 16 bytes is copied
    to and from shared memory in 4-byte pieces instead of 16-byte ones; the
    arithmetic is the same, so the results are the same bits as for an
    aligned state, and match the oracle."""
    B, T, H = 2, 3, 3
    q, k, v, la, be, S0 = _case(B, T, H, dk, dv, 11 + dk)
    args = (bf16_cuda(q), bf16_cuda(k), bf16_cuda(v), f32_cuda(la), f32_cuda(be))
    n = B * H * dk * dv
    raw_in = torch.empty(n + 1, dtype=torch.float32, device="cuda")
    raw_out = torch.empty(n + 1, dtype=torch.float32, device="cuda")
    S_in = raw_in[1:].view(B, H, dk, dv)          # 4-byte aligned, not 16
    S_in.copy_(f32_cuda(S0))
    S_out = raw_out[1:].view(B, H, dk, dv)
    o_e, _ = _lib.gdn_delta_rule_step(*args, S=S_in, S_out=S_out, o_fp32=True, decayed_read=decayed)
    o_a, S_a = _lib.gdn_delta_rule_step(*args, S=f32_cuda(S0), o_fp32=True, decayed_read=decayed)
    _lib.stream_check()
    assert torch.equal(o_e, o_a) and torch.equal(S_out, S_a)
    o_ref, S_ref = delta_rule_sequential(q, k, v, la, be, S0=S0, decayed_read=decayed)
    assert rel_fro(to_np(S_a).astype(np.float64), S_ref) < TOL
    assert rel_fro(to_np(o_a).astype(np.float64), o_ref) < TOL


def test_step_bf16_output():
    q, k, v, la, be, S0 = _case(2, 3, 4, 128, 128, 5)
    o, _ = _step(q, k, v, la, be, S0, o_fp32=False)
    o_ref, _ = delta_rule_sequential(q, k, v, la, be, S0=S0)
    assert rel_fro(o, round_bf16(o_ref)) < 5e-3


def test_step_in_place_zero_state_and_empty_call():
    q, k, v, la, be, S0 = _case(2, 2, 3, 128, 64, 6)
    _, S_a = _step(q, k, v, la, be, S0)
    S_dev = f32_cuda(S0)
    _lib.gdn_delta_rule_step(bf16_cuda(q), bf16_cuda(k), bf16_cuda(v), f32_cuda(la), f32_cuda(be), S=S_dev,
                             S_out=S_dev)
    _lib.stream_check()
    np.testing.assert_array_equal(to_np(S_dev).astype(np.float64), S_a)
    # no entry state is a zero state
    o_n, S_n = _step(q, k, v, la, be, None)
    o_z, S_z = _step(q, k, v, la, be, np.zeros_like(S0))
    np.testing.assert_array_equal(S_n, S_z)
    np.testing.assert_array_equal(o_n, o_z)
    # T = 0 copies the state through
    _, S_0 = _step(q[:, :0], k[:, :0], v[:, :0], la[:, :0], be[:, :0], S0)
    np.testing.assert_array_equal(S_0, S0.astype(np.float64))


def test_chunked_prefill_then_decode_steps():
    """A 300-token chunked prefill followed by five decode steps equals the
    sequential oracle over all 305 tokens."""
    B, H, dk, dv = 2, 3, 128, 128
    q, k, v, la, be, S0 = _case(B, 305, H, dk, dv, 7)
    _, S_pre = _lib.gdn_delta_rule_fwd(bf16_cuda(q[:, :300]), bf16_cuda(k[:, :300]), bf16_cuda(v[:, :300]),
                                       f32_cuda(la[:, :300]), f32_cuda(be[:, :300]), S0=f32_cuda(S0), o_fp32=True)
    o_dec, S_end = _lib.gdn_delta_rule_step(bf16_cuda(q[:, 300:]), bf16_cuda(k[:, 300:]), bf16_cuda(v[:, 300:]),
                                            f32_cuda(la[:, 300:]), f32_cuda(be[:, 300:]), S=S_pre, S_out=S_pre,
                                            o_fp32=True)
    _lib.stream_check()
    o_ref, S_ref = delta_rule_sequential(q, k, v, la, be, S0=S0)
    # the prefill's FP16 tensor-core operands bound the error (2e-3, as the scan)
    assert rel_fro(to_np(S_end), S_ref) < 2e-3
    assert rel_fro(to_np(o_dec), o_ref[:, 300:]) < 2e-3


def test_decode_batch_full_size():
    """Decode batch of 64 sequences x 32 heads x d 128, one token, every chain
    against the oracle."""
    B, H, d = 64, 32, 128
    q, k, v, la, be, S0 = _case(B, 1, H, d, d, 8)
    o, S = _step(q, k, v, la, be, S0)
    o_ref, S_ref = delta_rule_sequential(q, k, v, la, be, S0=S0)
    assert rel_fro(S, S_ref) < TOL
    assert rel_fro(o, o_ref) < TOL
