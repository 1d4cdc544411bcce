"""GPU parity of the short convolution, the gated output norm and the layer
that uses them (the Gated DeltaNet block's outside specification; the oracle
is oracle/conv_norm.py).

Tolerances: the convolution and the norm are FP32 on bf16 storage against the
FP64 oracle rounded to bf16: within one bf16 rounding (2e-3 relative
Frobenius); the carried convolution state is a copy of inputs (exact).  The
layer is checked stage by stage with the oracle fed the GPU's own stage
inputs, and end to end at 2e-2 (o requantized on both sides).
"""
import numpy as np
import pytest
import torch

from nvfp4_w4a4_gated_quant_b200 import _lib, inputs
from oracle import nvfp4
from oracle.conv_norm import gated_rmsnorm, short_conv
from oracle.gemm import gemm_bf16
from oracle.layer import layer_forward, quantize_weights
from tests._helpers import bf16_cuda, f32_cuda, rel_fro, tiled_to_linear, to_np

pytestmark = pytest.mark.gpu


def _bf16(a):
    return nvfp4.round_bf16(a)


@pytest.mark.parametrize("B,T,C,with_state", [(2, 150, 96, False), (1, 64, 8, True), (3, 1, 40, True),
                                              (1, 300, 6176, False)],
                         ids=["ragged", "one_block", "one_token", "layer_width"])
def test_short_conv_matches_oracle(B, T, C, with_state):
    rng = np.random.default_rng(C + T)
    x = inputs.to_bf16_values(rng.standard_normal((B, T, C)).astype(np.float32))
    w = rng.uniform(-0.8, 0.8, (C, 4)).astype(np.float32)
    st = inputs.to_bf16_values(rng.standard_normal((B, 3, C)).astype(np.float32)) if with_state else None
    st_out = torch.full((B, 3, C), float("nan"), dtype=torch.bfloat16, device="cuda")
    y = _lib.gdn_short_conv(bf16_cuda(x), f32_cuda(w), state_in=None if st is None else bf16_cuda(st),
                            state_out=st_out)
    _lib.stream_check()
    y_ref, st_ref = short_conv(x, w, state=st)
    assert rel_fro(to_np(y), _bf16(y_ref)) < 2e-3
    np.testing.assert_array_equal(to_np(st_out), st_ref)


def test_short_conv_carried_state_equals_one_call():
    rng = np.random.default_rng(3)
    B, T, C = 2, 500, 64
    x = bf16_cuda(rng.standard_normal((B, T, C)).astype(np.float32))
    w = f32_cuda(rng.uniform(-1, 1, (C, 4)))
    y_all = _lib.gdn_short_conv(x, w)
    st = torch.empty((B, 3, C), dtype=torch.bfloat16, device="cuda")
    y_a = _lib.gdn_short_conv(x[:, :123].contiguous(), w, state_out=st)
    y_b = _lib.gdn_short_conv(x[:, 123:].contiguous(), w, state_in=st)
    _lib.stream_check()
    assert torch.equal(torch.cat([y_a, y_b], dim=1), y_all)


@pytest.mark.parametrize("M,H,dv", [(333, 3, 128), (64, 2, 64), (17, 5, 32)])
def test_gated_rmsnorm_matches_oracle(M, H, dv):
    rng = np.random.default_rng(M)
    o = inputs.to_bf16_values(rng.standard_normal((M, H * dv)).astype(np.float32) * 3)
    g = inputs.to_bf16_values(rng.standard_normal((M, H * dv)).astype(np.float32))
    gamma = rng.uniform(0.5, 1.5, dv).astype(np.float32)
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    y = _lib.gdn_gated_rmsnorm(bf16_cuda(o), bf16_cuda(g), f32_cuda(gamma), H, amax=amax)
    _lib.stream_check()
    ref = gated_rmsnorm(o.reshape(M, H, dv), g.reshape(M, H, dv), gamma).reshape(M, H * dv)
    assert rel_fro(to_np(y), _bf16(ref)) < 2e-3
    assert to_np(amax)[0] == np.abs(to_np(y)).max()


@pytest.mark.parametrize("dims", [(1, 200, 256, 2, 128, 128), (2, 96, 256, 2, 32, 32)], ids=["tc", "mma_sync"])
def test_layer_with_conv_and_output_gate(dims):
    B, T, D, H, dk, dv = dims
    M, HK, HV = B * T, H * dk, H * dv
    NQKV = 2 * HK + HV
    d = inputs.layer_inputs(B, T, D, H, dk, dv, seed=31)
    rng = np.random.default_rng(32)
    W = dict(d["W"])
    W["g"] = inputs.weight(rng, HV, D)
    conv_w = rng.uniform(-0.6, 0.6, (NQKV, 4)).astype(np.float32)
    norm_w = rng.uniform(0.5, 1.5, dv).astype(np.float32)
    lw = _lib.QuantizedLayerWeights(W, d["A_log"], d["dt_bias"], H, dk, dv, conv_w=conv_w, norm_w=norm_w)
    x = torch.from_numpy(d["x"]).cuda().to(torch.bfloat16)
    y, S_T, ws = _lib.gdn_layer_fwd(lw, x)
    _lib.stream_check()
    off = _lib.gdn_layer_workspace_offsets(lw.cfg(B, T))

    def b16(i, n, cols):
        return to_np(ws[off[i]:off[i] + n * 2].view(torch.bfloat16).view(-1, cols))

    Wq = quantize_weights(W)
    xq = nvfp4.quantize(d["x"].reshape(M, D))
    qkv = b16(_lib.WS_QKV, M * NQKV, NQKV)
    g = b16(_lib.WS_G, M * HV, HV)
    assert rel_fro(g, gemm_bf16(xq, Wq["g"])) < 1e-3
    # the convolution on the GPU's own projections
    qkv_c = b16(_lib.WS_QKV_CONV, M * NQKV, NQKV)
    ref_c = _bf16(short_conv(qkv.reshape(B, T, NQKV), conv_w)[0]).reshape(M, NQKV)
    assert rel_fro(qkv_c, ref_c) < 2e-3
    # the gated norm on the GPU's own o and g, and its quantization
    o = b16(_lib.WS_O, M * HV, HV)
    og = b16(_lib.WS_O_GATED, M * HV, HV)
    ref_g = _bf16(gated_rmsnorm(o.reshape(M, H, dv), g.reshape(M, H, dv), norm_w)).reshape(M, HV)
    assert rel_fro(og, ref_g) < 2e-3
    oq = nvfp4.quantize(og.astype(np.float32))
    o_codes = to_np(ws[off[_lib.WS_O_CODES]:off[_lib.WS_O_CODES] + M * HV // 2].view(M, HV // 2))
    np.testing.assert_array_equal(o_codes, oq["codes"])
    assert rel_fro(to_np(y).reshape(M, D), gemm_bf16(oq, Wq["out"])) < 1e-3
    # end to end against the oracle layer with the same block
    y_ref, S_ref, _ = layer_forward(d["x"], Wq, d["A_log"], d["dt_bias"], H, dk, dv, conv_w=conv_w, norm_w=norm_w)
    e2e = rel_fro(to_np(y).reshape(M, D), y_ref.reshape(M, D))
    print(f"layer with convolution and output gate: y within {e2e:.2e} of the oracle")
    assert e2e < 2e-2
    assert rel_fro(to_np(S_T), S_ref) < 2e-3
