"""Per-module calibration of static activation scales ("Why Gated DeltaNet
Survives 4-Bit Quantization", section "Critical Lessons for Model Serving":
activation scales are calibrated for each module on its own, and fusing
modules must not mix up their global scales).

The layer quantizes two activations, x (the input of the fused q/k/v/a/b
projection) and o (the input of the output projection).  Each gets its own
calibrated scale: the encode scale of the largest |value| that module saw over
the calibration batches.  With those scales the layer must match the oracle
layer run with the same per-module scales (codes and scales bit-exact where
the inputs agree); handing each module the other's scale -- the pitfall the
page warns about -- visibly breaks the output.
"""
import numpy as np
import pytest
import torch

from nvfp4_w4a4_gated_quant_b200 import _lib, inputs
from oracle import nvfp4
from oracle.gemm import gemm_bf16
from oracle.layer import layer_forward, quantize_weights
from tests._helpers import bf16_cuda, f32_cuda, rel_fro, tiled_to_linear, to_np

pytestmark = pytest.mark.gpu


def test_amax_update_is_a_running_max_and_the_encode_scale_matches():
    rng = np.random.default_rng(5)
    batches = [inputs.activations(rng, (r, 320)) for r in (100, 257, 1)]
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    for b in batches:
        _lib.gdn_amax_update(bf16_cuda(b), amax)
    w = inputs.weight(rng, 64, 320) * 1e3             # an FP32 tensor with a larger amax
    _lib.gdn_amax_update(f32_cuda(w), amax)
    _lib.gdn_amax_update(bf16_cuda(np.zeros((0, 320), np.float32)), amax)     # empty: unchanged
    _lib.stream_check()
    want = max(max(nvfp4.tensor_amax(b) for b in batches), nvfp4.tensor_amax(w))
    assert to_np(amax)[0] == want
    g = _lib.gdn_encode_scale_from_amax(amax)
    _lib.stream_check()
    assert to_np(g)[0] == nvfp4.global_encode_scale(want)
    z = _lib.gdn_encode_scale_from_amax(torch.zeros(1, dtype=torch.float32, device="cuda"))
    assert to_np(z)[0] == np.float32(1.0)


@pytest.mark.parametrize("dims", [(2, 200, 512, 4, 128, 128), (1, 96, 256, 2, 32, 32)], ids=["tc", "mma_sync"])
def test_layer_with_per_module_calibrated_scales(dims):
    B, T, D, H, dk, dv = dims
    M, HV = B * T, H * dv
    d = inputs.layer_inputs(B, T, D, H, dk, dv, seed=21)
    lw = _lib.QuantizedLayerWeights(d["W"], d["A_log"], d["dt_bias"], H, dk, dv)
    rng = np.random.default_rng(22)
    cal = [torch.from_numpy(inputs.activations(rng, (B, T, D))).cuda().to(torch.bfloat16) for _ in range(2)]
    x_g, o_g = _lib.calibrate_layer(lw, cal)
    _lib.stream_check()
    # x's scale: the calibration batches' amax, bit for bit
    x_amax = max(nvfp4.tensor_amax(to_np(c).reshape(-1, D)) for c in cal)
    assert to_np(x_g)[0] == nvfp4.global_encode_scale(x_amax)
    # o's scale: the amax of the layer's own o on those batches
    o_amax = np.float32(0.0)
    for c in cal:
        _, _, ws = _lib.gdn_layer_fwd(lw, c, want_state=False)
        off = _lib.gdn_layer_workspace_offsets(_lib.layer_cfg(B, T, D, H, dk, dv))
        o = ws[off[_lib.WS_O]:off[_lib.WS_O] + M * HV * 2].view(torch.bfloat16).view(M, HV)
        o_amax = max(o_amax, nvfp4.tensor_amax(to_np(o)))
    assert to_np(o_g)[0] == nvfp4.global_encode_scale(o_amax)

    # the layer on a new batch with both static scales
    lw.x_g_enc, lw.o_g_enc = x_g, o_g
    x = torch.from_numpy(d["x"]).cuda().to(torch.bfloat16)
    y, S_T, ws = _lib.gdn_layer_fwd(lw, x)
    _lib.stream_check()
    off = _lib.gdn_layer_workspace_offsets(_lib.layer_cfg(B, T, D, H, dk, dv))
    xs = to_np(x_g)[0]
    os_ = to_np(o_g)[0]
    xq = nvfp4.quantize(d["x"].reshape(M, D), g_enc=xs)
    x_codes = ws[off[_lib.WS_X_CODES]:off[_lib.WS_X_CODES] + M * D // 2].view(M, D // 2)
    x_scales = ws[off[_lib.WS_X_SCALES]:off[_lib.WS_X_SCALES] + _lib.scales_tiled_bytes(M, D)]
    np.testing.assert_array_equal(to_np(x_codes), xq["codes"])
    np.testing.assert_array_equal(tiled_to_linear(to_np(x_scales), M, D), xq["scales"])
    o = to_np(ws[off[_lib.WS_O]:off[_lib.WS_O] + M * HV * 2].view(torch.bfloat16).view(M, HV))
    oq = nvfp4.quantize(o.astype(np.float32), g_enc=os_)
    o_codes = ws[off[_lib.WS_O_CODES]:off[_lib.WS_O_CODES] + M * HV // 2].view(M, HV // 2)
    o_scales = ws[off[_lib.WS_O_SCALES]:off[_lib.WS_O_SCALES] + _lib.scales_tiled_bytes(M, HV)]
    np.testing.assert_array_equal(to_np(o_codes), oq["codes"])
    np.testing.assert_array_equal(tiled_to_linear(to_np(o_scales), M, HV), oq["scales"])
    Wq = quantize_weights(d["W"])
    y_gpu = to_np(y).reshape(M, D)
    assert rel_fro(y_gpu, gemm_bf16(oq, Wq["out"])) < 1e-3
    # end to end against the oracle layer with the same per-module scales: the
    # stages above are exact or within 1e-3; what remains is o requantized on
    # both sides from values that differ by the scan's error, so 4-bit codes
    # flip at rounding boundaries (2e-2 here; the tiny layer measures 5.5e-3)
    y_ref, S_ref, _ = layer_forward(d["x"], Wq, d["A_log"], d["dt_bias"], H, dk, dv, x_g_enc=xs, o_g_enc=os_)
    e2e = rel_fro(y_gpu, y_ref.reshape(M, D))
    assert e2e < 2e-2 and rel_fro(to_np(S_T), S_ref) < 2e-3

    # the pitfall: each module handed the other module's scale
    lw.x_g_enc, lw.o_g_enc = o_g, x_g
    y_mixed, _, _ = _lib.gdn_layer_fwd(lw, x)
    _lib.stream_check()
    e_mixed = rel_fro(to_np(y_mixed).reshape(M, D), y_ref.reshape(M, D))
    print(f"per-module scales: y within {e2e:.2e} of the oracle; mixed-up scales: {e_mixed:.2e}")
    # o's small scale on x saturates the block scales of x's outlier blocks and
    # clips every |x| above the E2M1 range: a visible corruption
    assert e_mixed > 0.1
