"""GPU parity of the whole layer forward, stage by stage, plus end to end.

Each stage is compared with the oracle fed the GPU's own inputs to that stage
(read from the documented workspace offsets), so a stage's tolerance is its
own: x and o codes / scales bit-exact, projections 1e-3 (bf16 vs bf16), gates
1e-4, o 3e-3 (bf16 storage), y 1e-3.  End to end, with every stage's error
compounding through 4-bit requantisation of o, y is compared with the fully
independent oracle layer at 1e-2 relative Frobenius (4-bit codes of o flip at
rounding boundaries when o moves by its bf16 error; measured 5.5e-3 on the
tiny layer) and the final state at 2e-3, the scan's own tolerance (measured
3.0e-4).
"""
import numpy as np
import pytest
import torch

from nvfp4_w4a4_gated_quant_b200 import _lib, inputs
from oracle import nvfp4
from oracle.delta_rule import delta_rule_chunked
from oracle.gates import gates as oracle_gates
from oracle.gemm import gemm_bf16, gemm_fp64
from oracle.layer import layer_forward, quantize_weights
from tests._helpers import rel_fro, tiled_to_linear, to_np

pytestmark = pytest.mark.gpu


def _ws_views(ws, cfg_dims):
    B, T, D, H, dk, dv = cfg_dims
    cfg = _lib.layer_cfg(B, T, D, H, dk, dv)
    off = _lib.gdn_layer_workspace_offsets(cfg)
    M = B * T
    HV = H * dv
    NQKV = 2 * H * dk + HV
    u8 = ws

    def f32(o, n):
        return u8[o:o + 4 * n].view(torch.float32)

    def b16(o, n):
        return u8[o:o + 2 * n].view(torch.bfloat16)

    return {
        "x_codes": u8[off[_lib.WS_X_CODES]:off[_lib.WS_X_CODES] + M * D // 2].view(M, D // 2),
        "x_scales": u8[off[_lib.WS_X_SCALES]:off[_lib.WS_X_SCALES] + _lib.scales_tiled_bytes(M, D)],
        "x_g": f32(off[_lib.WS_X_G], 1),
        "qkv": b16(off[_lib.WS_QKV], M * NQKV).view(M, NQKV),
        "log_alpha": f32(off[_lib.WS_LOG_ALPHA], M * H).view(M, H),
        "beta": f32(off[_lib.WS_BETA], M * H).view(M, H),
        "o": b16(off[_lib.WS_O], M * HV).view(M, HV),
        "o_codes": u8[off[_lib.WS_O_CODES]:off[_lib.WS_O_CODES] + M * HV // 2].view(M, HV // 2),
        "o_scales": u8[off[_lib.WS_O_SCALES]:off[_lib.WS_O_SCALES] + _lib.scales_tiled_bytes(M, HV)],
        "o_g": f32(off[_lib.WS_O_G], 1),
    }


def _run_layer(d, S0=None):
    B, T, D, H, dk, dv = d["B"], d["T"], d["d_model"], d["H"], d["dk"], d["dv"]
    lw = _lib.QuantizedLayerWeights(d["W"], d["A_log"], d["dt_bias"], H, dk, dv)
    x = torch.from_numpy(d["x"]).cuda().to(torch.bfloat16)
    y, S_T, ws = _lib.gdn_layer_fwd(lw, x, S0=S0)
    _lib.stream_check()
    return y, S_T, _ws_views(ws, (B, T, D, H, dk, dv))


def test_tiny_layer_stagewise_and_end_to_end():
    d = inputs.tiny_layer()
    B, T, D, H, dk, dv = d["B"], d["T"], d["d_model"], d["H"], d["dk"], d["dv"]
    M, HK, HV = B * T, H * dk, H * dv
    y, S_T, v = _run_layer(d)
    Wq = quantize_weights(d["W"])
    # 1. quantize x: bit-exact
    xq = nvfp4.quantize(d["x"].reshape(M, D))
    np.testing.assert_array_equal(to_np(v["x_codes"]), xq["codes"])
    np.testing.assert_array_equal(tiled_to_linear(to_np(v["x_scales"]), M, D), xq["scales"])
    assert to_np(v["x_g"])[0] == xq["g"]
    # 2. projections (bf16 vs bf16)
    qkv = to_np(v["qkv"])
    for i, n in enumerate(("q", "k", "v")):
        lo = i * HK
        hi = lo + (HK if n != "v" else HV)
        assert rel_fro(qkv[:, lo:hi], gemm_bf16(xq, Wq[n])) < 1e-3, n
    # 3. gates
    la_ref, be_ref = oracle_gates(gemm_fp64(xq, Wq["a"]), gemm_fp64(xq, Wq["b"]), d["A_log"], d["dt_bias"])
    np.testing.assert_allclose(to_np(v["log_alpha"]), la_ref, rtol=1e-4, atol=1e-5)
    np.testing.assert_allclose(to_np(v["beta"]), be_ref, rtol=1e-4, atol=1e-5)
    # 4. scan on the GPU's own q, k, v and gates
    q = qkv[:, :HK].reshape(B, T, H, dk)
    k = qkv[:, HK:2 * HK].reshape(B, T, H, dk)
    vv = qkv[:, 2 * HK:].reshape(B, T, H, dv)
    o_ref, S_ref = delta_rule_chunked(q, k, vv, to_np(v["log_alpha"]).reshape(B, T, H),
                                      to_np(v["beta"]).reshape(B, T, H))
    o_gpu = to_np(v["o"])
    assert rel_fro(o_gpu, o_ref.reshape(M, HV)) < 3e-3
    assert rel_fro(to_np(S_T), S_ref) < 2e-3
    # 5. quantize o: bit-exact on the GPU's own o
    oq = nvfp4.quantize(o_gpu.astype(np.float32))
    np.testing.assert_array_equal(to_np(v["o_codes"]), oq["codes"])
    np.testing.assert_array_equal(tiled_to_linear(to_np(v["o_scales"]), M, HV), oq["scales"])
    # 6. output projection on the GPU's own quantized o
    y_gpu = to_np(y).reshape(M, D)
    assert rel_fro(y_gpu, gemm_bf16(oq, Wq["out"])) < 1e-3
    # 7. end to end against the independent oracle layer
    y_ref, S_ref2, _ = layer_forward(d["x"], Wq, d["A_log"], d["dt_bias"], H, dk, dv)
    e2e = rel_fro(y_gpu, y_ref.reshape(M, D))
    print(f"tiny layer end-to-end rel_fro {e2e:.3e}")
    assert e2e < 1e-2
    assert rel_fro(to_np(S_T), S_ref2) < 2e-3


def test_layer_workload_sampled():
    """The layer workload (B=4, T=8192, d_model=5120, H=32, d=128): every stage
    checked on sampled rows / chains against the oracle fed the GPU's inputs."""
    d = inputs.layer_workload()
    B, T, D, H, dk, dv = d["B"], d["T"], d["d_model"], d["H"], d["dk"], d["dv"]
    M, HK, HV = B * T, H * dk, H * dv
    y, S_T, v = _run_layer(d)
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(M, 128, replace=False))
    rows_t = torch.from_numpy(rows).cuda()
    x2 = d["x"].reshape(M, D)
    g_enc = nvfp4.global_encode_scale(nvfp4.tensor_amax(x2))
    xq = nvfp4.quantize(x2[rows], g_enc=g_enc)
    np.testing.assert_array_equal(to_np(v["x_codes"][rows_t]), xq["codes"])
    np.testing.assert_array_equal(tiled_to_linear(to_np(v["x_scales"]), M, D)[rows], xq["scales"])
    Wq = quantize_weights(d["W"])
    qkv = to_np(v["qkv"][rows_t])
    for i, n in enumerate(("q", "k", "v")):
        assert rel_fro(qkv[:, i * HK:(i + 1) * HK], gemm_bf16(xq, Wq[n])) < 1e-3, n
    la_ref, be_ref = oracle_gates(gemm_fp64(xq, Wq["a"]), gemm_fp64(xq, Wq["b"]), d["A_log"], d["dt_bias"])
    np.testing.assert_allclose(to_np(v["log_alpha"][rows_t]), la_ref, rtol=1e-3, atol=1e-4)
    np.testing.assert_allclose(to_np(v["beta"][rows_t]), be_ref, rtol=1e-3, atol=1e-4)
    # scan: 4 sampled (batch, head) chains over the full 8192 tokens
    qkv_all = v["qkv"].view(B, T, -1)
    la_all = to_np(v["log_alpha"]).reshape(B, T, H)
    be_all = to_np(v["beta"]).reshape(B, T, H)
    o_all = v["o"].view(B, T, H, dv)
    for b, h in ((0, 0), (1, 7), (2, 19), (3, 31)):
        q = to_np(qkv_all[b, :, h * dk:(h + 1) * dk])[None, :, None, :]
        k = to_np(qkv_all[b, :, HK + h * dk:HK + (h + 1) * dk])[None, :, None, :]
        vv = to_np(qkv_all[b, :, 2 * HK + h * dv:2 * HK + (h + 1) * dv])[None, :, None, :]
        o_ref, S_ref = delta_rule_chunked(q, k, vv, la_all[b, :, h][None, :, None], be_all[b, :, h][None, :, None])
        assert rel_fro(to_np(o_all[b, :, h]), o_ref[0, :, 0]) < 3e-3
        assert rel_fro(to_np(S_T[b, h]), S_ref[0, 0]) < 2e-3
    o_gpu = to_np(v["o"])
    og_enc = nvfp4.global_encode_scale(nvfp4.tensor_amax(o_gpu))
    oq = nvfp4.quantize(o_gpu[rows].astype(np.float32), g_enc=og_enc)
    np.testing.assert_array_equal(to_np(v["o_codes"][rows_t]), oq["codes"])
    y_gpu = to_np(y.view(M, D)[rows_t])
    assert rel_fro(y_gpu, gemm_bf16(oq, Wq["out"])) < 1e-3


@pytest.mark.parametrize("dims", [
    (2, 200, 512, 4, 128, 128),    # tensor-core scan, 64-column d_v slices, ragged last chunk
    (2, 70, 512, 40, 128, 128),    # tensor-core scan, whole 128-column slices
    (1, 96, 256, 2, 32, 32),       # mma.sync scan: o quantized by a given-scale pass
    (1, 2048, 256, 2, 128, 128),   # tensor-core scan in segments: o quantized in the last phase
], ids=["tc_dvs64", "tc_dvs128", "mma_sync", "tc_segmented"])
def test_layer_static_o_scale(dims):
    """A static encode scale for o (gdn_layer_weights_t.o_g_enc): the scan
    writes o's NVFP4 codes and scales itself.  Given the dynamic run's own
    scale, every byte and y are identical to the dynamic run; given another
    scale, the codes and scales equal the oracle's quantization of the same
    bf16 o with that scale, bit for bit."""
    B, T, D, H, dk, dv = dims
    M, HV = B * T, H * dv
    d = inputs.layer_inputs(B, T, D, H, dk, dv, seed=11)
    lw = _lib.QuantizedLayerWeights(d["W"], d["A_log"], d["dt_bias"], H, dk, dv)
    x = torch.from_numpy(d["x"]).cuda().to(torch.bfloat16)
    y0, S0, ws0 = _lib.gdn_layer_fwd(lw, x)
    _lib.stream_check()
    v0 = _ws_views(ws0, dims)
    o = to_np(v0["o"]).astype(np.float32)
    g_enc = nvfp4.global_encode_scale(nvfp4.tensor_amax(o))
    lw.o_g_enc = torch.tensor([g_enc], dtype=torch.float32, device="cuda")
    y1, S1, ws1 = _lib.gdn_layer_fwd(lw, x)
    _lib.stream_check()
    v1 = _ws_views(ws1, dims)
    assert torch.equal(v1["o"], v0["o"])
    assert torch.equal(v1["o_codes"], v0["o_codes"])
    np.testing.assert_array_equal(tiled_to_linear(to_np(v1["o_scales"]), M, HV),
                                  tiled_to_linear(to_np(v0["o_scales"]), M, HV))
    assert to_np(v1["o_g"])[0] == to_np(v0["o_g"])[0]
    assert torch.equal(y1, y0)
    assert torch.equal(S1, S0)
    # another static scale: compare with the oracle on the same o
    g2 = np.float32(g_enc * np.float32(0.37))
    lw.o_g_enc = torch.tensor([g2], dtype=torch.float32, device="cuda")
    _, _, ws2 = _lib.gdn_layer_fwd(lw, x)
    _lib.stream_check()
    v2 = _ws_views(ws2, dims)
    o2 = to_np(v2["o"]).astype(np.float32)
    ref = nvfp4.quantize(o2, g_enc=g2)
    np.testing.assert_array_equal(to_np(v2["o_codes"]), ref["codes"])
    np.testing.assert_array_equal(tiled_to_linear(to_np(v2["o_scales"]), M, HV), ref["scales"])
    assert to_np(v2["o_g"])[0] == np.float32(ref["g"])
