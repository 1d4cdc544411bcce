"""GPU parity of step 1 (NVFP4 quantizer, bit-exact) and step 3 (gates).

Quantizer: codes, scales and the FP32 decode scale must equal the oracle's bit
for bit ("Why Gated DeltaNet Survives 4-Bit Quantization", section "Why the
'Fragile' Recurrence is Actually Robust": 16-element block scaling).
Gates ("Anthology of the SOTA, theory-128", section "The account"): FP32 with
accurate expf / log1pf against the FP64 oracle, tolerance 2e-6 relative
(a few FP32 ulps).
"""
import numpy as np
import pytest
import torch

from nvfp4_w4a4_gated_quant_b200 import _lib, inputs
from oracle import nvfp4
from oracle.gates import gates as oracle_gates
from tests._helpers import f32_cuda, tiled_to_linear, to_np

pytestmark = pytest.mark.gpu


def _check_quant(x_np, x_dev, g_enc=None, layout="tiled"):
    g_dev = None if g_enc is None else torch.tensor([g_enc], dtype=torch.float32, device="cuda")
    codes, scales, g = _lib.gdn_quantize_nvfp4(x_dev, g_enc=g_dev, layout=layout)
    torch.cuda.synchronize()
    ref = nvfp4.quantize(x_np, g_enc=g_enc)
    rows, cols = x_np.shape
    got_scales = to_np(scales)
    got_scales = tiled_to_linear(got_scales, rows, cols) if layout == "tiled" else got_scales.reshape(rows, cols // 16)
    np.testing.assert_array_equal(to_np(codes), ref["codes"])
    np.testing.assert_array_equal(got_scales, ref["scales"])
    assert to_np(g)[0].view(np.uint32) == np.float32(ref["g"]).view(np.uint32)
    return codes, scales, g


@pytest.mark.parametrize("rows,cols,seed", [(64, 256, 0), (130, 320, 1), (1, 64, 2), (300, 5120, 3)])
def test_quantize_bf16_bit_exact(rows, cols, seed):
    x = inputs.activations(np.random.default_rng(seed), (rows, cols))
    _check_quant(x, torch.from_numpy(x).cuda().to(torch.bfloat16))


def test_quantize_linear_layout_and_given_scale():
    x = inputs.activations(np.random.default_rng(5), (96, 192))
    xd = torch.from_numpy(x).cuda().to(torch.bfloat16)
    _check_quant(x, xd, layout="linear")
    _check_quant(x, xd, g_enc=np.float32(37.5))


def test_quantize_given_amax_equals_dynamic():
    """Given-amax mode (the amax recorded by the producer of the tensor) gives
    the dynamic result without the amax pass."""
    x = inputs.activations(np.random.default_rng(12), (257, 320))
    xd = torch.from_numpy(x).cuda().to(torch.bfloat16)
    amax = torch.tensor([float(np.abs(x).max())], dtype=torch.float32, device="cuda")
    c1, s1, g1 = _lib.gdn_quantize_nvfp4(xd)
    c2, s2, g2 = _lib.gdn_quantize_nvfp4(xd, amax=amax)
    torch.cuda.synchronize()
    assert torch.equal(c1, c2) and torch.equal(s1, s2) and torch.equal(g1, g2)
    ref = nvfp4.quantize(x)
    np.testing.assert_array_equal(to_np(c2), ref["codes"])


def test_quantize_fp32_weights_bit_exact():
    w = inputs.weight(np.random.default_rng(6), 200, 256)
    _check_quant(w, f32_cuda(w))


def test_quantize_ties_signed_zero_and_saturation():
    """With g_enc = 1 and a block maximum of 6 the block scale is exactly 1,
    so x * inv = x hits every E2M1 tie point, -0, tiny negatives and the
    saturation edge."""
    row = np.array([6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -5.0, 0.0, -0.0, 0.1, -0.1, 4.9],
                   np.float32)
    x = np.stack([row, row * 2, row * 0.5, np.zeros(16, np.float32)]).astype(np.float32)
    x = inputs.to_bf16_values(np.concatenate([x, x, x, x], axis=1))    # 4 x 64
    _check_quant(x, torch.from_numpy(x).cuda().to(torch.bfloat16), g_enc=np.float32(1.0))
    _check_quant(x, torch.from_numpy(x).cuda().to(torch.bfloat16), layout="linear")


def test_quantize_zero_and_empty():
    z = np.zeros((3, 64), np.float32)
    _check_quant(z, torch.zeros((3, 64), dtype=torch.bfloat16, device="cuda"))
    codes, scales, g = _lib.gdn_quantize_nvfp4(torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    assert to_np(g)[0] == 1.0


def test_quantize_shared_tiled_buffer_row_offsets():
    """Separately scaled projections written into one tiled operand keep their
    own decode scales (the fused-module global-scale pitfall)."""
    rng = np.random.default_rng(8)
    parts = [inputs.weight(rng, n, 128) * s for n, s in ((64, 1.0), (32, 5.0), (2, 0.1), (2, 30.0))]
    total = sum(p.shape[0] for p in parts)
    codes = torch.empty((total, 64), dtype=torch.uint8, device="cuda")
    scales = torch.zeros(_lib.scales_tiled_bytes(total, 128), dtype=torch.uint8, device="cuda")
    gs, r0 = [], 0
    for p in parts:
        _, _, g = _lib.gdn_quantize_nvfp4(f32_cuda(p), codes=codes[r0:r0 + p.shape[0]], scales=scales,
                                          sf_row_offset=r0)
        gs.append(g)
        r0 += p.shape[0]
    torch.cuda.synchronize()
    lin = tiled_to_linear(to_np(scales), total, 128)
    r0 = 0
    for p, g in zip(parts, gs):
        ref = nvfp4.quantize(p)
        n = p.shape[0]
        np.testing.assert_array_equal(to_np(codes)[r0:r0 + n], ref["codes"])
        np.testing.assert_array_equal(lin[r0:r0 + n], ref["scales"])
        assert to_np(g)[0] == ref["g"]
        r0 += n


def test_quantize_full_layer_activation_sampled_rows():
    """x of the layer workload (4 x 8192 tokens x 5120): the full tensor on the
    GPU, the oracle on 256 sampled rows with the tensor's own amax."""
    x = inputs.layer_workload()["x"].reshape(-1, 5120)
    xd = torch.from_numpy(x).cuda().to(torch.bfloat16)
    codes, scales, g = _lib.gdn_quantize_nvfp4(xd)
    torch.cuda.synchronize()
    amax = nvfp4.tensor_amax(x)
    g_enc = nvfp4.global_encode_scale(amax)
    rows = np.sort(np.random.default_rng(0).choice(x.shape[0], 256, replace=False))
    ref = nvfp4.quantize(x[rows], g_enc=g_enc)
    np.testing.assert_array_equal(to_np(codes[torch.from_numpy(rows).cuda()]), ref["codes"])
    lin = tiled_to_linear(to_np(scales), x.shape[0], 5120)
    np.testing.assert_array_equal(lin[rows], ref["scales"])
    assert to_np(g)[0] == np.float32(np.float32(1) / g_enc)


@pytest.mark.parametrize("rows,cols", [(32768, 5120), (4099, 320), (1000, 5120), (7, 64)])
def test_quantize_dynamic_visits_every_row_once(rows, cols):
    """The dynamic path (amax pass, then quant pass) and the given-amax path
    (quant pass only) must, with the same amax, write the same codes and
    scales into buffers that start out different: no row is skipped or
    written from another row, at the layer's size and at ragged ones."""
    if rows == 32768:
        x = inputs.layer_workload()["x"].reshape(-1, 5120)
    else:
        x = inputs.activations(np.random.default_rng(rows), (rows, cols))
    xd = torch.from_numpy(x).cuda().to(torch.bfloat16)
    nsf = _lib.scales_tiled_bytes(rows, cols)
    c_dyn = torch.zeros((rows, cols // 2), dtype=torch.uint8, device="cuda")
    s_dyn = torch.zeros(nsf, dtype=torch.uint8, device="cuda")
    c_amx = torch.full((rows, cols // 2), 0xFF, dtype=torch.uint8, device="cuda")
    s_amx = torch.full((nsf,), 0xFF, dtype=torch.uint8, device="cuda")
    _, _, g_dyn = _lib.gdn_quantize_nvfp4(xd, codes=c_dyn, scales=s_dyn)
    amax = xd.float().abs().amax().reshape(1)
    _, _, g_amx = _lib.gdn_quantize_nvfp4(xd, codes=c_amx, scales=s_amx, amax=amax)
    torch.cuda.synchronize()
    assert torch.equal(c_dyn, c_amx)
    # tiled padding rows past `rows` are never written; compare the real ones
    lin_dyn = tiled_to_linear(to_np(s_dyn), rows, cols)
    lin_amx = tiled_to_linear(to_np(s_amx), rows, cols)
    np.testing.assert_array_equal(lin_dyn, lin_amx)
    assert to_np(g_dyn)[0].view(np.uint32) == to_np(g_amx)[0].view(np.uint32)


# ------------------------------------------------------------------ gates --
def test_gates_against_oracle():
    rng = np.random.default_rng(11)
    M, H = 4099, 7
    a = (rng.standard_normal((M, H)) * 4).astype(np.float32)
    b = (rng.standard_normal((M, H)) * 4).astype(np.float32)
    A = rng.uniform(-2, 1, H).astype(np.float32)
    dt = rng.uniform(-1, 1, H).astype(np.float32)
    la, be = _lib.gdn_gates(f32_cuda(a), f32_cuda(b), f32_cuda(A), f32_cuda(dt))
    torch.cuda.synchronize()
    la_ref, be_ref = oracle_gates(a, b, A, dt)
    np.testing.assert_allclose(to_np(la), la_ref, rtol=2e-6, atol=1e-30)
    np.testing.assert_allclose(to_np(be), be_ref, rtol=2e-6, atol=1e-30)
    # 1 - alpha keeps its accuracy too (where the decay is weak)
    np.testing.assert_allclose(-np.expm1(to_np(la).astype(np.float64)), -np.expm1(la_ref), rtol=5e-6)


def test_gates_special_values():
    a = np.zeros((1, 2), np.float32)
    A = np.array([0.0, np.log(2.0)], np.float32)
    la, be = _lib.gdn_gates(f32_cuda(a), f32_cuda(a), f32_cuda(A), f32_cuda(np.zeros(2, np.float32)))
    torch.cuda.synchronize()
    np.testing.assert_allclose(np.exp(to_np(la)[0].astype(np.float64)), [0.5, 0.25], rtol=1e-6)
    assert np.all(to_np(be) == 0.5)
