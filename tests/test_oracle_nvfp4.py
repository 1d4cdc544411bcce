"""Pins for the NVFP4 part of the oracle (CPU only).

Each test checks the oracle against something other than itself: the format
definitions worked by hand (tests/golden), brute-force nearest-value search,
torch's own float8_e4m3fn conversion, and the block-localisation property the
pages state ("Why Gated DeltaNet Survives 4-Bit Quantization", section "Why the
'Fragile' Recurrence is Actually Robust": an outlier's error stays inside its
own 16-element block).
"""
import os

import numpy as np
import pytest
import torch

from oracle import nvfp4

E2M1_MAGS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _read_pairs(path, conv):
    out = []
    with open(path) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                a, b = line.split()
                out.append((float(a), conv(b)))
    return out


def test_e2m1_decode_table():
    codes = np.arange(16)
    vals = nvfp4.e2m1_decode(codes)
    np.testing.assert_array_equal(np.abs(vals[:8]), E2M1_MAGS)
    np.testing.assert_array_equal(vals[8:], -E2M1_MAGS)
    assert np.signbit(vals[8])


def test_e2m1_roundtrip_all_codes():
    codes = np.arange(16, dtype=np.uint8)
    vals = nvfp4.e2m1_decode(codes).astype(np.float32)
    back = nvfp4.e2m1_encode(vals)
    np.testing.assert_array_equal(back, codes)


def test_e2m1_golden(golden_dir):
    cases = _read_pairs(os.path.join(golden_dir, "e2m1_rounding.txt"), int)
    x = np.array([c[0] for c in cases], np.float32)
    want = np.array([c[1] for c in cases], np.uint8)
    np.testing.assert_array_equal(nvfp4.e2m1_encode(x), want)


def _nearest_even(vals, table_mags, codes_of_mags):
    """Brute force: nearest magnitude in the table, ties to the even code."""
    out = []
    for v in vals:
        m = abs(float(v))
        d = np.abs(table_mags - m)
        best = np.flatnonzero(d == d.min())
        if len(best) > 1:
            best = [b for b in best if codes_of_mags[b] % 2 == 0]
        out.append(best[0])
    return np.array(out)


def test_e2m1_brute_force_random():
    rng = np.random.default_rng(123)
    x = (rng.standard_normal(20000) * 3).astype(np.float32)
    x = np.concatenate([x, np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)])
    idx = _nearest_even(x, E2M1_MAGS, np.arange(8))
    got = nvfp4.e2m1_encode(x)
    np.testing.assert_array_equal(got & 7, idx)
    np.testing.assert_array_equal(got >> 3, np.signbit(x).astype(np.uint8))


def test_e4m3_roundtrip_all_finite_and_torch_decode():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    assert len(codes) == 254
    vals = nvfp4.e4m3_decode(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(vals, ref)
    back = nvfp4.e4m3_encode(vals.astype(np.float32))
    # +0 and -0 both decode to a zero; -0 re-encodes to +0 (scales are >= 0)
    want = codes.copy()
    want[codes == 0x80] = 0x00
    np.testing.assert_array_equal(back, want)
    assert np.isnan(nvfp4.e4m3_decode(np.array([0x7F])))[0]


def test_e4m3_golden(golden_dir):
    cases = _read_pairs(os.path.join(golden_dir, "e4m3_rounding.txt"), lambda s: int(s, 16))
    x = np.array([c[0] for c in cases], np.float32)
    want = np.array([c[1] for c in cases], np.uint8)
    np.testing.assert_array_equal(nvfp4.e4m3_encode(x), want)


def test_e4m3_matches_torch_in_range():
    rng = np.random.default_rng(7)
    x = np.exp(rng.uniform(np.log(1e-4), np.log(448.0), 50000)).astype(np.float32)
    ties = (nvfp4.e4m3_decode(np.arange(0, 0x7E)) + nvfp4.e4m3_decode(np.arange(1, 0x7F))) / 2
    x = np.concatenate([x, ties.astype(np.float32)])
    got = nvfp4.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(got, ref)


def test_e4m3_saturates():
    x = np.array([448.0, 460.0, 464.0, 500.0, 1e30], np.float32)
    np.testing.assert_array_equal(nvfp4.e4m3_encode(x), np.full(5, 0x7E, np.uint8))


def test_round_bf16_matches_torch():
    rng = np.random.default_rng(11)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(nvfp4.round_bf16(x.astype(np.float64)), ref)


def test_packing_low_nibble_first():
    x = np.zeros((1, 16), np.float32)
    x[0, 0] = 6.0      # -> code 7 in the low nibble of byte 0
    x[0, 1] = -3.0     # -> code 13 in the high nibble of byte 0
    q = nvfp4.quantize(x)
    assert q["codes"][0, 0] == (7 | (13 << 4))
    np.testing.assert_array_equal(nvfp4.unpack_codes(q["codes"])[0, :2], [7, 13])


def test_zero_tensor():
    q = nvfp4.quantize(np.zeros((3, 32), np.float32))
    assert q["g_enc"] == np.float32(1.0) and q["g"] == np.float32(1.0)
    assert not q["codes"].any() and not q["scales"].any()


def test_global_scale_definition():
    # amax 2688 -> g_enc 1 exactly; amax 1 -> g_enc 2688; decode = 1 / encode
    assert nvfp4.global_encode_scale(np.float32(2688.0)) == np.float32(1.0)
    assert nvfp4.global_encode_scale(np.float32(1.0)) == np.float32(2688.0)
    q = nvfp4.quantize(np.full((1, 16), 2.0, np.float32))
    assert q["g_enc"] == np.float32(1344.0)
    assert q["g"] == np.float32(np.float32(1.0) / np.float32(1344.0))
    # the block amax maps to the largest code: s = E4M3(2/6 * 1344) = 448
    assert q["scales"][0, 0] == 0x7E
    np.testing.assert_array_equal(nvfp4.unpack_codes(q["codes"])[0], np.full(16, 7))


def test_dequant_error_bound():
    """|x - x_hat| <= half the E2M1 spacing at x's magnitude, in units of the
    block's decode scale s_val * g (2 at the top binade), plus the saturation
    excess when the E4M3 scale rounded down."""
    rng = np.random.default_rng(5)
    x = nvfp4.round_bf16(rng.standard_normal((64, 256)) * 3).astype(np.float32)
    q = nvfp4.quantize(x)
    xh = nvfp4.dequantize(q["codes"], q["scales"], q["g"])
    unit = (nvfp4.e4m3_decode(q["scales"]) * np.float64(q["g"]))
    unit = np.repeat(unit, 16, axis=1)
    r = np.abs(x) / unit
    half = np.where(r < 2, 0.25, np.where(r < 4, 0.5, 1.0))
    # 1e-6 relative slack: the quantizer forms x * inv in FP32, not exactly
    bound = half * unit + np.maximum(r - 6.0, 0) * unit + 1e-6 * np.abs(x)
    assert np.all(np.abs(x - xh) <= bound)
    # relative error of the whole tensor is the usual few percent of 4-bit
    rel = np.linalg.norm(x - xh) / np.linalg.norm(x)
    assert 0.02 < rel < 0.15


def test_outlier_localised_to_its_block_given_scale():
    """With a fixed per-tensor scale, a x50 outlier changes the codes and the
    scale of exactly one 16-element block."""
    rng = np.random.default_rng(9)
    x = nvfp4.round_bf16(rng.standard_normal((8, 128))).astype(np.float32)
    g_enc = nvfp4.global_encode_scale(np.float32(50 * np.abs(x).max()))
    base = nvfp4.quantize(x, g_enc=g_enc)
    x2 = x.copy()
    x2[3, 37] *= 50
    pert = nvfp4.quantize(x2, g_enc=g_enc)
    dc = nvfp4.unpack_codes(base["codes"]) != nvfp4.unpack_codes(pert["codes"])
    blocks_changed = np.unique(np.argwhere(dc)[:, 0] * 8 + np.argwhere(dc)[:, 1] // 16)
    assert set(blocks_changed.tolist()) <= {3 * 8 + 37 // 16}
    ds = base["scales"] != pert["scales"]
    assert np.argwhere(ds).tolist() == [[3, 37 // 16]]


def test_outlier_dynamic_scale_other_blocks_keep_accuracy():
    """Dynamic mode: the outlier raises amax_t, so other blocks change only
    through g; their dequantised values stay within the half-step bound."""
    rng = np.random.default_rng(10)
    x = nvfp4.round_bf16(rng.standard_normal((8, 128))).astype(np.float32)
    x[2, 5] *= 50
    q = nvfp4.quantize(x)
    xh = nvfp4.dequantize(q["codes"], q["scales"], q["g"])
    mask = np.ones_like(x, bool)
    mask[2, 0:16] = False
    rel = np.linalg.norm((x - xh)[mask]) / np.linalg.norm(x[mask])
    assert rel < 0.12


@pytest.mark.parametrize("shape", [(1, 16), (5, 48), (130, 64)])
def test_quantize_shapes_and_dtypes(shape):
    rng = np.random.default_rng(1)
    x = nvfp4.round_bf16(rng.standard_normal(shape)).astype(np.float32)
    q = nvfp4.quantize(x)
    assert q["codes"].shape == (shape[0], shape[1] // 2) and q["codes"].dtype == np.uint8
    assert q["scales"].shape == (shape[0], shape[1] // 16) and q["scales"].dtype == np.uint8
    assert not np.any(q["scales"] & 0x80)
