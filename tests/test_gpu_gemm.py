"""GPU parity of step 2, the block-scaled NVFP4 GEMM, against the FP64 oracle.

Tolerance: 1e-3 relative Frobenius on the bf16 output against the oracle's
bf16-rounded FP64 product (bf16 rounding alone is ~1.5e-3 against the exact
value, so the comparison is bf16-vs-bf16); FP32 outputs within 1e-5 of the
FP64 product.  Gate segments: the epilogue's gates against the oracle gates of
the FP64 projections.
"""
import numpy as np
import pytest
import torch

from nvfp4_w4a4_gated_quant_b200 import _lib, inputs
from oracle import nvfp4
from oracle.gates import gates as oracle_gates
from oracle.gemm import gemm_bf16, gemm_fp64
from tests._helpers import bf16_cuda, f32_cuda, rel_fro, to_np

pytestmark = pytest.mark.gpu


def _quant_dev(x, bf16=True):
    xd = bf16_cuda(x) if bf16 else f32_cuda(x)
    return _lib.gdn_quantize_nvfp4(xd)


def test_one_hot_layout():
    """A single nonzero code in A (row 77, k 300) and in B (row 200, k 300)
    gives exactly one nonzero output at (77, 200)."""
    M, N, K = 130, 260, 512
    a = np.zeros((M, K), np.float32)
    b = np.zeros((N, K), np.float32)
    a[77, 300] = 3.0
    b[200, 300] = -2.0
    b[13, 301] = 2.0          # same K block, other column: must not touch row 77
    ac, as_, ga = _quant_dev(a)
    bc, bs, gb = _quant_dev(b, bf16=False)
    y = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    _lib.gdn_gemm_nvfp4(ac, as_, ga, bc, bs, M, N, K,
                        [{"n_begin": 0, "n_end": N, "kind": _lib.EPI_STORE_F32, "g_b": gb, "out": y, "ld_out": N}])
    _lib.stream_check()
    yn = to_np(y)
    ref = gemm_fp64(nvfp4.quantize(a), nvfp4.quantize(b))
    assert np.count_nonzero(yn) == np.count_nonzero(ref) == 1
    np.testing.assert_allclose(yn, ref, rtol=1e-6)


@pytest.mark.parametrize("M,N,K,seed", [(64, 196, 256, 0), (200, 300, 320, 1), (257, 513, 1024, 2),
                                        (128, 256, 64, 3), (5, 12, 192, 4),
                                        # row strides of a multiple of 16 bytes: the TMA-store epilogue,
                                        # with ragged rows clipped by the tensor map
                                        (300, 384, 512, 6), (1000, 1024, 256, 7), (77, 640, 1280, 8)])
def test_gemm_matches_oracle(M, N, K, seed):
    rng = np.random.default_rng(seed)
    x = inputs.activations(rng, (M, K))
    w = inputs.weight(rng, N, K)
    xc, xs, gx = _quant_dev(x)
    wc, ws, gw = _quant_dev(w, bf16=False)
    y = _lib.gemm_bf16(xc, xs, gx, wc, ws, gw, M, N, K)
    y32 = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    _lib.gdn_gemm_nvfp4(xc, xs, gx, wc, ws, M, N, K,
                        [{"n_begin": 0, "n_end": N, "kind": _lib.EPI_STORE_F32, "g_b": gw, "out": y32, "ld_out": N}])
    _lib.stream_check()
    xq, wq = nvfp4.quantize(x), nvfp4.quantize(w)
    assert rel_fro(to_np(y), gemm_bf16(xq, wq)) < 1e-3
    assert rel_fro(to_np(y32), gemm_fp64(xq, wq)) < 1e-5


def test_fused_projection_segments_and_gates():
    """q | k | v | a | b in one GEMM, each weight quantized with its own
    decode scale (scales spread over three orders of magnitude), gates in the
    epilogue, bf16 outputs at an offset inside a shared buffer."""
    rng = np.random.default_rng(21)
    M, D, H, dk = 150, 256, 2, 32
    x = inputs.activations(rng, (M, D))
    W = {"q": inputs.weight(rng, H * dk, D), "k": inputs.weight(rng, H * dk, D) * 30,
         "v": inputs.weight(rng, H * dk, D) * 0.05, "a": inputs.weight(rng, H, D) * 3,
         "b": inputs.weight(rng, H, D)}
    A = rng.uniform(-1, 1, H).astype(np.float32)
    dt = rng.uniform(-1, 1, H).astype(np.float32)
    lw = _lib.QuantizedLayerWeights({**W, "out": inputs.weight(rng, D, H * dk)}, A, dt, H, dk, dk)
    xc, xs, gx = _quant_dev(x)
    HK = H * dk
    NQKV = 3 * HK
    qkv = torch.zeros((M, NQKV), dtype=torch.bfloat16, device="cuda")
    la = torch.zeros((M, H), dtype=torch.float32, device="cuda")
    be = torch.zeros((M, H), dtype=torch.float32, device="cuda")
    segs = [
        {"n_begin": 0, "n_end": HK, "kind": _lib.EPI_STORE_BF16, "g_b": lw.g["q"], "out": qkv, "ld_out": NQKV},
        {"n_begin": HK, "n_end": 2 * HK, "kind": _lib.EPI_STORE_BF16, "g_b": lw.g["k"], "out": qkv,
         "out_offset": HK, "ld_out": NQKV},
        {"n_begin": 2 * HK, "n_end": NQKV, "kind": _lib.EPI_STORE_BF16, "g_b": lw.g["v"], "out": qkv,
         "out_offset": 2 * HK, "ld_out": NQKV},
        {"n_begin": NQKV, "n_end": NQKV + H, "kind": _lib.EPI_LOG_ALPHA, "g_b": lw.g["a"], "out": la, "ld_out": H,
         "A_log": lw.A_log, "dt_bias": lw.dt_bias},
        {"n_begin": NQKV + H, "n_end": NQKV + 2 * H, "kind": _lib.EPI_BETA, "g_b": lw.g["b"], "out": be, "ld_out": H},
    ]
    _lib.gdn_gemm_nvfp4(xc, xs, gx, lw.codes, lw.scales, M, NQKV + 2 * H, D, segs)
    _lib.stream_check()
    xq = nvfp4.quantize(x)
    got = to_np(qkv)
    for i, n in enumerate(("q", "k", "v")):
        ref = gemm_bf16(xq, nvfp4.quantize(W[n]))
        assert rel_fro(got[:, i * HK:(i + 1) * HK], ref) < 1e-3, n
    a_ref = gemm_fp64(xq, nvfp4.quantize(W["a"]))
    b_ref = gemm_fp64(xq, nvfp4.quantize(W["b"]))
    la_ref, be_ref = oracle_gates(a_ref, b_ref, A, dt)
    # the gate inputs carry the FP32 accumulation error of a K = 256 sum
    np.testing.assert_allclose(to_np(la), la_ref, rtol=1e-4, atol=1e-5)
    np.testing.assert_allclose(to_np(be), be_ref, rtol=1e-4, atol=1e-5)


def test_gemm_workload_sampled_rows():
    """The GEMM workload: X 8192 x 5120 (quantized on the fly), W 12288 x 5120,
    bf16 Y; the oracle computes 64 sampled rows of Y."""
    d = inputs.gemm_workload()
    M, K = d["x"].shape
    N = d["w"].shape[0]
    xc, xs, gx = _quant_dev(d["x"])
    wc, ws, gw = _quant_dev(d["w"], bf16=False)
    y = _lib.gemm_bf16(xc, xs, gx, wc, ws, gw, M, N, K)
    _lib.stream_check()
    rows = np.sort(np.random.default_rng(1).choice(M, 64, replace=False))
    g_enc = nvfp4.global_encode_scale(nvfp4.tensor_amax(d["x"]))
    xq = nvfp4.quantize(d["x"][rows], g_enc=g_enc)
    wq = nvfp4.quantize(d["w"])
    ref = gemm_bf16(xq, wq)
    got = to_np(y[torch.from_numpy(rows).cuda()])
    e = rel_fro(got, ref)
    print(f"GEMM workload sampled rows: rel_fro {e:.3e}")
    assert e < 1e-3


def test_pair_and_single_tiles_agree():
    """M > 128 runs on CTA pairs (256-row tiles, cta_group::2), M <= 128 on
    single CTAs: the first 128 rows of a 300-row product and the same rows
    computed alone must agree (same k order; FP32 outputs)."""
    rng = np.random.default_rng(11)
    M, N, K = 300, 520, 1024
    x = inputs.activations(rng, (M, K))
    w = inputs.weight(rng, N, K)
    g = np.float32(2688.0) / np.float32(np.abs(x).max())      # one activation scale for both calls
    xd = bf16_cuda(x)
    gx = torch.tensor([g], dtype=torch.float32, device="cuda")
    xc, xs, ga = _lib.gdn_quantize_nvfp4(xd, g_enc=gx)
    xc1, xs1, _ = _lib.gdn_quantize_nvfp4(xd[:128].contiguous(), g_enc=gx)
    wc, ws, gw = _quant_dev(w, bf16=False)
    y = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    y1 = torch.zeros((128, N), dtype=torch.float32, device="cuda")
    seg = lambda out: [{"n_begin": 0, "n_end": N, "kind": _lib.EPI_STORE_F32, "g_b": gw, "out": out, "ld_out": N}]
    _lib.gdn_gemm_nvfp4(xc, xs, ga, wc, ws, M, N, K, seg(y))
    _lib.gdn_gemm_nvfp4(xc1, xs1, ga, wc, ws, 128, N, K, seg(y1))
    _lib.stream_check()
    np.testing.assert_allclose(to_np(y)[:128], to_np(y1), rtol=1e-6, atol=0)
