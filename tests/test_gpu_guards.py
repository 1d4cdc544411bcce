"""Guard regions around every output: no kernel writes outside its buffer, and
none leaves an element of its output unwritten.

Each output is carved out of a larger allocation with 4 KiB of 0xA5 canary
bytes before and after it, and the output itself is pre-filled with NaN (or
with two different byte patterns for integer outputs, whose results must then
agree).  After the call the canaries must be intact, no NaN may remain in the
output, and padding inside a row pitch (ld > N) must be untouched.  Shapes are
ragged on purpose: rows past a 128-row tile, columns past a 256-column tile,
sequences ending inside a 64-token chunk.  This stands in for a memory checker
on the GPU (compute-sanitizer is not available here).
"""
import numpy as np
import pytest
import torch

from nvfp4_w4a4_gated_quant_b200 import _lib, inputs
from oracle import nvfp4
from oracle.delta_rule import delta_rule_chunked, delta_rule_sequential
from oracle.gemm import gemm_bf16
from tests._helpers import bf16_cuda, f32_cuda, rel_fro, tiled_to_linear, to_np

pytestmark = pytest.mark.gpu

PAD = 4096
CANARY = 0xA5


class Guarded:
    """``n`` elements of ``dtype`` between two canary regions."""

    def __init__(self, n, dtype, fill):
        esize = torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((2 * PAD + n * esize,), CANARY, dtype=torch.uint8, device="cuda")
        self.t = self.raw[PAD:PAD + n * esize].view(dtype)
        self.t.fill_(fill)

    def canaries_intact(self):
        return bool((self.raw[:PAD] == CANARY).all()) and bool((self.raw[-PAD:] == CANARY).all())


def _nan_free(t):
    return not bool(torch.isnan(t.float()).any())


@pytest.mark.parametrize("rows,cols", [(200, 320), (1, 64), (129, 1088)])
def test_quantizer_stays_in_bounds_and_writes_everything(rows, cols):
    rng = np.random.default_rng(rows)
    x = inputs.activations(rng, (rows, cols))
    xd = bf16_cuda(x)
    ref = nvfp4.quantize(x)
    for fill in (0x00, 0xFF):
        codes = Guarded(rows * cols // 2, torch.uint8, fill)
        sbytes = _lib.scales_tiled_bytes(rows, cols)
        scales = Guarded(sbytes, torch.uint8, fill)
        g = Guarded(1, torch.float32, float("nan"))
        _lib.gdn_quantize_nvfp4(xd, codes=codes.t.view(rows, cols // 2), scales=scales.t, g_out=g.t)
        _lib.stream_check()
        assert codes.canaries_intact() and scales.canaries_intact() and g.canaries_intact()
        assert _nan_free(g.t)
        c = to_np(codes.t).reshape(rows, cols // 2)
        s = tiled_to_linear(to_np(scales.t), rows, cols)
        np.testing.assert_array_equal(c, ref["codes"])
        np.testing.assert_array_equal(s, ref["scales"])
    # linear scales: the whole buffer is the output
    for fill in (0x00, 0xFF):
        scales = Guarded(rows * cols // 16, torch.uint8, fill)
        codes = Guarded(rows * cols // 2, torch.uint8, fill)
        _lib.gdn_quantize_nvfp4(xd, layout="linear", codes=codes.t.view(rows, cols // 2), scales=scales.t)
        _lib.stream_check()
        assert codes.canaries_intact() and scales.canaries_intact()
        np.testing.assert_array_equal(to_np(scales.t).reshape(rows, cols // 16), ref["scales"])


@pytest.mark.parametrize("M,N,K,pitch", [(200, 200, 256, 0), (129, 264, 320, 0), (200, 150, 256, 3),
                                         (300, 40, 512, 5)],
                         ids=["tma_store", "tma_store_2", "per_element", "per_element_2"])
def test_gemm_stays_in_bounds_and_writes_everything(M, N, K, pitch):
    """bf16 out with the row pitch ld = N + pitch: pitch 0 (16-byte rows) takes
    the TMA-store epilogue, an odd pitch the per-element path; the padding
    columns between N and ld must stay untouched."""
    rng = np.random.default_rng(M + N)
    x = inputs.activations(rng, (M, K))
    w = inputs.weight(rng, N, K)
    xc, xs, gx = _lib.gdn_quantize_nvfp4(bf16_cuda(x))
    wc, wsc, gw = _lib.gdn_quantize_nvfp4(f32_cuda(w))
    ld = N + pitch
    out = Guarded(M * ld, torch.bfloat16, float("nan"))
    y = out.t.view(M, ld)
    _lib.gdn_gemm_nvfp4(xc, xs, gx, wc, wsc, M, N, K,
                        [{"n_begin": 0, "n_end": N, "kind": _lib.EPI_STORE_BF16, "g_b": gw, "out": y, "ld_out": ld}])
    _lib.stream_check()
    assert out.canaries_intact()
    assert _nan_free(y[:, :N])
    if pitch:
        assert bool(torch.isnan(y[:, N:].float()).all())
    assert rel_fro(to_np(y[:, :N]), gemm_bf16(nvfp4.quantize(x), nvfp4.quantize(w))) < 1e-3


@pytest.mark.parametrize("B,T,H,d,mma_sync,o_fp32", [(2, 200, 2, 128, False, False), (1, 77, 3, 128, False, True),
                                                    (2, 130, 2, 64, False, False), (1, 150, 2, 128, True, False),
                                                    (1, 2000, 2, 128, False, False)],
                         ids=["tc_bf16", "tc_f32", "mma_sync_d64", "mma_sync_bf16", "tc_segmented"])
def test_scan_stays_in_bounds_and_writes_everything(B, T, H, d, mma_sync, o_fp32):
    rng = np.random.default_rng(T)
    q = rng.standard_normal((B, T, H, d)).astype(np.float32)
    k = rng.standard_normal((B, T, H, d)).astype(np.float32)
    v = rng.standard_normal((B, T, H, d)).astype(np.float32)
    la = -rng.uniform(0, 1, (B, T, H)).astype(np.float32)
    be = rng.uniform(0, 1, (B, T, H)).astype(np.float32)
    qd, kd, vd = bf16_cuda(q), bf16_cuda(k), bf16_cuda(v)
    o = Guarded(B * T * H * d, torch.float32 if o_fp32 else torch.bfloat16, float("nan"))
    S = Guarded(B * H * d * d, torch.float32, float("nan"))
    o_t = o.t.view(B, T, H, d)
    S_t = S.t.view(B, H, d, d)
    _lib.gdn_delta_rule_fwd(qd, kd, vd, f32_cuda(la), f32_cuda(be), o=o_t, S_T=S_t, o_fp32=o_fp32, mma_sync=mma_sync)
    _lib.stream_check()
    assert o.canaries_intact() and S.canaries_intact()
    assert _nan_free(o_t) and _nan_free(S_t)
    o_ref, S_ref = delta_rule_chunked(to_np(qd), to_np(kd), to_np(vd), la, be)
    assert rel_fro(to_np(o_t), o_ref) < 3e-3
    assert rel_fro(to_np(S_t), S_ref) < 2e-3


def test_segmented_scan_workspace_stays_in_bounds():
    """Sequences cut into segments: the call writes the segment states and
    every chunk's inverse image into the caller's workspace, and nothing past
    either end of it; a second call on the same (now stale) workspace gives
    the same bits."""
    B, T, H, d = 1, 2000, 2, 128
    wsz = int(_lib.lib().gdn_delta_rule_workspace_size(B, T, H, d, d))
    assert wsz >= B * ((T + 63) // 64) * H * 16384
    rng = np.random.default_rng(5)
    q, k, v = (bf16_cuda(rng.standard_normal((B, T, H, d)).astype(np.float32)) for _ in range(3))
    la = f32_cuda(-rng.uniform(0, 1, (B, T, H)).astype(np.float32))
    be = f32_cuda(rng.uniform(0, 1, (B, T, H)).astype(np.float32))
    ws = Guarded(wsz, torch.uint8, 0x5A)
    o1, S1 = _lib.gdn_delta_rule_fwd(q, k, v, la, be, workspace=ws.t)
    o2, S2 = _lib.gdn_delta_rule_fwd(q, k, v, la, be, workspace=ws.t)
    _lib.stream_check()
    assert ws.canaries_intact()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    assert _nan_free(o1) and _nan_free(S1)


@pytest.mark.parametrize("B,T,C", [(2, 150, 96), (1, 77, 6176), (3, 1, 40)], ids=["ragged", "layer_width", "one_token"])
def test_short_conv_stays_in_bounds_and_writes_everything(B, T, C):
    """The convolution's output and carried state: rows staged through shared
    memory in groups of eight (ragged last group, a last token block shorter
    than 64), nothing written outside either buffer, nothing left unwritten."""
    from oracle.conv_norm import short_conv
    rng = np.random.default_rng(B * T + C)
    x = bf16_cuda(rng.standard_normal((B, T, C)).astype(np.float32))
    w = f32_cuda(rng.uniform(-0.8, 0.8, (C, 4)).astype(np.float32))
    st_in = bf16_cuda(rng.standard_normal((B, 3, C)).astype(np.float32))
    y = Guarded(B * T * C, torch.bfloat16, float("nan"))
    st = Guarded(B * 3 * C, torch.bfloat16, float("nan"))
    _lib.gdn_short_conv(x, w, state_in=st_in, y=y.t.view(B, T, C), state_out=st.t.view(B, 3, C))
    _lib.stream_check()
    assert y.canaries_intact() and st.canaries_intact()
    assert _nan_free(y.t) and _nan_free(st.t)
    y_ref, st_ref = short_conv(to_np(x), to_np(w), state=to_np(st_in))
    assert rel_fro(to_np(y.t).reshape(B, T, C), nvfp4.round_bf16(y_ref)) < 2e-3
    np.testing.assert_array_equal(to_np(st.t).reshape(B, 3, C), st_ref)


def test_gated_rmsnorm_stays_in_bounds_and_writes_everything():
    M, H, dv = 333, 3, 128
    rng = np.random.default_rng(7)
    o = bf16_cuda(rng.standard_normal((M, H * dv)).astype(np.float32))
    g = bf16_cuda(rng.standard_normal((M, H * dv)).astype(np.float32))
    gamma = f32_cuda(rng.uniform(0.5, 1.5, dv).astype(np.float32))
    y = Guarded(M * H * dv, torch.bfloat16, float("nan"))
    _lib.gdn_gated_rmsnorm(o, g, gamma, H, y=y.t.view(M, H * dv))
    _lib.stream_check()
    assert y.canaries_intact() and _nan_free(y.t)


def test_decode_step_stays_in_bounds_and_writes_everything():
    B, T, H, d = 3, 5, 2, 128
    rng = np.random.default_rng(5)
    q, k, v = (bf16_cuda(rng.standard_normal((B, T, H, d)).astype(np.float32)) for _ in range(3))
    la = -rng.uniform(0, 1, (B, T, H)).astype(np.float32)
    be = rng.uniform(0, 1, (B, T, H)).astype(np.float32)
    S0 = (rng.standard_normal((B, H, d, d)) * 0.3).astype(np.float32)
    o = Guarded(B * T * H * d, torch.float32, float("nan"))
    S = Guarded(B * H * d * d, torch.float32, float("nan"))
    _lib.gdn_delta_rule_step(q, k, v, f32_cuda(la), f32_cuda(be), S=f32_cuda(S0), o_fp32=True,
                             o=o.t.view(B, T, H, d), S_out=S.t.view(B, H, d, d))
    _lib.stream_check()
    assert o.canaries_intact() and S.canaries_intact()
    assert _nan_free(o.t) and _nan_free(S.t)
    o_ref, S_ref = delta_rule_sequential(to_np(q), to_np(k), to_np(v), la, be, S0=S0)
    assert rel_fro(to_np(o.t).reshape(B, T, H, d), o_ref) < 1e-5
    assert rel_fro(to_np(S.t).reshape(B, H, d, d), S_ref) < 1e-5


def test_gates_stay_in_bounds_and_write_everything():
    M, H = 333, 5
    rng = np.random.default_rng(9)
    a = f32_cuda(rng.standard_normal((M, H)))
    b = f32_cuda(rng.standard_normal((M, H)))
    A = f32_cuda(rng.uniform(-1, 1, H))
    dt = f32_cuda(rng.uniform(-1, 1, H))
    la = Guarded(M * H, torch.float32, float("nan"))
    be = Guarded(M * H, torch.float32, float("nan"))
    _lib.gdn_gates(a, b, A, dt, log_alpha=la.t.view(M, H), beta=be.t.view(M, H))
    _lib.stream_check()
    assert la.canaries_intact() and be.canaries_intact()
    assert _nan_free(la.t) and _nan_free(be.t)


@pytest.mark.parametrize("dims", [(2, 200, 512, 4, 128, 128), (1, 96, 256, 2, 32, 32), (1, 2048, 256, 2, 128, 128)],
                         ids=["tc", "mma_sync", "tc_segmented"])
def test_layer_stays_in_bounds_and_writes_everything(dims):
    """The layer's output, final state and workspace, each between canaries;
    y and S_T pre-filled with NaN."""
    B, T, D, H, dk, dv = dims
    d = inputs.layer_inputs(B, T, D, H, dk, dv, seed=17)
    lw = _lib.QuantizedLayerWeights(d["W"], d["A_log"], d["dt_bias"], H, dk, dv)
    x = torch.from_numpy(d["x"]).cuda().to(torch.bfloat16)
    y = Guarded(B * T * D, torch.bfloat16, float("nan"))
    S = Guarded(B * H * dk * dv, torch.float32, float("nan"))
    cfg = _lib.layer_cfg(B, T, D, H, dk, dv)
    nws = _lib.gdn_layer_workspace_size(cfg)
    ws = Guarded(nws, torch.uint8, 0xFF)
    # the workspace must be 256-byte aligned: PAD keeps the allocation's alignment
    _lib.gdn_layer_fwd(lw, x, y=y.t.view(B, T, D), S_T=S.t.view(B, H, dk, dv), ws=ws.t)
    _lib.stream_check()
    assert y.canaries_intact() and S.canaries_intact() and ws.canaries_intact()
    assert _nan_free(y.t) and _nan_free(S.t)
    y2, S2, _ = _lib.gdn_layer_fwd(lw, x)
    _lib.stream_check()
    assert torch.equal(y.t.view(B, T, D), y2) and torch.equal(S.t.view(B, H, dk, dv), S2)
