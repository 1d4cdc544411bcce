"""ctypes binding of ``libgdn.so`` (the C ABI in ``include/gdn.h``).

Argument marshalling only: every function checks dtype / device / contiguity of
its torch tensors, allocates missing outputs with torch (device memory is the
only thing PyTorch is used for), and passes raw pointers plus the current CUDA
stream to the C entry point of the same name.  There is no fallback: if the
library is missing or a call fails, a ``GdnError`` is raised.
"""
import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgdn.so")

GDN_OK = 0
ERR_TIMEOUT, ERR_WORKSPACE, ERR_RANGE = 5, 6, 7
QUANT_DYNAMIC, QUANT_GIVEN_SCALE, QUANT_GIVEN_AMAX = 0, 1, 2
DTYPE_BF16, DTYPE_F32 = 0, 1
SF_TILED, SF_LINEAR = 0, 1
EPI_STORE_BF16, EPI_STORE_F32, EPI_LOG_ALPHA, EPI_BETA = 0, 1, 2, 3
MAX_SEGMENTS = 8
DR_L2NORM_QK, DR_O_FP32, DR_MMA_SYNC, DR_DECAYED_READ = 1, 2, 4, 8
(WS_X_CODES, WS_X_SCALES, WS_X_G, WS_QKV, WS_LOG_ALPHA, WS_BETA, WS_O, WS_O_CODES,
 WS_O_SCALES, WS_O_G, WS_QUANT, WS_SCAN, WS_QKV_CONV, WS_G, WS_O_GATED, WS_COUNT) = range(16)

c_i64 = ctypes.c_int64
c_vp = ctypes.c_void_p


class GdnError(RuntimeError):
    pass


class Nvfp4(ctypes.Structure):
    _fields_ = [("codes", c_vp), ("scales", c_vp)]


class Segment(ctypes.Structure):
    _fields_ = [("n_begin", c_i64), ("n_end", c_i64), ("kind", ctypes.c_int), ("g_b", c_vp),
                ("out", c_vp), ("ld_out", c_i64), ("A_log", c_vp), ("dt_bias", c_vp)]


class LayerCfg(ctypes.Structure):
    _fields_ = [("B", c_i64), ("T", c_i64), ("d_model", c_i64), ("H", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("conv", ctypes.c_int), ("out_gate", ctypes.c_int)]


class LayerWeights(ctypes.Structure):
    _fields_ = [("w_qkvab", Nvfp4), ("g_q", c_vp), ("g_k", c_vp), ("g_v", c_vp), ("g_a", c_vp),
                ("g_b", c_vp), ("w_out", Nvfp4), ("g_out", c_vp), ("A_log", c_vp), ("dt_bias", c_vp),
                ("o_g_enc", c_vp), ("x_g_enc", c_vp), ("conv_w", c_vp), ("g_g", c_vp), ("norm_w", c_vp)]


_LIB = None


def lib():
    """Load libgdn.so once (raises if it was not built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise GdnError(f"{LIB_PATH} is missing: build it with python -m nvfp4_w4a4_gated_quant_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        sig = {
            "gdn_status_string": (ctypes.c_char_p, [ctypes.c_int]),
            "gdn_last_error": (ctypes.c_char_p, []),
            "gdn_version": (ctypes.c_char_p, []),
            "gdn_stream_check": (ctypes.c_int, [c_vp]),
            "gdn_selftest_bounded_wait": (ctypes.c_int, [ctypes.c_uint32, c_vp]),
            "gdn_fp4_mma_ceiling": (ctypes.c_int, [c_i64, ctypes.POINTER(ctypes.c_int), c_vp]),
            "gdn_quantize_workspace_size": (ctypes.c_size_t, []),
            "gdn_scales_tiled_bytes": (ctypes.c_size_t, [c_i64, c_i64]),
            "gdn_quantize_nvfp4": (ctypes.c_int, [c_vp, ctypes.c_int, c_i64, c_i64, c_i64, ctypes.c_int, c_vp,
                                                  c_vp, c_vp, ctypes.c_int, c_i64, c_vp, c_vp, ctypes.c_size_t,
                                                  c_vp]),
            "gdn_amax_update": (ctypes.c_int, [c_vp, ctypes.c_int, c_i64, c_i64, c_i64, c_vp, c_vp]),
            "gdn_encode_scale_from_amax": (ctypes.c_int, [c_vp, c_vp, c_vp]),
            "gdn_gemm_nvfp4": (ctypes.c_int, [ctypes.POINTER(Nvfp4), c_vp, ctypes.POINTER(Nvfp4), c_i64, c_i64,
                                              c_i64, ctypes.POINTER(Segment), ctypes.c_int, c_vp]),
            "gdn_gates": (ctypes.c_int, [c_vp, c_vp, c_i64, ctypes.c_int, c_vp, c_vp, c_vp, c_vp, c_vp]),
            "gdn_short_conv": (ctypes.c_int, [c_vp, c_i64, c_i64, c_i64, c_i64, c_vp, c_vp, c_vp, c_i64, c_vp, c_vp]),
            "gdn_gated_rmsnorm": (ctypes.c_int, [c_vp, c_vp, c_i64, ctypes.c_int, ctypes.c_int, c_vp, c_vp, c_vp,
                                                 c_vp]),
            "gdn_delta_rule_workspace_size": (ctypes.c_size_t, [c_i64, c_i64, ctypes.c_int, ctypes.c_int,
                                                                ctypes.c_int]),
            "gdn_delta_rule_fwd": (ctypes.c_int, [c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_vp, c_vp, c_vp, c_i64,
                                                  c_i64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                  c_vp, c_vp, c_vp, ctypes.c_size_t, c_vp]),
            "gdn_delta_rule_step": (ctypes.c_int, [c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_vp, c_vp, c_vp, c_vp,
                                                   c_i64, c_i64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_int, c_vp, c_vp]),
            "gdn_layer_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(LayerCfg)]),
            "gdn_layer_workspace_offsets": (ctypes.c_int, [ctypes.POINTER(LayerCfg), ctypes.POINTER(c_i64)]),
            "gdn_layer_fwd": (ctypes.c_int, [ctypes.POINTER(LayerWeights), ctypes.POINTER(LayerCfg), c_vp, c_vp,
                                             c_vp, c_vp, c_vp, ctypes.c_size_t, c_vp]),
            "gdn_layer_fwd_static_ws": (ctypes.c_int, [ctypes.POINTER(LayerWeights), ctypes.POINTER(LayerCfg), c_vp,
                                                       c_vp, c_vp, c_vp, c_vp]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


EXPORTED = ("gdn_status_string", "gdn_last_error", "gdn_version", "gdn_stream_check", "gdn_selftest_bounded_wait",
            "gdn_fp4_mma_ceiling",
            "gdn_quantize_workspace_size", "gdn_scales_tiled_bytes", "gdn_quantize_nvfp4", "gdn_amax_update",
            "gdn_encode_scale_from_amax", "gdn_gemm_nvfp4",
            "gdn_gates", "gdn_short_conv", "gdn_gated_rmsnorm", "gdn_delta_rule_workspace_size", "gdn_delta_rule_fwd", "gdn_delta_rule_step",
            "gdn_layer_workspace_size",
            "gdn_layer_workspace_offsets", "gdn_layer_fwd", "gdn_layer_fwd_static_ws")
LAYER_STATIC_WS_BYTES = 32 << 20


def check(status):
    if status != GDN_OK:
        L = lib()
        msg = L.gdn_status_string(status).decode()
        if status in (4, 6):
            msg += ": " + L.gdn_last_error().decode()
        raise GdnError(f"gdn status {status}: {msg}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _row_stride(x):
    """Elements between the rows of a 2-D tensor (its width when empty, whose
    strides torch leaves arbitrary)."""
    return x.stride(0) if x.numel() else x.shape[1]


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, name, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def stream_check(stream=None):
    """Synchronise the stream and raise if a bounded device wait ran out."""
    check(lib().gdn_stream_check(_stream(stream)))


def fp4_mma_ceiling(iters, stream=None):
    """Enqueue the FP4 MMA ceiling kernel (one CTA per SM, iters x 4 MMAs of
    128 x 256 x 64 each); returns the FLOPs it performs."""
    ctas = ctypes.c_int(0)
    check(lib().gdn_fp4_mma_ceiling(iters, ctypes.byref(ctas), _stream(stream)))
    return 2.0 * 128 * 256 * 64 * 4 * iters * ctas.value


# -------------------------------------------------------------- quantizer --
def scales_tiled_bytes(rows, cols):
    return int(lib().gdn_scales_tiled_bytes(rows, cols))


def gdn_quantize_nvfp4(x, g_enc=None, layout="tiled", codes=None, scales=None, sf_row_offset=0, g_out=None,
                       ws=None, stream=None, amax=None):
    """Quantize a 2-D bf16 / FP32 CUDA tensor (unit stride along columns).

    Dynamic per-tensor scale unless ``g_enc`` (a 1-element FP32 CUDA tensor
    holding the encode scale) or ``amax`` (a 1-element FP32 CUDA tensor holding
    the tensor's amax) is given.  Returns (codes, scales, g) where g is the
    1-element FP32 decode scale.  ``scales`` may be a shared TILED buffer
    filled from row ``sf_row_offset`` on."""
    if x.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("x must be bf16 or float32")
    if not x.is_cuda or x.dim() != 2 or (x.numel() and x.stride(1) != 1):
        raise ValueError("x must be a 2-D CUDA tensor with unit column stride")
    rows, cols = x.shape
    dev = x.device
    tiled = layout == "tiled"
    if codes is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    if scales is None:
        nbytes = scales_tiled_bytes(rows, cols) if tiled else rows * (cols // 16)
        scales = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    if g_out is None:
        g_out = torch.empty(1, dtype=torch.float32, device=dev)
    _need(codes, torch.uint8, "codes", dev)
    _need(scales, torch.uint8, "scales", dev)
    _need(g_out, torch.float32, "g_out", dev)
    mode = QUANT_DYNAMIC
    if g_enc is not None and amax is not None:
        raise ValueError("give g_enc or amax, not both")
    if g_enc is not None:
        _need(g_enc, torch.float32, "g_enc", dev)
        mode = QUANT_GIVEN_SCALE
    if amax is not None:
        _need(amax, torch.float32, "amax", dev)
        g_enc, mode = amax, QUANT_GIVEN_AMAX
    L = lib()
    wsz = int(L.gdn_quantize_workspace_size())
    if ws is None and mode == QUANT_DYNAMIC:
        ws = torch.empty(wsz, dtype=torch.uint8, device=dev)
    check(L.gdn_quantize_nvfp4(_ptr(x), DTYPE_F32 if x.dtype == torch.float32 else DTYPE_BF16, rows, cols,
                               _row_stride(x), mode, _ptr(g_enc), _ptr(codes), _ptr(scales),
                               SF_TILED if tiled else SF_LINEAR, sf_row_offset, _ptr(g_out), _ptr(ws),
                               wsz if ws is not None else 0, _stream(stream)))
    return codes, scales, g_out


# ------------------------------------------------------------ calibration --
def gdn_amax_update(x, amax, stream=None):
    """Fold max |x| of a 2-D bf16 / FP32 CUDA tensor (unit column stride) into
    ``amax``, a 1-element FP32 CUDA tensor holding a running maximum."""
    if x.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("x must be bf16 or float32")
    if not x.is_cuda or x.dim() != 2 or (x.numel() and x.stride(1) != 1):
        raise ValueError("x must be a 2-D CUDA tensor with unit column stride")
    _need(amax, torch.float32, "amax", x.device)
    rows, cols = x.shape
    check(lib().gdn_amax_update(_ptr(x), DTYPE_F32 if x.dtype == torch.float32 else DTYPE_BF16, rows, cols,
                                _row_stride(x), _ptr(amax), _stream(stream)))
    return amax


def gdn_encode_scale_from_amax(amax, g_enc=None, stream=None):
    """The encode scale 2688 / amax of a calibrated amax (1-element FP32 CUDA
    tensors)."""
    _need(amax, torch.float32, "amax")
    if g_enc is None:
        g_enc = torch.empty(1, dtype=torch.float32, device=amax.device)
    _need(g_enc, torch.float32, "g_enc", amax.device)
    check(lib().gdn_encode_scale_from_amax(_ptr(amax), _ptr(g_enc), _stream(stream)))
    return g_enc


def calibrate_layer(weights, batches, stream=None):
    """Static activation scales of the layer's two quantized inputs, each
    calibrated on its own: x (the input of the q/k/v/a/b projection) and o
    (the input of the output projection).  ``batches``: bf16 CUDA tensors
    [B, T, d_model].  Every batch's x folds into x's running amax; the layer
    runs on it with dynamic scales and its o folds into o's.  Returns
    (x_g_enc, o_g_enc), 1-element FP32 CUDA tensors for
    ``weights.x_g_enc`` / ``weights.o_g_enc``."""
    saved = (weights.x_g_enc, weights.o_g_enc)
    weights.x_g_enc = weights.o_g_enc = None
    try:
        dev = batches[0].device
        x_amax = torch.zeros(1, dtype=torch.float32, device=dev)
        o_amax = torch.zeros(1, dtype=torch.float32, device=dev)
        for x in batches:
            B, T, D = x.shape
            gdn_amax_update(x.view(B * T, D), x_amax, stream=stream)
            _, _, ws = gdn_layer_fwd(weights, x, want_state=False, stream=stream)
            off = gdn_layer_workspace_offsets(weights.cfg(B, T))
            HV = weights.H * weights.dv
            o = ws[off[WS_O]:off[WS_O] + B * T * HV * 2].view(torch.bfloat16).view(B * T, HV)
            gdn_amax_update(o, o_amax, stream=stream)
        return gdn_encode_scale_from_amax(x_amax, stream=stream), gdn_encode_scale_from_amax(o_amax, stream=stream)
    finally:
        weights.x_g_enc, weights.o_g_enc = saved


# ------------------------------------------------------------------- GEMM --
def gdn_gemm_nvfp4(a_codes, a_scales, g_a, b_codes, b_scales, M, N, K, segments, stream=None):
    """Block-scaled FP4 GEMM.  ``segments``: list of dicts with keys n_begin,
    n_end, kind (EPI_*), g_b (1-element FP32 tensor), out (tensor), ld_out,
    and for EPI_LOG_ALPHA A_log / dt_bias (FP32 tensors)."""
    for t, dt, n in ((a_codes, torch.uint8, "a_codes"), (a_scales, torch.uint8, "a_scales"),
                     (b_codes, torch.uint8, "b_codes"), (b_scales, torch.uint8, "b_scales"),
                     (g_a, torch.float32, "g_a")):
        _need(t, dt, n)
    if len(segments) > MAX_SEGMENTS:
        raise ValueError("too many segments")
    segs = (Segment * len(segments))()
    keep = []
    for i, s in enumerate(segments):
        out = s["out"]
        want = torch.bfloat16 if s["kind"] == EPI_STORE_BF16 else torch.float32
        _need(out, want, "segment out")
        _need(s["g_b"], torch.float32, "segment g_b")
        segs[i].n_begin = s["n_begin"]
        segs[i].n_end = s["n_end"]
        segs[i].kind = s["kind"]
        segs[i].g_b = s["g_b"].data_ptr()
        segs[i].out = out.data_ptr() + s.get("out_offset", 0) * out.element_size()
        segs[i].ld_out = s["ld_out"]
        if s["kind"] == EPI_LOG_ALPHA:
            _need(s["A_log"], torch.float32, "A_log")
            _need(s["dt_bias"], torch.float32, "dt_bias")
            segs[i].A_log = s["A_log"].data_ptr()
            segs[i].dt_bias = s["dt_bias"].data_ptr()
        keep.append(s)
    A = Nvfp4(a_codes.data_ptr(), a_scales.data_ptr())
    B = Nvfp4(b_codes.data_ptr(), b_scales.data_ptr())
    check(lib().gdn_gemm_nvfp4(ctypes.byref(A), _ptr(g_a), ctypes.byref(B), M, N, K, segs, len(segments),
                               _stream(stream)))


def gemm_bf16(a_codes, a_scales, g_a, b_codes, b_scales, g_b, M, N, K, out=None, stream=None):
    """Plain Y = A_hat B_hat^T in bf16 (one segment)."""
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a_codes.device)
    gdn_gemm_nvfp4(a_codes, a_scales, g_a, b_codes, b_scales, M, N, K,
                   [{"n_begin": 0, "n_end": N, "kind": EPI_STORE_BF16, "g_b": g_b, "out": out, "ld_out": out.stride(0)}],
                   stream)
    return out


# ------------------------------------------------------------------ gates --
def gdn_gates(a, b, A_log, dt_bias, log_alpha=None, beta=None, stream=None):
    """a, b: FP32 [M, H] contiguous; returns (log_alpha, beta) FP32 [M, H]."""
    for t, n in ((a, "a"), (b, "b"), (A_log, "A_log"), (dt_bias, "dt_bias")):
        _need(t, torch.float32, n)
    if not (a.is_contiguous() and b.is_contiguous()) or a.shape != b.shape or a.dim() != 2:
        raise ValueError("a, b must be contiguous [M, H]")
    M, H = a.shape
    if log_alpha is None:
        log_alpha = torch.empty_like(a)
    if beta is None:
        beta = torch.empty_like(b)
    check(lib().gdn_gates(_ptr(a), _ptr(b), M, H, _ptr(A_log), _ptr(dt_bias), _ptr(log_alpha), _ptr(beta),
                          _stream(stream)))
    return log_alpha, beta


# ------------------------------------------------- convolution and norm --
def gdn_short_conv(x, w, state_in=None, y=None, state_out=None, stream=None):
    """Causal depthwise convolution of width 4 + SiLU over the channels of x
    (bf16 [B, T, C], unit channel stride); w FP32 [C, 4]; state_in / state_out
    bf16 [B, 3, C] or None.  Returns y (bf16 [B, T, C])."""
    _need(x, torch.bfloat16, "x")
    _need(w, torch.float32, "w")
    if x.dim() != 3 or (x.numel() and x.stride(2) != 1):
        raise ValueError("x must be [B, T, C] with unit channel stride")
    B, T, C = x.shape
    if T > 1 and B > 1 and x.stride(0) != T * x.stride(1):
        raise ValueError("x: batch stride must be T * token stride")
    ld_x = x.stride(1) if T > 1 else (x.stride(0) if B > 1 else C)
    if y is None:
        y = torch.empty((B, T, C), dtype=torch.bfloat16, device=x.device)
    for t, n in ((state_in, "state_in"), (state_out, "state_out")):
        if t is not None:
            _need(t, torch.bfloat16, n)
            if not t.is_contiguous() or t.shape != (B, 3, C):
                raise ValueError(f"{n} must be a contiguous [B, 3, C] tensor")
    check(lib().gdn_short_conv(_ptr(x), B, T, C, ld_x, _ptr(w), _ptr(state_in), _ptr(y), C, _ptr(state_out),
                               _stream(stream)))
    return y


def gdn_gated_rmsnorm(o, g, gamma, H, y=None, amax=None, stream=None):
    """o, g bf16 [M, H*dv] contiguous; gamma FP32 [dv].  Returns
    y = o / sqrt(mean_dv(o^2) + 1e-6) * gamma * SiLU(g) per (token, head), bf16;
    folds max |y| into ``amax`` (1-element FP32) when given."""
    _need(o, torch.bfloat16, "o")
    _need(g, torch.bfloat16, "g")
    _need(gamma, torch.float32, "gamma")
    if not (o.is_contiguous() and g.is_contiguous()) or o.shape != g.shape or o.dim() != 2:
        raise ValueError("o, g must be contiguous [M, H*dv]")
    M, HV = o.shape
    if y is None:
        y = torch.empty_like(o)
    if amax is not None:
        _need(amax, torch.float32, "amax")
    check(lib().gdn_gated_rmsnorm(_ptr(o), _ptr(g), M, H, HV // H, _ptr(gamma), _ptr(y), _ptr(amax),
                                  _stream(stream)))
    return y


# ------------------------------------------------------------- delta rule --
def _token_stride(t, name):
    """Elements between consecutive tokens of a [B, T, H, d] tensor whose
    heads are contiguous; strides of size-1 dimensions are irrelevant."""
    B, T, H, d = t.shape
    if B * T == 0:
        return H * d
    if (d > 1 and t.stride(3) != 1) or (H > 1 and t.stride(2) != d):
        raise ValueError(f"{name} must have contiguous heads ([B, T, H, d] with unit stride over H*d)")
    if T > 1:
        ld = t.stride(1)
        if B > 1 and t.stride(0) != T * ld:
            raise ValueError(f"{name}: batch stride must be T * token stride")
        return ld
    return t.stride(0) if B > 1 else H * d


def gdn_delta_rule_fwd(q, k, v, log_alpha, beta, S0=None, l2norm=True, o_fp32=False, o=None, S_T=None,
                       want_state=True, stream=None, mma_sync=False, use_workspace=True, workspace_bytes=None,
                       workspace=None):
    """q, k [B, T, H, dk], v [B, T, H, dv] bf16 (heads contiguous, token stride
    free); log_alpha, beta FP32 [B, T, H] contiguous; S0 FP32 [B, H, dk, dv].
    ``mma_sync`` selects the warp-level mma.sync kernel where the tcgen05 one
    would run; ``use_workspace=False`` passes no workspace (long sequences on
    few chains then run in one piece instead of segments, and each chunk's
    inverse is computed inside the scan); ``workspace_bytes`` passes a
    workspace of that size instead of the queried one; ``workspace`` (a uint8
    tensor on the device) passes the caller's own.
    Returns (o [B, T, H, dv] bf16 or FP32, S_T FP32 or None)."""
    lds = []
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
        if t.dim() != 4:
            raise ValueError(f"{n} must be [B, T, H, d]")
        lds.append(_token_stride(t, n))
    for t, n in ((log_alpha, "log_alpha"), (beta, "beta")):
        _need(t, torch.float32, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    B, T, H, dk = q.shape
    dv = v.shape[3]
    dev = q.device
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=torch.float32 if o_fp32 else torch.bfloat16, device=dev)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    if S0 is not None:
        _need(S0, torch.float32, "S0")
        if not S0.is_contiguous():
            raise ValueError("S0 must be contiguous")
    flags = (DR_L2NORM_QK if l2norm else 0) | (DR_O_FP32 if o_fp32 else 0) | (DR_MMA_SYNC if mma_sync else 0)
    L = lib()
    wsz = int(L.gdn_delta_rule_workspace_size(B, T, H, dk, dv)) if use_workspace else 0
    if workspace_bytes is not None:
        wsz = int(workspace_bytes)
    ws = torch.empty(wsz, dtype=torch.uint8, device=dev) if wsz else None
    if workspace is not None:
        _need(workspace, torch.uint8, "workspace")
        ws, wsz = workspace, workspace.numel()
    check(L.gdn_delta_rule_fwd(_ptr(q), _ptr(k), _ptr(v), lds[0], lds[1], lds[2], _ptr(log_alpha),
                               _ptr(beta), _ptr(S0), B, T, H, dk, dv, flags, _ptr(o), _ptr(S_T), _ptr(ws), wsz,
                               _stream(stream)))
    return o, S_T


def gdn_delta_rule_step(q, k, v, log_alpha, beta, S=None, l2norm=True, o_fp32=False, decayed_read=False, o=None,
                        S_out=None, stream=None):
    """The recurrence token by token (decode, short continuations): q, k
    [B, T, H, dk], v [B, T, H, dv] bf16 (token stride free); log_alpha, beta
    FP32 [B, T, H]; S FP32 [B, H, dk, dv] entry state or None for zeros.
    ``S_out`` defaults to a new tensor; pass ``S_out=S`` to update in place.
    Returns (o [B, T, H, dv] bf16 or FP32, S_out)."""
    lds = []
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
        if t.dim() != 4:
            raise ValueError(f"{n} must be [B, T, H, d]")
        lds.append(_token_stride(t, n))
    for t, n in ((log_alpha, "log_alpha"), (beta, "beta")):
        _need(t, torch.float32, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    B, T, H, dk = q.shape
    dv = v.shape[3]
    dev = q.device
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=torch.float32 if o_fp32 else torch.bfloat16, device=dev)
    if S_out is None:
        S_out = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    for t, n in ((S, "S"), (S_out, "S_out")):
        if t is not None:
            _need(t, torch.float32, n)
            if not t.is_contiguous():
                raise ValueError(f"{n} must be contiguous")
    flags = (DR_L2NORM_QK if l2norm else 0) | (DR_O_FP32 if o_fp32 else 0) | (DR_DECAYED_READ if decayed_read else 0)
    check(lib().gdn_delta_rule_step(_ptr(q), _ptr(k), _ptr(v), lds[0], lds[1], lds[2], _ptr(log_alpha), _ptr(beta),
                                    _ptr(S), _ptr(S_out), B, T, H, dk, dv, flags, _ptr(o), _stream(stream)))
    return o, S_out


# ------------------------------------------------------------------ layer --
class QuantizedLayerWeights:
    """NVFP4 weights of one layer, quantized on the device by the library:
    q, k, v, a, b share one [2*H*dk + H*dv + 2*H, d_model] operand (each with
    its own decode scale), out is [d_model, H*dv].  ``x_g_enc`` and
    ``o_g_enc`` (1-element FP32 CUDA tensors, default None) are static encode
    scales for the two quantized activations, x and o (``calibrate_layer``);
    None quantizes that activation with its own amax."""

    def __init__(self, W, A_log, dt_bias, H, dk, dv, device="cuda", stream=None, conv_w=None, norm_w=None):
        d_model = W["q"].shape[1]
        self.H, self.dk, self.dv, self.d_model = H, dk, dv, d_model
        names = ["q", "k", "v", "a", "b"]
        rows = [H * dk, H * dk, H * dv, H, H]
        self.out_gate = 1 if "g" in W else 0
        if self.out_gate:
            if norm_w is None:
                raise ValueError("the output gate needs norm_w")
            names.append("g")
            rows.append(H * dv)
        n_total = sum(rows)
        self.codes = torch.empty((n_total, d_model // 2), dtype=torch.uint8, device=device)
        self.scales = torch.zeros(scales_tiled_bytes(n_total, d_model), dtype=torch.uint8, device=device)
        self.g = {}
        r0 = 0
        for name, nr in zip(names, rows):
            w = torch.as_tensor(W[name], dtype=torch.float32).to(device).contiguous()
            _, _, g = gdn_quantize_nvfp4(w, codes=self.codes[r0:r0 + nr], scales=self.scales, sf_row_offset=r0,
                                         stream=stream)
            self.g[name] = g
            r0 += nr
        wo = torch.as_tensor(W["out"], dtype=torch.float32).to(device).contiguous()
        self.out_codes, self.out_scales, self.g["out"] = gdn_quantize_nvfp4(wo, stream=stream)
        self.A_log = torch.as_tensor(A_log, dtype=torch.float32).to(device).contiguous()
        self.dt_bias = torch.as_tensor(dt_bias, dtype=torch.float32).to(device).contiguous()
        self.o_g_enc = None
        self.x_g_enc = None
        self.conv = 0 if conv_w is None else 1
        self.conv_w = None if conv_w is None else torch.as_tensor(conv_w, dtype=torch.float32).to(device).contiguous()
        self.norm_w = None if norm_w is None else torch.as_tensor(norm_w, dtype=torch.float32).to(device).contiguous()

    def cfg(self, B, T):
        return layer_cfg(B, T, self.d_model, self.H, self.dk, self.dv, self.conv, self.out_gate)

    def struct(self):
        s = LayerWeights()
        s.w_qkvab = Nvfp4(self.codes.data_ptr(), self.scales.data_ptr())
        s.g_q, s.g_k, s.g_v = self.g["q"].data_ptr(), self.g["k"].data_ptr(), self.g["v"].data_ptr()
        s.g_a, s.g_b = self.g["a"].data_ptr(), self.g["b"].data_ptr()
        s.w_out = Nvfp4(self.out_codes.data_ptr(), self.out_scales.data_ptr())
        s.g_out = self.g["out"].data_ptr()
        s.A_log, s.dt_bias = self.A_log.data_ptr(), self.dt_bias.data_ptr()
        if self.o_g_enc is not None:
            _need(self.o_g_enc, torch.float32, "o_g_enc")
            s.o_g_enc = self.o_g_enc.data_ptr()
        if self.x_g_enc is not None:
            _need(self.x_g_enc, torch.float32, "x_g_enc")
            s.x_g_enc = self.x_g_enc.data_ptr()
        if self.conv_w is not None:
            s.conv_w = self.conv_w.data_ptr()
        if self.out_gate:
            s.g_g = self.g["g"].data_ptr()
            s.norm_w = self.norm_w.data_ptr()
        return s


def layer_cfg(B, T, d_model, H, dk, dv, conv=0, out_gate=0):
    return LayerCfg(B, T, d_model, H, dk, dv, conv, out_gate)


def gdn_layer_workspace_size(cfg):
    return int(lib().gdn_layer_workspace_size(ctypes.byref(cfg)))


def gdn_layer_workspace_offsets(cfg):
    offs = (c_i64 * WS_COUNT)()
    check(lib().gdn_layer_workspace_offsets(ctypes.byref(cfg), offs))
    return list(offs)


def gdn_layer_fwd(weights, x, S0=None, want_state=True, y=None, S_T=None, ws=None, stream=None):
    """x: bf16 [B, T, d_model] contiguous.  Returns (y, S_T, ws)."""
    _need(x, torch.bfloat16, "x")
    if not x.is_contiguous() or x.dim() != 3:
        raise ValueError("x must be a contiguous [B, T, d_model] tensor")
    B, T, D = x.shape
    cfg = weights.cfg(B, T)
    dev = x.device
    if y is None:
        y = torch.empty_like(x)
    if S_T is None and want_state:
        S_T = torch.empty((B, weights.H, weights.dk, weights.dv), dtype=torch.float32, device=dev)
    need = gdn_layer_workspace_size(cfg)
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_struct = weights.struct()
    check(lib().gdn_layer_fwd(ctypes.byref(ws_struct), ctypes.byref(cfg), _ptr(x), _ptr(y), _ptr(S0), _ptr(S_T),
                              _ptr(ws), ws.numel(), _stream(stream)))
    return y, S_T, ws


def gdn_layer_fwd_static_ws(weights, x, S0=None, want_state=True, y=None, S_T=None, stream=None):
    """The layer forward with its scratch in the library's static device
    array (no workspace argument, nothing allocated by the call itself).
    Returns (y, S_T).  Calls that overlap on the GPU race on the shared
    array."""
    _need(x, torch.bfloat16, "x")
    if not x.is_contiguous() or x.dim() != 3:
        raise ValueError("x must be a contiguous [B, T, d_model] tensor")
    B, T, D = x.shape
    cfg = weights.cfg(B, T)
    if y is None:
        y = torch.empty_like(x)
    if S_T is None and want_state:
        S_T = torch.empty((B, weights.H, weights.dk, weights.dv), dtype=torch.float32, device=x.device)
    ws_struct = weights.struct()
    st = lib().gdn_layer_fwd_static_ws(ctypes.byref(ws_struct), ctypes.byref(cfg), _ptr(x), _ptr(y), _ptr(S0),
                                       _ptr(S_T), _stream(stream))
    if st == 6:
        raise GdnError(f"gdn status 6: {lib().gdn_last_error().decode()}")
    check(st)
    return y, S_T
