"""The W4A4 Gated DeltaNet layer forward, four steps composed (oracle).

Steps (task statement; pages "Why Gated DeltaNet Survives 4-Bit Quantization"
sections "Why the 'Fragile' Recurrence is Actually Robust" and "Performance and
Efficiency Gains" for W4A4 on every projection, gates included; "Anthology of
the SOTA, theory-128", section "The account" for the recurrence and gates):

  1. quantize x to NVFP4 (dynamic per-tensor amax);
  2. q, k, v, a, b = W4A4 projections of x; every weight is quantized on its
     own, with its own per-tensor scale (the pages warn that fusing modules
     that were scaled separately corrupts the gates when their global scales
     get mixed up: each projection keeps its own);
  3. log_alpha, beta = gates(a, b);
  4. o = gated delta rule over (L2-normalised) q, k and v; then
     y = W4A4 output projection of o (o quantized like x).

Readings: the four steps the task lists, no residual.  Optionally the rest of
a Gated DeltaNet block from its outside specification (``oracle.conv_norm``):
a short causal convolution with SiLU on q, k, v (``conv_w``) and an output
RMSNorm gated by SiLU of a sixth W4A4 projection g (``Wq["g"]`` with
``norm_w``).  Storage precision is mirrored where the GPU stores bf16: q, k,
v (before and after the convolution), g, o, the gated o and y are rounded to
bf16 (nearest-even); the gate pre-activations a, b stay unrounded.  FP64
except the quantizer (FP32).
"""
import numpy as np

from . import nvfp4
from .conv_norm import gated_rmsnorm, short_conv
from .gemm import gemm_fp64
from .gates import gates
from .delta_rule import delta_rule_chunked, delta_rule_sequential


def quantize_weights(W):
    """Each projection weight [out, in] quantized with its own amax / scale."""
    return {name: nvfp4.quantize(w) for name, w in W.items()}


def layer_forward(x, Wq, A_log, dt_bias, H, dk, dv, chunked=True, S0=None, x_g_enc=None, o_g_enc=None,
                  conv_w=None, norm_w=None):
    """x [B, T, d_model] (bf16 values); Wq: dict of quantized weights with keys
    q, k, v ([H*dk|H*dv, d_model]), a, b ([H, d_model]), out ([d_model, H*dv]),
    and optionally g ([H*dv, d_model], the output gate; needs ``norm_w``).
    ``x_g_enc`` / ``o_g_enc``: static (calibrated) FP32 encode scales of the
    two quantized activations, each module's own ("Critical Lessons for Model
    Serving"); None quantizes that activation with its own amax.
    ``conv_w`` [2*H*dk + H*dv, 4]: the short convolution over the q | k | v
    channels (None: none); ``norm_w`` [dv]: the output RMSNorm weight.
    Returns y [B, T, d_model] (bf16 values, FP64 array), the final state and a
    dict of intermediates."""
    B, T, D = x.shape
    xq = nvfp4.quantize(np.asarray(x, np.float32).reshape(B * T, D), g_enc=x_g_enc)
    gate = "g" in Wq
    proj = {n: gemm_fp64(xq, Wq[n]) for n in ("q", "k", "v", "a", "b") + (("g",) if gate else ())}
    qkv = np.concatenate([nvfp4.round_bf16(proj[n]) for n in ("q", "k", "v")], axis=1)
    if conv_w is not None:
        qkv = nvfp4.round_bf16(short_conv(qkv.reshape(B, T, -1), conv_w)[0]).reshape(B * T, -1)
    HK = H * dk
    q = qkv[:, :HK].reshape(B, T, H, dk)
    k = qkv[:, HK:2 * HK].reshape(B, T, H, dk)
    v = qkv[:, 2 * HK:].reshape(B, T, H, dv)
    log_alpha, beta = gates(proj["a"].reshape(B, T, H), proj["b"].reshape(B, T, H), A_log, dt_bias)
    scan = delta_rule_chunked if chunked else delta_rule_sequential
    o, S_T = scan(q, k, v, log_alpha, beta, S0=S0)
    o_bf = nvfp4.round_bf16(o).reshape(B * T, H * dv)
    o_in = o_bf
    if gate:
        g_bf = nvfp4.round_bf16(proj["g"])
        o_in = nvfp4.round_bf16(gated_rmsnorm(o_bf.reshape(B * T, H, dv), g_bf.reshape(B * T, H, dv),
                                              norm_w)).reshape(B * T, H * dv)
    oq = nvfp4.quantize(o_in.astype(np.float32), g_enc=o_g_enc)
    y = nvfp4.round_bf16(gemm_fp64(oq, Wq["out"])).reshape(B, T, D)
    inter = {"xq": xq, "q": q, "k": k, "v": v, "a": proj["a"], "b": proj["b"],
             "log_alpha": log_alpha, "beta": beta, "o": o, "o_bf16": o_bf, "oq": oq, "o_gated": o_in}
    return y, S_T, inter
