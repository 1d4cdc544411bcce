"""Recurrent-state trajectories through the library: the replay measurement.

"Why Gated DeltaNet Survives 4-Bit Quantization", section "Why the 'Fragile'
Recurrence is Actually Robust", follows the state of a GDN layer along long
sequences with every projection quantized to NVFP4 and compares it with a
clean trajectory; it also adds an impulse to the state and counts the tokens
until it has decayed.  This module produces the quantized side of that
measurement with the library's own kernels, so what it returns is the
product's state, not a model of it:

  * the activation and each weight are quantized by gdn_quantize_nvfp4, the
    q/k/v/a/b projections run as one block-scaled FP4 GEMM (gdn_gemm_nvfp4)
    and the gates are computed by gdn_gates;
  * the state is carried through gdn_delta_rule_fwd from checkpoint to
    checkpoint (the final state of one segment is the initial state of the
    next), so the states at the checkpoints are the ones a long prefill
    passes through;
  * an impulse is followed token by token with gdn_delta_rule_step.

Independent realisations of the quantization error come from a permutation of
the d_model axis applied to the activation and to every weight before
quantizing: x P (W P)^T = x W^T, but the 16-element blocks change.  The clean
reference trajectory is not computed here.  Every step of the method's
arithmetic runs in the library; torch supplies device memory and the norms
the measurement reads.
"""
import numpy as np
import torch

from . import _lib

PROJ = ("q", "k", "v", "a", "b")


def nvfp4_projections(x, W, H, dk, dv, perm=None, device="cuda"):
    """W4A4 projections of ``x`` ([M, d_model] bf16 values, numpy) with the
    FP32 weights ``W`` (dict q, k, v, a, b of [out, d_model]), the d_model axis
    permuted by ``perm`` first when given.  Returns device tensors: qkv bf16
    [M, 2*H*dk + H*dv] (q | k | v), a and b FP32 [M, H]."""
    x = np.asarray(x, dtype=np.float32)
    if perm is not None:
        x = x[:, perm]
        W = {n: np.asarray(W[n], dtype=np.float32)[:, perm] for n in PROJ}
    M, D = x.shape
    HK, HV = H * dk, H * dv
    NQKV = 2 * HK + HV
    dummy_out = np.zeros((64, HV), np.float32)     # the output projection is not used here
    lw = _lib.QuantizedLayerWeights({**{n: W[n] for n in PROJ}, "out": dummy_out}, np.zeros(H, np.float32),
                                    np.zeros(H, np.float32), H, dk, dv, device=device)
    xd = torch.from_numpy(np.ascontiguousarray(x)).to(device).to(torch.bfloat16)
    xc, xs, gx = _lib.gdn_quantize_nvfp4(xd)
    qkv = torch.empty((M, NQKV), dtype=torch.bfloat16, device=device)
    a = torch.empty((M, H), dtype=torch.float32, device=device)
    b = torch.empty((M, H), dtype=torch.float32, device=device)
    segs = [
        {"n_begin": 0, "n_end": HK, "kind": _lib.EPI_STORE_BF16, "g_b": lw.g["q"], "out": qkv, "ld_out": NQKV},
        {"n_begin": HK, "n_end": 2 * HK, "kind": _lib.EPI_STORE_BF16, "g_b": lw.g["k"], "out": qkv,
         "out_offset": HK, "ld_out": NQKV},
        {"n_begin": 2 * HK, "n_end": NQKV, "kind": _lib.EPI_STORE_BF16, "g_b": lw.g["v"], "out": qkv,
         "out_offset": 2 * HK, "ld_out": NQKV},
        {"n_begin": NQKV, "n_end": NQKV + H, "kind": _lib.EPI_STORE_F32, "g_b": lw.g["a"], "out": a, "ld_out": H},
        {"n_begin": NQKV + H, "n_end": NQKV + 2 * H, "kind": _lib.EPI_STORE_F32, "g_b": lw.g["b"], "out": b,
         "ld_out": H},
    ]
    _lib.gdn_gemm_nvfp4(xc, xs, gx, lw.codes, lw.scales, M, NQKV + 2 * H, D, segs)
    return qkv, a, b


def scan_inputs(qkv, a, b, A_log, dt_bias, T, H, dk, dv):
    """One sequence's scan inputs from the projections: q, k, v views
    [1, T, H, d] of ``qkv`` and the gates (gdn_gates) [1, T, H]."""
    HK = H * dk
    dev = qkv.device
    la, be = _lib.gdn_gates(a, b, torch.as_tensor(A_log, dtype=torch.float32).to(dev).contiguous(),
                            torch.as_tensor(dt_bias, dtype=torch.float32).to(dev).contiguous())
    qkv3 = qkv.view(1, T, -1)
    q = qkv3[:, :, :HK].unflatten(-1, (H, dk))
    k = qkv3[:, :, HK:2 * HK].unflatten(-1, (H, dk))
    v = qkv3[:, :, 2 * HK:].unflatten(-1, (H, dv))
    return q, k, v, la.view(1, T, H), be.view(1, T, H)


def states_at(q, k, v, la, be, checkpoints, S0=None):
    """The state [1, H, dk, dv] after each checkpoint token count, the scan
    run segment by segment with the state carried between segments."""
    out = []
    S, t_prev = S0, 0
    for t in checkpoints:
        _, S = _lib.gdn_delta_rule_fwd(q[:, t_prev:t], k[:, t_prev:t], v[:, t_prev:t], la[:, t_prev:t].contiguous(),
                                       be[:, t_prev:t].contiguous(), S0=S)
        out.append(S)
        t_prev = t
    _lib.stream_check()
    return out


def impulse_steps(q, k, v, la, be, t_imp, window, eps, seed):
    """Perturb the state after ``t_imp`` tokens by S (1 + eps z), z ~ N(0, 1)
    elementwise (numpy generator ``seed``), then carry the clean and the
    perturbed state token by token (gdn_delta_rule_step) over ``window``
    tokens.  Returns the number of tokens until ||dS|| per head first falls to
    1/e of its start (-1 if not within the window), numpy [H]."""
    H = q.shape[2]
    (S,) = states_at(q, k, v, la, be, (t_imp,))
    z = torch.from_numpy(np.random.default_rng(seed).standard_normal(S.shape).astype(np.float32)).to(S.device)
    S2 = torch.cat([S, S * (1.0 + eps * z)], dim=0).contiguous()      # [2, H, dk, dv]: clean, perturbed
    d = torch.empty((window + 1, H), dtype=torch.float32, device=S.device)
    d[0] = (S2[1] - S2[0]).flatten(1).norm(dim=1)
    for n in range(1, window + 1):
        t = t_imp + n - 1
        sl = slice(t, t + 1)
        q2, k2, v2 = (x[:, sl].expand(2, -1, -1, -1).contiguous() for x in (q, k, v))
        la2 = la[:, sl].expand(2, -1, -1).contiguous()
        be2 = be[:, sl].expand(2, -1, -1).contiguous()
        _lib.gdn_delta_rule_step(q2, k2, v2, la2, be2, S=S2, S_out=S2)
        d[n] = (S2[1] - S2[0]).flatten(1).norm(dim=1)
    _lib.stream_check()
    d = d.cpu().numpy()
    hit = d[1:] <= d[0][None, :] / np.e
    return np.where(hit.any(axis=0), hit.argmax(axis=0) + 1, -1)
