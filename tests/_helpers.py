"""Test-side helpers: layout conversions and error metrics (no method arithmetic)."""
import numpy as np
import torch


def tiled_to_linear(scales_tiled, rows, cols, row_offset=0):
    """Read a [rows, cols/16] linear scale matrix out of the tensor-core tiled
    layout documented in include/gdn.h (blocks of 128 rows x 4 scales = 512 B)."""
    s = np.asarray(scales_tiled, dtype=np.uint8).reshape(-1)
    kc = cols // 64
    r = np.arange(rows)[:, None] + row_offset
    j = np.arange(cols // 16)[None, :]
    off = (r // 128) * kc * 512 + (j // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (j % 4)
    return s[off]


def rel_fro(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def to_np(t):
    return t.detach().float().cpu().numpy() if t.dtype in (torch.bfloat16, torch.float16) else t.detach().cpu().numpy()


def bf16_cuda(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device).to(torch.bfloat16)


def f32_cuda(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)
