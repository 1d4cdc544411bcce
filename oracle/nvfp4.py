"""NVFP4 formats and the two-level NVFP4 quantizer (oracle; test infrastructure).

Method.  "Why Gated DeltaNet Survives 4-Bit Quantization" (franklineh.com
research summary), section "Why the 'Fragile' Recurrence is Actually Robust":
NVFP4 scales activations and weights in blocks of 16 elements, which keeps an
outlier's damage inside its own block.  The element format (E2M1), the block
scale format (E4M3, one per 16 elements) and the FP32 per-tensor scale are the
NVFP4 definition the task fixes; the pages give no bit-level recipe.

Reading of the recipe (the pages are silent; this is the plainest two-level
convention consistent with "E4M3 block scale + FP32 per-tensor scale").  All
arithmetic is IEEE FP32, round-to-nearest-even, one operation at a time:

  1. amax_t = max |x| over the tensor.  g_enc = 2688 / amax_t, where
     2688 = 6 * 448 (E2M1 max times E4M3 max).  amax_t == 0 gives g_enc = 1;
     a quotient that overflows FP32 is clamped to FLT_MAX.  The stored
     per-tensor *decode* scale is g = 1 / g_enc.
  2. Per block of 16 consecutive elements of a row: amax_b = max |x|,
     s_f = (amax_b / 6) * g_enc, s = E4M3(s_f) with RNE and saturation to 448.
  3. s_val = decode(s).  If s_val == 0 all 16 codes are 0x0.  Otherwise
     inv = g_enc / s_val and each element becomes code = E2M1(x * inv), RNE
     with saturation to 6; the sign bit is the sign of x * inv (a negative
     value that rounds to zero keeps its sign: code 0x8).
  4. Packing: element 2j of a row is the low nibble of byte j, element 2j+1
     the high nibble.
  5. Dequantised value: e2m1(code) * s_val * g, evaluated in FP64.

Rounding to a format is done on its value grid: inside the binade
[2^E, 2^(E+1)) a format with p significant bits has spacing 2^(E-p+1); below
the smallest normal the spacing is that of the smallest binade.  numpy.rint
rounds half to even, and an even multiple of the spacing is exactly a value
with an even last significand bit, so rint on the grid is RNE.
"""
import numpy as np

F32 = np.float32
FLT_MAX = np.finfo(np.float32).max

E2M1_MAX = 6.0
E4M3_MAX = 448.0


def round_to_grid(a, p, emin, maxval):
    """Round |a| (float64, exact copies of the inputs) to nearest-even on the
    grid of a binary format with ``p`` significant bits, smallest normal
    exponent ``emin`` and largest finite value ``maxval`` (saturating)."""
    a = np.abs(np.asarray(a, dtype=np.float64))
    _, e = np.frexp(a)                    # a = m * 2**e, m in [0.5, 1)
    E = np.maximum(e - 1, emin)           # binade exponent, clamped at emin
    spacing = np.ldexp(1.0, E - (p - 1))
    q = np.rint(a / spacing) * spacing    # exact: power-of-two scaling
    return np.minimum(q, maxval)


# ---------------------------------------------------------------- E2M1 ----
# E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit.
def e2m1_decode(codes):
    c = np.asarray(codes, dtype=np.int64) & 0xF
    exp = (c >> 1) & 3
    man = c & 1
    mag = np.where(exp == 0, man * 0.5, (1.0 + man / 2.0) * np.ldexp(1.0, exp - 1))
    return np.where(c & 8, -mag, mag)


def e2m1_encode(r):
    """FP32 values -> E2M1 codes (uint8 in [0, 15]), RNE, saturating."""
    r = np.asarray(r, dtype=np.float32)
    mag = round_to_grid(r, p=2, emin=0, maxval=E2M1_MAX)
    # magnitude -> 3-bit code: subnormal 0/0.5, then (1+m/2)*2^(e-1)
    _, e = np.frexp(mag)
    E = e - 1
    exp_field = np.where(mag < 1.0, 0, E + 1)
    man_field = np.where(mag < 1.0, (mag * 2).astype(np.int64),
                         np.rint((mag / np.ldexp(1.0, E) - 1.0) * 2).astype(np.int64))
    code = (exp_field.astype(np.int64) << 1) | man_field
    code = np.where(np.signbit(r), code | 8, code)
    return code.astype(np.uint8)


# ---------------------------------------------------------------- E4M3 ----
# E4M3 (the "FN" variant): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits,
# no infinities, S.1111.111 is NaN, largest finite 448.
def e4m3_decode(b):
    b = np.asarray(b, dtype=np.int64) & 0xFF
    exp = (b >> 3) & 15
    man = b & 7
    mag = np.where(exp == 0, man / 8.0 * 2.0 ** -6, (1.0 + man / 8.0) * np.ldexp(1.0, exp - 7))
    mag = np.where((exp == 15) & (man == 7), np.nan, mag)
    return np.where(b & 0x80, -mag, mag)


def e4m3_encode(v):
    """FP32 values -> E4M3 bytes, RNE, saturating to +-448 (satfinite)."""
    v = np.asarray(v, dtype=np.float32)
    assert np.all(np.isfinite(v)), "non-finite input is out of contract"
    mag = round_to_grid(v, p=4, emin=-6, maxval=E4M3_MAX)
    _, e = np.frexp(mag)
    E = e - 1
    normal = mag >= 2.0 ** -6
    exp_field = np.where(normal, E + 7, 0)
    man_field = np.where(normal,
                         np.rint((mag / np.ldexp(1.0, np.where(normal, E, 0)) - 1.0) * 8),
                         np.rint(mag / 2.0 ** -9)).astype(np.int64)
    out = (exp_field.astype(np.int64) << 3) | man_field
    out = np.where(np.signbit(v) & (mag > 0), out | 0x80, out)
    return out.astype(np.uint8)


# ------------------------------------------------------------ quantizer ----
def global_encode_scale(amax):
    """Step 1: g_enc = 2688 / amax_t in FP32 (1 for an all-zero tensor)."""
    amax = F32(amax)
    if amax == 0:
        return F32(1.0)
    with np.errstate(over="ignore", divide="ignore"):
        g = F32(F32(E2M1_MAX * E4M3_MAX) / amax)
    if not np.isfinite(g):
        g = F32(FLT_MAX)
    return g


def tensor_amax(x):
    x = np.asarray(x, dtype=np.float32)
    assert np.all(np.isfinite(x)), "non-finite input is out of contract"
    return F32(np.max(np.abs(x))) if x.size else F32(0.0)


def quantize(x, g_enc=None):
    """Quantize a [rows, K] FP32 array (bf16 values) to NVFP4.

    ``g_enc`` None means dynamic mode (amax over this tensor); otherwise the
    given FP32 encode scale is used.  Returns a dict with
      codes  uint8 [rows, K/2]   packed E2M1 (low nibble = even element)
      scales uint8 [rows, K/16]  E4M3 block scales, linear layout
      g      float32             per-tensor decode scale (1 / g_enc)
      g_enc  float32             per-tensor encode scale
      amax   float32             tensor amax (dynamic mode) or None
    """
    x = np.asarray(x, dtype=np.float32)
    assert x.ndim == 2 and x.shape[1] % 16 == 0
    rows, K = x.shape
    amax = None
    if g_enc is None:
        amax = tensor_amax(x)
        g_enc = global_encode_scale(amax)
    g_enc = F32(g_enc)
    blocks = x.reshape(rows, K // 16, 16)
    amax_b = np.max(np.abs(blocks), axis=2) if x.size else np.zeros((rows, 0), np.float32)
    s_f = (amax_b / F32(6.0)).astype(np.float32) * g_enc          # two FP32 ops
    s_f = s_f.astype(np.float32)
    scales = e4m3_encode(s_f)
    s_val = e4m3_decode(scales).astype(np.float32)                 # exact
    with np.errstate(divide="ignore", invalid="ignore"):
        inv = np.where(s_val > 0, g_enc / s_val, F32(0.0)).astype(np.float32)
    r = (blocks * inv[:, :, None]).astype(np.float32)              # FP32 mul
    codes = e2m1_encode(r)
    codes = np.where((s_val > 0)[:, :, None], codes, np.uint8(0)).astype(np.uint8)
    codes = codes.reshape(rows, K)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    g = F32(F32(1.0) / g_enc)
    return {"codes": packed, "scales": scales, "g": g, "g_enc": g_enc, "amax": amax}


def unpack_codes(packed):
    """[rows, K/2] packed bytes -> [rows, K] codes (low nibble first)."""
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty((packed.shape[0], packed.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out


def dequantize(codes, scales, g):
    """Step 5: x_hat = e2m1(code) * s_val * g in FP64, shape [rows, K]."""
    c = unpack_codes(codes)
    rows, K = c.shape
    vals = e2m1_decode(c).reshape(rows, K // 16, 16)
    s_val = e4m3_decode(scales)[:, :, None]
    return (vals * s_val * np.float64(g)).reshape(rows, K)


def round_bf16(a):
    """FP64 -> nearest-even bf16 value (returned as FP64).  bf16 has 8
    significant bits and FP32's exponent range; overflow is out of contract."""
    a = np.asarray(a, dtype=np.float64)
    mag = round_to_grid(a, p=8, emin=-126, maxval=np.inf)
    return np.where(np.signbit(a), -mag, mag)
