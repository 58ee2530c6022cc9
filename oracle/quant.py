"""Token-wise asymmetric quantizer (oracle; test infrastructure only).

Sources:
* "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM
  Serving", Abstract -- token-wise INT4 quantization of the (rotated) cache.
* "KV4-RL: Unlocking Faster Asynchronous Rollouts for RLVR with INT4 KV Cache
  Quantization", Abstract -- calibration-free INT4; a bounded set of positions
  kept in INT8.

One quantization group is the D rotated values of one (token, KV head, K or V).
Each group gets its own scale s and zero point z, stored as fp16; the codes
are unsigned b-bit integers (b = 4 or 8, Q = 2^b - 1; b = 2 for the INT2 page
format, the folded-scale INT2 variant of the "KV Cache Quantization" topic
page, item 2, with the same token-wise groups and rounding rule).

Rounding rule (a reading of this library; the pages fix none of it):

1. values are clamped to the finite fp16 range [-65504, 65504] (NaN maps to
   -65504, the behaviour of fmax/fmin); the CUDA path flags any clamp in its
   status word;
2. mn = min x_i, mx = max x_i (exact);
3. z16 = mn rounded toward -inf to fp16;  z = float(z16);
4. r = fp32(mx - z);  s_f = fp32(r / Q)  (IEEE division, round to nearest even);
5. s16 = s_f rounded toward +inf to fp16, or 1.0 when r == 0;  s = float(s16);
6. c_i = clamp(rint_half_even(fp32(fp32(x_i - z) / s)), 0, Q);
7. dequantized value x^_i = fp32(c_i * s + z) with a single rounding (fma).

Directed rounding of z (down) and s (up) keeps z <= mn and z + Q*s >= mx for
the STORED fp16 values, so every element satisfies |x_i - x^_i| <= s/2 up to a
few fp32 ulps.  "bf16_round" is IEEE round-to-nearest-even to bfloat16.
"""

import numpy as np

FP16_MAX = np.float32(65504.0)


def clamp_fp16_range(x):
    """Clamp to [-65504, 65504] in fp32; NaN becomes -65504 (fmax/fmin semantics)."""
    x = np.asarray(x, dtype=np.float32)
    return np.fmin(np.fmax(x, -FP16_MAX), FP16_MAX).astype(np.float32)


def fp16_round_down(x):
    """Largest fp16 value <= x (x fp32, inside the fp16 range)."""
    x = np.asarray(x, dtype=np.float32)
    h = np.atleast_1d(x.astype(np.float16))  # round to nearest even first
    xv = np.atleast_1d(x)
    over = h.astype(np.float32) > xv
    h[over] = np.nextafter(h[over], np.float16(-np.inf))
    return h.reshape(x.shape)


def fp16_round_up(x):
    """Smallest fp16 value >= x (x fp32, inside the fp16 range)."""
    x = np.asarray(x, dtype=np.float32)
    h = np.atleast_1d(x.astype(np.float16))
    xv = np.atleast_1d(x)
    under = h.astype(np.float32) < xv
    h[under] = np.nextafter(h[under], np.float16(np.inf))
    return h.reshape(x.shape)


def quantize_groups(x, bits):
    """Quantize each group (last axis) of fp32 values.

    Returns (codes uint8 [..., D], s16 float16 [...], z16 float16 [...]).
    """
    if bits not in (2, 4, 8):
        raise ValueError("bits must be 2, 4 or 8")
    Q = np.float32(2 ** bits - 1)
    x = clamp_fp16_range(x)
    mn = x.min(axis=-1)
    mx = x.max(axis=-1)
    z16 = fp16_round_down(mn)
    z = z16.astype(np.float32)
    r = (mx - z).astype(np.float32)
    s_f = (r / Q).astype(np.float32)
    s16 = fp16_round_up(s_f)
    s16 = np.where(r == 0, np.float16(1.0), s16).astype(np.float16)
    s = s16.astype(np.float32)
    t = ((x - z[..., None]).astype(np.float32) / s[..., None]).astype(np.float32)
    codes = np.clip(np.rint(t), 0, Q).astype(np.uint8)
    return codes, s16, z16


def dequantize_groups(codes, s16, z16):
    """x^ = fp32(c*s + z) with one rounding.

    c <= 255 and s, z are fp16, so c*s + z is a multiple of 2^-24 below 2^25
    in magnitude: it is exact in fp64, and the single fp64 -> fp32 conversion
    is the one rounding an fma would make.
    """
    c = np.asarray(codes, dtype=np.float64)
    s = np.asarray(s16, dtype=np.float64)[..., None]
    z = np.asarray(z16, dtype=np.float64)[..., None]
    return (c * s + z).astype(np.float32)


def bf16_round(x):
    """Round fp32 values to the nearest bfloat16 (ties to even); returns fp32 holding bf16 values.

    NaN stays NaN; infinities stay infinite.
    """
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    rounded = ((u + 0x7FFF + lsb) >> 16) << 16
    out = rounded.astype(np.uint32).view(np.float32)
    return np.where(np.isnan(x), x, out).astype(np.float32)
