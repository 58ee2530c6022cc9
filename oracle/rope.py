"""RoPE applied to keys and queries before the block Hadamard (oracle; test infrastructure only).

Source: the RoPE step in front of the cache's rotation -- the method's pages
take keys after RoPE ("SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for
Real-World LLM Serving", Abstract: a fused rotation-quantization step on the
projection outputs; the key transform is applied after RoPE).  RoPE itself is
the textbook rotary embedding: each pair of dimensions (a, b) with angle
theta is turned by theta, (a, b) -> (a cos - b sin, b cos + a sin).

Readings of this library:

* The angles come from a caller's table, fp32 [max_pos][R]: row p holds
  cos(theta_{p,i}) for the R/2 pairs, then sin(theta_{p,i}).
* Pairs: "neox" (i, i + R/2) or "gptj" (2i, 2i + 1), for dims < R; dims >= R
  pass through (partial rotary).
* Arithmetic: fp32 from the bf16 input, each product and each sum rounded to
  fp32 in that order (no fused multiply-add), and the fp32 result goes to the
  Hadamard rotation without a bf16 rounding in between, so that codes can be
  compared bit for bit.
"""

import numpy as np

NEOX, GPTJ = 0, 1


def rope_fp32(x, pos, cos_sin, R, style):
    """x: [..., D] fp32 values; pos: integer array broadcast to x.shape[:-1]; returns RoPE(x) in fp32."""
    x = np.asarray(x, np.float32)
    pos = np.broadcast_to(np.asarray(pos, np.int64), x.shape[:-1])
    cs = np.asarray(cos_sin, np.float32)[pos]                  # [..., R]
    half = R // 2
    c, s = cs[..., :half], cs[..., half:R]
    y = x.copy()
    if style == NEOX:
        a, b = x[..., :half], x[..., half:R]
        y[..., :half] = a * c - b * s                          # numpy fp32: every operation rounds
        y[..., half:R] = b * c + a * s
    elif style == GPTJ:
        a, b = x[..., 0:R:2], x[..., 1:R:2]
        y[..., 0:R:2] = a * c - b * s
        y[..., 1:R:2] = b * c + a * s
    else:
        raise ValueError("unknown RoPE style")
    return y
