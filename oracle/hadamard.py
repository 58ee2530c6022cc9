"""Block-diagonal Walsh-Hadamard rotation (oracle; test infrastructure only).

Source: "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM
Serving", Abstract -- keys and values are rotated by a block-diagonal Hadamard
transform before token-wise INT4 quantization.  Queries receive the same
rotation, so q.k is unchanged (an orthonormal H gives (Hq).(Hk) = q.k).

Readings of this library (the page gives none of these details):

* Sylvester ordering, normalised by 1/sqrt(Bh), no random sign flips.  The
  normalisation makes each block orthonormal (H H^T = I); a sign-randomised
  transform would be a different method (a randomised Hadamard).
* The rotation is applied independently to each of the D/Bh consecutive
  blocks of length Bh of a head vector (block-diagonal).  Bh = 1 is the
  identity (no rotation), which gives the page's "naive INT4" baseline.
* fp32 evaluation order, fixed so that the quantized codes are reproducible
  bit for bit: butterfly stages h = 1, 2, 4, ..., Bh/2 in ascending order,
  each pair (x_i, x_{i+h}) with (i & h) == 0 becomes (x_i + x_{i+h},
  x_i - x_{i+h}) rounded to fp32, and a single final multiply by
  c_Bh = fp32(1/sqrt(Bh)) rounded to nearest even.
"""

import numpy as np


def _is_pow2(n):
    return n >= 1 and (n & (n - 1)) == 0


def sylvester_hadamard(n):
    """Normalised Sylvester Hadamard matrix in fp64.

    Closed form: H[i, j] = (-1)^popcount(i AND j) / sqrt(n).
    """
    if not _is_pow2(n):
        raise ValueError("Hadamard order must be a power of two, got %r" % (n,))
    H = np.empty((n, n), dtype=np.float64)
    for i in range(n):
        for j in range(n):
            H[i, j] = -1.0 if bin(i & j).count("1") % 2 else 1.0
    return H / np.sqrt(n)


def block_diag_hadamard(D, Bh):
    """D x D block-diagonal matrix with D/Bh copies of sylvester_hadamard(Bh)."""
    if D % Bh:
        raise ValueError("block %d does not divide head_dim %d" % (Bh, D))
    H = np.zeros((D, D), dtype=np.float64)
    Hb = sylvester_hadamard(Bh)
    for b in range(D // Bh):
        H[b * Bh:(b + 1) * Bh, b * Bh:(b + 1) * Bh] = Hb
    return H


def rotation_constant_fp32(Bh):
    """c_Bh = 1/sqrt(Bh) rounded to the nearest fp32 (0.125 for 64, 0x3DB504F3 for 128)."""
    return np.float32(1.0 / np.sqrt(np.float64(Bh)))


def fwht_fp32(x, Bh):
    """Block-diagonal normalised Walsh-Hadamard transform of the last axis, in fp32.

    x: array [..., D] (any float dtype; widened to fp32 exactly when it holds
    bf16/fp16 values).  Returns fp32 [..., D] equal to H_blk @ x up to fp32
    rounding, evaluated in the fixed order stated in the module docstring.
    """
    x = np.asarray(x, dtype=np.float32)
    D = x.shape[-1]
    if not _is_pow2(Bh) or D % Bh:
        raise ValueError("bad Hadamard block %r for head_dim %r" % (Bh, D))
    lead = x.shape[:-1]
    nb = D // Bh
    y = x.reshape(lead + (nb, Bh)).copy()
    h = 1
    while h < Bh:
        # index inside a block: i = q*(2h) + s*h + r with s in {0, 1}; the pair
        # (s=0, s=1) at equal (q, r) is (x_i, x_{i+h}) with (i & h) == 0.
        y = y.reshape(lead + (nb, Bh // (2 * h), 2, h))
        a = y[..., 0, :]
        b = y[..., 1, :]
        y = np.stack([a + b, a - b], axis=-2)  # fp32 add / sub, round-to-nearest-even
        h *= 2
    y = y.reshape(lead + (D,))
    return (y * rotation_constant_fp32(Bh)).astype(np.float32)
