"""Pins of the oracle's block-diagonal Hadamard rotation against closed forms and a library routine."""

import numpy as np
import pytest
import scipy.linalg

from oracle import sylvester_hadamard, block_diag_hadamard, fwht_fp32, rotation_constant_fp32

ORDERS = [1, 2, 4, 8, 16, 32, 64, 128]


@pytest.mark.parametrize("n", ORDERS)
def test_closed_form_matches_scipy(n):
    np.testing.assert_array_equal(sylvester_hadamard(n), scipy.linalg.hadamard(n) / np.sqrt(n))


@pytest.mark.parametrize("n", ORDERS)
def test_orthonormal(n):
    H = sylvester_hadamard(n)
    np.testing.assert_allclose(H @ H.T, np.eye(n), atol=1e-15)
    np.testing.assert_array_equal(H, H.T)


def test_rotation_constants():
    assert rotation_constant_fp32(64) == np.float32(0.125)
    assert rotation_constant_fp32(128).view(np.uint32) == 0x3DB504F3
    assert rotation_constant_fp32(1) == np.float32(1.0)


@pytest.mark.parametrize("Bh", ORDERS)
def test_fwht_of_unit_vectors_is_the_column(Bh):
    # butterflies of a unit vector produce exact +-1, so the fp32 result is
    # exactly +-c_Bh: compare with the closed-form column rounded to fp32.
    I = np.eye(Bh, dtype=np.float32)
    out = fwht_fp32(I, Bh)           # row i = FWHT(e_i)
    expect = np.sign(sylvester_hadamard(Bh).T) * rotation_constant_fp32(Bh)
    np.testing.assert_array_equal(out, expect.astype(np.float32))


@pytest.mark.parametrize("D,Bh", [(64, 64), (128, 128), (128, 64), (128, 16), (64, 1), (128, 2)])
def test_fwht_equals_block_diag_matrix(D, Bh):
    rng = np.random.default_rng(0)
    x = rng.standard_normal((50, D)).astype(np.float32) * 3
    x[:, 5] *= 15
    got = fwht_fp32(x, Bh).astype(np.float64)
    ref = x.astype(np.float64) @ block_diag_hadamard(D, Bh).T
    # log2(Bh) fp32 add stages plus one multiply, each within one rounding of
    # the partial sums, whose magnitude is bounded by ||x_block||_1.
    stages = int(np.log2(Bh)) + 1
    bound = stages * 2.0 ** -23 * np.abs(x).sum(axis=1, keepdims=True)
    assert np.all(np.abs(got - ref) <= bound)


def test_block_diagonal_independence():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((1, 128)).astype(np.float32)
    y = x.copy()
    y[0, :64] += 1.0                 # change block 0 only
    a, b = fwht_fp32(x, 64), fwht_fp32(y, 64)
    np.testing.assert_array_equal(a[0, 64:], b[0, 64:])
    assert np.any(a[0, :64] != b[0, :64])


def test_fwht_is_an_involution_up_to_rounding():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((10, 128)).astype(np.float32)
    np.testing.assert_allclose(fwht_fp32(fwht_fp32(x, 128), 128), x, atol=2e-6)


def test_identity_block():
    x = np.random.default_rng(3).standard_normal((4, 64)).astype(np.float32)
    np.testing.assert_array_equal(fwht_fp32(x, 1), x)


def test_fixed_stage_order_is_pinned():
    # The fp32 result depends on the stage order; pin it against an explicit
    # loop over (h ascending, pairs (i, i+h) with i & h == 0).
    rng = np.random.default_rng(4)
    x = (rng.standard_normal(128) * 7).astype(np.float32)
    y = x.copy()
    h = 1
    while h < 128:
        z = y.copy()
        for i in range(128):
            if i & h == 0:
                z[i] = np.float32(y[i] + y[i + h])
                z[i + h] = np.float32(y[i] - y[i + h])
        y = z
        h *= 2
    y = (y * rotation_constant_fp32(128)).astype(np.float32)
    np.testing.assert_array_equal(fwht_fp32(x, 128), y)


def test_bad_block_rejected():
    with pytest.raises(ValueError):
        fwht_fp32(np.zeros(64, np.float32), 3)
    with pytest.raises(ValueError):
        fwht_fp32(np.zeros(64, np.float32), 128)
