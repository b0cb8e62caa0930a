"""Pins of the oracle's 1-bit weight variant to facts outside the oracle.

unite.ai "Microsofts Inference Framework bringt 1-Bit grosse Sprachmodelle auf
lokale Geraete", "Mathematische Grundlagen", item 1 "Gewichtsbinarisierung",
eq. 1: W_b = Sign(W - alpha), alpha = mean(W), Sign(d) = +1 for d > 0 and -1
otherwise.  The expected values come from the hand-worked example under
tests/golden/, math.fsum, numpy's float32 arithmetic and int64 matmul,
closed forms and brute force over small bit patterns.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            rows.setdefault(key, []).append(vals)
    return rows


HAND = _read("hand_binary_4x4.txt")


def _f32(key):
    return np.array([[float(v) for v in r] for r in HAND[key]], np.float32)


def _int(key, dt):
    return np.array([[int(v, 0) for v in r] for r in HAND[key]], dt)


# --------------------------------------------------------------------------
# Hand-worked example
# --------------------------------------------------------------------------

def test_hand_alpha_beta_and_signs():
    W = _f32("W")
    W_b, alpha, beta = oracle.binarize_weights(W)
    assert alpha == np.float32(HAND["alpha"][0][0])
    assert beta == np.float32(HAND["beta"][0][0])
    np.testing.assert_array_equal(W_b, _int("W_b", np.int8))


def test_hand_accumulators_and_output():
    r = oracle.forward(_f32("x"), _int("W_b", np.int8), np.float32(0.328125))
    np.testing.assert_array_equal(r["acc"], _int("acc", np.int32))
    exact = np.array([[float(Fraction(v)) for v in row] for row in HAND["y"]])
    np.testing.assert_allclose(r["y64"], exact, rtol=1e-15, atol=0)
    np.testing.assert_allclose(r["y"], exact, rtol=1e-6, atol=0)
    np.testing.assert_array_equal(r["y"][1], exact[1].astype(np.float32))


def test_hand_packed_word():
    row = np.full((1, 32), -1, np.int8)
    row[0, :16] = _int("W_b", np.int8).ravel()
    assert int(oracle.pack_bits(row)[0, 0]) == int(HAND["packed_word"][0][0], 16)


# --------------------------------------------------------------------------
# alpha: exact signed mean
# --------------------------------------------------------------------------

@pytest.mark.parametrize("seed,shape,scale,shift", [
    (0, (64, 48), 1.0, 0.0), (1, (333, 17), 1e-3, 1e-4), (2, (16, 4096), 1e30, 0.0),
    (3, (128, 128), 1e-38, 0.0),          # subnormal-heavy
    (4, (1000, 250), 0.02, -0.001),
    (5, (7, 9), 1.0, 3.0),                # all positive
])
def test_exact_sum_matches_fsum(seed, shape, scale, shift):
    W = (np.random.default_rng(seed).standard_normal(shape) * scale + shift * scale).astype(np.float32)
    s64 = W.astype(np.float64).ravel()
    assert oracle.exact_sum(W) == math.fsum(s64)
    assert oracle.mean_alpha(W) == np.float32(math.fsum(s64) / s64.size)


def test_exact_sum_cancellation_and_extremes():
    v = np.array([1e30, 1.0, -1e30], np.float32)
    assert oracle.exact_sum(v) == 1.0
    v = np.array([3.4028235e38, 3.4028235e38, -1.4e-45], np.float32)
    assert oracle.exact_sum(v) == math.fsum(v.astype(np.float64))
    # ties broken by a term 2^-149 below them (float(Fraction) rounds once, correctly)
    for terms in ([1.0, 2.0 ** -53, 2.0 ** -149], [1.0, -(2.0 ** -54), -(2.0 ** -149)],
                  [-1.0, -(2.0 ** -53), -(2.0 ** -149)], [1.0, -(2.0 ** -60), 2.0 ** -149, -1.0]):
        exact = sum(Fraction(t) for t in terms)
        assert oracle.exact_sum(np.array(terms, np.float32)) == float(exact)
    assert oracle.exact_sum(np.array([1.0, 2.0 ** -53, 2.0 ** -149], np.float32)) == 1.0 + 2.0 ** -52
    assert oracle.exact_sum(np.array([1.0, -(2.0 ** -54), -(2.0 ** -149)], np.float32)) == 1.0 - 2.0 ** -53
    # a sum that is exactly zero, and one whose sign flips on the last element
    assert oracle.exact_sum(np.array([0.1, 0.2, -0.3, -0.1, -0.2, 0.3], np.float32)) == 0.0
    v = np.array([0.5, 0.25, -0.75, -2.0 ** -100], np.float32)
    assert oracle.exact_sum(v) == -(2.0 ** -100)


def test_alpha_special_cases():
    assert oracle.mean_alpha(np.full((8, 32), -0.75, np.float32)) == np.float32(-0.75)
    assert oracle.mean_alpha(np.zeros((3, 32), np.float32)) == 0
    W = workloads.latent_weights(9, 64, 128)
    assert oracle.mean_alpha(np.concatenate([W, -W])) == 0      # symmetric: exactly zero
    assert oracle.mean_alpha(-W) == -oracle.mean_alpha(W)         # odd
    assert oracle.mean_alpha(W * np.float32(4)) == oracle.mean_alpha(W) * np.float32(4)  # power-of-two scale


def test_alpha_closed_form_gaussian():
    # W ~ 0.02 N(0, 1) over 4096 x 4096: the mean is N(0, (0.02 / 4096)^2)
    W = workloads.latent_weights(0, 4096, 4096)
    assert abs(float(oracle.mean_alpha(W))) < 5 * 0.02 / 4096


# --------------------------------------------------------------------------
# Sign(W - alpha)
# --------------------------------------------------------------------------

def test_binarize_matches_numpy_float32():
    for seed in range(3):
        W = (workloads.latent_weights(seed, 97, 64) + np.float32(0.003 * seed)).astype(np.float32)
        alpha = oracle.mean_alpha(W)
        d = W - alpha                                        # numpy binary32 subtraction
        W_b = oracle.binarize(W, alpha)
        np.testing.assert_array_equal(W_b, np.where(d > 0, 1, -1).astype(np.int8))
        nz = d != 0                                          # np.sign agrees away from zero
        np.testing.assert_array_equal(W_b[nz], np.sign(d[nz]).astype(np.int8))


def test_binarize_sign_of_zero_is_minus_one():
    a = np.float32(0.1015625)
    W = np.array([[a, np.nextafter(a, np.float32(1)), np.nextafter(a, np.float32(-1)), 0.0, -0.0, 1.0, -1.0, a]],
                 np.float32)
    np.testing.assert_array_equal(oracle.binarize(W, a)[0], [-1, 1, -1, -1, -1, 1, -1, -1])
    np.testing.assert_array_equal(oracle.binarize(W[:, 3:5], 0.0)[0], [-1, -1])
    # a constant matrix equals its own mean everywhere: every sign is -1
    W_b, alpha, beta = oracle.binarize_weights(np.full((4, 32), 0.3, np.float32))
    assert alpha == np.float32(0.3) and beta == np.float32(0.3) and (W_b == -1).all()


def test_binarize_invariants():
    W = workloads.latent_weights(3, 300, 512)
    W_b, alpha, beta = oracle.binarize_weights(W)
    assert set(np.unique(W_b)) <= {-1, 1}
    assert beta == oracle.absmean_beta(W)
    order = np.argsort(W.ravel(), kind="stable")
    assert np.all(np.diff(W_b.ravel()[order].astype(np.int16)) >= 0)   # monotone in W
    # Gaussian: P(W > mean) = 1/2; sd of the fraction over 153600 draws is 0.0013
    assert abs(float(np.mean(W_b == 1)) - 0.5) < 5 * 0.0013


# --------------------------------------------------------------------------
# 1-bit packing
# --------------------------------------------------------------------------

def test_pack_bits_constant_rows():
    np.testing.assert_array_equal(oracle.pack_bits(np.ones((2, 64), np.int8)), np.full((2, 2), 0xFFFFFFFF, np.uint32))
    np.testing.assert_array_equal(oracle.pack_bits(-np.ones((2, 64), np.int8)), np.zeros((2, 2), np.uint32))
    # values <= 0 are stored as -1
    np.testing.assert_array_equal(oracle.pack_bits(np.zeros((1, 32), np.int8)), np.zeros((1, 1), np.uint32))


def test_pack_bits_single_positions():
    for t in range(32):
        W_b = -np.ones((1, 32), np.int8)
        W_b[0, t] = 1
        s, b = divmod(t, 4)
        assert int(oracle.pack_bits(W_b)[0, 0]) == 1 << (8 * b + s)


def test_pack_bits_byte_lane_extraction():
    # (word >> s) & 0x01010101 holds, in byte b, the bit of k = 32j + 4s + b
    W_b = np.where(np.random.default_rng(5).random((40, 96)) < 0.5, 1, -1).astype(np.int8)
    P = oracle.pack_bits(W_b)
    for j in range(3):
        for s in range(8):
            lanes = (P[:, j] >> np.uint32(s)) & np.uint32(0x01010101)
            for b in range(4):
                got = (lanes >> np.uint32(8 * b)) & np.uint32(1)
                np.testing.assert_array_equal(got, (W_b[:, 32 * j + 4 * s + b] > 0).astype(np.uint32))


def test_pack_bits_brute_force_all_16bit_patterns():
    pats = np.arange(1 << 16, dtype=np.int64)
    W_b = -np.ones((pats.size, 32), np.int8)
    for t in range(16):
        W_b[:, t] = np.where((pats >> t) & 1, 1, -1)
    P = oracle.pack_bits(W_b)
    assert len(np.unique(P)) == pats.size
    np.testing.assert_array_equal(oracle.unpack_bits(P, 32), W_b)


# --------------------------------------------------------------------------
# The contraction with binary weights
# --------------------------------------------------------------------------

def test_binary_acc_identity():
    # sum_k w x = 2 * sum_{w = +1} x - sum_k x, with int64 matmuls
    rng = np.random.default_rng(11)
    x_q = rng.integers(-127, 128, (5, 320)).astype(np.int8)
    W_b = np.where(rng.random((77, 320)) < 0.5, 1, -1).astype(np.int8)
    pos = (W_b > 0).astype(np.int64)
    expect = 2 * (x_q.astype(np.int64) @ pos.T) - x_q.astype(np.int64).sum(1, keepdims=True)
    np.testing.assert_array_equal(oracle.ternary_acc(x_q, W_b), expect)
    # extremes: |acc| = 127 K
    K = 4096
    x = np.full((1, K), 127, np.int8)
    W = np.ones((2, K), np.int8)
    W[1] = -1
    np.testing.assert_array_equal(oracle.ternary_acc(x, W)[0], [127 * K, -127 * K])
