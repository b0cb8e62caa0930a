"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test names what fixes the expected value: the hand-worked example under
tests/golden/, a closed form, an invariant, brute force on tiny inputs, or a
library routine (math.fsum, numpy's int64 matmul).
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_hand():
    rows = {}
    with open(os.path.join(GOLDEN, "hand_4x4.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            rows.setdefault(key, []).append(vals)
    return rows


HAND = _read_hand()


def _f32(key):
    return np.array([[float(v) for v in r] for r in HAND[key]], np.float32)


def _int(key, dt=np.int64):
    return np.array([[int(v, 0) for v in r] for r in HAND[key]], dt)


# --------------------------------------------------------------------------
# Hand-worked 4x4 example
# --------------------------------------------------------------------------

def test_hand_beta_and_ternary_codes():
    W = _f32("W")
    beta = oracle.absmean_beta(W)
    assert beta == np.float32(HAND["beta"][0][0])
    W_t, beta2 = oracle.quantize_weights(W)
    assert beta2 == beta
    np.testing.assert_array_equal(W_t, _int("W_t", np.int8))


def test_hand_activation_quantiser_ties_to_even():
    x = _f32("x")
    x_q, gamma = oracle.quant_act(x)
    np.testing.assert_array_equal(gamma, np.array([float(v) for v in HAND["gamma"][0]], np.float32))
    np.testing.assert_array_equal(x_q, _int("x_q", np.int8))


def test_hand_accumulators_and_output():
    r = oracle.forward(_f32("x"), _int("W_t", np.int8), np.float32(0.28125))
    np.testing.assert_array_equal(r["acc"], _int("acc", np.int32))
    exact = np.array([[float(Fraction(v)) for v in row] for row in HAND["y"]])
    np.testing.assert_allclose(r["y64"], exact, rtol=1e-15, atol=0)
    np.testing.assert_allclose(r["y"], exact, rtol=1e-6, atol=0)
    np.testing.assert_array_equal(r["y"][1], exact[1].astype(np.float32))  # dyadic: exact
    bf = oracle.to_bf16(r["y"][1:2])
    np.testing.assert_array_equal(bf[0], _int("y_bf16_row1", np.uint16)[0])


def test_hand_packed_word():
    W_t = _int("W_t", np.int8).reshape(1, 16)
    assert int(oracle.pack(W_t)[0, 0]) == int(HAND["packed_word"][0][0], 16)


# --------------------------------------------------------------------------
# Packing
# --------------------------------------------------------------------------

@pytest.mark.parametrize("val,word", [(0, 0x55555555), (1, 0xAAAAAAAA), (-1, 0x00000000)])
def test_pack_constant_rows(val, word):
    # c = w + 1 repeated in every 2-bit field: 0b01.. = 0x55.., 0b10.. = 0xAA.., 0
    W_t = np.full((3, 64), val, np.int8)
    np.testing.assert_array_equal(oracle.pack(W_t), np.full((3, 4), word, np.uint32))


def test_pack_single_trit_positions():
    # a single +1 among zeros moves exactly one field from 01 to 10: the word
    # differs from 0x55555555 by the single bit pair at 8b + 2s for k = 4s + b.
    for t in range(16):
        W_t = np.zeros((1, 16), np.int8)
        W_t[0, t] = 1
        s, b = divmod(t, 4)
        expect = (0x55555555 & ~(3 << (8 * b + 2 * s))) | (2 << (8 * b + 2 * s))
        assert int(oracle.pack(W_t)[0, 0]) == expect


def test_pack_roundtrip_random_and_no_invalid_codes():
    g = np.random.default_rng(7)
    W_t = g.integers(-1, 2, size=(37, 16 * 23)).astype(np.int8)
    W_p = oracle.pack(W_t)
    back, bad = oracle.unpack(W_p, W_t.shape[1])
    assert bad == 0
    np.testing.assert_array_equal(back, W_t)
    # no field ever holds 3 (0b11): (w & (w >> 1)) has no set even bit
    assert not np.any((W_p & (W_p >> 1)) & 0x55555555)


def test_unpack_counts_invalid_fields():
    _, bad = oracle.unpack(np.array([[0xFFFFFFFF]], np.uint32), 16)
    assert bad == 16


def test_pack_brute_force_all_3pow8_halfwords():
    # every combination of the trits k = 0..7 (3^8 rows), trits 8..15 zero
    combos = np.array(np.meshgrid(*[[-1, 0, 1]] * 8, indexing="ij")).reshape(8, -1).T
    W_t = np.zeros((combos.shape[0], 16), np.int8)
    W_t[:, :8] = combos
    back, bad = oracle.unpack(oracle.pack(W_t), 16)
    assert bad == 0
    np.testing.assert_array_equal(back, W_t)
    assert len(np.unique(oracle.pack(W_t))) == 3 ** 8


# --------------------------------------------------------------------------
# absmean scale beta
# --------------------------------------------------------------------------

def _fsum_beta(W):
    a = np.abs(W.astype(np.float64)).ravel()
    return np.float32(math.fsum(a) / a.size)


@pytest.mark.parametrize("seed,shape,scale", [
    (0, (64, 48), 1.0), (1, (333, 17), 1e-3), (2, (16, 4096), 1e30),
    (3, (128, 128), 1e-38),             # subnormal-heavy
    (4, (1000, 250), 0.02),
])
def test_exact_abs_sum_matches_fsum(seed, shape, scale):
    W = (np.random.default_rng(seed).standard_normal(shape) * scale).astype(np.float32)
    assert oracle.exact_abs_sum(W) == math.fsum(np.abs(W.astype(np.float64)).ravel())
    assert oracle.absmean_beta(W) == _fsum_beta(W)


def test_exact_abs_sum_extreme_range():
    # largest and smallest binary32 magnitudes together: fsum is exact here too
    vals = np.array([3.4028235e38, 1.4e-45, -1.4e-45, 1.0, -2.5e-40, 1e20], np.float32)
    assert oracle.exact_abs_sum(vals) == math.fsum(np.abs(vals.astype(np.float64)))
    # exact rational check on a cancellation-prone set (all |.| so no cancellation
    # is possible; the sum must still carry the tiny terms)
    v = np.array([1.0, 2.0 ** -60, 2.0 ** -60, 2.0 ** -149], np.float32)
    exact = Fraction(1) + 2 * Fraction(2) ** -60 + Fraction(2) ** -149
    assert Fraction(oracle.exact_abs_sum(v)) == Fraction(float(exact))


def test_beta_special_cases():
    assert oracle.absmean_beta(np.zeros((8, 16), np.float32)) == 0
    assert oracle.absmean_beta(np.full((8, 16), -0.75, np.float32)) == np.float32(0.75)
    W_t, beta = oracle.quantize_weights(np.zeros((8, 16), np.float32))
    assert beta == 0 and not W_t.any()


def test_absmean_closed_form_gaussian():
    # W ~ 0.02 N(0,1): E|W| = 0.02 sqrt(2/pi); sd of the mean of 16.7M draws is
    # 0.02 sqrt(1 - 2/pi) / 4096 = 2.9e-6.  Zeros: |W| <= beta/2, so
    # P(0) = erf(0.5 sqrt(2/pi) / sqrt(2)) = 0.3101, each sign (1 - 0.3101)/2.
    W = workloads.latent_weights(0, 4096, 4096)
    W_t, beta = oracle.quantize_weights(W)
    mu = 0.02 * math.sqrt(2 / math.pi)
    assert abs(float(beta) - mu) < 5 * 2.9e-6
    p0 = math.erf(0.5 * math.sqrt(2 / math.pi) / math.sqrt(2))
    assert abs(p0 - 0.3101) < 1e-4
    frac0 = float(np.mean(W_t == 0))
    assert abs(frac0 - p0) < 1e-3
    assert abs(float(np.mean(W_t == 1)) - (1 - p0) / 2) < 1e-3
    assert abs(float(np.mean(W_t == -1)) - (1 - p0) / 2) < 1e-3


def test_ternarize_ties_and_clip():
    # with beta = 1 and eps = 0 the divisor is exactly 1, so q = W
    W = np.array([[0.5, -0.5, 1.5, -1.5, 2.5, 0.49999997, 0.50000006, -0.50000006,
                   0.0, -0.0, 100.0, -3e38, 1.0, -1.0, 0.75, -0.25]], np.float32)
    W_t = oracle.ternarize(W, 1.0, 0.0)
    np.testing.assert_array_equal(W_t[0], [0, 0, 1, -1, 1, 0, 1, -1, 0, 0, 1, -1, 1, -1, 1, 0])


def test_ternarize_invariants():
    W = workloads.latent_weights(3, 300, 512)
    W_t, beta = oracle.quantize_weights(W)
    assert set(np.unique(W_t)) <= {-1, 0, 1}
    # odd symmetry: ternarising -W gives -W_t (beta is unchanged)
    W_t2, beta2 = oracle.quantize_weights(-W)
    assert beta2 == beta
    np.testing.assert_array_equal(W_t2, -W_t)
    # monotone in W within a matrix
    order = np.argsort(W.ravel(), kind="stable")
    assert np.all(np.diff(W_t.ravel()[order].astype(np.int16)) >= 0)


# --------------------------------------------------------------------------
# Activation quantiser
# --------------------------------------------------------------------------

def test_quant_act_invariants():
    x = workloads.activations(5, 33, 1024, outliers=True)
    x_q, g = oracle.quant_act(x)
    assert np.all(np.abs(x_q.astype(np.int16)) <= 127)
    np.testing.assert_array_equal(np.abs(x_q.astype(np.int16)).max(axis=1), 127)
    np.testing.assert_array_equal(g, np.abs(x).max(axis=1))
    xn_q, gn = oracle.quant_act(-x)                        # odd symmetry
    np.testing.assert_array_equal(xn_q, -x_q)
    np.testing.assert_array_equal(gn, g)
    for j in (-3, 5):                                      # exact 2^j scaling
        xs_q, gs = oracle.quant_act(x * np.float32(2.0 ** j))
        np.testing.assert_array_equal(xs_q, x_q)
        np.testing.assert_array_equal(gs, g * np.float32(2.0 ** j))


def test_quant_act_zero_row_and_floor():
    x = np.zeros((2, 64), np.float32)
    x[1, 3] = 1e-7                                          # below the 1e-5 floor
    x_q, g = oracle.quant_act(x)
    np.testing.assert_array_equal(g, np.float32(1e-5))
    assert not x_q[0].any()
    assert x_q[1, 3] == 1                                   # 1e-7 * 127e5 = 1.27 -> 1


def test_quant_act_single_channel_levels():
    # x = k/127 * gamma for k = -127..127 maps back to k exactly
    k = np.arange(-127, 128, dtype=np.float32)
    x = (k * np.float32(2.0)).reshape(1, -1)                # gamma = 254, s = 0.5
    x_q, g = oracle.quant_act(x)
    assert g[0] == 254
    np.testing.assert_array_equal(x_q[0], k.astype(np.int8))


# --------------------------------------------------------------------------
# Ternary contraction
# --------------------------------------------------------------------------

def test_acc_brute_force_all_ternary_rows_k4():
    rows = np.array(np.meshgrid(*[[-1, 0, 1]] * 4, indexing="ij")).reshape(4, -1).T.astype(np.int8)
    assert rows.shape == (81, 4)
    g = np.random.default_rng(11)
    x_q = g.integers(-127, 128, size=(50, 4)).astype(np.int8)
    x_q[0] = 127
    x_q[1] = -127
    acc = oracle.ternary_acc(x_q, rows)
    np.testing.assert_array_equal(acc, x_q.astype(np.int64) @ rows.T.astype(np.int64))


def test_acc_matches_int64_matmul_and_bounds():
    g = np.random.default_rng(12)
    x_q = g.integers(-127, 128, size=(7, 1040)).astype(np.int8)
    W_t = g.integers(-1, 2, size=(129, 1040)).astype(np.int8)
    acc = oracle.ternary_acc(x_q, W_t)
    np.testing.assert_array_equal(acc, x_q.astype(np.int64) @ W_t.T.astype(np.int64))
    nnz = np.count_nonzero(W_t, axis=1)
    assert np.all(np.abs(acc) <= 127 * nnz[None, :])
    # extreme: every x = 127, every w = 1 -> 127 K
    K = 11008
    acc = oracle.ternary_acc(np.full((1, K), 127, np.int8), np.ones((1, K), np.int8))
    assert acc[0, 0] == 127 * K


def test_all_core_build_gives_the_same_accumulators():
    # the -fopenmp build of the same source (used for full-size checks) must
    # give the plain build's integers, which the int64 matmul pins
    g = np.random.default_rng(13)
    x_q = g.integers(-127, 128, size=(33, 2048)).astype(np.int8)
    W_t = g.integers(-1, 2, size=(301, 2048)).astype(np.int8)
    acc = oracle.ternary_acc_all_cores(x_q, W_t)
    np.testing.assert_array_equal(acc, oracle.ternary_acc(x_q, W_t))
    np.testing.assert_array_equal(acc, x_q.astype(np.int64) @ W_t.T.astype(np.int64))


# --------------------------------------------------------------------------
# Rescale and bf16
# --------------------------------------------------------------------------

def test_rescale_f32_within_tolerance_of_f64():
    g = np.random.default_rng(13)
    acc = g.integers(-1_398_016, 1_398_017, size=(9, 700)).astype(np.int32)
    gamma = (np.abs(g.standard_normal(9)) * 20 + 1e-3).astype(np.float32)
    beta = np.float32(0.0159577)
    y = oracle.rescale_f32(acc, beta, gamma)
    y64 = oracle.rescale_f64(acc, beta, gamma)
    # exact value as a fraction for a few entries
    for (m, n) in [(0, 0), (3, 17), (8, 699)]:
        exact = Fraction(int(acc[m, n])) * Fraction(float(beta)) * Fraction(float(gamma[m])) / 127
        assert abs(Fraction(float(y64[m, n])) - exact) <= abs(exact) * Fraction(1, 2 ** 50)
    nz = acc != 0
    rel = np.abs(y.astype(np.float64) - y64)[nz] / np.abs(y64[nz])
    assert rel.max() < 4 * 2.0 ** -24
    assert np.all(y[~nz] == 0)


def test_bf16_rounding_ties_to_even():
    vals = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 1.0 + 2 ** -8 + 2 ** -20,
                     0.0, -0.0, 65504.0], np.float32)
    bf = oracle.to_bf16(vals)
    np.testing.assert_array_equal(bf, np.array([0x3F80, 0x3F82, 0xBF80, 0x3F81, 0x0000, 0x8000, 0x4780],
                                               np.uint16))


# --------------------------------------------------------------------------
# Block glue
# --------------------------------------------------------------------------

def test_rms_rho_normalises_to_unit_rms():
    x = workloads.activations(9, 1, 2560)
    rho = oracle.rms_rho(x)
    h = x.astype(np.float64) * float(rho)
    assert abs(math.sqrt(np.mean(h * h)) - 1.0) < 1e-6
    # scale equivariance: rho(c x) = rho(x) / c for c a power of two (eps negligible)
    assert abs(float(oracle.rms_rho(x * 4)) * 4 / float(rho) - 1) < 1e-6


def test_quant_act_rmsnorm_folding():
    # the codes of Q(RMSNorm(x)) equal those of Q(x) up to the last-bit ties of
    # the binary32 product rho * x; the scale carries rho
    x = workloads.activations(10, 1, 2560)
    x_q, g_eff, rho = oracle.quant_act_rmsnorm(x)
    x_q0, g0 = oracle.quant_act(x)
    np.testing.assert_array_equal(x_q, x_q0)
    assert g_eff[0] == np.float32(g0[0] * rho)
    x_q_unfolded, g_unf = oracle.quant_act((x * rho).astype(np.float32))
    assert np.count_nonzero(x_q_unfolded != x_q) <= 3
    assert abs(float(g_unf[0]) / float(g_eff[0]) - 1) < 1e-6


def test_silu_mul_identities():
    g = np.random.default_rng(14).standard_normal(4096).astype(np.float32) * 6
    one = np.ones_like(g)
    s = oracle.silu_mul(g, one).astype(np.float64)
    sn = oracle.silu_mul(-g, one).astype(np.float64)
    # x sigma(x) - (-x) sigma(-x) = x (sigma(x) + sigma(-x)) = x
    np.testing.assert_allclose(s - sn, g.astype(np.float64), rtol=1e-6, atol=1e-6)
    z = oracle.silu_mul(np.array([0.0, 40.0, -40.0], np.float32), np.ones(3, np.float32))
    assert z[0] == 0 and z[1] == 40.0 and abs(z[2]) < 1e-15
    # sigma(x) in (0, 1): |silu(x)| < |x|
    assert np.all(np.abs(s) <= np.abs(g) + 1e-6)


def test_block_decode_structure():
    shapes = workloads.block_shapes()
    g = np.random.default_rng(15)
    tern = {}
    for p, (n, k, _) in shapes.items():
        Wt = g.integers(-1, 2, size=(n // 16, k // 16)).astype(np.int8)   # shrunken block
        tern[p] = (Wt, np.float32(0.01))
    x = workloads.activations(16, 1, 2560 // 16)
    r = oracle.block_decode(x, tern)
    # attention over a single token returns v; o consumes it
    xq_v, _ = oracle.quant_act(r["v"])
    np.testing.assert_array_equal(r["x_q_o"], xq_v)
    np.testing.assert_array_equal(r["out"], (r["h1"] + r["down"]).astype(np.float32))
    np.testing.assert_array_equal(r["h1"], (x + r["o"]).astype(np.float32))
    xq_u, _ = oracle.quant_act(r["u"])
    np.testing.assert_array_equal(r["x_q_down"], xq_u)


# --------------------------------------------------------------------------
# MatMul-free GLU (composition of pinned parts): structural pins
# --------------------------------------------------------------------------

def _glu_weights(D, F, seed):
    return {p: oracle.quantize_weights(workloads.latent_weights(seed + i, *shape))
            for i, (p, shape) in enumerate((("gate", (F, D)), ("up", (F, D)), ("down", (D, F))))}


def test_glu_zero_gate_gives_zero():
    # W_gate = 0: gate = 0, SiLU(0) = 0, u = 0, its codes 0, y = 0 exactly
    D, F = 128, 192
    tern = _glu_weights(D, F, 70)
    tern["gate"] = (np.zeros((F, D), np.int8), tern["gate"][1])
    r = oracle.glu(workloads.activations(71, 3, D, outliers=True), tern)
    assert not r["gate"].any() and not r["u"].any() and not r["u_q"].any() and not r["y"].any()


def test_glu_odd_in_up_and_down():
    # -W_up negates u exactly (binary64 product, symmetric rounding) and so y;
    # -W_down negates y exactly; the codes of x are untouched
    D, F = 256, 320
    tern = _glu_weights(D, F, 80)
    x = workloads.activations(81, 2, D, outliers=True)
    r = oracle.glu(x, tern)
    neg_up = dict(tern, up=(-tern["up"][0], tern["up"][1]))
    r2 = oracle.glu(x, neg_up)
    np.testing.assert_array_equal(r2["u"], -r["u"])
    np.testing.assert_array_equal(r2["y"], -r["y"])
    neg_down = dict(tern, down=(-tern["down"][0], tern["down"][1]))
    np.testing.assert_array_equal(oracle.glu(x, neg_down)["y"], -r["y"])


def test_glu_tokens_are_independent_and_match_the_block():
    D, F = 128, 256
    tern = _glu_weights(D, F, 90)
    x = workloads.activations(91, 4, D, outliers=True)
    r = oracle.glu(x, tern)
    for m in range(4):
        rm = oracle.glu(x[m:m + 1], tern)
        for k in ("gate", "up", "u", "y"):
            np.testing.assert_array_equal(rm[k][0], r[k][m])
    # the block's MLP half is the GLU of h1
    blk = {p: tern[p] for p in ("gate", "up", "down")}
    blk.update({p: oracle.quantize_weights(workloads.latent_weights(95 + i, D, D))
                for i, p in enumerate(("q", "k", "v", "o"))})
    ref = oracle.block_decode(x[0], blk)
    g = oracle.glu(ref["h1"], tern)
    for k, kb in (("gate", "gate"), ("up", "up"), ("u", "u"), ("y", "down")):
        np.testing.assert_array_equal(g[k].ravel(), np.asarray(ref[kb]).ravel())


# --------------------------------------------------------------------------
# Group quantisation: reductions to the ungrouped, pinned path
# --------------------------------------------------------------------------

def test_grouped_g1_is_the_ungrouped_path():
    W = workloads.latent_weights(120, 77, 256)
    x = workloads.activations(121, 3, 256, outliers=True)
    W_t, beta = oracle.quantize_weights_grouped(W, 1)
    W_t1, beta1 = oracle.quantize_weights(W)
    np.testing.assert_array_equal(W_t, W_t1)
    assert beta[0] == beta1
    r, r1 = oracle.forward_grouped(x, W_t, beta, 1), oracle.forward(x, W_t1, beta1)
    np.testing.assert_array_equal(r["acc"][0], r1["acc"])
    np.testing.assert_array_equal(r["y"], r1["y"])
    np.testing.assert_array_equal(r["gamma"][:, 0], r1["gamma"])


def test_grouped_error_bound_from_the_arithmetic():
    # binary32 evaluation against binary64: within (G + 2) 2^-24 of the sum of
    # the terms' magnitudes, even where the terms of different groups cancel
    W = workloads.latent_weights(150, 300, 2048)
    x = workloads.activations(151, 4, 2048, outliers=True)
    for G in (2, 4, 8):
        W_t, beta = oracle.quantize_weights_grouped(W, G)
        r = oracle.forward_grouped(x, W_t, beta, G)
        assert (np.abs(r["y"] - r["y64"]) <= (G + 2) * 2.0 ** -24 * r["yabs64"]).all()
        assert (r["yabs64"] >= np.abs(r["y64"])).all()


def test_grouped_duplicate_halves_double_exactly():
    # W = [A | A], x = [a | a], G = 2: equal parameters and accumulators in both
    # groups, so y = fl(t + t) = 2 t exactly
    A = workloads.latent_weights(130, 50, 128)
    a = workloads.activations(131, 2, 128, outliers=True)
    W_t, beta = oracle.quantize_weights_grouped(np.hstack([A, A]), 2)
    assert beta[0] == beta[1] == oracle.absmean_beta(A)
    r = oracle.forward_grouped(np.hstack([a, a]), W_t, beta, 2)
    At, bA = oracle.quantize_weights(A)
    np.testing.assert_array_equal(r["y"], 2 * oracle.forward(a, At, bA)["y"])


def test_grouped_zero_group_and_group_scales():
    # a zero column group contributes exactly 0; scaling one group by 2^3
    # scales only its beta and leaves every code unchanged
    W = workloads.latent_weights(140, 40, 256)
    x = workloads.activations(141, 2, 256)
    W0 = W.copy()
    W0[:, 128:] = 0
    W_t, beta = oracle.quantize_weights_grouped(W0, 2)
    assert beta[1] == 0 and not W_t[:, 128:].any()
    r = oracle.forward_grouped(x, W_t, beta, 2)
    Wt_a, b_a = oracle.quantize_weights(W[:, :128])
    np.testing.assert_array_equal(r["y"], oracle.forward(x[:, :128], Wt_a, b_a)["y"])
    W8 = W.copy()
    W8[:, 64:128] *= np.float32(8)
    # (eps = 0: the divisor guard would break the exact power-of-two scaling)
    W_t4, beta4 = oracle.quantize_weights_grouped(W, 4, eps=0.0)
    W_t8, beta8 = oracle.quantize_weights_grouped(W8, 4, eps=0.0)
    np.testing.assert_array_equal(W_t8, W_t4)
    assert beta8[1] == 8 * beta4[1] and all(beta8[g] == beta4[g] for g in (0, 2, 3))
    # activation groups: gamma per group is that group's absmax
    _, gam = oracle.quant_act_grouped(x, 4)
    for g in range(4):
        np.testing.assert_array_equal(gam[:, g], np.maximum(np.abs(x[:, 64 * g:64 * (g + 1)]).max(1), 1e-5))


def test_hand_grouped_example():
    rows = {}
    with open(os.path.join(GOLDEN, "hand_grouped_2x8.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, *vals = line.split()
                rows.setdefault(key, []).append(vals)
    W = np.array([[float(v) for v in r] for r in rows["W"]], np.float32)
    W_t, beta = oracle.quantize_weights_grouped(W, 2)
    np.testing.assert_array_equal(beta, np.array([float(v) for v in rows["beta"][0]], np.float32))
    np.testing.assert_array_equal(W_t, np.array([[int(v) for v in r] for r in rows["W_t"]], np.int8))
    x = np.array([[float(v) for v in rows["x"][0]]], np.float32)
    r = oracle.forward_grouped(x, W_t, beta, 2)
    np.testing.assert_array_equal(r["gamma"][0], [float(v) for v in rows["gamma"][0]])
    np.testing.assert_array_equal(r["x_q"][0], [int(v) for v in rows["x_q"][0]])
    np.testing.assert_array_equal(r["acc"][:, 0, :], [[int(v) for v in rows["acc0"][0]], [int(v) for v in rows["acc1"][0]]])
    exact = np.array([float(Fraction(v)) for v in rows["y"][0]])
    np.testing.assert_allclose(r["y64"][0], exact, rtol=1e-15, atol=0)
    assert (np.abs(r["y"][0] - exact) <= 4 * 2.0 ** -24 * r["yabs64"][0]).all()
