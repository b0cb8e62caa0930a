"""CPU restatement of the library's exact sum of |W| (and of the positive and
negative parts, for the 1-bit mean) against the oracle's 384-bit sum.

The weight-preparation kernels add every |w| exactly: an element whose
exponent is within 38 of the largest one is an integer on the grid
2^(E - 188) and goes into a 128-bit sum; a smaller one is an integer on the
grid 2^-149, split by exponent block of 16 into sixteen 128-bit sums.  The
last CTA places all sums into one multi-word integer (32-bit words) and
rounds it once to binary64 (top 64 bits, the sticky bit OR-ed into the
lowest).  This test restates those steps in Python -- the element split, the
word placement, the word-wise subtraction with borrow and the rounding -- and
requires the result to equal the oracle's exactly, on inputs built to reach
every branch: subnormals, elements far below the maximum, cancellation, all
zeros, one element.  The GPU parity tests then check the kernels themselves on
the same kinds of input.
"""
import math
import struct

import numpy as np
import pytest

import oracle

SMALL_BLOCKS, SMALL_BITS, WORDS = 16, 16, 24


def bits(x):
    return struct.unpack("<I", struct.pack("<f", float(x)))[0]


def split(w, E):
    """(fast sum on grid 2^(E-188), [block sums on grid 2^-149]) of |w|."""
    fast, small = 0, [0] * SMALL_BLOCKS
    for v in np.asarray(w, np.float32).ravel():
        u = bits(v) & 0x7FFFFFFF
        e = u >> 23
        m = (u & 0x7FFFFF) | (0x800000 if e else 0)
        if m == 0:
            continue
        ee = e if e else 1
        sh = ee - E + 38
        if sh >= 0:
            assert (m << sh) < 2 ** 62
            fast += m << sh
        else:
            t = ee - 1
            small[t // SMALL_BITS] += m << (t % SMALL_BITS)
    assert fast < 2 ** 128 and all(s < 2 ** 128 for s in small)
    return fast, small


def big_add(words, v, shift):
    for k in range(4):
        piece = (v >> (32 * k)) & 0xFFFFFFFF
        pos = shift + 32 * k
        x = piece << (pos & 31)
        words[pos >> 5] += x & 0xFFFFFFFF
        words[(pos >> 5) + 1] += x >> 32


def normalise(words):
    for i in range(WORDS - 1):
        words[i + 1] += words[i] >> 32
        words[i] &= 0xFFFFFFFF
    assert words[-1] < 2 ** 32


def exact_total(fast, small, E):
    w = [0] * WORDS
    if E < 39:
        big_add(w, fast, 0)
        unit = E - 188
    else:
        big_add(w, fast, E - 39)
        for b in range(SMALL_BLOCKS):
            big_add(w, small[b], SMALL_BITS * b)
        unit = -149
    normalise(w)
    return w, unit


def bits64(w, lo):
    L, o = lo >> 5, lo & 31
    t = w[L] >> o
    if L + 1 < WORDS:
        t |= w[L + 1] << (32 - o)
    if L + 2 < WORDS and o:
        t |= w[L + 2] << (64 - o)
    return t & (2 ** 64 - 1)


def to_double(w, unit):
    top = WORDS - 1
    while top >= 0 and w[top] == 0:
        top -= 1
    if top < 0:
        return 0.0
    msb = 32 * top + w[top].bit_length() - 1
    lsb = msb - 63
    if lsb <= 0:
        return math.ldexp(float(bits64(w, 0)), unit)
    t = bits64(w, lsb)
    sticky = (w[lsb >> 5] & ((1 << (lsb & 31)) - 1)) != 0 or any(w[i] for i in range(lsb >> 5))
    return math.ldexp(float(t | int(sticky)), lsb + unit)   # float(int) rounds to nearest even


def lib_abs_sum(w):
    a = np.abs(np.asarray(w, np.float32)).view(np.uint32).max()
    E = max(int(a) >> 23, 1)
    fast, small = split(w, E)
    return to_double(*exact_total(fast, small, E))


def lib_signed_sums(w):
    """(sum |w|, sum w) as the 1-bit preparation forms them."""
    w = np.asarray(w, np.float32).ravel()
    a = np.abs(w).view(np.uint32).max()
    E = max(int(a) >> 23, 1)
    P, up = exact_total(*split(w[~np.signbit(w)], E), E)
    Q, _ = exact_total(*split(w[np.signbit(w)], E), E)
    top = WORDS - 1
    while top > 0 and P[top] == Q[top]:
        top -= 1
    neg = Q[top] > P[top]
    hi, lo = (Q, P) if neg else (P, Q)
    A, D, borrow = [0] * WORDS, [0] * WORDS, 0
    for i in range(WORDS):
        A[i] = P[i] + Q[i]
        D[i] = (hi[i] - lo[i] - borrow) & 0xFFFFFFFF
        borrow = 1 if hi[i] < lo[i] + borrow else 0
    assert borrow == 0
    normalise(A)
    s = to_double(D, up)
    return to_double(A, up), -s if neg else s


def cases():
    g = np.random.default_rng(0)
    yield "gaussian", (g.standard_normal(4096) * 0.02).astype(np.float32)
    yield "subnormals", (g.standard_normal(300) * 1e-42).astype(np.float32)
    yield "far_below_max", np.concatenate([[3.0e3], g.standard_normal(500) * 2.0 ** -45,
                                           g.standard_normal(500) * 2.0 ** -60]).astype(np.float32)
    yield "every_exponent", np.array([math.ldexp(1.0 + i / 300.0, e) * (-1) ** i for i, e in
                                      enumerate(range(-149, 128))], np.float32)
    yield "wide_random", (g.standard_normal(2000) * np.exp2(g.uniform(-140, 120, 2000))).astype(np.float32)
    yield "tiny_max", (g.standard_normal(100) * 2.0 ** -120).astype(np.float32)    # E < 39
    yield "all_zero", np.zeros(64, np.float32)
    yield "one_element", np.array([-7.5e-39], np.float32)
    yield "max_float", np.array([3.4028235e38, 3.4028235e38, -1e-45], np.float32)
    yield "cancel", np.array([1.0, -1.0, 2.0 ** -140, -(2.0 ** -149)], np.float32)
    # sums that land on binary64 ties: the sticky bit must break them
    yield "tie", np.array([2.0 ** 60, 1.0, 2.0 ** -80], np.float32)


@pytest.mark.parametrize("name,w", list(cases()), ids=[c[0] for c in cases()])
def test_abs_sum_scheme_equals_the_oracle(name, w):
    assert lib_abs_sum(w) == oracle.exact_abs_sum(w)


@pytest.mark.parametrize("name,w", list(cases()), ids=[c[0] for c in cases()])
def test_signed_sum_scheme_equals_the_oracle(name, w):
    a, s = lib_signed_sums(w)
    assert a == oracle.exact_abs_sum(w)
    assert s == oracle.exact_sum(w)
