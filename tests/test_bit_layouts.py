"""CPU checks of the bit-level schemes the CUDA kernels are built on.

The kernels never unpack a weight to a value in {-1, 0, +1}: they mask
packed words so that each byte holds 2^e times a code, feed the bytes to
4-way byte dot products, and undo the scale with shifts.  These tests
restate those steps in numpy on words packed by the oracle and require the
result to equal the oracle's contraction, so a changed mask, shift or layout
constant fails here before any GPU run.  They also check the two shared-
memory layouts: the x_hat chunk swizzle (distinct bank groups for the eight
lanes of one shared-memory phase) and the 128-byte swizzle of the unpacked
GEMM operand.
"""
import numpy as np
import pytest

import oracle


def _bytes(words: np.ndarray) -> np.ndarray:
    """uint32 [...] -> unsigned byte lanes [..., 4] (lane b = bits 8b..8b+7)."""
    return ((words[..., None] >> (8 * np.arange(4, dtype=np.uint32))) & 0xFF).astype(np.int64)


def _dp4a_us(w_masked: np.ndarray, x4: np.ndarray) -> np.ndarray:
    """Sum over the 4 byte lanes of unsigned(w byte) * signed(x byte)."""
    return (_bytes(w_masked) * x4).sum(-1)


def _x_lanes(x_q: np.ndarray, k0: int) -> np.ndarray:
    """The 4 signed x bytes of k = k0 .. k0+3 for every token: [M, 4]."""
    return x_q[:, k0:k0 + 4].astype(np.int64)


@pytest.mark.parametrize("seed", [0, 1])
def test_two_bit_masked_dot_products_give_the_contraction(seed):
    # word j holds trit k = 16j + 4s + b at bits 8b + 2s; w & (0x03030303 << 2s)
    # leaves 4^s * code in byte b; a_s accumulates 4^s * sum(code * x) and
    # a0 + a1/4 + a2/16 + a3/64 - rowsum is the ternary contraction
    rng = np.random.default_rng(seed)
    M, N, K = 3, 7, 128
    W_t = rng.integers(-1, 2, (N, K)).astype(np.int8)
    x_q = rng.integers(-127, 128, (M, K)).astype(np.int8)
    W_p = oracle.pack(W_t)
    acc = np.zeros((M, N), np.int64)
    for n in range(N):
        a = np.zeros((M, 4), np.int64)
        for j in range(K // 16):
            w = np.uint32(W_p[n, j])
            for s in range(4):
                a[:, s] += _dp4a_us(np.uint32(w & np.uint32(0x03030303 << (2 * s))), _x_lanes(x_q, 16 * j + 4 * s))
        assert (a[:, 1] % 4 == 0).all() and (a[:, 2] % 16 == 0).all() and (a[:, 3] % 64 == 0).all()
        dot = a[:, 0] + (a[:, 1] >> 2) + (a[:, 2] >> 4) + (a[:, 3] >> 6)
        acc[:, n] = dot - x_q.astype(np.int64).sum(1)
    np.testing.assert_array_equal(acc, oracle.ternary_acc(x_q, W_t))


@pytest.mark.parametrize("seed", [0, 1])
def test_one_bit_masked_dot_products_give_the_contraction(seed):
    # word j holds the sign of k = 32j + 4s + b at bit 8b + s; masks
    # 0x01010101 << s (s < 4) on w and on w >> 4 leave 2^s * bit; the row
    # result is 2 * sum(bit * x) - rowsum
    rng = np.random.default_rng(seed + 10)
    M, N, K = 2, 5, 256
    W_b = np.where(rng.random((N, K)) < 0.5, 1, -1).astype(np.int8)
    x_q = rng.integers(-127, 128, (M, K)).astype(np.int8)
    W_p = oracle.pack_bits(W_b)
    acc = np.zeros((M, N), np.int64)
    for n in range(N):
        a = np.zeros((M, 4), np.int64)
        for j in range(K // 32):
            w = np.uint32(W_p[n, j])
            h = np.uint32(w >> np.uint32(4))
            for s in range(4):
                m = np.uint32(0x01010101 << s)
                a[:, s] += _dp4a_us(np.uint32(w & m), _x_lanes(x_q, 32 * j + 4 * s))
                a[:, s] += _dp4a_us(np.uint32(h & m), _x_lanes(x_q, 32 * j + 16 + 4 * s))
        dot = a[:, 0] + (a[:, 1] >> 1) + (a[:, 2] >> 2) + (a[:, 3] >> 3)
        acc[:, n] = 2 * dot - x_q.astype(np.int64).sum(1)
    np.testing.assert_array_equal(acc, oracle.ternary_acc(x_q, W_b))


def _xq_slot(c: int, wb: int) -> int:
    return c ^ ((c >> 3) & (3 if wb == 2 else 7))


@pytest.mark.parametrize("wb,chunks_per_group", [(2, 4), (1, 8)])
def test_x_hat_swizzle_is_a_permutation_with_distinct_bank_groups(wb, chunks_per_group):
    G = 4096 // 16                                       # 16-byte chunks of one token's x_hat
    slots = [_xq_slot(c, wb) for c in range(G)]
    assert sorted(slots) == list(range(G))               # a permutation of the row
    # the chunks of one weight group stay inside their aligned block
    for idx in range(G // chunks_per_group):
        block = {_xq_slot(chunks_per_group * idx + q, wb) for q in range(chunks_per_group)}
        assert block == set(range(chunks_per_group * idx, chunks_per_group * (idx + 1)))
    # eight consecutive lanes (one 128-byte shared-memory phase of 16-byte
    # loads) reading chunk q of their groups hit eight distinct bank groups
    for base in range(0, G // chunks_per_group - 8, 3):
        for q in range(chunks_per_group):
            banks = {_xq_slot(chunks_per_group * (base + l) + q, wb) % 8 for l in range(8)}
            assert len(banks) == 8


def test_gemm_unpack_codes_and_swizzled_placement():
    # 2-bit: chunk t_s = (w >> 2s) & 0x03030303 holds codes of k = 16j+4s..+3;
    # 1-bit: t_0 = (w << 1) & 0x02020202, t_s = (w >> (s-1)) & 0x02020202 hold
    # 2 * bit of k = 32j+4s..+3.  Chunk c of row n sits at 16-byte slot
    # c ^ (n % 8) of the row's 128 bytes (the 128-byte swizzle).
    rng = np.random.default_rng(3)
    W_t = rng.integers(-1, 2, (16, 64)).astype(np.int8)
    W_b = np.where(rng.random((16, 128)) < 0.5, 1, -1).astype(np.int8)
    P2, P1 = oracle.pack(W_t), oracle.pack_bits(W_b)
    for n in range(16):
        row2 = np.zeros(128, np.int64)
        for j in range(4):                       # 4 words = 64 trits = 4 chunks of 16 codes
            w = np.uint32(P2[n, j])
            chunk = np.concatenate([_bytes(np.uint32((w >> np.uint32(2 * s)) & np.uint32(0x03030303)))
                                    for s in range(4)])
            slot = (j ^ (n & 7)) * 16
            row2[slot:slot + 16] = chunk
        row1 = np.zeros(128, np.int64)
        for j in range(4):                       # 4 words = 128 signs = 8 chunks of 16 codes
            w = np.uint32(P1[n, j])
            t = [np.uint32((w << np.uint32(1)) & np.uint32(0x02020202))] + \
                [np.uint32((w >> np.uint32(s - 1)) & np.uint32(0x02020202)) for s in range(1, 8)]
            lo = (2 * j ^ (n & 7)) * 16
            hi = lo ^ 16                         # chunk 2j + 1
            assert hi == ((2 * j + 1) ^ (n & 7)) * 16
            row1[lo:lo + 16] = np.concatenate([_bytes(v) for v in t[:4]])
            row1[hi:hi + 16] = np.concatenate([_bytes(v) for v in t[4:]])
        # undo the swizzle and compare with the codes of the oracle's weights
        un2 = np.concatenate([row2[((c ^ (n & 7)) * 16):((c ^ (n & 7)) * 16) + 16] for c in range(4)])
        np.testing.assert_array_equal(un2, W_t[n].astype(np.int64) + 1)
        un1 = np.concatenate([row1[((c ^ (n & 7)) * 16):((c ^ (n & 7)) * 16) + 16] for c in range(8)])
        np.testing.assert_array_equal(un1, W_b[n].astype(np.int64) + 1)


def test_rms_cluster_slices_cover_every_chunk_once():
    # The RMS-folded quantiser shares a row among a cluster of 8 CTAs: CTA r
    # takes 16-element chunks [G r / 8, G (r + 1) / 8) and keeps them in a
    # shared-memory slice sized for ceil(G / 8) chunks (at most 40 KiB).
    C = 8
    for K in list(range(16, 4096, 16)) + [6912, 11008, 65536, 81920]:
        G = K // 16
        cap = (G + C - 1) // C
        assert cap * 16 * 4 <= 40 * 1024
        seen = []
        for r in range(C):
            g0, g1 = G * r // C, G * (r + 1) // C
            assert 0 <= g1 - g0 <= cap
            seen += range(g0, g1)
        assert seen == list(range(G))
