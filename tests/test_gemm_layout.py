"""CPU emulation of the prefill GEMM's tile walk and operand layouts.

The tcgen05 GEMM is persistent: CTA b takes tiles b, b + grid, ... in
m-fastest order (128 x 256 output tiles), and per 128-byte K-block a TMA
box of x_q (128 rows, 128-byte swizzle, zero fill past M and K) and a box of
packed words (256 rows, zero fill) land in a stage; unpack warps expand each
word into 16-byte code chunks of the K-major, 128-byte-swizzled B operand
(2-bit trits: one chunk per word; 1-bit signs: two chunks per word, codes
{0, 2}); four MMAs of K = 32 walk both swizzled operands; the epilogue
subtracts the token's row sum.  This test restates those steps in numpy,
with garbage in the stage before every fill, and requires the oracle's
contraction, for ternary and for 1-bit weights.
"""
import numpy as np
import pytest

import oracle

BM, BN, BK = 128, 256, 128


def sw128_off(row, chunk):
    return row * 128 + ((chunk ^ (row & 7)) << 4)


def tma_box(src: np.ndarray, r0: int, c0: int, rows: int, cols: int) -> np.ndarray:
    """A [rows, cols] box of src starting at (r0, c0); zero outside src."""
    box = np.zeros((rows, cols), src.dtype)
    r1, c1 = min(src.shape[0], r0 + rows), min(src.shape[1], c0 + cols)
    if r1 > r0 and c1 > c0:
        box[:r1 - r0, :c1 - c0] = src[r0:r1, c0:c1]
    return box


def emulate(x_q, W_p, K, N, wbits, grid, rng):
    M = x_q.shape[0]
    tiles_m, tiles_n, num_kb = (M + BM - 1) // BM, (N + BN - 1) // BN, (K + BK - 1) // BK
    wpr = BK * wbits // 32                            # packed words per row and K-block
    xq_u8 = x_q.view(np.uint8)
    rowsum = x_q.astype(np.int64).sum(1)
    y = np.full((M, N), -(2 ** 40), np.int64)
    for cta in range(grid):
        for t in range(cta, tiles_m * tiles_n, grid):
            mb, nb = t % tiles_m, t // tiles_m
            D = np.zeros((BM, BN), np.int64)
            for kb in range(num_kb):
                a_st = rng.integers(0, 256, BM * BK, dtype=np.int64).astype(np.uint8)
                b_st = rng.integers(0, 256, BN * BK, dtype=np.int64).astype(np.uint8)
                # x_q box with the 128-byte swizzle
                box = tma_box(xq_u8, mb * BM, kb * BK, BM, BK)
                for r in range(BM):
                    for c in range(8):
                        a_st[sw128_off(r, c):sw128_off(r, c) + 16] = box[r, 16 * c:16 * c + 16]
                # packed words (no swizzle), then the unpack into swizzled code chunks
                words = tma_box(W_p, nb * BN, kb * wpr, BN, wpr)
                for n in range(BN):
                    for j in range(wpr):
                        w = int(words[n, j])
                        if wbits == 2:
                            t4 = [(w >> (2 * s)) & 0x03030303 for s in range(4)]
                            chunks = {j: t4}
                        else:
                            t8 = [(w << 1) & 0x02020202] + [(w >> (s - 1)) & 0x02020202 for s in range(1, 8)]
                            chunks = {2 * j: t8[:4], 2 * j + 1: t8[4:]}
                        for c, ts in chunks.items():
                            o = sw128_off(n, c)
                            b_st[o:o + 16] = np.array(ts, np.uint32).view(np.uint8)
                # four MMAs of K = 32 bytes: both operands read through the swizzle
                A = np.stack([np.concatenate([a_st[sw128_off(r, c):sw128_off(r, c) + 16] for c in range(8)])
                              for r in range(BM)]).view(np.int8).astype(np.int64)
                B = np.stack([np.concatenate([b_st[sw128_off(n, c):sw128_off(n, c) + 16] for c in range(8)])
                              for n in range(BN)]).view(np.int8).astype(np.int64)
                for k in range(BK // 32):
                    D += A[:, 32 * k:32 * k + 32] @ B[:, 32 * k:32 * k + 32].T
            for r in range(BM):
                m = mb * BM + r
                if m < M:
                    n0, n1 = nb * BN, min(N, nb * BN + BN)
                    y[m, n0:n1] = D[r, :n1 - n0] - rowsum[m]
    return y


@pytest.mark.parametrize("M,K,N,grid", [(130, 320, 300, 2), (64, 128, 513, 3), (257, 192, 40, 1)])
def test_ternary_gemm_emulation_matches_the_oracle(M, K, N, grid):
    rng = np.random.default_rng(M + K + N)
    W_t = rng.integers(-1, 2, (N, K)).astype(np.int8)
    x_q = rng.integers(-127, 128, (M, K)).astype(np.int8)
    y = emulate(x_q, oracle.pack(W_t), K, N, 2, grid, rng)
    np.testing.assert_array_equal(y, oracle.ternary_acc(x_q, W_t))


@pytest.mark.parametrize("M,K,N,grid", [(130, 384, 300, 2), (5, 128, 260, 1)])
def test_one_bit_gemm_emulation_matches_the_oracle(M, K, N, grid):
    rng = np.random.default_rng(M * 3 + K + N)
    W_b = np.where(rng.random((N, K)) < 0.5, 1, -1).astype(np.int8)
    x_q = rng.integers(-127, 128, (M, K)).astype(np.int8)
    y = emulate(x_q, oracle.pack_bits(W_b), K, N, 1, grid, rng)
    np.testing.assert_array_equal(y, oracle.ternary_acc(x_q, W_b))
