"""CPU emulation of the prefill GEMM's tile walk and operand layouts.

The tcgen05 GEMM is persistent: CTA b takes work units b, b + grid, ...;
a unit is a 128 MT x 256 output tile (m-fastest order) and, when there are few
tiles, one of `splits` ranges of its K-blocks.  From 256 tokens on (and no
split) a tile is two 128-row sub-tiles (MT = 2) whose two MMAs, into two
accumulators, read the same unpacked B block.  Per 128-byte K-block a TMA
box of x_q (128 rows, 128-byte swizzle, zero fill past M and K) and a box of
packed words (256 rows, zero fill) land in a stage; unpack warps expand each
word into 16-byte code chunks of the K-major, 128-byte-swizzled B operand
(2-bit trits: one chunk per word; 1-bit signs: two chunks per word, codes
{0, 2}); four MMAs of K = 32 walk both swizzled operands; the epilogue
subtracts the token's row sum.  With splits, each unit stores its int32 tile
to the workspace and a separate kernel adds the partial tiles of every
output, four columns per thread.  This test restates those steps in
numpy, with garbage in the stage before every fill and in the workspace,
restates the host's choice of splits and workspace size, checks every
partial-tile index against that size, and requires the oracle's
contraction, for ternary and for 1-bit weights.
"""
import numpy as np
import pytest

import oracle

BM, BN, BK = 128, 256, 128
SPLIT_UNITS_TARGET = 148
MT2_MIN_M = 256


def plan(M, N, K, allow_split=True):
    tiles_m, tiles_n, num_kb = (M + BM - 1) // BM, (N + BN - 1) // BN, (K + BK - 1) // BK
    tiles = tiles_m * tiles_n
    splits = max(1, min(SPLIT_UNITS_TARGET // tiles, num_kb)) if allow_split else 1
    mt, nfull = 1, 0
    if splits == 1:
        if M >= MT2_MIN_M:
            mt, tiles_m = 2, (M + 2 * BM - 1) // (2 * BM)
        nfull = tiles_m * tiles_n               # every tile whole
    cut = tiles_m * tiles_n - nfull
    part_rows = min(M, mt * BM)
    rowsum_bytes = (M * 4 + 255) // 256 * 256
    part_bytes = cut * splits * part_rows * BN * 4 if splits > 1 else 0
    return dict(mt=mt, nfull=nfull, tiles_m=tiles_m, tiles_n=tiles_n, num_kb=num_kb, splits=splits,
                part_rows=part_rows,
                ws_bytes=rowsum_bytes + part_bytes, part_off=rowsum_bytes)


def sw128_off(row, chunk):
    return row * 128 + ((chunk ^ (row & 7)) << 4)


def tma_box(src: np.ndarray, r0: int, c0: int, rows: int, cols: int) -> np.ndarray:
    """A [rows, cols] box of src starting at (r0, c0); zero outside src."""
    box = np.zeros((rows, cols), src.dtype)
    r1, c1 = min(src.shape[0], r0 + rows), min(src.shape[1], c0 + cols)
    if r1 > r0 and c1 > c0:
        box[:r1 - r0, :c1 - c0] = src[r0:r1, c0:c1]
    return box


def emulate(x_q, W_p, K, N, wbits, grid, rng, allow_split=False):
    M = x_q.shape[0]
    pl = plan(M, N, K, allow_split)
    tiles_m, tiles_n, num_kb, splits, part_rows = (pl[k] for k in ("tiles_m", "tiles_n", "num_kb", "splits",
                                                                    "part_rows"))
    TBM = BM * pl["mt"]                               # rows of a tile: MT sub-tiles of 128
    wpr = BK * wbits // 32                            # packed words per row and K-block
    xq_u8 = x_q.view(np.uint8)
    rowsum = x_q.astype(np.int64).sum(1)
    y = np.full((M, N), -(2 ** 40), np.int64)
    nfull = pl["nfull"]
    units = nfull + (tiles_m * tiles_n - nfull) * splits
    part_ints = (pl["ws_bytes"] - pl["part_off"]) // 4
    part = rng.integers(-2 ** 31, 2 ** 31, max(part_ints, 1), dtype=np.int64)   # garbage on entry
    kb_seen = np.zeros((tiles_m * tiles_n, num_kb), np.int64)
    for cta in range(grid):
        for u in range(cta, units, grid):
            if u < nfull:                             # a whole tile
                t, sp, kb0, kb1, cut = u, 0, 0, num_kb, False
            else:                                     # a K range of a cut tile
                t, sp = nfull + (u - nfull) // splits, (u - nfull) % splits
                kb0, kb1, cut = num_kb * sp // splits, num_kb * (sp + 1) // splits, splits > 1
            mb, nb = t % tiles_m, t // tiles_m
            D = np.zeros((TBM, BN), np.int64)             # MT accumulators of 128 rows
            for kb in range(kb0, kb1):
                kb_seen[t, kb] += 1
                a_st = rng.integers(0, 256, TBM * BK, dtype=np.int64).astype(np.uint8)
                b_st = rng.integers(0, 256, BN * BK, dtype=np.int64).astype(np.uint8)
                # x_q box with the 128-byte swizzle
                box = tma_box(xq_u8, mb * TBM, kb * BK, TBM, BK)
                for r in range(TBM):
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
                # four MMAs of K = 32 bytes per sub-tile: sub-tile a's A operand starts
                # 16 KiB into the stage, its rows read through the same swizzle
                B = np.stack([np.concatenate([b_st[sw128_off(n, c):sw128_off(n, c) + 16] for c in range(8)])
                              for n in range(BN)]).view(np.int8).astype(np.int64)
                for a in range(pl["mt"]):
                    base = a * BM * BK
                    A = np.stack([np.concatenate([a_st[base + sw128_off(r, c):base + sw128_off(r, c) + 16]
                                                  for c in range(8)])
                                  for r in range(BM)]).view(np.int8).astype(np.int64)
                    for k in range(BK // 32):
                        D[a * BM:(a + 1) * BM] += A[:, 32 * k:32 * k + 32] @ B[:, 32 * k:32 * k + 32].T
            if not cut:
                for r in range(TBM):                  # epilogue warp (sub-tile r // 128, lanes of r % 128)
                    m = mb * TBM + r
                    if m < M:
                        n0, n1 = nb * BN, min(N, nb * BN + BN)
                        y[m, n0:n1] = D[r, :n1 - n0] - rowsum[m]
                continue
            for r in range(TBM):                      # this unit's partial tile
                if r < part_rows and mb * TBM + r < M:
                    o = ((u - nfull) * part_rows + r) * BN
                    assert o + BN <= part_ints
                    part[o:o + BN] = D[r]
    assert np.all(kb_seen == 1)                       # every (tile, K-block) exactly once
    if splits > 1:                                    # the finishing kernel over the cut tiles' outputs
        ncut = tiles_m * tiles_n - nfull
        for e in range(ncut * part_rows * (BN // 4)):
            tt, rem = divmod(e, part_rows * (BN // 4))
            r, c = rem // (BN // 4), rem % (BN // 4) * 4
            t = nfull + tt
            m, n = (t % tiles_m) * TBM + r, (t // tiles_m) * BN + c
            if m < M and n < N:
                tot = np.zeros(4, np.int64)
                for s2 in range(splits):
                    o = ((tt * splits + s2) * part_rows + r) * BN + c
                    assert o + 4 <= part_ints
                    tot += part[o:o + 4]
                for j in range(4):
                    if n + j < N:
                        y[m, n + j] = tot[j] - rowsum[m]
    return y


@pytest.mark.parametrize("M,K,N,grid", [(130, 320, 300, 2), (64, 128, 513, 3), (257, 192, 40, 1)])
def test_ternary_gemm_emulation_matches_the_oracle(M, K, N, grid):
    rng = np.random.default_rng(M + K + N)
    W_t = rng.integers(-1, 2, (N, K)).astype(np.int8)
    x_q = rng.integers(-127, 128, (M, K)).astype(np.int8)
    y = emulate(x_q, oracle.pack(W_t), K, N, 2, grid, rng)
    np.testing.assert_array_equal(y, oracle.ternary_acc(x_q, W_t))


@pytest.mark.parametrize("M,K,N,grid", [(64, 1024, 1300, 40), (17, 640, 260, 7), (130, 512, 1000, 148),
                                        (64, 4096, 300, 16)])
def test_split_k_gemm_emulation_matches_the_oracle(M, K, N, grid):
    # few tiles: units of (tile, K range), partial tiles summed by the last
    # warp of each quarter; the chosen splits and the workspace they need
    pl = plan(M, N, K)
    assert pl["splits"] > 1
    assert pl["tiles_m"] * pl["tiles_n"] * pl["splits"] <= SPLIT_UNITS_TARGET
    rng = np.random.default_rng(M * 7 + K + N)
    W_t = rng.integers(-1, 2, (N, K)).astype(np.int8)
    x_q = rng.integers(-127, 128, (M, K)).astype(np.int8)
    y = emulate(x_q, oracle.pack(W_t), K, N, 2, grid, rng, allow_split=True)
    np.testing.assert_array_equal(y, oracle.ternary_acc(x_q, W_t))


def test_split_k_plan_of_the_small_batch_shapes():
    # M = 16 and 64 on K = 4096: 16 or 43 tiles, cut into 9 or 3 K ranges
    for M in (16, 64):
        assert plan(M, 4096, 4096)["splits"] == 9
        assert plan(M, 11008, 4096)["splits"] == 3
    # prefill: enough tiles, no split
    assert plan(2048, 4096, 4096)["splits"] == 1 and plan(2048, 11008, 4096)["splits"] == 1


@pytest.mark.parametrize("M,K,N,grid", [(130, 384, 300, 2), (5, 128, 260, 1)])
def test_one_bit_gemm_emulation_matches_the_oracle(M, K, N, grid):
    rng = np.random.default_rng(M * 3 + K + N)
    W_b = np.where(rng.random((N, K)) < 0.5, 1, -1).astype(np.int8)
    x_q = rng.integers(-127, 128, (M, K)).astype(np.int8)
    y = emulate(x_q, oracle.pack_bits(W_b), K, N, 1, grid, rng)
    np.testing.assert_array_equal(y, oracle.ternary_acc(x_q, W_b))


@pytest.mark.parametrize("M,K,N,grid,wbits,split", [(300, 128, 520, 3, 2, True), (600, 128, 260, 2, 1, True),
                                                     (256, 384, 300, 1, 2, False), (513, 256, 40, 2, 2, False)])
def test_two_sub_tile_gemm_emulation_matches_the_oracle(M, K, N, grid, wbits, split):
    # small shapes take two sub-tiles when K is not cut: one K-block, or no
    # split allowed (the workspace-free entry point)
    pl = plan(M, N, K, split)
    assert pl["mt"] == 2 and pl["splits"] == 1
    rng = np.random.default_rng(M * 5 + K + N + wbits)
    if wbits == 2:
        W = rng.integers(-1, 2, (N, K)).astype(np.int8)
        W_p = oracle.pack(W)
    else:
        W = np.where(rng.random((N, K)) < 0.5, 1, -1).astype(np.int8)
        W_p = oracle.pack_bits(W)
    x_q = rng.integers(-127, 128, (M, K)).astype(np.int8)
    np.testing.assert_array_equal(emulate(x_q, W_p, K, N, wbits, grid, rng, allow_split=split),
                                  oracle.ternary_acc(x_q, W))


def test_sub_tiles_of_the_prefill_shapes():
    for N in (4096, 11008):
        pl = plan(2048, N, 4096)
        assert pl["mt"] == 2 and pl["tiles_m"] == 8
    assert plan(64, 4096, 4096)["mt"] == 1 and plan(200, 4096, 4096)["mt"] == 1


@pytest.mark.parametrize("unpack_warps", [4, 8])
@pytest.mark.parametrize("mt", [1, 2])
def test_epilogue_warps_cover_every_tile_row_once(unpack_warps, mt):
    # Epilogue warps start after the producer, the MMA issuer and the unpack
    # warps; warp w may read only TMEM lanes 32 (w % 4) .. 32 (w % 4) + 31, so
    # it takes those lanes of sub-tile (w - first) / 4.  Every row of the
    # 128 MT-row tile must be read by exactly one thread.
    first = 2 + unpack_warps
    rows = []
    for w in range(first, first + 4 * mt):
        sub, q = (w - first) // 4, w % 4
        rows += [sub * BM + q * 32 + lane for lane in range(32)]
    assert sorted(rows) == list(range(BM * mt))
