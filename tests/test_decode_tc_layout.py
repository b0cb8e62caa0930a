"""CPU emulation of the swap-AB tensor-core decode kernel's index arithmetic.

The kernel (tcgen05, weight rows on the MMA's 128 lanes, tokens on N) moves
every operand through a layout of its own: a 2-D TMA ring with the 128-byte
swizzle, unpacked code bytes in tensor memory (4 K-bytes per 32-bit column,
one lane per weight row), x_hat in shared memory as 128-byte-swizzled K-major
rows in S slice blocks and G column groups, and an epilogue that adds column
groups (>> 2s) and slices.  This test restates those steps in numpy -- the
host split (slices, tiles, lanes, ring slots), the ring contents including
the stale bytes of slices past K, the unpack of each 128-trit quarter, the
MMA walk over K and the epilogue -- for packed words from the oracle, and
requires the oracle's contraction.  Garbage fills every byte the kernel does
not write, so a read of an unwritten byte changes the result.
"""
import numpy as np
import pytest

import oracle

STAGE_K, QK, NBUF, MAX_NMMA, MAX_SLOTS, MAX_M, HDR = 512, 128, 6, 64, 16, 16, 3072


def ru(v, a):
    return (v + a - 1) // a * a


def pow2(v):
    r = 1
    while r < v:
        r <<= 1
    return r


def split(mp, K, R):
    """Slices S (placed in different TMEM subpartitions) and row tiles: the
    fewest tiles x slice length (MMAs per CTA), ties to fewer tiles."""
    best = None
    for s in (1, 2, 4):
        if s * mp > MAX_NMMA:
            continue
        lf = ru((K + s - 1) // s, STAGE_K)
        if (s - 1) * lf >= K:
            continue
        nt = (R + 128 // s - 1) // (128 // s)
        if best is None or nt * lf < best[0]:
            best = (nt * lf, dict(S=s, Lfull=lf, ntiles=nt, Rt=(R + nt - 1) // nt))
    return (best[1], True) if best else (None, False)


def layout(G, M, K, N, sms, budget):
    if M < 1 or M > MAX_M or K < 64 or K % 64 or N < 1:
        return None
    mp = pow2(M)
    R = (N + sms - 1) // sms
    sp, ok = split(mp, K, R)
    if not ok or (G == 4 and 4 * sp["S"] * mp > 16):
        return None
    p = dict(sp, G=G, M=M, K=K, N=N, R=R, mp=mp, grid=(N + R - 1) // R)
    S, Rt = p["S"], p["Rt"]
    p["T"] = p["Lfull"] // STAGE_K
    p["Rt8"] = ru(Rt, 8)
    p["L"] = (Rt + (4 // S) - 1) // (4 // S)
    p["stage_bytes"] = S * p["Rt8"] * 128
    p["brow"] = ru(S * mp * G, 8)
    p["nmma"] = max(16, ru(S * mp * G, 16))
    if p["nmma"] > MAX_NMMA or p["L"] > 32:
        return None
    p["b_off"] = ru(HDR + Rt * mp * 4, 1024)
    b_bytes = p["T"] * (STAGE_K // QK) * p["brow"] * 128 + (1024 if p["nmma"] > p["brow"] else 0)
    p["ring_off"] = p["b_off"] + b_bytes
    avail = budget - 1024 - p["ring_off"]
    units = p["ntiles"] * p["T"]
    slots = min(units, MAX_SLOTS, avail // p["stage_bytes"])
    if slots < min(units, 2):
        return None
    p["slots"] = slots
    p["smem"] = p["ring_off"] + slots * p["stage_bytes"]
    return p


def configure(M, K, N, sms, budget):
    return layout(4, M, K, N, sms, budget) or layout(1, M, K, N, sms, budget)


def sw128(row, chunk):
    """Byte offset of 16-byte chunk `chunk` of 128-byte row `row` in a 128-byte-swizzled tile."""
    return (row // 8) * 1024 + (row % 8) * 128 + ((chunk ^ (row % 8)) << 4)


NW = 12                  # unpack warps


def row_rowsum(x_q, M, K, mp, S, KC, Lfull):
    """Row sums of x_hat as the staging pass forms them: B row j = q * mp + m
    (slice q, token m) to warp j % NW, its KC chunks to the lanes (lane l
    takes chunks l, l + 32, ...), a warp sum per row and one shared add per
    row into token m's total."""
    rows = [0] * mp
    for w in range(NW):
        for j in range(w, S * mp, NW):
            q, m = divmod(j, mp)
            ls = min(Lfull, K - q * Lfull) if m < M else 0
            lane_sums = [0] * 32
            for lane in range(32):
                for kc in range(lane, KC, 32):
                    if kc * 16 < ls:
                        k0 = q * Lfull + kc * 16
                        lane_sums[lane] += int(x_q[m, k0:k0 + 16].astype(np.int64).sum())
            if sum(lane_sums) != 0:
                rows[m] += sum(lane_sums)
    return rows


def emulate(p, Wbytes, x_q, rng):
    """acc [M, N] as the kernel computes it."""
    M, K, N, G, S, T, mp = p["M"], p["K"], p["N"], p["G"], p["S"], p["T"], p["mp"]
    Rt, Rt8, L, brow, nmma, Lfull = p["Rt"], p["Rt8"], p["L"], p["brow"], p["nmma"], p["Lfull"]
    acc = np.full((M, N), -(2 ** 40), np.int64)
    for cta in range(p["grid"]):
        r0 = cta * p["R"]
        nrows = min(p["R"], N - r0)
        smem = rng.integers(0, 256, p["smem"] + 1024, dtype=np.int64).astype(np.uint8)   # garbage
        # ---- B: x_hat rows j = (q * mp + m) * G + g per 128-trit K-block of the slice
        KC = T * (STAGE_K // 16)
        for m in range(mp):
            for idx in range(S * KC):
                q, kc = divmod(idx, KC)
                kl, ls = kc * 16, min(Lfull, K - q * Lfull)
                v = np.zeros(16, np.int8)
                if m < M and kl < ls:
                    v = x_q[m, q * Lfull + kl:q * Lfull + kl + 16]
                kb_off = (kc >> 3) * brow * 128
                for g in range(G):
                    j = (q * mp + m) * G + g
                    vg = v.copy()
                    if G == 4:                                   # group g keeps bytes 4g .. 4g+3
                        vg[:] = 0
                        vg[4 * g:4 * g + 4] = v[4 * g:4 * g + 4]
                    o = p["b_off"] + kb_off + j * 128 + (((kc & 7) ^ (j & 7)) << 4)
                    smem[o:o + 16] = vg.view(np.uint8)
        rowsum = row_rowsum(x_q, M, K, mp, S, KC, Lfull)
        part = np.zeros((Rt, mp), np.int64)
        u4 = 0
        for tile in range(p["ntiles"]):
            y0 = r0 + tile * Rt
            D = np.zeros((128, nmma), np.int64)
            for t in range(T):
                u = tile * T + t
                base = p["ring_off"] + (u % p["slots"]) * p["stage_bytes"]
                # ---- TMA: 128 bytes of each of Rt rows per slice, zero fill outside [N, K/4)
                for q in range(S):
                    k0 = q * Lfull + t * STAGE_K
                    if k0 >= K:
                        continue                                 # not loaded: stale bytes stay
                    x0, dst = k0 // 4, base + q * Rt8 * 128
                    assert dst % 1024 == 0 and x0 % 16 == 0
                    for r in range(Rt):
                        row = np.zeros(128, np.uint8)
                        if y0 + r < N:
                            seg = Wbytes[y0 + r, x0:x0 + 128]
                            row[:len(seg)] = seg
                        for c in range(8):
                            o = dst + sw128(r, c)
                            smem[o:o + 16] = row[16 * c:16 * c + 16]
                # ---- four 128-trit quarters: unpack into a TMEM A buffer, then 4 MMAs of K = 32
                for qq in range(4):
                    kq = 4 * t + qq
                    A = np.zeros((128, 32), np.uint32)           # TMEM lanes x 32 columns of 4 K-bytes
                    for sp in range(4):
                        P = 4 // S
                        q = sp // P
                        for lane in range(32):
                            n = (sp % P) * L + lane
                            nr = n if (lane < L and n < Rt) else 0
                            rowaddr = base + (q * Rt8 + nr) * 128
                            words = []
                            for cc in range(2):
                                o = rowaddr + (((2 * qq + cc) ^ (nr & 7)) << 4)
                                words += list(smem[o:o + 16].view(np.uint32))
                            v = []
                            for w in words:
                                w = int(w)
                                for s in range(4):
                                    v.append(w & (0x03030303 << (2 * s)) if G == 4 else (w >> (2 * s)) & 0x03030303)
                            A[sp * 32 + lane] = v
                    Ab = A.view(np.uint8).reshape(128, 128).astype(np.int64)          # unsigned A bytes
                    kbase = p["b_off"] + kq * brow * 128
                    for kk in range(QK // 32):
                        Bm = np.zeros((nmma, 32), np.int64)
                        for j in range(nmma):
                            for kb in range(32):
                                logical = kk * 32 + kb
                                o = kbase + (j // 8) * 1024 + (j % 8) * 128 + (((logical >> 4) ^ (j % 8)) << 4) + (logical & 15)
                                Bm[j, kb] = np.int64(np.int8(smem[o]))
                        D += Ab[:, kk * 32:(kk + 1) * 32] @ Bm.T
                    u4 += 1
            # ---- epilogue: column groups and slices into part[n][m]
            for sp in range(4):
                P = 4 // S
                q = sp // P
                for lane in range(32):
                    n = (sp % P) * L + lane
                    if lane < L and n < Rt:
                        d = D[sp * 32 + lane, q * mp * G:(q + 1) * mp * G]
                        for m in range(M):
                            a = int(d[m * G])
                            if G == 4:
                                a += (int(d[m * 4 + 1]) >> 2) + (int(d[m * 4 + 2]) >> 4) + (int(d[m * 4 + 3]) >> 6)
                            part[n, m] += a
            tn = max(0, min(Rt, nrows - tile * Rt))
            for m in range(M):
                for nn in range(tn):
                    acc[m, r0 + tile * Rt + nn] = part[nn, m] - rowsum[m]
            part[:] = 0
    return acc


BUDGET = (232448 - 1024) // 2        # two CTAs per SM on B200 (227 KiB opt-in each block)

CASES = [
    # (M, K, N, SMs): slices S = 4 / 2 / 1, G = 4 and G = 1, several tiles, ragged K and N
    (1, 1024, 40, 8),
    (1, 576, 20, 8),
    (2, 2048, 70, 8),
    (3, 1088, 100, 4),
    (5, 640, 33, 4),
    (16, 512, 24, 4),
    (1, 512, 2000, 4),
    (8, 1024, 9, 8),
    (1, 17 * 512, 65, 1),            # 17 stages through 4 ring slots
    (16, 2048, 300, 4),              # 75 rows per CTA: 4 slices in 3 tiles
    (2, 2048, 600, 4),               # 150 rows per CTA: 4 slices in 5 tiles
]


@pytest.mark.parametrize("M,K,N,sms", CASES)
def test_swap_ab_decode_emulation_matches_the_oracle(M, K, N, sms):
    p = configure(M, K, N, sms, BUDGET)
    assert p is not None
    rng = np.random.default_rng(M * 1000 + K + N)
    W_t = rng.integers(-1, 2, (N, K)).astype(np.int8)
    x_q = rng.integers(-127, 128, (M, K)).astype(np.int8)
    Wbytes = oracle.pack(W_t).view(np.uint8).reshape(N, K // 4)
    np.testing.assert_array_equal(emulate(p, Wbytes, x_q, rng), oracle.ternary_acc(x_q, W_t))


def test_emulated_cases_cover_the_kernel_shapes():
    shapes = [configure(M, K, N, sms, BUDGET) for M, K, N, sms in CASES]
    assert {p["S"] for p in shapes} == {1, 2, 4}
    assert {p["G"] for p in shapes} == {1, 4}
    assert max(p["ntiles"] for p in shapes) > 1
    assert any(p["ntiles"] > 1 and p["S"] > 1 for p in shapes)      # sliced tiles
    assert any(p["slots"] < p["ntiles"] * p["T"] for p in shapes)     # a recycled ring
    assert any(p["nmma"] > p["brow"] for p in shapes)                  # B read past its rows


def test_staging_row_sums_match_the_token_sums():
    rng = np.random.default_rng(3)
    for M, K, S in ((16, 4096, 4), (5, 1088, 2), (1, 640, 1), (9, 2048, 1)):
        mp = pow2(M)
        Lfull = ru(-(-K // S), STAGE_K)
        T = Lfull // STAGE_K
        x_q = rng.integers(-127, 128, (M, K)).astype(np.int8)
        rows = row_rowsum(x_q, M, K, mp, S, T * (STAGE_K // 16), Lfull)
        assert rows == [int(x_q[m].astype(np.int64).sum()) if m < M else 0 for m in range(mp)]


def test_lone_problem_takes_the_whole_sm_when_its_ring_is_short():
    # At two CTAs per SM a problem whose ring cannot hold all of its stages
    # (M = 16, N = 11008: 6 stages of 16 KiB, 2 slots) is laid out for the
    # whole SM instead, where every stage is in flight at once.
    FULL = 232448 - 1024
    half = configure(16, 4096, 11008, 148, BUDGET)
    assert half["slots"] < half["ntiles"] * half["T"]
    full = configure(16, 4096, 11008, 148, FULL)
    assert full["slots"] == full["ntiles"] * full["T"]
    assert full["smem"] + 1024 <= 232448
    # one tile of a 4096-row problem already fits two CTAs per SM
    p = configure(16, 4096, 4096, 148, BUDGET)
    assert p["slots"] == p["ntiles"] * p["T"]
