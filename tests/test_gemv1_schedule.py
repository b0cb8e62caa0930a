"""CPU check of the one-token streaming GEMV's plan and index walk.

The one-token kernel gives every CTA (one per SM) a contiguous slab of rows
of every problem and binds every warp to one K slice of one problem, with
that slice of x_hat in registers; every lane streams its own 16-byte groups
of the warp's rows with cp.async through a per-warp ring of DEPTH slots.
Its correctness rests on host-side planning that the GPU parity tests only
sample.  This test restates the plan and the device-side walk in Python and
checks, over a sweep of problem sets:
  * shared memory: header, x_hat areas and rings are disjoint and fit half an
    SM (two CTAs per SM); slice-sum indices fit their table;
  * the staging threads cover every 16-element activation chunk exactly once
    and write inside the problem's x_hat area;
  * every copy stays inside its ring slot and inside its row of W_p, and
    every read of a slot reads back exactly the bytes the same lane copied
    into it for the same row (the commit-group accounting: DEPTH groups in
    flight, one committed per row consumed);
  * every (row, K slice) of every CTA is computed exactly once, each x_hat
    read lies inside the problem's K;
  * the slice partition reproduces the oracle's integer accumulators.
"""
import numpy as np
import pytest

import oracle
import workloads

NUM_SMS, SMEM_OPTIN = 148, 232448                 # B200
MAX_PROBS, WARPS, DEPTH, SLOT, PART_MAX = 8, 16, 5, 1024, 512
SLICE_UNITS, XC = 64, 2
THREADS = WARPS * 32
MAX_SUMK = XC * THREADS * 16
# G1Shared: rowsum/beta/fscale[8], red[16][8], part[512]
HDR = ((3 * MAX_PROBS * 4 + WARPS * MAX_PROBS * 4 + PART_MAX * 4 + 3) // 4 * 4 + 127) // 128 * 128


def cost(rows, upl, n):
    best, best_r = 1 << 30, 1
    for R in (4, 2, 1):
        if R * upl > 4:
            continue
        batches = (rows + R - 1) // R
        per_warp = (batches + n - 1) // n
        c = per_warp * (300 + R * (upl * 35 + 10))
        if c < best:
            best, best_r = c, R
    return best, best_r


def plan(probs):
    """probs: list of (K, N).  Returns the plan dict or None (kernel not used)."""
    if not 1 <= len(probs) <= MAX_PROBS:
        return None
    if any(K % 64 or K < 64 * 32 for K, _ in probs):
        return None
    sumK = sum(K for K, _ in probs)
    pairs = sum((K // 64 + SLICE_UNITS - 1) // SLICE_UNITS for K, _ in probs)
    if sumK > MAX_SUMK or pairs > WARPS:
        return None
    grid = max(1, min(NUM_SMS, max(N for _, N in probs)))
    budget = min(SMEM_OPTIN, 233472 // 2 - 1024)
    off, part = HDR, 0
    P = []
    for K, N in probs:
        q = dict(K=K, N=N, rb=K // 4, xq_off=off)
        off += (K + 127) // 128 * 128
        U = K // 64
        q["nslice"] = (U + SLICE_UNITS - 1) // SLICE_UNITS
        q["slice_w"] = (U + q["nslice"] - 1) // q["nslice"]
        if q["nslice"] > 1:
            q["part_off"] = part
            part += (N + grid - 1) // grid
        P.append(q)
    if part > PART_MAX:
        return None
    ring_off = off
    off += WARPS * DEPTH * SLOT
    if off > budget:
        return None
    pr = []
    for i, q in enumerate(P):
        U = q["K"] // 64
        for s in range(q["nslice"]):
            width = min(q["slice_w"], U - s * q["slice_w"])
            pr.append(dict(p=i, s=s, rows=(q["N"] + grid - 1) // grid, upl=2 if width > 32 else 1, n=1))
    for _ in range(len(pr), WARPS):
        worst = max(range(len(pr)), key=lambda k: (cost(pr[k]["rows"], pr[k]["upl"], pr[k]["n"])[0], -k))
        pr[worst]["n"] += 1
    roles = []
    for e in pr:
        R = cost(e["rows"], e["upl"], e["n"])[1]
        for j in range(e["n"]):
            roles.append((e["p"], e["s"], j, e["n"], R))
    assert len(roles) == WARPS
    return dict(P=P, grid=grid, smem=off, budget=budget, roles=roles, ring_off=ring_off)


def rows_of(q, cta, ncta):
    r0 = q["N"] * cta // ncta
    return r0, q["N"] * (cta + 1) // ncta - r0


def check_plan(pl):
    P, grid = pl["P"], pl["grid"]
    assert pl["smem"] <= pl["budget"] and 2 * (pl["smem"] + 1024) <= 233472
    areas = [(0, HDR)] + [(q["xq_off"], q["xq_off"] + q["K"]) for q in P] + \
            [(pl["ring_off"], pl["ring_off"] + WARPS * DEPTH * SLOT)]
    areas.sort()
    for (a0, a1), (b0, b1) in zip(areas, areas[1:]):
        assert a1 <= b0
    for q in P:
        assert q["xq_off"] % 16 == 0
    assert pl["ring_off"] % 16 == 0
    # staging: chunk g of the concatenation -> thread g % THREADS, cache slot g // THREADS
    seen = set()
    for tid in range(THREADS):
        for i in range(XC):
            gi, p = tid + i * THREADS, -1
            for j, q in enumerate(P):
                gj = q["K"] >> 4
                if p < 0 and gi < gj:
                    p = j
                if p < 0:
                    gi -= gj
            if p >= 0:
                assert 0 <= gi < P[p]["K"] // 16
                seen.add((p, gi))
    assert len(seen) == sum(q["K"] // 16 for q in P)
    for cta in range(grid):
        done = set()
        for w, (p, s, j, n, R) in enumerate(pl["roles"]):
            q = P[p]
            r0, nrows = rows_of(q, cta, grid)
            U = q["K"] // 64
            u0 = s * q["slice_w"]
            width = min(q["slice_w"], U - u0)
            assert width > 0
            upl = 2 if width > 32 else 1
            assert R * upl <= 4
            ring = pl["ring_off"] + w * DEPTH * SLOT

            def row(t):
                i = (j + (t // R) * n) * R + t % R
                return i if i < nrows else -1

            def groups(lane):
                return [u for u in (u0 + lane, u0 + lane + 32) if u - u0 < width]

            for lane in range(32):
                for u in groups(lane):
                    assert 64 * u + 64 <= q["K"]                       # x_hat read
                    if u == u0 + lane + 32:
                        assert upl == 2
            # commit groups: DEPTH fetches, then one per consumed row; slot
            # contents tracked per lane and byte offset
            slot_row = {}
            committed = []
            for d in range(DEPTH):
                slot_row[d] = row(d)
                committed.append(row(d))
            batches = (nrows + R - 1) // R
            t = 0
            b = j
            while b < batches:
                # wait_group(DEPTH - R): rows t .. t+R-1 have landed
                assert R <= DEPTH
                assert len(committed) - (t + R) <= DEPTH - R
                for r in range(R):
                    slot = (t + r) % DEPTH
                    i = row(t + r)
                    assert slot_row[slot] == i                       # the slot holds row t + r
                    assert (i == b * R + r) if b * R + r < nrows else (i == -1)
                    if i >= 0:
                        for lane in range(32):
                            for u in groups(lane):
                                dst = ring + slot * SLOT + 16 * (u - u0)
                                assert ring <= dst and dst + 16 <= ring + DEPTH * SLOT
                                src = (r0 + i) * q["rb"] + 16 * u
                                assert src + 16 <= (r0 + i + 1) * q["rb"] <= q["N"] * q["rb"]
                        key = (p, i, s)
                        assert key not in done
                        done.add(key)
                        if q["nslice"] > 1:
                            assert q["part_off"] + i < PART_MAX
                        assert r0 + i < q["N"]
                for r in range(R):                                   # refills after the batch
                    slot_row[(t + r) % DEPTH] = row(t + r + DEPTH)
                    committed.append(row(t + r + DEPTH))
                t += R
                b += n
        for p, q in enumerate(P):
            r0, nrows = rows_of(q, cta, grid)
            assert sum(1 for (pp, _, _) in done if pp == p) == nrows * q["nslice"]


DECODE_SETS = {
    "ffn_up_down": [(4096, 11008), (11008, 4096)],
    "up": [(4096, 11008)],
    "down": [(11008, 4096)],
    "qkv": [(2560, 2560)] * 3,
    "o": [(2560, 2560)],
    "gate_up": [(2560, 6912)] * 2,
    "block_down": [(6912, 2560)],
}


@pytest.mark.parametrize("name", sorted(DECODE_SETS))
def test_decode_sets_take_the_one_token_kernel(name):
    pl = plan(DECODE_SETS[name])
    assert pl is not None, name
    check_plan(pl)


SWEEP = [
    [(2048, 1)], [(2048, 5)], [(2048, 147)], [(2048, 149)], [(4096, 300)], [(4096, 40000)],
    [(15360, 4096)], [(15296, 1000)], [(8192, 18945)], [(6144, 148 * 9 + 5)], [(4160, 7)],
    [(2048, 100)] * 7, [(2048, 8)] * 8, [(4096, 2000), (2048, 3000), (3072, 148)],
    [(2560, 6912), (2560, 6912), (2560, 2560)], [(11008, 4096), (4096, 11008)],
    [(12288, 65536)], [(14336, 300), (1024, 10)],
]


@pytest.mark.parametrize("probs", SWEEP, ids=lambda p: "+".join(f"{k}x{n}" for k, n in p))
def test_plan_and_walk_in_bounds(probs):
    pl = plan(probs)
    if pl is None:
        # rejected sets run on the general small-M kernel; only the structural
        # limits may reject
        grid = min(NUM_SMS, max(n for _, n in probs))
        assert (any(K < 2048 or K % 64 for K, _ in probs) or sum(K for K, _ in probs) > MAX_SUMK
                or sum((K // 64 + 63) // 64 for K, _ in probs) > WARPS
                or sum((N + grid - 1) // grid for K, N in probs if K > 4096) > PART_MAX)
        return
    check_plan(pl)


@pytest.mark.parametrize("K,N", [(2048, 37), (11008, 300), (6912, 149)])
def test_slice_partition_reproduces_the_oracle(K, N):
    """Sum over the kernel's K slices (and over the 16-byte groups of each
    lane) of sum c x_hat, minus the row sum of x_hat, equals the oracle's
    accumulator for every row."""
    pl = plan([(K, N)])
    assert pl is not None
    q = pl["P"][0]
    W = workloads.latent_weights(11, N, K)
    x = workloads.activations(12, 1, K, outliers=True)
    W_t, beta = oracle.quantize_weights(W)
    ref = oracle.forward(x, W_t, beta)
    xq = ref["x_q"][0].astype(np.int64)
    codes = W_t.astype(np.int64) + 1
    U = K // 64
    acc = np.zeros(N, dtype=np.int64)
    for s in range(q["nslice"]):
        u0 = s * q["slice_w"]
        width = min(q["slice_w"], U - u0)
        for lane in range(32):
            for u in (u0 + lane, u0 + lane + 32):
                if u - u0 < width and (u == u0 + lane or width > 32):
                    ks = slice(64 * u, 64 * u + 64)
                    acc += codes[:, ks] @ xq[ks]
    acc -= xq.sum()
    assert np.array_equal(acc, ref["acc"][0].astype(np.int64))
