"""CPU check of the one-token streaming GEMV's plan and index walk.

The one-token kernel gives every CTA (one per SM) a contiguous slab of rows
of every problem, streams each problem's slab through its own ring of chunk
slots (a power-of-two number of rows each) and binds every consumer warp to
one K slice of one problem, with that slice of x_hat in registers.  Its
correctness rests on host-side planning that the GPU parity tests only
sample.  This test restates the plan and the device-side walk in Python and
checks, over a sweep of problem sets:
  * shared memory: header, x_hat areas and rings are disjoint and fit half an
    SM (two CTAs per SM); barrier and slice-sum indices fit their tables;
  * the staging threads cover every 16-element activation chunk exactly once
    and write inside the problem's x_hat area;
  * every bulk copy stays inside its slot and inside W_p;
  * every (row, K slice) of every CTA is computed exactly once, each weight
    read lies inside the bytes its chunk brought in, each x_hat read inside
    the problem's K;
  * a warp's batch of rows never spans more chunks than its ring holds (so
    no warp waits for a slot it still holds), and every chunk but the last of
    a slab collects exactly the arrivals its empty barrier counts;
  * the slice partition reproduces the oracle's integer accumulators.
"""
import numpy as np
import pytest

import oracle
import workloads

NUM_SMS, SMEM_OPTIN = 148, 232448                 # B200
MAX_PROBS, CWARPS, MAX_BARS, PART_MAX = 8, 15, 64, 512
SLICE_UNITS, CHUNK_TARGET, XC = 64, 8192, 2
MAX_SUMK = XC * CWARPS * 32 * 16
# G1Shared: 2 x 64 mbarriers, abort flag, rowsum/beta/fscale[8], red[15][8], part[512]
HDR = ((2 * MAX_BARS * 8 + 4 + 3 * MAX_PROBS * 4 + CWARPS * MAX_PROBS * 4 + PART_MAX * 4 + 7) // 8 * 8 + 127) \
    // 128 * 128


def cost(rows, upl, n):
    best, best_r = 1 << 30, 1
    for R in (4, 2, 1):
        batches = (rows + R - 1) // R
        per_warp = (batches + n - 1) // n * R
        red = 10 if R == 1 else 5 if R == 2 else 3
        c = per_warp * (upl * 33 + 4 + red)
        if c < best:
            best, best_r = c, R
    return best, best_r


def plan(probs):
    """probs: list of (K, N).  Returns the plan dict or None (kernel not used)."""
    if not 1 <= len(probs) <= MAX_PROBS:
        return None
    sumK = sum(K for K, _ in probs)
    if any(K % 64 or K < 64 * 32 for K, _ in probs):
        return None
    pairs = sum((K // 64 + SLICE_UNITS - 1) // SLICE_UNITS for K, _ in probs)
    if sumK > MAX_SUMK or pairs > CWARPS:
        return None
    grid = max(1, min(NUM_SMS, max(N for _, N in probs)))
    budget = min(SMEM_OPTIN, 233472 // 2 - 1024)
    off, part, total = HDR, 0, 0
    P = []
    for K, N in probs:
        q = dict(K=K, N=N, rb=K // 4, xq_off=off)
        off += (K + 127) // 128 * 128
        U = K // 64
        q["nslice"] = (U + SLICE_UNITS - 1) // SLICE_UNITS
        q["slice_w"] = (U + q["nslice"] - 1) // q["nslice"]
        rows_max = (N + grid - 1) // grid
        rpc = 1
        while rpc * 2 * q["rb"] <= CHUNK_TARGET and rpc * 2 <= max(1, rows_max):
            rpc *= 2
        q["rpc"] = rpc
        q["shift"] = rpc.bit_length() - 1
        q["slot"] = rpc * q["rb"]
        if q["nslice"] > 1:
            q["part_off"] = part
            part += rows_max
        q["slab"] = rows_max * q["rb"]
        total += q["slab"]
        P.append(q)
    if part > PART_MAX:
        return None
    ring_budget = budget - off
    if ring_budget <= 0:
        return None
    bars = 0
    for q in P:
        rows_max = (q["N"] + grid - 1) // grid
        nch = (rows_max + q["rpc"] - 1) >> q["shift"]
        share = ring_budget * q["slab"] // max(1, total)
        st = min(share // q["slot"], nch)
        span = min(nch, 4 // q["rpc"] + 1 + (1 if 4 % q["rpc"] else 0))
        if st < span:
            return None
        q["stages"], q["ring_off"], q["bar0"] = st, off, bars
        off += st * q["slot"]
        bars += st
    if bars > MAX_BARS or off > budget:
        return None
    pr = []
    for i, q in enumerate(P):
        U = q["K"] // 64
        for s in range(q["nslice"]):
            width = min(q["slice_w"], U - s * q["slice_w"])
            pr.append(dict(p=i, s=s, rows=(q["N"] + grid - 1) // grid, upl=2 if width > 32 else 1, n=1))
    for _ in range(len(pr), CWARPS):
        worst = max(range(len(pr)), key=lambda k: (cost(pr[k]["rows"], pr[k]["upl"], pr[k]["n"])[0], -k))
        pr[worst]["n"] += 1
    roles = []
    for e in pr:
        R = cost(e["rows"], e["upl"], e["n"])[1]
        for j in range(e["n"]):
            roles.append((e["p"], e["s"], j, e["n"], R))
    assert len(roles) == CWARPS
    return dict(P=P, grid=grid, smem=off, budget=budget, roles=roles, bars=bars)


def rows_of(q, cta, ncta):
    r0 = q["N"] * cta // ncta
    return r0, q["N"] * (cta + 1) // ncta - r0


def check_plan(pl):
    P, grid = pl["P"], pl["grid"]
    assert pl["smem"] <= pl["budget"] and 2 * (pl["smem"] + 1024) <= 233472
    # disjoint, 16-byte aligned areas
    areas = [(0, HDR)] + [(q["xq_off"], q["xq_off"] + q["K"]) for q in P] + \
            [(q["ring_off"], q["ring_off"] + q["stages"] * q["slot"]) for q in P]
    areas.sort()
    for (a0, a1), (b0, b1) in zip(areas, areas[1:]):
        assert a1 <= b0
    for q in P:
        assert q["xq_off"] % 16 == 0 and q["ring_off"] % 16 == 0 and q["slot"] % 16 == 0
        assert q["bar0"] + q["stages"] <= MAX_BARS
    # staging: chunk g of the concatenation -> thread g % 480, cache slot g // 480
    seen = set()
    for ctid in range(CWARPS * 32):
        for i in range(XC):
            gi, p = ctid + i * CWARPS * 32, -1
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
        done = {}
        for w, (p, s, j, n, R) in enumerate(pl["roles"]):
            q = P[p]
            r0, nrows = rows_of(q, cta, grid)
            U = q["K"] // 64
            u0 = s * q["slice_w"]
            width = min(q["slice_w"], U - u0)
            assert width > 0
            upl = 2 if width > 32 else 1
            for lane in range(32):  # x_hat reads
                for u in (u0 + lane, u0 + lane + 32):
                    if u - u0 < width and (u == u0 + lane or upl == 2):
                        assert 64 * u + 64 <= q["K"]
            b = j
            while b * R < nrows:
                i0 = b * R
                nv = min(R, nrows - i0)
                ks = [(i0 + r) >> q["shift"] for r in range(nv)]
                assert max(ks) - min(ks) + 1 <= q["stages"]       # no wait on a slot still held
                for r in range(nv):
                    i = i0 + r
                    k = i >> q["shift"]
                    rows_k = min(q["rpc"], nrows - k * q["rpc"])
                    base = (i & (q["rpc"] - 1)) * q["rb"]
                    hi = base + 16 * (u0 + min(width, 64 if upl == 2 else 32))
                    assert hi <= rows_k * q["rb"] <= q["slot"]
                    if q["nslice"] > 1:
                        assert q["part_off"] + i < PART_MAX
                    assert r0 + i < q["N"]
                    key = (p, i, s)
                    assert key not in done
                    done[key] = w
                b += n
        for p, q in enumerate(P):
            r0, nrows = rows_of(q, cta, grid)
            assert sum(1 for (pp, _, _) in done if pp == p) == nrows * q["nslice"]
            # bulk copies
            nch = (nrows + q["rpc"] - 1) >> q["shift"]
            for k in range(nch):
                rows = min(q["rpc"], nrows - (k << q["shift"]))
                assert rows > 0
                assert (r0 + (k << q["shift"]) + rows) * q["rb"] <= q["N"] * q["rb"]
                assert rows * q["rb"] <= q["slot"]
                if k < nch - 1:   # reused slots: arrivals == count
                    arrivals = sum(1 for (pp, i, _) in done if pp == p and (i >> q["shift"]) == k)
                    assert arrivals == q["rpc"] * q["nslice"]


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
        assert (any(K < 2048 for K, _ in probs) or sum(K for K, _ in probs) > MAX_SUMK
                or sum((K // 64 + 63) // 64 for K, _ in probs) > CWARPS
                or any((N + min(NUM_SMS, max(n for _, n in probs)) - 1) // min(NUM_SMS, max(n for _, n in probs))
                       > PART_MAX for K, N in probs if K > 4096))
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
