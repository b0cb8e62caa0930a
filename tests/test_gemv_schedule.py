"""CPU check of the CUDA-core decode GEMV's launch shaping and work schedule.

The small GEMV kernel (M <= 4) gives every CTA a contiguous slab of rows,
streams it through a shared-memory ring of chunks (a power-of-two number of
rows each) and lets teams of LPR lanes take (R rows x one K slice) items,
iteration by iteration.  Its correctness rests on host-side sizing that the
parity tests only sample.  This test restates the sizing (launch shape, ring
geometry, the reuse adjustments) and the device-side item walk in Python and
checks, over a sweep of shapes, decode and batched (several problems per SM)
budgets, for 2-bit and 1-bit weights:
  * every (row, 16-byte weight group) of every CTA is computed exactly once
    (each row's K slices once, and the slices tile the row);
  * shared memory fits the device, the ring has at most 32 slots of 16-byte
    multiples, K-slice partial sums fit their table;
  * with a recycled ring, the rows of one iteration lie within
    max(1, (stages - 1) * rows-per-chunk) (the sizing rule), which keeps every chunk
    an iteration waits for at most 2 * stages - 1 chunks past the oldest one
    still held -- beyond that an mbarrier parity wait could see the phase of
    the chunk two loads earlier.
"""
import itertools

import pytest

NUM_SMS, SMEM_OPTIN = 148, 232448                 # B200
HDR, MAX_STAGES, CHUNK_TARGET, KS_MAX_ROWS, XQ_MAX = 4096, 32, 8192, 64, 64 * 1024


def small_mt(M):
    return 1 if M <= 1 else 2 if M <= 2 else 4


def ring_geometry(rb, rows_per_cta, ring_bytes):
    cap = max(1, min(rows_per_cta, CHUNK_TARGET // rb))
    shift = 0
    while (2 << shift) <= cap:
        shift += 1
    rpc = 1 << shift
    stride = rpc * rb
    nchunks = (rows_per_cta + rpc - 1) // rpc
    fit = max(1, min(ring_bytes // stride, MAX_STAGES))
    reuse = nchunks > fit
    return dict(rpc=rpc, shift=shift, stride=stride, reuse=reuse, stages=fit if reuse else nchunks)


def configure_small(M, K, N, wbits, co_resident):
    rb = K * wbits // 8
    grid = max(1, min(N, NUM_SMS))
    rows_per_cta = (N + grid - 1) // grid
    K4 = rb // 16
    mt = small_mt(M)
    cw_target = 10
    r = max(1, 2 // mt)
    teams_needed = (rows_per_cta + r - 1) // r
    lpr = 8
    for l in (32, 16, 8):
        if teams_needed * l <= cw_target * 32:
            lpr = l
            break
    ks = 1
    if rows_per_cta <= KS_MAX_ROWS and lpr == 32 and (cw_target * 32 // lpr) * r >= 2 * rows_per_cta:
        ks = 2
    slice4 = (K4 + ks - 1) // ks
    items = (rows_per_cta + r - 1) // r * ks
    cwarps = max(1, min(cw_target, (items * lpr + 31) // 32))
    xq_bytes = (mt * K + 127) // 128 * 128
    budget = (SMEM_OPTIN - 1024) // co_resident
    ring_bytes = max(budget - HDR - xq_bytes, 2 * rb)
    g = ring_geometry(rb, rows_per_cta, ring_bytes)
    if g["reuse"]:
        window = max(1, (g["stages"] - 1) * g["rpc"])
        lpr = 32
        r = min(r, window)
        while r > 1 and (r & (r - 1)):
            r -= 1
        teams_max = max(1, window // r * ks)
        cwarps = max(1, min(cwarps, teams_max))
        if cwarps >= ks:
            cwarps = cwarps // ks * ks
        else:
            while ks % cwarps:
                cwarps -= 1
    return dict(g, rb=rb, K4=K4, grid=grid, lpr=lpr, r=r, ks=ks, slice4=slice4, cwarps=cwarps,
                xq_bytes=xq_bytes, smem=HDR + xq_bytes + g["stages"] * g["stride"])


def cta_rows(N, cta, ncta):
    r0 = N * cta // ncta
    return r0, N * (cta + 1) // ncta - r0


def check_schedule(M, K, N, wbits, co_resident):
    p = configure_small(M, K, N, wbits, co_resident)
    assert p["stride"] % 16 == 0 and 1 <= p["stages"] <= MAX_STAGES
    assert p["smem"] <= SMEM_OPTIN - 1024
    assert p["xq_bytes"] >= small_mt(M) * K
    T = p["cwarps"] * 32 // p["lpr"]                       # teams
    R, KS, K4 = p["r"], p["ks"], p["K4"]
    # the K slices tile the row's 16-byte weight groups exactly once (lanes tl
    # of a team take k_lo + tl, k_lo + tl + LPR, ... < k_hi)
    cover = [0] * K4
    for sl in range(KS):
        for idx in range(sl * p["slice4"], min(K4, sl * p["slice4"] + p["slice4"])):
            cover[idx] += 1
    assert all(c == 1 for c in cover)
    for cta in range(p["grid"]):
        r0, nrows = cta_rows(N, cta, p["grid"])
        if KS > 1:
            assert nrows <= KS_MAX_ROWS
        items = (nrows + R - 1) // R * KS
        iters = (items + T - 1) // T
        done = [[0] * KS for _ in range(nrows)]
        for it in range(iters):
            rows = set()
            for team in range(T):
                item = it * T + team
                if item >= items:
                    continue
                b, sl = (item // KS) * R, item % KS
                for rr in range(max(0, min(R, nrows - b))):
                    rows.add(b + rr)
                    done[b + rr][sl] += 1
            if p["reuse"] and rows:
                lo, hi = min(rows), max(rows)
                assert hi - lo + 1 <= max(1, (p["stages"] - 1) * p["rpc"])
                span = (hi >> p["shift"]) - (lo >> p["shift"]) + 1
                assert span <= 2 * p["stages"] - 1
        assert all(c == 1 for row in done for c in row), (M, K, N, wbits, co_resident, cta)
    return p


NS = [1, 2, 5, 147, 148, 149, 300, 1000, 3000, 4096, 6000, 11008, 20000]
KS_ = [64, 128, 576, 1024, 2560, 4096, 6912, 8192, 11008, 16384, 32768, 65536]


@pytest.mark.parametrize("wbits", [2, 1])
@pytest.mark.parametrize("co_resident", [1, 2, 3, 8])
def test_gemv_schedule_covers_every_row_once(wbits, co_resident):
    seen_reuse = False
    for M, K, N in itertools.product([1, 2, 3, 4], KS_, NS):
        if small_mt(M) * K > XQ_MAX or K % (64 if wbits == 2 else 128):
            continue
        p = check_schedule(M, K, N, wbits, co_resident)
        seen_reuse |= p["reuse"]
    assert seen_reuse                                  # the sweep reaches recycled rings
