"""CPU checks of the benchmark's per-shape small-batch bounds.

The bound of a call is the larger of the HBM time of its algorithmic bytes
and the compute time of its path's instruction stream at the measured B200
rates (a kind::i8 MMA of 128 x N x 32 per ~186 cycles whatever N; dp4a alone
at 64 lanes per cycle per SM, an even dp4a / LOP3 mix at 85).  These tests
restate the arithmetic for the config-3 shapes."""
import bench
import workloads

SMS, HBM = 148, 6650.0
CLK = bench.NOMINAL_SM_HZ


def test_bound_is_the_larger_of_memory_and_compute():
    for s in workloads.W3.shapes:
        for path in ("cuda_cores", "swap_ab", "gemm"):
            b = bench.small_batch_bound(s.M, s.K, s.N, s.algorithmic_bytes, HBM, SMS, path)
            assert abs(b["hbm_us"] - s.algorithmic_bytes / (HBM * 1e3)) < 1e-9
            assert b["bound_us"] == max(b["hbm_us"], b["compute_us"])
            assert b["bound"] == ("hbm" if b["hbm_us"] >= b["compute_us"] else b["compute"].split()[0])


def test_compute_time_of_each_path():
    M, K, N = 16, 4096, 11008
    nb = 1
    # swap-AB: 128 weight rows x 32 k per MMA
    b = bench.small_batch_bound(M, K, N, nb, HBM, SMS, "swap_ab")
    assert abs(b["compute_us"] - (N * K / 4096) / SMS * 186 / CLK * 1e6) < 1e-9
    # GEMM: 128 tokens x 256 weight rows x 32 k per MMA (tokens padded to 128)
    b = bench.small_batch_bound(M, K, N, nb, HBM, SMS, "gemm")
    assert abs(b["compute_us"] - (1 * 43 * K / 32) / SMS * 186 / CLK * 1e6) < 1e-9
    # CUDA cores at M = 4: 4 M dp4a and 4 LOP3 per 16 trits; the dp4a pipe binds
    b = bench.small_batch_bound(4, K, N, nb, HBM, SMS, "cuda_cores")
    dp4a, lop3 = N * K / 16 * 16, N * K / 16 * 4
    assert abs(b["compute_us"] - max(dp4a / 64, (dp4a + lop3) / 85) / SMS / CLK * 1e6) < 1e-9
    # the swap-AB kernel moves half the weights per MMA of the GEMM's
    g = bench.small_batch_bound(M, K, N, nb, HBM, SMS, "gemm")["compute_us"]
    w = bench.small_batch_bound(M, K, N, nb, HBM, SMS, "swap_ab")["compute_us"]
    assert 1.9 < w / g < 2.1


def test_lead_spin_covers_graph_submission():
    # about a millisecond ahead of the start event, more with more graphs
    assert bench.lead_cycles(1) >= 2_000_000
    assert bench.lead_cycles(8) > bench.lead_cycles(1)
