"""How often the kernels' summation order changes the RMS factor rho.

rho = 1 / sqrt(sum_k h_k^2 / K + 1e-6), rounded once to binary32, with the sum
in binary64 (each h_k^2 of a binary32 h_k is exact there).  The oracle adds in
k order; the kernels add per-thread strided partials, then the warp and block
trees (the one-CTA-per-row form), and for up to 64 rows also the 8 CTA
partials of the row's cluster in rank order.  Both binary64 sums carry a
rounding error of about K 2^-53 relative, so the binary32 rho can differ only
when the exact value lies that close to a binary32 rounding boundary.  This
test replays both kernel orders exactly (numpy float64 adds, elementwise over
many rows) on seeded rows of the decoder block's widths and counts the rows
whose rho differs from the oracle order's."""
import numpy as np

import workloads

THREADS, CLUSTER = 256, 8


def k_order_sum(h):
    s = np.zeros(h.shape[0])
    for k in range(h.shape[1]):
        s = s + h[:, k] * h[:, k]
    return s


def block_sum(part):
    """block_sum_f64 over [rows, 256] thread partials: xor-shuffle trees in
    each warp, lane 0's value per warp, then the same tree over the 8 warp
    sums (lanes 8..31 contribute 0.0); thread 0's value."""
    rows = part.shape[0]
    w = part.reshape(rows, THREADS // 32, 32)
    for off in (16, 8, 4, 2, 1):
        w = w + w[:, :, np.arange(32) ^ off]
    sm = np.zeros((rows, 32))
    sm[:, :THREADS // 32] = w[:, :, 0]
    for off in (16, 8, 4, 2, 1):
        sm = sm + sm[:, np.arange(32) ^ off]
    return sm[:, 0]


def thread_partials(h, g0, g1):
    """Per-thread strided partials over chunks [g0, g1) of 16 elements."""
    rows = h.shape[0]
    part = np.zeros((rows, THREADS))
    for t in range(THREADS):
        for g in range(g0 + t, g1, THREADS):
            for i in range(16):
                v = h[:, 16 * g + i]
                part[:, t] = part[:, t] + v * v
    return part


def one_cta_sum(h):
    return block_sum(thread_partials(h, 0, h.shape[1] // 16))


def cluster_sum(h):
    G = h.shape[1] // 16
    tot = np.zeros(h.shape[0])
    for r in range(CLUSTER):
        tot = tot + block_sum(thread_partials(h, G * r // CLUSTER, G * (r + 1) // CLUSTER))
    return tot


def rho(s, K):
    return (1.0 / np.sqrt(s / K + 1e-6)).astype(np.float32)


def test_kernel_orders_rarely_change_rho():
    rows = 4000
    for K in (2560, 6912):
        h = workloads.activations(K + 7, rows, K, outliers=True).astype(np.float64)
        ref = rho(k_order_sum(h), K)
        for name, s in (("one CTA per row", one_cta_sum(h)), ("cluster of 8", cluster_sum(h))):
            # the sums agree to a few units in the last place of binary64
            rel = np.abs(s - k_order_sum(h)) / k_order_sum(h)
            assert rel.max() < K * 2.0 ** -52, (name, K, rel.max())
            diff = int((rho(s, K) != ref).sum())
            assert diff <= 1, (name, K, diff)
