"""The 1-bit weight variant on the GPU against the CPU oracle.

unite.ai "Microsofts Inference Framework bringt 1-Bit grosse Sprachmodelle auf
lokale Geraete", "Mathematische Grundlagen", item 1 "Gewichtsbinarisierung",
eq. 1 (W_b = Sign(W - alpha), alpha = mean(W)) with eq. 2 and eq. 3 as for
ternary weights.  alpha, beta, the signs, the packed words, x_q and the int32
accumulators must equal the oracle's bit for bit; float outputs equal the
oracle's binary32 values (same operation order) and lie within 1e-6 of its
binary64 rescale.  The shapes cover the decode GEMV (1-bit words streamed
from HBM, M <= 4) and the tcgen05 GEMM (every other M), ragged N, K at the
128 granularity, several ring slots, the fused quantiser and the full-size
decode and prefill shapes.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import ternary_weight_linear_forward_b200 as bl

pytestmark = pytest.mark.gpu

REL_TOL = 1e-6


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    d = torch.device("cuda:0")
    torch.cuda.set_device(d)
    return d


@pytest.fixture(autouse=True)
def _status_clean(dev):
    yield
    bl.device_status()


def T(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def u32(t):
    return t.cpu().numpy().view(np.uint32)


def gpu_binarize(W, dev):
    W_b, alpha, beta = bl.binarize_weights(T(W, dev))
    return W_b, alpha, beta, bl.pack_bits(W_b)


def check_weights(W, dev):
    W_b, alpha, beta, W_p = gpu_binarize(W, dev)
    oW_b, oalpha, obeta = oracle.binarize_weights(W)
    assert alpha.item() == float(oalpha) and beta.item() == float(obeta)
    np.testing.assert_array_equal(W_b.cpu().numpy(), oW_b)
    np.testing.assert_array_equal(u32(W_p), oracle.pack_bits(oW_b))
    return W_p, beta, oW_b, obeta


def check_y(y, ref, y_dtype):
    if y_dtype == "bf16":
        bits = y.cpu().view(torch.int16).numpy().view(np.uint16)
        lo = oracle.to_bf16((ref["y64"] * (1 - REL_TOL)).astype(np.float32))
        hi = oracle.to_bf16((ref["y64"] * (1 + REL_TOL)).astype(np.float32))
        assert ((bits == lo) | (bits == hi)).all()
    else:
        yv = y.cpu().numpy()
        np.testing.assert_array_equal(yv, ref["y"])
        nz = ref["y64"] != 0
        if nz.any():
            assert (np.abs(yv[nz] - ref["y64"][nz]) / np.abs(ref["y64"][nz])).max() <= REL_TOL


def run_case(dev, M, K, N, seed, y_dtype="f32"):
    W = workloads.latent_weights(seed, N, K)
    x = workloads.activations(seed + 7, M, K, outliers=True)
    W_p, beta, oW_b, obeta = check_weights(W, dev)
    ref = oracle.forward(x, oW_b, obeta)
    x_q, gamma = bl.quant_act(T(x, dev))
    np.testing.assert_array_equal(x_q.cpu().numpy(), ref["x_q"])
    acc = bl.forward_binary_acc(x_q, W_p)
    np.testing.assert_array_equal(acc.cpu().numpy(), ref["acc"])
    od = torch.bfloat16 if y_dtype == "bf16" else torch.float32
    check_y(bl.forward_binary(x_q, gamma, W_p, beta, out_dtype=od), ref, y_dtype)


# --------------------------------------------------------------------------
# weight preparation
# --------------------------------------------------------------------------

@pytest.mark.parametrize("N,K,seed", [(1, 32, 0), (64, 32, 1), (333, 96, 2), (1000, 4096, 3), (4096, 4096, 4),
                                      (11008, 4096, 5)])
def test_binarize_and_pack_bit_exact(dev, N, K, seed):
    W = workloads.latent_weights(seed, N, K) + np.float32(0.001 * (seed - 2))  # nonzero means of both signs
    check_weights(W.astype(np.float32), dev)


def test_binarize_special_matrices(dev):
    # constant: every element equals the mean -> all -1
    W = np.full((8, 64), 0.3, np.float32)
    W_b, alpha, beta, W_p = gpu_binarize(W, dev)
    assert alpha.item() == np.float32(0.3) and beta.item() == np.float32(0.3)
    assert (W_b == -1).all() and not u32(W_p).any()
    # symmetric: mean exactly 0
    half = workloads.latent_weights(77, 32, 128)
    check_weights(np.concatenate([half, -half]), dev)
    # many elements equal to the mean (values a - d, a, a + d balanced): ties -> -1
    a, d = np.float32(0.125), np.float32(0.5)
    vals = np.array([a - d, a, a + d], np.float32)
    W = vals[np.random.default_rng(3).permutation(np.arange(3 * 1024) % 3)].reshape(96, 32)
    W_p, beta, oW_b, _ = check_weights(W, dev)
    assert (oW_b[W == a] == -1).all()
    # zeros and two large elements that cancel in the sum
    W = workloads.latent_weights(5, 64, 64)
    W[0, :8] = 0.0
    W[1, 0] = 30.0
    W[2, 0] = -30.0
    check_weights(W, dev)


@pytest.mark.parametrize("name", ["gaussian_with_tiny_tail", "every_exponent", "subnormal_only", "one_huge",
                                  "small_mass", "above_a_tie"])
def test_binarize_exact_over_the_whole_binary32_range(dev, name):
    # alpha (the signed mean) and beta (the absmean) are the exact means
    # whatever the ratio of an element to the largest; the small elements are
    # given a nonzero signed total
    from test_gpu_parity import _wide_range_matrices
    W = _wide_range_matrices()[name].copy()
    W[W.shape[0] // 2:] = np.abs(W[W.shape[0] // 2:])
    check_weights(W, dev)


def test_pack_bits_of_arbitrary_codes(dev):
    rng = np.random.default_rng(8)
    W_b = rng.integers(-2, 3, (300, 512)).astype(np.int8)   # values <= 0 pack as -1
    np.testing.assert_array_equal(u32(bl.pack_bits(T(W_b, dev))), oracle.pack_bits(W_b))


# --------------------------------------------------------------------------
# forward: GEMV (M <= 4) and GEMM
# --------------------------------------------------------------------------

@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 16, 64, 130])
@pytest.mark.parametrize("K,N", [(128, 5), (1024, 149), (2560, 300), (4096, 1111)])
def test_binary_parity_sweep(dev, M, K, N):
    run_case(dev, M, K, N, seed=M * 17 + K + N)


@pytest.mark.parametrize("K", [128, 256, 640, 1152, 6912, 16384])
def test_binary_m1_k_range(dev, K):
    run_case(dev, 1, K, 333, seed=K + 3)


@pytest.mark.parametrize("N", [1, 2, 147, 148, 149, 296, 5000, 18945])
def test_binary_row_partition(dev, N):
    run_case(dev, 1, 512, N, seed=N)
    run_case(dev, 3, 1024, N, seed=N + 1)


@pytest.mark.parametrize("M,K,N", [(1, 65536, 3000), (4, 16384, 3000), (4, 32768, 200), (2, 32768, 500)])
def test_binary_large_k(dev, M, K, N):
    # K so large that the ring recycles; M * K beyond the GEMV's x_hat stage runs the GEMM
    run_case(dev, M, K, N, seed=K + N + M)


def test_binary_bf16_output(dev):
    run_case(dev, 1, 4096, 2000, 21, y_dtype="bf16")
    run_case(dev, 3, 2560, 700, 22, y_dtype="bf16")
    run_case(dev, 200, 2048, 777, 23, y_dtype="bf16")


def test_binary_extreme_values(dev):
    # |acc| = 127 K on both paths
    K, N = 11008, 64
    W_b = np.ones((N, K), np.int8)
    W_b[1::2] = -1
    W_p = bl.pack_bits(T(W_b, dev))
    for M in (1, 4, 70):
        x_q = torch.full((M, K), 127, dtype=torch.int8, device=dev)
        x_q[:, 1::2] = -127
        acc = bl.forward_binary_acc(x_q, W_p).cpu().numpy()
        np.testing.assert_array_equal(acc, oracle.ternary_acc(x_q.cpu().numpy(), W_b))
        x_q.fill_(-127)
        acc = bl.forward_binary_acc(x_q, W_p).cpu().numpy()
        assert (acc[:, 0] == -127 * K).all() and (acc[:, 1] == 127 * K).all()


@pytest.mark.parametrize("M", [1, 2, 4, 7, 64])
@pytest.mark.parametrize("K,N,x_dtype", [(1024, 300, "bf16"), (4096, 1111, "f32"), (11008, 4096, "bf16")])
def test_binary_fused_quantiser(dev, M, K, N, x_dtype):
    W = workloads.latent_weights(M + K + N, N, K)
    x = workloads.activations(M + K, M, K, outliers=True)
    if x_dtype == "bf16":
        bits = workloads.bf16_bits(x)
        xt = T(bits.view(np.int16), dev).view(torch.bfloat16)
        x = workloads.bf16_to_f32(bits)
    else:
        xt = T(x, dev)
    W_p, beta, oW_b, obeta = check_weights(W, dev)
    y = bl.forward_binary_fp(xt, W_p, beta)
    check_y(y, oracle.forward(x, oW_b, obeta), "f32")
    x_q, gamma = bl.quant_act(xt)
    assert torch.equal(y, bl.forward_binary(x_q, gamma, W_p, beta))


def test_binary_gemm_matches_gemv(dev):
    # rows computed at the dispatch boundary agree: GEMM (M = 130) against GEMV (M <= 4)
    K, N = 4096, 1000
    W_p, beta, _, _ = check_weights(workloads.latent_weights(41, N, K), dev)
    x_q, gamma = bl.quant_act(T(workloads.activations(42, 130, K, outliers=True), dev))
    y = bl.forward_binary(x_q, gamma, W_p, beta).cpu().numpy()
    for lo in (0, 64, 126):
        for m in (1, 2, 4):
            y4 = bl.forward_binary(x_q[lo:lo + m].clone(), gamma[lo:lo + m].clone(), W_p, beta).cpu().numpy()
            np.testing.assert_array_equal(y[lo:lo + m], y4)


# --------------------------------------------------------------------------
# full-size shapes
# --------------------------------------------------------------------------

@pytest.mark.parametrize("shape", workloads.W2.shapes, ids=lambda s: s.name)
def test_binary_workload_decode_m1(dev, shape):
    # the decode shapes with bf16 activations, quantiser fused (one kernel)
    W = shape.weights()
    bits = shape.inputs_bf16_bits()
    x = workloads.bf16_to_f32(bits)
    W_p, beta, oW_b, obeta = check_weights(W, dev)
    y = bl.forward_binary_fp(T(bits.view(np.int16), dev).view(torch.bfloat16), W_p, beta)
    check_y(y, oracle.forward(x, oW_b, obeta), "f32")


@pytest.mark.parametrize("shape", workloads.W4.shapes, ids=lambda s: s.name)
def test_binary_workload_prefill_sampled_rows(dev, shape):
    # M = 2048 on the GEMM; the oracle checks a sample of whole output rows
    W = shape.weights()
    x = shape.inputs()
    W_p, beta, oW_b, obeta = check_weights(W, dev)
    x_q, gamma = bl.quant_act(T(x, dev))
    acc = bl.forward_binary_acc(x_q, W_p).cpu().numpy()
    y = bl.forward_binary(x_q, gamma, W_p, beta, out_dtype=torch.bfloat16)
    rows = np.random.default_rng(shape.M + shape.N + 1).choice(shape.M, 48, replace=False)
    rows[:2] = [0, shape.M - 1]
    ref = oracle.forward(x[rows], oW_b, obeta)
    np.testing.assert_array_equal(acc[rows], ref["acc"])
    check_y(y[torch.from_numpy(rows).to(dev)], ref, "bf16")


def test_binary_kernels_that_run(dev):
    # the 1-bit GEMV streams the packed signs for M <= 4; the GEMM runs otherwise
    from kernel_trace import kernel_names
    W_p, beta, _, _ = check_weights(workloads.latent_weights(3, 2048, 4096), dev)
    for M, name in ((1, "gemv_small_kernel"), (64, "gemm_kernel")):
        x = T(workloads.activations(4, M, 4096), dev)
        names = kernel_names(lambda: bl.forward_binary_fp(x, W_p, beta))
        if not names:
            pytest.skip("profiler reported no kernel records")
        assert any(name in n for n in names), (M, names)
