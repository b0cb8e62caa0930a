"""The tensor-core decode engine (tcgen05, M <= 16 tokens) against the CPU
oracle and against the CUDA-core engine.

Integers (x_q, int32 accumulators) must match the oracle bit for bit and the
float outputs must equal the oracle's binary32 values (same op order); the two
engines must agree bit for bit on every output.  The shapes exercise what is
particular to this kernel: K cut into 1, 2 or 4 slices, K not a multiple of
the 512-trit stage, rows split into several TMEM tiles per CTA, a recycled
stage ring, token counts padded to 2, 4, 8 or 16, the quantiser fused in the
prologue, several problems in one launch and the allocation-free entry point.
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


def prep(dev, M, K, N, seed, x_dtype="f32"):
    W = workloads.latent_weights(seed, N, K)
    x = workloads.activations(seed + 7, M, K, outliers=True)
    if x_dtype == "bf16":
        bits = workloads.bf16_bits(x)
        xt = T(bits.view(np.int16), dev).view(torch.bfloat16)
        x = workloads.bf16_to_f32(bits)
    else:
        xt = T(x, dev)
    W_t = bl.quantize_weights(T(W, dev))
    W_p = bl.pack(W_t[0])
    oW_t, obeta = oracle.quantize_weights(W)
    return xt, W_p, W_t[1], oracle.forward(x, oW_t, obeta)


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


def both_engines(fn):
    """fn() -> list of tensors, under each engine; returns the tensor-core results after
    checking they equal the CUDA-core results bit for bit."""
    with bl.decode_engine("cuda_cores"):
        a = [t.clone() for t in fn()]
    with bl.decode_engine("tensor_cores"):
        b = fn()
    for u, v in zip(a, b):
        assert torch.equal(u.view(torch.uint8) if u.dtype == torch.bfloat16 else u,
                           v.view(torch.uint8) if v.dtype == torch.bfloat16 else v)
    return b


def run_quantised(dev, M, K, N, seed, y_dtype="f32"):
    xt, W_p, beta, ref = prep(dev, M, K, N, seed)
    x_q, gamma = bl.quant_act(xt)
    np.testing.assert_array_equal(x_q.cpu().numpy(), ref["x_q"])
    od = torch.bfloat16 if y_dtype == "bf16" else torch.float32
    acc, y = both_engines(lambda: [bl.forward_acc(x_q, W_p), bl.forward(x_q, gamma, W_p, beta, out_dtype=od)])
    np.testing.assert_array_equal(acc.cpu().numpy(), ref["acc"])
    check_y(y, ref, y_dtype)


# K slices: 4 when a CTA holds <= 32 rows, 2 for <= 64, else 1; ragged K
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 11, 16])
@pytest.mark.parametrize("K,N", [(64, 5), (576, 149), (1024, 1024), (2752, 300)])
def test_tc_parity_sweep(dev, M, K, N):
    run_quantised(dev, M, K, N, seed=M * 31 + K + N)


@pytest.mark.parametrize("M", [1, 4, 16])
@pytest.mark.parametrize("K,N", [(4096, 11008), (11008, 4096), (4096, 4096)])
def test_tc_ffn_shapes(dev, M, K, N):
    run_quantised(dev, M, K, N, seed=M * 31 + K + N)


@pytest.mark.parametrize("K", [64, 128, 512, 1088, 2560, 6912, 16384, 16448])
def test_tc_m1_k_range(dev, K):
    run_quantised(dev, 1, K, 333, seed=K + 5)


@pytest.mark.parametrize("N", [1, 2, 147, 148, 149, 296, 5000, 18944, 18945, 40000])
def test_tc_row_partition_and_tiles(dev, N):
    # N > 148 * 128 rows puts several 128-lane tiles in one CTA
    run_quantised(dev, 1, 512, N, seed=N)
    run_quantised(dev, 3, 1024, N, seed=N + 1)


@pytest.mark.parametrize("M,K,N", [(1, 16384, 2000), (4, 8192, 4000), (16, 2048, 600)])
def test_tc_ring_reuse(dev, M, K, N):
    # more stages per CTA than ring slots: slots recycle
    run_quantised(dev, M, K, N, seed=K + N + M)


def test_tc_bf16_output(dev):
    run_quantised(dev, 1, 4096, 2000, 21, y_dtype="bf16")
    run_quantised(dev, 9, 2560, 700, 22, y_dtype="bf16")


def test_tc_extreme_values(dev):
    # |acc| = 127 K, every code at the ends of its range
    K, N = 11008, 64
    x_q = torch.full((1, K), 127, dtype=torch.int8, device=dev)
    x_q[0, 1::2] = -127
    W_t = np.ones((N, K), np.int8)
    W_t[1::2] = -1
    W_t[2] = 0
    W_p = bl.pack(T(W_t, dev))
    with bl.decode_engine("tensor_cores"):
        acc = bl.forward_acc(x_q, W_p).cpu().numpy()
        np.testing.assert_array_equal(acc, oracle.ternary_acc(x_q.cpu().numpy(), W_t))
        x_q.fill_(127)
        acc = bl.forward_acc(x_q, W_p).cpu().numpy()
    assert acc[0, 0] == 127 * K and acc[0, 1] == -127 * K and acc[0, 2] == 0


@pytest.mark.parametrize("M", [1, 2, 4, 7, 16])
@pytest.mark.parametrize("K,N,x_dtype", [(1024, 300, "bf16"), (4096, 1111, "f32"), (11008, 4096, "bf16")])
def test_tc_fused_quantiser(dev, M, K, N, x_dtype):
    xt, W_p, beta, ref = prep(dev, M, K, N, seed=M + K + N, x_dtype=x_dtype)
    (y,) = both_engines(lambda: [bl.forward_fp(xt, W_p, beta)])
    check_y(y, ref, "f32")
    x_q, gamma = bl.quant_act(xt)
    np.testing.assert_array_equal(y.cpu().numpy(), bl.forward(x_q, gamma, W_p, beta).cpu().numpy())


@pytest.mark.parametrize("M,x_dtype,shapes", [
    (1, "bf16", [(4096, 11008), (11008, 4096)]),
    (1, "f32", [(2560, 2560), (2560, 2560), (2560, 2560)]),
    (4, "bf16", [(4096, 1000), (2560, 777)]),
    (3, "f32", [(128, 7), (256, 9), (512, 11), (1024, 13), (2048, 17), (4096, 19), (8192, 23), (16384, 29)]),
])
def test_tc_batch(dev, M, x_dtype, shapes):
    probs, refs = [], []
    for i, (K, N) in enumerate(shapes):
        xt, W_p, beta, ref = prep(dev, M, K, N, seed=900 + 13 * i + M, x_dtype=x_dtype)
        probs.append({"x": xt, "W_p": W_p, "beta": beta})
        refs.append(ref)
    outs = both_engines(lambda: bl.forward_fp_batch(probs))
    for out, ref in zip(outs, refs):
        check_y(out, ref, "f32")
    outs = both_engines(lambda: bl.forward_fp_batch(probs, out_dtype=torch.bfloat16))
    for out, ref in zip(outs, refs):
        check_y(out, ref, "bf16")


def test_tc_noalloc(dev):
    xt, W_p, beta, ref = prep(dev, 2, 4096, 3000, seed=4242)
    x_q, gamma = bl.quant_act(xt)
    with bl.decode_engine("tensor_cores"):
        y1 = bl.forward_noalloc(x_q, gamma, W_p, beta)
        y2 = bl.forward(x_q, gamma, W_p, beta)
    assert torch.equal(y1, y2)
    check_y(y1, ref, "f32")


def test_tc_workload_decode_m1(dev):
    # the bench's decode workload (bf16 activations with outliers), fused quantiser
    for shape in workloads.W2.shapes:
        W = shape.weights()
        bits = shape.inputs_bf16_bits()
        x = workloads.bf16_to_f32(bits)
        W_t, beta = bl.quantize_weights(T(W, dev))
        W_p = bl.pack(W_t)
        oW_t, obeta = oracle.quantize_weights(W)
        ref = oracle.forward(x, oW_t, obeta)
        with bl.decode_engine("tensor_cores"):
            y = bl.forward_fp(T(bits.view(np.int16), dev).view(torch.bfloat16), W_p, beta)
        check_y(y, ref, "f32")


def test_tc_engine_is_the_one_that_runs(dev):
    # the tensor-core kernel is what runs for a supported shape (kernel names from the profiler)
    xt, W_p, beta, _ = prep(dev, 1, 4096, 2048, seed=3)
    from kernel_trace import kernel_names
    for engine, name in (("tensor_cores", "decode_tc_kernel"), ("cuda_cores", "gemv1_kernel"),
                         ("cuda_cores_general", "gemv_small_kernel")):
        with bl.decode_engine(engine):
            names = kernel_names(lambda: bl.forward_fp(xt, W_p, beta))
        if not names:
            pytest.skip("profiler reported no kernel records")
        assert any(name in n for n in names), (engine, names)


@pytest.mark.parametrize("M,N", [(1, 4096), (4, 11008), (8, 11008), (16, 4096), (16, 11008), (64, 4096)])
def test_forward_path_names_the_kernel_that_runs(dev, M, N):
    # the library's path query (used by the bench for its labels and bounds)
    # names the kernel family the forward launches, under the automatic engine
    from kernel_trace import kernel_names
    K = 4096
    with bl.decode_engine("auto"):
        path = bl.forward_path(M, N, K)
        W_p = torch.randint(-2**31, 2**31 - 1, (N, K // 16), dtype=torch.int32, device=dev)
        beta = torch.tensor([0.02], device=dev)
        x = torch.randn((M, K), device=dev)
        names = kernel_names(lambda: bl.forward_fp(x, W_p, beta))
    if not names:
        pytest.skip("profiler reported no kernel records")
    want = {"cuda_cores": "gemv_small_kernel", "swap_ab": "decode_tc_kernel", "gemm": "gemm_kernel"}[path]
    assert any(want in n for n in names), (M, N, path, names)
    if M == 16 and N == 11008:
        assert path == "gemm"
    if M == 16 and N == 4096:
        assert path == "swap_ab"
