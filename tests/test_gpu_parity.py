"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Integers (ternary codes, packed words, int8 activations, int32 accumulators)
must match bit for bit; the absmean scale beta and the per-token gamma too
(both are binary32 values that decide integer codes, computed in the same
precision on both sides).  Float outputs must lie within 1e-6 relative error
of the oracle's binary64 rescale; bf16 outputs must be one of the bf16
roundings of a value within that tolerance.
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


def gpu_prep(W, dev):
    W_t, beta = bl.quantize_weights(T(W, dev))
    return W_t, beta, bl.pack(W_t)


def assert_f32_close(y_gpu, y64):
    y = y_gpu.astype(np.float64)
    nz = y64 != 0
    assert np.all(y[~nz] == 0)
    if nz.any():
        rel = np.abs(y[nz] - y64[nz]) / np.abs(y64[nz])
        assert rel.max() <= REL_TOL, f"max rel err {rel.max():.3g}"


def assert_bf16_ok(y_bits, y64):
    lo = oracle.to_bf16((y64 * (1 - REL_TOL)).astype(np.float32))
    hi = oracle.to_bf16((y64 * (1 + REL_TOL)).astype(np.float32))
    ok = (y_bits == lo) | (y_bits == hi)
    assert ok.all(), f"{(~ok).sum()} bf16 outputs outside tolerance"


# --------------------------------------------------------------------------
# weight preparation
# --------------------------------------------------------------------------

@pytest.mark.parametrize("N,K,seed", [(1, 16, 0), (7, 48, 1), (300, 1024, 2), (1024, 1024, 3),
                                      (149, 4096, 4), (4096, 11008, 1002), (11008, 4096, 1012)])
def test_quantize_and_pack_bit_exact(dev, N, K, seed):
    W = workloads.latent_weights(seed, N, K)
    W_t, beta, W_p = gpu_prep(W, dev)
    oW_t, obeta = oracle.quantize_weights(W)
    assert beta.item() == float(obeta)
    np.testing.assert_array_equal(W_t.cpu().numpy(), oW_t)
    np.testing.assert_array_equal(W_p.cpu().numpy().view(np.uint32), oracle.pack(oW_t))


def test_quantize_special_matrices(dev):
    z = np.zeros((8, 32), np.float32)
    W_t, beta, W_p = gpu_prep(z, dev)
    assert beta.item() == 0.0 and not W_t.any()
    assert np.all(W_p.cpu().numpy().view(np.uint32) == 0x55555555)
    # mean |W| = 1 exactly and eps = 0: q = W, so +-0.5 ties go to 0, +-1.5 clips to +-1
    W = np.array([[0.5, -0.5, 1.5, -1.5] * 4] * 3, np.float32)
    W_t, beta = bl.quantize_weights(T(W, dev), eps=0.0)
    assert beta.item() == 1.0
    np.testing.assert_array_equal(W_t.cpu().numpy(), oracle.ternarize(W, 1.0, 0.0))
    np.testing.assert_array_equal(W_t.cpu().numpy()[0, :4], [0, 0, 1, -1])
    # wide dynamic range
    g = np.random.default_rng(5)
    W = (g.standard_normal((64, 256)) * np.exp(g.uniform(-20, 20, (64, 256)))).astype(np.float32)
    W_t, beta, _ = gpu_prep(W, dev)
    oW_t, obeta = oracle.quantize_weights(W)
    assert beta.item() == float(obeta)
    np.testing.assert_array_equal(W_t.cpu().numpy(), oW_t)


def _wide_range_matrices():
    """Matrices whose |W| spans the whole binary32 range: the mean must be
    the exact one whatever the ratio of an element to the largest."""
    g = np.random.default_rng(55)
    base = g.standard_normal((96, 512)).astype(np.float32)
    out = {}
    W = base * np.float32(0.02)
    W[0, :200] = g.standard_normal(200) * 2.0 ** -45 * 0.02      # 2^-45 .. 2^-60 of the max
    W[1, :200] = g.standard_normal(200) * 2.0 ** -60 * 0.02
    W[2, :64] = g.standard_normal(64) * 1e-42                      # subnormals
    W[3, :8] = [1e-45, -1e-45, 2e-45, 3e-44, -7e-40, 1.1754942e-38, -1.1754944e-38, 5.877472e-39]
    out["gaussian_with_tiny_tail"] = W.astype(np.float32)
    out["every_exponent"] = (base * np.exp2(g.integers(-149, 120, base.shape))).astype(np.float32)
    out["subnormal_only"] = (base * 1e-41).astype(np.float32)
    W = np.zeros((64, 128), np.float32)
    W[5, 7] = 3.0e38                                               # one huge element, the rest tiny
    W[6, :] = g.standard_normal(128) * 1e-40
    out["one_huge"] = W
    # many small elements whose total reaches the big ones' scale: a sum
    # that truncation below 2^-38 of the max would change
    W = np.full((128, 1024), np.float32(2.0 ** -40) * np.float32(1.0000001), np.float32)
    W[0, 0] = 1.0
    out["small_mass"] = W
    # a mean one tiny step above a binary32 tie: 2^16, 2^-9 and 16384 copies
    # of 2^-23 (1 + 2^-23) among 65536 elements sum to 2^16 + 2^-8 + 2^-32, so
    # the mean is 1 + 2^-24 + 2^-48 and rounds up to 1 + 2^-23; dropping the
    # copies' lowest bit (anything coarser than exact) leaves the tie 1 + 2^-24,
    # which rounds to even, 1
    W = np.zeros((64, 1024), np.float32)
    W.flat[0] = 2.0 ** 16
    W.flat[1] = 2.0 ** -9
    W.flat[2:2 + 16384] = np.float32(2.0 ** -23) * np.float32(1.0000001)
    out["above_a_tie"] = W
    return out


@pytest.mark.parametrize("name", sorted(_wide_range_matrices()))
def test_quantize_exact_over_the_whole_binary32_range(dev, name):
    W = _wide_range_matrices()[name]
    W_t, beta, W_p = gpu_prep(W, dev)
    oW_t, obeta = oracle.quantize_weights(W)
    assert beta.item() == float(obeta), (beta.item(), float(obeta))
    np.testing.assert_array_equal(W_t.cpu().numpy(), oW_t)
    np.testing.assert_array_equal(W_p.cpu().numpy().view(np.uint32), oracle.pack(oW_t))


def test_pack_of_arbitrary_trits(dev):
    g = np.random.default_rng(6)
    W_t = g.integers(-1, 2, size=(333, 16 * 37)).astype(np.int8)
    W_p = bl.pack(T(W_t, dev))
    np.testing.assert_array_equal(W_p.cpu().numpy().view(np.uint32), oracle.pack(W_t))


# --------------------------------------------------------------------------
# activation quantiser
# --------------------------------------------------------------------------

@pytest.mark.parametrize("M,K,dtype", [(1, 16, "f32"), (1, 4096, "bf16"), (1, 11008, "bf16"), (5, 1024, "f32"),
                                       (64, 4096, "f32"), (2048, 4096, "f32"), (3, 2560, "bf16")])
def test_quant_act_bit_exact(dev, M, K, dtype):
    x = workloads.activations(100 + M, M, K, outliers=True)
    if dtype == "bf16":
        bits = workloads.bf16_bits(x)
        xt = T(bits.view(np.int16), dev).view(torch.bfloat16)
        x = workloads.bf16_to_f32(bits)
    else:
        xt = T(x, dev)
    x_q, gamma = bl.quant_act(xt)
    ox_q, og = oracle.quant_act(x)
    np.testing.assert_array_equal(x_q.cpu().numpy(), ox_q)
    np.testing.assert_array_equal(gamma.cpu().numpy(), og)


def test_quant_act_edge_rows(dev):
    x = np.zeros((4, 64), np.float32)
    x[1, 5] = 3e-6                       # below the gamma floor
    x[2, :4] = [1, -2, 0.5, 4]           # the hand-worked token: -63.5 -> -64
    x[3, :4] = [127, 62.5, -0.5, 1.5]    # ties to even: 62, 0, 2
    x_q, gamma = bl.quant_act(T(x, dev))
    ox_q, og = oracle.quant_act(x)
    np.testing.assert_array_equal(x_q.cpu().numpy(), ox_q)
    np.testing.assert_array_equal(gamma.cpu().numpy(), og)
    np.testing.assert_array_equal(x_q.cpu().numpy()[3, :4], [127, 62, 0, 2])


# --------------------------------------------------------------------------
# forward: accumulators bit-exact, outputs within tolerance
# --------------------------------------------------------------------------

def run_case(dev, M, K, N, seed, x_dtype="f32", y_dtype="f32", outliers=False):
    W = workloads.latent_weights(seed, N, K)
    x = workloads.activations(seed + 7, M, K, outliers)
    if x_dtype == "bf16":
        bits = workloads.bf16_bits(x)
        xt = T(bits.view(np.int16), dev).view(torch.bfloat16)
        x = workloads.bf16_to_f32(bits)
    else:
        xt = T(x, dev)
    W_t, beta, W_p = gpu_prep(W, dev)
    oW_t, obeta = oracle.quantize_weights(W)
    x_q, gamma = bl.quant_act(xt)
    acc = bl.forward_acc(x_q, W_p)
    y = bl.forward(x_q, gamma, W_p, beta, out_dtype=torch.bfloat16 if y_dtype == "bf16" else torch.float32)
    ref = oracle.forward(x, oW_t, obeta)
    np.testing.assert_array_equal(acc.cpu().numpy(), ref["acc"])
    if y_dtype == "bf16":
        assert_bf16_ok(y.cpu().view(torch.int16).numpy().view(np.uint16), ref["y64"])
    else:
        yv = y.cpu().numpy()
        assert_f32_close(yv, ref["y64"])
        np.testing.assert_array_equal(yv, ref["y"])      # same binary32 op order: identical
    return ref


@pytest.mark.parametrize("engine", ["cuda_cores", "tensor_cores", "cuda_cores_general"])
@pytest.mark.parametrize("M", [1, 2, 3, 4, 7, 16, 33, 64])
@pytest.mark.parametrize("K,N", [(64, 5), (1024, 148), (1024, 149), (2560, 1000), (6912, 300)])
def test_gemv_parity_sweep(dev, M, K, N, engine):
    # shapes the tensor-core engine does not take run on CUDA cores
    with bl.decode_engine(engine):
        run_case(dev, M, K, N, seed=10 * M + K % 97 + N)


@pytest.mark.parametrize("K", [64, 128, 1024, 1088, 2048, 2560, 4096, 6912, 11008, 16384, 16448, 32768])
def test_gemv_m1_all_team_shapes(dev, K):
    run_case(dev, 1, K, 333, seed=K)


@pytest.mark.parametrize("N", [1, 2, 147, 148, 149, 296, 5000])
def test_gemv_row_partition_tails(dev, N):
    run_case(dev, 1, 4096, N, seed=N)
    run_case(dev, 5, 1024, N, seed=N + 1)


@pytest.mark.parametrize("M,K,N", [(1, 32768, 5000), (3, 16384, 9000), (2, 65536, 700)])
def test_gemv_ring_reuse(dev, M, K, N):
    # slabs larger than the shared-memory ring: chunks recycle ring slots
    run_case(dev, M, K, N, seed=K + N)


def test_gemv_bf16_output(dev):
    run_case(dev, 1, 4096, 2000, 21, y_dtype="bf16")
    run_case(dev, 9, 2560, 700, 22, y_dtype="bf16")


def test_gemv_extreme_values(dev):
    # every activation at +-127 and every weight +1: |acc| = 127 K at the int32 bound of the kernel
    K, N = 11008, 64
    x_q = torch.full((1, K), 127, dtype=torch.int8, device=dev)
    x_q[0, 1::2] = -127
    W_t = np.ones((N, K), np.int8)
    W_t[1::2] = -1
    W_t[2] = 0
    W_p = bl.pack(T(W_t, dev))
    acc = bl.forward_acc(x_q, W_p).cpu().numpy()
    np.testing.assert_array_equal(acc, oracle.ternary_acc(x_q.cpu().numpy(), W_t))
    x_q.fill_(127)
    acc = bl.forward_acc(x_q, W_p).cpu().numpy()
    assert acc[0, 0] == 127 * K and acc[0, 1] == -127 * K and acc[0, 2] == 0


# --------------------------------------------------------------------------
# the workloads at full size
# --------------------------------------------------------------------------

def test_workload_single_layer_m1_k1024(dev):
    s = workloads.W1.shapes[0]
    run_case(dev, s.M, s.K, s.N, s.w_seed)


@pytest.mark.parametrize("shape", workloads.W2.shapes, ids=lambda s: s.name)
def test_workload_decode_m1_bf16(dev, shape):
    # the bench's workload, same weights, activations and launch path
    W = shape.weights()
    bits = shape.inputs_bf16_bits()
    x = workloads.bf16_to_f32(bits)
    W_t, beta, W_p = gpu_prep(W, dev)
    oW_t, obeta = oracle.quantize_weights(W)
    x_q, gamma = bl.quant_act(T(bits.view(np.int16), dev).view(torch.bfloat16))
    y = bl.forward(x_q, gamma, W_p, beta)
    ref = oracle.forward(x, oW_t, obeta)
    np.testing.assert_array_equal(x_q.cpu().numpy(), ref["x_q"])
    np.testing.assert_array_equal(bl.forward_acc(x_q, W_p).cpu().numpy(), ref["acc"])
    assert_f32_close(y.cpu().numpy(), ref["y64"])
    zero_frac = float((W_t == 0).float().mean())
    assert abs(zero_frac - 0.3101) < 2e-3


@pytest.mark.parametrize("shape", workloads.W3.shapes, ids=lambda s: s.name)
def test_workload_small_batch(dev, shape):
    run_case(dev, shape.M, shape.K, shape.N, shape.w_seed)


# --------------------------------------------------------------------------
# fused quantise + forward: bit-identical to quant_act followed by forward
# --------------------------------------------------------------------------

@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 17])
@pytest.mark.parametrize("K,N,x_dtype", [(1024, 300, "bf16"), (4096, 1111, "f32"), (16384, 150, "bf16"),
                                         (6912, 149, "f32")])
def test_forward_fp_matches_two_calls_and_oracle(dev, M, K, N, x_dtype):
    W = workloads.latent_weights(M + K + N, N, K)
    x = workloads.activations(M * 3 + K, M, K, outliers=True)
    if x_dtype == "bf16":
        bits = workloads.bf16_bits(x)
        xt = T(bits.view(np.int16), dev).view(torch.bfloat16)
        x = workloads.bf16_to_f32(bits)
    else:
        xt = T(x, dev)
    W_t, beta, W_p = gpu_prep(W, dev)
    y_fused = bl.forward_fp(xt, W_p, beta)
    x_q, gamma = bl.quant_act(xt)
    y_two = bl.forward(x_q, gamma, W_p, beta)
    np.testing.assert_array_equal(y_fused.cpu().numpy(), y_two.cpu().numpy())
    oW_t, obeta = oracle.quantize_weights(W)
    ref = oracle.forward(x, oW_t, obeta)
    assert_f32_close(y_fused.cpu().numpy(), ref["y64"])
    yb = bl.forward_fp(xt, W_p, beta, out_dtype=torch.bfloat16)
    assert_bf16_ok(yb.cpu().view(torch.int16).numpy().view(np.uint16), ref["y64"])


def test_forward_fp_zero_and_tiny_tokens(dev):
    K, N = 1024, 64
    W = workloads.latent_weights(3, N, K)
    x = np.zeros((3, K), np.float32)
    x[1, 7] = 2e-6                                  # gamma floor
    x[2] = workloads.activations(4, 1, K)[0]
    W_t, beta, W_p = gpu_prep(W, dev)
    y = bl.forward_fp(T(x, dev), W_p, beta).cpu().numpy()
    oW_t, obeta = oracle.quantize_weights(W)
    ref = oracle.forward(x, oW_t, obeta)
    assert np.all(y[0] == 0)
    assert_f32_close(y, ref["y64"])


# --------------------------------------------------------------------------
# prefill GEMM (M > 64, tcgen05): accumulators bit-exact, tails in M, N, K
# --------------------------------------------------------------------------

@pytest.mark.parametrize("M,K,N", [(128, 128, 256), (65, 64, 5), (200, 1088, 300), (129, 4096, 257),
                                   (511, 1024, 512), (512, 2048, 256), (513, 640, 1000), (300, 6912, 64),
                                   (2047, 256, 130), (2049, 512, 260)])
def test_gemm_parity_tails(dev, M, K, N):
    run_case(dev, M, K, N, seed=M + 3 * K + N)


@pytest.mark.parametrize("y_dtype", ["f32", "bf16"])
def test_gemm_output_dtypes(dev, y_dtype):
    run_case(dev, 300, 2048, 777, 31, y_dtype=y_dtype, outliers=True)


def test_gemm_matches_gemv_on_same_inputs(dev):
    # the dispatch boundary: rows computed by the GEMM equal those of the GEMV
    K, N = 4096, 1000
    W = workloads.latent_weights(41, N, K)
    x = workloads.activations(42, 130, K, outliers=True)
    W_t, beta, W_p = gpu_prep(W, dev)
    x_q, gamma = bl.quant_act(T(x, dev))
    y_gemm = bl.forward(x_q, gamma, W_p, beta).cpu().numpy()
    for lo in (0, 64, 66):
        # slices are cloned: the ABI requires 16-byte aligned pointers
        for m, engine in ((64, "cuda_cores"), (64, "auto"), (4, "auto"), (16, "tensor_cores")):
            with bl.decode_engine(engine):
                y_gemv = bl.forward(x_q[lo:lo + m].clone(), gamma[lo:lo + m].clone(), W_p, beta).cpu().numpy()
            np.testing.assert_array_equal(y_gemm[lo:lo + m], y_gemv)


def _sampled_rows_check(dev, shape, n_rows=48):
    W = shape.weights()
    x = shape.inputs()
    W_t, beta, W_p = gpu_prep(W, dev)
    x_q, gamma = bl.quant_act(T(x, dev))
    acc = bl.forward_acc(x_q, W_p).cpu().numpy()
    y = bl.forward(x_q, gamma, W_p, beta, out_dtype=torch.bfloat16).cpu().view(torch.int16).numpy().view(np.uint16)
    oW_t, obeta = oracle.quantize_weights(W)
    assert beta.item() == float(obeta)
    rows = np.random.default_rng(shape.M + shape.N).choice(shape.M, n_rows, replace=False)
    rows[:2] = [0, shape.M - 1]
    ref = oracle.forward(x[rows], oW_t, obeta)     # per-token quantiser: a row subset is exact
    np.testing.assert_array_equal(x_q.cpu().numpy()[rows], ref["x_q"])
    np.testing.assert_array_equal(acc[rows], ref["acc"])
    assert_bf16_ok(y[rows], ref["y64"])


@pytest.mark.parametrize("M,K,N", [(1024, 512, 11008), (700, 1024, 18000)])
def test_gemm_multi_wave_full_output(dev, M, K, N):
    # more 128 x 256 tiles than SMs (344 and 216): every CTA walks several
    # tiles, alternating its two TMEM accumulators; every output is compared
    run_case(dev, M, K, N, seed=M + K + N, y_dtype="bf16", outliers=True)
    run_case(dev, M, K, N, seed=M + K + N + 1)


@pytest.mark.parametrize("shape", workloads.W4.shapes, ids=lambda s: s.name)
def test_workload_prefill_full_output(dev, shape):
    # full-size prefill (M = 2048) in the launch configuration the benchmark
    # times, every output against the oracle (its all-core build of the
    # integer contraction)
    W = shape.weights()
    x = shape.inputs()
    W_t, beta, W_p = gpu_prep(W, dev)
    x_q, gamma = bl.quant_act(T(x, dev))
    acc = bl.forward_acc(x_q, W_p).cpu().numpy()
    y = bl.forward(x_q, gamma, W_p, beta, out_dtype=torch.bfloat16).cpu().view(torch.int16).numpy().view(np.uint16)
    oW_t, obeta = oracle.quantize_weights(W)
    assert beta.item() == float(obeta)
    ox_q, ogamma = oracle.quant_act(x)
    np.testing.assert_array_equal(x_q.cpu().numpy(), ox_q)
    np.testing.assert_array_equal(gamma.cpu().numpy(), ogamma)
    oacc = oracle.ternary_acc_all_cores(ox_q, oW_t)
    np.testing.assert_array_equal(acc, oacc)
    assert_bf16_ok(y, oracle.rescale_f64(oacc, obeta, ogamma))
    np.testing.assert_array_equal(y, oracle.to_bf16(oracle.rescale_f32(oacc, obeta, ogamma)))


@pytest.mark.parametrize("shape", workloads.W4.shapes, ids=lambda s: s.name)
def test_workload_prefill_sampled_rows(dev, shape):
    # full-size prefill (M = 2048) in the launch configuration the benchmark
    # times; the oracle checks a sample of whole output rows
    _sampled_rows_check(dev, shape)


# --------------------------------------------------------------------------
# batched independent projections in one launch
# --------------------------------------------------------------------------

def _prep_batch(dev, shapes, M, x_dtype, seed):
    probs, refs = [], []
    for i, (K, N) in enumerate(shapes):
        W = workloads.latent_weights(seed + i, N, K)
        x = workloads.activations(seed + 50 + i, M, K, outliers=True)
        if x_dtype == "bf16":
            bits = workloads.bf16_bits(x)
            xt = T(bits.view(np.int16), dev).view(torch.bfloat16)
            x = workloads.bf16_to_f32(bits)
        else:
            xt = T(x, dev)
        W_t, beta, W_p = gpu_prep(W, dev)
        probs.append({"x": xt, "W_p": W_p, "beta": beta})
        oW_t, obeta = oracle.quantize_weights(W)
        refs.append(oracle.forward(x, oW_t, obeta))
    return probs, refs


@pytest.mark.parametrize("M,x_dtype,shapes", [
    (1, "bf16", [(4096, 11008), (11008, 4096)]),
    (1, "f32", [(2560, 2560), (2560, 2560), (2560, 2560)]),
    (2, "f32", [(1024, 300), (6912, 149), (64, 5)]),
    (4, "bf16", [(4096, 1000), (2560, 777)]),
    (1, "f32", [(1024, 1024)]),
    (3, "f32", [(128, 7), (256, 9), (512, 11), (1024, 13), (2048, 17), (4096, 19), (8192, 23), (16384, 29)]),
])
def test_forward_fp_batch_matches_single_calls(dev, M, x_dtype, shapes):
    probs, refs = _prep_batch(dev, shapes, M, x_dtype, seed=M * 100 + len(shapes))
    outs = bl.forward_fp_batch(probs)
    for pr, out, ref in zip(probs, outs, refs):
        single = bl.forward_fp(pr["x"], pr["W_p"], pr["beta"])
        np.testing.assert_array_equal(out.cpu().numpy(), single.cpu().numpy())
        assert_f32_close(out.cpu().numpy(), ref["y64"])
    # bf16 outputs
    outs = bl.forward_fp_batch(probs, out_dtype=torch.bfloat16)
    for out, ref in zip(outs, refs):
        assert_bf16_ok(out.cpu().view(torch.int16).numpy().view(np.uint16), ref["y64"])


def test_forward_fp_batch_quantised_inputs(dev):
    # q / k / v style: one x_q shared by three projections
    K = 2560
    x = workloads.activations(77, 1, K)
    x_q, gamma = bl.quant_act(T(x, dev))
    probs = []
    for i, N in enumerate((2560, 2560, 1280)):
        W_t, beta, W_p = gpu_prep(workloads.latent_weights(80 + i, N, K), dev)
        probs.append({"x": x_q, "gamma": gamma, "W_p": W_p, "beta": beta})
    outs = bl.forward_fp_batch(probs)
    for pr, out in zip(probs, outs):
        np.testing.assert_array_equal(out.cpu().numpy(), bl.forward(x_q, gamma, pr["W_p"], pr["beta"]).cpu().numpy())


def test_batch_plan_matches_call(dev):
    # the marshal-once plan runs the same launch as forward_fp_batch, call after call
    probs, refs = _prep_batch(dev, [(4096, 1000), (2560, 777)], 1, "bf16", seed=7)
    outs = bl.forward_fp_batch(probs)
    plan = bl.BatchPlan([dict(pr, out=torch.empty_like(o)) for pr, o in zip(probs, outs)])
    for _ in range(2):
        got = plan.run()
        for a, b, ref in zip(outs, got, refs):
            assert torch.equal(a, b)
            assert_f32_close(b.cpu().numpy(), ref["y64"])
