"""The one-token streaming GEMV (CUDA cores, several projections per launch)
against the CPU oracle and against the general small-M kernel.

For M = 1 the decode calls run a kernel that keeps one CTA per SM at half an
SM, so that the next launch streams its weights while this one computes, and
keeps each warp's K slice of x_hat in registers.  Integers must equal the
oracle's bit for bit and float outputs its binary32 values; the general
CUDA-core kernel (engine 'cuda_cores_general') must give identical outputs.
The shapes cover one and several K slices per row (K = 2048 ... 15360),
rows per CTA from 0 to 271 (N = 1 ... 40000), rings that recycle their slots,
every input mode (fp32, bf16, int8 with gamma), every output mode and batches
of up to eight problems.
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
    # the 'cuda_cores' engine runs one token on the streaming kernel wherever it applies
    with bl.decode_engine("cuda_cores"):
        yield
    bl.device_status()


def T(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def prep(dev, K, N, seed, x_dtype="f32"):
    W = workloads.latent_weights(seed, N, K)
    x = workloads.activations(seed + 1, 1, K, outliers=True)
    if x_dtype == "bf16":
        bits = workloads.bf16_bits(x)
        xt = T(bits.view(np.int16), dev).view(torch.bfloat16)
        x = workloads.bf16_to_f32(bits)
    else:
        xt = T(x, dev)
    W_t, beta = bl.quantize_weights(T(W, dev))
    W_p = bl.pack(W_t)
    oW_t, obeta = oracle.quantize_weights(W)
    return xt, W_p, beta, oracle.forward(x, oW_t, obeta)


def check_f32(y, ref):
    yv = y.cpu().numpy()
    np.testing.assert_array_equal(yv, ref["y"])             # same binary32 op order
    y64 = ref["y64"]
    nz = y64 != 0
    assert np.all(yv[~nz] == 0)
    if nz.any():
        assert (np.abs(yv[nz].astype(np.float64) - y64[nz]) / np.abs(y64[nz])).max() <= REL_TOL


def check_bf16(y, ref):
    np.testing.assert_array_equal(y.cpu().view(torch.int16).numpy().view(np.uint16), oracle.to_bf16(ref["y"]))


SHAPES = [(2048, 1), (2048, 149), (2560, 2560), (2560, 6912), (4096, 11008), (4096, 40000), (4160, 7),
          (6912, 2560), (8192, 18945), (11008, 4096), (12288, 300), (15360, 4096)]


@pytest.mark.parametrize("K,N", SHAPES)
def test_gemv1_all_modes_against_oracle(dev, K, N):
    xt, W_p, beta, ref = prep(dev, K, N, seed=K + N, x_dtype="bf16" if N % 2 else "f32")
    # fused quantiser (fp32 / bf16 x) and quantised input (x_q, gamma)
    check_f32(bl.forward_fp(xt, W_p, beta), ref)
    check_bf16(bl.forward_fp(xt, W_p, beta, out_dtype=torch.bfloat16), ref)
    x_q, gamma = bl.quant_act(xt)
    np.testing.assert_array_equal(x_q.cpu().numpy(), ref["x_q"])
    check_f32(bl.forward(x_q, gamma, W_p, beta), ref)
    np.testing.assert_array_equal(bl.forward_acc(x_q, W_p).cpu().numpy(), ref["acc"])


@pytest.mark.parametrize("K,N", [(2048, 149), (4096, 11008), (11008, 4096), (15360, 4096), (8192, 18945)])
def test_gemv1_equals_general_kernel(dev, K, N):
    xt, W_p, beta, _ = prep(dev, K, N, seed=3 * K + N)
    x_q, gamma = bl.quant_act(xt)

    def outs():
        return [bl.forward_fp(xt, W_p, beta), bl.forward(x_q, gamma, W_p, beta, out_dtype=torch.bfloat16),
                bl.forward_acc(x_q, W_p)]
    a = outs()
    with bl.decode_engine("cuda_cores_general"):
        b = outs()
    for u, v in zip(a, b):
        assert torch.equal(u, v)


@pytest.mark.parametrize("x_dtype,shapes", [
    ("bf16", [(4096, 11008), (11008, 4096)]),
    ("f32", [(2560, 2560)] * 3),
    ("bf16", [(2560, 6912)] * 2),
    ("f32", [(2048, 100)] * 7),
    ("bf16", [(4096, 2000), (2048, 3000), (3072, 148)]),
    ("f32", [(2560, 6912), (2560, 6912), (2560, 2560)]),
])
def test_gemv1_batches(dev, x_dtype, shapes):
    probs, refs = [], []
    for i, (K, N) in enumerate(shapes):
        xt, W_p, beta, ref = prep(dev, K, N, seed=40 * i + K % 101 + N, x_dtype=x_dtype)
        probs.append({"x": xt, "W_p": W_p, "beta": beta})
        refs.append(ref)
    for out, ref in zip(bl.forward_fp_batch(probs), refs):
        check_f32(out, ref)
    for out, ref in zip(bl.forward_fp_batch(probs, out_dtype=torch.bfloat16), refs):
        check_bf16(out, ref)
    # quantised inputs
    qprobs = []
    for pr in probs:
        x_q, gamma = bl.quant_act(pr["x"])
        qprobs.append({"x": x_q, "gamma": gamma, "W_p": pr["W_p"], "beta": pr["beta"]})
    for out, ref in zip(bl.forward_fp_batch(qprobs), refs):
        check_f32(out, ref)


def test_gemv1_back_to_back_launches(dev):
    # consecutive launches overlap (each starts streaming while the previous
    # one computes); outputs of a chain of dependent calls stay exact
    K, N = 4096, 4096
    Ws = [workloads.latent_weights(900 + i, N if i % 2 == 0 else K, K if i % 2 == 0 else N) for i in range(4)]
    x = workloads.activations(950, 1, K, outliers=True)
    layers = []
    for W in Ws:
        W_t, beta = bl.quantize_weights(T(W, dev))
        layers.append((bl.pack(W_t), beta, oracle.quantize_weights(W)))
    h = T(x, dev)
    hs = []
    for W_p, beta, _ in layers:
        h = bl.forward_fp(h, W_p, beta)
        hs.append(h)
    torch.cuda.synchronize()
    hx = x
    for (W_p, beta, (oW_t, obeta)), hg in zip(layers, hs):
        ref = oracle.forward(hx, oW_t, obeta)
        check_f32(hg, ref)
        hx = hg.cpu().numpy()          # the next layer's input is this layer's exact output


def test_gemv1_is_the_kernel_that_runs(dev):
    xt, W_p, beta, _ = prep(dev, 4096, 11008, seed=5)
    from kernel_trace import kernel_names
    names = kernel_names(lambda: bl.forward_fp(xt, W_p, beta))
    if not names:
        pytest.skip("profiler reported no kernel records")
    assert any("gemv1_kernel" in n for n in names), names

