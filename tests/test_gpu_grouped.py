"""Group quantisation along K against the CPU oracle.

unite.ai "Microsofts Inference Framework bringt 1-Bit grosse Sprachmodelle auf
lokale Geraete", section "Gruppenquantisierung und -normalisierung": weights
and activations divided into G groups with their own parameters (here G
contiguous blocks of K; beta_g per weight group, gamma_{m,g} per token and
group; per-group binary32 terms added in increasing g).  Codes, scales and
int32 accumulators must equal the oracle's bit for bit; y equals the
oracle's binary32 value and lies within 1e-6 * sum_g |term_g| of its binary64
sum (a bf16 y is the oracle's binary32 y rounded to nearest-even).
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


def prep(dev, N, K, G, seed):
    W = workloads.latent_weights(seed, N, K)
    W_t, beta = bl.quantize_weights_grouped(T(W, dev), G)
    oW_t, obeta = oracle.quantize_weights_grouped(W, G)
    np.testing.assert_array_equal(beta.cpu().numpy(), obeta)
    np.testing.assert_array_equal(W_t.cpu().numpy(), oracle.group_major(oW_t, G))
    W_p = bl.pack_grouped(W_t)
    np.testing.assert_array_equal(W_p.cpu().numpy().view(np.uint32),
                                  np.stack([oracle.pack(oracle.group_major(oW_t, G)[g]) for g in range(G)]))
    return W_p, beta, oW_t, obeta


def check_y(y, ref, y_dtype):
    # Terms of different groups can cancel, so the binary32 result is bounded
    # relative to the sum of the terms' magnitudes: each term carries three
    # roundings and each of the G - 1 adds one, (G + 2) 2^-24 < 1e-6 for G <= 8.
    if y_dtype == "bf16":
        bits = y.cpu().view(torch.int16).numpy().view(np.uint16)
        np.testing.assert_array_equal(bits, oracle.to_bf16(ref["y"]))
    else:
        yv = y.cpu().numpy()
        np.testing.assert_array_equal(yv, ref["y"])
        assert (np.abs(yv - ref["y64"]) <= REL_TOL * ref["yabs64"]).all()


def run_case(dev, M, K, N, G, seed, y_dtype="f32", x_dtype="f32"):
    W_p, beta, oW_t, obeta = prep(dev, N, K, G, seed)
    x = workloads.activations(seed + 3, M, K, outliers=True)
    if x_dtype == "bf16":
        bits = workloads.bf16_bits(x)
        xt = T(bits.view(np.int16), dev).view(torch.bfloat16)
        x = workloads.bf16_to_f32(bits)
    else:
        xt = T(x, dev)
    ref = oracle.forward_grouped(x, oW_t, obeta, G)
    x_q, gamma = bl.quant_act_grouped(xt, G)
    np.testing.assert_array_equal(x_q.cpu().numpy(), oracle.group_major(ref["x_q"], G))
    np.testing.assert_array_equal(gamma.cpu().numpy(), ref["gamma"])
    np.testing.assert_array_equal(bl.forward_grouped_acc(x_q, W_p).cpu().numpy(), ref["acc"])
    od = torch.bfloat16 if y_dtype == "bf16" else torch.float32
    y = bl.forward_grouped(x_q, gamma, W_p, beta, out_dtype=od)
    check_y(y, ref, y_dtype)
    y2 = bl.forward_grouped_fp(xt, W_p, beta, out_dtype=od)
    assert torch.equal(y.view(torch.int16) if y_dtype == "bf16" else y,
                       y2.view(torch.int16) if y_dtype == "bf16" else y2)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("M", [1, 3, 4, 5, 64, 130])
def test_grouped_parity(dev, M, G):
    run_case(dev, M, 2048, 333, G, seed=M * 11 + G)


@pytest.mark.parametrize("M,K,N,G", [(1, 512, 5, 8), (2, 1024, 149, 2), (4, 64 * 8 * 9, 700, 8), (7, 4096, 2000, 4)])
def test_grouped_ragged_and_small(dev, M, K, N, G):
    run_case(dev, M, K, N, G, seed=K + N + G)


def test_grouped_bf16(dev):
    run_case(dev, 1, 4096, 1000, 4, 61, y_dtype="bf16", x_dtype="bf16")
    run_case(dev, 200, 2048, 600, 2, 62, y_dtype="bf16", x_dtype="bf16")


@pytest.mark.parametrize("engine", ["cuda_cores", "tensor_cores"])
def test_grouped_engines(dev, engine):
    with bl.decode_engine(engine):
        run_case(dev, 1, 4096, 3000, 4, 69)      # one token: quantiser fused per group
        run_case(dev, 1, 2048, 500, 8, 68, y_dtype="bf16", x_dtype="bf16")
        run_case(dev, 2, 4096, 3000, 4, 70)
        run_case(dev, 12, 4096, 900, 2, 71)


def test_grouped_g1_equals_ungrouped(dev):
    W = workloads.latent_weights(80, 1111, 4096)
    x = T(workloads.activations(81, 3, 4096, outliers=True), dev)
    W_t, beta = bl.quantize_weights_grouped(T(W, dev), 1)
    W_t1, beta1 = bl.quantize_weights(T(W, dev))
    assert torch.equal(W_t[0], W_t1) and torch.equal(beta, beta1)
    y = bl.forward_grouped_fp(x, bl.pack_grouped(W_t), beta)
    assert torch.equal(y, bl.forward_fp(x, bl.pack(W_t1), beta1))


@pytest.mark.parametrize("shape", workloads.W2.shapes, ids=lambda s: s.name)
def test_grouped_workload_decode_m1(dev, shape):
    # the decode shapes with 4 groups (K/4 = 1024 and 2752 channels per group)
    W_p, beta, oW_t, obeta = prep(dev, shape.N, shape.K, 4, 90)
    bits = shape.inputs_bf16_bits()
    x = workloads.bf16_to_f32(bits)
    y = bl.forward_grouped_fp(T(bits.view(np.int16), dev).view(torch.bfloat16), W_p, beta)
    check_y(y, oracle.forward_grouped(x, oW_t, obeta, 4), "f32")
