"""The MatMul-free GLU channel mixer (bitlinear_glu_forward) against the CPU
oracle: MatMul-free blog, section "Kerncomponenten: MLGRU en GLU" (two
BitLinears on one input, SiLU of one times the other, a third BitLinear),
every BitLinear input RMS-normalised (figure item "RMS norm").

The gated intermediate u and the output y must equal the oracle's binary32
values; u is SiLU(gate) * up computed in binary64 and rounded once on both
sides, with exp a library routine on each side (the one step whose parity
is not pinned beyond its binary64 error bound).  Shapes cover the one-launch
gate/up path (M <= 4, both decode engines), the GEMM path and the decoder
block's dimensions; large M is checked on sampled tokens.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import ternary_weight_linear_forward_b200 as bl

pytestmark = pytest.mark.gpu


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


def prep(dev, D, F, seed):
    shapes = {"gate": (F, D), "up": (F, D), "down": (D, F)}
    Ws = {p: workloads.latent_weights(seed + i, *shapes[p]) for i, p in enumerate(shapes)}
    layers = {p: bl.BitLinear.from_float(T(W, dev)) for p, W in Ws.items()}
    tern = {p: oracle.quantize_weights(W) for p, W in Ws.items()}
    for p in shapes:
        assert layers[p].beta.item() == float(tern[p][1])
    return layers, tern


def check(dev, M, D, F, seed, rows=None):
    layers, tern = prep(dev, D, F, seed)
    x = workloads.activations(seed + 50, M, D, outliers=True)
    y, u = bl.glu_forward(T(x, dev), layers["gate"], layers["up"], layers["down"], want_u=True)
    y, u = y.cpu().numpy(), u.cpu().numpy()
    rows = np.arange(M) if rows is None else rows
    ref = oracle.glu(x[rows], tern)
    np.testing.assert_array_equal(u[rows], ref["u"])
    np.testing.assert_array_equal(y[rows], ref["y"])
    return layers, x, y


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 16, 64, 130])
@pytest.mark.parametrize("D,F", [(256, 384), (1024, 2816)])
def test_glu_parity(dev, M, D, F):
    check(dev, M, D, F, seed=M + D + F)


@pytest.mark.parametrize("engine", ["cuda_cores", "tensor_cores"])
@pytest.mark.parametrize("M", [1, 4, 9])
def test_glu_block_dims_both_engines(dev, engine, M):
    # hidden 2560, intermediate 6912 (the decoder block's MLP)
    with bl.decode_engine(engine):
        check(dev, M, 2560, 6912, seed=300 + M)


def test_glu_large_m_sampled_tokens(dev):
    M = 700
    rows = np.random.default_rng(5).choice(M, 10, replace=False)
    rows[:2] = [0, M - 1]
    check(dev, M, 2560, 6912, seed=400, rows=rows)


def test_glu_equals_the_calls_one_by_one(dev):
    M, D, F = 3, 1024, 2816
    layers, x, y = check(dev, M, D, F, seed=500)
    xt = T(x, dev)
    _, xq, g = bl.quant_act_rms(xt)
    gate = bl.forward(xq, g, layers["gate"].W_p, layers["gate"].beta)
    up = bl.forward(xq, g, layers["up"].W_p, layers["up"].beta)
    _, uq, gu = bl.quant_act_rms(gate, up, "silu_mul")
    y2 = bl.forward(uq, gu, layers["down"].W_p, layers["down"].beta)
    np.testing.assert_array_equal(y, y2.cpu().numpy())


def test_glu_without_u_output(dev):
    layers, tern = prep(dev, 512, 1024, 600)
    x = workloads.activations(601, 2, 512)
    y = bl.glu_forward(T(x, dev), layers["gate"], layers["up"], layers["down"])
    np.testing.assert_array_equal(y.cpu().numpy(), oracle.glu(x, tern)["y"])
