"""Decoder block at batch-1 decode (hidden 2560, intermediate 6912): the fused
combine + RMSNorm + int8 quantiser and the seven-projection chain, against
the CPU oracle.  Codes must match bit for bit; float values within 1e-6
relative (the binary32 op order is the oracle's, so they match exactly)."""
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


def T(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def close(got, ref):
    g = np.asarray(got, np.float64).ravel()
    r = np.asarray(ref, np.float64).ravel()
    nz = r != 0
    assert np.all(g[~nz] == 0)
    if nz.any():
        rel = np.abs(g[nz] - r[nz]) / np.abs(r[nz])
        assert rel.max() <= REL_TOL, rel.max()


# up to 64 rows a row is shared by a cluster of 8 CTAs (K = 64: most CTAs have
# an empty slice; K = 81920: 40 KiB slices); from 65 rows, or beyond 81920
# channels, one CTA per row
@pytest.mark.parametrize("M,K", [(1, 2560), (1, 6912), (3, 1024), (1, 16), (2, 64), (64, 2560), (65, 1024),
                                 (1, 81920), (1, 81936)])
def test_quant_act_rms_none(dev, M, K):
    x = workloads.activations(M + K, M, K, outliers=True)
    h, x_q, g = bl.quant_act_rms(T(x, dev), want_h=True)
    for m in range(M):
        ox_q, og, _ = oracle.quant_act_rmsnorm(x[m:m + 1])
        np.testing.assert_array_equal(x_q.cpu().numpy()[m], ox_q[0])
        assert g.cpu().numpy()[m] == og[0]
    np.testing.assert_array_equal(h.cpu().numpy(), x)


def test_quant_act_rms_add_and_silu_mul(dev):
    K = 6912
    a = workloads.activations(1, 2, K) * np.float32(3)
    b = workloads.activations(2, 2, K)
    h, x_q, g = bl.quant_act_rms(T(a, dev), T(b, dev), "add", want_h=True)
    ref_h = (a + b).astype(np.float32)
    np.testing.assert_array_equal(h.cpu().numpy(), ref_h)
    for m in range(2):
        ox_q, og, _ = oracle.quant_act_rmsnorm(ref_h[m:m + 1])
        np.testing.assert_array_equal(x_q.cpu().numpy()[m], ox_q[0])
        assert g.cpu().numpy()[m] == og[0]
    h, x_q, g = bl.quant_act_rms(T(a, dev), T(b, dev), "silu_mul", want_h=True)
    ref_u = np.stack([oracle.silu_mul(a[m], b[m]) for m in range(2)])
    close(h.cpu().numpy(), ref_u)
    np.testing.assert_array_equal(h.cpu().numpy(), ref_u)     # binary64 then one rounding: identical
    for m in range(2):
        ox_q, og, _ = oracle.quant_act_rmsnorm(ref_u[m:m + 1])
        np.testing.assert_array_equal(x_q.cpu().numpy()[m], ox_q[0])
    # residual-only form: no quantiser, only h
    h2, xq2, g2 = bl.quant_act_rms(T(a, dev), T(b, dev), "add", want_h=True, quantize=False)
    assert xq2 is None and g2 is None
    np.testing.assert_array_equal(h2.cpu().numpy(), ref_h)


def test_decoder_block_matches_oracle(dev):
    weights = workloads.block_weights()
    x = workloads.block_input()
    blk = bl.DecoderBlock.from_float({p: T(w, dev) for p, w in weights.items()})
    out = blk(T(x, dev))
    torch.cuda.synchronize()
    tern = {p: oracle.quantize_weights(w) for p, w in weights.items()}
    for p in bl.DecoderBlock.PROJ:
        assert blk.layers[p].beta.item() == float(tern[p][1])
    ref = oracle.block_decode(x, tern)
    for key in ("q", "k", "v", "o", "h1", "gate", "up", "u", "down", "out"):
        close(out[key].cpu().numpy(), ref[key])
        np.testing.assert_array_equal(out[key].cpu().numpy().ravel(), np.asarray(ref[key]).ravel())
    bl.device_status()
