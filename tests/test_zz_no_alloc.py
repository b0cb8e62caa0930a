"""bitlinear_forward_noalloc: the forward for callers that cannot allocate
device memory (a runtime with a fixed arena and no device allocator to give
the library, or code recorded into a stream capture).  Its prefill scratch is
a static device array inside the library.  It must give the same outputs as
bitlinear_forward with a caller workspace, call after call (the shared
scratch keeps the previous call's contents).

This file is collected last so a run that stops at the first failure has run
every other test first."""
import pytest
import torch

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


def _calls(dev, seq, K, N, y_dtype):
    """forward_noalloc and forward on the same inputs for each M of `seq`, in
    that order; both run the same kernels, so the outputs must be equal bit
    for bit, whatever the shared scratch held from the call before."""
    W = torch.from_numpy(workloads.latent_weights(7 + N, N, K)).to(dev)
    W_t, beta = bl.quantize_weights(W)
    W_p = bl.pack(W_t)
    outs = []
    for call, M in enumerate(seq):
        x = torch.from_numpy(workloads.activations(100 * call + M, M, K, outliers=True)).to(dev)
        x_q, gamma = bl.quant_act(x)
        ref = bl.forward(x_q, gamma, W_p, beta, out_dtype=y_dtype)
        got = bl.forward_noalloc(x_q, gamma, W_p, beta, out_dtype=y_dtype)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), (call, M)
        outs.append(got.clone())
    bl.device_status()
    return outs


@pytest.mark.parametrize("y_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("M,K,N", [(300, 1024, 520), (2048, 4096, 256), (1, 4096, 1000), (65, 2560, 333)])
def test_noalloc_matches_forward_on_consecutive_calls(dev, M, K, N, y_dtype):
    outs = _calls(dev, [M, M], K, N, y_dtype)
    assert not torch.equal(outs[0], outs[1])      # the second call did new work


@pytest.mark.parametrize("y_dtype", [torch.float32, torch.bfloat16])
def test_noalloc_smaller_call_after_a_larger_one(dev, y_dtype):
    # the scratch keeps the larger call's row sums beyond the smaller M; the
    # smaller call must neither read them nor be disturbed by them
    _calls(dev, [2048, 100, 1500, 65, 2048], 2048, 384, y_dtype)


def test_noalloc_rejects_more_rows_than_its_scratch(dev):
    M, K, N = 16385, 64, 8
    x_q = torch.zeros((M, K), dtype=torch.int8, device=dev)
    gamma = torch.ones(M, dtype=torch.float32, device=dev)
    W_p = torch.zeros((N, K // 16), dtype=torch.int32, device=dev)
    beta = torch.ones(4, dtype=torch.float32, device=dev)[:1]
    with pytest.raises(bl.BitLinearError) as e:
        bl.forward_noalloc(x_q, gamma, W_p, beta)
    assert e.value.status == 5  # BL_ERR_WORKSPACE
