"""Failure detection: a bounded wait that runs out is reported, and the
context stays usable.

Every spin of the library's kernels on an mbarrier gives up after a limit,
raises the device error word and returns; bitlinear_device_status then
reports BL_ERR_TIMEOUT.  The test hook bitlinear_test_expire_next_wait makes
the next launch of the general small-M decode kernel wait for weights that
its first CTA's producer never requests, with a limit of ~1e5 cycles: no copy
is in flight when the consumers give up, so nothing hangs.  The next normal
call must be exact again.
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


def test_bounded_wait_expires_and_reports_timeout(dev):
    K, N = 4096, 11008
    W = workloads.latent_weights(77, N, K)
    x = workloads.activations(78, 1, K, outliers=True)
    W_t, beta = bl.quantize_weights(torch.from_numpy(W).to(dev))
    W_p = bl.pack(W_t)
    xt = torch.from_numpy(x).to(dev)
    oW_t, obeta = oracle.quantize_weights(W)
    ref = oracle.forward(x, oW_t, obeta)
    prob = [{"x": xt, "W_p": W_p, "beta": beta}]
    bl.device_status()
    with bl.decode_engine("cuda_cores_general"):
        bl.lib().bitlinear_test_expire_next_wait(1)
        try:
            bl.forward_fp_batch(prob)
            with pytest.raises(bl.BitLinearError) as e:
                bl.device_status()
            assert e.value.status == 8          # BL_ERR_TIMEOUT
        finally:
            bl.lib().bitlinear_test_expire_next_wait(0)
        (y,) = bl.forward_fp_batch(prob)
    np.testing.assert_array_equal(y.cpu().numpy(), ref["y"])
    bl.device_status()
