"""The bounded waits of the tensor-core prefill: a wait that runs out records
GDN_ERR_TIMEOUT, the kernel drains what it has in flight, frees its tensor
memory and returns, and the context stays usable. The wait limit is set to 0
(every hand-off wait that is not already complete at its first probe gives
up), so the timeout is certain and nothing waits on anything that cannot
finish: the kernel's own copies and tensor-core operations always complete."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import gated_deltanet_linear_silu_b200 as gdn
import gdn_inputs as gi
from gpu_util import DEV, TOL_BF16, err, prefill_gpu, prefill_oracle


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(DEV)


def test_prefill_wait_timeout_is_reported_and_recovered():
    P = gi.random_prefill(41, [128], H=1, dk=128, dv=128, with_h0=True)
    gdn.set_wait_limit_ns(0)
    try:
        with pytest.raises(gdn.GDNError, match="TIMEOUT"):
            prefill_gpu(P, algo="tensor")  # raises from the device status check
    finally:
        gdn.set_wait_limit_ns(-1)
    torch.cuda.synchronize()
    gdn.check_device_status(DEV)  # the status word was cleared by the report
    o, hT = prefill_gpu(P, algo="tensor")
    o_ref, h_ref = prefill_oracle(P)
    assert err(o, o_ref) <= TOL_BF16 and err(hT, h_ref) <= TOL_BF16
    assert np.isfinite(o).all()
