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
import oracle
from gpu_util import DEV, TOL_BF16, dev_tensor, err, host, prefill_gpu, prefill_oracle


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


def test_decode_layer_wait_timeout_is_reported_and_recovered():
    """The streaming whole-mixer decode step: with the wait limit at 0 each
    CTA's first wait for a state copy, probed right after the copy is issued,
    cannot be complete, so the step records GDN_ERR_TIMEOUT, lets the copy land
    and returns; the next step runs normally."""
    r = np.random.default_rng(42)
    N, H, d, K = 60, 10, 128, 4
    C = 3 * H * d
    bf = lambda a: gi.to_bf16_bits(a.astype(np.float32))
    x, cw, cs = bf(r.normal(size=(N, C))), bf(r.normal(size=(C, K)) * 0.5), bf(r.normal(size=(N, C, K - 1)))
    g = -np.abs(r.normal(size=(N, H))).astype(np.float32)
    beta = r.uniform(size=(N, H)).astype(np.float32)
    s0 = r.normal(0, 0.1, size=(N, H, d, d)).astype(np.float32)
    xd, cwd, gd, bd = dev_tensor(x, "bf16"), dev_tensor(cw, "bf16"), dev_tensor(g, "f32"), dev_tensor(beta, "f32")
    gdn.set_wait_limit_ns(0)
    try:
        gdn.decode_layer_step(xd, cwd, dev_tensor(cs, "bf16"), gd, bd, dev_tensor(s0, "f32"), H=H, dk=d, dv=d)
        with pytest.raises(gdn.GDNError, match="TIMEOUT"):
            gdn.check_device_status(DEV)
    finally:
        gdn.set_wait_limit_ns(-1)
    cs_d, state = dev_tensor(cs, "bf16"), dev_tensor(s0, "f32")
    o = gdn.decode_layer_step(xd, cwd, cs_d, gd, bd, state, H=H, dk=d, dv=d)
    gdn.check_device_status(DEV)
    o_ref, cs_ref, s_ref = oracle.decode_layer_step(x, cw, cs, g, beta, s0.astype(np.float64), dtype="bf16",
                                                    H=H, dk=d, dv=d)
    assert err(host(o), o_ref) <= TOL_BF16 and err(host(state), s_ref) <= TOL_BF16
