"""gdn_prefill_noalloc: the prefill entry point for callers that cannot
allocate device memory where they run the mixer (a runtime whose memory
planner owns the whole device arena, a serving loop that must not call
cudaMalloc once running). It keeps its scratch in a fixed array inside the
library instead of a caller workspace.

These tests call it through the C ABI and compare it with gdn_prefill (the
workspace entry point) on two different problems in a row, so a stale
schedule left in the shared array by the first call would show up in the
second. This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import gated_deltanet_linear_silu_b200 as gdn
import gdn_inputs as gi
from gpu_util import DEV, TOL_BF16, dev_tensor, err, host


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(DEV)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _device_problem(P):
    q, k, v = (dev_tensor(a, P.dtype) for a in (P.q, P.k, P.v))
    g, beta = dev_tensor(P.g, "f32"), dev_tensor(P.beta, "f32")
    cu = torch.from_numpy(P.cu_seqlens.astype(np.int32)).to(DEV)
    h0 = None if P.h0 is None else dev_tensor(P.h0, "f32")
    return q, k, v, g, beta, cu, h0


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    L = gdn.lib()
    problems = [
        gi.random_prefill(31, [200, 0, 64, 129, 7, 300], H=3, dk=128, dv=128, with_h0=True),
        gi.random_prefill(32, [90, 450], H=2, dk=128, dv=128, with_h0=False),
    ]
    for P in problems:
        q, k, v, g, beta, cu, h0 = _device_problem(P)
        T, H, dk = q.shape
        dv = v.shape[2]
        N = P.N
        o_ref, hT_ref = gdn.prefill(q, k, v, g, beta, cu, initial_state=h0)
        o = torch.empty_like(o_ref)
        hT = torch.empty_like(hT_ref)
        stream = ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream)
        st = L.gdn_prefill_noalloc(_p(q), _p(k), _p(v), gdn.GDN_BF16, _p(g), _p(beta), _p(cu), None,
                                   N, T, H, 0, dk, dv, 0, 0, 0, 1.0, 1, 1e-6, 0, 64, _p(h0), _p(hT),
                                   _p(o), 0, stream)
        assert st == 0, gdn.STATUS.get(st, st)
        gdn.check_device_status(DEV)
        assert err(host(o), host(o_ref)) <= TOL_BF16
        assert err(host(hT), host(hT_ref)) <= TOL_BF16


def test_noalloc_rejects_problems_larger_than_its_scratch():
    L = gdn.lib()
    cap = L.gdn_prefill_noalloc_max_scratch()
    assert cap == 64 * 1024
    too_many = cap // 4  # the schedule needs 4 bytes per sequence plus a header
    fake = ctypes.c_void_p(1 << 20)
    st = L.gdn_prefill_noalloc(fake, fake, fake, gdn.GDN_BF16, fake, fake, fake, None, too_many,
                               too_many, 1, 0, 128, 128, 0, 0, 0, 1.0, 1, 1e-6, 0, 64, None, None, fake, 0,
                               None)
    assert st == 3  # GDN_ERR_WORKSPACE, before anything is launched
