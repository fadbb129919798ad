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
from gpu_util import DEV, TOL_BF16, dev_tensor, err, host, prefill_oracle


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
        # and against the fp64 oracle, so a fault shared by both entry points shows
        o_or, h_or = prefill_oracle(P)
        assert err(host(o), o_or) <= TOL_BF16
        assert err(host(hT), h_or) <= TOL_BF16


def _call_empty(L, N, hT):
    """N empty sequences (T_tot = 0, zero initial state): only the schedule and
    the final-state copies run, through the shared array."""
    cu = torch.zeros(N + 1, dtype=torch.int32, device=DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream)
    return L.gdn_prefill_noalloc(None, None, None, gdn.GDN_F32, None, None, _p(cu), None, N, 0, 1,
                                 0, 16, 16, 0, 0, 0, 1.0, 1, 1e-6, 0, 64, None, _p(hT), None, 0,
                                 stream)


def test_noalloc_size_limit_boundary():
    """The array holds a 256-byte header plus 4 bytes per sequence: 16320
    sequences fit (the identity-order schedule used above 8192 sequences runs
    through the shared array), 16321 are refused with GDN_ERR_WORKSPACE."""
    L = gdn.lib()
    cap = L.gdn_prefill_noalloc_max_scratch()
    assert cap == 64 * 1024
    n_max = (cap - 256) // 4
    assert n_max == 16320
    hT = torch.full((n_max, 1, 16, 16), 7.0, dtype=torch.float32, device=DEV)
    assert _call_empty(L, n_max, hT) == 0
    gdn.check_device_status(DEV)
    assert torch.count_nonzero(hT).item() == 0  # empty sequences: hT = h0 = 0
    hT2 = torch.empty((n_max + 1, 1, 16, 16), dtype=torch.float32, device=DEV)
    assert _call_empty(L, n_max + 1, hT2) == 3  # GDN_ERR_WORKSPACE, nothing launched
    gdn.check_device_status(DEV)


def test_noalloc_checks_arguments_before_the_size_limit():
    """An invalid problem reports the same error as gdn_prefill would, even when
    it is also too large for the array."""
    L = gdn.lib()
    fake = ctypes.c_void_p(1 << 20)
    too_many = 20000
    # H = 3 value heads on Hk = 2 q/k heads: INVALID_ARG from the argument checks
    st = L.gdn_prefill_noalloc(fake, fake, fake, gdn.GDN_BF16, fake, fake, fake, None, too_many,
                               too_many, 3, 2, 128, 128, 0, 0, 0, 1.0, 1, 1e-6, 0, 64, None, None,
                               fake, 0, None)
    assert st == 1
    # a valid problem of that size: WORKSPACE, before anything is launched
    st = L.gdn_prefill_noalloc(fake, fake, fake, gdn.GDN_BF16, fake, fake, fake, None, too_many,
                               too_many, 1, 0, 128, 128, 0, 0, 0, 1.0, 1, 1e-6, 0, 64, None, None,
                               fake, 0, None)
    assert st == 3
