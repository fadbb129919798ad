"""Randomised properties of the CPU oracle (hypothesis): over random shapes,
sequence-length mixes, chunk sizes, head groupings and both recurrence orders,
the fp64 chunked evaluator equals the token loop, the conv equals torch's
conv1d, and packing sequences equals running them one by one."""
import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle

SETTINGS = settings(max_examples=25, deadline=None,
                    suppress_health_check=[HealthCheck.too_slow, HealthCheck.data_too_large])


@st.composite
def problems(draw):
    lens = draw(st.lists(st.integers(0, 40), min_size=1, max_size=4))
    Hk = draw(st.integers(1, 2))
    H = Hk * draw(st.integers(1, 3))
    dk, dv = draw(st.integers(1, 6)), draw(st.integers(1, 6))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    r = np.random.default_rng(seed)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    T = int(cu[-1])
    g_scale = draw(st.sampled_from([0.0, 0.3, 2.0, 9.0]))
    return dict(q=r.normal(size=(T, Hk, dk)), k=r.normal(size=(T, Hk, dk)),
                v=r.normal(size=(T, H, dv)), g=-g_scale * np.abs(r.normal(size=(T, H))),
                beta=r.uniform(size=(T, H)), h0=r.normal(size=(len(lens), H, dk, dv)),
                cu=cu, chunk=draw(st.sampled_from([1, 2, 5, 16, 64])),
                undecayed=draw(st.booleans()), l2=draw(st.booleans()))


@SETTINGS
@given(problems())
def test_chunked_evaluator_equals_token_loop(P):
    kw = dict(dtype="f64", h0=P["h0"], scale=0.9, qk_l2norm=P["l2"], threads=1,
              undecayed=P["undecayed"])
    if not P["l2"]:
        P["q"], P["k"] = 0.4 * P["q"], 0.4 * P["k"]
    args = (P["q"], P["k"], P["v"], P["g"], P["beta"], P["cu"])
    o1, h1 = oracle.recurrence(*args, **kw)
    o2, h2 = oracle.chunked(*args, chunk=P["chunk"], **kw)
    scale_o = max(np.abs(o1).max(), 1.0) if o1.size else 1.0
    assert np.abs(o1 - o2).max(initial=0.0) <= 1e-10 * scale_o
    assert np.abs(h1 - h2).max() <= 1e-10 * max(np.abs(h1).max(), 1.0)


@SETTINGS
@given(problems())
def test_packing_equals_separate_sequences(P):
    kw = dict(dtype="f64", scale=0.9, threads=1, undecayed=P["undecayed"])
    args = (P["q"], P["k"], P["v"], P["g"], P["beta"])
    o, hT = oracle.recurrence(*args, P["cu"], h0=P["h0"], **kw)
    cu = P["cu"]
    for n in range(len(cu) - 1):
        a, b = int(cu[n]), int(cu[n + 1])
        on, hn = oracle.recurrence(*(x[a:b] for x in args), [0, b - a], h0=P["h0"][n:n + 1], **kw)
        assert np.array_equal(o[a:b], on) and np.array_equal(hT[n], hn[0])


@SETTINGS
@given(st.integers(1, 30), st.integers(1, 12), st.integers(1, 4), st.booleans(),
       st.integers(0, 2 ** 31 - 1))
def test_conv_equals_torch_conv1d(T, C, K, with_state, seed):
    r = np.random.default_rng(seed)
    x, w = r.normal(size=(T, C)), r.normal(size=(C, K))
    state = r.normal(size=(1, C, K - 1)) if with_state else None
    y, st_out = oracle.conv_silu(x, w, [0, T], dtype="f64", state_in=state, apply_silu=False)
    xt = torch.from_numpy(x.T.copy())[None]
    pre = torch.from_numpy(state[0].copy())[None] if with_state else torch.zeros(1, C, K - 1,
                                                                                  dtype=torch.float64)
    ref = torch.nn.functional.conv1d(torch.cat([pre, xt], 2), torch.from_numpy(w.copy())[:, None, :],
                                     groups=C)[0].T.numpy()
    assert np.abs(y - ref).max() <= 1e-12 * max(np.abs(ref).max(), 1.0)
    # the state out is the last K-1 inputs of (state, x), oldest first
    full = np.concatenate([pre[0].numpy(), x.T], axis=1)
    assert np.array_equal(st_out[0], full[:, full.shape[1] - (K - 1):])
