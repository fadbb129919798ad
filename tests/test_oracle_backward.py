"""Pins for the oracle's gradients (oracle/backward.py): its torch forward is
checked against the C oracle's token loop, and its gradients against central
finite differences of that forward (every input element of a tiny problem) and
against the closed form of the beta = 0 case; the chunk-form gradient evaluator
is checked against those gradients."""
import numpy as np
import pytest

import oracle
from oracle import backward as ob


def _rng(seed):
    return np.random.default_rng(seed)


def _problem(seed, lens, H, Hk, dk, dv):
    r = _rng(seed)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    T, N = int(cu[-1]), len(lens)
    return dict(q=r.normal(size=(T, Hk, dk)), k=r.normal(size=(T, Hk, dk)),
                v=r.normal(size=(T, H, dv)), g=-0.5 * np.abs(r.normal(size=(T, H))),
                beta=r.uniform(size=(T, H)), h0=r.normal(size=(N, H, dk, dv))), cu


@pytest.mark.parametrize("H,Hk,l2", [(2, 2, True), (4, 2, True), (2, 2, False)])
def test_torch_forward_equals_c_oracle(H, Hk, l2):
    P, cu = _problem(1, [9, 0, 14], H, Hk, 5, 4)
    o1, h1 = ob.forward(P["q"], P["k"], P["v"], P["g"], P["beta"], cu, h0=P["h0"], scale=0.7,
                        qk_l2norm=l2)
    o2, h2 = oracle.recurrence(P["q"], P["k"], P["v"], P["g"], P["beta"], cu, dtype="f64",
                               h0=P["h0"], scale=0.7, qk_l2norm=l2, threads=1)
    assert np.abs(o1 - o2).max() < 1e-13 and np.abs(h1 - h2).max() < 1e-13


@pytest.mark.parametrize("H,Hk,l2", [(2, 1, True), (2, 2, False)])
def test_gradients_equal_central_differences(H, Hk, l2):
    # every element of every input of a tiny problem of two sequences
    P, cu = _problem(2, [4, 3], H, Hk, 3, 2)
    r = _rng(3)
    T, N = int(cu[-1]), 2
    do = r.normal(size=(T, H, 2))
    dhT = r.normal(size=(N, H, 3, 2))
    kw = dict(scale=0.8, qk_l2norm=l2)
    grads = ob.recurrence_backward(P["q"], P["k"], P["v"], P["g"], P["beta"], cu, do, dhT,
                                   h0=P["h0"], **kw)
    names = ["q", "k", "v", "g", "beta", "h0"]

    def loss(args):
        o, hT = ob.forward(*(args[n] for n in names[:5]), cu, h0=args["h0"], **kw)
        return float((o * do).sum() + (hT * dhT).sum())

    h = 1e-6
    worst = 0.0
    for a, name in enumerate(names):
        for idx in np.ndindex(P[name].shape):
            args = {n: P[n].copy() for n in names}
            args[name][idx] += h
            lp = loss(args)
            args[name][idx] -= 2 * h
            lm = loss(args)
            fd = (lp - lm) / (2 * h)
            worst = max(worst, abs(fd - grads[a][idx]) / max(1.0, abs(fd)))
    assert worst < 1e-7, worst


def test_beta0_closed_form_gradients():
    # beta = 0: o_t = e^{gamma_t} S_0^T q_t and S_T = e^{gamma_T} S_0 (no L2 norm), so
    # dv = dk = 0, dh0 = sum_t e^{gamma_t} q_t do_t^T + e^{gamma_T} dS_T,
    # dq_t = e^{gamma_t} S_0 do_t, and dg_t sums the terms of every gamma_t' with t' >= t.
    r = _rng(4)
    T, dk, dv = 6, 4, 3
    q, k, v = r.normal(size=(T, 1, dk)), r.normal(size=(T, 1, dk)), r.normal(size=(T, 1, dv))
    g = -np.abs(r.normal(size=(T, 1)))
    beta = np.zeros((T, 1))
    S0 = r.normal(size=(1, 1, dk, dv))
    do, dhT = r.normal(size=(T, 1, dv)), r.normal(size=(1, 1, dk, dv))
    dq, dk_, dv_, dg, dbeta, dh0 = ob.recurrence_backward(q, k, v, g, beta, [0, T], do, dhT, h0=S0,
                                                          qk_l2norm=False)
    gam = np.cumsum(g[:, 0])
    S = S0[0, 0]
    assert np.abs(dv_).max() == 0.0
    ref_dh0 = sum(np.exp(gam[t]) * np.outer(q[t, 0], do[t, 0]) for t in range(T)) + \
        np.exp(gam[-1]) * dhT[0, 0]
    assert np.abs(dh0[0, 0] - ref_dh0).max() < 1e-12
    ref_dq = np.stack([np.exp(gam[t]) * S @ do[t, 0] for t in range(T)])
    assert np.abs(dq[:, 0] - ref_dq).max() < 1e-12
    # g_t enters gamma_t' for every t' >= t and the final state
    contrib = np.array([np.exp(gam[t]) * (q[t, 0] @ S @ do[t, 0]) for t in range(T)])
    final = np.exp(gam[-1]) * np.sum(S * dhT[0, 0])
    ref_dg = np.array([contrib[t:].sum() + final for t in range(T)])
    assert np.abs(dg[:, 0] - ref_dg).max() < 1e-12
    assert np.abs(dk_).max() < 1e-15  # k enters only through beta-weighted terms


@pytest.mark.parametrize("lens,H,Hk,l2,chunk,g_scale", [
    ([37, 0, 9, 70], 2, 1, True, 16, 0.5),   # ragged, empty, grouped heads
    ([33], 1, 1, False, 4, 0.2),              # no L2 norm
    ([20, 65], 2, 2, True, 64, 3.0),          # strong decay across a full chunk
    ([19], 1, 1, True, 1, 1.0),               # chunk of one token
])
def test_chunked_backward_equals_autograd(lens, H, Hk, l2, chunk, g_scale):
    # the chunk-level gradient algebra (what a tensor-core backward evaluates)
    # against autograd of the token loop
    r = _rng(30 + chunk)
    cu = np.concatenate([[0], np.cumsum(lens)])
    T, N, dk, dv = int(cu[-1]), len(lens), 6, 5
    q, k = r.normal(size=(T, Hk, dk)), r.normal(size=(T, Hk, dk))
    if not l2:
        q, k = 0.3 * q, 0.3 * k
    v = r.normal(size=(T, H, dv))
    g = -g_scale * np.abs(r.normal(size=(T, H)))
    beta = r.uniform(size=(T, H))
    h0, dhT = r.normal(size=(N, H, dk, dv)), r.normal(size=(N, H, dk, dv))
    do = r.normal(size=(T, H, dv))
    kw = dict(h0=h0, scale=0.8, qk_l2norm=l2)
    ref = ob.recurrence_backward(q, k, v, g, beta, cu, do, dhT, **kw)
    got = ob.chunked_backward(q, k, v, g, beta, cu, do, dhT, chunk=chunk, **kw)
    for name, a_, b_ in zip(["dq", "dk", "dv", "dg", "dbeta", "dh0"], got, ref):
        assert np.abs(a_ - b_).max() <= 1e-12 * max(np.abs(b_).max(), 1.0), name
