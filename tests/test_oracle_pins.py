"""Pins for the CPU oracle: each check compares the oracle with something other
than itself -- closed forms, exact retrieval identities, explicit unrolled
matrix products, a hand-worked example, a library conv1d, linearity, a norm
bound and the independent fp64 chunkwise evaluator.

The recurrence pinned here is the decay-first gated delta rule of the
Qwen3.5-MoE source walkthrough, section 4.3; in matrix form (state [d_k, d_v])
S_t = a_t (I - b_t k_t k_t^T) S_{t-1} + b_t k_t v_t^T and o_t = S_t^T q_t,
the transpose of the form S_t = a_t S_{t-1}(I - b_t k k^T) + b_t v k^T,
o_t = S_t q_t, in which the state is [d_v, d_k].

The last test plants each plausible mistake in the oracle (on the CPU) and
checks that at least one pin catches it.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rec(planted=0):
    def f(q, k, v, g, beta, cu, **kw):
        kw.setdefault("dtype", "f64")
        return oracle.recurrence(np.asarray(q, np.float64), np.asarray(k, np.float64),
                                 np.asarray(v, np.float64), np.asarray(g, np.float64),
                                 np.asarray(beta, np.float64), cu, _planted=planted,
                                 threads=2, **kw)
    return f


# --------------------------------------------------------------------------
# Pins as functions of the recurrence under test; each returns an error.
# --------------------------------------------------------------------------

def pin_beta0_pure_decay(rec):
    """beta = 0: S_T = exp(sum g) S_0 and o_t = exp(gamma_t) S_0^T q_t."""
    r = _rng(1)
    T, H, dk, dv = 9, 2, 5, 3
    q, k = r.normal(size=(T, H, dk)), r.normal(size=(T, H, dk))
    v = r.normal(size=(T, H, dv))
    g = -np.abs(r.normal(size=(T, H)))
    beta = np.zeros((T, H))
    h0 = r.normal(size=(1, H, dk, dv))
    o, hT = rec(q, k, v, g, beta, [0, T], h0=h0, qk_l2norm=False)
    gam = np.cumsum(g, axis=0)
    o_ref = np.einsum("th,hij,thi->thj", np.exp(gam), h0[0], q)
    hT_ref = np.exp(gam[-1])[:, None, None] * h0[0]
    return max(np.abs(o - o_ref).max(), np.abs(hT[0] - hT_ref).max())


def pin_orthonormal_retrieval(rec):
    """alpha = 1, beta = 1, S_0 = 0, orthonormal keys: after writing the pairs,
    querying with k_j returns v_j exactly (later tokens have beta = 0)."""
    r = _rng(2)
    dk, dv, m = 8, 6, 5
    Qm, _ = np.linalg.qr(r.normal(size=(dk, dk)))
    keys = Qm[:, :m].T                                  # m orthonormal rows
    vals = r.normal(size=(m, dv))
    T = 2 * m
    q = np.zeros((T, 1, dk)); k = np.zeros((T, 1, dk)); v = np.zeros((T, 1, dv))
    beta = np.zeros((T, 1)); g = np.zeros((T, 1))
    k[:m, 0], v[:m, 0], beta[:m, 0] = keys, vals, 1.0
    q[m:, 0] = keys[::-1]
    k[m:, 0] = keys[0]                                  # any key; beta=0 so no write
    o, hT = rec(q, k, v, g, beta, [0, T], qk_l2norm=False)
    err_read = np.abs(o[m:, 0] - vals[::-1]).max()
    err_state = np.abs(hT[0, 0] - keys.T @ vals).max()
    return max(err_read, err_state)


def pin_overwrite_identity(rec):
    """For any S_0 and unit k, one step with alpha = beta = 1 stores v at k:
    S_1^T k = v."""
    r = _rng(3)
    dk, dv = 6, 6
    h0 = r.normal(size=(1, 1, dk, dv))
    kk = _unit(r.normal(size=dk))
    vv = r.normal(size=dv)
    q = np.stack([r.normal(size=dk), kk])[:, None]
    k = np.stack([kk, kk])[:, None]
    v = np.stack([vv, r.normal(size=dv)])[:, None]
    g = np.zeros((2, 1)); beta = np.array([[1.0], [0.0]])
    o, hT = rec(q, k, v, g, beta, [0, 2], h0=h0, qk_l2norm=False)
    return np.abs(o[1, 0] - vv).max()


def pin_decay_first(rec):
    """Decay-first reading (the walkthrough's order): for unit k, one step gives
    S_1^T k = a(1-b) S_0^T k + b v. The retrieve-before-decay reading of the
    7.6.2 formula would give (a-b) S_0^T k + b v instead."""
    r = _rng(4)
    dk, dv = 5, 5
    h0 = r.normal(size=(1, 1, dk, dv))
    kk = _unit(r.normal(size=dk))
    vv = r.normal(size=dv)
    a, b = 0.5, 0.3
    _, hT = rec(kk[None, None], kk[None, None], vv[None, None], [[math.log(a)]], [[b]],
                [0, 1], h0=h0, qk_l2norm=False)
    ref = a * (1 - b) * (h0[0, 0].T @ kk) + b * vv
    return np.abs(hT[0, 0].T @ kk - ref).max()


def _unrolled(q, k, v, alpha, beta, S0, undecayed=False):
    """Transposed orientation P = S^T ([d_v, d_k]); P_t = P_0 prod B_j +
    sum_i b_i v_i k_i^T prod_{j>i} B_j with B_j = a_j (I - b_j k_j k_j^T)
    (or B_j = a_j I - b_j k_j k_j^T for the read-before-decay order), every
    product formed explicitly left to right. Returns (o [T,dv], P_T)."""
    T, dk = k.shape
    I = np.eye(dk)
    if undecayed:
        B = [alpha[j] * I - beta[j] * np.outer(k[j], k[j]) for j in range(T)]
    else:
        B = [alpha[j] * (I - beta[j] * np.outer(k[j], k[j])) for j in range(T)]
    outs, P = [], None
    for t in range(1, T + 1):
        P = S0.T.copy()
        for j in range(t):
            P = P @ B[j]
        for i in range(t):
            term = beta[i] * np.outer(v[i], k[i])
            for j in range(i + 1, t):
                term = term @ B[j]
            P = P + term
        outs.append(P @ q[t - 1])
    return np.array(outs), P


def pin_brute_force(rec):
    err = 0.0
    for seed, (T, dk, dv) in enumerate([(1, 1, 1), (3, 2, 3), (6, 4, 4), (5, 3, 2), (6, 3, 3)]):
        r = _rng(100 + seed)
        q, k = r.normal(size=(T, dk)), r.normal(size=(T, dk))
        v = r.normal(size=(T, dv))
        g = -np.abs(r.normal(size=T)); beta = r.uniform(size=T)
        S0 = r.normal(size=(dk, dv))
        scale = 0.7
        qn = _unit(q) * scale  # the oracle normalises with eps; use eps=0 here
        kn = _unit(k)
        o_ref, P = _unrolled(qn, kn, v, np.exp(g), beta, S0)
        o, hT = rec(q[:, None], k[:, None], v[:, None], g[:, None], beta[:, None], [0, T],
                    h0=S0[None, None], scale=scale, qk_l2norm=True, eps=0.0)
        err = max(err, np.abs(o[:, 0] - o_ref).max(), np.abs(hT[0, 0] - P.T).max())
    return err


def pin_scalar_closed_form(rec):
    """d_k = d_v = 1: s_t = a_t (1 - b_t k_t^2) s_{t-1} + b_t k_t v_t, o_t = s_t q_t."""
    r = _rng(5)
    T = 12
    q, k, v = r.normal(size=T), r.normal(size=T), r.normal(size=T)
    g = -np.abs(r.normal(size=T)); beta = r.uniform(size=T)
    s = 0.37
    o_ref = []
    for t in range(T):
        s = math.exp(g[t]) * (1 - beta[t] * k[t] ** 2) * s + beta[t] * k[t] * v[t]
        o_ref.append(s * q[t])
    o, hT = rec(q[:, None, None], k[:, None, None], v[:, None, None], g[:, None], beta[:, None],
                [0, T], h0=np.full((1, 1, 1, 1), 0.37), qk_l2norm=False)
    return max(np.abs(o[:, 0, 0] - o_ref).max(), abs(hT[0, 0, 0, 0] - s))


def pin_hand_worked(rec):
    d = json.load(open(os.path.join(GOLD, "hand_worked_d2.json")))
    q, k, v = (np.array(d[x])[:, None] for x in ("q", "k", "v"))
    g = np.log(np.array(d["alpha"]))[:, None]
    beta = np.array(d["beta"])[:, None]
    o, hT = rec(q, k, v, g, beta, [0, 2], h0=np.array(d["h0"])[None, None], qk_l2norm=False)
    return max(np.abs(o[:, 0] - np.array(d["o"])).max(), np.abs(hT[0, 0] - np.array(d["hT"])).max())


ALL_PINS = [pin_beta0_pure_decay, pin_orthonormal_retrieval, pin_overwrite_identity,
            pin_decay_first, pin_brute_force, pin_scalar_closed_form, pin_hand_worked]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_recurrence_pin(pin):
    assert pin(_rec()) < 1e-12


def test_linearity_in_values_and_state():
    r = _rng(6)
    T, H, dk, dv = 11, 2, 4, 3
    q, k = r.normal(size=(T, H, dk)), r.normal(size=(T, H, dk))
    g = -np.abs(r.normal(size=(T, H))); beta = r.uniform(size=(T, H))
    V1, V2 = r.normal(size=(T, H, dv)), r.normal(size=(T, H, dv))
    S1, S2 = r.normal(size=(1, H, dk, dv)), r.normal(size=(1, H, dk, dv))
    a, b = 1.7, -0.4
    rec = _rec()
    o1, h1 = rec(q, k, V1, g, beta, [0, T], h0=S1)
    o2, h2 = rec(q, k, V2, g, beta, [0, T], h0=S2)
    o3, h3 = rec(q, k, a * V1 + b * V2, g, beta, [0, T], h0=a * S1 + b * S2)
    assert np.abs(o3 - (a * o1 + b * o2)).max() < 1e-12
    assert np.abs(h3 - (a * h1 + b * h2)).max() < 1e-12


def test_contraction_bound_and_state_carry():
    """||S_t||_2 <= a_t ||S_{t-1}||_2 + b_t ||v_t|| for unit keys, beta in [0,1];
    chaining one-token calls through h0/hT equals one call."""
    r = _rng(7)
    T, dk, dv = 20, 6, 5
    q, k, v = r.normal(size=(T, 1, dk)), r.normal(size=(T, 1, dk)), 3 * r.normal(size=(T, 1, dv))
    g = -np.abs(r.normal(size=(T, 1))); beta = r.uniform(size=(T, 1))
    S = r.normal(size=(1, 1, dk, dv))
    rec = _rec()
    o_all, h_all = rec(q, k, v, g, beta, [0, T], h0=S, eps=0.0)
    for t in range(T):
        o_t, S_new = rec(q[t:t + 1], k[t:t + 1], v[t:t + 1], g[t:t + 1], beta[t:t + 1], [0, 1],
                         h0=S, eps=0.0)
        bound = math.exp(g[t, 0]) * np.linalg.norm(S[0, 0], 2) + beta[t, 0] * np.linalg.norm(v[t, 0])
        assert np.linalg.norm(S_new[0, 0], 2) <= bound * (1 + 1e-12)
        assert np.abs(o_t[0] - o_all[t]).max() < 1e-12
        S = S_new
    assert np.abs(S - h_all).max() < 1e-12


def test_varlen_packing_equals_separate_calls():
    r = _rng(8)
    lens = [5, 1, 0, 9, 3]
    cu = np.concatenate([[0], np.cumsum(lens)])
    H, dk, dv = 2, 4, 3
    T = int(cu[-1])
    q, k, v = r.normal(size=(T, H, dk)), r.normal(size=(T, H, dk)), r.normal(size=(T, H, dv))
    g = -np.abs(r.normal(size=(T, H))); beta = r.uniform(size=(T, H))
    h0 = r.normal(size=(len(lens), H, dk, dv))
    rec = _rec()
    o, hT = rec(q, k, v, g, beta, cu, h0=h0)
    for n in range(len(lens)):
        a, b = cu[n], cu[n + 1]
        on, hn = rec(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], [0, b - a], h0=h0[n:n + 1])
        if b > a:
            assert np.abs(o[a:b] - on).max() == 0.0
        assert np.abs(hT[n] - hn[0]).max() == 0.0
    assert np.array_equal(hT[2], h0[2])  # empty sequence: state passes through


@pytest.mark.parametrize("chunk", [1, 4, 16, 64])
def test_chunked_evaluator_equals_token_loop(chunk):
    r = _rng(9)
    lens = [70, 3, 64, 129, 1]
    cu = np.concatenate([[0], np.cumsum(lens)])
    H, dk, dv = 2, 8, 6
    T = int(cu[-1])
    q, k, v = r.normal(size=(T, H, dk)), r.normal(size=(T, H, dk)), r.normal(size=(T, H, dv))
    g = -0.3 * np.abs(r.normal(size=(T, H))); beta = r.uniform(size=(T, H))
    h0 = r.normal(size=(len(lens), H, dk, dv))
    kw = dict(dtype="f64", h0=h0, scale=0.8, threads=2)
    o1, h1 = oracle.recurrence(q, k, v, g, beta, cu, **kw)
    o2, h2 = oracle.chunked(q, k, v, g, beta, cu, chunk=chunk, **kw)
    assert np.abs(o1 - o2).max() <= 1e-12 * np.abs(o1).max()
    assert np.abs(h1 - h2).max() <= 1e-12 * np.abs(h1).max()


def test_chunked_handles_strong_decay_without_overflow():
    """g down to -10 per token: exp(gamma) underflows across a chunk; the
    evaluator only forms exp of non-positive differences and stays finite."""
    r = _rng(10)
    T, H, d = 130, 1, 4
    q, k, v = r.normal(size=(T, H, d)), r.normal(size=(T, H, d)), r.normal(size=(T, H, d))
    g = -10 * r.uniform(size=(T, H)); beta = r.uniform(size=(T, H))
    o1, h1 = oracle.recurrence(q, k, v, g, beta, [0, T], dtype="f64", threads=1)
    o2, h2 = oracle.chunked(q, k, v, g, beta, [0, T], dtype="f64", chunk=64, threads=1)
    assert np.isfinite(o2).all() and np.isfinite(h2).all()
    assert np.abs(o1 - o2).max() <= 1e-12 * np.abs(o1).max()


# --------------------------------------------------------------------------
# Conv stage
# --------------------------------------------------------------------------

def _torch_conv(x, w, state=None):
    """Library reference: torch conv1d (groups=C, padding K-1), first T outputs,
    with the conv state prepended as the K-1 preceding inputs."""
    T, C = x.shape
    K = w.shape[1]
    xt = torch.from_numpy(x.T.copy())[None]
    if state is not None:
        xt = torch.cat([torch.from_numpy(state.copy())[None], xt], dim=2)
        y = torch.nn.functional.conv1d(xt, torch.from_numpy(w.copy())[:, None, :], groups=C)
    else:
        y = torch.nn.functional.conv1d(xt, torch.from_numpy(w.copy())[:, None, :], padding=K - 1,
                                       groups=C)[..., :T]
    return y[0].T.numpy()


def test_conv_matches_library_conv1d():
    r = _rng(11)
    T, C, K = 37, 24, 4
    x, w = r.normal(size=(T, C)), r.normal(size=(C, K))
    y, _ = oracle.conv_silu(x, w, [0, T], dtype="f64", apply_silu=False)
    assert np.abs(y - _torch_conv(x, w)).max() < 1e-12
    y2, _ = oracle.conv_silu(x, w, [0, T], dtype="f64", apply_silu=True)
    ref = torch.nn.functional.silu(torch.from_numpy(_torch_conv(x, w))).numpy()
    assert np.abs(y2 - ref).max() < 1e-12


def test_conv_delta_input_returns_taps_and_silu_zero():
    C, K, T = 3, 4, 8
    w = np.arange(1, C * K + 1, dtype=np.float64).reshape(C, K)
    x = np.zeros((T, C)); x[0, :] = 1.0
    y, _ = oracle.conv_silu(x, w, [0, T], dtype="f64", apply_silu=False)
    for t in range(K):
        assert np.array_equal(y[t], w[:, K - 1 - t])      # taps reversed in time
    assert np.array_equal(y[K:], np.zeros((T - K, C)))
    y0, _ = oracle.conv_silu(np.zeros((T, C)), w, [0, T], dtype="f64", apply_silu=True)
    assert np.array_equal(y0, np.zeros((T, C)))           # SiLU(0) = 0


@pytest.mark.parametrize("split", [1, 2, 3, 10, 20])
def test_conv_state_continuation(split):
    """Splitting a sequence at `split` and carrying the conv state equals one
    call (the state holds the K-1 latest inputs, zero-padded on the left)."""
    r = _rng(12)
    T, C, K = 21, 10, 4
    x, w = r.normal(size=(T, C)), r.normal(size=(C, K))
    st0 = r.normal(size=(1, C, K - 1))
    y, st = oracle.conv_silu(x, w, [0, T], dtype="f64", state_in=st0)
    ya, sa = oracle.conv_silu(x[:split], w, [0, split], dtype="f64", state_in=st0)
    yb, sb = oracle.conv_silu(x[split:], w, [0, T - split], dtype="f64", state_in=sa)
    assert np.abs(np.concatenate([ya, yb]) - y).max() < 1e-12
    assert np.array_equal(sb, st)
    assert np.array_equal(st[0], x[-(K - 1):].T)
    ref = torch.nn.functional.silu(torch.from_numpy(_torch_conv(x, w, st0[0]))).numpy()
    assert np.abs(y - ref).max() < 1e-12


def test_conv_state_short_sequence_and_fresh_start():
    C, K = 2, 4
    x = np.array([[1.0, 2.0]])
    _, st = oracle.conv_silu(x, np.ones((C, K)), [0, 1], dtype="f64")
    assert np.array_equal(st[0], np.array([[0, 0, 1.0], [0, 0, 2.0]]))


def test_conv_varlen_no_mixing_and_l2norm():
    r = _rng(13)
    lens = [6, 1, 0, 9]
    cu = np.concatenate([[0], np.cumsum(lens)])
    hd, C, K = 4, 12, 4           # q: 0..3, k: 4..7, v: 8..11
    x, w = r.normal(size=(int(cu[-1]), C)), r.normal(size=(C, K))
    y, st = oracle.conv_silu(x, w, cu, dtype="f64", qk_l2norm=True, n_qk=8, head_dim=hd, eps=0.0)
    for n in range(len(lens)):
        a, b = cu[n], cu[n + 1]
        yn, sn = oracle.conv_silu(x[a:b], w, [0, b - a], dtype="f64", qk_l2norm=True, n_qk=8,
                                  head_dim=hd, eps=0.0)
        assert np.array_equal(y[a:b], yn) and np.array_equal(st[n], sn[0])
    norms = np.linalg.norm(y[:, :8].reshape(-1, 2, hd), axis=-1)
    assert np.abs(norms - 1.0).max() < 1e-12
    raw, _ = oracle.conv_silu(x, w, cu, dtype="f64")
    assert np.array_equal(y[:, 8:], raw[:, 8:])           # v channels are not normalised


def test_bf16_decode_is_exact():
    import gdn_inputs
    vals = np.array([1.0, -2.5, 3.140625, 1e-3, 65504.0], np.float32)
    bits = gdn_inputs.to_bf16_bits(vals)
    widened = gdn_inputs.bf16_bits_to_f32(bits).astype(np.float64)
    y, _ = oracle.conv_silu(bits[:, None], gdn_inputs.to_bf16_bits(np.array([[0, 0, 0, 1.0]], np.float32)),
                            [0, len(vals)], dtype="bf16", apply_silu=False)
    assert np.array_equal(y[:, 0], widened)


# --------------------------------------------------------------------------
# Gated RMSNorm output ("Qwen3.5 ... linear-attention hybrid", 7.6.2 and 7.6.3)
# --------------------------------------------------------------------------

def test_gated_rmsnorm_hand_example():
    # one head, d_v = 2: y = (3, 4), mean(y^2) = 12.5, eps = 0.5 -> rms = sqrt(13)
    # z = (0, ln 3): SiLU(0) = 0, SiLU(ln 3) = ln 3 * 3/4; w = (2, 5)
    y = np.array([[3.0, 4.0]])
    z = np.array([[0.0, math.log(3.0)]])
    out = oracle.gated_rmsnorm(y, z, np.array([2.0, 5.0]), dtype="f64", eps=0.5)
    want = np.array([[0.0, 4.0 / math.sqrt(13.0) * 5.0 * math.log(3.0) * 0.75]])
    assert np.abs(out - want).max() < 1e-15


def test_gated_rmsnorm_per_head_scale_invariance():
    # eps = 0: scaling one head's y by any c > 0 leaves every output unchanged, so
    # the norm runs over that head's d_v values only (not over tokens or heads)
    r = _rng(21)
    y, z, w = r.normal(size=(5, 3, 8)), r.normal(size=(5, 3, 8)), r.normal(size=8)
    base = oracle.gated_rmsnorm(y, z, w, dtype="f64", eps=0.0)
    y2 = y.copy()
    y2[2, 1] *= 37.0
    assert np.abs(oracle.gated_rmsnorm(y2, z, w, dtype="f64", eps=0.0) - base).max() < 1e-13
    y3 = y.copy()
    y3[:, 1] *= 0.01
    assert np.abs(oracle.gated_rmsnorm(y3, z, w, dtype="f64", eps=0.0) - base).max() < 1e-13


def test_gated_rmsnorm_gate_is_silu():
    # SiLU(z) - SiLU(-z) = z: the difference of the two gated outputs is the plain
    # normalised, scaled y times z; w = 1 and eps = 0 make it unit-RMS per head
    r = _rng(22)
    y, z = r.normal(size=(4, 2, 16)), r.normal(size=(4, 2, 16))
    w = np.ones(16)
    d = oracle.gated_rmsnorm(y, z, w, dtype="f64", eps=0.0) - \
        oracle.gated_rmsnorm(y, -z, w, dtype="f64", eps=0.0)
    ratio = d / z
    assert np.abs(np.sqrt(np.mean(ratio ** 2, axis=-1)) - 1.0).max() < 1e-12
    assert np.abs(ratio * np.sqrt(np.mean(y ** 2, axis=-1, keepdims=True)) - y).max() < 1e-12


@pytest.mark.parametrize("Hk", [2, 1])
def test_decode_layer_steps_equal_packed_layer(Hk):
    # Token-by-token decode of the whole mixer (conv state and recurrent state
    # carried across calls) equals the packed path: conv over the sequence, then
    # the recurrence over it -- so the conv-state shift and hand-off are right.
    # Hk = 1 shares one q, k head between both value heads.
    r = _rng(23)
    H, dk, dv, K, T = 2, 4, 3, 4, 7
    C = 2 * Hk * dk + H * dv
    x = r.normal(size=(T, C))
    cw = r.normal(size=(C, K))
    cs0 = r.normal(size=(1, C, K - 1))
    h0 = r.normal(size=(1, H, dk, dv)) * 0.3
    g = -np.abs(r.normal(size=(T, H))) * 0.3
    b = 1.0 / (1.0 + np.exp(-r.normal(size=(T, H))))
    y, cs_ref = oracle.conv_silu(x, cw, [0, T], dtype="f64", state_in=cs0, qk_l2norm=True,
                                 n_qk=2 * Hk * dk, head_dim=dk, eps=1e-6)
    o_ref, h_ref = oracle.recurrence(y[:, :Hk * dk].reshape(T, Hk, dk),
                                     y[:, Hk * dk:2 * Hk * dk].reshape(T, Hk, dk),
                                     y[:, 2 * Hk * dk:].reshape(T, H, dv), g, b, [0, T],
                                     dtype="f64", h0=h0, qk_l2norm=False)
    cs, st = cs0, h0
    for t in range(T):
        o, cs, st = oracle.decode_layer_step(x[t:t + 1], cw, cs, g[t:t + 1], b[t:t + 1], st,
                                             dtype="f64", H=H, dk=dk, dv=dv, Hk=Hk)
        assert np.abs(o[0] - o_ref[t]).max() < 1e-12
    assert np.abs(cs - cs_ref).max() < 1e-15 and np.abs(st - h_ref).max() < 1e-12
    # the final conv state is the last K-1 inputs, oldest first
    assert np.array_equal(cs[0], x[T - (K - 1):].T)


def test_decode_layer_step_gate_and_input_encoding():
    # With a gate the step's output is the gated RMSNorm of the ungated output;
    # bf16-encoded inputs give exactly the result of their decoded fp64 values.
    import gdn_inputs
    r = _rng(24)
    N, H, dk, dv, K = 2, 2, 4, 4, 4
    C = 2 * H * dk + H * dv
    bits = lambda a: gdn_inputs.to_bf16_bits(a.astype(np.float32))
    dec = lambda b: gdn_inputs.bf16_bits_to_f32(b).astype(np.float64)
    x, cw, cs0 = bits(r.normal(size=(N, C))), bits(r.normal(size=(C, K))), bits(r.normal(size=(N, C, K - 1)))
    z = bits(r.normal(size=(N, H, dv)))
    st = r.normal(size=(N, H, dk, dv)) * 0.2
    g, b = -np.abs(r.normal(size=(N, H))), np.full((N, H), 0.5)
    nw = 1.0 + 0.1 * r.normal(size=dv)
    o_b, cs_b, st_b = oracle.decode_layer_step(x, cw, cs0, g, b, st, dtype="bf16", H=H, dk=dk, dv=dv,
                                               z=z, norm_w=nw)
    o_f, cs_f, st_f = oracle.decode_layer_step(dec(x), dec(cw), dec(cs0), g, b, st, dtype="f64",
                                               H=H, dk=dk, dv=dv, z=dec(z), norm_w=nw)
    assert np.array_equal(o_b, o_f) and np.array_equal(cs_b, cs_f) and np.array_equal(st_b, st_f)
    o_u, _, _ = oracle.decode_layer_step(dec(x), dec(cw), dec(cs0), g, b, st, dtype="f64", H=H,
                                         dk=dk, dv=dv)
    assert np.array_equal(o_f, oracle.gated_rmsnorm(o_u, dec(z), nw, dtype="f64"))


# --------------------------------------------------------------------------
# Grouped value heads: the config's linear_num_value_heads may exceed
# linear_num_key_heads; each q, k head then serves G consecutive value heads.
# --------------------------------------------------------------------------

@pytest.mark.parametrize("fn", ["recurrence", "chunked"])
def test_grouped_value_heads_equal_repeated_keys(fn):
    # Hk key heads shared by G = H / Hk value heads: the result equals the plain
    # (pinned) rule with every q, k head repeated G times in place
    r = _rng(26)
    lens = [37, 0, 70]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T, Hk, G, dk, dv = int(cu[-1]), 2, 3, 8, 5
    H = Hk * G
    q, k = r.normal(size=(T, Hk, dk)), r.normal(size=(T, Hk, dk))
    v = r.normal(size=(T, H, dv))
    g = -0.3 * np.abs(r.normal(size=(T, H))); beta = r.uniform(size=(T, H))
    h0 = r.normal(size=(len(lens), H, dk, dv))
    kw = dict(dtype="f64", h0=h0, scale=0.7, threads=2)
    if fn == "chunked":
        kw["chunk"] = 16
    f = getattr(oracle, fn)
    o, hT = f(q, k, v, g, beta, cu, **kw)
    o_r, h_r = f(np.repeat(q, G, axis=1), np.repeat(k, G, axis=1), v, g, beta, cu, **kw)
    assert np.array_equal(o, o_r) and np.array_equal(hT, h_r)
    # the other conceivable sharing (value head h reading key head h mod Hk)
    # gives a different result, so the check above tells the two apart
    o_t, _ = f(np.tile(q, (1, G, 1)), np.tile(k, (1, G, 1)), v, g, beta, cu, **kw)
    assert np.abs(o_t - o).max() > 1e-3


def test_grouped_value_heads_reject_uneven_groups():
    r = _rng(27)
    q, k, v = r.normal(size=(4, 2, 3)), r.normal(size=(4, 2, 3)), r.normal(size=(4, 3, 3))
    g, b = np.zeros((4, 3)), np.zeros((4, 3))
    with pytest.raises(ValueError):
        oracle.recurrence(q, k, v, g, b, [0, 4], dtype="f64", threads=1)


# --------------------------------------------------------------------------
# The order "7.6 Qwen3.5: linear-attention hybrid", 7.6.2 writes: the memory
# is read from S_{t-1} before the decay, S_t = a S_{t-1} + k [b (v - S_{t-1}^T k)]^T,
# i.e. S_t = (a I - b k k^T) S_{t-1} + b k v^T (the oracle's undecayed=True).
# --------------------------------------------------------------------------

def test_undecayed_brute_force():
    for seed, (T, dk, dv) in enumerate([(1, 1, 1), (3, 2, 3), (6, 4, 4), (5, 3, 2)]):
        r = _rng(200 + seed)
        q, k = r.normal(size=(T, dk)), r.normal(size=(T, dk))
        v = r.normal(size=(T, dv))
        g = -np.abs(r.normal(size=T)); beta = r.uniform(size=T)
        S0 = r.normal(size=(dk, dv))
        o_ref, P = _unrolled(_unit(q) * 0.7, _unit(k), v, np.exp(g), beta, S0, undecayed=True)
        o, hT = _rec()(q[:, None], k[:, None], v[:, None], g[:, None], beta[:, None], [0, T],
                       h0=S0[None, None], scale=0.7, eps=0.0, undecayed=True)
        assert np.abs(o[:, 0] - o_ref).max() < 1e-12 and np.abs(hT[0, 0] - P.T).max() < 1e-12


def test_undecayed_unit_key_one_step():
    # for unit k: S_1^T k = (a - b) S_0^T k + b v (the decay-first order gives a (1 - b) S_0^T k + b v)
    r = _rng(210)
    dk = dv = 5
    h0 = r.normal(size=(1, 1, dk, dv))
    kk = _unit(r.normal(size=dk)); vv = r.normal(size=dv)
    a, b = 0.5, 0.3
    _, hT = _rec()(kk[None, None], kk[None, None], vv[None, None], [[math.log(a)]], [[b]], [0, 1],
                   h0=h0, qk_l2norm=False, undecayed=True)
    assert np.abs(hT[0, 0].T @ kk - ((a - b) * (h0[0, 0].T @ kk) + b * vv)).max() < 1e-13


def test_undecayed_equals_reparametrised_default():
    # (a I - b k k^T) S + b k v^T = a (I - (b/a) k k^T) S + (b/a) k (a v)^T: the read-before-decay
    # order with (beta, v) is the decay-first order with (beta / alpha, alpha v)
    r = _rng(211)
    T, H, dk, dv = 40, 2, 6, 4
    q, k, v = r.normal(size=(T, H, dk)), r.normal(size=(T, H, dk)), r.normal(size=(T, H, dv))
    g = -0.5 * np.abs(r.normal(size=(T, H))); beta = r.uniform(size=(T, H))
    h0 = r.normal(size=(1, H, dk, dv))
    a = np.exp(g)
    o1, h1 = _rec()(q, k, v, g, beta, [0, T], h0=h0, undecayed=True)
    o2, h2 = _rec()(q, k, v * a[..., None], g, beta / a, [0, T], h0=h0)
    assert np.abs(o1 - o2).max() < 1e-12 * np.abs(o1).max()
    assert np.abs(h1 - h2).max() < 1e-12 * np.abs(h1).max()
    # with no decay the two orders coincide exactly; with decay they differ
    o3, _ = _rec()(q, k, v, np.zeros_like(g), beta, [0, T], h0=h0, undecayed=True)
    o4, _ = _rec()(q, k, v, np.zeros_like(g), beta, [0, T], h0=h0)
    assert np.array_equal(o3, o4)
    o5, _ = _rec()(q, k, v, g, beta, [0, T], h0=h0)
    assert np.abs(o5 - o1).max() > 1e-2


@pytest.mark.parametrize("chunk", [1, 4, 16, 64])
def test_undecayed_chunked_evaluator_equals_token_loop(chunk):
    # chunk form of the read-before-decay order: row decay e^{gamma_{r-1}} in A and W
    r = _rng(212)
    lens = [70, 3, 64, 129, 1]
    cu = np.concatenate([[0], np.cumsum(lens)])
    H, dk, dv = 2, 8, 6
    T = int(cu[-1])
    q, k, v = r.normal(size=(T, H, dk)), r.normal(size=(T, H, dk)), r.normal(size=(T, H, dv))
    g = -0.3 * np.abs(r.normal(size=(T, H))); beta = r.uniform(size=(T, H))
    g[5:9] = -9.0  # strong decay inside a chunk
    h0 = r.normal(size=(len(lens), H, dk, dv))
    kw = dict(dtype="f64", h0=h0, scale=0.8, threads=2, undecayed=True)
    o1, h1 = oracle.recurrence(q, k, v, g, beta, cu, **kw)
    o2, h2 = oracle.chunked(q, k, v, g, beta, cu, chunk=chunk, **kw)
    assert np.abs(o1 - o2).max() <= 1e-12 * np.abs(o1).max()
    assert np.abs(h1 - h2).max() <= 1e-12 * np.abs(h1).max()


def test_undecayed_decode_layer_steps_equal_packed_layer():
    r = _rng(213)
    H, dk, dv, K, T = 2, 4, 3, 4, 6
    C = 2 * H * dk + H * dv
    x, cw = r.normal(size=(T, C)), r.normal(size=(C, K))
    cs0, h0 = r.normal(size=(1, C, K - 1)), r.normal(size=(1, H, dk, dv)) * 0.3
    g = -np.abs(r.normal(size=(T, H))) * 0.3
    b = 1.0 / (1.0 + np.exp(-r.normal(size=(T, H))))
    y, _ = oracle.conv_silu(x, cw, [0, T], dtype="f64", state_in=cs0, qk_l2norm=True,
                            n_qk=2 * H * dk, head_dim=dk, eps=1e-6)
    o_ref, h_ref = oracle.recurrence(y[:, :H * dk].reshape(T, H, dk),
                                     y[:, H * dk:2 * H * dk].reshape(T, H, dk),
                                     y[:, 2 * H * dk:].reshape(T, H, dv), g, b, [0, T],
                                     dtype="f64", h0=h0, qk_l2norm=False, undecayed=True)
    cs, st = cs0, h0
    for t in range(T):
        o, cs, st = oracle.decode_layer_step(x[t:t + 1], cw, cs, g[t:t + 1], b[t:t + 1], st,
                                             dtype="f64", H=H, dk=dk, dv=dv, undecayed=True)
        assert np.abs(o[0] - o_ref[t]).max() < 1e-12
    assert np.abs(st - h_ref).max() < 1e-12


# --------------------------------------------------------------------------
# Pin sensitivity: each planted mistake must fail at least one pin.
# --------------------------------------------------------------------------

@pytest.mark.parametrize("planted", [1, 2, 3, 4],
                         ids=["retrieve_before_decay", "transposed_state", "dropped_decay",
                              "wrong_sign_delta"])
def test_pins_catch_planted_mistakes(planted):
    errs = {p.__name__: p(_rec(planted)) for p in ALL_PINS}
    assert max(errs.values()) > 1e-6, errs
