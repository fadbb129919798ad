"""Gradients of the gated delta rule -- TEST INFRASTRUCTURE ONLY (part of the
CPU oracle; the CUDA library never imports it).

The forward here is the token loop of the Qwen3.5-MoE source walkthrough,
section 4.3, restated with plain PyTorch CPU ops in fp64 (the same steps as
``gdn_oracle.c``'s recurrence, which the tests check it against):

    k^ = L2(k_t), q^ = scale * L2(q_t)     (L2(x) = x / sqrt(sum x^2 + eps))
    S <- exp(g_t) S;  m = S^T k^;  delta = beta_t (v_t - m);
    S <- S + k^ delta^T;  o_t = S^T q^

and the gradients are torch.autograd's of that function: for upstream
gradients dO [T, H, dv] and dS_T [N, H, dk, dv] it returns dq, dk, dv, dg,
dbeta and dh0 -- the vector-Jacobian product of the definition, with nothing
reordered or fused. Value head h reads q, k head h // (H // Hk); the q, k
gradients of a shared head are the sums over its value heads.
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch


def _f64(a) -> torch.Tensor:
    return torch.as_tensor(np.asarray(a, dtype=np.float64))


def _forward(q, k, v, g, beta, cu, h0, *, scale, qk_l2norm, eps):
    """o [T, H, dv], hT [N, H, dk, dv] as torch fp64 tensors (autograd-tracked)."""
    T, Hk, dk = q.shape
    H, dv = v.shape[1], v.shape[2]
    G = H // Hk
    N = len(cu) - 1
    outs = [None] * T
    finals = []
    for n in range(N):
        heads = []
        for h in range(H):
            hk = h // G
            S = h0[n, h] if h0 is not None else torch.zeros(dk, dv, dtype=torch.float64)
            for t in range(int(cu[n]), int(cu[n + 1])):
                qt, kt = q[t, hk], k[t, hk]
                if qk_l2norm:
                    qt = qt / torch.sqrt((qt * qt).sum() + eps)
                    kt = kt / torch.sqrt((kt * kt).sum() + eps)
                qt = qt * scale
                S = torch.exp(g[t, h]) * S
                m = S.T @ kt
                delta = beta[t, h] * (v[t, h] - m)
                S = S + torch.outer(kt, delta)
                if outs[t] is None:
                    outs[t] = [None] * H
                outs[t][h] = S.T @ qt
            heads.append(S)
        finals.append(torch.stack(heads))
    o = torch.stack([torch.stack(row) for row in outs]) if T > 0 else torch.zeros(0, H, dv,
                                                                                   dtype=torch.float64)
    return o, torch.stack(finals)


def forward(q, k, v, g, beta, cu_seqlens, *, h0=None, scale: float = 1.0,
            qk_l2norm: bool = True, eps: float = 1e-6):
    """The torch restatement's forward, as numpy fp64 (o, hT)."""
    with torch.no_grad():
        o, hT = _forward(_f64(q), _f64(k), _f64(v), _f64(g), _f64(beta),
                         np.asarray(cu_seqlens, np.int64), None if h0 is None else _f64(h0),
                         scale=scale, qk_l2norm=qk_l2norm, eps=eps)
    return o.numpy(), hT.numpy()


def recurrence_backward(q, k, v, g, beta, cu_seqlens, do, dhT=None, *, h0=None,
                        scale: float = 1.0, qk_l2norm: bool = True, eps: float = 1e-6):
    """(dq, dk, dv, dg, dbeta, dh0) in fp64 for upstream gradients do [T, H, dv]
    and dhT [N, H, dk, dv] (None: zero). dh0 is returned even when h0 is None
    (the gradient with respect to a zero initial state)."""
    cu = np.asarray(cu_seqlens, np.int64)
    ts = [_f64(x).requires_grad_(True) for x in (q, k, v, g, beta)]
    N, H = len(cu) - 1, v.shape[1]
    dk_, dv_ = q.shape[2], v.shape[2]
    h0t = (_f64(h0) if h0 is not None else torch.zeros(N, H, dk_, dv_, dtype=torch.float64))
    h0t.requires_grad_(True)
    o, hT = _forward(*ts, cu, h0t, scale=scale, qk_l2norm=qk_l2norm, eps=eps)
    outs, grads = [o], [_f64(do)]
    if dhT is not None:
        outs.append(hT)
        grads.append(_f64(dhT))
    res = torch.autograd.grad(outs, ts + [h0t], grads, allow_unused=True)
    return tuple(np.zeros(x.shape) if r is None else r.numpy()
                 for r, x in zip(res, ts + [h0t]))
