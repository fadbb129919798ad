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

``chunked_backward`` evaluates the same gradients from the chunk form of the
forward (the WY/UT regrouping of "Parallelizing Linear Transformers with the
Delta Rule over Sequence Length" and "Gated Delta Networks", Yang et al.,
2024, restated for the decay-first order), differentiated step by step; the
tests check it against the autograd gradients.
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


def _l2_rows(x, eps, on):
    """(x / |x|_eps per row, the row norms) -- the norm used by the forward."""
    n = np.sqrt((x * x).sum(-1) + eps) if on else np.ones(x.shape[0])
    return x / n[:, None], n


def chunked_backward(q, k, v, g, beta, cu_seqlens, do, dhT=None, *, h0=None,
                     scale: float = 1.0, qk_l2norm: bool = True, eps: float = 1e-6,
                     chunk: int = 64):
    """The same gradients as recurrence_backward, evaluated chunk by chunk in
    fp64 numpy: the reverse-mode derivative of the chunk form (cumulative decay
    gamma, A = strict_lower(beta_r e^{gamma_r - gamma_j} k_r.k_j), T = (I + A)^-1,
    W = T diag(beta e^gamma) K, U~ = T diag(beta) V, U = U~ - W S,
    O = diag(e^gamma) Q S + (QK^T o Gamma o lower) U,
    S' = e^{gamma_L} S + (diag(e^{gamma_L - gamma}) K)^T U), taken step by step
    backwards through each chunk, last chunk first, with the chunk-start states
    from a forward pass. It exists to check that chunk-level gradient algebra
    (the form a tensor-core backward evaluates) against autograd of the token
    loop; no kernel calls it."""
    q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
    g, beta, do = (np.asarray(x, np.float64) for x in (g, beta, do))
    cu = np.asarray(cu_seqlens, np.int64)
    T_tot, Hk, dk = q.shape
    H, dv = v.shape[1], v.shape[2]
    G = H // Hk
    N = len(cu) - 1
    dq, dkk = np.zeros_like(q), np.zeros_like(k)
    dvv, dg, db = np.zeros_like(v), np.zeros_like(g), np.zeros_like(beta)
    dh0 = np.zeros((N, H, dk, dv))
    for n in range(N):
        a, b = int(cu[n]), int(cu[n + 1])
        for h in range(H):
            hk = h // G
            Kh, nk = _l2_rows(k[a:b, hk], eps, qk_l2norm)
            Qt, nq = _l2_rows(q[a:b, hk], eps, qk_l2norm)
            Qh = scale * Qt
            V, bt, gg, dO = v[a:b, h], beta[a:b, h], g[a:b, h], do[a:b, h]
            # forward: chunk-start states
            starts = list(range(0, b - a, chunk))
            S = np.zeros((dk, dv)) if h0 is None else np.asarray(h0, np.float64)[n, h].copy()
            S_in, saved = [], []
            for c0 in starts:
                sl = slice(c0, min(c0 + chunk, b - a))
                K, Q, Vc, B, gam = Kh[sl], Qh[sl], V[sl], bt[sl], np.cumsum(gg[sl])
                L = K.shape[0]
                Gm = np.exp(gam[:, None] - gam[None, :])
                low = np.tril(np.ones((L, L)), -1)
                A = low * (B[:, None] * (K @ K.T) * Gm)
                Tm = np.linalg.inv(np.eye(L) + A)
                E = B * np.exp(gam)
                W = Tm @ (E[:, None] * K)
                Ut = Tm @ (B[:, None] * Vc)
                U = Ut - W @ S
                cK = np.exp(gam[-1] - gam)
                S_in.append(S)
                saved.append((sl, K, Q, Vc, B, gam, Gm, A, Tm, E, W, U, cK))
                S = np.exp(gam[-1]) * S + (cK[:, None] * K).T @ U
            # backward, last chunk first
            dS = np.zeros((dk, dv)) if dhT is None else np.asarray(dhT, np.float64)[n, h].copy()
            dKh, dQh = np.zeros_like(Kh), np.zeros_like(Qh)
            for S0, (sl, K, Q, Vc, B, gam, Gm, A, Tm, E, W, U, cK) in zip(S_in[::-1], saved[::-1]):
                L = K.shape[0]
                dOc = dO[sl]
                dgam = np.zeros(L)
                incl = np.tril(np.ones((L, L)))
                low = np.tril(np.ones((L, L)), -1)
                # S' = e^{gamma_L} S0 + Kt^T U, Kt = cK o K
                dSp = dS
                dS = np.exp(gam[-1]) * dSp
                dgam[-1] += np.exp(gam[-1]) * np.sum(S0 * dSp)
                dKt = U @ dSp.T
                dU = (cK[:, None] * K) @ dSp
                dK = cK[:, None] * dKt
                dc = np.sum(dKt * K, axis=1) * cK
                dgam[-1] += dc.sum()
                dgam -= dc
                # O = (e^gamma o Q) S0 + Pm U, Pm = incl o (QK^T) o Gamma
                eg = np.exp(gam)
                dS += (eg[:, None] * Q).T @ dOc
                dQ = eg[:, None] * (dOc @ S0.T)
                dgam += eg * np.sum((Q @ S0) * dOc, axis=1)
                Pm = incl * (Q @ K.T) * Gm
                dPm = incl * (dOc @ U.T)
                dU += Pm.T @ dOc
                Z = dPm * Gm * incl
                dQ += Z @ K
                dK += Z.T @ Q
                pp = dPm * Pm
                dgam += pp.sum(1)
                dgam -= pp.sum(0)
                # U = U~ - W S0
                dW = -dU @ S0.T
                dS += -W.T @ dU
                # U~ = T (B o V)
                dT = dU @ (B[:, None] * Vc).T
                TtdU = Tm.T @ dU
                dVc = B[:, None] * TtdU
                dB = np.sum(Vc * TtdU, axis=1)
                # W = T (E o K)
                dT += dW @ (E[:, None] * K).T
                TtdW = Tm.T @ dW
                dK += E[:, None] * TtdW
                dE = np.sum(K * TtdW, axis=1)
                dB += dE * eg
                dgam += dE * E
                # T = (I + A)^-1, A strictly lower
                dA = low * (-(Tm.T @ dT @ Tm.T))
                # A = low o (B_r (K K^T) o Gamma)
                Y = dA * Gm * B[:, None]
                dK += Y @ K + Y.T @ K
                dB += np.sum(dA * Gm * (K @ K.T), axis=1)
                aa = dA * A
                dgam += aa.sum(1)
                dgam -= aa.sum(0)
                # gamma = cumsum(g) within the chunk
                dg[a:b, h][sl] = np.cumsum(dgam[::-1])[::-1]
                db[a:b, h][sl] = dB
                dvv[a:b, h][sl] = dVc
                dKh[sl] += dK
                dQh[sl] += dQ
            dh0[n, h] = dS
            # through the L2 norms (and the query scale)
            dQt = scale * dQh
            if qk_l2norm:
                dkk[a:b, hk] += (dKh - Kh * np.sum(Kh * dKh, 1, keepdims=True)) / nk[:, None]
                dq[a:b, hk] += (dQt - Qt * np.sum(Qt * dQt, 1, keepdims=True)) / nq[:, None]
            else:
                dkk[a:b, hk] += dKh
                dq[a:b, hk] += dQt
    return dq, dkk, dvv, dg, db, dh0
