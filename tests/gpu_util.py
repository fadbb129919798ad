"""Helpers shared by the GPU parity tests: move the seeded inputs to the
device, run the library, run the oracle on the same bytes, compare."""
from __future__ import annotations

import numpy as np
import torch

import gated_deltanet_linear_silu_b200 as gdn
import oracle

DEV = torch.device("cuda", 0)
TOL_F32 = 1e-4   # fp32 inputs, fp32 arithmetic
TOL_BF16 = 2e-2  # bf16 inputs/outputs, fp32 accumulation


def err(x, ref) -> float:
    """max |x - ref| / max |ref| (max-abs-normalised error)."""
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    assert np.isfinite(x).all(), "non-finite values"
    return float(np.abs(x - ref).max() / max(np.abs(ref).max(), 1e-30))


def dev_tensor(a: np.ndarray, kind: str) -> torch.Tensor:
    """kind 'bf16': a holds uint16 bf16 bits; otherwise a float array."""
    if kind == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(DEV).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV)


def host(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


def tol(kind: str) -> float:
    return TOL_BF16 if kind == "bf16" else TOL_F32


def prefill_gpu(P, *, algo="auto", chunk=None, h0=None, give_host_cu=True, undecayed=False):
    kind = P.dtype
    q, k, v = (dev_tensor(a, kind) for a in (P.q, P.k, P.v))
    g, beta = dev_tensor(P.g, "f32"), dev_tensor(P.beta, "f32")
    cu = torch.from_numpy(P.cu_seqlens.astype(np.int32)).to(DEV)
    h0 = P.h0 if h0 is None else h0
    h0d = None if h0 is None else dev_tensor(h0, "f32")
    o, hT = gdn.prefill(q, k, v, g, beta, cu, initial_state=h0d, scale=P.scale,
                        qk_l2norm=P.qk_l2norm, eps=P.eps, chunk=chunk or P.chunk, algo=algo,
                        undecayed=undecayed,
                        cu_seqlens_host=torch.from_numpy(P.cu_seqlens.astype(np.int32))
                        if give_host_cu else None)
    gdn.check_device_status(DEV)
    return host(o), host(hT)


def prefill_oracle(P, h0=None, undecayed=False):
    h0 = P.h0 if h0 is None else h0
    return oracle.recurrence(P.q, P.k, P.v, P.g, P.beta, P.cu_seqlens, dtype=P.dtype, h0=h0,
                             scale=P.scale, qk_l2norm=P.qk_l2norm, eps=P.eps, undecayed=undecayed)


def oracle_unit(P, n: int, h: int):
    """Oracle on one (sequence, head) of a packed problem: (o [T_n, dv], hT [dk, dv])."""
    a, b = int(P.cu_seqlens[n]), int(P.cu_seqlens[n + 1])
    sl = lambda x, i=h: np.ascontiguousarray(x[a:b, i:i + 1])
    hk = h // (P.H // P.Hk)  # the q, k head of value head h
    h0 = None if P.h0 is None else P.h0[n:n + 1, h:h + 1]
    o, hT = oracle.recurrence(sl(P.q, hk), sl(P.k, hk), sl(P.v), sl(P.g), sl(P.beta), [0, b - a],
                              dtype=P.dtype, h0=h0, scale=P.scale, qk_l2norm=P.qk_l2norm,
                              eps=P.eps, threads=1)
    return o[:, 0], hT[0, 0]


def oracle_seq(P, n: int):
    """Oracle on every head of one sequence of a packed problem:
    (o [T_n, H, dv], hT [H, dk, dv]); threads over heads."""
    a, b = int(P.cu_seqlens[n]), int(P.cu_seqlens[n + 1])
    sl = lambda x: np.ascontiguousarray(x[a:b])
    h0 = None if P.h0 is None else P.h0[n:n + 1]
    o, hT = oracle.recurrence(sl(P.q), sl(P.k), sl(P.v), sl(P.g), sl(P.beta), [0, b - a],
                              dtype=P.dtype, h0=h0, scale=P.scale, qk_l2norm=P.qk_l2norm,
                              eps=P.eps)
    return o, hT[0]


def longest_first(cu_seqlens) -> np.ndarray:
    """Sequence indices in the order the persistent prefill kernels take them:
    longest first, ties by index."""
    lens = np.diff(np.asarray(cu_seqlens, np.int64))
    return np.lexsort((np.arange(lens.size), -lens))
