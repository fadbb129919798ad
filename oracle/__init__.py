"""CPU oracle for the Gated DeltaNet token mixer -- TEST INFRASTRUCTURE ONLY.

A plain fp64 restatement (C, threads over (sequence, head)) of what the mixer
computes, used by the tests, the smoke check and the benchmark's CPU baseline.
The CUDA library never imports or links it, and it shares no code with it.

The recurrence, chunked evaluator and conv marshal numpy arrays into the C
library built from ``gdn_oracle.c`` (see that file's header for the sources
each step follows). The gated RMSNorm output is plain numpy in fp64, and the
decode layer step is the composition of the conv, the recurrence and that norm.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

from . import build as _build

_F32, _BF16, _F64 = 0, 1, 2
_lib = None


def _rec_argtypes():
    vp, i32, f64, i64p = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
    return [vp, vp, vp, i32, vp, vp, i32, i64p, i32, i32, i32, i32, i32, f64, i32, f64, i32, vp,
            i32, vp, vp, i32]


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        vp, i32, f64, i64p = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        L.gdn_oracle_recurrence.argtypes = _rec_argtypes()
        L.gdn_oracle_recurrence.restype = i32
        L.gdn_oracle_chunked.argtypes = [vp, vp, vp, i32, vp, vp, i32, i64p, i32, i32, i32, i32,
                                         i32, f64, i32, f64, i32, vp, i32, vp, vp, i32, i32]
        L.gdn_oracle_chunked.restype = i32
        L.gdn_oracle_conv_silu.argtypes = [vp, i32, vp, i32, i64p, i32, i32, i32, vp, i32, vp,
                                           i32, i32, i32, i32, f64, vp, i32]
        L.gdn_oracle_conv_silu.restype = i32
        _lib = L
    return _lib


def _pincheck_entry():
    """The recurrence with a planted mistake, from the pin-check build of the
    same source (used only by the pin-sensitivity test)."""
    L = ctypes.CDLL(_build.build_pincheck())
    fn = L.gdn_oracle_recurrence_planted
    fn.argtypes = _rec_argtypes() + [ctypes.c_int]
    fn.restype = ctypes.c_int
    return fn


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def _arr(a: np.ndarray, kind: str):
    """(contiguous array, dtype code). kind 'bf16' means uint16 bit patterns."""
    if kind == "bf16":
        a = np.ascontiguousarray(a, dtype=np.uint16)
        return a, _BF16
    if a.dtype == np.float64:
        return np.ascontiguousarray(a), _F64
    return np.ascontiguousarray(a, dtype=np.float32), _F32


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def recurrence(q, k, v, g, beta, cu_seqlens, *, dtype: str, h0=None, scale: float = 1.0,
               qk_l2norm: bool = True, eps: float = 1e-6, threads: Optional[int] = None,
               want_o: bool = True, undecayed: bool = False, _planted: int = 0):
    """Token-by-token gated delta rule in fp64.

    Default order (Qwen3.5-MoE source walkthrough, 4.3): decay the state, then
    read kv_mem = S^T k. undecayed=True takes the order of "7.6 Qwen3.5:
    linear-attention hybrid", 7.6.2: kv_mem is read from S_{t-1} before the
    decay, S_t = alpha S_{t-1} + k [beta (v - S_{t-1}^T k)]^T.

    q,k [T,Hk,dk], v [T,H,dv] (uint16 bf16 bits when dtype=='bf16', else
    float), g/beta [T,H], cu_seqlens [N+1], h0 [N,H,dk,dv] or None.
    Value head h reads q, k head h // (H // Hk) (grouped value heads; Hk == H
    is the plain layer).
    Returns (o [T,H,dv] float64 or None, hT [N,H,dk,dv] float64).
    `_planted` (1..4) is for the pin-sensitivity test only: it runs the
    pin-check build with that deliberate mistake.
    """
    T, Hk, dk = q.shape
    H, dv = v.shape[1], v.shape[2]
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int64)
    N = cu.shape[0] - 1
    q, dt = _arr(q, dtype)
    k, _ = _arr(k, dtype)
    v, _ = _arr(v, dtype)
    g, gdt = _arr(np.asarray(g), "f")
    beta = np.ascontiguousarray(beta, dtype=g.dtype)
    h0a, h0dt = (None, _F64) if h0 is None else _arr(np.asarray(h0), "f")
    hT = np.empty((N, H, dk, dv), np.float64)
    o = np.empty((T, H, dv), np.float64) if want_o else None
    args = [_ptr(q), _ptr(k), _ptr(v), dt, _ptr(g), _ptr(beta), gdt, _ptr(cu), N, H, Hk, dk, dv,
            float(scale), int(qk_l2norm), float(eps), int(undecayed), _ptr(h0a), h0dt, _ptr(hT),
            _ptr(o), threads or default_threads()]
    if _planted:
        rc = _pincheck_entry()(*args, int(_planted))
    else:
        rc = lib().gdn_oracle_recurrence(*args)
    if rc != 0:
        raise ValueError("oracle recurrence: bad arguments")
    return o, hT


def chunked(q, k, v, g, beta, cu_seqlens, *, dtype: str, chunk: int, h0=None,
            scale: float = 1.0, qk_l2norm: bool = True, eps: float = 1e-6,
            threads: Optional[int] = None, undecayed: bool = False):
    """fp64 chunkwise (UT-transform) evaluation of the same recurrence; used
    only to check that the chunk algebra equals the token loop."""
    T, Hk, dk = q.shape
    H, dv = v.shape[1], v.shape[2]
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int64)
    N = cu.shape[0] - 1
    q, dt = _arr(q, dtype)
    k, _ = _arr(k, dtype)
    v, _ = _arr(v, dtype)
    g, gdt = _arr(np.asarray(g), "f")
    beta = np.ascontiguousarray(beta, dtype=g.dtype)
    h0a, h0dt = (None, _F64) if h0 is None else _arr(np.asarray(h0), "f")
    hT = np.empty((N, H, dk, dv), np.float64)
    o = np.empty((T, H, dv), np.float64)
    rc = lib().gdn_oracle_chunked(
        _ptr(q), _ptr(k), _ptr(v), dt, _ptr(g), _ptr(beta), gdt, _ptr(cu), N, H, Hk, dk, dv,
        float(scale), int(qk_l2norm), float(eps), int(undecayed), _ptr(h0a), h0dt, _ptr(hT),
        _ptr(o), int(chunk), threads or default_threads())
    if rc != 0:
        raise ValueError("oracle chunked: bad arguments")
    return o, hT


def conv_silu(x, w, cu_seqlens, *, dtype: str, state_in=None, apply_silu: bool = True,
              qk_l2norm: bool = False, n_qk: int = 0, head_dim: int = 128, eps: float = 1e-6,
              threads: Optional[int] = None):
    """Causal depthwise conv (+SiLU, + per-head L2 norm of the first n_qk
    channels) over packed sequences, fp64.

    x [T,C], w [C,K], state_in [N,C,K-1] or None (same encoding as x).
    Returns (y [T,C] float64, state_out [N,C,K-1] float64).
    """
    T, C = x.shape
    K = w.shape[1]
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int64)
    N = cu.shape[0] - 1
    x, dt = _arr(x, dtype)
    w, wdt = _arr(w, dtype)
    st, sdt = (None, _F64) if state_in is None else _arr(state_in, dtype)
    y = np.empty((T, C), np.float64)
    st_out = np.empty((N, C, K - 1), np.float64)
    rc = lib().gdn_oracle_conv_silu(
        _ptr(x), dt, _ptr(w), wdt, _ptr(cu), N, C, K, _ptr(st), sdt, _ptr(st_out),
        int(apply_silu), int(qk_l2norm), int(n_qk), int(head_dim), float(eps), _ptr(y),
        threads or default_threads())
    if rc != 0:
        raise ValueError("oracle conv: bad arguments")
    return y, st_out


def _to_f64(a: np.ndarray, kind: str) -> np.ndarray:
    """Inputs as float64; kind 'bf16' decodes uint16 bit patterns exactly."""
    if kind == "bf16":
        b = np.ascontiguousarray(a, dtype=np.uint16).astype(np.uint32) << 16
        return b.view(np.float32).astype(np.float64)
    return np.asarray(a, dtype=np.float64)


def gated_rmsnorm(y, z, w, *, dtype: str, eps: float = 1e-6):
    """Output gate of the linear-attention layer ("Qwen3.5 ... linear-attention
    hybrid", 7.6.2, gated RMSNorm output; RMSNorm as in 7.6.3):
        out = y / sqrt(mean(y^2) + eps) * w * SiLU(z),   SiLU(z) = z / (1 + e^-z)
    over the last axis (one head's d_v values), in fp64. The scale vector w is
    applied as given (a caller with zero-centred parameters passes 1 + w).
    y, z [..., dv] in `dtype` encoding, w [dv] float. Returns float64."""
    y = _to_f64(y, dtype)
    z = _to_f64(z, dtype)
    w = np.asarray(w, dtype=np.float64)
    ms = np.mean(y * y, axis=-1, keepdims=True)
    return y / np.sqrt(ms + eps) * w * (z / (1.0 + np.exp(-z)))


def decode_layer_step(x, conv_w, conv_state, g, beta, state, *, dtype: str, H: int, dk: int,
                      dv: int, z=None, norm_w=None, norm_eps: float = 1e-6, scale: float = 1.0,
                      qk_l2norm: bool = True, eps: float = 1e-6, Hk: Optional[int] = None,
                      undecayed: bool = False):
    """One decode token of the whole mixer per sequence: the conv update over the
    fused [q | k | v] channels from the conv state (then SiLU and the per-head L2
    norm of q and k), one step of the gated delta rule from `state`, and, when z
    is given, the gated RMSNorm output. Composed from `conv_silu`, `recurrence`
    and `gated_rmsnorm`, each run as documented there.

    x [N, C] (C = 2 Hk dk + H dv; Hk key heads, default H), conv_w [C, K],
    conv_state [N, C, K-1] in `dtype` encoding; g, beta [N, H]; state
    [N, H, dk, dv] float.
    Returns (o [N, H, dv], new conv state [N, C, K-1], new state [N, H, dk, dv]),
    all float64."""
    Hk = H if Hk is None else Hk
    N, C = x.shape
    cu = np.arange(N + 1, dtype=np.int64)
    y, cs = conv_silu(x, conv_w, cu, dtype=dtype, state_in=conv_state, qk_l2norm=qk_l2norm,
                      n_qk=2 * Hk * dk, head_dim=dk, eps=eps, threads=1)
    q = y[:, :Hk * dk].reshape(N, Hk, dk)
    k = y[:, Hk * dk:2 * Hk * dk].reshape(N, Hk, dk)
    v = y[:, 2 * Hk * dk:].reshape(N, H, dv)
    o, hT = recurrence(q, k, v, np.asarray(g, np.float64), np.asarray(beta, np.float64), cu,
                       dtype="f64", h0=np.asarray(state, np.float64), scale=scale,
                       qk_l2norm=False, threads=1, undecayed=undecayed)
    if z is not None:  # o is already fp64; z arrives in the inputs' encoding
        o = gated_rmsnorm(o, _to_f64(z, dtype), norm_w, dtype="f64", eps=norm_eps)
    return o, cs, hT
