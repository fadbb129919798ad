"""Seeded synthetic inputs for the Gated DeltaNet token mixer.

This module only draws random numbers and encodes them (bf16 rounding). It
holds none of the mixer's arithmetic: no convolution, no SiLU, no L2 norm, no
delta-rule recurrence. Both the CUDA path and the CPU oracle consume the exact
bytes produced here, so any disagreement between them is arithmetic, not data.

Every tensor is drawn from its own numpy PCG64 stream, seeded by
``(workload id, tensor tag, index)`` through ``numpy.random.SeedSequence``, so a
single sequence (or a single decode step) can be regenerated on its own when a
parity test samples it. The draw recipes follow the five workloads of the
token mixer (Qwen3.5 linear-attention layer shapes, "7.6 Qwen3.5" config table:
16 key/value heads, head dim 128, conv kernel 4):

* ``tiny_fp32``    1 x 64 tokens, 2 heads, d=16, fp32 q/k/v ~ N(0,1),
                   beta = sigmoid(N(0,1)), g = -softplus(N(0,1)), zero state.
* ``layer_0p8b``   one 0.8B-shaped layer prefill: x[4096,1024] ~ N(0,1) (bf16),
                   projections std 0.02 (bf16), mixed_qkv = bf16(x @ W_qkv) with
                   fp32 accumulation, conv taps ~ N(0, 0.5) (bf16),
                   beta = sigmoid(x @ w_beta), g = -softplus(x @ w_a) * exp(A_log),
                   A_log ~ U(0, 2.7) per head.
* ``long_prefill`` 8 x 16384 tokens, 16 heads, d=128, bf16 q/k/v ~ N(0,1),
                   beta = sigmoid(N(0,1)), g = -0.1 * softplus(N(0,1)).
* ``decode``       256 sequences x 16 heads, d=128, state ~ N(0, 0.1) fp32,
                   per step bf16 q/k/v ~ N(0,1), beta = sigmoid(N(0,1)),
                   g = -softplus(N(0,1)); 100 steps.
* ``varlen``       64 lengths ~ U[256, 32768] (inclusive), packed; q/k/v/beta/g
                   as ``long_prefill``; initial state ~ N(0, 0.1) fp32.
* ``grouped``      grouped value heads (the config table lists the value-head
                   and key-head counts separately): 8 x 8192 tokens, 32 value
                   heads on 16 q/k heads, d=128, draws as ``long_prefill``.

q and k are drawn raw; the per-head L2 normalisation the workloads call for is
part of the computed path (both sides apply it), not of the data. The gate
parametrisation (sigmoid / softplus) is input synthesis: the mixer consumes
beta and g = log(alpha) as given.
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import os
from typing import Optional

import numpy as np

# Workload ids (seed roots).
TINY_FP32 = 0
LAYER_0P8B = 1
LONG_PREFILL = 2
DECODE = 3
VARLEN = 4
GROUPED = 5

WORKLOAD_NAMES = {
    TINY_FP32: "tiny_fp32",
    LAYER_0P8B: "layer_0p8b",
    LONG_PREFILL: "long_prefill",
    DECODE: "decode",
    VARLEN: "varlen",
    GROUPED: "grouped",
}

# Tensor tags of the seed tree (stable: changing one changes every draw).
_TAG = {"q": 1, "k": 2, "v": 3, "beta": 4, "g": 5, "h0": 6, "x": 7, "wqkv": 8,
        "convw": 9, "wbeta": 10, "wa": 11, "alog": 12, "lens": 13, "state": 14,
        "convstate": 15}


def rng(workload: int, tag: str, index: int = 0) -> np.random.Generator:
    """Independent PCG64 stream for (workload, tensor tag, index)."""
    return np.random.default_rng(np.random.SeedSequence([workload, _TAG[tag], index]))


# ---------------------------------------------------------------------------
# bf16 encoding (round to nearest even), stored as uint16 bit patterns.
# ---------------------------------------------------------------------------

def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return uint16 bits."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    rounded = (u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal(r: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    x = r.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return (1.0 / (1.0 + np.exp(-x.astype(np.float64)))).astype(np.float32)


def _softplus(x: np.ndarray) -> np.ndarray:
    x = x.astype(np.float64)
    return (np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))).astype(np.float32)


# ---------------------------------------------------------------------------
# Workload containers
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class Prefill:
    """Packed prefill batch. q/k are [T_tot, Hk, dk], v [T_tot, H, dv] (uint16
    bf16 bits or float32), g/beta [T_tot, H] float32, cu_seqlens [N+1] int32,
    h0 [N,H,dk,dv] float32 or None. Hk = H unless value heads are grouped."""
    name: str
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    g: np.ndarray
    beta: np.ndarray
    cu_seqlens: np.ndarray
    h0: Optional[np.ndarray]
    dtype: str          # "bf16" or "f32"
    H: int
    dk: int
    dv: int
    chunk: int = 64
    scale: float = 1.0
    qk_l2norm: bool = True
    eps: float = 1e-6

    @property
    def N(self) -> int:
        return int(self.cu_seqlens.shape[0] - 1)

    @property
    def T_tot(self) -> int:
        return int(self.cu_seqlens[-1])

    @property
    def Hk(self) -> int:
        return int(self.q.shape[1])


@dataclasses.dataclass
class Layer:
    """One 0.8B-shaped layer prefill: the conv stage input plus gates.
    mixed_qkv [T, 6144] bf16 bits, conv_w [6144, 4] bf16 bits, g/beta [T,16]."""
    name: str
    mixed_qkv: np.ndarray
    conv_w: np.ndarray
    g: np.ndarray
    beta: np.ndarray
    cu_seqlens: np.ndarray
    H: int
    dk: int
    dv: int
    K: int = 4
    chunk: int = 64
    eps: float = 1e-6

    @property
    def C(self) -> int:
        return int(self.mixed_qkv.shape[1])

    @property
    def N(self) -> int:
        return int(self.cu_seqlens.shape[0] - 1)

    @property
    def T_tot(self) -> int:
        return int(self.cu_seqlens[-1])


# ---------------------------------------------------------------------------
# Generators
# ---------------------------------------------------------------------------

def tiny_fp32() -> Prefill:
    T, H, d = 64, 2, 16
    w = TINY_FP32
    q = _normal(rng(w, "q"), (T, H, d))
    k = _normal(rng(w, "k"), (T, H, d))
    v = _normal(rng(w, "v"), (T, H, d))
    beta = _sigmoid(_normal(rng(w, "beta"), (T, H)))
    g = -_softplus(_normal(rng(w, "g"), (T, H)))
    cu = np.array([0, T], dtype=np.int32)
    return Prefill("tiny_fp32", q, k, v, g, beta, cu, None, "f32", H, d, d)


def layer_0p8b(T: int = 4096, emb: int = 1024, H: int = 16, d: int = 128) -> Layer:
    w = LAYER_0P8B
    C = 3 * H * d  # conv_dim = 2 * key_dim + value_dim
    x = bf16_bits_to_f32(to_bf16_bits(_normal(rng(w, "x"), (T, emb))))
    wqkv = bf16_bits_to_f32(to_bf16_bits(_normal(rng(w, "wqkv"), (emb, C), 0.02)))
    mixed = to_bf16_bits(x @ wqkv)
    conv_w = to_bf16_bits(_normal(rng(w, "convw"), (C, 4), 0.5))
    wb = bf16_bits_to_f32(to_bf16_bits(_normal(rng(w, "wbeta"), (emb, H), 0.02)))
    wa = bf16_bits_to_f32(to_bf16_bits(_normal(rng(w, "wa"), (emb, H), 0.02)))
    a_log = rng(w, "alog").uniform(0.0, 2.7, size=H).astype(np.float32)
    beta = _sigmoid(x @ wb)
    g = (-_softplus(x @ wa) * np.exp(a_log.astype(np.float64))).astype(np.float32)
    cu = np.array([0, T], dtype=np.int32)
    return Layer("layer_0p8b", mixed, conv_w, np.ascontiguousarray(g),
                 np.ascontiguousarray(beta), cu, H, d, d)


def sequence_tensors(workload: int, n: int, T: int, H: int, d: int,
                     g_scale: float, Hk: Optional[int] = None) -> dict:
    """q/k/v (bf16 bits), beta, g of sequence n of a packed prefill workload
    (q, k with Hk heads, default H)."""
    Hk = H if Hk is None else Hk
    q = to_bf16_bits(_normal(rng(workload, "q", n), (T, Hk, d)))
    k = to_bf16_bits(_normal(rng(workload, "k", n), (T, Hk, d)))
    v = to_bf16_bits(_normal(rng(workload, "v", n), (T, H, d)))
    beta = _sigmoid(_normal(rng(workload, "beta", n), (T, H)))
    g = (-_softplus(_normal(rng(workload, "g", n), (T, H))) * np.float32(g_scale)).astype(np.float32)
    return {"q": q, "k": k, "v": v, "beta": beta, "g": g}


def varlen_lengths(N: int = 64, lo: int = 256, hi: int = 32768) -> np.ndarray:
    return rng(VARLEN, "lens").integers(lo, hi, size=N, endpoint=True).astype(np.int64)


def _packed(workload: int, name: str, lengths, H: int, d: int, g_scale: float,
            h0: Optional[np.ndarray], Hk: Optional[int] = None) -> Prefill:
    Hk = H if Hk is None else Hk
    lengths = np.asarray(lengths, dtype=np.int64)
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(lengths)
    T_tot = int(cu[-1])
    q = np.empty((T_tot, Hk, d), np.uint16)
    k = np.empty_like(q)
    v = np.empty((T_tot, H, d), np.uint16)
    beta = np.empty((T_tot, H), np.float32)
    g = np.empty_like(beta)

    def fill(n):  # numpy releases the GIL while drawing, so sequences fill in parallel
        s = sequence_tensors(workload, n, int(lengths[n]), H, d, g_scale, Hk)
        a, b = int(cu[n]), int(cu[n + 1])
        q[a:b], k[a:b], v[a:b], beta[a:b], g[a:b] = s["q"], s["k"], s["v"], s["beta"], s["g"]

    with concurrent.futures.ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
        list(ex.map(fill, range(len(lengths))))
    return Prefill(name, q, k, v, g, beta, cu.astype(np.int32), h0, "bf16", H, d, d)


def long_prefill(N: int = 8, T: int = 16384, H: int = 16, d: int = 128) -> Prefill:
    return _packed(LONG_PREFILL, "long_prefill", [T] * N, H, d, 0.1, None)


def grouped_prefill(N: int = 8, T: int = 8192, H: int = 32, Hk: int = 16, d: int = 128) -> Prefill:
    return _packed(GROUPED, "grouped", [T] * N, H, d, 0.1, None, Hk)


def initial_state(workload: int, n: int, H: int, dk: int, dv: int, std: float = 0.1) -> np.ndarray:
    return _normal(rng(workload, "h0", n), (H, dk, dv), std)


def varlen(N: int = 64, H: int = 16, d: int = 128, lo: int = 256, hi: int = 32768,
           lengths=None) -> Prefill:
    if lengths is None:
        lengths = varlen_lengths(N, lo, hi)
    h0 = np.stack([initial_state(VARLEN, n, H, d, d) for n in range(len(lengths))])
    return _packed(VARLEN, "varlen", lengths, H, d, 0.1, h0)


@dataclasses.dataclass
class DecodeStep:
    q: np.ndarray      # [N,H,dk] bf16 bits
    k: np.ndarray
    v: np.ndarray      # [N,H,dv]
    g: np.ndarray      # [N,H] f32
    beta: np.ndarray   # [N,H] f32


def decode_state(N: int = 256, H: int = 16, d: int = 128) -> np.ndarray:
    return _normal(rng(DECODE, "state"), (N, H, d, d), 0.1)


def decode_step(step: int, N: int = 256, H: int = 16, d: int = 128) -> DecodeStep:
    w = DECODE
    q = to_bf16_bits(_normal(rng(w, "q", step), (N, H, d)))
    k = to_bf16_bits(_normal(rng(w, "k", step), (N, H, d)))
    v = to_bf16_bits(_normal(rng(w, "v", step), (N, H, d)))
    beta = _sigmoid(_normal(rng(w, "beta", step), (N, H)))
    g = -_softplus(_normal(rng(w, "g", step), (N, H)))
    return DecodeStep(q, k, v, g, beta)


def random_prefill(seed: int, lengths, H: int, dk: int, dv: int, dtype: str = "bf16",
                   g_scale: float = 1.0, with_h0: bool = False, h0_std: float = 0.1,
                   chunk: int = 64, qk_l2norm: bool = True, scale: float = 1.0,
                   Hk: Optional[int] = None) -> Prefill:
    """A small packed prefill problem for parity tests (any shapes); Hk < H
    gives grouped value heads (q, k with Hk heads)."""
    Hk = H if Hk is None else Hk
    r = np.random.default_rng(np.random.SeedSequence([1000, seed]))
    lengths = np.asarray(lengths, dtype=np.int64)
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(lengths)
    T_tot = int(cu[-1])
    q = _normal(r, (T_tot, Hk, dk))
    k = _normal(r, (T_tot, Hk, dk))
    v = _normal(r, (T_tot, H, dv))
    beta = _sigmoid(_normal(r, (T_tot, H)))
    g = (-_softplus(_normal(r, (T_tot, H))) * np.float32(g_scale)).astype(np.float32)
    h0 = _normal(r, (len(lengths), H, dk, dv), h0_std) if with_h0 else None
    if dtype == "bf16":
        q, k, v = to_bf16_bits(q), to_bf16_bits(k), to_bf16_bits(v)
    return Prefill(f"random{seed}", q, k, v, g, beta, cu.astype(np.int32), h0, dtype,
                   H, dk, dv, chunk=chunk, qk_l2norm=qk_l2norm, scale=scale)


def random_mixed(seed: int, lengths, C: int, K: int = 4, dtype: str = "bf16",
                 w_std: float = 0.5, with_state: bool = False):
    """Random conv-stage input (x [T_tot, C], taps [C, K], optional conv state
    [N, C, K-1]) for conv parity tests."""
    r = np.random.default_rng(np.random.SeedSequence([2000, seed]))
    lengths = np.asarray(lengths, dtype=np.int64)
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(lengths)
    x = _normal(r, (int(cu[-1]), C))
    w = _normal(r, (C, K), w_std)
    st = _normal(r, (len(lengths), C, K - 1)) if with_state else None
    if dtype == "bf16":
        x, w = to_bf16_bits(x), to_bf16_bits(w)
        if st is not None:
            st = to_bf16_bits(st)
    return x, w, cu.astype(np.int32), st
