"""Gated DeltaNet token mixer on B200 (sm_100a): Python binding of libgdn.so.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in include/gdn.h. PyTorch supplies device
memory and the current stream. There is no CPU fallback: if libgdn.so has not
been built (``python -m gated_deltanet_linear_silu_b200.build``) every call
raises.

Operations (the Qwen3.5 linear-attention layer's token mixer):
  conv_silu     causal depthwise conv1d (k <= 4) + SiLU over [q | k | v]
                channels, optional per-head L2 norm of q and k, conv state.
  prefill       chunked gated delta rule over packed sequences (cu_seqlens),
                optional initial state, fp32 final state.
  decode_step   one token per sequence, fp32 state updated in place.
  decode_layer_step  the whole mixer for one decode token (conv update, SiLU,
                L2 norm, recurrent step, optional gated RMSNorm) in one kernel.
  gated_rmsnorm the gated RMSNorm output for prefill outputs.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn.so")
ABI_VERSION = 205  # gdn_version() of the C ABI these argument lists describe

GDN_F32, GDN_BF16 = 0, 1
ALGOS = {"auto": 0, "simt": 1, "tensor": 2}
STATUS = {0: "GDN_OK", 1: "GDN_ERR_INVALID_ARG", 2: "GDN_ERR_UNSUPPORTED",
          3: "GDN_ERR_WORKSPACE", 4: "GDN_ERR_CUDA", 5: "GDN_ERR_TIMEOUT"}

_lib = None


class GDNError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


def lib() -> ctypes.CDLL:
    """The loaded libgdn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m gated_deltanet_linear_silu_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                                 ctypes.c_size_t)
        L.gdn_conv_silu.argtypes = [vp, i32, vp, vp, i32, i64, i32, i32, vp, vp, i32, i32, i32, f32,
                                    vp, vp]
        L.gdn_conv_silu.restype = i32
        L.gdn_prefill_workspace_size.argtypes = [i32, i64, i32, i32, i32, i32]
        L.gdn_prefill_workspace_size.restype = sz
        L.gdn_prefill.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32,
                                  i64, i64, i64, f32, i32, f32, i32, i32, vp, vp, vp, vp, sz, i32,
                                  vp]
        L.gdn_prefill.restype = i32
        L.gdn_prefill_gated.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, i32, i64, i32, i32, i32,
                                        i32, i64, i64, i64, f32, i32, f32, i32, i32, vp, vp, vp, vp,
                                        vp, f32, vp, sz, i32, vp]
        L.gdn_prefill_gated.restype = i32
        L.gdn_prefill_layer.argtypes = [vp, vp, i32, vp, vp, i32, vp, vp, vp, vp, i32, i64, i32, i32,
                                        i32, i32, f32, i32, f32, i32, vp, vp, vp, vp, vp, f32, vp, sz,
                                        vp]
        L.gdn_prefill_layer.restype = i32
        L.gdn_prefill_layer_workspace_size.argtypes = [i32, i64, i32, i32, i32, i32]
        L.gdn_prefill_layer_workspace_size.restype = sz
        L.gdn_decode_step.argtypes = [vp, vp, vp, i32, vp, vp, vp, i32, i32, i32, i32, i32, f32, i32,
                                      f32, i32, vp, vp]
        L.gdn_decode_layer_step.argtypes = [vp, vp, vp, i32, i32, vp, vp, vp, vp, vp, f32, i32, i32,
                                            i32, i32, i32, f32, i32, f32, i32, vp, vp]
        L.gdn_decode_layer_step.restype = i32
        L.gdn_gated_rmsnorm.argtypes = [vp, vp, vp, i32, i64, i32, f32, vp, vp]
        L.gdn_gated_rmsnorm.restype = i32
        L.gdn_decode_step.restype = i32
        L.gdn_status_string.argtypes = [i32]
        L.gdn_status_string.restype = ctypes.c_char_p
        L.gdn_check_device_status.argtypes = [vp]
        L.gdn_check_device_status.restype = i32
        L.gdn_prefill_noalloc.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, i32, i64, i32, i32, i32,
                                          i32, i64, i64, i64, f32, i32, f32, i32, i32, vp, vp, vp,
                                          i32, vp]
        L.gdn_prefill_noalloc.restype = i32
        L.gdn_prefill_noalloc_max_scratch.argtypes = []
        L.gdn_prefill_noalloc_max_scratch.restype = sz
        L.gdn_prefill_selected_algo.argtypes = [i32, i32, i32, i32, i32]
        L.gdn_prefill_selected_algo.restype = i32
        L.gdn_backward_workspace_size.argtypes = [i32, i64, i32, i32, i32]
        L.gdn_backward_workspace_size.restype = sz
        L.gdn_backward_workspace_size_kept.argtypes = [i32, i64, i32, i32, i32]
        L.gdn_backward_workspace_size_kept.restype = sz
        L.gdn_backward.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32,
                                   f32, i32, f32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.gdn_backward.restype = i32
        L.gdn_set_wait_limit_ns.argtypes = [i64]
        L.gdn_set_wait_limit_ns.restype = None
        L.gdn_version.argtypes = []
        L.gdn_version.restype = i32
        if L.gdn_version() != ABI_VERSION:  # argument lists differ between versions
            raise RuntimeError(f"{LIB_PATH} has ABI {L.gdn_version()}, this binding needs "
                               f"{ABI_VERSION}: rebuild with `python -m gated_deltanet_linear_silu_b200.build`")
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev: torch.device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _on(dev: torch.device):
    """The C ABI works on the current device (its status word and the no-alloc
    scratch array are per device): make the tensors' device current."""
    return torch.cuda.device(dev)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _check(status: int, what: str):
    if status != 0:
        raise GDNError(status, what)


def _cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def _check_heads(q, k, v, g, beta):
    """Shapes the C ABI cannot see: q, k [T, Hk, dk] alike, v [T, H, dv],
    g, beta [T, H], H a multiple of Hk."""
    T, Hk, dk = q.shape
    if tuple(k.shape) != (T, Hk, dk) or v.dim() != 3 or v.shape[0] != T:
        raise ValueError("q and k must be [T, Hk, dk] and v [T, H, dv]")
    H = v.shape[1]
    if H % Hk != 0:
        raise ValueError(f"{H} value heads cannot share {Hk} q/k heads evenly")
    if tuple(g.shape) != (T, H) or tuple(beta.shape) != (T, H):
        raise ValueError("g and beta must be [T, H]")


def _token_stride(t: torch.Tensor) -> int:
    """Elements between consecutive tokens of a [T, H, d] tensor whose rows
    may be views into a wider fused buffer (each row itself dense)."""
    if not t.is_cuda:
        raise ValueError("tensors must be CUDA tensors")
    T, H, d = t.shape
    if t.stride(2) != 1 or (H > 1 and t.stride(1) != d) or t.stride(0) < H * d:
        raise ValueError("q, k, v must have dense [H, d] rows (token stride may be larger)")
    return int(t.stride(0))


def conv_silu(x: torch.Tensor, w: torch.Tensor, cu_seqlens: torch.Tensor, *,
              conv_state: Optional[torch.Tensor] = None, conv_state_out: Optional[torch.Tensor] = None,
              return_state: bool = True, qk_l2norm: bool = True, n_qk_channels: Optional[int] = None,
              head_dim: int = 128, eps: float = 1e-6, out: Optional[torch.Tensor] = None
              ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """y = SiLU(causal depthwise conv(x)) (+ L2 norm of the first n_qk_channels
    per head). x [T, C], w [C, K], cu_seqlens int32 [N+1] on the device,
    conv_state [N, C, K-1] or None. Returns (y, conv_state_out)."""
    T, C = x.shape
    K = w.shape[1]
    N = cu_seqlens.shape[0] - 1
    if n_qk_channels is None:
        n_qk_channels = 2 * (C // 3)
    y = torch.empty_like(x) if out is None else out
    st_out = conv_state_out
    if st_out is None and return_state:
        st_out = torch.empty((N, C, K - 1), dtype=x.dtype, device=x.device)
    _cuda(x, w, cu_seqlens, conv_state, st_out, y)
    with _on(x.device):
        st = lib().gdn_conv_silu(_ptr(x), _dtype_code(x), _ptr(w), _ptr(cu_seqlens), N, T, C, K,
                                 _ptr(conv_state), _ptr(st_out), int(qk_l2norm), int(n_qk_channels),
                                 int(head_dim), float(eps), _ptr(y), _stream(x.device))
    _check(st, "gdn_conv_silu")
    return y, st_out


def prefill_workspace_size(N: int, T_tot: int, H: int, dk: int, dv: int, chunk: int = 64) -> int:
    return int(lib().gdn_prefill_workspace_size(N, T_tot, H, dk, dv, chunk))


def prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor, beta: torch.Tensor,
            cu_seqlens: torch.Tensor, *, initial_state: Optional[torch.Tensor] = None,
            output_final_state: bool = True, final_state: Optional[torch.Tensor] = None,
            scale: float = 1.0, qk_l2norm: bool = True, eps: float = 1e-6, chunk: int = 64,
            cu_seqlens_host: Optional[torch.Tensor] = None, algo: str = "auto",
            workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
            undecayed: bool = False, z: Optional[torch.Tensor] = None,
            norm_w: Optional[torch.Tensor] = None, norm_eps: float = 1e-6
            ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunked gated delta rule. q,k [T,Hk,dk], v [T,H,dv] (bf16 or fp32; each
    may be a token-strided view, e.g. a slice of the fused conv output; Hk < H
    groups H / Hk value heads on each q, k head), g,beta [T,H] fp32, cu_seqlens
    int32 [N+1] (device). Returns (o, hT); final_state may be initial_state
    itself for an in-place update. undecayed=True reads each token's memory
    from the state before its decay (the 7.6.2 order). With z [T,H,dv] (and
    norm_w [dv] fp32) the output is the gated RMSNorm RMSNorm(y) * norm_w *
    SiLU(z) of the recurrence's output y, applied before the output is stored."""
    _check_heads(q, k, v, g, beta)
    T, Hk, dk = q.shape
    H, dv = v.shape[1], v.shape[2]
    N = cu_seqlens.shape[0] - 1
    o = torch.empty((T, H, dv), dtype=q.dtype, device=q.device) if out is None else out
    hT = final_state
    if hT is None and output_final_state:
        hT = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    with _on(q.device):  # the workspace can depend on the device's SM count
        ws_bytes = prefill_workspace_size(N, T, H, dk, dv, chunk)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    ld = [_token_stride(t) for t in (q, k, v)]
    _cuda(g, beta, cu_seqlens, initial_state, hT, o, workspace)
    host_cu = None
    if cu_seqlens_host is not None:
        host_cu = cu_seqlens_host.to(torch.int32).contiguous()
    common = (_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), _ptr(g), _ptr(beta), _ptr(cu_seqlens),
              None if host_cu is None else ctypes.c_void_p(host_cu.data_ptr()), N, T, H, Hk, dk, dv,
              ld[0], ld[1], ld[2], float(scale), int(qk_l2norm), float(eps), int(undecayed),
              int(chunk), _ptr(initial_state), _ptr(hT), _ptr(o))
    if z is None:
        with _on(q.device):
            st = lib().gdn_prefill(*common, _ptr(workspace), workspace.numel(), ALGOS[algo],
                                   _stream(q.device))
        _check(st, "gdn_prefill")
    else:
        if norm_w is None:
            raise ValueError("a gated prefill needs norm_w")
        _cuda(z, norm_w)
        if tuple(z.shape) != (T, H, dv) or z.dtype != q.dtype:
            raise ValueError("z must be [T, H, dv] in the dtype of q")
        with _on(q.device):
            st = lib().gdn_prefill_gated(*common, _ptr(z), _ptr(norm_w), float(norm_eps),
                                         _ptr(workspace), workspace.numel(), ALGOS[algo],
                                         _stream(q.device))
        _check(st, "gdn_prefill_gated")
    return o, hT


def prefill_layer_workspace_size(N: int, T_tot: int, H: int, Hk: int, dk: int = 128, dv: int = 128) -> int:
    return int(lib().gdn_prefill_layer_workspace_size(N, T_tot, H, Hk, dk, dv))


def prefill_layer(x: torch.Tensor, conv_w: torch.Tensor, g: torch.Tensor, beta: torch.Tensor,
                  cu_seqlens: torch.Tensor, *, H: int, Hk: Optional[int] = None, dk: int = 128,
                  dv: int = 128, conv_state_in: Optional[torch.Tensor] = None,
                  conv_state_out: Optional[torch.Tensor] = None,
                  initial_state: Optional[torch.Tensor] = None, output_final_state: bool = True,
                  final_state: Optional[torch.Tensor] = None, scale: float = 1.0,
                  qk_l2norm: bool = True, eps: float = 1e-6, undecayed: bool = False,
                  z: Optional[torch.Tensor] = None, norm_w: Optional[torch.Tensor] = None,
                  norm_eps: float = 1e-6, cu_seqlens_host: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None
                  ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """The whole mixer for a prefill with the conv fused into the chunked
    prefill: x [T, C] bf16 fused [q | k | v] projections before the conv
    (C = 2 Hk dk + H dv), conv_w [C, K] bf16, conv windows [N, C, K-1] bf16 in
    (nullable: zeros) and out (nullable; may be conv_state_in), g, beta [T, H]
    fp32, optional gate z [T, H, dv] with norm_w [dv] fp32. Returns (o, hT).
    The default workspace (prefill_layer_workspace_size) lets a call whose
    prefill runs as the sequence split convolve once into it instead of in
    each pass; a workspace of prefill_workspace_size bytes keeps it fused."""
    Hk = H if Hk is None else Hk
    T, C = x.shape
    K = conv_w.shape[1]
    if Hk <= 0 or C != 2 * Hk * dk + H * dv:
        raise ValueError(f"x has {C} channels; expected 2*Hk*dk + H*dv")
    N = cu_seqlens.shape[0] - 1
    o = torch.empty((T, H, dv), dtype=x.dtype, device=x.device) if out is None else out
    hT = final_state
    if hT is None and output_final_state:
        hT = torch.empty((N, H, dk, dv), dtype=torch.float32, device=x.device)
    if workspace is None:
        with _on(x.device):  # the workspace can depend on the device's SM count
            ws_bytes = prefill_layer_workspace_size(N, T, H, Hk, dk, dv)
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=x.device)
    if z is not None and norm_w is None:
        raise ValueError("a gated prefill needs norm_w")
    _cuda(x, conv_w, conv_state_in, conv_state_out, g, beta, cu_seqlens, initial_state, hT, o, z,
          norm_w, workspace)
    host_cu = None
    if cu_seqlens_host is not None:
        host_cu = cu_seqlens_host.to(torch.int32).contiguous()
    with _on(x.device):
        st = lib().gdn_prefill_layer(
            _ptr(x), _ptr(conv_w), K, _ptr(conv_state_in), _ptr(conv_state_out), _dtype_code(x), _ptr(g),
            _ptr(beta), _ptr(cu_seqlens), None if host_cu is None else ctypes.c_void_p(host_cu.data_ptr()),
            N, T, H, Hk, dk, dv, float(scale), int(qk_l2norm), float(eps), int(undecayed),
            _ptr(initial_state), _ptr(hT), _ptr(o), _ptr(z), _ptr(norm_w), float(norm_eps),
            _ptr(workspace), workspace.numel(), _stream(x.device))
    _check(st, "gdn_prefill_layer")
    return o, hT


def prefill_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                    beta: torch.Tensor, cu_seqlens: torch.Tensor, *,
                    initial_state: Optional[torch.Tensor] = None, final_state: torch.Tensor,
                    out: torch.Tensor, scale: float = 1.0, qk_l2norm: bool = True,
                    eps: float = 1e-6, chunk: int = 64, algo: str = "auto",
                    undecayed: bool = False) -> None:
    """gdn_prefill_noalloc: prefill with the library's fixed scratch array
    instead of a workspace; the caller passes every output buffer, so nothing
    is allocated."""
    _check_heads(q, k, v, g, beta)
    T, Hk, dk = q.shape
    H, dv = v.shape[1], v.shape[2]
    N = cu_seqlens.shape[0] - 1
    ld = [_token_stride(t) for t in (q, k, v)]
    _cuda(g, beta, cu_seqlens, initial_state, final_state, out)
    with _on(q.device):
        st = lib().gdn_prefill_noalloc(
            _ptr(q), _ptr(k), _ptr(v), _dtype_code(q), _ptr(g), _ptr(beta), _ptr(cu_seqlens), None,
            N, T, H, Hk, dk, dv, ld[0], ld[1], ld[2], float(scale), int(qk_l2norm), float(eps),
            int(undecayed), int(chunk),
            _ptr(initial_state), _ptr(final_state), _ptr(out), ALGOS[algo], _stream(q.device))
    _check(st, "gdn_prefill_noalloc")


def selected_algo(dtype: str, dk: int, dv: int, chunk: int = 64, algo: str = "auto") -> str:
    """Name of the prefill kernel ("simt" or "tensor") that would run; raises
    if the combination is unsupported."""
    code = lib().gdn_prefill_selected_algo(GDN_BF16 if dtype == "bf16" else GDN_F32, dk, dv,
                                            chunk, ALGOS[algo])
    if code < 0:
        raise GDNError(2, "gdn_prefill_selected_algo")
    return {1: "simt", 2: "tensor"}[code]


def decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                beta: torch.Tensor, state: torch.Tensor, *, scale: float = 1.0,
                qk_l2norm: bool = True, eps: float = 1e-6, out: Optional[torch.Tensor] = None,
                undecayed: bool = False) -> torch.Tensor:
    """One recurrent token per sequence. q,k [N,Hk,dk], v [N,H,dv], g,beta
    [N,H] fp32, state [N,H,dk,dv] fp32 updated in place. Returns o [N,H,dv]."""
    _check_heads(q, k, v, g, beta)
    N, Hk, dk = q.shape
    H, dv = v.shape[1], v.shape[2]
    o = torch.empty((N, H, dv), dtype=q.dtype, device=q.device) if out is None else out
    _cuda(q, k, v, g, beta, state, o)
    with _on(q.device):
        st = lib().gdn_decode_step(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), _ptr(g), _ptr(beta),
                                   _ptr(state), N, H, Hk, dk, dv, float(scale), int(qk_l2norm), float(eps),
                                   int(undecayed), _ptr(o), _stream(q.device))
    _check(st, "gdn_decode_step")
    return o


def decode_layer_step(x: torch.Tensor, conv_w: torch.Tensor, conv_state: Optional[torch.Tensor],
                      g: torch.Tensor, beta: torch.Tensor, state: torch.Tensor, *, H: int, dk: int,
                      dv: int, z: Optional[torch.Tensor] = None,
                      norm_w: Optional[torch.Tensor] = None, norm_eps: float = 1e-6,
                      scale: float = 1.0, qk_l2norm: bool = True, eps: float = 1e-6,
                      out: Optional[torch.Tensor] = None, Hk: Optional[int] = None,
                      undecayed: bool = False) -> torch.Tensor:
    """One decode token of the whole mixer per sequence. x [N, C] fused
    [q | k | v] projections (C = 2 Hk dk + H dv; Hk q, k heads, default H),
    conv_w [C, K], conv_state [N, C, K-1] and state [N, H, dk, dv] fp32 updated
    in place, g/beta [N, H] fp32, optional gate z [N, H, dv] with norm_w [dv]
    fp32. Returns o [N, H, dv]."""
    Hk = H if Hk is None else Hk
    N, C = x.shape
    K = conv_w.shape[1]
    if Hk <= 0 or C != 2 * Hk * dk + H * dv:
        raise ValueError(f"x has {C} channels; expected 2*Hk*dk + H*dv")
    o = torch.empty((N, H, dv), dtype=x.dtype, device=x.device) if out is None else out
    _cuda(x, conv_w, conv_state, g, beta, state, z, norm_w, o)
    with _on(x.device):
        st = lib().gdn_decode_layer_step(_ptr(x), _ptr(conv_w), _ptr(conv_state), K, _dtype_code(x),
                                         _ptr(g), _ptr(beta), _ptr(state), _ptr(z), _ptr(norm_w),
                                         float(norm_eps), N, H, Hk, dk, dv, float(scale), int(qk_l2norm),
                                         float(eps), int(undecayed), _ptr(o), _stream(x.device))
    _check(st, "gdn_decode_layer_step")
    return o


def backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
             beta: torch.Tensor, cu_seqlens: torch.Tensor, do: torch.Tensor, *,
             initial_state: Optional[torch.Tensor] = None, dhT: Optional[torch.Tensor] = None,
             scale: float = 1.0, qk_l2norm: bool = True, eps: float = 1e-6,
             cu_seqlens_host: Optional[torch.Tensor] = None, want_dh0: bool = True,
             workspace: Optional[torch.Tensor] = None, keep_states: bool = False):
    """Gradients of the recurrence for upstream gradients do [T, H, dv] (fp32)
    and dhT [N, H, dk, dv] (fp32, optional). q, k [T, Hk, dk] and v [T, H, dv]
    dense (bf16 or fp32). Returns (dq, dk, dv, dg, dbeta, dh0), fp32; dh0 is
    None unless want_dh0. keep_states=True allocates the workspace with which
    every token's state is kept from the forward pass (T * H * dk * dv * 4
    bytes) instead of recomputed; a given workspace of that size does the same."""
    _check_heads(q, k, v, g, beta)
    T, Hk, dk = q.shape
    H, dv = v.shape[1], v.shape[2]
    N = cu_seqlens.shape[0] - 1
    dev = q.device
    f32 = dict(dtype=torch.float32, device=dev)
    dq, dkt = torch.empty((T, Hk, dk), **f32), torch.empty((T, Hk, dk), **f32)
    dvt, dg, db = torch.empty((T, H, dv), **f32), torch.empty((T, H), **f32), torch.empty((T, H), **f32)
    dh0 = torch.empty((N, H, dk, dv), **f32) if want_dh0 else None
    size_fn = lib().gdn_backward_workspace_size_kept if keep_states else lib().gdn_backward_workspace_size
    ws_bytes = int(size_fn(N, T, H, dk, dv))
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    _cuda(q, k, v, g, beta, cu_seqlens, do, initial_state, dhT, workspace)
    host_cu = None
    if cu_seqlens_host is not None:
        host_cu = cu_seqlens_host.to(torch.int32).contiguous()
    with _on(dev):
        st = lib().gdn_backward(
            _ptr(q), _ptr(k), _ptr(v), _dtype_code(q), _ptr(g), _ptr(beta), _ptr(cu_seqlens),
            None if host_cu is None else ctypes.c_void_p(host_cu.data_ptr()), N, T, H, Hk, dk, dv,
            float(scale), int(qk_l2norm), float(eps), _ptr(initial_state), _ptr(do), _ptr(dhT),
            _ptr(dq), _ptr(dkt), _ptr(dvt), _ptr(dg), _ptr(db), _ptr(dh0), _ptr(workspace),
            workspace.numel(), _stream(dev))
    _check(st, "gdn_backward")
    return dq, dkt, dvt, dg, db, dh0


def gated_rmsnorm(y: torch.Tensor, z: torch.Tensor, w: torch.Tensor, *, eps: float = 1e-6,
                  out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """out = y / sqrt(mean(y^2) + eps) * w * SiLU(z) over the last axis (d_v).
    y, z [..., dv] bf16 or fp32, w [dv] fp32 (applied as given)."""
    dv = y.shape[-1]
    o = torch.empty_like(y) if out is None else out
    _cuda(y, z, w, o)
    with _on(y.device):
        st = lib().gdn_gated_rmsnorm(_ptr(y), _ptr(z), _ptr(w), _dtype_code(y), y.numel() // dv, dv,
                                     float(eps), _ptr(o), _stream(y.device))
    _check(st, "gdn_gated_rmsnorm")
    return o


def set_wait_limit_ns(ns: int) -> None:
    """Diagnostic: limit of the tensor-core prefill's bounded hand-off waits
    (ns; negative restores the 2 s default, 0 makes them give up at once)."""
    lib().gdn_set_wait_limit_ns(int(ns))


def check_device_status(device: Optional[torch.device] = None) -> None:
    """Synchronise and raise if a kernel skipped work (bad cu_seqlens, timeout)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with _on(dev):
        _check(lib().gdn_check_device_status(_stream(dev)), "device status")


def state_bytes(n_layers: int, heads: int, dk: int, dv: int, elem_bytes: int = 4) -> int:
    """Bytes of recurrent state for n_layers mixer layers (independent of length)."""
    return n_layers * heads * dk * dv * elem_bytes


def conv_channels(key_heads: int, key_head_dim: int, value_heads: int, value_head_dim: int) -> int:
    """Channels of the fused conv input: q and k (key_dim each) then v."""
    return 2 * key_heads * key_head_dim + value_heads * value_head_dim
