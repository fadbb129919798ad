"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/gdn.h declares, and rejects bad arguments before
touching a device."""
import ctypes
import json
import os
import re
import subprocess

import pytest
import torch

import gated_deltanet_linear_silu_b200 as gdn
from gated_deltanet_linear_silu_b200 import build as gbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


@pytest.fixture(scope="module")
def L():
    gbuild.build()
    return gdn.lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GDN_API\s+[\w\s\*]+?\b(gdn_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for required in ["gdn_conv_silu", "gdn_prefill", "gdn_prefill_workspace_size",
                     "gdn_decode_step", "gdn_status_string", "gdn_check_device_status"]:
        assert required in names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", gdn.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s+(\w+)$", out, re.M))
    missing = [s for s in declared_symbols() if s not in exported]
    assert not missing, missing
    for s in declared_symbols():
        assert hasattr(L, s)
    # internal symbols stay hidden
    assert all(s.startswith("gdn_") for s in exported)


def test_status_strings(L):
    for code, name in gdn.STATUS.items():
        assert L.gdn_status_string(code).decode() == name
    assert L.gdn_status_string(99).decode() == "GDN_ERR_UNKNOWN"
    assert L.gdn_version() == gdn.ABI_VERSION


def test_workspace_size_is_aligned_and_grows(L):
    a = L.gdn_prefill_workspace_size(1, 10, 16, 128, 128, 64)
    b = L.gdn_prefill_workspace_size(10000, 10, 16, 128, 128, 64)
    assert a > 0 and a % 256 == 0 and b % 256 == 0 and b > a


def test_workspace_size_covers_the_sequence_split(L):
    """Few (sequence, head) units on the tensor-core shape: the size also holds
    the split's segment bounds, four state arrays of N*S*H states and a bf16 zero
    value buffer (S segments, S >= 6); many units, other head dims or chunks:
    only the schedule (256 + 4 N, rounded up to 256)."""
    base = lambda N: 256 + (4 * N + 255) // 256 * 256
    assert L.gdn_prefill_workspace_size(8, 8 * 16384, 16, 128, 128, 64) == base(8)  # 128 units
    assert L.gdn_prefill_workspace_size(1, 4096, 16, 64, 64, 64) == base(1)        # not d = 128
    assert L.gdn_prefill_workspace_size(1, 4096, 16, 128, 128, 32) == base(1)      # not chunk 64
    assert L.gdn_prefill_workspace_size(1, 256, 16, 128, 128, 64) == base(1)       # too short
    split = L.gdn_prefill_workspace_size(1, 4096, 16, 128, 128, 64)
    state = 128 * 128 * 4
    zeros = 4096 * 16 * 128 * 2
    assert split % 256 == 0
    # S between 6 and 16 segments: four [S, 16] state arrays plus the zero values
    assert base(1) + 4 * 6 * 16 * state + zeros <= split <= 2 * base(16) + 512 + 4 * 16 * 16 * state + zeros


FAKE = ctypes.c_void_p(1 << 20)  # aligned, never dereferenced: validation fails first


def _prefill(L, **kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, dt=1, g=FAKE, beta=FAKE, cu=FAKE, cu_host=None, N=1,
                T=64, H=2, Hk=0, dk=128, dv=128, ldq=0, ldk=0, ldv=0, scale=1.0, l2=1, eps=1e-6, und=0, chunk=64, h0=None, hT=None,
                o=FAKE, ws=FAKE, ws_bytes=1 << 20, algo=0, stream=None)
    args.update(kw)
    return L.gdn_prefill(*args.values())


@pytest.mark.parametrize("kw,expect", [
    (dict(dt=7), 1), (dict(N=-1), 1), (dict(H=0), 1), (dict(N=0, T=5), 1),
    (dict(dk=80 + 1), 2), (dict(dv=144), 2), (dict(chunk=48), 2), (dict(algo=9), 1),
    (dict(q=None), 1), (dict(o=ctypes.c_void_p((1 << 20) + 4)), 1), (dict(cu=None), 1),
    (dict(ws=None), 3), (dict(ws_bytes=16), 3), (dict(ws=ctypes.c_void_p((1 << 20) + 16)), 3),
    (dict(eps=float("nan")), 1),
    (dict(ldq=255), 1), (dict(ldk=257), 1), (dict(ldv=8), 1), (dict(dt=0, ldq=258), 1),
    # grouped value heads: Hk must divide H; dense strides follow Hk for q, k
    (dict(Hk=-1), 1), (dict(H=6, Hk=4), 1), (dict(H=4, Hk=2, ldq=255), 1),
    (dict(H=4, Hk=2, ldv=256), 1),
    (dict(und=2), 1), (dict(und=-1), 1),     # the order flag is 0 or 1
])
def test_prefill_rejects_bad_arguments(L, kw, expect):
    assert _prefill(L, **kw) == expect


def test_prefill_host_seqlens_checked(L):
    bad = [(0, 30, 20), (1, 64, 64), (0, 10, 70)]  # decreasing / not starting at 0 / != T
    for cu in bad:
        arr = (ctypes.c_int32 * 3)(*cu)
        assert _prefill(L, N=2, cu_host=ctypes.cast(arr, ctypes.c_void_p)) == 1


def test_prefill_empty_batch_is_noop(L):
    assert _prefill(L, N=0, T=0, q=None, k=None, v=None, o=None, cu=None) == 0


def _prefill_layer(L, **kw):
    args = dict(x=FAKE, cw=FAKE, K=4, si=None, so=None, dt=1, g=FAKE, beta=FAKE, cu=FAKE, cu_host=None,
                N=2, T=100, H=16, Hk=0, dk=128, dv=128, scale=1.0, l2=1, eps=1e-6, und=0, h0=None,
                hT=None, o=ctypes.c_void_p(1 << 21), z=None, nw=None, neps=1e-6, ws=None, ws_bytes=0,
                stream=None)
    args.update(kw)
    return L.gdn_prefill_layer(*args.values())


@pytest.mark.parametrize("kw,expect", [
    (dict(dt=0), 2), (dict(dt=5), 1), (dict(dk=64), 2), (dict(dv=64), 2), (dict(K=0), 2),
    (dict(K=5), 2), (dict(H=6, Hk=4), 1), (dict(Hk=-1), 1), (dict(N=-1), 1), (dict(x=None), 1),
    (dict(cw=None), 1), (dict(x=ctypes.c_void_p((1 << 20) + 8)), 1),
    (dict(si=ctypes.c_void_p((1 << 20) + 2)), 1), (dict(o=FAKE), 1),   # o must not alias x
    (dict(z=FAKE), 1),                                                   # a gate needs norm_w
    (dict(z=ctypes.c_void_p(1 << 22), nw=FAKE, neps=-1.0), 1),
    (dict(und=2), 1), (dict(eps=float("nan")), 1),
    (dict(), 3), (dict(ws=ctypes.c_void_p(1 << 23), ws_bytes=16), 3),  # valid: the workspace is missing
])
def test_prefill_layer_rejects_bad_arguments(L, kw, expect):
    assert _prefill_layer(L, **kw) == expect


def test_prefill_layer_workspace_size(L):
    """The layer workspace adds y (T * C bf16) only where the prefill splits."""
    pre = L.gdn_prefill_workspace_size(1, 4096, 16, 128, 128, 64)
    lay = L.gdn_prefill_layer_workspace_size(1, 4096, 16, 0, 128, 128)
    if pre > 256 + 256:  # one 4096-token sequence on 16 heads splits (on >= 96 SMs)
        assert lay == (pre + 255) // 256 * 256 + 4096 * 3 * 16 * 128 * 2
        assert L.gdn_prefill_layer_workspace_size(1, 4096, 16, 8, 128, 128) == \
            (pre + 255) // 256 * 256 + 4096 * (2 * 8 + 16) * 128 * 2
    else:
        assert lay == pre
    # eight 16384-token sequences on 16 heads fill the GPU: no split, no y
    assert L.gdn_prefill_layer_workspace_size(8, 131072, 16, 16, 128, 128) == \
        L.gdn_prefill_workspace_size(8, 131072, 16, 128, 128, 64)
    assert lay % 256 == 0


def test_prefill_layer_empty_batch_is_noop(L):
    assert _prefill_layer(L, N=0, T=0, x=None, cw=None, o=None, cu=None, g=None, beta=None) == 0


def _conv(L, **kw):
    args = dict(x=FAKE, dt=1, w=FAKE, cu=FAKE, N=1, T=16, C=6144, K=4, si=None, so=None, l2=1,
                nqk=4096, hd=128, eps=1e-6, y=ctypes.c_void_p(1 << 21), stream=None)
    args.update(kw)
    return L.gdn_conv_silu(*args.values())


@pytest.mark.parametrize("kw,expect", [
    (dict(dt=3), 1), (dict(K=5), 2), (dict(K=0), 1), (dict(C=6145), 2), (dict(hd=96), 2),
    (dict(nqk=100), 1), (dict(nqk=8192), 1), (dict(y=FAKE), 1), (dict(x=None), 1),
    (dict(N=0, T=3), 1),
])
def test_conv_rejects_bad_arguments(L, kw, expect):
    assert _conv(L, **kw) == expect


def _decode(L, **kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, dt=1, g=FAKE, beta=FAKE, state=FAKE, N=4, H=2, Hk=0, dk=128,
                dv=128, scale=1.0, l2=1, eps=1e-6, und=0, o=FAKE, stream=None)
    args.update(kw)
    return L.gdn_decode_step(*args.values())


@pytest.mark.parametrize("kw,expect", [
    (dict(dt=2), 1), (dict(dk=8), 2), (dict(dv=130), 2), (dict(state=None), 1),
    (dict(state=ctypes.c_void_p((1 << 20) + 8)), 1), (dict(H=-1), 1),
    (dict(Hk=-2), 1), (dict(H=4, Hk=3), 1), (dict(Hk=4), 1), (dict(und=3), 1),
])
def test_decode_rejects_bad_arguments(L, kw, expect):
    assert _decode(L, **kw) == expect


def test_decode_empty_batch_is_noop(L):
    assert _decode(L, N=0, q=None, k=None, v=None, state=None, o=None) == 0


@pytest.mark.parametrize("shapes", [
    ((8, 2, 16), (8, 1, 16), (8, 2, 16), (8, 2)),   # k unlike q
    ((8, 2, 16), (8, 2, 16), (8, 3, 16), (8, 3)),   # 3 value heads on 2 q/k heads
    ((8, 2, 16), (8, 2, 16), (7, 2, 16), (8, 2)),   # v has another token count
    ((8, 2, 16), (8, 2, 16), (8, 4, 16), (8, 2)),   # gates not per value head
])
def test_binding_rejects_head_shapes_the_abi_cannot_see(shapes):
    q, k, v, gg = (torch.zeros(s_) for s_ in shapes)
    cu = torch.tensor([0, 8], dtype=torch.int32)
    with pytest.raises(ValueError):
        gdn.prefill(q, k, v, gg, gg, cu)
    with pytest.raises(ValueError):
        gdn.backward(q, k, v, gg, gg, cu, torch.zeros(8, v.shape[1], 16))


@pytest.mark.parametrize("C,H,Hk", [(768, 2, 2), (1024, 2, 1), (512, 3, 1)])
def test_binding_rejects_layer_channel_counts(C, H, Hk):
    """prefill_layer needs C = 2 Hk dk + H dv channels (before any device work)."""
    x = torch.zeros(8, C, dtype=torch.bfloat16)
    w = torch.zeros(C, 4, dtype=torch.bfloat16)
    gg = torch.zeros(8, H)
    with pytest.raises(ValueError, match="channels"):
        gdn.prefill_layer(x, w, gg, gg, torch.tensor([0, 8], dtype=torch.int32), H=H, Hk=Hk, dk=64, dv=64)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(gdn, "LIB_PATH", str(tmp_path / "absent.so"))
    monkeypatch.setattr(gdn, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        gdn.lib()


def _layer_step(L, **kw):
    args = dict(x=FAKE, cw=FAKE, cs=FAKE, K=4, dt=1, g=FAKE, beta=FAKE, st=FAKE, z=None, nw=None,
                neps=1e-6, N=2, H=16, Hk=0, dk=128, dv=128, scale=1.0, l2=1, eps=1e-6, und=0, o=FAKE,
                stream=None)
    args.update(kw)
    return L.gdn_decode_layer_step(*args.values())


@pytest.mark.parametrize("kw,expect", [
    (dict(dt=5), 1), (dict(N=-1), 1), (dict(H=0), 1), (dict(K=0), 1), (dict(K=5), 2),
    (dict(dk=96 + 8), 2), (dict(dv=256), 2), (dict(x=None), 1), (dict(cs=None), 1),
    (dict(z=FAKE), 1),                       # a gate needs norm_w
    (dict(z=FAKE, nw=FAKE, neps=-1.0), 1), (dict(o=ctypes.c_void_p((1 << 20) + 8)), 1),
    (dict(cs=ctypes.c_void_p((1 << 20) + 2)), 1), (dict(eps=float("nan")), 1),
    (dict(Hk=3), 1), (dict(Hk=-1), 1),
    (dict(und=7), 1),
])
def test_decode_layer_step_rejects_bad_arguments(L, kw, expect):
    assert _layer_step(L, **kw) == expect


def test_decode_layer_step_k1_needs_no_conv_state_and_empty_is_noop(L):
    assert _layer_step(L, N=0) == 0
    # K = 1 has no conv state: only the state pointer check remains (NULL state -> invalid)
    assert _layer_step(L, K=1, cs=None, st=None) == 1


def _bwd(L, **kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, dt=1, g=FAKE, beta=FAKE, cu=FAKE, cu_host=None, N=1, T=64,
                H=2, Hk=0, dk=128, dv=128, scale=1.0, l2=1, eps=1e-6, h0=None, dO=FAKE, dhT=None,
                dq=FAKE, dkk=FAKE, dvv=FAKE, dg=FAKE, db=FAKE, dh0=None, ws=FAKE, ws_bytes=1 << 20,
                stream=None)
    args.update(kw)
    return L.gdn_backward(*args.values())


@pytest.mark.parametrize("kw,expect", [
    (dict(dt=4), 1), (dict(N=-1), 1), (dict(H=0), 1), (dict(H=6, Hk=4), 1), (dict(Hk=-1), 1),
    (dict(N=0, T=3), 1), (dict(dk=40), 2), (dict(dv=144), 2), (dict(cu=None), 1),
    (dict(dO=None), 1), (dict(dq=None), 1), (dict(db=None), 1),
    (dict(h0=ctypes.c_void_p((1 << 20) + 4)), 1), (dict(eps=float("nan")), 1),
    (dict(ws=None), 3), (dict(ws_bytes=1024), 3), (dict(ws=ctypes.c_void_p((1 << 20) + 64)), 3),
])
def test_backward_rejects_bad_arguments(L, kw, expect):
    assert _bwd(L, **kw) == expect


def test_backward_workspace_size_formula(L):
    # checkpoints every 16 tokens + 16 recomputed states per (sequence, head)
    N, T, H, dk, dv = 3, 100, 2, 64, 32
    floats = ((2 * N + (T + 15) // 16 + 1) * H + N * H * 16) * dk * dv
    got = L.gdn_backward_workspace_size(N, T, H, dk, dv)
    assert got % 256 == 0 and floats * 4 <= got <= floats * 4 + 512
    # every state kept: a checkpoint slot per token, no recompute buffer
    kept = (2 * N + T + 1) * H * dk * dv
    got_k = L.gdn_backward_workspace_size_kept(N, T, H, dk, dv)
    assert got_k % 256 == 0 and kept * 4 <= got_k <= kept * 4 + 512 and got_k > got
    assert _bwd(L, N=0, T=0, q=None, k=None, v=None, dO=None, dq=None, dkk=None, dvv=None,
                dg=None, db=None, cu=None) == 0  # empty batch: nothing to do


def _gnorm(L, **kw):
    args = dict(y=FAKE, z=FAKE, w=FAKE, dt=1, rows=10, dv=128, eps=1e-6, out=FAKE, stream=None)
    args.update(kw)
    return L.gdn_gated_rmsnorm(*args.values())


@pytest.mark.parametrize("kw,expect", [
    (dict(dt=9), 1), (dict(rows=-1), 1), (dict(dv=130), 2), (dict(dv=2), 2), (dict(dv=260), 2),
    (dict(y=None), 1), (dict(w=None), 1), (dict(out=ctypes.c_void_p((1 << 20) + 4)), 1),
    (dict(eps=-1.0), 1),
])
def test_gated_rmsnorm_rejects_bad_arguments(L, kw, expect):
    assert _gnorm(L, **kw) == expect


def test_gated_rmsnorm_empty_is_noop(L):
    assert _gnorm(L, rows=0, y=None, z=None, w=None, out=None) == 0


def test_sizing_helpers_match_printed_figures():
    d = json.load(open(os.path.join(ROOT, "tests", "golden", "pages_sizing.json")))
    for c in d["cases"]:
        b = gdn.state_bytes(c["layers"], c["heads"], c["dk"], c["dv"], c["elem_bytes"])
        mb = b / (1e6 if c["mb_is_1e6"] else 2 ** 20)
        assert abs(mb - c["printed_mb"]) <= 0.05 * c["printed_mb"], (c["source"], mb)
    cd = d["conv_dim"]
    assert gdn.conv_channels(cd["key_heads"], cd["key_head_dim"], cd["value_heads"],
                             cd["value_head_dim"]) == cd["conv_dim"]


def test_product_path_does_not_import_oracle():
    """The binding and build script never reach the oracle."""
    pkg = os.path.join(ROOT, "gated_deltanet_linear_silu_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "gdn_oracle" not in text, f
