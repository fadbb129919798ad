"""GPU parity: the CUDA path against the CPU oracle on the same seeded bytes,
element by element at sizes the oracle finishes in seconds (several chunks,
ragged tails, empty sequences), and on sampled (sequence, head) units at the
full workload sizes. Tolerances (max-abs-normalised error): 1e-4 for fp32
inputs, 2e-2 for bf16 inputs with fp32 accumulation."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import gated_deltanet_linear_silu_b200 as gdn
import gdn_inputs as gi
import oracle
from gpu_util import (DEV, TOL_BF16, TOL_F32, dev_tensor, err, host, longest_first, oracle_seq,
                      oracle_unit, prefill_gpu, prefill_oracle, tol)

ALGOS = ["auto", "simt", "tensor"]


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(DEV)


# ----------------------------------------------------------------------------
# prefill
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("chunk", [64, 32, 16])
def test_tiny_fp32_workload(chunk):
    P = gi.tiny_fp32()
    o, hT = prefill_gpu(P, chunk=chunk)
    o_ref, h_ref = prefill_oracle(P)
    assert err(o, o_ref) <= TOL_F32
    assert err(hT, h_ref) <= TOL_F32


@pytest.mark.parametrize("algo", ALGOS)
def test_prefill_bf16_ragged_with_state(algo):
    P = gi.random_prefill(1, [1, 63, 64, 65, 0, 200, 130, 3], H=3, dk=128, dv=128, with_h0=True)
    o, hT = prefill_gpu(P, algo=algo)
    o_ref, h_ref = prefill_oracle(P)
    assert err(o, o_ref) <= TOL_BF16
    assert err(hT, h_ref) <= TOL_BF16
    n_empty = 4
    assert np.array_equal(hT[n_empty], P.h0[n_empty])  # empty sequence passes its state through


@pytest.mark.parametrize("algo", ALGOS)
def test_prefill_degenerate_gates(algo):
    """beta = 0 leaves only the decay: S_T = e^{sum g} S_0 and o_t = e^{gamma_t} S_0^T q^_t
    (closed form); with g = 0 as well the state passes through unchanged. Zero q rows give
    zero outputs."""
    P = gi.random_prefill(14, [200, 64, 1], H=2, dk=128, dv=128, with_h0=True)
    P.beta = np.zeros_like(P.beta)
    P.q[5] = 0
    o, hT = prefill_gpu(P, algo=algo)
    q = gi.bf16_bits_to_f32(P.q).astype(np.float64)
    qn = q / np.sqrt((q * q).sum(-1, keepdims=True) + P.eps)
    for n in range(P.N):
        a, b = int(P.cu_seqlens[n]), int(P.cu_seqlens[n + 1])
        gam = np.cumsum(P.g[a:b].astype(np.float64), axis=0)          # [L, H]
        h_cf = np.exp(gam[-1])[:, None, None] * P.h0[n]
        o_cf = np.exp(gam)[:, :, None] * np.einsum("lhi,hij->lhj", qn[a:b], P.h0[n])
        assert err(hT[n], h_cf) <= TOL_BF16
        assert err(o[a:b], o_cf) <= TOL_BF16
    assert np.all(o[5] == 0)
    P.g = np.zeros_like(P.g)
    o, hT = prefill_gpu(P, algo=algo)
    assert err(hT, P.h0) <= TOL_BF16


@pytest.mark.parametrize("g_scale", [1.0, 4.0])
def test_prefill_bf16_decay_ranges(g_scale):
    """Chunks whose cumulative decay |gamma| (about 51 * g_scale at a chunk's end
    here) stays below or exceeds the bound under which the tensor-core path
    factors e^{gamma_r - gamma_j} into e^{gamma_r} e^{-gamma_j} (60): both ways of
    forming the decay, against the oracle."""
    P = gi.random_prefill(13, [130, 64, 200], H=2, dk=128, dv=128, g_scale=g_scale, with_h0=True)
    o, hT = prefill_gpu(P, algo="tensor")
    o_ref, h_ref = prefill_oracle(P)
    assert err(o, o_ref) <= TOL_BF16
    assert err(hT, h_ref) <= TOL_BF16


@pytest.mark.parametrize("dk,dv", [(16, 16), (64, 128), (128, 64), (32, 96), (48, 80), (128, 128)])
def test_prefill_fp32_shapes(dk, dv):
    P = gi.random_prefill(2, [70, 5, 129], H=2, dk=dk, dv=dv, dtype="f32", with_h0=True, chunk=32,
                          scale=0.5)
    o, hT = prefill_gpu(P)
    o_ref, h_ref = prefill_oracle(P)
    assert err(o, o_ref) <= TOL_F32
    assert err(hT, h_ref) <= TOL_F32


def test_prefill_without_l2norm_and_strong_decay():
    P = gi.random_prefill(3, [150, 64], H=2, dk=64, dv=64, dtype="f32", g_scale=10.0,
                          qk_l2norm=False)
    P.q = (P.q / np.linalg.norm(P.q, axis=-1, keepdims=True)).astype(np.float32)
    P.k = (P.k / np.linalg.norm(P.k, axis=-1, keepdims=True)).astype(np.float32)
    o, hT = prefill_gpu(P)
    o_ref, h_ref = prefill_oracle(P)
    assert err(o, o_ref) <= TOL_F32 and err(hT, h_ref) <= TOL_F32


@pytest.mark.parametrize("algo", ALGOS)
def test_prefill_token_strided_views_equal_dense(algo):
    """q, k, v as views into one padded fused buffer give the dense result bit for bit."""
    P = gi.random_prefill(12, [70, 129, 0, 64], H=2, dk=128, dv=128, with_h0=True)
    o_d, h_d = prefill_gpu(P, algo=algo)
    T, H, d = P.q.shape
    ld = 3 * H * d + 64
    fused = torch.zeros((T, ld), dtype=torch.bfloat16, device=DEV)
    views = []
    for i, a in enumerate((P.q, P.k, P.v)):
        fused[:, i * H * d:(i + 1) * H * d] = dev_tensor(a, "bf16").view(T, H * d)
        views.append(fused[:, i * H * d:(i + 1) * H * d].view(T, H, d))
    assert views[0].stride(0) == ld and not views[0].is_contiguous()
    o, hT = gdn.prefill(*views, dev_tensor(P.g, "f32"), dev_tensor(P.beta, "f32"),
                        torch.from_numpy(P.cu_seqlens).to(DEV),
                        initial_state=dev_tensor(P.h0, "f32"), algo=algo)
    gdn.check_device_status(DEV)
    assert np.array_equal(host(o), o_d) and np.array_equal(host(hT), h_d)


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("H,Hk", [(6, 3), (8, 2)])
def test_prefill_grouped_value_heads(algo, H, Hk):
    """H value heads on Hk q, k heads (value head h reads q, k head h // (H // Hk)),
    ragged lengths with an empty sequence and an initial state."""
    P = gi.random_prefill(15, [1, 130, 0, 64, 77], H=H, Hk=Hk, dk=128, dv=128, with_h0=True)
    o, hT = prefill_gpu(P, algo=algo)
    o_ref, h_ref = prefill_oracle(P)
    assert err(o, o_ref) <= TOL_BF16
    assert err(hT, h_ref) <= TOL_BF16


@pytest.mark.parametrize("algo", ALGOS)
def test_prefill_grouped_value_heads_from_fused_buffer(algo):
    """Grouped heads read in place from one fused [T, 2 Hk dk + H dv (+pad)] buffer
    (the conv output's layout) give the dense result bit for bit."""
    H, Hk, d = 4, 2, 128
    P = gi.random_prefill(16, [70, 129, 64], H=H, Hk=Hk, dk=d, dv=d, with_h0=True)
    o_d, h_d = prefill_gpu(P, algo=algo)
    T = P.T_tot
    widths = [Hk * d, Hk * d, H * d]
    ld = sum(widths) + 32
    fused = torch.zeros((T, ld), dtype=torch.bfloat16, device=DEV)
    views, c0 = [], 0
    for a, wdt, nh in zip((P.q, P.k, P.v), widths, (Hk, Hk, H)):
        fused[:, c0:c0 + wdt] = dev_tensor(a, "bf16").view(T, wdt)
        views.append(fused[:, c0:c0 + wdt].view(T, nh, d))
        c0 += wdt
    o, hT = gdn.prefill(*views, dev_tensor(P.g, "f32"), dev_tensor(P.beta, "f32"),
                        torch.from_numpy(P.cu_seqlens).to(DEV),
                        initial_state=dev_tensor(P.h0, "f32"), algo=algo)
    gdn.check_device_status(DEV)
    assert np.array_equal(host(o), o_d) and np.array_equal(host(hT), h_d)


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("g_scale", [1.0, 4.0])
def test_prefill_undecayed_read(algo, g_scale):
    """The 7.6.2 order (memory read from the state before the decay): ragged
    sequences with an initial state; g_scale 4 takes chunks past the factored-decay
    range, so both epilogue paths run."""
    P = gi.random_prefill(17, [1, 63, 64, 65, 0, 200, 130], H=3, dk=128, dv=128, with_h0=True,
                          g_scale=g_scale)
    o, hT = prefill_gpu(P, algo=algo, undecayed=True)
    o_ref, h_ref = prefill_oracle(P, undecayed=True)
    assert err(o, o_ref) <= TOL_BF16
    assert err(hT, h_ref) <= TOL_BF16
    o_std, _ = prefill_oracle(P)
    assert err(o_std, o_ref) > 2 * TOL_BF16  # the two orders are told apart at this tolerance


@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_prefill_undecayed_read_fp32(chunk):
    P = gi.random_prefill(18, [100, 37, 1], H=2, dk=64, dv=48, dtype="f32", with_h0=True,
                          chunk=chunk)
    o, hT = prefill_gpu(P, undecayed=True)
    o_ref, h_ref = prefill_oracle(P, undecayed=True)
    assert err(o, o_ref) <= TOL_F32 and err(hT, h_ref) <= TOL_F32


def test_chunk_sizes_agree():
    P = gi.random_prefill(4, [100, 37], H=2, dk=32, dv=32, dtype="f32", with_h0=True)
    outs = [prefill_gpu(P, chunk=c) for c in (16, 32, 64)]
    for o, hT in outs[1:]:
        assert err(o, outs[0][0]) <= TOL_F32 and err(hT, outs[0][1]) <= TOL_F32


@pytest.mark.parametrize("algo", ALGOS)
def test_split_and_resume_equals_one_call(algo):
    T, m = 300, 117
    P = gi.random_prefill(5, [T], H=2, dk=128, dv=128, with_h0=True)
    o_all, h_all = prefill_gpu(P, algo=algo)
    A = gi.random_prefill(5, [T], H=2, dk=128, dv=128, with_h0=True)
    for name in ("q", "k", "v", "g", "beta"):
        setattr(A, name, getattr(P, name)[:m])
    A.cu_seqlens = np.array([0, m], np.int32)
    o1, h1 = prefill_gpu(A, algo=algo)
    B = gi.random_prefill(5, [T], H=2, dk=128, dv=128)
    for name in ("q", "k", "v", "g", "beta"):
        setattr(B, name, getattr(P, name)[m:])
    B.cu_seqlens = np.array([0, T - m], np.int32)
    o2, h2 = prefill_gpu(B, algo=algo, h0=h1)
    # Moving the chunk boundary changes which values the tensor-core path
    # rounds to bf16 (2^-9 relative per operand): half the bf16 tolerance there.
    # The CUDA-core path computes in fp32 from the same decoded inputs and only
    # rounds o to bf16 at the end: 1e-3.
    bound = 1e-3 if algo == "simt" else TOL_BF16 / 2
    assert err(np.concatenate([o1, o2]), o_all) <= bound
    assert err(h2, h_all) <= bound


@pytest.mark.parametrize("algo", ["simt", "tensor"])
def test_prefill_in_place_state(algo):
    """final_state may be initial_state itself (hT == h0): the update happens in
    place and equals the out-of-place result bit for bit."""
    P = gi.random_prefill(22, [130, 0, 64, 5], H=3, dk=128, dv=128, with_h0=True)
    o_ref, h_ref = prefill_gpu(P, algo=algo)
    q, k, v = (dev_tensor(a, "bf16") for a in (P.q, P.k, P.v))
    state = dev_tensor(P.h0, "f32")
    o, hT = gdn.prefill(q, k, v, dev_tensor(P.g, "f32"), dev_tensor(P.beta, "f32"),
                        torch.from_numpy(P.cu_seqlens).to(DEV), initial_state=state,
                        final_state=state, algo=algo)
    gdn.check_device_status(DEV)
    assert hT.data_ptr() == state.data_ptr()
    assert np.array_equal(host(o), o_ref) and np.array_equal(host(state), h_ref)
    o_or, h_or = prefill_oracle(P)
    assert err(host(state), h_or) <= TOL_BF16


@pytest.mark.parametrize("algo", ["simt", "tensor"])
def test_prefill_more_units_than_sms(algo):
    """48 sequences x 4 heads = 192 (sequence, head) units, more than the 148 SMs,
    lengths 0..300 with initial states: the persistent kernel's CTAs each take
    a second unit after the first (the hand-over between units); every element
    against the oracle."""
    lens = np.random.default_rng(23).integers(0, 301, size=48)
    lens[[5, 17]] = 0
    P = gi.random_prefill(23, lens.tolist(), H=4, dk=128, dv=128, with_h0=True)
    sms = torch.cuda.get_device_properties(DEV).multi_processor_count
    assert P.N * P.H > sms
    o, hT = prefill_gpu(P, algo=algo)
    o_ref, h_ref = prefill_oracle(P)
    assert err(o, o_ref) <= TOL_BF16
    assert err(hT, h_ref) <= TOL_BF16
    assert np.array_equal(hT[5], P.h0[5]) and np.array_equal(hT[17], P.h0[17])


def test_prefill_many_short_units_work_counter():
    """750 sequences of 0..150 tokens x 4 heads = 3000 units on the tensor-core
    kernel: each CTA takes about twenty units from the work counter, so the
    shared-memory ring that hands a unit to every role wraps around (16 slots)
    and the roles meet units of one to three chunks back to back; every element
    and every final state against the oracle."""
    lens = np.random.default_rng(29).integers(0, 151, size=750)
    lens[[3, 400, 749]] = 0
    P = gi.random_prefill(29, lens.tolist(), H=4, dk=128, dv=128, with_h0=True)
    sms = torch.cuda.get_device_properties(DEV).multi_processor_count
    assert P.N * P.H > 16 * sms
    o, hT = prefill_gpu(P, algo="tensor")
    o_ref, h_ref = prefill_oracle(P)
    assert err(o, o_ref) <= TOL_BF16
    assert err(hT, h_ref) <= TOL_BF16
    assert np.array_equal(hT[400], P.h0[400])


@pytest.mark.parametrize("algo", ["tensor", "simt"])
@pytest.mark.parametrize("undecayed", [False, True])
def test_prefill_gated_output(algo, undecayed):
    """The gated RMSNorm output fused into the prefill (7.6.2: RMSNorm(y) * w *
    SiLU(z)) against the oracle's gate applied to the oracle's recurrence: ragged
    lengths with partial chunks, an empty sequence and initial states."""
    P = gi.random_prefill(24, [1, 63, 64, 65, 0, 200, 130], H=3, dk=128, dv=128, with_h0=True)
    r = np.random.default_rng(25)
    z = gi.to_bf16_bits((r.normal(size=(P.T_tot, P.H, 128)) * 2).astype(np.float32))
    w = (1.0 + 0.1 * r.normal(size=128)).astype(np.float32)
    q, k, v = (dev_tensor(a, "bf16") for a in (P.q, P.k, P.v))
    o, hT = gdn.prefill(q, k, v, dev_tensor(P.g, "f32"), dev_tensor(P.beta, "f32"),
                        torch.from_numpy(P.cu_seqlens).to(DEV), initial_state=dev_tensor(P.h0, "f32"),
                        algo=algo, undecayed=undecayed, z=dev_tensor(z, "bf16"),
                        norm_w=torch.from_numpy(w).to(DEV), norm_eps=1e-6)
    gdn.check_device_status(DEV)
    y_ref, h_ref = prefill_oracle(P, undecayed=undecayed)
    ref = oracle.gated_rmsnorm(y_ref, gi.bf16_bits_to_f32(z).astype(np.float64), w, dtype="f64",
                               eps=1e-6)
    assert err(host(o), ref) <= TOL_BF16
    assert err(host(hT), h_ref) <= TOL_BF16
    # the gate does not change the state
    o2, hT2 = prefill_gpu(P, algo=algo, undecayed=undecayed)
    assert np.array_equal(host(hT), hT2)


def test_varlen_packing_equals_separate_calls():
    P = gi.random_prefill(6, [33, 0, 97, 64], H=2, dk=64, dv=64, dtype="f32", with_h0=True)
    o, hT = prefill_gpu(P)
    for n in range(P.N):
        a, b = P.cu_seqlens[n], P.cu_seqlens[n + 1]
        Q = gi.random_prefill(6, [b - a], H=2, dk=64, dv=64, dtype="f32")
        for name in ("q", "k", "v", "g", "beta"):
            setattr(Q, name, getattr(P, name)[a:b])
        Q.h0 = P.h0[n:n + 1]
        on, hn = prefill_gpu(Q)
        if b > a:
            assert err(o[a:b], on) <= 1e-6
        assert err(hT[n:n + 1], hn) <= 1e-6


def test_decode_steps_equal_prefill():
    T = 40
    P = gi.random_prefill(7, [T, T], H=2, dk=64, dv=32, dtype="f32", with_h0=True)
    o_p, h_p = prefill_gpu(P)
    state = dev_tensor(P.h0, "f32").clone()
    idx = np.array([0, T])
    for t in range(T):
        rows = idx + t
        args = [dev_tensor(getattr(P, nm)[rows], "f32") for nm in ("q", "k", "v", "g", "beta")]
        o_t = gdn.decode_step(*args, state, scale=P.scale)
        assert err(host(o_t), o_p[rows]) <= TOL_F32
    assert err(host(state), h_p) <= TOL_F32


# ----------------------------------------------------------------------------
# decode
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("kind,dk,dv", [("f32", 16, 16), ("f32", 128, 128), ("bf16", 128, 128),
                                        ("f32", 48, 80), ("bf16", 64, 128)])
def test_decode_step_matches_oracle(kind, dk, dv):
    r = np.random.default_rng(8)
    N, H = 5, 3
    q, k = r.normal(size=(N, H, dk)).astype(np.float32), r.normal(size=(N, H, dk)).astype(np.float32)
    v = r.normal(size=(N, H, dv)).astype(np.float32)
    if kind == "bf16":
        q, k, v = gi.to_bf16_bits(q), gi.to_bf16_bits(k), gi.to_bf16_bits(v)
    g = -np.abs(r.normal(size=(N, H))).astype(np.float32)
    beta = r.uniform(size=(N, H)).astype(np.float32)
    s0 = r.normal(0, 0.1, size=(N, H, dk, dv)).astype(np.float32)
    state = dev_tensor(s0, "f32")
    o = gdn.decode_step(dev_tensor(q, kind), dev_tensor(k, kind), dev_tensor(v, kind),
                        dev_tensor(g, "f32"), dev_tensor(beta, "f32"), state, scale=0.9)
    o_ref, s_ref = oracle.recurrence(q, k, v, g, beta, np.arange(N + 1), dtype=kind, h0=s0,
                                     scale=0.9)
    assert err(host(o), o_ref) <= tol(kind)
    assert err(host(state), s_ref) <= TOL_F32  # the state never passes through bf16


@pytest.mark.parametrize("kind", ["f32", "bf16"])
def test_decode_step_grouped_value_heads(kind):
    r = np.random.default_rng(9)
    N, H, Hk, dk, dv = 5, 6, 2, 128, 128
    q, k = r.normal(size=(N, Hk, dk)).astype(np.float32), r.normal(size=(N, Hk, dk)).astype(np.float32)
    v = r.normal(size=(N, H, dv)).astype(np.float32)
    if kind == "bf16":
        q, k, v = gi.to_bf16_bits(q), gi.to_bf16_bits(k), gi.to_bf16_bits(v)
    g = -np.abs(r.normal(size=(N, H))).astype(np.float32)
    beta = r.uniform(size=(N, H)).astype(np.float32)
    s0 = r.normal(0, 0.1, size=(N, H, dk, dv)).astype(np.float32)
    state = dev_tensor(s0, "f32")
    o = gdn.decode_step(dev_tensor(q, kind), dev_tensor(k, kind), dev_tensor(v, kind),
                        dev_tensor(g, "f32"), dev_tensor(beta, "f32"), state)
    o_ref, s_ref = oracle.recurrence(q, k, v, g, beta, np.arange(N + 1), dtype=kind, h0=s0)
    assert err(host(o), o_ref) <= tol(kind)
    assert err(host(state), s_ref) <= TOL_F32


@pytest.mark.parametrize("kind", ["f32", "bf16"])
def test_decode_step_undecayed_read(kind):
    r = np.random.default_rng(10)
    N, H, dk, dv = 5, 3, 128, 64
    q, k = r.normal(size=(N, H, dk)).astype(np.float32), r.normal(size=(N, H, dk)).astype(np.float32)
    v = r.normal(size=(N, H, dv)).astype(np.float32)
    if kind == "bf16":
        q, k, v = gi.to_bf16_bits(q), gi.to_bf16_bits(k), gi.to_bf16_bits(v)
    g = -np.abs(r.normal(size=(N, H))).astype(np.float32)
    beta = r.uniform(size=(N, H)).astype(np.float32)
    s0 = r.normal(0, 0.1, size=(N, H, dk, dv)).astype(np.float32)
    state = dev_tensor(s0, "f32")
    o = gdn.decode_step(dev_tensor(q, kind), dev_tensor(k, kind), dev_tensor(v, kind),
                        dev_tensor(g, "f32"), dev_tensor(beta, "f32"), state, undecayed=True)
    o_ref, s_ref = oracle.recurrence(q, k, v, g, beta, np.arange(N + 1), dtype=kind, h0=s0,
                                     undecayed=True)
    assert err(host(o), o_ref) <= tol(kind)
    assert err(host(state), s_ref) <= TOL_F32


def test_decode_workload_full_100_steps():
    """256 sequences x 16 heads, d=128, 100 in-place steps; every output of
    every step and the final state against the oracle's own trajectory."""
    N, H, d = 256, 16, 128
    s0 = gi.decode_state(N, H, d)
    state = dev_tensor(s0, "f32")
    ref_state = s0.astype(np.float64)
    worst_o = 0.0
    for step in range(100):
        D = gi.decode_step(step, N, H, d)
        o = gdn.decode_step(dev_tensor(D.q, "bf16"), dev_tensor(D.k, "bf16"), dev_tensor(D.v, "bf16"),
                            dev_tensor(D.g, "f32"), dev_tensor(D.beta, "f32"), state)
        o_ref, ref_state = oracle.recurrence(D.q, D.k, D.v, D.g, D.beta, np.arange(N + 1),
                                             dtype="bf16", h0=ref_state)
        worst_o = max(worst_o, err(host(o), o_ref))
    assert worst_o <= TOL_BF16
    assert err(host(state), ref_state) <= TOL_BF16


# ----------------------------------------------------------------------------
# conv
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("kind", ["bf16", "f32"])
@pytest.mark.parametrize("with_state", [False, True])
@pytest.mark.parametrize("K", [4, 3, 1])
def test_conv_matches_oracle(kind, with_state, K):
    lens = [5, 1, 0, 2, 40, 33, 70]
    H, d = 2, 128
    C = 3 * H * d
    x, w, cu, st = gi.random_mixed(9, lens, C, K=K, dtype=kind, with_state=with_state)
    y, st_out = gdn.conv_silu(dev_tensor(x, kind), dev_tensor(w, kind),
                              torch.from_numpy(cu).to(DEV),
                              conv_state=None if st is None else dev_tensor(st, kind),
                              n_qk_channels=2 * H * d, head_dim=d)
    gdn.check_device_status(DEV)
    y_ref, st_ref = oracle.conv_silu(x, w, cu, dtype=kind, state_in=st, qk_l2norm=True,
                                     n_qk=2 * H * d, head_dim=d)
    assert err(host(y), y_ref) <= (1e-2 if kind == "bf16" else 1e-5)
    if K > 1:
        assert np.array_equal(host(st_out), st_ref.astype(np.float32))  # a pure copy: bit exact


def test_conv_state_in_place_and_continuation():
    C, K = 384, 4
    x, w, cu, st = gi.random_mixed(10, [50], C, K=K, dtype="f32", with_state=True)
    st_d = dev_tensor(st, "f32")
    xd, wd = dev_tensor(x, "f32"), dev_tensor(w, "f32")
    y_all, _ = gdn.conv_silu(xd, wd, torch.tensor([0, 50], dtype=torch.int32, device=DEV),
                             conv_state=st_d.clone(), qk_l2norm=False)
    m = 23
    s = st_d.clone()
    y1, _ = gdn.conv_silu(xd[:m].contiguous(), wd, torch.tensor([0, m], dtype=torch.int32, device=DEV),
                          conv_state=s, conv_state_out=s, qk_l2norm=False)
    y2, _ = gdn.conv_silu(xd[m:].contiguous(), wd, torch.tensor([0, 50 - m], dtype=torch.int32,
                                                                device=DEV),
                          conv_state=s, conv_state_out=s, qk_l2norm=False)
    assert err(host(torch.cat([y1, y2])), host(y_all)) <= 1e-6
    assert np.array_equal(host(s)[0], x[-3:].T)


# ----------------------------------------------------------------------------
# gated RMSNorm output, whole-mixer decode step
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("kind", ["bf16", "f32"])
@pytest.mark.parametrize("dv", [128, 64, 256, 20])
def test_gated_rmsnorm_matches_oracle(kind, dv):
    r = np.random.default_rng(31)
    rows = 1000 + 7
    y = (r.normal(size=(rows, dv)) * 3).astype(np.float32)
    z = (r.normal(size=(rows, dv)) * 2).astype(np.float32)
    w = (1.0 + 0.1 * r.normal(size=dv)).astype(np.float32)
    yb, zb = (gi.to_bf16_bits(y), gi.to_bf16_bits(z)) if kind == "bf16" else (y, z)
    out = gdn.gated_rmsnorm(dev_tensor(yb, kind), dev_tensor(zb, kind),
                            torch.from_numpy(w).to(DEV), eps=1e-6)
    ref = oracle.gated_rmsnorm(yb, zb, w, dtype=kind, eps=1e-6)
    assert err(host(out), ref) <= (TOL_BF16 if kind == "bf16" else 1e-5)


@pytest.mark.parametrize("kind", ["bf16", "f32"])
@pytest.mark.parametrize("gate", [False, True])
@pytest.mark.parametrize("K", [4, 2])
def test_decode_layer_step_matches_oracle(kind, gate, K):
    """Five decode tokens through the fused kernel (conv state and recurrent state
    carried in place) against the oracle's conv + recurrence + gate."""
    r = np.random.default_rng(32)
    N, H, dk, dv = 5, 3, 64, 128
    C = 2 * H * dk + H * dv
    to = (lambda a: gi.to_bf16_bits(a.astype(np.float32))) if kind == "bf16" else (
        lambda a: a.astype(np.float32))
    cw = to(r.normal(size=(C, K)) * 0.5)
    cs = to(r.normal(size=(N, C, K - 1)))
    st = (r.normal(size=(N, H, dk, dv)) * 0.1).astype(np.float32)
    nw = (1.0 + 0.1 * r.normal(size=dv)).astype(np.float32)
    cs_d, st_d = dev_tensor(cs, kind), torch.from_numpy(st).to(DEV)
    cs_o, st_o = cs, st.astype(np.float64)
    worst = 0.0
    for t in range(5):
        x = to(r.normal(size=(N, C)))
        z = to(r.normal(size=(N, H, dv))) if gate else None
        g = (-np.log1p(np.exp(r.normal(size=(N, H))))).astype(np.float32)
        b = (1.0 / (1.0 + np.exp(-r.normal(size=(N, H))))).astype(np.float32)
        o = gdn.decode_layer_step(dev_tensor(x, kind), dev_tensor(cw, kind), cs_d,
                                  torch.from_numpy(g).to(DEV), torch.from_numpy(b).to(DEV), st_d,
                                  H=H, dk=dk, dv=dv,
                                  z=None if z is None else dev_tensor(z, kind),
                                  norm_w=torch.from_numpy(nw).to(DEV) if gate else None)
        o_ref, cs_n, st_o = oracle.decode_layer_step(x, cw, cs_o, g, b, st_o, dtype=kind, H=H,
                                                     dk=dk, dv=dv, z=z, norm_w=nw if gate else None)
        cs_o = to(cs_n) if kind == "bf16" else cs_n  # the conv state is stored in dtype
        worst = max(worst, err(host(o), o_ref))
    gdn.check_device_status(DEV)
    tol = TOL_BF16 if kind == "bf16" else TOL_F32
    assert worst <= tol
    assert err(host(st_d), st_o) <= tol
    assert np.array_equal(host(cs_d), (gi.bf16_bits_to_f32(cs_o) if kind == "bf16" else cs_o)
                          .astype(np.float32))  # a pure shift: bit exact


@pytest.mark.parametrize("kind", ["bf16", "f32"])
@pytest.mark.parametrize("G", [2, 4, 8, 16])
def test_decode_layer_step_grouped_value_heads(kind, G):
    """G value heads per q, k head share the q, k conv channels (one CTA runs a
    group's value heads back to back); three tokens in a row check that the
    shared conv state is shifted exactly once per token."""
    r = np.random.default_rng(34 + G)
    N, Hk, dk, dv, K = 5, 2, 128, 128, 4
    H = G * Hk
    C = 2 * Hk * dk + H * dv
    to = (lambda a: gi.to_bf16_bits(a.astype(np.float32))) if kind == "bf16" else (
        lambda a: a.astype(np.float32))
    cw = to(r.normal(size=(C, K)) * 0.5)
    cs = to(r.normal(size=(N, C, K - 1)))
    st = (r.normal(size=(N, H, dk, dv)) * 0.1).astype(np.float32)
    nw = (1.0 + 0.1 * r.normal(size=dv)).astype(np.float32)
    cs_d, st_d = dev_tensor(cs, kind), torch.from_numpy(st).to(DEV)
    cs_o, st_o = cs, st.astype(np.float64)
    worst = 0.0
    for t in range(3):
        x = to(r.normal(size=(N, C)))
        z = to(r.normal(size=(N, H, dv)))
        g = (-np.log1p(np.exp(r.normal(size=(N, H))))).astype(np.float32)
        b = (1.0 / (1.0 + np.exp(-r.normal(size=(N, H))))).astype(np.float32)
        o = gdn.decode_layer_step(dev_tensor(x, kind), dev_tensor(cw, kind), cs_d,
                                  torch.from_numpy(g).to(DEV), torch.from_numpy(b).to(DEV), st_d,
                                  H=H, Hk=Hk, dk=dk, dv=dv, z=dev_tensor(z, kind),
                                  norm_w=torch.from_numpy(nw).to(DEV))
        o_ref, cs_n, st_o = oracle.decode_layer_step(x, cw, cs_o, g, b, st_o, dtype=kind, H=H,
                                                     Hk=Hk, dk=dk, dv=dv, z=z, norm_w=nw)
        cs_o = to(cs_n) if kind == "bf16" else cs_n
        worst = max(worst, err(host(o), o_ref))
    gdn.check_device_status(DEV)
    tol_ = TOL_BF16 if kind == "bf16" else TOL_F32
    assert worst <= tol_
    assert err(host(st_d), st_o) <= tol_
    assert np.array_equal(host(cs_d), (gi.bf16_bits_to_f32(cs_o) if kind == "bf16" else cs_o)
                          .astype(np.float32))


@pytest.mark.parametrize("kind", ["bf16", "f32"])
def test_decode_layer_step_undecayed_read(kind):
    r = np.random.default_rng(45)
    N, H, Hk, dk, dv, K = 4, 4, 2, 128, 128, 4
    C = 2 * Hk * dk + H * dv
    to = (lambda a: gi.to_bf16_bits(a.astype(np.float32))) if kind == "bf16" else (
        lambda a: a.astype(np.float32))
    cw, cs = to(r.normal(size=(C, K)) * 0.5), to(r.normal(size=(N, C, K - 1)))
    st = (r.normal(size=(N, H, dk, dv)) * 0.1).astype(np.float32)
    nw = (1.0 + 0.1 * r.normal(size=dv)).astype(np.float32)
    cs_d, st_d = dev_tensor(cs, kind), torch.from_numpy(st).to(DEV)
    cs_o, st_o = cs, st.astype(np.float64)
    worst = 0.0
    for t in range(3):
        x, z = to(r.normal(size=(N, C))), to(r.normal(size=(N, H, dv)))
        g = (-np.log1p(np.exp(r.normal(size=(N, H))))).astype(np.float32)
        b = (1.0 / (1.0 + np.exp(-r.normal(size=(N, H))))).astype(np.float32)
        o = gdn.decode_layer_step(dev_tensor(x, kind), dev_tensor(cw, kind), cs_d,
                                  torch.from_numpy(g).to(DEV), torch.from_numpy(b).to(DEV), st_d,
                                  H=H, Hk=Hk, dk=dk, dv=dv, z=dev_tensor(z, kind),
                                  norm_w=torch.from_numpy(nw).to(DEV), undecayed=True)
        o_ref, cs_n, st_o = oracle.decode_layer_step(x, cw, cs_o, g, b, st_o, dtype=kind, H=H,
                                                     Hk=Hk, dk=dk, dv=dv, z=z, norm_w=nw,
                                                     undecayed=True)
        cs_o = to(cs_n) if kind == "bf16" else cs_n
        worst = max(worst, err(host(o), o_ref))
    gdn.check_device_status(DEV)
    tol_ = TOL_BF16 if kind == "bf16" else TOL_F32
    assert worst <= tol_ and err(host(st_d), st_o) <= tol_


@pytest.mark.parametrize("kind,K,gate,G", [("bf16", 4, True, 1), ("f32", 4, True, 1), ("bf16", 1, False, 1),
                                           ("f32", 3, False, 1), ("bf16", 4, True, 2), ("f32", 4, True, 4)])
def test_decode_layer_step_many_units_per_sm(kind, K, gate, G):
    """More q/k groups than the streaming kernel's CTAs (two per SM), so CTAs
    take several groups and each CTA's prefetch slot is refilled many times;
    with G > 1 a CTA runs a group's G value heads back to back on shared q, k;
    K = 1 runs without a conv state."""
    r = np.random.default_rng(46 + K + 10 * G)
    H, dk, dv = 16, 128, 128
    Hk = H // G
    N = 640 // Hk
    C = 2 * Hk * dk + H * dv
    to = (lambda a: gi.to_bf16_bits(a.astype(np.float32))) if kind == "bf16" else (
        lambda a: a.astype(np.float32))
    cw = to(r.normal(size=(C, K)) * 0.5)
    cs = to(r.normal(size=(N, C, K - 1))) if K > 1 else None
    st = (r.normal(size=(N, H, dk, dv)) * 0.1).astype(np.float32)
    nw = (1.0 + 0.1 * r.normal(size=dv)).astype(np.float32)
    cs_d = dev_tensor(cs, kind) if K > 1 else None
    st_d = torch.from_numpy(st).to(DEV)
    cs_o, st_o = cs, st.astype(np.float64)
    worst = 0.0
    for t in range(2):
        x = to(r.normal(size=(N, C)))
        z = to(r.normal(size=(N, H, dv))) if gate else None
        g = (-np.log1p(np.exp(r.normal(size=(N, H))))).astype(np.float32)
        b = (1.0 / (1.0 + np.exp(-r.normal(size=(N, H))))).astype(np.float32)
        o = gdn.decode_layer_step(dev_tensor(x, kind), dev_tensor(cw, kind), cs_d,
                                  torch.from_numpy(g).to(DEV), torch.from_numpy(b).to(DEV), st_d,
                                  H=H, Hk=Hk, dk=dk, dv=dv, z=None if z is None else dev_tensor(z, kind),
                                  norm_w=torch.from_numpy(nw).to(DEV) if gate else None)
        o_ref, cs_n, st_o = oracle.decode_layer_step(x, cw, cs_o, g, b, st_o, dtype=kind, H=H, Hk=Hk,
                                                     dk=dk, dv=dv, z=z, norm_w=nw if gate else None)
        if K > 1:
            cs_o = to(cs_n) if kind == "bf16" else cs_n
        worst = max(worst, err(host(o), o_ref))
    gdn.check_device_status(DEV)
    tol_ = TOL_BF16 if kind == "bf16" else TOL_F32
    assert worst <= tol_
    assert err(host(st_d), st_o) <= tol_
    if K > 1:
        assert np.array_equal(host(cs_d), (gi.bf16_bits_to_f32(cs_o) if kind == "bf16" else cs_o)
                              .astype(np.float32))


@pytest.mark.parametrize("kind,dk,dv", [("f32", 128, 128), ("bf16", 48, 80), ("bf16", 16, 32)])
def test_decode_step_many_units_per_sm(kind, dk, dv):
    """More (sequence, head) units than SMs, shapes with 1, 4 and 16 state rows
    per thread."""
    r = np.random.default_rng(47)
    N, H = 70, 9
    q, k = r.normal(size=(N, H, dk)).astype(np.float32), r.normal(size=(N, H, dk)).astype(np.float32)
    v = r.normal(size=(N, H, dv)).astype(np.float32)
    if kind == "bf16":
        q, k, v = gi.to_bf16_bits(q), gi.to_bf16_bits(k), gi.to_bf16_bits(v)
    g = -np.abs(r.normal(size=(N, H))).astype(np.float32)
    beta = r.uniform(size=(N, H)).astype(np.float32)
    s0 = r.normal(0, 0.1, size=(N, H, dk, dv)).astype(np.float32)
    state = dev_tensor(s0, "f32")
    o = gdn.decode_step(dev_tensor(q, kind), dev_tensor(k, kind), dev_tensor(v, kind),
                        dev_tensor(g, "f32"), dev_tensor(beta, "f32"), state, scale=0.7)
    gdn.check_device_status(DEV)
    o_ref, s_ref = oracle.recurrence(q, k, v, g, beta, np.arange(N + 1), dtype=kind, h0=s0,
                                     scale=0.7)
    assert err(host(o), o_ref) <= tol(kind)
    assert err(host(state), s_ref) <= TOL_F32


def test_decode_layer_step_equals_separate_kernels():
    """The fused step equals conv_silu, then decode_step, then gated_rmsnorm run as
    three library calls (fp32, same arithmetic order up to rounding)."""
    r = np.random.default_rng(33)
    N, H, dk, dv, K = 4, 2, 32, 64, 4
    C = 2 * H * dk + H * dv
    x = torch.from_numpy(r.normal(size=(N, C)).astype(np.float32)).to(DEV)
    cw = torch.from_numpy((r.normal(size=(C, K)) * 0.5).astype(np.float32)).to(DEV)
    cs = torch.from_numpy(r.normal(size=(N, C, K - 1)).astype(np.float32)).to(DEV)
    st = torch.from_numpy((r.normal(size=(N, H, dk, dv)) * 0.1).astype(np.float32)).to(DEV)
    z = torch.from_numpy(r.normal(size=(N, H, dv)).astype(np.float32)).to(DEV)
    nw = torch.from_numpy((1.0 + 0.1 * r.normal(size=dv)).astype(np.float32)).to(DEV)
    g = torch.from_numpy((-np.abs(r.normal(size=(N, H)))).astype(np.float32)).to(DEV)
    b = torch.from_numpy((1.0 / (1.0 + np.exp(-r.normal(size=(N, H))))).astype(np.float32)).to(DEV)
    cs2, st2 = cs.clone(), st.clone()
    o = gdn.decode_layer_step(x, cw, cs, g, b, st, H=H, dk=dk, dv=dv, z=z, norm_w=nw)
    cu = torch.arange(N + 1, dtype=torch.int32, device=DEV)
    y, _ = gdn.conv_silu(x, cw, cu, conv_state=cs2, conv_state_out=cs2, n_qk_channels=2 * H * dk,
                         head_dim=dk)
    q = y[:, :H * dk].reshape(N, H, dk).contiguous()
    k = y[:, H * dk:2 * H * dk].reshape(N, H, dk).contiguous()
    v = y[:, 2 * H * dk:].reshape(N, H, dv).contiguous()
    o2 = gdn.decode_step(q, k, v, g, b, st2, qk_l2norm=False)
    o2 = gdn.gated_rmsnorm(o2, z, nw)
    gdn.check_device_status(DEV)
    assert err(host(o), host(o2)) <= 1e-5
    assert err(host(st), host(st2)) <= 1e-5
    assert torch.equal(cs, cs2)


# ----------------------------------------------------------------------------
# backward
# ----------------------------------------------------------------------------

def _backward_case(P, seed, with_dhT, keep_states=False):
    from oracle import backward as ob
    r = np.random.default_rng(seed)
    T, N = P.T_tot, P.N
    do = r.normal(size=(T, P.H, P.dv)).astype(np.float32)
    dhT = r.normal(size=(N, P.H, P.dk, P.dv)).astype(np.float32) if with_dhT else None
    dec = (lambda a: gi.bf16_bits_to_f32(a).astype(np.float64)) if P.dtype == "bf16" else (
        lambda a: np.asarray(a, np.float64))
    ref = ob.recurrence_backward(dec(P.q), dec(P.k), dec(P.v), P.g, P.beta, P.cu_seqlens, do, dhT,
                                 h0=P.h0, scale=P.scale, qk_l2norm=P.qk_l2norm, eps=P.eps)
    got = gdn.backward(dev_tensor(P.q, P.dtype), dev_tensor(P.k, P.dtype), dev_tensor(P.v, P.dtype),
                       dev_tensor(P.g, "f32"), dev_tensor(P.beta, "f32"),
                       torch.from_numpy(P.cu_seqlens.astype(np.int32)).to(DEV),
                       dev_tensor(do, "f32"),
                       initial_state=None if P.h0 is None else dev_tensor(P.h0, "f32"),
                       dhT=None if dhT is None else dev_tensor(dhT, "f32"), scale=P.scale,
                       qk_l2norm=P.qk_l2norm, eps=P.eps,
                       cu_seqlens_host=torch.from_numpy(P.cu_seqlens.astype(np.int32)),
                       keep_states=keep_states)
    gdn.check_device_status(DEV)
    return [host(x) for x in got], ref


@pytest.mark.parametrize("keep_states", [False, True])
@pytest.mark.parametrize("kind,H,Hk,dk,dv,with_h0,with_dhT", [
    ("bf16", 2, 2, 128, 128, True, True),
    ("f32", 4, 2, 64, 48, False, True),
    ("f32", 3, 3, 32, 128, True, False),
])
def test_backward_matches_oracle(kind, H, Hk, dk, dv, with_h0, with_dhT, keep_states):
    """Gradients of q, k, v, g, beta and h0 against autograd of the fp64 oracle:
    ragged sequences (an empty one, one shorter than a checkpoint block, one spanning
    several blocks), grouped heads, with and without initial state and final-state
    gradient, with the states recomputed per 16-token block or all kept from the
    forward pass. The inputs are the same values on both sides; the kernel computes in fp32."""
    P = gi.random_prefill(19, [40, 0, 7, 35], H=H, Hk=Hk, dk=dk, dv=dv, dtype=kind,
                          with_h0=with_h0, scale=0.9)
    got, ref = _backward_case(P, 20, with_dhT, keep_states)
    for name, a_, b_ in zip(["dq", "dk", "dv", "dg", "dbeta", "dh0"], got, ref):
        assert err(a_, b_) <= TOL_F32, name


def test_backward_without_l2norm():
    P = gi.random_prefill(21, [33, 18], H=2, dk=16, dv=16, dtype="f32", with_h0=True,
                          qk_l2norm=False)
    P.q *= 0.25
    P.k *= 0.25
    got, ref = _backward_case(P, 22, True)
    for name, a_, b_ in zip(["dq", "dk", "dv", "dg", "dbeta", "dh0"], got, ref):
        assert err(a_, b_) <= TOL_F32, name


# ----------------------------------------------------------------------------
# full-size workloads
# ----------------------------------------------------------------------------

def test_layer_0p8b_conv_then_prefill():
    """One 0.8B-shaped layer: T=4096, 16 heads of 128, conv + SiLU + L2 norm,
    chunked prefill (chunk 64), fp32 final state; every element checked."""
    Lw = gi.layer_0p8b()
    T, H, d = Lw.T_tot, Lw.H, Lw.dk
    cu = torch.from_numpy(Lw.cu_seqlens).to(DEV)
    y, _ = gdn.conv_silu(dev_tensor(Lw.mixed_qkv, "bf16"), dev_tensor(Lw.conv_w, "bf16"), cu,
                         n_qk_channels=2 * H * d, head_dim=d)
    qkv = y.view(T, 3, H, d)
    q, k, v = (qkv[:, i] for i in range(3))  # token-strided views of the conv output
    o, hT = gdn.prefill(q, k, v, dev_tensor(Lw.g, "f32"), dev_tensor(Lw.beta, "f32"), cu,
                        qk_l2norm=False)
    gdn.check_device_status(DEV)
    y_ref, _ = oracle.conv_silu(Lw.mixed_qkv, Lw.conv_w, Lw.cu_seqlens, dtype="bf16",
                                qk_l2norm=True, n_qk=2 * H * d, head_dim=d)
    assert err(host(y), y_ref) <= 1e-2
    yr = y_ref.reshape(T, 3, H, d)
    o_ref, h_ref = oracle.recurrence(yr[:, 0], yr[:, 1], yr[:, 2], Lw.g, Lw.beta, Lw.cu_seqlens,
                                     dtype="f64", qk_l2norm=False)
    assert err(host(o), o_ref) <= TOL_BF16
    assert err(host(hT), h_ref) <= TOL_BF16


def _layer_inputs(seed, lens, H, Hk, K, with_state, with_h0, gate, d=128):
    """Seeded layer-prefill inputs: pre-conv x [T, C] bf16, taps, conv windows,
    gates, initial state and the output gate."""
    C = 2 * Hk * d + H * d
    x, w, cu, st = gi.random_mixed(seed, lens, C, K=K, dtype="bf16", with_state=with_state)
    r = np.random.default_rng(np.random.SeedSequence([3000, seed]))
    T, N = int(cu[-1]), len(lens)
    g = (-np.log1p(np.exp(r.normal(size=(T, H)) + 1.0))).astype(np.float32)
    beta = (1.0 / (1.0 + np.exp(-r.normal(size=(T, H))))).astype(np.float32)
    h0 = (r.normal(size=(N, H, d, d)) * 0.1).astype(np.float32) if with_h0 else None
    z = gi.to_bf16_bits(r.normal(size=(T, H, d)).astype(np.float32)) if gate else None
    nw = (1.0 + 0.1 * r.normal(size=d)).astype(np.float32) if gate else None
    return dict(x=x, w=w, cu=cu, st=st, g=g, beta=beta, h0=h0, z=z, nw=nw, H=H, Hk=Hk, d=d)


def _layer_oracle(L, undecayed=False):
    """The oracle's conv + SiLU (fp64, unnormalised), then its recurrence with
    the L2 norms of q and k, then the gate."""
    H, Hk, d = L["H"], L["Hk"], L["d"]
    y, st_out = oracle.conv_silu(L["x"], L["w"], L["cu"], dtype="bf16", state_in=L["st"])
    T = y.shape[0]
    q = y[:, :Hk * d].reshape(T, Hk, d)
    k = y[:, Hk * d:2 * Hk * d].reshape(T, Hk, d)
    v = y[:, 2 * Hk * d:].reshape(T, H, d)
    o, hT = oracle.recurrence(q, k, v, L["g"], L["beta"], L["cu"], dtype="f64", h0=L["h0"],
                              qk_l2norm=True, undecayed=undecayed)
    if L["z"] is not None:
        o = oracle.gated_rmsnorm(o, gi.bf16_bits_to_f32(L["z"]).astype(np.float64), L["nw"], dtype="f64")
    return o, hT, st_out


def _layer_gpu(L, undecayed=False, in_place_state=False, workspace=None):
    cu = torch.from_numpy(L["cu"].astype(np.int32)).to(DEV)
    st_in = None if L["st"] is None else dev_tensor(L["st"], "bf16")
    K = L["w"].shape[1]
    st_out = st_in if in_place_state else torch.empty((len(L["cu"]) - 1, L["x"].shape[1], K - 1),
                                                      dtype=torch.bfloat16, device=DEV)
    o, hT = gdn.prefill_layer(dev_tensor(L["x"], "bf16"), dev_tensor(L["w"], "bf16"),
                              dev_tensor(L["g"], "f32"), dev_tensor(L["beta"], "f32"), cu,
                              H=L["H"], Hk=L["Hk"], conv_state_in=st_in, conv_state_out=st_out,
                              initial_state=None if L["h0"] is None else dev_tensor(L["h0"], "f32"),
                              undecayed=undecayed,
                              z=None if L["z"] is None else dev_tensor(L["z"], "bf16"),
                              norm_w=None if L["nw"] is None else dev_tensor(L["nw"], "f32"),
                              workspace=workspace)
    gdn.check_device_status(DEV)
    return host(o), host(hT), host(st_out)


@pytest.mark.parametrize("lens,H,Hk,K,with_state,with_h0,gate,undecayed,in_place", [
    ([130, 0, 64, 1, 200, 3], 2, 2, 4, True, True, True, False, False),
    ([130, 0, 64, 1, 200, 3], 2, 2, 4, True, False, False, False, True),
    ([70, 129, 5], 4, 2, 3, False, True, False, True, False),
    ([70, 129, 5], 2, 1, 2, True, False, True, False, False),
    ([100, 2], 2, 2, 1, False, False, False, False, False),
])
def test_prefill_layer_matches_oracle(lens, H, Hk, K, with_state, with_h0, gate, undecayed, in_place):
    """The conv fused into the tensor-core prefill against the oracle's conv,
    recurrence and gate: every element of o and hT, and the conv windows out
    bit-exact (a copy of inputs). Ragged, empty and one-token sequences, conv
    windows reaching into the caller's state, grouped heads, K = 1 .. 4, the
    read-before-decay order and the conv state updated in place."""
    L = _layer_inputs(70 + K + H, lens, H, Hk, K, with_state, with_h0, gate)
    o, hT, st = _layer_gpu(L, undecayed=undecayed, in_place_state=in_place and with_state)
    o_ref, h_ref, st_ref = _layer_oracle(L, undecayed=undecayed)
    assert err(o, o_ref) <= TOL_BF16
    assert err(hT, h_ref) <= TOL_BF16
    if K > 1:
        assert np.array_equal(st, gi.bf16_bits_to_f32(gi.to_bf16_bits(st_ref.astype(np.float32))))


def test_prefill_layer_equals_conv_then_prefill():
    """Fused and two-call layer (gdn_conv_silu without the norms, then
    gdn_prefill with them on strided views of its output) agree to bf16
    rounding of the conv output."""
    L = _layer_inputs(81, [300, 17, 0, 96], 2, 2, 4, True, True, False)
    o, hT, _ = _layer_gpu(L)
    H, d = 2, 128
    cu = torch.from_numpy(L["cu"].astype(np.int32)).to(DEV)
    y, _ = gdn.conv_silu(dev_tensor(L["x"], "bf16"), dev_tensor(L["w"], "bf16"), cu,
                         conv_state=dev_tensor(L["st"], "bf16"), qk_l2norm=False)
    T = y.shape[0]
    qkv = y.view(T, 3, H, d)
    o2, h2 = gdn.prefill(qkv[:, 0], qkv[:, 1], qkv[:, 2], dev_tensor(L["g"], "f32"),
                         dev_tensor(L["beta"], "f32"), cu, initial_state=dev_tensor(L["h0"], "f32"))
    gdn.check_device_status(DEV)
    assert err(o, host(o2)) <= 1e-2 and err(hT, host(h2)) <= 1e-2


@pytest.mark.parametrize("lens,H,Hk,with_state,undecayed,in_place", [
    ([4096], 2, 2, True, False, True),
    ([3000, 0, 5000], 2, 1, True, True, False),
    ([2500, 700], 2, 2, False, False, False),
])
def test_prefill_layer_sequence_split(lens, H, Hk, with_state, undecayed, in_place):
    """Few units, so the prefill runs as the sequence split. With the layer
    workspace the conv goes first into it (once) and the split prefill reads y;
    with the prefill's workspace the conv stays fused into all three passes
    (segments that start inside a sequence take their conv window from x, the
    v = 0 pass leaves v unconvolved); with only the schedule's workspace the
    fused prefill runs in one pass. All three against the oracle, with the conv
    state updated in place (read before it is rewritten) and the
    read-before-decay order."""
    L = _layer_inputs(90 + len(lens), lens, H, Hk, 4, with_state, True, False)
    N, T = len(lens), int(L["cu"][-1])
    pre = gdn.prefill_workspace_size(N, T, H, 128, 128)
    assert pre > 256 + (4 * N + 255) // 256 * 256  # the split applies
    assert gdn.prefill_layer_workspace_size(N, T, H, Hk) >= pre + T * (2 * Hk + H) * 128 * 2
    o, hT, st = _layer_gpu(L, undecayed=undecayed, in_place_state=in_place)
    o_f, h_f, st_f = _layer_gpu(L, undecayed=undecayed, in_place_state=in_place,
                                workspace=torch.empty(pre, dtype=torch.uint8, device=DEV))
    base_ws = torch.empty(256 + (4 * N + 255) // 256 * 256, dtype=torch.uint8, device=DEV)
    o1, h1, _ = _layer_gpu(L, undecayed=undecayed, workspace=base_ws)
    o_ref, h_ref, st_ref = _layer_oracle(L, undecayed=undecayed)
    st_bits = gi.bf16_bits_to_f32(gi.to_bf16_bits(st_ref.astype(np.float32)))
    for oo, hh in ((o, hT), (o_f, h_f), (o1, h1)):
        assert err(oo, o_ref) <= TOL_BF16 and err(hh, h_ref) <= TOL_BF16
    assert np.array_equal(st, st_bits) and np.array_equal(st_f, st_bits)


def test_prefill_layer_more_units_than_sms():
    """40 sequences x 4 heads (160 units on 148 SMs): CTAs move from unit to
    unit, reloading taps and conv windows at each unit's first chunk."""
    lens = [(37 * i) % 150 + 1 for i in range(40)]
    L = _layer_inputs(95, lens, 4, 4, 4, True, False, False)
    o, hT, _ = _layer_gpu(L)
    o_ref, h_ref, _ = _layer_oracle(L)
    assert err(o, o_ref) <= TOL_BF16 and err(hT, h_ref) <= TOL_BF16


def test_layer_0p8b_prefill_layer():
    """The 0.8B-shaped layer (T=4096, 16 heads of 128) through gdn_prefill_layer
    with its default workspace (the prefill splits, so the conv runs first, once),
    every element against the oracle."""
    Lw = gi.layer_0p8b()
    L = dict(x=Lw.mixed_qkv, w=Lw.conv_w, cu=np.asarray(Lw.cu_seqlens), st=None, g=Lw.g,
             beta=Lw.beta, h0=None, z=None, nw=None, H=Lw.H, Hk=Lw.H, d=Lw.dk)
    o, hT, _ = _layer_gpu(L)
    o_ref, h_ref, _ = _layer_oracle(L)
    assert err(o, o_ref) <= TOL_BF16 and err(hT, h_ref) <= TOL_BF16


@pytest.mark.parametrize("lengths,H,Hk,undecayed,with_h0,in_place", [
    ([3000, 0, 1400, 4200], 2, 1, False, True, True),
    ([4096], 8, 8, True, False, False),
    ([640, 9000], 2, 2, False, True, False),
])
def test_prefill_sequence_split(lengths, H, Hk, undecayed, with_h0, in_place):
    """Few (sequence, head) units: the sequences are cut into segments (zero-
    and identity-start passes, the fp32 chain of segment start states, then
    the output pass). Every element against the oracle, and against the plain
    launch, which a workspace of only the schedule's size selects. Covers an
    empty sequence, sequences with fewer chunks than segments, grouped heads,
    the read-before-decay order and hT == h0 in place."""
    P = gi.random_prefill(61 + H, lengths, H=H, dk=128, dv=128, with_h0=with_h0, Hk=Hk)
    assert gdn.prefill_workspace_size(P.N, P.T_tot, H, 128, 128) > 256 + 4 * P.N + 255  # splits
    q, k, v = (dev_tensor(a, "bf16") for a in (P.q, P.k, P.v))
    g, beta = dev_tensor(P.g, "f32"), dev_tensor(P.beta, "f32")
    cu = torch.from_numpy(P.cu_seqlens.astype(np.int32)).to(DEV)
    h0 = dev_tensor(P.h0, "f32") if with_h0 else None
    h0_copy = None if h0 is None else h0.clone()
    o, hT = gdn.prefill(q, k, v, g, beta, cu, initial_state=h0, undecayed=undecayed,
                        final_state=h0 if in_place else None)
    gdn.check_device_status(DEV)
    base_ws = torch.empty(256 + (4 * P.N + 255) // 256 * 256, dtype=torch.uint8, device=DEV)
    o1, h1 = gdn.prefill(q, k, v, g, beta, cu, initial_state=h0_copy, undecayed=undecayed,
                         workspace=base_ws)
    gdn.check_device_status(DEV)
    o_ref, h_ref = prefill_oracle(P, undecayed=undecayed)
    assert err(host(o), o_ref) <= TOL_BF16 and err(host(hT), h_ref) <= TOL_BF16
    assert err(host(o1), o_ref) <= TOL_BF16 and err(host(h1), h_ref) <= TOL_BF16
    assert err(host(o), host(o1)) <= TOL_BF16


def _check_sequences(P, seqs, o, hT):
    worst = 0.0
    for n in seqs:
        a, b = int(P.cu_seqlens[n]), int(P.cu_seqlens[n + 1])
        o_ref, h_ref = oracle_seq(P, n)
        worst = max(worst, err(o[a:b], o_ref), err(hT[n], h_ref))
    return worst


def test_long_prefill_full_size_every_element():
    """The headline workload (8 x 16384 tokens, 16 heads, d = 128, bf16): every
    output element and every final-state element against the oracle."""
    P = gi.long_prefill()
    o, hT = prefill_gpu(P)
    assert np.isfinite(o).all() and np.isfinite(hT).all()
    worst = _check_sequences(P, range(P.N), o, hT)
    assert worst <= TOL_BF16, worst


def test_varlen_full_size_sixteen_sequences():
    """The 64-sequence packed workload with initial states: every element of 16
    sequences (all heads) against the oracle -- the four longest, four short and
    eight from the middle of the longest-first order. Unit u = rank * H + h runs
    on CTA u mod grid, so every unit past the first 148 is a CTA's second or
    later unit: the middle and short ones are (8 sequences x 16 heads)."""
    P = gi.varlen()
    order = longest_first(P.cu_seqlens)
    ranks = [0, 1, 2, 3, 20, 21, 22, 23, 40, 41, 42, 43, 60, 61, 62, 63]
    sms = torch.cuda.get_device_properties(DEV).multi_processor_count
    assert sum(1 for r in ranks for h in range(P.H) if r * P.H + h >= sms) >= 8
    o, hT = prefill_gpu(P)
    assert np.isfinite(o).all() and np.isfinite(hT).all()
    worst = _check_sequences(P, [int(order[r]) for r in ranks], o, hT)
    assert worst <= TOL_BF16, worst


# ----------------------------------------------------------------------------
# device-side argument checks
# ----------------------------------------------------------------------------

def test_bad_device_seqlens_reported_not_faulted():
    P = gi.random_prefill(11, [64, 64], H=1, dk=32, dv=32, dtype="f32")
    bad = torch.tensor([0, 100, 64], dtype=torch.int32, device=DEV)  # decreasing, no host copy
    q, k, v = (dev_tensor(a, "f32") for a in (P.q, P.k, P.v))
    g, beta = dev_tensor(P.g, "f32"), dev_tensor(P.beta, "f32")
    gdn.prefill(q, k, v, g, beta, bad)
    with pytest.raises(gdn.GDNError, match="INVALID_ARG"):
        gdn.check_device_status(DEV)
    x = torch.zeros((128, 384), dtype=torch.float32, device=DEV)
    gdn.conv_silu(x, torch.zeros((384, 4), device=DEV), bad, qk_l2norm=False)
    with pytest.raises(gdn.GDNError, match="INVALID_ARG"):
        gdn.check_device_status(DEV)
    # the context is still usable
    o, hT = prefill_gpu(P)
    o_ref, h_ref = prefill_oracle(P)
    assert err(o, o_ref) <= TOL_F32
