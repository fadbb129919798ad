#!/usr/bin/env python
"""Benchmark of the Gated DeltaNet token mixer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline workload (one step): chunked gated-delta-rule prefill of 8 sequences x
16384 tokens, 16 heads, d_k = d_v = 128, bf16 q/k/v, fp32 gates and fp32 final
state, chunk 64 -- one gdn_prefill call over the packed batch. Inputs stay
resident in HBM (q, k, v, gates and o: about 2.2 GB, far larger than the 126 MB L2). The same JSON line
carries two more measured workloads of the same hot path: batched decode
(256 sequences, 100 in-place steps) and one 0.8B-shaped layer prefill
(conv + SiLU + L2 norm, then the chunked prefill, T = 4096).

Multi-GPU: one process per GPU (torchrun), each rank runs its own replica of
the workload (weak scaling, no data-path collective); the step time is the max
over ranks.

--impl reference times the CPU oracle (fp64, C, host threads) on a bounded
sample of the same workload; it is the reference arm of this benchmark.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN prefill tokens/s & % bf16 TC roofline; decode tokens/s & % HBM BW (1×B200)"
UNIT = "tokens/s"
H, D, CHUNK = 16, 128, 64
SEQS, SEQ_LEN = 8, 16384
# Algorithmic work per (token, head) of the chunked prefill (chunk C, d = 128):
# five C x C x d products and three C x d x d products, 2 flops per MAC.
FLOP_PER_TOKEN_HEAD = 10 * CHUNK * D + 6 * D * D          # 180,224
# q, k, v, o in bf16 plus g, beta in fp32.
BYTES_PER_TOKEN_HEAD = 3 * D * 2 + D * 2 + 2 * 4          # 1,032
STATE_BYTES = D * D * 4                                    # per (sequence, head)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "gated_deltanet_linear_silu_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, sources, units_this_launch: float):
    """dram bytes per launch from the committed ncu summary, scaled to this
    launch's units; None when the kernel source changed since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(kernel)
    if not rec or rec.get("source_hash") != source_hash(*sources):
        return None
    return rec["dram_bytes_per_unit"] * units_this_launch


# ----------------------------------------------------------------------------
# clocks during the timed regions
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index: int):
        self.samples, self.proc, self.err = [], None, None
        self.active = False
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            target = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            target = str(device_index)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", target, f"--query-gpu={','.join(self.FIELDS)}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception as e:  # no nvidia-smi
            self.err = str(e)

    def _read(self):
        for line in self.proc.stdout:
            if self.active:
                self.samples.append([x.strip() for x in line.split(",")])

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        sm = [float(s[0]) for s in self.samples if len(s) >= 7 and s[0].replace(".", "").isdigit()]
        mx = [float(s[1]) for s in self.samples if len(s) >= 7 and s[1].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for s in self.samples:
            if len(s) >= 7:
                for nm, val in zip(names, s[3:7]):
                    if val.lower() == "active":
                        reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------
# distributed plumbing (barrier + max over ranks only)
# ----------------------------------------------------------------------------

class Dist:
    def __init__(self, want: int):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False
        if self.world != want:
            raise SystemExit(f"--gpus {want} but WORLD_SIZE={self.world}")

    def init(self):
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(self.local)
        if self.world > 1:
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", self.local))
            self.pg = True

    def barrier(self):
        if self.pg:
            import torch.distributed as dist
            dist.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        import torch
        import torch.distributed as dist
        t = torch.tensor([x], dtype=torch.float64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as dist
            dist.destroy_process_group()


# ----------------------------------------------------------------------------
# CPU oracle (the reference arm and the cpu_baseline)
# ----------------------------------------------------------------------------

def oracle_sample(P, tokens: int, n_seq: int):
    """Oracle over the first `tokens` tokens of the first n_seq sequences, all
    heads. Returns (token count processed, seconds, threads)."""
    import numpy as np
    import oracle
    qs, ks, vs, gs, bs, cu = [], [], [], [], [], [0]
    for n in range(n_seq):
        a = int(P.cu_seqlens[n])
        b = min(int(P.cu_seqlens[n + 1]), a + tokens)
        for lst, arr in ((qs, P.q), (ks, P.k), (vs, P.v), (gs, P.g), (bs, P.beta)):
            lst.append(arr[a:b])
        cu.append(cu[-1] + (b - a))
    cat = lambda xs: np.ascontiguousarray(np.concatenate(xs))
    threads = min(oracle.default_threads(), n_seq * P.H)
    t0 = time.perf_counter()
    oracle.recurrence(cat(qs), cat(ks), cat(vs), cat(gs), cat(bs), cu, dtype=P.dtype,
                      qk_l2norm=P.qk_l2norm, threads=threads, want_o=True)
    return cu[-1], time.perf_counter() - t0, threads


def calibrated_sample(P, target_s: float):
    """Pick (tokens, n_seq) so one oracle pass takes about target_s seconds
    (at most the whole workload): a prefix of every sampled sequence while
    that fits, whole sequences beyond it."""
    import oracle
    n0 = max(1, min(P.N, oracle.default_threads() // P.H or 1))  # sequences filling the cores
    tok, dt, _ = oracle_sample(P, 512, n0)
    budget = tok / max(dt, 1e-6) * target_s  # tokens the cores get through in target_s
    if budget <= n0 * SEQ_LEN:
        return int(max(256, budget / n0)), n0
    return SEQ_LEN, int(min(P.N, math.ceil(budget / SEQ_LEN)))


def run_reference(args, dist: Dist):
    import gdn_inputs as gi
    if dist.rank != 0:
        return
    P = gi.long_prefill(SEQS, SEQ_LEN, H, D)
    tokens, n_seq = calibrated_sample(P, 3.0)
    for _ in range(args.warmup):
        oracle_sample(P, min(tokens, 1024), n_seq)
    times, toks, threads = [], 0, 1
    for _ in range(args.steps):
        tk, dt, threads = oracle_sample(P, tokens, n_seq)
        times.append(dt)
        toks = tk
    step_s = statistics.mean(times)
    value = toks / step_s
    sample = f"first {tokens} tokens of {n_seq} of the 8 sequences, all 16 heads, fp64 token loop"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(args.gpus),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def config_block(n):
    return {"workload": f"long_prefill_{SEQS}x{SEQ_LEN}_h16_d128_bf16", "global_batch": SEQS * n,
            "seq_len": SEQ_LEN, "heads": H, "head_dim": D, "chunk": CHUNK,
            "parallelism": f"replicas{n}" if n > 1 else "single",
            "l2": f"inputs larger than L2 ({resident_bytes() / 1e9:.2f} GB resident per step, L2 126 MB)"}


def resident_bytes():
    """q/k/v/o bf16 and g/beta fp32 of the timed prefill: what one step touches."""
    return SEQS * SEQ_LEN * H * (4 * D * 2 + 2 * 4)


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

def timed(fn, steps, stream, per_call=True):
    """Run fn `steps` times between two events; returns (total ms, per-call ms).
    per_call=False records no event between the calls (back-to-back calls may
    then overlap a launch with the previous kernel's tail, as in a user's loop);
    the per-call list is then empty."""
    import torch
    n_ev = steps + 1 if per_call else 2
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    evs[0].record(stream)
    for i in range(steps):
        fn()
        if per_call:
            evs[i + 1].record(stream)
    if not per_call:
        evs[1].record(stream)
    torch.cuda.synchronize()
    per = [evs[i].elapsed_time(evs[i + 1]) for i in range(steps)] if per_call else []
    return evs[0].elapsed_time(evs[-1]), per


def bench_prefill(args, dist, pk):
    import numpy as np
    import torch
    import gated_deltanet_linear_silu_b200 as gdn
    import gdn_inputs as gi

    dev = torch.device("cuda", dist.local)
    P = gi.long_prefill(SEQS, SEQ_LEN, H, D)
    T = P.T_tot

    def pinned(a, dtype):
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16) if dtype == torch.bfloat16
                             else np.ascontiguousarray(a))
        t = t.view(dtype) if dtype == torch.bfloat16 else t
        return t.pin_memory()

    hq, hk, hv = (pinned(a, torch.bfloat16) for a in (P.q, P.k, P.v))
    hg, hb = pinned(P.g, torch.float32), pinned(P.beta, torch.float32)
    hcu = torch.from_numpy(P.cu_seqlens.astype(np.int32)).pin_memory()
    q, k, v, g, beta = (t.to(dev) for t in (hq, hk, hv, hg, hb))
    cu = hcu.to(dev)
    o = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
    hT = torch.empty((SEQS, H, D, D), dtype=torch.float32, device=dev)
    ws = torch.empty(gdn.prefill_workspace_size(SEQS, T, H, D, D, CHUNK), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        gdn.prefill(q, k, v, g, beta, cu, final_state=hT, out=o, workspace=ws, chunk=CHUNK,
                    algo=args.algo)

    for _ in range(args.warmup):
        step()
    gdn.check_device_status(dev)
    dist.barrier()
    torch.cuda.synchronize()
    total_ms, per = timed(step, args.steps, stream)
    dist.barrier()
    total_ms = dist.max(total_ms)
    kernel_ms = dist.max(statistics.mean(per))
    gdn.check_device_status(dev)

    # end to end: pinned host inputs -> device -> library -> host outputs, as a
    # serving loop would run it: two device buffer sets, the host-to-device copy
    # of step i+1 on one copy stream while step i computes, the device-to-host
    # copy of step i on another (PCIe carries both directions at once). Every
    # step's copies are inside the timed region.
    ho = torch.empty((T, H, D), dtype=torch.bfloat16).pin_memory()
    hhT = torch.empty((SEQS, H, D, D), dtype=torch.float32).pin_memory()
    bufs = [dict(q=q, k=k, v=v, g=g, beta=beta, cu=torch.empty_like(cu), o=o, hT=hT)]
    bufs.append({n: torch.empty_like(t) for n, t in bufs[0].items()})
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    done_in = [ev(), ev()]      # inputs of buffer set b are on the device
    done_comp = [ev(), ev()]    # the prefill on buffer set b finished
    done_out = [ev(), ev()]     # the results of buffer set b are on the host
    e2e_i = [0]

    def e2e_step():
        b = e2e_i[0] % 2
        e2e_i[0] += 1
        B = bufs[b]
        with torch.cuda.stream(s_in):
            s_in.wait_event(done_comp[b])  # the previous prefill on this set has read its inputs
            for n, src in (("q", hq), ("k", hk), ("v", hv), ("g", hg), ("beta", hb), ("cu", hcu)):
                B[n].copy_(src, non_blocking=True)
            done_in[b].record(s_in)
        stream.wait_event(done_in[b])
        stream.wait_event(done_out[b])  # the previous results of this set have left
        gdn.prefill(B["q"], B["k"], B["v"], B["g"], B["beta"], B["cu"], final_state=B["hT"], out=B["o"],
                    workspace=ws, chunk=CHUNK, algo=args.algo)
        done_comp[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done_comp[b])
            ho.copy_(B["o"], non_blocking=True)
            hhT.copy_(B["hT"], non_blocking=True)
            done_out[b].record(s_out)

    def e2e_run(n):
        for _ in range(n):
            e2e_step()
        for b in range(2):  # the timed region ends when the last results are on the host
            stream.wait_event(done_out[b])

    e2e_run(2)
    dist.barrier()
    torch.cuda.synchronize()
    e2e_steps = max(1, min(args.steps, 5))
    e2e_ms, _ = timed(lambda: e2e_run(e2e_steps), 1, stream)
    dist.barrier()
    e2e_ms = dist.max(e2e_ms)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hg, hb, hcu))
    d2h = ho.numel() * ho.element_size() + hhT.numel() * hhT.element_size()
    res = {"P": P, "tokens": T, "total_ms": total_ms, "kernel_ms": kernel_ms,
           "e2e_ms_per_step": e2e_ms / e2e_steps, "h2d": h2d, "d2h": d2h}
    del q, k, v, g, beta, o, hT, hq, hk, hv, ho, hhT, bufs
    torch.cuda.empty_cache()
    return res


def bench_prefill_gated(args, dist, pk):
    """The headline prefill with the layer's gated RMSNorm output
    (gdn_prefill_gated: the recurrence, then the gate over o in place), against
    the same call without the gate, alternated on the same inputs."""
    import numpy as np
    import torch
    import gated_deltanet_linear_silu_b200 as gdn
    import gdn_inputs as gi
    dev = torch.device("cuda", dist.local)
    P = gi.long_prefill(SEQS, SEQ_LEN, H, D)
    T = P.T_tot
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)
    q, k, v = bf(P.q), bf(P.k), bf(P.v)
    g, beta = torch.from_numpy(P.g).to(dev), torch.from_numpy(P.beta).to(dev)
    cu = torch.from_numpy(P.cu_seqlens).to(dev)
    r = np.random.default_rng(7)
    z = torch.from_numpy(r.standard_normal((T, H, D), dtype=np.float32)).to(dev).to(torch.bfloat16)
    w = torch.from_numpy((1.0 + 0.1 * r.standard_normal(D)).astype(np.float32)).to(dev)
    o = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
    hT = torch.empty((SEQS, H, D, D), dtype=torch.float32, device=dev)
    ws = torch.empty(gdn.prefill_workspace_size(SEQS, T, H, D, D, CHUNK), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def plain():
        gdn.prefill(q, k, v, g, beta, cu, final_state=hT, out=o, workspace=ws, algo=args.algo)

    def gated():
        gdn.prefill(q, k, v, g, beta, cu, final_state=hT, out=o, workspace=ws, algo=args.algo, z=z,
                    norm_w=w)

    for fn in (plain, gated, plain, gated):
        fn()
    torch.cuda.synchronize()
    reps = max(3, min(args.steps, 10))
    p_ms, g_ms = [], []
    for _ in range(2):
        p_ms.append(timed(plain, reps, stream)[0] / reps)
        g_ms.append(timed(gated, reps, stream)[0] / reps)
    gdn.check_device_status(dev)
    pm, gm = dist.max(min(p_ms)), dist.max(min(g_ms))
    th = T * H
    bytes_g = th * (BYTES_PER_TOKEN_HEAD + 3 * D * 2) + SEQS * H * STATE_BYTES  # + z, o in and out
    res = {"ms": gm, "ms_ungated": pm, "ratio": gm / pm,
           "workload": f"long_prefill_{SEQS}x{SEQ_LEN}_h16_d128_bf16_gated_rmsnorm",
           "roofline": {"bound": "hbm", "achieved": bytes_g / (gm * 1e-3) / 1e9, "peak": pk["hbm_gbs"],
                        "unit": "GB/s", "frac": bytes_g / (gm * 1e-3) / 1e9 / pk["hbm_gbs"],
                        "algorithmic_bytes": bytes_g},
           "gpu_launches": 2 * reps}
    del q, k, v, z, o, hT
    torch.cuda.empty_cache()
    return res


def bench_decode(args, dist, pk):
    """256 sequences x 16 heads, d=128, 100 in-place steps (one call each)."""
    import torch
    import gated_deltanet_linear_silu_b200 as gdn
    import gdn_inputs as gi
    dev = torch.device("cuda", dist.local)
    N, steps = 256, 100
    state = torch.from_numpy(gi.decode_state(N, H, D)).to(dev)
    ins = []
    for s in range(steps):
        Dd = gi.decode_step(s, N, H, D)
        bf = lambda a: torch.from_numpy(a.view("int16")).to(dev).view(torch.bfloat16)
        ins.append((bf(Dd.q), bf(Dd.k), bf(Dd.v), torch.from_numpy(Dd.g).to(dev),
                    torch.from_numpy(Dd.beta).to(dev)))
    o = torch.empty((N, H, D), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    it = iter(range(10 ** 9))

    def step():
        i = next(it) % steps
        gdn.decode_step(*ins[i], state, out=o)

    for _ in range(5):
        step()
    torch.cuda.synchronize()
    total_ms, _ = timed(step, steps, stream, per_call=False)
    total_ms = dist.max(total_ms)
    step_ms = total_ms / steps
    # the same 100 steps captured once in a CUDA graph and replayed (launch cost
    # of the library call and ctypes marshalling out of the loop)
    graph_ms = None
    try:
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            with torch.cuda.graph(g, stream=cap):
                for i in range(steps):
                    gdn.decode_step(*ins[i], state, out=o)
        stream.wait_stream(cap)
        for _ in range(2):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        graph_ms = dist.max(e0.elapsed_time(e1)) / steps
        del g
    except Exception as exc:  # reported, not fatal: the eager number stands
        graph_ms = f"unavailable: {type(exc).__name__}: {exc}"[:200]
    bytes_step = 2 * N * H * STATE_BYTES + N * H * (4 * D * 2 + 8)
    return {"value": N / (step_ms * 1e-3) * dist.world, "unit": UNIT, "ms_per_step": step_ms,
            "ms_per_step_graph": graph_ms,
            "workload": "decode_256x16_d128_100steps",
            "roofline": {"bound": "hbm", "achieved": bytes_step / (step_ms * 1e-3) / 1e9,
                         "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": bytes_step / (step_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                         "traffic": profiled_traffic("decode_step_kernel", ["decode.cu"], N * H),
                         "algorithmic_bytes": bytes_step},
            "gpu_launches": steps}


def bench_varlen(args, dist, pk):
    """64 packed sequences of 256..32768 tokens (about 1.06 M), 16 heads, h0 and hT."""
    import numpy as np
    import torch
    import gated_deltanet_linear_silu_b200 as gdn
    import gdn_inputs as gi
    dev = torch.device("cuda", dist.local)
    P = gi.varlen()
    T = int(P.cu_seqlens[-1])
    bf = lambda a: torch.from_numpy(a.view("int16")).to(dev).view(torch.bfloat16)
    q, k, v = bf(P.q), bf(P.k), bf(P.v)
    g, beta = torch.from_numpy(P.g).to(dev), torch.from_numpy(P.beta).to(dev)
    cu = torch.from_numpy(P.cu_seqlens).to(dev)
    h0 = torch.from_numpy(P.h0).to(dev)
    N = P.N
    o = torch.empty_like(q)
    hT = torch.empty_like(h0)
    ws = torch.empty(gdn.prefill_workspace_size(N, T, H, D, D, CHUNK), dtype=torch.uint8, device=dev)
    host_cu = torch.from_numpy(P.cu_seqlens)
    del P
    stream = torch.cuda.current_stream(dev)

    def step():
        gdn.prefill(q, k, v, g, beta, cu, initial_state=h0, final_state=hT, out=o, workspace=ws,
                    cu_seqlens_host=host_cu)

    for _ in range(2):
        step()
    torch.cuda.synchronize()
    reps = 5
    total_ms, _ = timed(step, reps, stream)
    ms = dist.max(total_ms) / reps
    flops = T * H * FLOP_PER_TOKEN_HEAD
    byts = T * H * BYTES_PER_TOKEN_HEAD + 2 * N * H * STATE_BYTES
    # per-CTA work of the tensor-core kernel: (sequence, head) units in longest-first
    # order; CTA c starts with unit c and each later unit goes to the CTA that runs
    # out of work first (the kernel's work counter), emulated in tokens
    import heapq
    lens = np.diff(host_cu.numpy().astype(np.int64))
    order = sorted(range(N), key=lambda n: (-int(lens[n]), n))
    grid = min(torch.cuda.get_device_properties(dev).multi_processor_count, N * H)
    work = np.zeros(grid)
    heap = []
    for u in range(N * H):
        c = u if u < grid else heapq.heappop(heap)[1]
        work[c] += lens[order[u // H]]
        heapq.heappush(heap, (work[c], c))
    return {"value": T / (ms * 1e-3) * dist.world, "unit": UNIT, "ms_per_step": ms,
            "workload": f"varlen_64seqs_{T}tok_h16_d128_bf16_h0",
            "tc_roofline": {"achieved": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                            "peak": pk["bf16_tflops"],
                            "frac": flops / (ms * 1e-3) / 1e12 / pk["bf16_tflops"]},
            "roofline": {"bound": "hbm", "achieved": byts / (ms * 1e-3) / 1e9, "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": byts / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                         "algorithmic_bytes": byts},
            "tail_imbalance": {"max_over_mean_cta_tokens": float(work.max() / work.mean()),
                               "ctas": grid}}


def bench_decode_layer(args, dist, pk):
    """The whole mixer for one decode token (conv update + SiLU + L2 norm +
    recurrent step + gated RMSNorm output) in one kernel: 256 sequences x 16
    heads, d=128, conv k=4, 100 in-place steps."""
    import numpy as np
    import torch
    import gated_deltanet_linear_silu_b200 as gdn
    import gdn_inputs as gi
    dev = torch.device("cuda", dist.local)
    N, steps, K = 256, 100, 4
    C = 3 * H * D
    r = np.random.default_rng(7)
    bf = lambda a: torch.from_numpy(gi.to_bf16_bits(a.astype(np.float32)).view("int16")).to(dev) \
        .view(torch.bfloat16)
    state = torch.from_numpy(gi.decode_state(N, H, D)).to(dev)
    conv_state = bf(r.normal(size=(N, C, K - 1)))
    conv_w = bf(r.normal(size=(C, K)) * 0.5)
    norm_w = torch.ones(D, dtype=torch.float32, device=dev)
    ins = []
    for s_ in range(8):  # a few distinct inputs, cycled
        ins.append((bf(r.normal(size=(N, C))), torch.from_numpy(
            (-np.log1p(np.exp(r.normal(size=(N, H))))).astype(np.float32)).to(dev),
            torch.from_numpy((1 / (1 + np.exp(-r.normal(size=(N, H))))).astype(np.float32)).to(dev),
            bf(r.normal(size=(N, H, D)))))
    o = torch.empty((N, H, D), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    it = iter(range(10 ** 9))

    def step():
        x, g, b, z = ins[next(it) % len(ins)]
        gdn.decode_layer_step(x, conv_w, conv_state, g, b, state, H=H, dk=D, dv=D, z=z,
                              norm_w=norm_w, out=o)

    for _ in range(5):
        step()
    torch.cuda.synchronize()
    total_ms, _ = timed(step, steps, stream, per_call=False)
    step_ms = dist.max(total_ms) / steps
    # state in and out, x, conv state in and out, z, o, gates; taps once
    bytes_step = (2 * N * H * STATE_BYTES + N * C * 2 + 2 * N * C * (K - 1) * 2
                  + 2 * N * H * D * 2 + N * H * 8 + C * K * 2)
    return {"value": N / (step_ms * 1e-3) * dist.world, "unit": UNIT, "ms_per_step": step_ms,
            "workload": "decode_layer_256x16_d128_conv4_gated_100steps",
            "roofline": {"bound": "hbm", "achieved": bytes_step / (step_ms * 1e-3) / 1e9,
                         "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": bytes_step / (step_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                         "traffic": profiled_traffic("decode_layer_stream_kernel", ["decode_stream.cu"], N * H),
                         "algorithmic_bytes": bytes_step},
            "gpu_launches": steps}


def bench_grouped(args, dist, pk):
    """Grouped value heads: 32 value heads on 16 q, k heads, d=128. The prefill
    of 8 sequences x 8192 tokens (fp32 final state), and the whole-mixer decode
    step for 256 sequences (a CTA runs the two value heads of a q, k head back
    to back), 100 steps."""
    import numpy as np
    import torch
    import gated_deltanet_linear_silu_b200 as gdn
    import gdn_inputs as gi
    dev = torch.device("cuda", dist.local)
    P = gi.grouped_prefill()
    Hv, Hk, N, T = P.H, P.Hk, P.N, P.T_tot
    bf = lambda a: torch.from_numpy(a.view("int16")).to(dev).view(torch.bfloat16)
    q, k, v = bf(P.q), bf(P.k), bf(P.v)
    g, beta = torch.from_numpy(P.g).to(dev), torch.from_numpy(P.beta).to(dev)
    cu = torch.from_numpy(P.cu_seqlens).to(dev)
    del P
    o = torch.empty((T, Hv, D), dtype=torch.bfloat16, device=dev)
    hT = torch.empty((N, Hv, D, D), dtype=torch.float32, device=dev)
    ws = torch.empty(gdn.prefill_workspace_size(N, T, Hv, D, D, CHUNK), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        gdn.prefill(q, k, v, g, beta, cu, final_state=hT, out=o, workspace=ws, chunk=CHUNK)

    for _ in range(3):
        step()
    gdn.check_device_status(dev)
    torch.cuda.synchronize()
    reps = 5
    total_ms, _ = timed(step, reps, stream)
    ms = dist.max(total_ms) / reps
    flops = T * Hv * FLOP_PER_TOKEN_HEAD
    # q, k once per q, k head; v, o, gates per value head; the final state
    byts = T * (2 * Hk * D * 2 + Hv * (2 * D * 2 + 8)) + N * Hv * STATE_BYTES
    pre = {"value": T / (ms * 1e-3) * dist.world, "unit": UNIT, "ms_per_step": ms,
           "workload": f"grouped_prefill_{N}x{T // N}_hv{Hv}_hk{Hk}_d128_bf16",
           "tc_roofline": {"achieved": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                           "peak": pk["bf16_tflops"],
                           "frac": flops / (ms * 1e-3) / 1e12 / pk["bf16_tflops"]},
           "roofline": {"bound": "hbm", "achieved": byts / (ms * 1e-3) / 1e9, "peak": pk["hbm_gbs"],
                        "unit": "GB/s", "frac": byts / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                        "algorithmic_bytes": byts},
           "gpu_launches": 2 * reps}
    del q, k, v, g, beta, o, hT
    torch.cuda.empty_cache()

    Nd, steps, K = 256, 100, 4
    C = 2 * Hk * D + Hv * D
    r = np.random.default_rng(8)
    bfr = lambda a: torch.from_numpy(gi.to_bf16_bits(a.astype(np.float32)).view("int16")).to(dev) \
        .view(torch.bfloat16)
    state = torch.from_numpy(gi.decode_state(Nd, Hv, D)).to(dev)
    conv_state = bfr(r.normal(size=(Nd, C, K - 1)))
    conv_w = bfr(r.normal(size=(C, K)) * 0.5)
    norm_w = torch.ones(D, dtype=torch.float32, device=dev)
    ins = []
    for _ in range(8):
        ins.append((bfr(r.normal(size=(Nd, C))), torch.from_numpy(
            (-np.log1p(np.exp(r.normal(size=(Nd, Hv))))).astype(np.float32)).to(dev),
            torch.from_numpy((1 / (1 + np.exp(-r.normal(size=(Nd, Hv))))).astype(np.float32)).to(dev),
            bfr(r.normal(size=(Nd, Hv, D)))))
    od = torch.empty((Nd, Hv, D), dtype=torch.bfloat16, device=dev)
    it = iter(range(10 ** 9))

    def dstep():
        x, gg, bb, z = ins[next(it) % len(ins)]
        gdn.decode_layer_step(x, conv_w, conv_state, gg, bb, state, H=Hv, Hk=Hk, dk=D, dv=D, z=z,
                              norm_w=norm_w, out=od)

    for _ in range(5):
        dstep()
    gdn.check_device_status(dev)
    torch.cuda.synchronize()
    total_ms, _ = timed(dstep, steps, stream, per_call=False)
    step_ms = dist.max(total_ms) / steps
    bytes_step = (2 * Nd * Hv * STATE_BYTES + Nd * C * 2 + 2 * Nd * C * (K - 1) * 2
                  + 2 * Nd * Hv * D * 2 + Nd * Hv * 8 + C * K * 2)
    dec = {"value": Nd / (step_ms * 1e-3) * dist.world, "unit": UNIT, "ms_per_step": step_ms,
           "workload": f"decode_layer_{Nd}_hv{Hv}_hk{Hk}_d128_conv4_gated_{steps}steps",
           "roofline": {"bound": "hbm", "achieved": bytes_step / (step_ms * 1e-3) / 1e9,
                        "peak": pk["hbm_gbs"], "unit": "GB/s",
                        "frac": bytes_step / (step_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                        "traffic": profiled_traffic("decode_layer_grouped_kernel", ["decode_stream.cu"],
                                                    Nd * Hv),
                        "algorithmic_bytes": bytes_step},
           "gpu_launches": steps}
    return {"prefill": pre, "decode_layer": dec}


def bench_undecayed(args, dist, pk):
    """The read-before-decay order (memory read from the state before the decay)
    on the headline prefill workload (8 x 16384 tokens, 16 heads, d=128) and on
    the decode workload (256 x 16 heads, 100 in-place steps)."""
    import numpy as np
    import torch
    import gated_deltanet_linear_silu_b200 as gdn
    import gdn_inputs as gi
    dev = torch.device("cuda", dist.local)
    P = gi.long_prefill(SEQS, SEQ_LEN, H, D)
    T = P.T_tot
    bf = lambda a: torch.from_numpy(a.view("int16")).to(dev).view(torch.bfloat16)
    q, k, v = bf(P.q), bf(P.k), bf(P.v)
    g, beta = torch.from_numpy(P.g).to(dev), torch.from_numpy(P.beta).to(dev)
    cu = torch.from_numpy(P.cu_seqlens).to(dev)
    del P
    o = torch.empty_like(v)
    hT = torch.empty((SEQS, H, D, D), dtype=torch.float32, device=dev)
    ws = torch.empty(gdn.prefill_workspace_size(SEQS, T, H, D, D, CHUNK), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        gdn.prefill(q, k, v, g, beta, cu, final_state=hT, out=o, workspace=ws, chunk=CHUNK,
                    undecayed=True)

    for _ in range(3):
        step()
    gdn.check_device_status(dev)
    torch.cuda.synchronize()
    reps = 5
    total_ms, _ = timed(step, reps, stream)
    ms = dist.max(total_ms) / reps
    flops = T * H * FLOP_PER_TOKEN_HEAD
    byts = T * H * BYTES_PER_TOKEN_HEAD + SEQS * H * STATE_BYTES
    pre = {"value": T / (ms * 1e-3) * dist.world, "unit": UNIT, "ms_per_step": ms,
           "workload": f"long_prefill_{SEQS}x{SEQ_LEN}_h16_d128_bf16_undecayed",
           "tc_roofline": {"achieved": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                           "peak": pk["bf16_tflops"],
                           "frac": flops / (ms * 1e-3) / 1e12 / pk["bf16_tflops"]},
           "roofline": {"bound": "hbm", "achieved": byts / (ms * 1e-3) / 1e9, "peak": pk["hbm_gbs"],
                        "unit": "GB/s", "frac": byts / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                        "algorithmic_bytes": byts},
           "gpu_launches": 2 * reps}
    del q, k, v, g, beta, o, hT
    torch.cuda.empty_cache()

    N, steps = 256, 100
    state = torch.from_numpy(gi.decode_state(N, H, D)).to(dev)
    ins = []
    for s_ in range(8):
        Dd = gi.decode_step(s_, N, H, D)
        ins.append((bf(Dd.q), bf(Dd.k), bf(Dd.v), torch.from_numpy(Dd.g).to(dev),
                    torch.from_numpy(Dd.beta).to(dev)))
    od = torch.empty((N, H, D), dtype=torch.bfloat16, device=dev)
    it = iter(range(10 ** 9))

    def dstep():
        qq, kk, vv, gg, bb = ins[next(it) % len(ins)]
        gdn.decode_step(qq, kk, vv, gg, bb, state, out=od, undecayed=True)

    for _ in range(5):
        dstep()
    torch.cuda.synchronize()
    total_ms, _ = timed(dstep, steps, stream, per_call=False)
    step_ms = dist.max(total_ms) / steps
    bytes_step = N * H * (2 * STATE_BYTES + 4 * D * 2 + 8)
    dec = {"value": N / (step_ms * 1e-3) * dist.world, "unit": UNIT, "ms_per_step": step_ms,
           "workload": f"decode_{N}x16_d128_{steps}steps_undecayed",
           "roofline": {"bound": "hbm", "achieved": bytes_step / (step_ms * 1e-3) / 1e9,
                        "peak": pk["hbm_gbs"], "unit": "GB/s",
                        "frac": bytes_step / (step_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                        "algorithmic_bytes": bytes_step},
           "gpu_launches": steps}
    return {"prefill": pre, "decode": dec}


def bench_backward(args, dist, pk):
    """Gradients of the recurrence (fp32 CUDA cores, token by token): 8 sequences x
    4096 tokens, 16 heads, d=128, bf16 q/k/v, fp32 dO and dS_T."""
    import numpy as np
    import torch
    import gated_deltanet_linear_silu_b200 as gdn
    import gdn_inputs as gi
    dev = torch.device("cuda", dist.local)
    N, T1 = SEQS, min(4096, SEQ_LEN)  # --seq-len below 4096 gives a smaller profiling case
    P = gi.long_prefill(N, T1, H, D)
    T = P.T_tot
    bf = lambda a: torch.from_numpy(a.view("int16")).to(dev).view(torch.bfloat16)
    q, k, v = bf(P.q), bf(P.k), bf(P.v)
    g, beta = torch.from_numpy(P.g).to(dev), torch.from_numpy(P.beta).to(dev)
    cu = torch.from_numpy(P.cu_seqlens).to(dev)
    host_cu = torch.from_numpy(P.cu_seqlens)
    del P
    r = np.random.default_rng(9)
    do = torch.from_numpy(r.standard_normal((T, H, D), dtype=np.float32)).to(dev)
    dhT = torch.from_numpy(r.standard_normal((N, H, D, D), dtype=np.float32)).to(dev)
    # the workspace that keeps every token's state from the forward pass (34 GB
    # here): one token-sequential pass fewer than recomputing 16-token blocks
    ws = torch.empty(gdn.lib().gdn_backward_workspace_size_kept(N, T, H, D, D), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        gdn.backward(q, k, v, g, beta, cu, do, dhT=dhT, cu_seqlens_host=host_cu, workspace=ws)

    for _ in range(3):
        step()
    gdn.check_device_status(dev)
    torch.cuda.synchronize()
    reps = 3
    total_ms, _ = timed(step, reps, stream)
    ms = dist.max(total_ms) / reps
    # read q, k, v (bf16), g, beta, dO (fp32), dS_T; write dq, dk, dv (fp32), dg, dbeta, dh0
    per_th = 3 * D * 2 + 8 + D * 4 + 3 * D * 4 + 8
    byts = T * H * per_th + 2 * N * H * STATE_BYTES
    return {"value": T / (ms * 1e-3) * dist.world, "unit": UNIT, "ms_per_step": ms,
            "workload": f"backward_{N}x{T1}_h16_d128_bf16_inputs_fp32_grads",
            "roofline": {"bound": "hbm", "achieved": byts / (ms * 1e-3) / 1e9, "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": byts / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                         "algorithmic_bytes": byts,
                         "note": "token-sequential fp32 kernel: bound by per-token barriers, "
                                 "not by HBM"},
            "gpu_launches": reps}


def bench_gated_norm(args, dist, pk):
    """Gated RMSNorm output over the long-prefill output: 8 x 16384 tokens x 16
    heads, d_v = 128, bf16 (read o and z, write the gated output)."""
    import torch
    import gated_deltanet_linear_silu_b200 as gdn
    dev = torch.device("cuda", dist.local)
    rows = SEQS * SEQ_LEN * H
    gen = torch.Generator(device=dev).manual_seed(11)
    y = torch.randn((rows, D), generator=gen, device=dev).to(torch.bfloat16)
    z = torch.randn((rows, D), generator=gen, device=dev).to(torch.bfloat16)
    w = torch.ones(D, dtype=torch.float32, device=dev)
    out = torch.empty_like(y)
    stream = torch.cuda.current_stream(dev)

    def step():
        gdn.gated_rmsnorm(y, z, w, out=out)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    reps = 10
    total_ms, _ = timed(step, reps, stream)
    ms = dist.max(total_ms) / reps
    byts = 3 * rows * D * 2
    return {"ms": ms, "workload": f"gated_rmsnorm_{rows}x{D}_bf16",
            "roofline": {"bound": "hbm", "achieved": byts / (ms * 1e-3) / 1e9, "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": byts / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                         "traffic": profiled_traffic("gated_rmsnorm_kernel", ["gated_norm.cu"], rows),
                         "algorithmic_bytes": byts}}


def bench_layer(args, dist, pk):
    """0.8B-shaped layer prefill: conv + SiLU + L2 norm, then chunked prefill."""
    import torch
    import gated_deltanet_linear_silu_b200 as gdn
    import gdn_inputs as gi
    dev = torch.device("cuda", dist.local)
    Lw = gi.layer_0p8b()
    T = Lw.T_tot
    bf = lambda a: torch.from_numpy(a.view("int16")).to(dev).view(torch.bfloat16)
    x, w = bf(Lw.mixed_qkv), bf(Lw.conv_w)
    g, beta = torch.from_numpy(Lw.g).to(dev), torch.from_numpy(Lw.beta).to(dev)
    cu = torch.from_numpy(Lw.cu_seqlens).to(dev)
    y = torch.empty_like(x)
    st = torch.empty((1, Lw.C, 3), dtype=torch.bfloat16, device=dev)
    qkv = y.view(T, 3, H, D)
    q, k, v = qkv[:, 0], qkv[:, 1], qkv[:, 2]  # token-strided views: no copies
    o = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
    hT = torch.empty((1, H, D, D), dtype=torch.float32, device=dev)
    ws = torch.empty(gdn.prefill_workspace_size(1, T, H, D, D, CHUNK), dtype=torch.uint8, device=dev)
    flush = torch.empty(512 * 2 ** 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def conv():
        gdn.conv_silu(x, w, cu, conv_state_out=st, out=y, n_qk_channels=2 * H * D, head_dim=D)

    def layer():
        conv()
        gdn.prefill(q, k, v, g, beta, cu, final_state=hT, out=o, workspace=ws, qk_l2norm=False)

    st2 = torch.empty_like(st)
    ws_layer = torch.empty(gdn.prefill_layer_workspace_size(1, T, H, H), dtype=torch.uint8, device=dev)

    def layer_call():  # gdn_prefill_layer with its own workspace: the split applies, so conv first
        gdn.prefill_layer(x, w, g, beta, cu, H=H, conv_state_out=st2, final_state=hT, out=o,
                          workspace=ws_layer)

    def fused():  # the conv inside each of the split's three prefill passes
        gdn.prefill_layer(x, w, g, beta, cu, H=H, conv_state_out=st2, final_state=hT, out=o,
                          workspace=ws)

    conv_ms, layer_ms, call_ms, fused_ms = [], [], [], []
    for rep in range(8):
        for fn, acc in ((conv, conv_ms), (layer, layer_ms), (layer_call, call_ms), (fused, fused_ms)):
            flush.fill_(rep & 0xFF)  # L2 flush: the layer's inputs fit in L2
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record(stream)
            fn()
            e.record(stream)
            torch.cuda.synchronize()
            if rep >= 3:
                acc.append(s.elapsed_time(e))
    cms, lms, ams, fms = (statistics.median(v) for v in (conv_ms, layer_ms, call_ms, fused_ms))
    conv_bytes = 2 * T * Lw.C * 2 + Lw.C * 4 * 2
    return {"value": T / (lms * 1e-3) * dist.world, "unit": UNIT, "ms_per_step": lms,
            "workload": "layer_0p8b_T4096_conv_then_prefill",
            "note": "two launches (conv, prefill); the prefill reads q, k, v as strided views of the conv output",
            "prefill_layer": {"value": T / (ams * 1e-3) * dist.world, "unit": UNIT, "ms_per_step": ams,
                              "note": "gdn_prefill_layer, its own workspace: the prefill splits, so the "
                                      "conv runs first into the workspace"},
            "fused": {"value": T / (fms * 1e-3) * dist.world, "unit": UNIT, "ms_per_step": fms,
                      "note": "gdn_prefill_layer with the prefill's workspace: the conv inside each "
                              "of the split's three passes (no y round trip)"},
            "conv": {"ms": cms, "roofline": {
                "bound": "hbm", "achieved": conv_bytes / (cms * 1e-3) / 1e9, "peak": pk["hbm_gbs"],
                "unit": "GB/s", "frac": conv_bytes / (cms * 1e-3) / 1e9 / pk["hbm_gbs"],
                "traffic": profiled_traffic("conv_silu_kernel", ["conv_silu.cu"], T),
                "algorithmic_bytes": conv_bytes}}}


def bench_layer_long(args, dist, pk):
    """The layer prefill at the headline's size: the long-prefill workload's
    q, k, v side by side as the pre-conv layer input x (8 x 16384 tokens,
    C = 6144), conv taps ~ N(0, 0.5) bf16 (seeded), its gates. Conv then prefill
    (two calls, y through HBM) against gdn_prefill_layer (the conv inside the
    single-pass prefill), alternated; inputs larger than L2."""
    import numpy as np
    import torch
    import gated_deltanet_linear_silu_b200 as gdn
    import gdn_inputs as gi
    dev = torch.device("cuda", dist.local)
    P = gi.long_prefill(SEQS, SEQ_LEN, H, D)
    T = P.T_tot
    C = 3 * H * D
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)
    x = torch.cat([bf(P.q).view(T, -1), bf(P.k).view(T, -1), bf(P.v).view(T, -1)], dim=1).contiguous()
    r = np.random.default_rng(11)
    w = bf(gi.to_bf16_bits((0.5 * r.standard_normal((C, 4))).astype(np.float32)))
    g, beta = torch.from_numpy(P.g).to(dev), torch.from_numpy(P.beta).to(dev)
    cu = torch.from_numpy(P.cu_seqlens).to(dev)
    del P
    y = torch.empty_like(x)
    st = torch.empty((SEQS, C, 3), dtype=torch.bfloat16, device=dev)
    st2 = torch.empty_like(st)
    o = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
    hT = torch.empty((SEQS, H, D, D), dtype=torch.float32, device=dev)
    ws = torch.empty(gdn.prefill_layer_workspace_size(SEQS, T, H, H), dtype=torch.uint8, device=dev)
    qkv = y.view(T, 3, H, D)
    stream = torch.cuda.current_stream(dev)

    def two():
        gdn.conv_silu(x, w, cu, conv_state_out=st, out=y, n_qk_channels=2 * H * D, head_dim=D)
        gdn.prefill(qkv[:, 0], qkv[:, 1], qkv[:, 2], g, beta, cu, final_state=hT, out=o, workspace=ws,
                    qk_l2norm=False)

    def fused():
        gdn.prefill_layer(x, w, g, beta, cu, H=H, conv_state_out=st2, final_state=hT, out=o, workspace=ws)

    times = {"two": [], "fused": []}
    for rep in range(max(args.warmup, 3) + 5):
        for name, fn in (("two", two), ("fused", fused)):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record(stream)
            fn()
            e.record(stream)
            torch.cuda.synchronize()
            if rep >= max(args.warmup, 3):
                times[name].append(s.elapsed_time(e))
    gdn.check_device_status(dev)
    tms, fms = statistics.median(times["two"]), statistics.median(times["fused"])
    return {"value": T / (fms * 1e-3) * dist.world, "unit": UNIT, "ms_per_step": fms,
            "workload": "layer_8x16384_h16_d128_bf16_conv_k4",
            "note": "gdn_prefill_layer: conv + SiLU inside the single-pass tensor-core prefill",
            "two_calls": {"value": T / (tms * 1e-3) * dist.world, "unit": UNIT, "ms_per_step": tms,
                          "note": "gdn_conv_silu, then gdn_prefill on token-strided views of y"},
            "gpu_launches": 2 * 5}


def run_ours(args, dist: Dist):
    import torch
    import gated_deltanet_linear_silu_b200 as gdn
    gdn.lib()  # fail loudly if the library is missing
    pk = peaks()
    clocks = ClockSampler(dist.local)

    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        import gdn_inputs as gi
        P = gi.long_prefill(SEQS, SEQ_LEN, H, D)
        tokens, n_seq = calibrated_sample(P, 15.0)
        tok, dt, threads = oracle_sample(P, tokens, n_seq)
        cpu = {"value": tok / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"first {tokens} tokens of {n_seq} of the 8 sequences, all 16 heads "
                         f"({tok} tokens, {dt:.1f} s, fp64 token loop)"}
        del P

    clocks.active = True
    pre = bench_prefill(args, dist, pk)
    extras = {}
    if not args.no_extras:
        extras["decode"] = bench_decode(args, dist, pk)
        extras["layer"] = bench_layer(args, dist, pk)
        extras["layer_long"] = bench_layer_long(args, dist, pk)
        extras["varlen"] = bench_varlen(args, dist, pk)
        extras["decode_layer"] = bench_decode_layer(args, dist, pk)
        extras["gated_rmsnorm"] = bench_gated_norm(args, dist, pk)
        extras["prefill_gated"] = bench_prefill_gated(args, dist, pk)
        extras["grouped"] = bench_grouped(args, dist, pk)
        extras["undecayed"] = bench_undecayed(args, dist, pk)
        extras["backward"] = bench_backward(args, dist, pk)
    clocks.active = False
    clk = clocks.stop()

    tokens_all = pre["tokens"] * dist.world
    ms_per_step = pre["total_ms"] / args.steps
    kernel_s = pre["kernel_ms"] * 1e-3
    th = pre["tokens"] * H
    flops = th * FLOP_PER_TOKEN_HEAD
    bytes_alg = th * BYTES_PER_TOKEN_HEAD + SEQS * H * STATE_BYTES
    hbm_ach = bytes_alg / kernel_s / 1e9
    tc_ach = flops / kernel_s / 1e12
    algo = gdn.selected_algo("bf16", D, D, CHUNK, args.algo)
    tc_used = algo == "tensor"
    line = {
        "metric": METRIC, "value": tokens_all / (ms_per_step * 1e-3), "unit": UNIT,
        "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if tc_used else "f32", "data": "synthetic",
        "config": config_block(dist.world),
        "roofline": {"bound": "hbm", "achieved": hbm_ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": hbm_ach / pk["hbm_gbs"],
                     "traffic": profiled_traffic("prefill", ["prefill_simt.cu", "prefill_tc.cu", "tc_ptx.cuh"],
                                                 th),
                     "kernel": "gdn_prefill (schedule + chunk kernel), CUDA events per call",
                     "algorithmic_bytes": bytes_alg, "peak_source": pk["source"]},
        "tc_roofline": {"achieved": tc_ach, "unit": "TFLOP/s", "peak": pk["bf16_tflops"],
                        "frac": tc_ach / pk["bf16_tflops"],
                        "frac_sustained": tc_ach / pk["bf16_tflops_sustained"]
                        if pk.get("bf16_tflops_sustained") else None,
                        "algorithmic_flops": flops},
        "e2e": {"value": tokens_all / (pre["e2e_ms_per_step"] * 1e-3), "unit": UNIT,
                "h2d_bytes_per_step": pre["h2d"], "d2h_bytes_per_step": pre["d2h"],
                "how": "gdn.prefill on two device buffer sets; each step's H2D (pinned) and D2H on "
                       "their own streams, overlapping the neighbouring steps"},
        "gpu_launches": 2 * args.steps,
        "clocks": clk,
        "algo": algo,
    }
    if cpu:
        line["cpu_baseline"] = cpu
    # Details first, the headline keys and a compact summary of every workload
    # last: readers that keep only the end of the output still see all numbers.
    out = dict(extras)
    out.update(line)
    out["summary"] = summarize(line, extras)
    if dist.rank == 0:
        print(json.dumps(out), flush=True)


def summarize(line, extras):
    """One short object: per workload its time and its roofline fraction(s)."""
    def r(x, n=4):
        return None if not isinstance(x, (int, float)) else round(float(x), n)

    def obj(d, t_key="ms_per_step"):
        o = {"ms": r(d.get(t_key, d.get("ms")))}
        if "roofline" in d:
            o["hbm"] = r(d["roofline"]["frac"], 3)
        if "tc_roofline" in d:
            o["tc"] = r(d["tc_roofline"]["frac"], 3)
        if "ratio" in d:
            o["ratio"] = r(d["ratio"], 3)
        if "conv" in d:
            o["conv_ms"] = r(d["conv"]["ms"])
            o["conv_hbm"] = r(d["conv"]["roofline"]["frac"], 3)
        return o

    s = {"prefill": {"ms": r(line["ms_per_step"]), "hbm": r(line["roofline"]["frac"], 3),
                     "tc": r(line["tc_roofline"]["frac"], 3)}}
    for name in ("decode", "decode_layer", "layer", "varlen", "gated_rmsnorm", "prefill_gated", "backward"):
        if name in extras:
            s[name] = obj(extras[name])
    if "decode" in extras and isinstance(extras["decode"].get("ms_per_step_graph"), float):
        s["decode"]["ms_graph"] = r(extras["decode"]["ms_per_step_graph"])
    if "grouped" in extras:
        s["grouped"] = {k: obj(v) for k, v in extras["grouped"].items()}
    if "undecayed" in extras:
        s["undecayed"] = {k: obj(v) for k, v in extras["undecayed"].items()}
    if "layer" in extras and "prefill_layer" in extras["layer"]:
        s["layer"]["prefill_layer_ms"] = r(extras["layer"]["prefill_layer"]["ms_per_step"])
        s["layer"]["fused_ms"] = r(extras["layer"]["fused"]["ms_per_step"])
    if "layer_long" in extras:
        s["layer_long"] = {"ms": r(extras["layer_long"]["ms_per_step"]),
                           "two_calls_ms": r(extras["layer_long"]["two_calls"]["ms_per_step"])}
    return s


def main():
    global SEQS, SEQ_LEN
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--algo", choices=["auto", "simt", "tensor"], default="auto")
    ap.add_argument("--no-extras", action="store_true", help="headline workload only")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seqs", type=int, default=SEQS, help="sequences (profiling runs only)")
    ap.add_argument("--seq-len", type=int, default=SEQ_LEN, help="tokens per sequence (profiling)")
    ap.add_argument("--only", choices=sorted(ONLY), default=None,
                    help="run one secondary workload alone and print its object (profiling runs)")
    args = ap.parse_args()
    SEQS, SEQ_LEN = args.seqs, args.seq_len
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    dist = Dist(args.gpus)
    if args.impl == "reference":
        run_reference(args, dist)
        return
    dist.init()
    try:
        if args.only:
            import gated_deltanet_linear_silu_b200 as gdn
            gdn.lib()
            res = ONLY[args.only](args, dist, peaks())
            if dist.rank == 0:
                print(json.dumps({"only": args.only, **res}), flush=True)
        else:
            run_ours(args, dist)
    finally:
        dist.close()


ONLY = {"decode": bench_decode, "layer": bench_layer, "varlen": bench_varlen,
        "decode_layer": bench_decode_layer, "gated_rmsnorm": bench_gated_norm,
        "grouped": bench_grouped, "undecayed": bench_undecayed, "backward": bench_backward,
        "prefill_gated": bench_prefill_gated, "layer_long": bench_layer_long}

if __name__ == "__main__":
    main()
