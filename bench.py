"""Benchmark of the KDA operator on B200 (one JSON line on stdout, rank 0).

Default: one GPU, the prefill workload B=4, H=32, T=8192, D_k=D_v=128, C=64
(BF16 q/k/v, FP32 g/beta/state, zero initial state) as the headline, plus the
decode workload (512 sequences x 32 heads, 256 steps captured in one CUDA
graph, FP32 state N(0, 0.02)) as a second object on the same line, and the
append-prefill (8 sequences of 1K-32K tokens, checkpoints every 4096) and
1M-token (snapshots every 32K) prefill workloads as two more.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload prefill|decode|append_varlen|long|many_seqs|many_seqs_small|prefill_small] [--no-decode] [--no-backward]
                  [--no-extra-prefill]

For N > 1 it is launched by torchrun, one rank per GPU; every rank runs its
own copy of the workload (the operator's (sequence, head) units are
independent, so nothing is exchanged on the data path) and the job time is
the maximum over ranks.  ``--impl reference`` times the FP64 CPU oracle on a
bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_attention_08_b200 import inputs as kin  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# --------------------------------------------------------------------------------------
# Algorithmic counts ("LLM - Semianalysis, Kimi K3 아키텍처" (charstring.tistory.com/2557),
# Methods 1: prefill costs
# 12C^3 + 8C^2 D + 6 C D^2 FLOPs per chunk; decode about 7 D^2 FLOPs and 8 D^2 bytes
# of FP32 state traffic per head per token).
# --------------------------------------------------------------------------------------
def prefill_flops_per_chunk(C: int, D: int) -> int:
    return 12 * C ** 3 + 8 * C ** 2 * D + 6 * C * D ** 2


def prefill_io_bytes_per_token_head(Dk: int, Dv: int, qkv_bytes: int) -> int:
    # q, k (Dk each) and v (Dv) in the qkv dtype; g (Dk) and beta FP32; o (Dv) in the qkv dtype
    return qkv_bytes * (2 * Dk + Dv) + 4 * Dk + 4 + qkv_bytes * Dv


def decode_state_bytes_per_token_head(Dk: int, Dv: int) -> int:
    return 8 * Dk * Dv           # FP32 state read + write


def decode_flops_per_token_head(D: int) -> int:
    return 7 * D * D


def prefill_algorithmic(lengths, H, Dk, Dv, C, qkv_bytes, interval, has_init):
    T = sum(lengths)
    chunks = sum(-(-n // C) for n in lengths)
    flops = chunks * H * prefill_flops_per_chunk(C, Dk)
    state = Dk * Dv * 4 * H * len(lengths)
    n_ck = sum(n // interval for n in lengths) if interval else 0
    byts = T * H * prefill_io_bytes_per_token_head(Dk, Dv, qkv_bytes) + state \
        + (state if has_init else 0) + n_ck * H * Dk * Dv * 4
    return flops, byts


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return p, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


KERNEL_SOURCES = {
    "decode": ("kda_decode.cu", "kda_common.cuh"),
    # BF16, D = 128, drafts up to 16 tokens: the tensor-core form; others: CUDA cores
    "decode_multi": ("kda_decode_multi.cu", "kda_decode_multi_tc.cu", "kda_tc_util.cuh",
                     "kda_tma.cuh", "kda_common.cuh"),
    "prefill_tc": ("kda_prefill_tc.cu", "kda_tc_util.cuh", "kda_tma.cuh", "kda_common.cuh"),
    # two-pass path: intra-chunk pass + chain pass, one prefill call = one launch of each
    "prefill_split": ("kda_prefill_split.cu", "kda_tc_util.cuh", "kda_tma.cuh", "kda_common.cuh"),
    "prefill_simt": ("kda_prefill_simt.cu", "kda_common.cuh"),
    # chunked tensor-core backward: the forward recomputation (two-pass prefill)
    # and the backward's own kernels, one call
    "backward_tc": ("kda_backward_tc.cu", "kda_prefill_split.cu", "kda_tc_util.cuh", "kda_tma.cuh",
                    "kda_common.cuh"),
}
PATH_KERNEL = {2: "prefill_split", 1: "prefill_tc", 0: "prefill_simt"}


def kernel_source_sha(kernel: str) -> str:
    """Hash of the source files a kernel is built from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "linear_attention_08_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as fh:
            h.update(name.encode() + fh.read())
    return h.hexdigest()[:16]


def scaled_traffic(kernel: str, token_heads: int):
    """DRAM bytes of one call on another workload, scaled by token-heads from the
    committed small-case capture of the same kernels (traffic grows in
    proportion to the chunks processed); None if that capture is stale."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        rec = json.load(fh).get(kernel + "_small")
    if not rec or rec.get("source_sha") != kernel_source_sha(kernel):
        return None
    return rec["bytes_per_launch"] * token_heads / rec["token_heads"]


def ncu_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current sources of that kernel (else None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        rec = json.load(fh).get(kernel)
    if not rec or rec.get("source_sha") != kernel_source_sha(kernel):
        return None
    return rec.get("bytes_per_launch")


# --------------------------------------------------------------------------------------
# Clocks during the timed region
# --------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.proc = None
        self.index = index

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.result = None
        if self.proc is None:
            return False
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(",") for r in out.strip().splitlines() if r.count(",") >= 7]
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[0]))
                mx = max(mx, float(r[1]))
            except ValueError:
                continue
            for name, val in zip(names, r[4:8]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        if sm:
            busy = [x for x in sm if x > 0.5 * mx] or sm
            self.result = {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx,
                           "reasons": sorted(reasons), "samples": len(sm)}
        return False


# --------------------------------------------------------------------------------------
# Distributed plumbing
# --------------------------------------------------------------------------------------
def dist_setup(gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------------------------
# Our arm
# --------------------------------------------------------------------------------------
def time_prefill(name, steps, warmup, world, local, e2e=True):
    from linear_attention_08_b200 import kda
    w = kin.WORKLOADS[name]
    d = kin.make_workload(name, device="cuda", seed=local)
    lengths, cu = d["lengths"], d["cu_seqlens"]
    cu_dev = torch.tensor(cu, dtype=torch.int32, device="cuda")
    C, H, Dk, Dv = w["chunk"], w["H"], w["Dk"], w["Dv"]
    interval = w["ckpt_interval"]
    init = d["init_state"] if w["state_std"] > 0 else None
    out = torch.empty_like(d["v"])
    fin = torch.empty(len(lengths), H, Dk, Dv, device="cuda")
    n_ck = kda.kda_ckpt_count(cu, interval) if interval else 0
    ck = torch.empty(max(n_ck, 1), H, Dk, Dv, device="cuda") if interval else None
    stream = torch.cuda.current_stream()

    def step():
        kda.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], cu_dev, init_state=init,
                        chunk=C, ckpt_interval=interval, out=out, final_state=fin,
                        ckpt_states=ck, cu_seqlens_host=cu, stream=stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        barrier(world)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(steps):
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
    total_ms = t0.elapsed_time(t1)
    launch_ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    barrier(world)
    total_ms = max_over_ranks(total_ms, world)
    launch_ms = max_over_ranks(launch_ms, world)

    tokens = sum(lengths)
    flops, byts = prefill_algorithmic(lengths, H, Dk, Dv, C, 2 if w["dtype"] == "bf16" else 4,
                                      interval, init is not None)
    shape = kda.make_shape(len(lengths), tokens, H, Dk, Dv, C, 1 if w["dtype"] == "bf16" else 0)
    path = kda.kda_prefill_path(shape)
    launches = 1
    if path == 2:   # one intra-chunk pass and one chain pass per window of chunks
        ws = kda.workspace_for(shape, "meta")
        launches = 2 * prefill_windows(len(lengths), H, tokens, ws.numel(),
                                       kda.kda_prefill_workspace_bytes(shape))
    res = dict(tokens=tokens, steps=steps, total_ms=total_ms, launch_ms=launch_ms,
               launches_per_step=launches, flops=flops, bytes=byts, clocks=clk.result,
               kernel=PATH_KERNEL[path], w=w, lengths=lengths, token_heads=tokens * H)
    if not e2e:
        return res

    # End to end through the public API: pinned host inputs -> device -> kernel -> host.
    host = {x: d[x].to("cpu").pin_memory() for x in ("q", "k", "v", "g", "beta")}
    h_init = init.to("cpu").pin_memory() if init is not None else None
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h_fin = torch.empty(fin.shape, dtype=fin.dtype).pin_memory()
    dev = {x: torch.empty_like(d[x]) for x in host}
    d_init = torch.empty_like(init) if init is not None else None
    bi = sum(t.numel() * t.element_size() for t in host.values()) + \
        (h_init.numel() * 4 if h_init is not None else 0)
    bo = h_out.numel() * h_out.element_size() + h_fin.numel() * 4
    e2e_steps = max(1, min(steps, 5))

    def e2e_step():
        for x in host:
            dev[x].copy_(host[x], non_blocking=True)
        if d_init is not None:
            d_init.copy_(h_init, non_blocking=True)
        kda.kda_prefill(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], cu_dev,
                        init_state=d_init, chunk=C, ckpt_interval=interval, out=out,
                        final_state=fin, ckpt_states=ck, cu_seqlens_host=cu, stream=stream)
        h_out.copy_(out, non_blocking=True)
        h_fin.copy_(fin, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(b) / e2e_steps, world)
    res.update(e2e_ms=e2e_ms, bi=bi, bo=bo)
    return res


def prefill_object(r, world, hbm, tflops, peaks_src):
    """The bench object of one more prefill workload (no end-to-end leg)."""
    w = r["w"]
    ms = r["total_ms"] / r["steps"]
    gbs = r["bytes"] / (r["launch_ms"] / 1e3) / 1e9
    tfs = r["flops"] / (r["launch_ms"] / 1e3) / 1e12
    return {
        "metric": "KDA prefill tokens/s", "value": world * r["tokens"] / (ms / 1e3),
        "unit": "tokens/s", "ms_per_call": ms, "steps": r["steps"],
        "config": {"workload": w_name(w), "num_seqs": len(r["lengths"]),
                   "total_tokens": r["tokens"],
                   "seq_lens": sorted(r["lengths"]) if len(r["lengths"]) <= 16 else
                   {"min": min(r["lengths"]), "max": max(r["lengths"])},
                   "heads": w["H"], "d": w["Dk"], "chunk": w["chunk"],
                   "ckpt_interval": w["ckpt_interval"],
                   "init_state": "N(0, 0.02)" if w["state_std"] > 0 else "zero"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                     "frac": gbs / hbm, "traffic": scaled_traffic(r["kernel"], r["token_heads"]),
                     "kernel": r["kernel"], "peak_source": peaks_src,
                     "tensor_tflops": tfs, "tensor_frac": tfs / tflops,
                     "algorithmic_bytes_per_launch": r["bytes"],
                     "algorithmic_flops_per_launch": r["flops"]},
        "gpu_launches": r["steps"] * r["launches_per_step"], "clocks": r["clocks"],
    }


def w_name(w):
    for name, spec in kin.WORKLOADS.items():
        if spec is w:
            return name
    return "?"


def prefill_windows(N, H, T, ws_bytes, full_bytes, packet=74240, chunk=64):
    """Windows of chunks the two-pass prefill runs for a workspace of ws_bytes
    (with a final-state buffer, as the benchmark passes one)."""
    if ws_bytes >= full_bytes:
        return 1
    wc = (ws_bytes - 256) // (N * H * packet)
    max_chunks = -(-T // chunk)
    return -(-max_chunks // wc)


def time_decode(steps_graph, warmup, world, local, decode_steps=None):
    from linear_attention_08_b200 import kda
    w = dict(kin.WORKLOADS["decode"])
    if decode_steps:
        w["steps"] = decode_steps
    d = kin.make_inputs((w["steps"], w["num_seqs"]), w["H"], w["Dk"], w["Dv"],
                        kin.torch_dtype(w["dtype"]), local, num_states=w["num_seqs"],
                        state_std=w["state_std"], device="cuda")
    S, N, H, Dk, Dv = w["steps"], w["num_seqs"], w["H"], w["Dk"], w["Dv"]
    state = d["init_state"].clone()
    outs = torch.empty_like(d["v"])
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for t in range(S):   # warm the kernels before capture
            kda.kda_decode(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], state,
                           out=outs[t], stream=side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        for t in range(S):
            kda.kda_decode(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], state,
                           out=outs[t], stream=side)
    stream = torch.cuda.current_stream()
    for _ in range(max(warmup, 1)):
        graph.replay()
    torch.cuda.synchronize()
    barrier(world)
    with ClockSampler(local) as clk:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps_graph):
            graph.replay()
        b.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b) / steps_graph, world)
    # end to end: per-step host inputs in, per-step outputs out (state stays resident)
    hq = {x: d[x].to("cpu").pin_memory() for x in ("q", "k", "v", "g", "beta")}
    h_out = torch.empty(outs.shape, dtype=outs.dtype).pin_memory()
    bi = sum(t.numel() * t.element_size() for t in hq.values())
    bo = h_out.numel() * h_out.element_size()

    def e2e():
        for x in hq:
            d[x].copy_(hq[x], non_blocking=True)
        graph.replay()
        h_out.copy_(outs, non_blocking=True)

    e2e()
    torch.cuda.synchronize()
    a2, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a2.record(stream)
    e2e()
    b2.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a2.elapsed_time(b2), world)
    del graph
    token_heads = S * N * H
    byts = token_heads * (decode_state_bytes_per_token_head(Dk, Dv)
                          + prefill_io_bytes_per_token_head(Dk, Dv, 2))
    return dict(tokens=S * N, ms=ms, launches=S, e2e_ms=e2e_ms, bi=bi, bo=bo, bytes=byts,
                flops=token_heads * decode_flops_per_token_head(Dk), clocks=clk.result)


def time_prefill_at(steps, warmup, world, local, positions=(1000, 3000, 5000, 7777)):
    """Prefill with states at explicit positions (prompt boundaries): the
    headline workload (4 x 8192 tokens, H=32, D=128, BF16) with the state also
    taken after each of `positions` tokens of every sequence (kda_prefill_at)."""
    from linear_attention_08_b200 import kda
    w = kin.WORKLOADS["prefill"]
    d = kin.make_workload("prefill", device="cuda", seed=local)
    lengths, cu = d["lengths"], d["cu_seqlens"]
    N, H, Dk, Dv, C = len(lengths), w["H"], w["Dk"], w["Dv"], w["chunk"]
    cu_dev = torch.tensor(cu, dtype=torch.int32, device="cuda")
    pos_cu = torch.tensor([len(positions) * n for n in range(N + 1)], dtype=torch.int32, device="cuda")
    pos = torch.tensor(list(positions) * N, dtype=torch.int32, device="cuda")
    out = torch.empty_like(d["v"])
    fin = torch.empty(N, H, Dk, Dv, device="cuda")
    pos_states = torch.empty(N * len(positions), H, Dk, Dv, device="cuda")
    lib = kda.load()
    shape = kda.make_shape(N, sum(lengths), H, Dk, Dv, C, kda.KDA_DTYPE_BF16)
    stream = torch.cuda.current_stream()
    P = kda._ptr

    def step():
        st = lib.kda_prefill_at(P(d["q"]), P(d["k"]), P(d["v"]), P(d["g"]), P(d["beta"]), None,
                                P(cu_dev), P(out), P(fin), 0, None, P(pos_cu), P(pos),
                                P(pos_states), kda.ctypes.byref(shape), kda._stream(stream))
        assert st == kda.KDA_OK, st

    for _ in range(max(warmup, 1)):
        step()
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b) / steps, world)
    flops, byts = prefill_algorithmic(lengths, H, Dk, Dv, C, 2, 0, False)
    byts += N * len(positions) * H * Dk * Dv * 4
    return dict(tokens=sum(lengths), ms=ms, bytes=byts, flops=flops, positions=list(positions), N=N,
                H=H, T=lengths[0])


def time_spec_decode(steps, warmup, world, local, T_new=8, N=512):
    """Multi-token decode: N (512) sequences x 32 heads, T_new draft tokens each,
    all accepted.  One call moves the FP32 state once for T_new tokens."""
    from linear_attention_08_b200 import kda
    H, D = 32, 128
    d = kin.make_inputs((N, T_new), H, D, D, torch.bfloat16, local, num_states=N,
                        state_std=0.02, device="cuda")
    state = d["init_state"].clone()
    out = torch.empty_like(d["v"])
    stream = torch.cuda.current_stream()

    def step():
        kda.kda_decode_multi(d["q"], d["k"], d["v"], d["g"], d["beta"], state, out=out,
                             stream=stream)

    for _ in range(max(warmup, 1)):
        step()
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b) / steps, world)
    byts = N * H * (decode_state_bytes_per_token_head(D, D)
                    + T_new * prefill_io_bytes_per_token_head(D, D, 2))
    return dict(tokens=N * T_new, ms=ms, bytes=byts, T_new=T_new, N=N)


def time_backward(steps, warmup, world, local, N=4, H=32, T=1024, D=128):
    """Backward pass: B=4 x 1024 tokens, 32 heads, D=128, BF16 inputs, random
    upstream gradients on the outputs and the final states."""
    from linear_attention_08_b200 import kda
    lengths = [T] * N
    d = kin.make_inputs((N * T,), H, D, D, torch.bfloat16, local, num_states=N, state_std=0.02,
                        device="cuda")
    cu = torch.tensor(kin.cu_seqlens_of(lengths), dtype=torch.int32, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(1000 + local)
    d_out = torch.randn(N * T, H, D, device="cuda", generator=gen)
    d_fin = torch.randn(N, H, D, D, device="cuda", generator=gen)
    shape = kda.make_shape(N, N * T, H, D, D, 0, kda.KDA_DTYPE_BF16)
    ws = torch.empty(kda.load().kda_backward_workspace_bytes(kda.ctypes.byref(shape)),
                     dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        kda.kda_backward(d["q"], d["k"], d["v"], d["g"], d["beta"], cu, d_out,
                         init_state=d["init_state"], d_final=d_fin, workspace=ws, stream=stream)

    for _ in range(max(warmup, 1)):
        step()
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b) / steps, world)
    path = kda.kda_last_backward_path()
    # algorithmic bytes per token-head: q, k, v (BF16), g, d_out, the five
    # FP32 gradients and beta; plus three states per unit (init, d_final, d_init)
    per_th = 3 * D * 2 + D * 4 + D * 4 + 4 + 3 * D * 4 + D * 4 + 4
    byts = N * T * H * per_th + 3 * N * H * D * D * 4
    return dict(tokens=N * T, ms=ms, bytes=byts, N=N, H=H, T=T, D=D,
                kernel="backward_tc" if path == 1 else "backward_simt")


def run_ours(args, rank, world, local):
    peaks, peaks_src = load_peaks()
    hbm = peaks["hbm_gbs"]
    tflops = peaks["bf16_tflops"]
    name = args.workload
    res = time_prefill(name, args.steps, args.warmup, world, local) if name != "decode" else None
    spec = None
    if not args.no_decode:
        spec = time_spec_decode(max(args.steps, 5), args.warmup, world, local)
    extra = {}
    if name == "prefill" and not args.no_extra_prefill:
        for other in ("append_varlen", "long", "many_seqs"):
            extra[other] = time_prefill(other, 3 if other == "long" else 10, args.warmup, world,
                                        local, e2e=False)
            torch.cuda.empty_cache()
    pat = None
    if name == "prefill" and not args.no_extra_prefill:
        pat = time_prefill_at(10, args.warmup, world, local)
    bwd = None
    if not args.no_backward and name == "prefill":
        bwd = time_backward(max(1, min(args.steps, 3)), args.warmup, world, local)
    dec = None
    if name == "decode" or not args.no_decode:
        dec = time_decode(max(1, args.steps // 2) if name != "decode" else args.steps,
                          args.warmup, world, local, args.decode_steps)
    if rank != 0:
        return None
    if res is not None:
        r = res
        w = r["w"]
        ms_step = r["total_ms"] / r["steps"]
        value = world * r["tokens"] / (ms_step / 1e3)
        gbs = r["bytes"] / (r["launch_ms"] / 1e3) / 1e9
        tfs = r["flops"] / (r["launch_ms"] / 1e3) / 1e12
        traffic = ncu_traffic(r["kernel"])
        line = {
            "metric": "KDA prefill tokens/s", "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": r["steps"], "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if w["dtype"] == "bf16" else "f32",
            "data": "synthetic",
            "config": {"workload": name, "num_seqs": w["num_seqs"], "seq_lens": sorted(set(r["lengths"]))[:4],
                       "total_tokens": r["tokens"], "heads": w["H"], "d_k": w["Dk"], "d_v": w["Dv"],
                       "chunk": w["chunk"], "ckpt_interval": w["ckpt_interval"],
                       "state": "fp32", "parallelism": f"replicas{world}",
                       "l2": "inputs larger than L2 (%.2f GB per step)" % (r["bytes"] / 1e9)},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                         "frac": gbs / hbm, "traffic": traffic,
                         "kernel": r["kernel"], "peak_source": peaks_src,
                         "tensor_tflops": tfs, "tensor_frac": tfs * 1e12 / (tflops * 1e12),
                         "algorithmic_bytes_per_launch": r["bytes"],
                         "algorithmic_flops_per_launch": r["flops"]},
            "e2e": {"value": world * r["tokens"] / (r["e2e_ms"] / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": r["bi"], "d2h_bytes_per_step": r["bo"]},
            "gpu_launches": r["steps"] * r["launches_per_step"],
            "clocks": r["clocks"],
        }
        for other, ro in extra.items():
            line[other] = prefill_object(ro, world, hbm, tflops, peaks_src)
        if pat is not None:
            pgbs = pat["bytes"] / (pat["ms"] / 1e3) / 1e9
            line["prefill_at"] = {
                "metric": "KDA prefill tokens/s, states at prompt boundaries",
                "value": world * pat["tokens"] / (pat["ms"] / 1e3), "unit": "tokens/s",
                "ms_per_call": pat["ms"],
                "config": {"workload": "prefill_at", "num_seqs": pat["N"], "seq_len": pat["T"],
                           "heads": pat["H"], "d": 128, "positions_per_seq": pat["positions"]},
                "roofline": {"bound": "hbm", "achieved": pgbs, "peak": hbm, "unit": "GB/s",
                             "frac": pgbs / hbm, "kernel": "prefill_tc", "traffic": None,
                             "note": "single-pass kernel (explicit positions); operator bytes incl. the position states"}}
        if bwd is not None:
            bgbs = bwd["bytes"] / (bwd["ms"] / 1e3) / 1e9
            line["backward"] = {
                "metric": "KDA backward tokens/s",
                "value": world * bwd["tokens"] / (bwd["ms"] / 1e3), "unit": "tokens/s",
                "ms_per_call": bwd["ms"],
                "config": {"num_seqs": bwd["N"], "seq_len": bwd["T"], "heads": bwd["H"],
                           "d": bwd["D"], "dtype": "bf16 inputs, fp32 gradients"},
                "roofline": {"bound": "hbm", "achieved": bgbs, "peak": hbm, "unit": "GB/s",
                             "frac": bgbs / hbm, "kernel": bwd["kernel"],
                             "traffic": ncu_traffic(bwd["kernel"]) if bwd["kernel"] == "backward_tc" else None,
                             "note": "operator bytes (inputs, upstream gradients, gradients, states) over the whole call; "
                                     "traffic = DRAM bytes of all eight kernels of one call"}}
    if dec is not None:
        dgbs = dec["bytes"] / (dec["ms"] / dec["launches"] / 1e3) / 1e9 / dec["launches"]
        dobj = {
            "metric": "KDA decode tokens/s", "value": world * dec["tokens"] / (dec["ms"] / 1e3),
            "unit": "tokens/s", "ms_per_step": dec["ms"] / dec["launches"], "ms_per_graph": dec["ms"],
            "steps_per_graph": dec["launches"],
            "config": {"workload": "decode", "num_seqs": 512, "heads": 32, "d": 128,
                       "steps": dec["launches"], "l2": "state 2.1 GB > L2"},
            "roofline": {"bound": "hbm", "achieved": dgbs, "peak": hbm, "unit": "GB/s",
                         "frac": dgbs / hbm, "traffic": ncu_traffic("decode"),
                         "kernel": "decode", "peak_source": peaks_src},
            "e2e": {"value": world * dec["tokens"] / (dec["e2e_ms"] / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": dec["bi"], "d2h_bytes_per_step": dec["bo"]},
            "gpu_launches": dec["launches"], "clocks": dec["clocks"],
        }
        if spec is not None:
            sgbs = spec["bytes"] / (spec["ms"] / 1e3) / 1e9
            dobj["spec_decode"] = {
                "metric": "KDA multi-token decode tokens/s",
                "value": world * spec["tokens"] / (spec["ms"] / 1e3), "unit": "tokens/s",
                "ms_per_call": spec["ms"],
                "config": {"num_seqs": 512, "heads": 32, "d": 128, "tokens_per_seq": spec["T_new"],
                           "accepted": "all"},
                "roofline": {"bound": "hbm", "achieved": sgbs, "peak": hbm, "unit": "GB/s",
                             "frac": sgbs / hbm, "traffic": ncu_traffic("decode_multi"),
                             "kernel": "decode_multi", "peak_source": peaks_src}}
        if res is None:
            line = dict(dobj)
            line.update({"n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                         "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                         "dtype": "bf16", "data": "synthetic"})
        else:
            line["decode"] = dobj
    return line


# --------------------------------------------------------------------------------------
# CPU baseline: the FP64 oracle on a bounded sample of the same workload
# --------------------------------------------------------------------------------------
def oracle_sample(name, budget_s=12.0):
    """Time the oracle on the first tokens of a few (sequence, head) units of the
    workload, growing the sample until about budget_s seconds of CPU work."""
    import oracle
    w = kin.WORKLOADS[name]
    threads = oracle.max_threads()
    H = w["H"]
    units = max(threads, 1)
    tokens = 256
    if name == "decode":
        d = kin.make_inputs((w["steps"], 1), units, w["Dk"], w["Dv"], kin.torch_dtype(w["dtype"]),
                            0, num_states=1, state_std=w["state_std"])
    while True:
        if name == "decode":
            n_steps = min(tokens, w["steps"])
            sl = lambda x: x[:n_steps]
            t0 = time.perf_counter()
            oracle.decode(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["g"]), sl(d["beta"]),
                          d["init_state"], nthreads=threads)
            dt = time.perf_counter() - t0
            token_heads = n_steps * units
        else:
            L = tokens
            di = kin.make_inputs((L,), units, w["Dk"], w["Dv"], kin.torch_dtype(w["dtype"]), 0,
                                 num_states=1, state_std=w["state_std"])
            t0 = time.perf_counter()
            oracle.prefill(di["q"], di["k"], di["v"], di["g"], di["beta"], [0, L],
                           di["init_state"], 0, 0, threads)
            dt = time.perf_counter() - t0
            token_heads = L * units
        if dt > budget_s / 4 or (name == "decode" and tokens >= w["steps"]):
            break
        if name != "decode" and tokens * 2 > max(kin.workload_lengths(name)):
            units *= 2          # longer than a sequence of the workload: add heads instead
        else:
            tokens *= 2
    tok_per_s = token_heads / dt / H   # a token is H token-heads
    return {"value": tok_per_s, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{token_heads} token-heads ({units} heads x {token_heads // units} tokens) "
                      f"of the {name} workload, FP64 recurrence, {dt:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    name = args.workload
    per_step = []
    for _ in range(args.warmup):
        oracle_sample(name, budget_s=2.0)
    base = None
    for _ in range(args.steps):
        base = oracle_sample(name, budget_s=8.0)
        per_step.append(base["value"])
    value = statistics.median(per_step)
    base["value"] = value
    return {"metric": "KDA decode tokens/s" if name == "decode" else "KDA prefill tokens/s",
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": {"workload": name},
            "cpu_baseline": base,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill",
                    choices=["prefill", "decode", "append_varlen", "long", "many_seqs",
                             "many_seqs_small", "prefill_small"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-extra-prefill", action="store_true",
                    help="skip the append-varlen and 1M-token prefill objects")
    ap.add_argument("--decode-steps", type=int, default=0,
                    help="decode steps per graph (default: the workload's 256)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--spec-only", type=int, default=0, metavar="NUM_SEQS",
                    help="time only the multi-token decode (8 draft tokens) on NUM_SEQS "
                         "sequences x 32 heads (a small case for profiling); prints its object alone")
    ap.add_argument("--backward-only", type=int, default=0, metavar="SEQ_LEN",
                    help="time only the backward pass on 4 sequences of SEQ_LEN tokens "
                         "(a small case for profiling); prints its object alone")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        line = run_reference(args, rank, int(os.environ.get("WORLD_SIZE", "1")))
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    rank, world, local = dist_setup(args.gpus)
    if args.spec_only > 0:
        spec = time_spec_decode(args.steps, args.warmup, world, local, N=args.spec_only)
        if rank == 0:
            print(json.dumps({"metric": "KDA multi-token decode tokens/s", "unit": "tokens/s",
                              "value": world * spec["tokens"] / (spec["ms"] / 1e3),
                              "ms_per_call": spec["ms"], "n_gpus": world,
                              "config": {"num_seqs": spec["N"], "heads": 32, "d": 128,
                                         "draft_tokens": spec["T_new"]}}), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
        return
    if args.backward_only > 0:
        bwd = time_backward(args.steps, args.warmup, world, local, T=args.backward_only)
        if rank == 0:
            print(json.dumps({"metric": "KDA backward tokens/s", "unit": "tokens/s",
                              "value": world * bwd["tokens"] / (bwd["ms"] / 1e3),
                              "ms_per_call": bwd["ms"], "n_gpus": world,
                              "config": {"num_seqs": bwd["N"], "seq_len": bwd["T"],
                                         "heads": bwd["H"], "d": bwd["D"]}}), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
        return
    line = run_ours(args, rank, world, local)
    if rank == 0 and line is not None:
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = oracle_sample(args.workload)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
