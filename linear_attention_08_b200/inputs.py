"""Seeded synthetic inputs for the KDA operator.

This module only draws random tensors with the distributions the workloads
state; it holds none of the operator's arithmetic.  Both the CUDA path and the
FP64 oracle consume what it returns, so that they see identical bits.

Distributions (one value per token-head unless noted):

* q, k ~ N(0, 1) per channel, then L2-normalised over the key dimension in
  FP32, then cast to the compute dtype;
* v ~ N(0, 1), cast to the compute dtype;
* beta = sigmoid(N(0, 1)) in FP32;
* g = max(-softplus(N(0, 1)), -5) in FP32 per key channel: a natural-log decay
  with the lower bound of -5 for the lower-bounded decay that
  "MoonshotAI/Kimi-K3 딥다이브" (fiv.co.kr/repos/kimi-k3-deep-dive.html), section 4-1, describes;
* the initial state, when requested, ~ N(0, std^2) in FP32.

Draw order from one generator: q, k, v, beta-logits, g-logits, init_state.
Sequence lengths of a varlen batch come from a separate generator.

Layouts (token-major, packed over sequences):
q, k, g: [T_tot, H, D_k]; v: [T_tot, H, D_v]; beta: [T_tot, H];
init_state: [N, H, D_k, D_v].  Decode inputs carry a leading step axis.
"""
from __future__ import annotations

import torch

GATE_FLOOR = -5.0


def make_lengths(num_seqs: int, lo: int, hi: int, seed: int = 1) -> list[int]:
    """Uniform integer lengths in [lo, hi] from their own generator."""
    gen = torch.Generator("cpu").manual_seed(seed)
    return torch.randint(lo, hi + 1, (num_seqs,), generator=gen).tolist()


def cu_seqlens_of(lengths: list[int]) -> list[int]:
    out = [0]
    for n in lengths:
        out.append(out[-1] + int(n))
    return out


def _gen(seed: int, device: str) -> torch.Generator:
    return torch.Generator(device).manual_seed(seed)


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def make_inputs(lead: tuple, H: int, Dk: int, Dv: int, dtype: torch.dtype,
                seed: int, num_states: int = 0, state_std: float = 0.0,
                device: str = "cpu") -> dict:
    """Draw one batch of inputs.

    ``lead`` is the leading shape: ``(T_tot,)`` for prefill, ``(steps, N)``
    for decode.  ``num_states`` > 0 also draws an initial state
    [num_states, H, Dk, Dv] with standard deviation ``state_std`` (0 gives
    zeros without a draw).
    """
    gen = _gen(seed, device)
    f32 = torch.float32
    q = torch.randn(*lead, H, Dk, generator=gen, device=device, dtype=f32)
    q = _unit_rows(q).to(dtype)
    k = torch.randn(*lead, H, Dk, generator=gen, device=device, dtype=f32)
    k = _unit_rows(k).to(dtype)
    v = torch.randn(*lead, H, Dv, generator=gen, device=device, dtype=f32).to(dtype)
    beta = torch.sigmoid(torch.randn(*lead, H, generator=gen, device=device, dtype=f32))
    g = torch.randn(*lead, H, Dk, generator=gen, device=device, dtype=f32)
    g = torch.clamp(-torch.nn.functional.softplus(g), min=GATE_FLOOR)
    init = None
    if num_states > 0:
        if state_std > 0:
            init = torch.randn(num_states, H, Dk, Dv, generator=gen, device=device,
                               dtype=f32) * state_std
        else:
            init = torch.zeros(num_states, H, Dk, Dv, device=device, dtype=f32)
    return {"q": q.contiguous(), "k": k.contiguous(), "v": v.contiguous(),
            "g": g.contiguous(), "beta": beta.contiguous(), "init_state": init}


# The five workloads the operator is specified on.  Lengths of the varlen
# batch are drawn from seed 1; everything else from seed 0.
WORKLOADS = {
    "tiny": dict(kind="prefill", num_seqs=1, seq_len=64, H=2, Dk=32, Dv=32, chunk=16,
                 dtype="f32", state_std=0.0, ckpt_interval=0),
    "prefill": dict(kind="prefill", num_seqs=4, seq_len=8192, H=32, Dk=128, Dv=128,
                    chunk=64, dtype="bf16", state_std=0.0, ckpt_interval=0),
    "decode": dict(kind="decode", num_seqs=512, steps=256, H=32, Dk=128, Dv=128,
                   dtype="bf16", state_std=0.02),
    "append_varlen": dict(kind="prefill", num_seqs=8, len_range=(1024, 32768), H=32,
                          Dk=128, Dv=128, chunk=64, dtype="bf16", state_std=0.02,
                          ckpt_interval=4096),
    "long": dict(kind="prefill", num_seqs=1, seq_len=1048576, H=32, Dk=128, Dv=128,
                 chunk=64, dtype="bf16", state_std=0.0, ckpt_interval=32768),
    # many short sequences: 32,768 (sequence, head) units, past the 2048 the
    # two-pass path takes, so the single-pass kernel runs
    "many_seqs": dict(kind="prefill", num_seqs=1024, seq_len=1024, H=32, Dk=128, Dv=128,
                      chunk=64, dtype="bf16", state_std=0.0, ckpt_interval=0),
    # the single-pass kernel on 128 x 1024 tokens (4096 units), for profiler
    # captures whose traffic is scaled to many_seqs
    "many_seqs_small": dict(kind="prefill", num_seqs=128, seq_len=1024, H=32, Dk=128, Dv=128,
                            chunk=64, dtype="bf16", state_std=0.0, ckpt_interval=0),
    # a smaller case of the prefill kernels, in the same launch configuration as
    # "prefill" (more than 74 (sequence, head) units), for profiler captures
    "prefill_small": dict(kind="prefill", num_seqs=2, seq_len=4096, H=40, Dk=128, Dv=128,
                          chunk=64, dtype="bf16", state_std=0.0, ckpt_interval=0),
}


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def workload_lengths(name: str) -> list[int]:
    w = WORKLOADS[name]
    if "len_range" in w:
        lo, hi = w["len_range"]
        return make_lengths(w["num_seqs"], lo, hi, seed=1)
    return [w["seq_len"]] * w["num_seqs"]


def make_workload(name: str, device: str = "cpu", seed: int = 0) -> dict:
    """Inputs of one named workload, plus its lengths and cu_seqlens."""
    w = WORKLOADS[name]
    dt = torch_dtype(w["dtype"])
    if w["kind"] == "decode":
        lead = (w["steps"], w["num_seqs"])
        d = make_inputs(lead, w["H"], w["Dk"], w["Dv"], dt, seed, num_states=w["num_seqs"],
                        state_std=w["state_std"], device=device)
        d["lengths"] = [w["steps"]] * w["num_seqs"]
        return d
    lengths = workload_lengths(name)
    d = make_inputs((sum(lengths),), w["H"], w["Dk"], w["Dv"], dt, seed,
                    num_states=len(lengths), state_std=w["state_std"], device=device)
    d["lengths"] = lengths
    d["cu_seqlens"] = cu_seqlens_of(lengths)
    return d
