"""Helpers shared by the GPU parity tests: run the CUDA path and the FP64 oracle
on the same seeded inputs and compare them."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from linear_attention_08_b200 import inputs as kin
from linear_attention_08_b200 import kda

TOL = {torch.float32: 1e-4, torch.bfloat16: 1e-2}


def rel_l2(x, ref) -> float:
    x = np.asarray(x.detach().to("cpu", torch.float64).numpy() if hasattr(x, "detach") else x,
                   dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    den = np.linalg.norm(ref)
    if den == 0.0:
        return float(np.linalg.norm(x))
    return float(np.linalg.norm(x - ref) / den)


def make_case(lengths, H, Dk, Dv, dtype, seed=0, state_std=0.02, device="cuda"):
    d = kin.make_inputs((int(sum(lengths)),), H, Dk, Dv, dtype, seed,
                        num_states=len(lengths), state_std=state_std, device="cpu")
    d["lengths"] = list(lengths)
    d["cu_seqlens"] = kin.cu_seqlens_of(lengths)
    return d


def to_device(d, device="cuda"):
    out = {}
    for key, val in d.items():
        out[key] = val.to(device) if isinstance(val, torch.Tensor) else val
    out["cu_dev"] = torch.tensor(d["cu_seqlens"], dtype=torch.int32, device=device)
    return out


def gpu_prefill(dd, chunk, interval=0, use_init=True, **kw):
    return kda.kda_prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["cu_dev"],
                           init_state=dd["init_state"] if use_init else None, chunk=chunk,
                           ckpt_interval=interval, cu_seqlens_host=dd["cu_seqlens"], **kw)


def oracle_full(d, interval=0, use_init=True, nthreads=0):
    return oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"],
                          d["init_state"] if use_init else None, interval, 0, nthreads)


def unit_slice(d, seq, h):
    """Inputs of one (sequence, head) unit as host tensors."""
    cu = d["cu_seqlens"]
    a, b = cu[seq], cu[seq + 1]
    cpu = lambda t: t.detach().to("cpu")
    sl = {key: cpu(d[key][a:b, h:h + 1]) for key in ("q", "k", "v", "g")}
    sl["beta"] = cpu(d["beta"][a:b, h:h + 1])
    init = d.get("init_state")
    sl["init_state"] = None if init is None else cpu(init[seq:seq + 1, h:h + 1])
    sl["cu_seqlens"] = [0, b - a]
    return sl


def oracle_unit(d, seq, h, interval=0, use_init=True):
    sl = unit_slice(d, seq, h)
    return oracle.prefill(sl["q"], sl["k"], sl["v"], sl["g"], sl["beta"], sl["cu_seqlens"],
                          sl["init_state"] if use_init else None, interval, 0, 1)


def ckpt_base(lengths, seq, interval):
    return sum(int(n) // interval for n in lengths[:seq]) if interval > 0 else 0
