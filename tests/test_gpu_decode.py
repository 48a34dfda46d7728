"""Decode parity: kda_decode through the C ABI against the FP64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_08_b200 import inputs as kin
from linear_attention_08_b200 import kda
from parity import TOL, gpu_prefill, rel_l2, to_device

pytestmark = pytest.mark.gpu


def run_decode_steps(d, device="cuda"):
    q, k, v, g, b = (d[x].to(device) for x in ("q", "k", "v", "g", "beta"))
    state = d["init_state"].to(device).clone()
    outs = torch.empty_like(v)
    for t in range(q.shape[0]):
        kda.kda_decode(q[t], k[t], v[t], g[t], b[t], state, out=outs[t])
    torch.cuda.synchronize()
    return outs, state


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dims", [(32, 32), (32, 128), (64, 64), (128, 32), (128, 128)])
def test_decode_small(dtype, dims):
    Dk, Dv = dims
    d = kin.make_inputs((12, 5), 3, Dk, Dv, dtype, seed=11, num_states=5, state_std=0.3)
    outs, state = run_decode_steps(d)
    ro, rf = oracle.decode(d["q"], d["k"], d["v"], d["g"], d["beta"], d["init_state"])
    assert rel_l2(outs, ro) <= TOL[dtype]
    assert rel_l2(state, rf) <= TOL[dtype]


def test_decode_extremes():
    d = kin.make_inputs((6, 4), 2, 128, 128, torch.bfloat16, seed=12, num_states=4, state_std=1.0)
    d["g"].fill_(-5.0)
    d["beta"].fill_(1.0)
    outs, state = run_decode_steps(d)
    ro, rf = oracle.decode(d["q"], d["k"], d["v"], d["g"], d["beta"], d["init_state"])
    assert rel_l2(outs, ro) <= 1e-2 and rel_l2(state, rf) <= 1e-2


def test_decode_matches_prefill():
    """T decode steps == a prefill over the same T tokens (per sequence)."""
    steps, N, H = 20, 3, 2
    d = kin.make_inputs((steps, N), H, 128, 128, torch.float32, seed=13, num_states=N,
                        state_std=0.2)
    outs, state = run_decode_steps(d)
    seqmajor = lambda x: x.transpose(0, 1).reshape(N * steps, *x.shape[2:]).contiguous()
    p = {key: seqmajor(d[key]) for key in ("q", "k", "v", "g", "beta")}
    p["init_state"] = d["init_state"]
    p["cu_seqlens"] = [i * steps for i in range(N + 1)]
    dd = to_device(p)
    po, pf, _ = gpu_prefill(dd, 16)
    torch.cuda.synchronize()
    po = po.reshape(N, steps, H, 128).transpose(0, 1)
    assert rel_l2(outs, po.double().cpu().numpy()) <= 1e-4
    assert rel_l2(state, pf.double().cpu().numpy()) <= 1e-4


def test_decode_full_workload_sampled():
    """512 sequences x 32 heads x 256 steps from an N(0, 0.02) state, as benchmarked;
    the oracle replays sampled (sequence, head) units over all 256 steps."""
    w = kin.WORKLOADS["decode"]
    d = kin.make_workload("decode", device="cuda")
    state = d["init_state"].clone()
    outs = torch.empty_like(d["v"])
    for t in range(w["steps"]):
        kda.kda_decode(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], state,
                       out=outs[t])
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    units = {(0, 0), (511, 31)} | {(int(rng.integers(512)), int(rng.integers(32))) for _ in range(4)}
    for n, h in sorted(units):
        sl = lambda x: x[:, n:n + 1, h:h + 1].to("cpu")
        ro, rf = oracle.decode(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["g"]), sl(d["beta"]),
                               d["init_state"][n:n + 1, h:h + 1].to("cpu"))
        assert rel_l2(outs[:, n:n + 1, h:h + 1], ro) <= 1e-2
        assert rel_l2(state[n:n + 1, h:h + 1], rf) <= 1e-2
