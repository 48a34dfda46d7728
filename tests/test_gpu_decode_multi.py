"""Multi-token (speculative-verify) decode through the C ABI against the FP64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_08_b200 import inputs as kin
from linear_attention_08_b200 import kda
from parity import TOL, rel_l2

pytestmark = pytest.mark.gpu


def reference(d, N, T_new, accept):
    """Oracle outputs for all draft tokens and the state after each accepted prefix."""
    cu = [n * T_new for n in range(N + 1)]
    flat = {x: d[x].reshape(N * T_new, *d[x].shape[2:]) for x in ("q", "k", "v", "g", "beta")}
    out, fin, ck = oracle.prefill(flat["q"], flat["k"], flat["v"], flat["g"], flat["beta"], cu,
                                  d["init_state"], ckpt_interval=1)
    H = d["q"].shape[2]
    states = d["init_state"].double().numpy().copy()
    for n in range(N):
        a = int(accept[n])
        if a > 0:
            states[n] = ck[n * T_new + a - 1]     # checkpoint after a tokens of sequence n
    return out.reshape(N, T_new, H, -1), states


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dims", [(32, 32), (64, 128), (128, 128)])
@pytest.mark.parametrize("T_new", [1, 4, 16])
def test_decode_multi_against_oracle(dtype, dims, T_new):
    Dk, Dv = dims
    N, H = 6, 3
    d = kin.make_inputs((N, T_new), H, Dk, Dv, dtype, seed=31, num_states=N, state_std=0.3)
    accept = np.array([0, T_new, 1, T_new // 2, T_new, max(T_new - 1, 0)])[:N]
    dev = {x: d[x].cuda() for x in ("q", "k", "v", "g", "beta")}
    state = d["init_state"].cuda().clone()
    acc = torch.tensor(accept, dtype=torch.int32, device="cuda")
    out = kda.kda_decode_multi(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], state,
                               accept_len=acc)
    torch.cuda.synchronize()
    ro, rs = reference(d, N, T_new, accept)
    assert rel_l2(out, ro) <= TOL[dtype]
    assert rel_l2(state, rs) <= TOL[dtype]


def test_decode_multi_all_accepted_and_single_step():
    N, H, T_new = 4, 2, 8
    d = kin.make_inputs((N, T_new), H, 128, 128, torch.bfloat16, seed=32, num_states=N,
                        state_std=0.1)
    dev = {x: d[x].cuda() for x in ("q", "k", "v", "g", "beta")}
    s1 = d["init_state"].cuda().clone()
    out = kda.kda_decode_multi(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], s1)
    # the same tokens one decode step at a time
    s2 = d["init_state"].cuda().clone()
    outs = [kda.kda_decode(dev["q"][:, t].contiguous(), dev["k"][:, t].contiguous(),
                           dev["v"][:, t].contiguous(), dev["g"][:, t].contiguous(),
                           dev["beta"][:, t].contiguous(), s2)
            for t in range(T_new)]
    torch.cuda.synchronize()
    # same arithmetic up to the summation order of q . k
    assert rel_l2(out, torch.stack(outs, 1).double().cpu().numpy()) <= 2e-3   # bf16 outputs
    assert rel_l2(s1, s2.double().cpu().numpy()) <= 1e-6


def test_decode_multi_full_batch_sampled():
    """512 sequences x 32 heads, 8 draft tokens each, random accepted lengths."""
    N, H, T_new = 512, 32, 8
    d = kin.make_inputs((N, T_new), H, 128, 128, torch.bfloat16, seed=33, num_states=N,
                        state_std=0.02, device="cuda")
    gen = torch.Generator("cpu").manual_seed(3)
    accept = torch.randint(0, T_new + 1, (N,), generator=gen, dtype=torch.int32)
    state = d["init_state"].clone()
    out = kda.kda_decode_multi(d["q"], d["k"], d["v"], d["g"], d["beta"], state,
                               accept_len=accept.cuda())
    torch.cuda.synchronize()
    for n, h in [(0, 0), (511, 31), (137, 5), (300, 17)]:
        sl = {x: d[x][n:n + 1, :, h:h + 1].cpu() for x in ("q", "k", "v", "g", "beta")}
        sl["init_state"] = d["init_state"][n:n + 1, h:h + 1].cpu()
        ro, rs = reference(sl, 1, T_new, accept[n:n + 1].numpy())
        assert rel_l2(out[n:n + 1, :, h:h + 1], ro) <= 1e-2
        assert rel_l2(state[n:n + 1, h:h + 1], rs) <= 1e-2
