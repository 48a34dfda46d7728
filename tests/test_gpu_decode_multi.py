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


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_multi_all_accepted_and_single_step(dtype):
    N, H, T_new = 4, 2, 8
    d = kin.make_inputs((N, T_new), H, 128, 128, dtype, seed=32, num_states=N, state_std=0.1)
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
    ref_out = torch.stack(outs, 1).double().cpu().numpy()
    if dtype == torch.float32:
        # The same recurrence in FP32 on the CUDA cores.  The multi-token kernel
        # applies a group's decay as exp of the cumulative log-decay instead of
        # one factor per token, so the two differ by FP32 rounding over 8 steps.
        assert rel_l2(out, ref_out) <= 1e-5
        assert rel_l2(s1, s2.double().cpu().numpy()) <= 1e-5
    else:
        # BF16 with D = 128 runs the draft as one chunk on the tensor cores,
        # which round S0 and the chunk's operands to BF16: the two paths agree
        # to the BF16 bound, not to FP32 rounding.
        assert rel_l2(out, ref_out) <= TOL[torch.bfloat16]
        assert rel_l2(s1, s2.double().cpu().numpy()) <= TOL[torch.bfloat16]


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


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_multi_extreme_decay(dtype):
    """Log-decays far below the workload's floor of -5 (down to -40 per token and
    -1e4 on whole channels): the group's cumulative decay passes e^-60, where the
    kernel's lazy scale stops, and the result must still match the oracle."""
    N, H, T_new = 3, 2, 16
    d = kin.make_inputs((N, T_new), H, 128, 128, dtype, seed=34, num_states=N, state_std=0.3)
    gen = torch.Generator().manual_seed(5)
    g = d["g"].clone()
    mask = torch.rand(g.shape, generator=gen) < 0.3
    g[mask] = -40.0 * torch.rand(int(mask.sum()), generator=gen)
    g[0, :, 0, 5] = -1.0e4          # channel 5 of (sequence 0, head 0) forgets at every token
    g[2, 3:, 1, 77] = -1.0e4        # one channel forgets from the 4th token on
    d["g"] = g.contiguous()
    accept = np.array([T_new, 5, 12])
    dev = {x: d[x].cuda() for x in ("q", "k", "v", "g", "beta")}
    state = d["init_state"].cuda().clone()
    out = kda.kda_decode_multi(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], state,
                               accept_len=torch.tensor(accept, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(state).all()
    ro, rs = reference(d, N, T_new, accept)
    assert rel_l2(out, ro) <= TOL[dtype]
    assert rel_l2(state, rs) <= TOL[dtype]


@pytest.mark.parametrize("T_new", [9, 64])
def test_decode_multi_long_drafts(T_new):
    """Drafts longer than one staging group: later groups are staged from global
    memory and start from the rescaled state of the group before."""
    N, H = 2, 3
    d = kin.make_inputs((N, T_new), H, 128, 128, torch.float32, seed=35, num_states=N,
                        state_std=0.3)
    accept = np.array([T_new, T_new - 1])
    dev = {x: d[x].cuda() for x in ("q", "k", "v", "g", "beta")}
    state = d["init_state"].cuda().clone()
    out = kda.kda_decode_multi(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], state,
                               accept_len=torch.tensor(accept, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    ro, rs = reference(d, N, T_new, accept)
    assert rel_l2(out, ro) <= TOL[torch.float32]
    assert rel_l2(state, rs) <= TOL[torch.float32]


def test_decode_multi_many_units_per_cta():
    """512 (sequence, head) units, more than two per CTA of the persistent grid:
    every unit against the oracle, accepted lengths 0..8."""
    N, H, T_new = 64, 8, 8
    d = kin.make_inputs((N, T_new), H, 128, 128, torch.bfloat16, seed=36, num_states=N,
                        state_std=0.05)
    accept = np.arange(N) % (T_new + 1)
    dev = {x: d[x].cuda() for x in ("q", "k", "v", "g", "beta")}
    state = d["init_state"].cuda().clone()
    out = kda.kda_decode_multi(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], state,
                               accept_len=torch.tensor(accept, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    ro, rs = reference(d, N, T_new, accept)
    assert rel_l2(out, ro) <= TOL[torch.bfloat16]
    assert rel_l2(state, rs) <= TOL[torch.bfloat16]
    untouched = accept == 0
    assert torch.equal(state[torch.from_numpy(untouched).cuda()].cpu(),
                       d["init_state"][torch.from_numpy(untouched)])


@pytest.mark.parametrize("T_new", [2, 15, 16, 17])
def test_decode_multi_bf16_draft_lengths(T_new):
    """Drafts around the 16-token limit of the tensor-core form (17 runs the
    CUDA-core kernel)."""
    N, H = 3, 4
    d = kin.make_inputs((N, T_new), H, 128, 128, torch.bfloat16, seed=37, num_states=N,
                        state_std=0.2)
    accept = np.array([T_new, 1, T_new // 2])
    dev = {x: d[x].cuda() for x in ("q", "k", "v", "g", "beta")}
    state = d["init_state"].cuda().clone()
    out = kda.kda_decode_multi(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], state,
                               accept_len=torch.tensor(accept, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    ro, rs = reference(d, N, T_new, accept)
    assert rel_l2(out, ro) <= TOL[torch.bfloat16]
    assert rel_l2(state, rs) <= TOL[torch.bfloat16]
