"""Backward pass on the GPU against the FP64 backward oracle (which is pinned to
finite differences of the forward oracle in test_oracle_backward.py)."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_08_b200 import kda
from parity import make_case, rel_l2, to_device

pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "dg", "dbeta", "d_init")


def run_both(lengths, H, Dk, Dv, dtype, seed, use_init=True, use_dfin=True, tol=1e-4):
    d = make_case(lengths, H, Dk, Dv, dtype, seed=seed, state_std=0.1)
    dd = to_device(d)
    rng = np.random.default_rng(seed + 100)
    T = sum(lengths)
    d_out = torch.tensor(rng.normal(size=(T, H, Dv)), dtype=torch.float32)
    d_fin = torch.tensor(rng.normal(size=(len(lengths), H, Dk, Dv)) * 0.5, dtype=torch.float32)
    init = dd["init_state"] if use_init else None
    got = kda.kda_backward(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["cu_dev"],
                           d_out.cuda(), init_state=init,
                           d_final=d_fin.cuda() if use_dfin else None)
    torch.cuda.synchronize()
    ref = oracle.backward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], d_out,
                          init_state=d["init_state"] if use_init else None,
                          d_final=d_fin if use_dfin else None)
    errs = {n: rel_l2(x, r) for n, x, r in zip(NAMES, got, ref)}
    for n, e in errs.items():
        assert e <= tol, f"{n}: rel-L2 {e:.3e} > {tol:.0e} ({errs})"
    return errs


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dims", [(32, 32), (64, 128), (128, 64), (128, 128)])
def test_backward_matches_oracle(dtype, dims):
    """Ragged sequences around the 4-token replay blocks (last blocks of 1, 2, 3 and 4
    tokens), nonzero initial state and final-state gradient.  D_v of 64 and 128 run
    2 and 4 column slices whose row-sum parts are added by the second kernel.  The
    GPU reads the same bits as the oracle, so the bound is the FP32 one for both
    input dtypes."""
    Dk, Dv = dims
    run_both([1, 2, 15, 16, 17, 42], 2, Dk, Dv, dtype, seed=5)


def test_backward_without_init_or_final_gradient():
    run_both([33, 7], 2, 128, 128, torch.bfloat16, seed=6, use_init=False, use_dfin=False)


def test_backward_empty_sequence_passes_final_gradient_through():
    errs = run_both([0, 20, 0], 1, 32, 32, torch.float32, seed=7)
    assert errs["d_init"] <= 1e-6


def test_backward_bench_shape_sampled_heads():
    """The bench's backward workload (4 sequences x 1024 tokens, H = 32, D = 128,
    BF16 q/k/v, FP32 state N(0, 0.02^2), N(0, 1) upstream gradients), run whole
    on the GPU in the launch configuration the bench times (4 column slices per
    head plus the slice-sum kernel).  Three heads are recomputed by the oracle
    and compared in full."""
    lengths, H, D = [1024] * 4, 32, 128
    d = make_case(lengths, H, D, D, torch.bfloat16, seed=11, state_std=0.02)
    dd = to_device(d)
    rng = np.random.default_rng(111)
    T = sum(lengths)
    d_out = torch.tensor(rng.normal(size=(T, H, D)), dtype=torch.float32)
    d_fin = torch.tensor(rng.normal(size=(len(lengths), H, D, D)), dtype=torch.float32)
    got = kda.kda_backward(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["cu_dev"],
                           d_out.cuda(), init_state=dd["init_state"], d_final=d_fin.cuda())
    torch.cuda.synchronize()
    got = [x.cpu() for x in got]
    for h in (0, 13, 31):
        hs = slice(h, h + 1)
        ref = oracle.backward(d["q"][:, hs], d["k"][:, hs], d["v"][:, hs], d["g"][:, hs],
                              d["beta"][:, hs], d["cu_seqlens"], d_out[:, hs],
                              init_state=d["init_state"][:, hs], d_final=d_fin[:, hs])
        for name, x, r in zip(NAMES, got, ref):
            e = rel_l2(x[:, hs], r)
            assert e <= 1e-4, f"head {h} {name}: rel-L2 {e:.3e}"
