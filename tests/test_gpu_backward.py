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


def chunked_path(dtype, Dk, Dv):
    """BF16 with D_k = D_v = 128 runs the chunked tensor-core backward."""
    return dtype == torch.bfloat16 and Dk == 128 and Dv == 128


def bound(dtype, Dk, Dv):
    """FP32 SIMT: the FP32 bound for either input dtype (it reads the exact bits
    the oracle reads).  Chunked tensor-core path: the BF16 bound of the forward,
    since its products take BF16 operands with FP32 accumulation."""
    return 1e-2 if chunked_path(dtype, Dk, Dv) else 1e-4


def run_both(lengths, H, Dk, Dv, dtype, seed, use_init=True, use_dfin=True, tol=None,
             mutate=None):
    d = make_case(lengths, H, Dk, Dv, dtype, seed=seed, state_std=0.1)
    if mutate is not None:
        mutate(d)
    tol = tol or bound(dtype, Dk, Dv)
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
    if sum(lengths) > 0:
        assert kda.kda_last_backward_path() == (1 if chunked_path(dtype, Dk, Dv) else 0)
    ref = oracle.backward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], d_out,
                          init_state=d["init_state"] if use_init else None,
                          d_final=d_fin if use_dfin else None)
    errs = {n: rel_l2(x, r) for n, x, r in zip(NAMES, got, ref)}
    for n, e in errs.items():
        if n == "dg" and chunked_path(dtype, Dk, Dv):
            check_dg(got[3], ref, d, lengths)
            continue
        assert e <= tol, f"{n}: rel-L2 {e:.3e} > {tol:.0e} ({errs})"
    return errs


def dg_term_scale(ref, d, lengths):
    """dg is the reverse cumulative sum, inside each 64-token chunk, of
    dGam = q * dq + k * (dk_plus - dk_minus): products that largely cancel.
    This returns that sum taken over the magnitudes |q * dq| + |k * dk|
    instead (FP64, from the oracle's dq and dk), the scale against which a
    cancelling sum's rounding error is measured."""
    q = d["q"].double().numpy()
    k = d["k"].double().numpy()
    mag = np.abs(q * ref[0]) + np.abs(k * ref[1])
    out = np.zeros_like(mag)
    cu = d["cu_seqlens"]
    for a, b in zip(cu[:-1], cu[1:]):
        for c0 in range(a, b, 64):
            blk = mag[c0:min(c0 + 64, b)]
            out[c0:c0 + blk.shape[0]] = np.cumsum(blk[::-1], axis=0)[::-1]
    return out


def check_dg(dg, ref, d, lengths):
    """dg on the chunked tensor-core path: rel-L2 1e-2 of dg, plus 2e-5 (a
    hundredth of the BF16 unit roundoff 2^-9) of the scale of the terms it
    is summed from.  For ordinary gates that scale is about 60x |dg| and the
    second part adds about 1e-3; at the decay floor (g = -5 everywhere) dg is
    about 5000x smaller than its terms, and a bound on dg alone would ask the
    BF16 products for more digits than they carry."""
    err = float(np.linalg.norm(dg.detach().double().cpu().numpy() - ref[3]))
    scale = float(np.linalg.norm(dg_term_scale(ref, d, lengths)))
    bound = 1e-2 * float(np.linalg.norm(ref[3])) + 2e-5 * scale
    assert err <= bound, f"dg: |err| {err:.3e} > {bound:.3e} (|dg| {np.linalg.norm(ref[3]):.3e}, term scale {scale:.3e})"


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dims", [(32, 32), (64, 128), (128, 64), (128, 128)])
def test_backward_matches_oracle(dtype, dims):
    """Ragged sequences around the 4-token replay blocks (last blocks of 1, 2, 3 and 4
    tokens), nonzero initial state and final-state gradient.  D_v of 64 and 128 run
    2 and 4 column slices whose row-sum parts are added by the second kernel.  The
    SIMT kernel reads the same bits as the oracle, so its bound is the FP32 one for
    both input dtypes; BF16 at D = 128 runs the chunked tensor-core kernels."""
    Dk, Dv = dims
    run_both([1, 2, 15, 16, 17, 42], 2, Dk, Dv, dtype, seed=5)


@pytest.mark.parametrize("lengths", [[1, 63, 64, 65], [130, 200, 7], [256]],
                         ids=["around_one_chunk", "ragged_multi_chunk", "four_chunks"])
def test_chunked_backward_ragged(lengths):
    """The chunked tensor-core backward on ragged sequences: partial last chunks
    (identity-token padding), several chunks per sequence (the chain carries dS
    across chunk ends), three heads."""
    run_both(lengths, 3, 128, 128, torch.bfloat16, seed=len(lengths) + lengths[0])


def test_chunked_backward_with_empty_sequences():
    """Empty sequences inside a batch on the chunked path: they own no chunk,
    so their d_init is the final-state gradient passed through, and the
    sequences around them keep their packet, state and item numbering."""
    errs = run_both([0, 70, 0, 5, 0], 2, 128, 128, torch.bfloat16, seed=79)
    assert errs["d_init"] <= 1e-2


def test_chunked_backward_many_items_per_cta():
    """More (chunk, head) items than CTAs (one per SM), over ragged sequences:
    every CTA walks several items, so the next item's inputs are copied in
    during the current item's reverse scan, across sequence boundaries, partial
    chunks and first chunks (initial state); the state part's S0 then comes
    from the initial-state tiles and the forward's chunk-end tiles alike."""
    rng = np.random.default_rng(77)
    lengths = [int(x) for x in rng.integers(1, 400, size=24)] + [64, 128, 1]
    run_both(lengths, 8, 128, 128, torch.bfloat16, seed=78)


@pytest.mark.parametrize("case", ["g_floor", "g_zero", "beta_zero", "beta_one",
                                  "strong_decay_16_32", "alternate_8"])
def test_chunked_backward_gate_extremes(case):
    """Gates at the floor (g = -5: the cumulative decay spans e^-320 inside a chunk,
    so every gated product needs its factored form), no decay, beta at 0 and 1,
    and strong decay confined to parts of each chunk."""
    def mutate(d):
        T = d["g"].shape[0]
        pos = torch.cat([torch.arange(n) for n in d["lengths"]]) % 64
        if case == "g_floor":
            d["g"].fill_(-5.0)
        elif case == "g_zero":
            d["g"].zero_()
        elif case == "beta_zero":
            d["beta"].zero_()
        elif case == "beta_one":
            d["beta"].fill_(1.0)
        else:
            mask = ((pos >= 16) & (pos < 32)) if case == "strong_decay_16_32" else ((pos // 8) % 2 == 0)
            d["g"] = torch.where(mask[:, None, None], torch.full_like(d["g"], -5.0),
                                 torch.zeros_like(d["g"])).contiguous()
        assert d["g"].shape[0] == T
    run_both([150, 64], 2, 128, 128, torch.bfloat16, seed=31, mutate=mutate)


def test_backward_without_init_or_final_gradient():
    run_both([33, 7], 2, 128, 128, torch.bfloat16, seed=6, use_init=False, use_dfin=False)


def test_backward_empty_sequence_passes_final_gradient_through():
    errs = run_both([0, 20, 0], 1, 32, 32, torch.float32, seed=7)
    assert errs["d_init"] <= 1e-6


def test_backward_bench_shape_sampled_heads():
    """The bench's backward workload (4 sequences x 1024 tokens, H = 32, D = 128,
    BF16 q/k/v, FP32 state N(0, 0.02^2), N(0, 1) upstream gradients), run whole
    on the GPU in the launch configuration the bench times (the chunked
    tensor-core backward).  Three heads are recomputed by the oracle and
    compared in full."""
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
    assert kda.kda_last_backward_path() == 1
    got = [x.cpu() for x in got]
    for h in (0, 13, 31):
        hs = slice(h, h + 1)
        ref = oracle.backward(d["q"][:, hs], d["k"][:, hs], d["v"][:, hs], d["g"][:, hs],
                              d["beta"][:, hs], d["cu_seqlens"], d_out[:, hs],
                              init_state=d["init_state"][:, hs], d_final=d_fin[:, hs])
        for name, x, r in zip(NAMES, got, ref):
            e = rel_l2(x[:, hs], r)
            print(f"backward, head {h}, {name}: rel-L2 {e:.3e}")
            assert e <= 1e-2, f"head {h} {name}: rel-L2 {e:.3e}"
