"""States at explicit positions (prompt boundaries) through kda_prefill_at, against the oracle."""
import pytest
import torch

import oracle
from linear_attention_08_b200 import kda
from parity import TOL, make_case, rel_l2, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,dims,chunk", [(torch.bfloat16, (128, 128), 64),
                                              (torch.float32, (64, 32), 16),
                                              (torch.bfloat16, (128, 128), 16)])
def test_positions_against_oracle(dtype, dims, chunk):
    Dk, Dv = dims
    lengths = [300, 70, 1, 129]
    positions = [[0, 37, 64, 64, 100, 191, 256, 299, 300, 5000],   # mid-chunk, aligned,
                 [69, 70],                                           # duplicate, past end
                 [1],
                 []]
    interval = 2 * chunk
    d = make_case(lengths, 2, Dk, Dv, dtype, seed=41, state_std=0.2)
    dd = to_device(d)
    out, fin, ck, ps = kda.kda_prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["cu_dev"],
                                       init_state=dd["init_state"], chunk=chunk,
                                       ckpt_interval=interval, cu_seqlens_host=d["cu_seqlens"],
                                       positions=positions)
    torch.cuda.synchronize()
    ro, rf, rc, rp = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"],
                                    d["init_state"], interval, positions=positions)
    tol = TOL[dtype]
    assert ps.shape[0] == rp.shape[0] == sum(len(p) for p in positions)
    for name, x, ref in (("o", out, ro), ("S", fin, rf), ("ckpt", ck, rc), ("pos", ps, rp)):
        e = rel_l2(x, ref)
        assert e <= tol, f"{name}: {e:.3e}"
    # cutting chunks at positions does not change the outputs
    o2, f2, _ = kda.kda_prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["cu_dev"],
                                init_state=dd["init_state"], chunk=chunk)
    torch.cuda.synchronize()
    assert rel_l2(out, o2.double().cpu().numpy()) <= tol
    assert rel_l2(fin, f2.double().cpu().numpy()) <= tol


def test_position_state_resumes_exactly():
    """Resuming from the state stored at an unaligned prompt boundary reproduces the rest:
    to rounding when the resumed call runs the same single-pass kernel (no workspace),
    within the parity tolerance when it runs the two-pass kernels."""
    L, cut = 500, 173
    d = make_case([L], 2, 128, 128, torch.bfloat16, seed=42, state_std=0.1)
    dd = to_device(d)
    out, fin, _, ps = kda.kda_prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["cu_dev"],
                                      init_state=dd["init_state"], chunk=64, positions=[[cut]])
    for ws, tol in ((None, 1e-5), ("auto", 1e-2)):
        o_r, f_r, _ = kda.kda_prefill(dd["q"][cut:].contiguous(), dd["k"][cut:].contiguous(),
                                      dd["v"][cut:].contiguous(), dd["g"][cut:].contiguous(),
                                      dd["beta"][cut:].contiguous(),
                                      torch.tensor([0, L - cut], dtype=torch.int32, device="cuda"),
                                      init_state=ps[0:1].contiguous(), chunk=64, workspace=ws)
        torch.cuda.synchronize()
        assert rel_l2(o_r, out[cut:].double().cpu().numpy()) <= tol
        assert rel_l2(f_r, fin.double().cpu().numpy()) <= tol
