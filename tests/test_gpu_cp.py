"""Context parallelism on one GPU: a long sequence split into segments, each
run as a rank would run it (two prefill calls), the segments' transitions
composed and the outputs corrected with the library's affine kernels; the
result must match one prefill over the whole sequence and the FP64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_08_b200 import cp, kda
from parity import make_case, rel_l2, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("interval", [0, 128])
def test_segments_match_one_call(interval):
    bounds = [0, 256, 384, 700]
    d = make_case([bounds[-1]], 4, 128, 128, torch.bfloat16, seed=12, state_std=0.05)
    dd = to_device(d)
    segs = []
    for a, b in zip(bounds[:-1], bounds[1:]):
        segs.append(cp.segment_pass(*(dd[n][a:b].contiguous() for n in ("q", "k", "v", "g", "beta")),
                                    chunk=64, ckpt_interval=interval))
    As, Bs = [s["A"] for s in segs], [s["B"] for s in segs]
    outs, cks = [], []
    for r, seg in enumerate(segs):
        S_in = cp.incoming_state(As, Bs, r, dd["init_state"][0].contiguous())
        out, fin, ck = cp.finish_segment(seg, S_in)
        outs.append(out)
        if ck is not None:
            cks.append(ck)
    torch.cuda.synchronize()
    out = torch.cat(outs)
    whole_o, whole_f, whole_c = kda.kda_prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"],
                                                dd["cu_dev"], init_state=dd["init_state"], chunk=64,
                                                ckpt_interval=interval, cu_seqlens_host=d["cu_seqlens"])
    ro, rf, rc = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"],
                                d["init_state"], interval, 0)
    torch.cuda.synchronize()
    assert rel_l2(out, ro) <= 1e-2
    assert rel_l2(fin, rf[0]) <= 1e-2
    assert rel_l2(out, whole_o.double().cpu().numpy()) <= 1e-2
    if interval:
        assert rel_l2(torch.cat(cks), rc) <= 1e-2


def test_affine_kernels_against_fp64():
    rng = np.random.default_rng(3)
    H, Dk, Dv, R = 3, 64, 128, 300
    x = torch.tensor(rng.normal(size=(R, H, Dk)), dtype=torch.float32, device="cuda")
    M = torch.tensor(rng.normal(size=(H, Dk, Dv)), dtype=torch.float32, device="cuda")
    y0 = torch.tensor(rng.normal(size=(R, H, Dv)), dtype=torch.float32, device="cuda")
    y = y0.clone()
    kda.kda_affine_rows(x, M, y, accumulate=True)
    A = torch.tensor(rng.normal(size=(H, Dk, Dk)), dtype=torch.float32, device="cuda")
    S = torch.tensor(rng.normal(size=(H, Dk, Dv)), dtype=torch.float32, device="cuda")
    B = torch.tensor(rng.normal(size=(H, Dk, Dv)), dtype=torch.float32, device="cuda")
    Z = kda.kda_affine_state(A, S, B)
    S2 = S.clone()
    kda.kda_affine_state(A, S2, B, S_out=S2)          # in place over S_in
    torch.cuda.synchronize()
    ref_y = y0.double() + torch.einsum("rhc,hcd->rhd", x.double(), M.double())
    ref_z = torch.einsum("hci,hid->hcd", A.double(), S.double()) + B.double()
    assert rel_l2(y, ref_y.cpu().numpy()) <= 1e-5
    assert rel_l2(Z, ref_z.cpu().numpy()) <= 1e-5
    assert torch.equal(S2, Z)


def test_many_segments_match_one_call():
    """Six segments: the correction o = o(B) + S_in^T (A_t^T q_t) rounds o(B) and
    A_t^T q_t to BF16 before the FP32 affine map (two more roundings than one
    prefill call), and the incoming state folds five transitions for the last
    segment.  Both the outputs and the final state must stay within the BF16
    bound of one prefill call and of the oracle."""
    bounds = [0, 128, 256, 320, 512, 640, 777]
    d = make_case([bounds[-1]], 2, 128, 128, torch.bfloat16, seed=13, state_std=0.05)
    dd = to_device(d)
    segs = [cp.segment_pass(*(dd[n][a:b].contiguous() for n in ("q", "k", "v", "g", "beta")),
                            chunk=64, ckpt_interval=64)
            for a, b in zip(bounds[:-1], bounds[1:])]
    As, Bs = [s["A"] for s in segs], [s["B"] for s in segs]
    outs, cks = [], []
    for r, seg in enumerate(segs):
        out, fin, ck = cp.finish_segment(seg, cp.incoming_state(As, Bs, r, dd["init_state"][0].contiguous()))
        outs.append(out)
        cks.append(ck)
    torch.cuda.synchronize()
    out = torch.cat(outs)
    whole_o, whole_f, whole_c = kda.kda_prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"],
                                                dd["cu_dev"], init_state=dd["init_state"], chunk=64,
                                                ckpt_interval=64, cu_seqlens_host=d["cu_seqlens"])
    ro, rf, rc = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"],
                                d["init_state"], 64, 0)
    torch.cuda.synchronize()
    e_call = rel_l2(out, whole_o.double().cpu().numpy())
    e_oracle = rel_l2(out, ro)
    print(f"six segments: o vs one call {e_call:.3e}, vs oracle {e_oracle:.3e}, "
          f"one call vs oracle {rel_l2(whole_o, ro):.3e}")
    assert e_call <= 1e-2 and e_oracle <= 1e-2
    assert rel_l2(fin, rf[0]) <= 1e-2
    assert rel_l2(torch.cat(cks), rc) <= 1e-2
