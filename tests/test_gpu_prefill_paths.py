"""Prefill routes against the FP64 oracle: the two-pass tensor-core path in one
and in several windows of chunks (caller workspace), the single-pass kernel
(no workspace), and the plain C entry that takes its workspace from the
library's pool."""
import ctypes

import pytest
import torch

from linear_attention_08_b200 import kda
from parity import TOL, make_case, oracle_full, rel_l2, to_device

pytestmark = pytest.mark.gpu

LENGTHS = [200, 64, 1, 130, 257]


def run(dd, interval, workspace, want_final=True, use_init=True):
    return kda.kda_prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["cu_dev"],
                           init_state=dd["init_state"] if use_init else None, chunk=64,
                           ckpt_interval=interval, cu_seqlens_host=dd["cu_seqlens"],
                           want_final=want_final, workspace=workspace)


def shape_of(dd):
    T, H, Dk = dd["q"].shape
    return kda.make_shape(len(dd["cu_seqlens"]) - 1, T, H, Dk, dd["v"].shape[2], 64,
                          kda.KDA_DTYPE_BF16)


def check(d, out, fin, ck, interval, use_init=True, tol=TOL[torch.bfloat16]):
    ro, rf, rc = oracle_full(d, interval, use_init)
    assert rel_l2(out, ro) <= tol
    if fin is not None:
        assert rel_l2(fin, rf) <= tol
    if interval > 0 and rc.shape[0]:
        assert rel_l2(ck, rc) <= tol


def test_path_query():
    d = to_device(make_case(LENGTHS, 3, 128, 128, torch.bfloat16, seed=3))
    assert kda.kda_prefill_path(shape_of(d)) == 2
    s = shape_of(d)
    s.chunk = 16      # the same tensor-core kernels (64-token chunks inside)
    assert kda.kda_prefill_path(s) == 2
    s.qkv_dtype = kda.KDA_DTYPE_F32
    assert kda.kda_prefill_path(s) == 0
    s = shape_of(d)
    s.num_seqs = 4096   # too many sequences for the two-pass path
    assert kda.kda_prefill_path(s) == 1
    assert kda.kda_prefill_workspace_bytes(shape_of(d)) >= kda.kda_prefill_workspace_min_bytes(shape_of(d)) > 0


@pytest.mark.parametrize("windows_of", [1, 2, 3, None])
@pytest.mark.parametrize("want_final", [True, False])
def test_two_pass_windows(windows_of, want_final):
    """Workspace for windows of 1, 2 or 3 chunks (None: one window), checkpoints every two
    chunks, nonzero initial state; without final_state the carried state lives in the
    workspace."""
    d = make_case(LENGTHS, 3, 128, 128, torch.bfloat16, seed=4, state_std=0.1)
    dd = to_device(d)
    shape = shape_of(dd)
    if windows_of is None:
        nbytes = kda.kda_prefill_workspace_bytes(shape)
    else:
        N, H = len(LENGTHS), 3
        nbytes = (kda.kda_prefill_workspace_min_bytes(shape)
                  + (windows_of - 1) * N * H * 74240)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    out, fin, ck = run(dd, 128, ws, want_final=want_final)
    torch.cuda.synchronize()
    check(d, out, fin if want_final else None, ck, 128)


@pytest.mark.parametrize("H", [3, 12, 16])
def test_chain_value_slices(H):
    """The chain pass splits each (sequence, head)'s value columns over 4, 2 or 1
    CTAs when N*H is at most a quarter, a half, or more than half the SM count:
    5 sequences x H = 3, 12, 16 reach all three widths on a 148-SM B200.  Each
    against the oracle, with checkpoints every 64 tokens and the final state."""
    d = make_case(LENGTHS, H, 128, 128, torch.bfloat16, seed=40 + H)
    dd = to_device(d)
    out, fin, ck = run(dd, 64, "auto")
    torch.cuda.synchronize()
    assert kda.kda_last_prefill_path() == 2
    check(d, out, fin, ck, 64)


def test_single_pass_and_two_pass_agree():
    d = make_case(LENGTHS, 4, 128, 128, torch.bfloat16, seed=5, state_std=0.05)
    dd = to_device(d)
    o1, f1, c1 = run(dd, 64, None)
    o2, f2, c2 = run(dd, 64, "auto")
    torch.cuda.synchronize()
    check(d, o1, f1, c1, 64)
    check(d, o2, f2, c2, 64)
    assert rel_l2(o1, o2.double().cpu().numpy()) <= 1e-2
    assert rel_l2(f1, f2.double().cpu().numpy()) <= 1e-2


def test_plain_entry_uses_pool():
    """kda_prefill (no workspace argument) twice, then the pool is released."""
    d = make_case(LENGTHS, 3, 128, 128, torch.bfloat16, seed=6, state_std=0.02)
    dd = to_device(d)
    lib = kda.load()
    T, H, Dk = dd["q"].shape
    N = len(LENGTHS)
    out = torch.empty(T, H, 128, dtype=torch.bfloat16, device="cuda")
    fin = torch.empty(N, H, 128, 128, device="cuda")
    shape = shape_of(dd)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        st = lib.kda_prefill(P(dd["q"]), P(dd["k"]), P(dd["v"]), P(dd["g"]), P(dd["beta"]),
                             P(dd["init_state"]), P(dd["cu_dev"]), P(out), P(fin), 0, None,
                             ctypes.byref(shape), stream)
        assert st == kda.KDA_OK
    torch.cuda.synchronize()
    check(d, out, fin, None, 0)
    assert lib.kda_release_workspace_pool() == kda.KDA_OK


def test_many_sequences_single_pass():
    """More sequences than the two-pass path takes: the single-pass kernel runs."""
    lengths = [3, 70] * 520
    d = make_case(lengths, 1, 128, 128, torch.bfloat16, seed=7, state_std=0.02)
    dd = to_device(d)
    out, fin, _ = run(dd, 0, "auto")
    torch.cuda.synchronize()
    check(d, out, fin, None, 0)


@pytest.mark.parametrize("interval,path", [(0, 2), (64, 2), (128, 2), (32, 1), (48, 1)])
def test_chunk16_runs_on_tensor_cores(interval, path):
    """A BF16, D = 128 request for 16-token chunks runs the tensor-core kernels:
    the two-pass ones when the checkpoint interval is a multiple of 64, the
    single-pass one (which cuts its chunks at every checkpoint) otherwise."""
    d = make_case(LENGTHS, 3, 128, 128, torch.bfloat16, seed=8, state_std=0.05)
    dd = to_device(d)
    out, fin, ck = kda.kda_prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["cu_dev"],
                                   init_state=dd["init_state"], chunk=16, ckpt_interval=interval,
                                   cu_seqlens_host=dd["cu_seqlens"])
    torch.cuda.synchronize()
    assert kda.kda_last_prefill_path() == path
    check(d, out, fin, ck, interval)


def test_pool_cap_fallback_is_visible():
    """With the pool cap below the smallest window kda_prefill takes nothing from
    the pool and runs the single-pass kernel; kda_last_prefill_path says so, and
    the result still matches the oracle.  Restoring the cap restores the path."""
    d = make_case(LENGTHS, 3, 128, 128, torch.bfloat16, seed=9, state_std=0.05)
    dd = to_device(d)
    lib = kda.load()
    T, H, _ = dd["q"].shape
    N = len(LENGTHS)
    shape = shape_of(dd)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    try:
        for cap, path in ((0, 1), (kda.kda_prefill_workspace_min_bytes(shape) - 1, 1),
                          (8 << 30, 2)):
            kda.kda_set_workspace_pool_cap(cap)
            out = torch.empty(T, H, 128, dtype=torch.bfloat16, device="cuda")
            fin = torch.empty(N, H, 128, 128, device="cuda")
            ck = torch.empty(kda.kda_ckpt_count(dd["cu_seqlens"], 128), H, 128, 128, device="cuda")
            st = lib.kda_prefill(P(dd["q"]), P(dd["k"]), P(dd["v"]), P(dd["g"]), P(dd["beta"]),
                                 P(dd["init_state"]), P(dd["cu_dev"]), P(out), None, 128, P(ck),
                                 ctypes.byref(shape), stream)
            assert st == kda.KDA_OK
            assert kda.kda_last_prefill_path() == path, cap
            torch.cuda.synchronize()
            check(d, out, None, ck, 128)
    finally:
        kda.kda_set_workspace_pool_cap(8 << 30)


def test_many_windows_run_the_single_pass():
    """64 sequences x 256 tokens x 32 heads with the smallest caller workspace:
    the two-pass path would run 256 one-chunk windows (most of them past every
    sequence), so the single-pass kernel runs; with room for one window the
    two-pass path runs.  Both against the oracle."""
    lengths = [256] * 64
    d = make_case(lengths, 32, 128, 128, torch.bfloat16, seed=41, state_std=0.02)
    dd = to_device(d)
    shape = shape_of(dd)
    ws = torch.empty(kda.kda_prefill_workspace_min_bytes(shape), dtype=torch.uint8, device="cuda")
    out, fin, _ = run(dd, 0, ws)
    torch.cuda.synchronize()
    assert kda.kda_last_prefill_path() == 1
    check(d, out, fin, None, 0)
    ws = torch.empty(kda.kda_prefill_workspace_bytes(shape), dtype=torch.uint8, device="cuda")
    out, fin, _ = run(dd, 0, ws)
    torch.cuda.synchronize()
    assert kda.kda_last_prefill_path() == 2
    check(d, out, fin, None, 0)


def test_many_units_take_the_single_pass_from_the_pool():
    """600 sequences x 4 heads = 2400 (sequence, head) units through the plain C
    entry (workspace from the library's pool): the single-pass kernel runs and
    nothing is taken from the pool; against the oracle."""
    lengths = [8, 1, 17, 64] * 150
    d = make_case(lengths, 4, 128, 128, torch.bfloat16, seed=42, state_std=0.05)
    dd = to_device(d)
    lib = kda.load()
    T, H, _ = dd["q"].shape
    N = len(lengths)
    out = torch.empty(T, H, 128, dtype=torch.bfloat16, device="cuda")
    fin = torch.empty(N, H, 128, 128, device="cuda")
    shape = shape_of(dd)
    assert kda.kda_prefill_path(shape) == 1
    assert kda.kda_prefill_workspace_bytes(shape) == 0
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.kda_prefill(P(dd["q"]), P(dd["k"]), P(dd["v"]), P(dd["g"]), P(dd["beta"]),
                         P(dd["init_state"]), P(dd["cu_dev"]), P(out), P(fin), 0, None,
                         ctypes.byref(shape), stream)
    assert st == kda.KDA_OK
    assert kda.kda_last_prefill_path() == 1
    torch.cuda.synchronize()
    check(d, out, fin, None, 0)
