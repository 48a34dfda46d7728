"""kda_prefill_noalloc, the prefill entry point for callers that cannot allocate
device memory when they call (an engine that has given all free memory to its
own pool, or a runtime whose allocator the library cannot reach): its output
must match kda_prefill's on two calls in a row through the C ABI.  This file
sorts last so that a run stopping at the first failure has run the rest."""
import ctypes

import pytest
import torch

from linear_attention_08_b200 import kda
from parity import TOL, make_case, oracle_full, rel_l2, to_device

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 128 << 20      # KDA_NOALLOC_SCRATCH_BYTES in include/kda.h
PACKET_BYTES = 74240


def noalloc_lib():
    lib = kda.load()
    P = ctypes.c_void_p
    lib.kda_prefill_noalloc.argtypes = [P, P, P, P, P, P, P, P, P, ctypes.c_int64, P,
                                        ctypes.POINTER(kda.KdaShape), P]
    lib.kda_prefill_noalloc.restype = ctypes.c_int
    return lib


def ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_prefill_two_calls():
    """16 sequences x 32 heads: one chunk of every (sequence, head) takes 38 MB, so
    the fixed array holds windows of three chunks and the batch runs in several
    windows.  Checkpoints every 128 tokens, nonzero initial state.

    Windows change where the FP32 state waits between chunks (tensor memory or
    global memory), not how any chunk is computed, so the result must equal
    kda_prefill's (one window) bit for bit; both are also held to the FP64
    oracle."""
    lib = noalloc_lib()
    lengths = [700, 64, 1, 1000, 333, 512, 97, 800] * 2
    H, interval = 32, 128
    assert len(lengths) * H * PACKET_BYTES * 4 > SCRATCH_BYTES   # several windows
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for seed in (11, 12):
        d = make_case(lengths, H, 128, 128, torch.bfloat16, seed=seed, state_std=0.05)
        dd = to_device(d)
        ref_o, ref_f, ref_c = kda.kda_prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"],
                                              dd["cu_dev"], init_state=dd["init_state"],
                                              chunk=64, ckpt_interval=interval,
                                              cu_seqlens_host=dd["cu_seqlens"])
        out = torch.empty_like(ref_o)
        fin = torch.empty_like(ref_f)
        ck = torch.empty_like(ref_c)
        shape = kda.make_shape(len(lengths), sum(lengths), H, 128, 128, 64, kda.KDA_DTYPE_BF16)
        st = lib.kda_prefill_noalloc(ptr(dd["q"]), ptr(dd["k"]), ptr(dd["v"]), ptr(dd["g"]),
                                     ptr(dd["beta"]), ptr(dd["init_state"]), ptr(dd["cu_dev"]),
                                     ptr(out), ptr(fin), interval, ptr(ck), ctypes.byref(shape),
                                     stream)
        assert st == kda.KDA_OK, st
        torch.cuda.synchronize()
        assert torch.equal(out, ref_o)
        assert torch.equal(fin, ref_f)
        assert torch.equal(ck, ref_c)
        tol = TOL[torch.bfloat16]
        ro, rf, rc = oracle_full(d, interval)
        assert rel_l2(out, ro) <= tol
        assert rel_l2(fin, rf) <= tol
        assert rel_l2(ck, rc) <= tol


def test_noalloc_rejects_what_does_not_fit():
    """Too many (sequence, head) pairs for one chunk each, or a shape off the
    two-pass path: KDA_ERR_UNSUPPORTED before any work is queued."""
    lib = noalloc_lib()
    a = ctypes.c_void_p(1 << 20)
    b = ctypes.c_void_p(1 << 34)
    big = kda.make_shape(64, 64 * 100, 32, 128, 128, 64, kda.KDA_DTYPE_BF16)
    assert 64 * 32 * PACKET_BYTES > SCRATCH_BYTES
    assert lib.kda_prefill_noalloc(a, a, a, a, a, None, a, b, b, 0, None, ctypes.byref(big),
                                   None) == kda.KDA_ERR_UNSUPPORTED
    fp32 = kda.make_shape(2, 100, 2, 128, 128, 64, kda.KDA_DTYPE_F32)
    assert lib.kda_prefill_noalloc(a, a, a, a, a, None, a, b, b, 0, None, ctypes.byref(fp32),
                                   None) == kda.KDA_ERR_UNSUPPORTED
