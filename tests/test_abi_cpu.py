"""Host-side checks of the C ABI that need no GPU: exports and argument validation."""
import ctypes
import os
import re

import pytest

from linear_attention_08_b200 import kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    text = open(os.path.join(ROOT, "include", "kda.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_function():
    lib = kda.load()
    names = header_functions()
    assert "kda_prefill" in names and "kda_decode" in names
    for name in names:
        assert hasattr(lib, name), f"{name} declared in include/kda.h but not exported"
    assert set(kda.EXPORTED) <= set(names)


def test_version_and_strings():
    lib = kda.load()
    assert lib.kda_version() >= 100
    for s in range(5):
        assert lib.kda_status_string(s)


def test_ckpt_count():
    assert kda.kda_ckpt_count([0, 5000, 9000, 9000], 4096) == 1
    assert kda.kda_ckpt_count([0, 8192, 16384], 4096) == 4
    assert kda.kda_ckpt_count([0, 100], 0) == 0
    # the 1M-token workload with 32K snapshots stores 32 of them
    assert kda.kda_ckpt_count([0, 1 << 20], 32768) == 32


def _shape(**kw):
    base = dict(num_seqs=2, total_tokens=64, H=2, Dk=32, Dv=32, chunk=16, dtype_code=0)
    base.update(kw)
    return kda.make_shape(base["num_seqs"], base["total_tokens"], base["H"], base["Dk"],
                          base["Dv"], base["chunk"], base["dtype_code"])


@pytest.mark.parametrize("kw,status", [
    (dict(Dk=48), kda.KDA_ERR_UNSUPPORTED),
    (dict(Dv=256), kda.KDA_ERR_UNSUPPORTED),
    (dict(chunk=32), kda.KDA_ERR_UNSUPPORTED),
    (dict(num_seqs=0), kda.KDA_ERR_INVALID_ARGUMENT),
    (dict(H=0), kda.KDA_ERR_INVALID_ARGUMENT),
    (dict(dtype_code=7), kda.KDA_ERR_INVALID_ARGUMENT),
    (dict(total_tokens=-1), kda.KDA_ERR_INVALID_ARGUMENT),
])
def test_prefill_rejects_bad_shapes_before_launch(kw, status):
    lib = kda.load()
    s = _shape(**kw)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    st = lib.kda_prefill(fake, fake, fake, fake, fake, None, fake, fake, None, 0, None,
                         ctypes.byref(s), None)
    assert st == status


def test_prefill_rejects_bad_pointers_and_intervals():
    lib = kda.load()
    s = _shape()
    a = ctypes.c_void_p(1 << 20)
    b = ctypes.c_void_p(1 << 24)
    c = ctypes.c_void_p(1 << 28)
    mis = ctypes.c_void_p((1 << 20) + 4)
    call = lambda *args: lib.kda_prefill(*args, ctypes.byref(s), None)
    # null cu_seqlens / null q
    assert call(a, a, a, a, a, None, None, b, None, 0, None) == kda.KDA_ERR_INVALID_ARGUMENT
    assert call(None, a, a, a, a, None, a, b, None, 0, None) == kda.KDA_ERR_INVALID_ARGUMENT
    # misaligned q
    assert call(mis, a, a, a, a, None, a, b, None, 0, None) == kda.KDA_ERR_INVALID_ARGUMENT
    # interval not a multiple of the chunk; interval without a buffer; buffer without interval
    assert call(a, a, a, a, a, None, a, b, None, 24, c) == kda.KDA_ERR_INVALID_ARGUMENT
    assert call(a, a, a, a, a, None, a, b, None, 32, None) == kda.KDA_ERR_INVALID_ARGUMENT
    assert call(a, a, a, a, a, None, a, b, None, 0, c) == kda.KDA_ERR_INVALID_ARGUMENT
    # out overlapping an input
    assert call(a, a, a, a, a, None, c, a, None, 0, None) == kda.KDA_ERR_INVALID_ARGUMENT


def test_decode_rejects_bad_arguments():
    lib = kda.load()
    a = ctypes.c_void_p(1 << 20)
    b = ctypes.c_void_p(1 << 26)
    s = kda.make_shape(4, 5, 2, 32, 32, 0, 1)   # total_tokens != num_seqs
    assert lib.kda_decode(a, a, a, a, a, b, ctypes.c_void_p(1 << 28), ctypes.byref(s),
                          None) == kda.KDA_ERR_INVALID_ARGUMENT
    s = kda.make_shape(4, 4, 2, 32, 32, 0, 1)
    # out aliasing the state
    assert lib.kda_decode(a, a, a, a, a, b, b, ctypes.byref(s), None) == kda.KDA_ERR_INVALID_ARGUMENT
    assert lib.kda_decode(a, a, a, a, a, b, ctypes.c_void_p(1 << 28), None,
                          None) == kda.KDA_ERR_INVALID_ARGUMENT


def test_workspace_and_path_queries():
    lib = kda.load()
    s = _shape()
    assert lib.kda_prefill_workspace_bytes(ctypes.byref(s)) == 0
    assert kda.kda_prefill_path(s) == 0            # FP32 runs on the SIMT kernel
    bad = _shape(Dk=12)
    assert kda.kda_prefill_path(bad) == -1
    assert lib.kda_prefill_workspace_bytes(ctypes.byref(bad)) == (1 << 64) - 1
    # BF16, D = 128, C = 64: the two-pass path, 74240 bytes per (chunk, head) packet
    s2 = kda.make_shape(2, 1000, 4, 128, 128, 64, kda.KDA_DTYPE_BF16)
    assert kda.kda_prefill_path(s2) == 2
    chunks_bound = (1000 + 63 * 2) // 64
    state = 2 * 4 * 128 * 128 * 4
    assert lib.kda_prefill_workspace_bytes(ctypes.byref(s2)) == 4 * chunks_bound * 74240 + state + 256
    assert lib.kda_prefill_workspace_min_bytes(ctypes.byref(s2)) == 2 * 4 * 74240 + state + 256
    s3 = kda.make_shape(2000, 4000, 4, 128, 128, 64, kda.KDA_DTYPE_BF16)
    assert kda.kda_prefill_path(s3) == 1          # too many sequences for the two-pass path
    assert lib.kda_prefill_workspace_bytes(ctypes.byref(s3)) == 0
    # chunk 16 names the same tensor-core kernels (64-token chunks inside)
    s4 = kda.make_shape(2, 1000, 4, 128, 128, 16, kda.KDA_DTYPE_BF16)
    assert kda.kda_prefill_path(s4) == 2
    assert lib.kda_prefill_workspace_bytes(ctypes.byref(s4)) == \
        lib.kda_prefill_workspace_bytes(ctypes.byref(s2))
    s5 = kda.make_shape(2000, 4000, 4, 128, 128, 16, kda.KDA_DTYPE_BF16)
    assert kda.kda_prefill_path(s5) == 1
    assert kda.kda_prefill_path(kda.make_shape(2, 1000, 4, 128, 128, 16, kda.KDA_DTYPE_F32)) == 0


def test_path_rules_units_and_windows():
    """The two-pass path takes at most 2048 (sequence, head) units, and only
    when the windows its workspace allows do not cost more than the work."""
    lib = kda.load()
    bf = kda.KDA_DTYPE_BF16
    # 600 x 4 = 2400 units: the single pass, and no workspace is asked for
    many = kda.make_shape(600, 600 * 64, 4, 128, 128, 64, bf)
    assert kda.kda_prefill_path(many) == 1
    assert lib.kda_prefill_workspace_bytes(ctypes.byref(many)) == 0
    assert lib.kda_prefill_workspace_min_bytes(ctypes.byref(many)) == 0
    # exactly 2048 units in one window: the two-pass path
    assert kda.kda_prefill_path(kda.make_shape(64, 64 * 256, 32, 128, 128, 64, bf)) == 2
    # one 1M-token sequence, 32 heads: five windows of an 8 GiB workspace, all of them real
    assert kda.kda_prefill_path(kda.make_shape(1, 1 << 20, 32, 128, 128, 64, bf)) == 2
    # 1000 sequences x 2 heads over 10^8 tokens: ~27K windows, most past the
    # longest sequence, against ~2.9 s of work
    assert kda.kda_prefill_path(kda.make_shape(1000, 100_000_000, 2, 128, 128, 64, bf)) == 1
    # the pool cap bounds the workspace kda_prefill takes: at the minimum, the
    # 64 x 256-token batch would run 256 one-chunk windows
    small = kda.make_shape(64, 64 * 256, 32, 128, 128, 64, bf)
    try:
        kda.kda_set_workspace_pool_cap(lib.kda_prefill_workspace_min_bytes(ctypes.byref(small)))
        assert kda.kda_prefill_path(small) == 1
    finally:
        kda.kda_set_workspace_pool_cap(8 << 30)
    assert kda.kda_prefill_path(small) == 2


def test_last_path_and_pool_cap():
    """The last-path query is untouched by a call that fails validation; the pool
    cap setter accepts any size (0 keeps the pool unused)."""
    lib = kda.load()
    before = kda.kda_last_prefill_path()
    assert before in (-1, 0, 1, 2)
    s = kda.make_shape(2, 1000, 4, 128, 128, 64, kda.KDA_DTYPE_BF16)
    a = ctypes.c_void_p(1 << 20)
    assert lib.kda_prefill(None, a, a, a, a, None, a, a, None, 0, None, ctypes.byref(s),
                           None) == kda.KDA_ERR_INVALID_ARGUMENT
    assert kda.kda_last_prefill_path() == before
    for cap in (0, 1 << 20, 8 << 30):
        kda.kda_set_workspace_pool_cap(cap)
    assert kda.kda_last_prefill_path() == before


def test_affine_state_rejects_partial_overlap():
    """S_out may be exactly S_in or B; shifted by one head it would race across CTAs."""
    lib = kda.load()
    s = kda.make_shape(1, 1, 4, 64, 64, 0, kda.KDA_DTYPE_F32)
    head = 64 * 64 * 4
    A = ctypes.c_void_p(1 << 30)
    S = ctypes.c_void_p(1 << 32)
    B = ctypes.c_void_p(1 << 34)
    shifted_S = ctypes.c_void_p((1 << 32) + head)
    shifted_B = ctypes.c_void_p((1 << 34) - head)
    call = lambda out: lib.kda_affine_state(A, S, B, out, ctypes.byref(s), None)
    assert call(shifted_S) == kda.KDA_ERR_INVALID_ARGUMENT
    assert call(shifted_B) == kda.KDA_ERR_INVALID_ARGUMENT
    assert call(A) == kda.KDA_ERR_INVALID_ARGUMENT
    assert lib.kda_affine_state(A, S, None, shifted_S, ctypes.byref(s), None) == \
        kda.KDA_ERR_INVALID_ARGUMENT


def test_prefill_ws_rejects_bad_workspace():
    lib = kda.load()
    s = kda.make_shape(2, 1000, 4, 128, 128, 64, kda.KDA_DTYPE_BF16)
    a = ctypes.c_void_p(1 << 20)
    b = ctypes.c_void_p(1 << 30)
    call = lambda ws, nbytes: lib.kda_prefill_ws(a, a, a, a, a, None, a, b, None, 0, None, ws,
                                                 nbytes, ctypes.byref(s), None)
    # misaligned workspace; workspace overlapping out
    assert call(ctypes.c_void_p((1 << 34) + 8), 1 << 20) == kda.KDA_ERR_INVALID_ARGUMENT
    assert call(ctypes.c_void_p((1 << 30) - 4096), 1 << 20) == kda.KDA_ERR_INVALID_ARGUMENT


def test_binding_fails_loudly_without_library(tmp_path):
    with pytest.raises(ImportError):
        kda.load(str(tmp_path / "missing.so"))


def test_decode_multi_rejects_bad_arguments():
    lib = kda.load()
    a = ctypes.c_void_p(1 << 20)
    st = ctypes.c_void_p(1 << 26)
    o = ctypes.c_void_p(1 << 28)
    good = kda.make_shape(4, 4 * 8, 2, 32, 32, 0, 1)
    for tokens in (0, 65):
        assert lib.kda_decode_multi(a, a, a, a, a, st, o, None, tokens, ctypes.byref(good),
                                    None) == kda.KDA_ERR_INVALID_ARGUMENT
    bad = kda.make_shape(4, 4 * 8 + 1, 2, 32, 32, 0, 1)       # total_tokens != N * T_new
    assert lib.kda_decode_multi(a, a, a, a, a, st, o, None, 8, ctypes.byref(bad),
                                None) == kda.KDA_ERR_INVALID_ARGUMENT
    mis = ctypes.c_void_p((1 << 20) + 2)                        # misaligned accept_len
    assert lib.kda_decode_multi(a, a, a, a, a, st, o, mis, 8, ctypes.byref(good),
                                None) == kda.KDA_ERR_INVALID_ARGUMENT


def test_prefill_at_requires_all_position_pointers():
    lib = kda.load()
    s = _shape()
    a = ctypes.c_void_p(1 << 20)
    b = ctypes.c_void_p(1 << 24)
    c = ctypes.c_void_p(1 << 28)
    # positions without pos_cu / pos_states
    assert lib.kda_prefill_at(a, a, a, a, a, None, a, b, None, 0, None, None, a, None,
                              ctypes.byref(s), None) == kda.KDA_ERR_INVALID_ARGUMENT
    assert lib.kda_prefill_at(a, a, a, a, a, None, a, b, None, 0, None, a, a, None,
                              ctypes.byref(s), None) == kda.KDA_ERR_INVALID_ARGUMENT
    # misaligned pos_states
    assert lib.kda_prefill_at(a, a, a, a, a, None, a, b, None, 0, None, a, a,
                              ctypes.c_void_p((1 << 28) + 4), ctypes.byref(s),
                              None) == kda.KDA_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("Dk,Dv", [(32, 32), (64, 64), (128, 128), (128, 32)])
def test_backward_workspace_covers_states_and_slice_parts(Dk, Dv):
    """A stored state per 4-token block of every sequence (ragged lengths round
    up), plus, for each 32-column value slice after the first, the slice's
    dq, dk, dg and dbeta parts."""
    lib = kda.load()
    lengths = [5, 0, 8, 1]
    T, N, H = sum(lengths), len(lengths), 3
    s = kda.make_shape(N, T, H, Dk, Dv, 0, kda.KDA_DTYPE_F32)
    need = lib.kda_backward_workspace_bytes(ctypes.byref(s))
    bound_blocks = (T + 3 * N) // 4            # >= sum of ceil(T_n / 4) = 2 + 0 + 2 + 1
    assert bound_blocks >= sum((L + 3) // 4 for L in lengths)
    extra = Dv // 32 - 1
    assert need == bound_blocks * H * Dk * Dv * 4 + extra * T * H * (3 * Dk + 1) * 4


def test_backward_workspace_and_validation():
    lib = kda.load()
    s = kda.make_shape(2, 1000, 4, 128, 64, 0, kda.KDA_DTYPE_BF16)
    need = lib.kda_backward_workspace_bytes(ctypes.byref(s))
    # a state every 4 tokens (bound), plus the dq, dk, dg, dbeta parts of the second
    # 32-column slice of D_v = 64
    assert need == ((1000 + 3 * 2) // 4) * 4 * 128 * 64 * 4 + 1000 * 4 * (3 * 128 + 1) * 4
    P = ctypes.c_void_p
    base = 1 << 30
    ptr = lambda i: P(base + i * (1 << 26))   # distinct, non-overlapping fake device addresses
    args = [ptr(i) for i in range(5)] + [None, ptr(5), ptr(6), None] + [ptr(7 + i) for i in range(5)] + [None]
    lib.kda_backward.argtypes = [P] * 16 + [ctypes.c_size_t, ctypes.POINTER(kda.KdaShape), P]
    ws = ptr(12)
    # workspace too small; null d_out; misaligned dq; dq overlapping q
    assert lib.kda_backward(*args, ws, need - 16, ctypes.byref(s), None) == kda.KDA_ERR_INVALID_ARGUMENT
    bad = list(args)
    bad[7] = None
    assert lib.kda_backward(*bad, ws, need, ctypes.byref(s), None) == kda.KDA_ERR_INVALID_ARGUMENT
    bad = list(args)
    bad[9] = P(base + 7 * (1 << 26) + 4)
    assert lib.kda_backward(*bad, ws, need, ctypes.byref(s), None) == kda.KDA_ERR_INVALID_ARGUMENT
    bad = list(args)
    bad[9] = ptr(0)
    assert lib.kda_backward(*bad, ws, need, ctypes.byref(s), None) == kda.KDA_ERR_INVALID_ARGUMENT
    # head size outside {32, 64, 128}
    s_bad = kda.make_shape(2, 1000, 4, 96, 64, 0, kda.KDA_DTYPE_BF16)
    assert lib.kda_backward(*args, ws, need, ctypes.byref(s_bad), None) == kda.KDA_ERR_UNSUPPORTED


def test_chunked_backward_workspace():
    """BF16, D_k = D_v = 128: the chunked tensor-core backward's workspace holds, per
    (64-token chunk, head) of an upper bound of the chunk count, the forward's
    74,240-byte packet, dS at the chunk's end as a BF16 tile (32 KiB), the -dU and
    dO tiles (16 KiB each), dT as a BF16 tile, dP placed as BF16 tile rows and dP^T in
    FP32 (40 KiB together); per full chunk the stored
    forward state as a BF16 operand tile (32 KiB); per (sequence, head) the initial
    state as such a tile; per (chunk, head) the forward's T and (I + M)^-1 as BF16
    tiles (16 KiB); the forward's output (BF16); two prefix tables; per (chunk,
    head) a 32-byte record of where it sits."""
    lib = kda.load()
    al = lambda x: (x + 255) // 256 * 256
    for lengths, H in (([1024] * 4, 32), ([5, 0, 130, 64], 3)):
        N, T = len(lengths), sum(lengths)
        s = kda.make_shape(N, T, H, 128, 128, 0, kda.KDA_DTYPE_BF16)
        P = H * ((T + 63 * N) // 64)
        assert P >= H * sum(-(-L // 64) for L in lengths)
        want = (al(P * 74240 + 256) + al((T // 64) * H * 32768) + al(N * H * 32768) + al(P * 16384)
                + al(P * 32768) + al(P * 16384)
                + al(P * 16384) + al(P * 40960) + al(T * H * 256) + 2 * al((N + 1) * 8) + al(P * 32) + 256)
        assert lib.kda_backward_workspace_bytes(ctypes.byref(s)) == want
    # FP32 inputs keep the SIMT kernel's workspace
    s = kda.make_shape(4, 4096, 32, 128, 128, 0, kda.KDA_DTYPE_F32)
    assert lib.kda_backward_workspace_bytes(ctypes.byref(s)) == (4096 + 12) // 4 * 32 * 128 * 128 * 4 + 3 * 4096 * 32 * 385 * 4
