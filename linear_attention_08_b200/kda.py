"""Thin ctypes binding of libkda.so (the C ABI declared in include/kda.h).

Argument marshalling only: every step of the operator runs in the CUDA
kernels behind the C ABI.  PyTorch provides device memory and streams.  There
is no fallback: if the library is missing or a call fails, this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkda.so")

KDA_OK, KDA_ERR_INVALID_ARGUMENT, KDA_ERR_UNSUPPORTED, KDA_ERR_CUDA, KDA_ERR_TIMEOUT = range(5)
KDA_DTYPE_F32, KDA_DTYPE_BF16 = 0, 1

EXPORTED = ("kda_prefill", "kda_prefill_ws", "kda_prefill_at", "kda_decode", "kda_decode_multi",
            "kda_ckpt_count", "kda_prefill_workspace_bytes", "kda_prefill_workspace_min_bytes",
            "kda_release_workspace_pool", "kda_prefill_path", "kda_selftest_bounded_wait",
            "kda_last_cuda_error", "kda_status_string", "kda_version", "kda_backward",
            "kda_backward_workspace_bytes", "kda_affine_rows", "kda_affine_state",
            "kda_last_prefill_path", "kda_set_workspace_pool_cap", "kda_last_backward_path")

# Largest workspace the binding allocates for the two-pass prefill; longer
# inputs run in windows of chunks.
WORKSPACE_CAP = int(os.environ.get("KDA_WORKSPACE_CAP", 8 << 30))


class KdaShape(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("total_tokens", ctypes.c_int64),
                ("num_heads", ctypes.c_int32), ("head_dim_k", ctypes.c_int32),
                ("head_dim_v", ctypes.c_int32), ("chunk", ctypes.c_int32),
                ("qkv_dtype", ctypes.c_int32), ("dev_status", ctypes.c_void_p)]


class KdaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = _lib_or_none().kda_status_string(status).decode() if _lib_or_none() else str(status)
        if status == KDA_ERR_CUDA and _lib_or_none():
            msg += f" (cudaError {_lib_or_none().kda_last_cuda_error()})"
        super().__init__(f"{what}: {msg}")


_lib = None


def _lib_or_none():
    return _lib


def load(path: str | None = None):
    """Load libkda.so (cached); raises if it has not been built.  An explicit
    ``path`` loads that file without touching the cache."""
    global _lib
    if path is None and _lib is not None:
        return _lib
    explicit = path is not None
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m linear_attention_08_b200.build`")
    lib = ctypes.CDLL(path)
    P, I32, I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    SP = ctypes.POINTER(KdaShape)
    lib.kda_prefill.argtypes = [P, P, P, P, P, P, P, P, P, I64, P, SP, P]
    lib.kda_prefill.restype = ctypes.c_int
    lib.kda_prefill_ws.argtypes = [P, P, P, P, P, P, P, P, P, I64, P, P, ctypes.c_size_t, SP, P]
    lib.kda_prefill_ws.restype = ctypes.c_int
    lib.kda_prefill_at.argtypes = [P, P, P, P, P, P, P, P, P, I64, P, P, P, P, SP, P]
    lib.kda_prefill_at.restype = ctypes.c_int
    lib.kda_decode.argtypes = [P, P, P, P, P, P, P, SP, P]
    lib.kda_decode.restype = ctypes.c_int
    lib.kda_decode_multi.argtypes = [P, P, P, P, P, P, P, P, I32, SP, P]
    lib.kda_decode_multi.restype = ctypes.c_int
    lib.kda_ckpt_count.argtypes = [P, I32, I64]
    lib.kda_ckpt_count.restype = I64
    lib.kda_prefill_workspace_bytes.argtypes = [SP]
    lib.kda_prefill_workspace_bytes.restype = ctypes.c_size_t
    lib.kda_affine_rows.argtypes = [P, P, P, I64, I32, SP, P]
    lib.kda_affine_rows.restype = ctypes.c_int
    lib.kda_affine_state.argtypes = [P, P, P, P, SP, P]
    lib.kda_affine_state.restype = ctypes.c_int
    lib.kda_backward.argtypes = [P] * 16 + [ctypes.c_size_t, SP, P]
    lib.kda_backward.restype = ctypes.c_int
    lib.kda_backward_workspace_bytes.argtypes = [SP]
    lib.kda_backward_workspace_bytes.restype = ctypes.c_size_t
    lib.kda_prefill_workspace_min_bytes.argtypes = [SP]
    lib.kda_prefill_workspace_min_bytes.restype = ctypes.c_size_t
    lib.kda_release_workspace_pool.restype = ctypes.c_int
    lib.kda_prefill_path.argtypes = [SP]
    lib.kda_prefill_path.restype = ctypes.c_int
    lib.kda_last_prefill_path.restype = ctypes.c_int
    lib.kda_last_backward_path.restype = ctypes.c_int
    lib.kda_set_workspace_pool_cap.argtypes = [ctypes.c_size_t]
    lib.kda_set_workspace_pool_cap.restype = ctypes.c_int
    lib.kda_selftest_bounded_wait.argtypes = [P, I64, P]
    lib.kda_selftest_bounded_wait.restype = ctypes.c_int
    lib.kda_last_cuda_error.restype = ctypes.c_int
    lib.kda_status_string.argtypes = [ctypes.c_int]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_version.restype = ctypes.c_int
    if not explicit:
        _lib = lib
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_DTYPE_BF16
    if t.dtype == torch.float32:
        return KDA_DTYPE_F32
    raise TypeError(f"q/k/v must be float32 or bfloat16, got {t.dtype}")


def make_shape(num_seqs, total_tokens, H, Dk, Dv, chunk, dtype_code, dev_status=None) -> KdaShape:
    return KdaShape(int(num_seqs), int(total_tokens), int(H), int(Dk), int(Dv), int(chunk),
                    int(dtype_code), None if dev_status is None else dev_status.data_ptr())


def kda_ckpt_count(cu_seqlens_host, ckpt_interval: int) -> int:
    cu = (ctypes.c_int32 * len(cu_seqlens_host))(*[int(x) for x in cu_seqlens_host])
    n = load().kda_ckpt_count(cu, len(cu_seqlens_host) - 1, int(ckpt_interval))
    if n < 0:
        raise ValueError("bad cu_seqlens")
    return int(n)


def kda_prefill_path(shape: KdaShape) -> int:
    return int(load().kda_prefill_path(ctypes.byref(shape)))


def kda_last_prefill_path() -> int:
    """Kernel the last prefill call on this thread launched (2, 1, 0; -1 none)."""
    return int(load().kda_last_prefill_path())


def kda_last_backward_path() -> int:
    """Backward kernel the last kda_backward on this thread launched (1 chunked
    tensor-core, 0 SIMT; -1 none)."""
    return int(load().kda_last_backward_path())


def kda_set_workspace_pool_cap(nbytes: int) -> None:
    st = load().kda_set_workspace_pool_cap(int(nbytes))
    if st != KDA_OK:
        raise KdaError(st, "kda_set_workspace_pool_cap")


def kda_prefill_workspace_bytes(shape: KdaShape) -> int:
    return int(load().kda_prefill_workspace_bytes(ctypes.byref(shape)))


def kda_prefill_workspace_min_bytes(shape: KdaShape) -> int:
    return int(load().kda_prefill_workspace_min_bytes(ctypes.byref(shape)))


def workspace_for(shape: KdaShape, device, cap: int | None = None):
    """A torch-owned workspace for the two-pass prefill of ``shape`` (None when
    the shape runs on a single-pass kernel): the single-window size, capped
    at ``cap`` bytes (but never below the minimum)."""
    full = kda_prefill_workspace_bytes(shape)
    if full in (0, (1 << 64) - 1):
        return None
    cap = WORKSPACE_CAP if cap is None else int(cap)
    nbytes = max(min(full, cap), kda_prefill_workspace_min_bytes(shape))
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def kda_prefill(q, k, v, g, beta, cu_seqlens, *, init_state=None, chunk: int = 64,
                ckpt_interval: int = 0, cu_seqlens_host=None, out=None, final_state=None,
                ckpt_states=None, dev_status=None, stream=None, want_final: bool = True,
                positions=None, pos_states=None, workspace="auto"):
    """Chunked KDA prefill over a packed batch (see kda_prefill in include/kda.h).

    q, k, g: [T, H, Dk]; v: [T, H, Dv]; beta: [T, H]; cu_seqlens: int32 device
    [N+1]; init_state: [N, H, Dk, Dv] FP32 or None.  Outputs are allocated
    with torch when not given.  ``cu_seqlens_host`` (a list) avoids a device
    read when checkpoints are requested.  ``positions`` (one list of token
    counts per sequence) also stores the states after those counts
    (kda_prefill_at).  ``workspace``: "auto" allocates one with torch
    (``workspace_for``), a uint8 device tensor is used as given, None runs
    the single-pass kernels.  Returns (out, final_state, ckpt_states), plus
    pos_states when positions are given.
    """
    lib = load()
    T, H, Dk = q.shape
    Dv = v.shape[2]
    N = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty(T, H, Dv, dtype=q.dtype, device=q.device)
    if final_state is None and want_final:
        final_state = torch.empty(N, H, Dk, Dv, dtype=torch.float32, device=q.device)
    if ckpt_interval > 0 and ckpt_states is None:
        host = cu_seqlens_host if cu_seqlens_host is not None else cu_seqlens.tolist()
        n = kda_ckpt_count(host, ckpt_interval)
        ckpt_states = torch.empty(max(n, 1), H, Dk, Dv, dtype=torch.float32, device=q.device)[:n]
    shape = make_shape(N, T, H, Dk, Dv, chunk, _dtype_code(q), dev_status)
    ck_ptr = _ptr(ckpt_states) if ckpt_interval > 0 else None
    if ckpt_interval > 0 and ckpt_states.numel() == 0:
        ck_ptr = ctypes.c_void_p(ckpt_states.untyped_storage().data_ptr())
    if positions is None:
        if isinstance(workspace, str):
            assert workspace == "auto"
            # the two-pass kernels take intervals that are multiples of 64 only
            workspace = workspace_for(shape, q.device) if ckpt_interval % 64 == 0 else None
        nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        st = lib.kda_prefill_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(init_state),
                                _ptr(cu_seqlens), _ptr(out), _ptr(final_state),
                                int(ckpt_interval), ck_ptr, _ptr(workspace), nbytes,
                                ctypes.byref(shape), _stream(stream))
        if st != KDA_OK:
            raise KdaError(st, "kda_prefill_ws")
        return out, final_state, ckpt_states
    counts = [0]
    for lst in positions:
        counts.append(counts[-1] + len(lst))
    assert len(counts) == N + 1, "one list of positions per sequence"
    pos_cu = torch.tensor(counts, dtype=torch.int32, device=q.device)
    flat = [int(x) for lst in positions for x in lst]
    pos = torch.tensor(flat or [0], dtype=torch.int32, device=q.device)
    if pos_states is None:
        pos_states = torch.empty(max(counts[-1], 1), H, Dk, Dv, dtype=torch.float32,
                                 device=q.device)[:counts[-1]]
    ps_ptr = ctypes.c_void_p(pos_states.untyped_storage().data_ptr()) if counts[-1] == 0 \
        else _ptr(pos_states)
    st = lib.kda_prefill_at(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(init_state),
                            _ptr(cu_seqlens), _ptr(out), _ptr(final_state), int(ckpt_interval),
                            ck_ptr, _ptr(pos_cu), _ptr(pos), ps_ptr, ctypes.byref(shape),
                            _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_prefill_at")
    return out, final_state, ckpt_states, pos_states


def kda_backward(q, k, v, g, beta, cu_seqlens, d_out, *, init_state=None, d_final=None,
                 want_d_init: bool = True, workspace=None, stream=None):
    """Gradients of the recurrence (see kda_backward in include/kda.h) for the
    upstream gradient d_out [T, H, Dv] (FP32) and d_final [N, H, Dk, Dv] (FP32
    or None).  Returns (dq, dk, dv, dg, dbeta, d_init) as FP32 tensors; d_init
    is None unless want_d_init."""
    lib = load()
    T, H, Dk = q.shape
    Dv = v.shape[2]
    N = cu_seqlens.numel() - 1
    dev = q.device
    dq = torch.empty(T, H, Dk, dtype=torch.float32, device=dev)
    dk = torch.empty_like(dq)
    dg = torch.empty_like(dq)
    dv = torch.empty(T, H, Dv, dtype=torch.float32, device=dev)
    dbeta = torch.empty(T, H, dtype=torch.float32, device=dev)
    d_init = torch.empty(N, H, Dk, Dv, dtype=torch.float32, device=dev) if want_d_init else None
    shape = make_shape(N, T, H, Dk, Dv, 0, _dtype_code(q))
    if workspace is None:
        nbytes = int(lib.kda_backward_workspace_bytes(ctypes.byref(shape)))
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    st = lib.kda_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(init_state),
                          _ptr(cu_seqlens), _ptr(d_out), _ptr(d_final), _ptr(dq), _ptr(dk),
                          _ptr(dv), _ptr(dg), _ptr(dbeta), _ptr(d_init), _ptr(workspace),
                          workspace.numel(), ctypes.byref(shape), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_backward")
    return dq, dk, dv, dg, dbeta, d_init


def kda_affine_rows(x, M, y, *, accumulate: bool = False, stream=None):
    """y[r, h, :] = x[r, h, :] @ M[h] (+ y when accumulate): x [rows, H, Dk],
    y [rows, H, Dv] (same dtype, BF16 or FP32), M [H, Dk, Dv] FP32."""
    rows, H, Dk = x.shape
    Dv = y.shape[2]
    shape = make_shape(1, rows, H, Dk, Dv, 0, _dtype_code(x))
    st = load().kda_affine_rows(_ptr(x), _ptr(M), _ptr(y), int(rows), int(bool(accumulate)),
                                ctypes.byref(shape), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_affine_rows")
    return y


def kda_affine_state(A, S_in, B=None, S_out=None, *, stream=None):
    """S_out[h] = A[h] @ S_in[h] + B[h] (FP32): A [H, Dk, Dk], S_in, B [H, Dk, Dv]."""
    H, Dk, Dv = S_in.shape
    if S_out is None:
        S_out = torch.empty_like(S_in)
    shape = make_shape(1, 1, H, Dk, Dv, 0, KDA_DTYPE_F32)
    st = load().kda_affine_state(_ptr(A), _ptr(S_in), _ptr(B), _ptr(S_out), ctypes.byref(shape),
                                 _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_affine_state")
    return S_out


def kda_decode(q, k, v, g, beta, state, *, out=None, dev_status=None, stream=None):
    """One decode step: q, k, g [N, H, Dk]; v [N, H, Dv]; beta [N, H]; state
    [N, H, Dk, Dv] FP32 updated in place.  Returns out [N, H, Dv]."""
    lib = load()
    N, H, Dk = q.shape
    Dv = v.shape[2]
    if out is None:
        out = torch.empty(N, H, Dv, dtype=q.dtype, device=q.device)
    shape = make_shape(N, N, H, Dk, Dv, 0, _dtype_code(q), dev_status)
    st = lib.kda_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state), _ptr(out),
                        ctypes.byref(shape), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_decode")
    return out


def kda_decode_multi(q, k, v, g, beta, state, *, accept_len=None, out=None, dev_status=None,
                     stream=None):
    """Multi-token decode: q, k, g [N, T_new, H, Dk]; v [N, T_new, H, Dv]; beta
    [N, T_new, H]; state [N, H, Dk, Dv] FP32, replaced by the state after the
    first accept_len[n] tokens (int32 device tensor, or None for all).
    Returns out [N, T_new, H, Dv]."""
    lib = load()
    N, T_new, H, Dk = q.shape
    Dv = v.shape[3]
    if out is None:
        out = torch.empty(N, T_new, H, Dv, dtype=q.dtype, device=q.device)
    shape = make_shape(N, N * T_new, H, Dk, Dv, 0, _dtype_code(q), dev_status)
    st = lib.kda_decode_multi(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state),
                              _ptr(out), _ptr(accept_len), int(T_new), ctypes.byref(shape),
                              _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_decode_multi")
    return out


def kda_selftest_bounded_wait(dev_status, max_polls: int, stream=None) -> None:
    st = load().kda_selftest_bounded_wait(_ptr(dev_status), int(max_polls), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_selftest_bounded_wait")
