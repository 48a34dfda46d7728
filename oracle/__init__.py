"""FP64 CPU oracle of Kimi Delta Attention -- test infrastructure only.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never does, and shares no code with it.

The arithmetic lives in ``kda_oracle.c`` (plain C, double precision); this
module builds it with gcc on first use and marshals numpy arrays to it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkda_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def load(path: str | None = None):
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _bind(lib):
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    common = [I64, P, I64, I64, I64, P, P, P, P, P, P, I64, P, P, P, ctypes.c_int]
    lib.kda_oracle_recurrent.argtypes = common
    lib.kda_oracle_recurrent.restype = ctypes.c_int
    lib.kda_oracle_chunked.argtypes = common + [I64]
    lib.kda_oracle_chunked.restype = ctypes.c_int
    lib.kda_oracle_recurrent_pos.argtypes = common + [P, P, P]
    lib.kda_oracle_recurrent_pos.restype = ctypes.c_int
    lib.kda_oracle_max_threads.restype = ctypes.c_int
    lib.kda_oracle_backward.argtypes = [I64, P, I64, I64, I64, P, P, P, P, P, P, P, P, P, P, P, P,
                                        P, P, ctypes.c_int]
    lib.kda_oracle_backward.restype = ctypes.c_int
    return lib


def max_threads() -> int:
    return int(load().kda_oracle_max_threads())


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: exact upcast (bf16/f32 -> f64)
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def ckpt_count(lengths, interval: int) -> int:
    if interval <= 0:
        return 0
    return int(sum(int(n) // interval for n in lengths))


def prefill(q, k, v, g, beta, cu_seqlens, init_state=None, ckpt_interval: int = 0,
            chunk: int = 0, nthreads: int = 0, lib=None, positions=None):
    """Run the oracle over a packed batch.

    q, k, g: [T_tot, H, Dk]; v: [T_tot, H, Dv]; beta: [T_tot, H];
    cu_seqlens: N+1 offsets; init_state: [N, H, Dk, Dv] or None (zeros).
    ``chunk`` = 0 runs the token-by-token recurrence, > 0 the chunked form.
    Returns (out [T_tot, H, Dv], final_state [N, H, Dk, Dv],
    checkpoints [n_ckpt, H, Dk, Dv]) as float64 numpy arrays.  With
    ``positions`` (one list of token counts per sequence) a fourth array
    [n_pos, H, Dk, Dv] holds the states after those counts.
    """
    lib = lib or load()
    q, k, v, g, beta = (_f64(a) for a in (q, k, v, g, beta))
    init = _f64(init_state)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    T, H, Dk = q.shape
    Dv = v.shape[2]
    N = len(cu) - 1
    assert k.shape == (T, H, Dk) and g.shape == (T, H, Dk) and v.shape == (T, H, Dv)
    assert beta.shape == (T, H) and int(cu[-1]) == T
    if init is not None:
        assert init.shape == (N, H, Dk, Dv)
    out = np.zeros((T, H, Dv))
    fin = np.zeros((N, H, Dk, Dv))
    nck = ckpt_count(np.diff(cu), ckpt_interval)
    ck = np.zeros((max(nck, 1), H, Dk, Dv))
    args = [N, _ptr(cu), H, Dk, Dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(init),
            int(ckpt_interval), _ptr(out), _ptr(fin), _ptr(ck), int(nthreads)]
    if positions is not None:
        if chunk != 0:
            raise ValueError("explicit positions are supported by the recurrent form only")
        pos_cu = np.zeros(N + 1, dtype=np.int64)
        for i, lst in enumerate(positions):
            pos_cu[i + 1] = pos_cu[i] + len(lst)
        pos = np.ascontiguousarray(np.concatenate([np.asarray(l, dtype=np.int64) for l in positions])
                                   if pos_cu[-1] else np.zeros(1, dtype=np.int64))
        ps = np.zeros((max(int(pos_cu[-1]), 1), H, Dk, Dv))
        rc = lib.kda_oracle_recurrent_pos(*args, _ptr(pos_cu), _ptr(pos), _ptr(ps))
        if rc != 0:
            raise ValueError(f"oracle rejected its arguments (status {rc})")
        return out, fin, ck[:nck], ps[:int(pos_cu[-1])]
    if chunk == 0:
        rc = lib.kda_oracle_recurrent(*args)
    else:
        rc = lib.kda_oracle_chunked(*args, int(chunk))
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (status {rc})")
    return out, fin, ck[:nck]


def decode(q, k, v, g, beta, init_state, nthreads: int = 0, lib=None):
    """Oracle of ``steps`` decode calls: inputs [steps, N, H, D], state [N, H, Dk, Dv].

    A run of decode steps on sequence n is the recurrence over that
    sequence's tokens in step order, so the steps are regrouped into one
    packed sequence per n and handed to ``prefill``.
    Returns (out [steps, N, H, Dv], final_state [N, H, Dk, Dv]).
    """
    q, k, v, g, beta = (_f64(a) for a in (q, k, v, g, beta))
    steps, N, H, Dk = q.shape
    Dv = v.shape[3]

    def seq_major(a):
        return np.ascontiguousarray(np.swapaxes(a, 0, 1).reshape(N * steps, *a.shape[2:]))

    cu = np.arange(N + 1, dtype=np.int64) * steps
    out, fin, _ = prefill(seq_major(q), seq_major(k), seq_major(v), seq_major(g),
                          seq_major(beta), cu, init_state, 0, 0, nthreads, lib)
    out = np.ascontiguousarray(np.swapaxes(out.reshape(N, steps, H, Dv), 0, 1))
    return out, fin


def backward(q, k, v, g, beta, cu_seqlens, d_out, init_state=None, d_final=None,
             nthreads: int = 0, lib=None):
    """Gradients of the recurrence (FP64) for an upstream gradient d_out
    [T_tot, H, Dv] on the outputs and d_final [N, H, Dk, Dv] on the final
    states (None = 0).  Returns (dq, dk, dv, dg, dbeta, d_init) as float64
    numpy arrays with the shapes of the inputs."""
    lib = lib or load()
    q, k, v, g, beta, d_out = (_f64(a) for a in (q, k, v, g, beta, d_out))
    init = _f64(init_state)
    dfin = _f64(d_final)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    T, H, Dk = q.shape
    Dv = v.shape[2]
    N = len(cu) - 1
    dq, dk, dg = (np.zeros((T, H, Dk)) for _ in range(3))
    dv = np.zeros((T, H, Dv))
    dbeta = np.zeros((T, H))
    dinit = np.zeros((N, H, Dk, Dv))
    rc = lib.kda_oracle_backward(N, _ptr(cu), H, Dk, Dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                 _ptr(beta), _ptr(init), _ptr(d_out), _ptr(dfin), _ptr(dq),
                                 _ptr(dk), _ptr(dv), _ptr(dg), _ptr(dbeta), _ptr(dinit),
                                 int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (status {rc})")
    return dq, dk, dv, dg, dbeta, dinit
