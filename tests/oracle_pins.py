"""Checks that pin the FP64 oracle to facts other than itself.

Each function takes a loaded oracle library (so that a deliberately broken
build can be checked too) and returns the largest error it saw; the caller
compares it with the stated bound.  None of them re-types the oracle's own
loop: they use closed forms, exact rational arithmetic, explicit matrix
products, automatic differentiation, a hand-worked example and invariants of
the recurrence.
"""
from __future__ import annotations

import os
from fractions import Fraction

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def rand_problem(rng, lengths, H, Dk, Dv, unit_k=True, state_std=0.5, beta=None, g=None):
    T = int(sum(lengths))
    q = rng.standard_normal((T, H, Dk))
    k = rng.standard_normal((T, H, Dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, Dv))
    b = rng.uniform(0.0, 1.0, (T, H)) if beta is None else np.full((T, H), float(beta))
    gg = -rng.uniform(0.0, 5.0, (T, H, Dk)) if g is None else np.full((T, H, Dk), float(g))
    S0 = rng.standard_normal((len(lengths), H, Dk, Dv)) * state_std
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    return dict(q=q, k=k, v=v, g=gg, beta=b, init_state=S0, cu_seqlens=cu)


def _run(lib, p, chunk=0, ckpt_interval=0):
    return oracle.prefill(p["q"], p["k"], p["v"], p["g"], p["beta"], p["cu_seqlens"],
                          p["init_state"], ckpt_interval, chunk, nthreads=2, lib=lib)


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# --- I1: beta = 0 and g = 0 (alpha = 1) leave the state unchanged --------------------
def pin_identity_tokens(lib):
    rng = np.random.default_rng(11)
    p = rand_problem(rng, [7, 5], 2, 4, 3, beta=0.0, g=0.0)
    out, fin, _ = _run(lib, p)
    err = np.abs(fin - p["init_state"]).max()
    for n in range(2):
        a, b = p["cu_seqlens"][n], p["cu_seqlens"][n + 1]
        want = np.einsum("thc,hcj->thj", p["q"][a:b], p["init_state"][n])
        err = max(err, np.abs(out[a:b] - want).max())
    return float(err)


# --- I2: beta = 1 and |k| = 1 make S_t^T k_t return v_t exactly ----------------------
def pin_delta_retrieval(lib):
    rng = np.random.default_rng(12)
    p = rand_problem(rng, [9], 3, 5, 4, beta=1.0)
    p["q"] = p["k"].copy()          # o_t = S_t^T k_t
    out, _, _ = _run(lib, p)
    return float(np.abs(out - p["v"]).max())


# --- I3: beta = 0 is pure per-channel decay: S_t = Diag(exp(sum g)) S_0 ---------------
def pin_pure_decay(lib):
    rng = np.random.default_rng(13)
    p = rand_problem(rng, [6, 4], 2, 3, 5, beta=0.0)
    out, fin, _ = _run(lib, p)
    err = 0.0
    for n in range(2):
        a, b = p["cu_seqlens"][n], p["cu_seqlens"][n + 1]
        cum = np.cumsum(p["g"][a:b], axis=0)                      # [L, H, Dk]
        St = np.exp(cum)[..., None] * p["init_state"][n][None]    # [L, H, Dk, Dv]
        want = np.einsum("thc,thcj->thj", p["q"][a:b], St)
        err = max(err, np.abs(out[a:b] - want).max(), np.abs(fin[n] - St[-1]).max())
    return float(err)


# --- I3: one gate for all channels (gated DeltaNet) is DeltaNet on rescaled values ----
# With g_t,c = gamma_t for every channel, Diag(alpha_t) = e^{gamma_t} I commutes
# with (I - b k k^T).  Dividing by P_t = exp(gamma_1 + ... + gamma_t) gives
# S_t / P_t = (I - b k k^T)(S_{t-1} / P_{t-1}) + b k (v_t / P_t)^T: the g = 0
# recurrence (DeltaNet) on values v_t / P_t.  A decay applied after the delta
# step, or a gate taken from the wrong token, breaks the identity.
def pin_scalar_gate(lib):
    rng = np.random.default_rng(17)
    p = rand_problem(rng, [7, 5], 2, 4, 3)
    T, H = p["q"].shape[:2]
    gamma = -rng.uniform(0.0, 0.6, (T, H))
    p["g"] = np.repeat(gamma[:, :, None], 4, axis=2)
    out, fin, _ = _run(lib, p)
    P = np.empty((T, H))
    for n in range(2):
        a, b = p["cu_seqlens"][n], p["cu_seqlens"][n + 1]
        P[a:b] = np.exp(np.cumsum(gamma[a:b], axis=0))
    q = dict(p, g=np.zeros_like(p["g"]), v=p["v"] / P[:, :, None])
    out0, fin0, _ = _run(lib, q)
    err = np.abs(out - out0 * P[:, :, None]).max()
    for n in range(2):
        last = p["cu_seqlens"][n + 1] - 1
        err = max(err, np.abs(fin[n] - fin0[n] * P[last][:, None, None]).max())
    return float(err)


# --- I5: the explicit matrix product form (I - b k k^T) Diag(a) S + b k v^T -----------
def pin_matrix_form(lib):
    rng = np.random.default_rng(14)
    p = rand_problem(rng, [6, 3], 2, 4, 3, unit_k=False)
    out, fin, _ = _run(lib, p)
    err = 0.0
    for n in range(2):
        a, b = p["cu_seqlens"][n], p["cu_seqlens"][n + 1]
        for h in range(2):
            S = p["init_state"][n, h].copy()
            for t in range(a, b):
                kk = p["k"][t, h][:, None]
                A = (np.eye(4) - p["beta"][t, h] * kk @ kk.T) @ np.diag(np.exp(p["g"][t, h]))
                S = A @ S + p["beta"][t, h] * kk @ p["v"][t, h][None, :]
                err = max(err, np.abs(out[t, h] - S.T @ p["q"][t, h]).max())
            err = max(err, np.abs(fin[n, h] - S).max())
    return float(err)


# --- I5: the same, summed in closed form: S_T = Phi_T S_0 + sum_t Phi_{t+1..T} b k v^T -
def pin_closed_form_sum(lib):
    rng = np.random.default_rng(15)
    p = rand_problem(rng, [5], 1, 3, 2, unit_k=False)
    _, fin, _ = _run(lib, p)
    mats = []
    for t in range(5):
        kk = p["k"][t, 0][:, None]
        mats.append((np.eye(3) - p["beta"][t, 0] * kk @ kk.T) @ np.diag(np.exp(p["g"][t, 0])))

    def phi(lo):  # product A_{T-1} ... A_lo
        M = np.eye(3)
        for t in range(lo, 5):
            M = mats[t] @ M
        return M

    want = phi(0) @ p["init_state"][0, 0]
    for t in range(5):
        kk = p["k"][t, 0][:, None]
        want = want + phi(t + 1) @ (p["beta"][t, 0] * kk @ p["v"][t, 0][None, :])
    return float(np.abs(fin[0, 0] - want).max())


# --- I5: exact rational arithmetic on a tiny case ------------------------------------
def pin_exact_rational(lib):
    # alpha are dyadic rationals, so exp(log(alpha)) is alpha to within an ulp;
    # everything else is exact in Fraction arithmetic.
    alphas = [[Fraction(1, 2), Fraction(3, 4)], [Fraction(1, 4), Fraction(1, 1)],
              [Fraction(7, 8), Fraction(1, 2)]]
    ks = [[Fraction(3, 5), Fraction(4, 5)], [Fraction(1), Fraction(0)],
          [Fraction(-5, 13), Fraction(12, 13)]]
    vs = [[Fraction(1), Fraction(-2), Fraction(1, 2)], [Fraction(3), Fraction(0), Fraction(-1)],
          [Fraction(1, 4), Fraction(2), Fraction(5)]]
    qs = [[Fraction(1), Fraction(2)], [Fraction(-1), Fraction(1, 2)], [Fraction(0), Fraction(1)]]
    bs = [Fraction(1, 2), Fraction(3, 4), Fraction(1, 8)]
    S = [[Fraction(1, 3), Fraction(0), Fraction(-1)], [Fraction(2), Fraction(1, 5), Fraction(1)]]
    S0 = [row[:] for row in S]
    outs = []
    for t in range(3):
        a, k, v, q, b = alphas[t], ks[t], vs[t], qs[t], bs[t]
        A = [[a[c] * S[c][j] for j in range(3)] for c in range(2)]
        # (I - b k k^T) A + b k v^T, written as the matrix product it is
        S = [[sum(((1 if c == d else 0) - b * k[c] * k[d]) * A[d][j] for d in range(2))
              + b * k[c] * v[j] for j in range(3)] for c in range(2)]
        outs.append([sum(S[c][j] * q[c] for c in range(2)) for j in range(3)])
    f = lambda x: np.array(x, dtype=np.float64)
    p = dict(q=f(qs)[:, None, :], k=f(ks)[:, None, :], v=f(vs)[:, None, :],
             g=np.log(f(alphas))[:, None, :], beta=f(bs)[:, None],
             init_state=f(S0)[None, None], cu_seqlens=np.array([0, 3], dtype=np.int64))
    out, fin, _ = _run(lib, p)
    return float(max(np.abs(out[:, 0] - f(outs)).max(), np.abs(fin[0, 0] - f(S)).max()))


# --- derivation: one gradient step on the L2 retrieval loss (Background section) -----
def pin_gradient_step(lib):
    import torch
    rng = np.random.default_rng(16)
    p = rand_problem(rng, [1], 1, 4, 3, unit_k=False)
    _, fin, _ = _run(lib, p)
    A = torch.tensor(np.exp(p["g"][0, 0])[:, None] * p["init_state"][0, 0], requires_grad=True)
    k = torch.tensor(p["k"][0, 0])
    v = torch.tensor(p["v"][0, 0])
    loss = 0.5 * ((A.T @ k - v) ** 2).sum()
    (grad,) = torch.autograd.grad(loss, A)
    want = (A - p["beta"][0, 0] * grad).detach().numpy()
    return float(np.abs(fin[0, 0] - want).max())


# --- hand-worked golden example -----------------------------------------------------
def load_hand_example():
    rows = {}
    with open(os.path.join(GOLDEN, "kda_hand_example.txt")) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            rows.setdefault(key, []).append([float(x) for x in vals])
    return {k: np.array(v) for k, v in rows.items()}


def pin_hand_example(lib):
    ex = load_hand_example()
    T = ex["k"].shape[0]
    p = dict(q=ex["q"][:, None], k=ex["k"][:, None], v=ex["v"][:, None],
             g=np.log(ex["alpha"])[:, None], beta=ex["beta"].reshape(T, 1),
             init_state=np.zeros((1, 1, 2, 2)), cu_seqlens=np.array([0, T], dtype=np.int64))
    out, fin, _ = _run(lib, p)
    return float(max(np.abs(out[:, 0] - ex["o"]).max(),
                     np.abs(fin.reshape(-1) - ex["S_final"].reshape(-1)).max()))


# --- I4: chunked regrouping == token recurrence -------------------------------------
def pin_chunked(lib, chunk):
    rng = np.random.default_rng(17 + chunk)
    lengths = [chunk * 2 + 3, chunk - 1, 1, chunk]
    p = rand_problem(rng, lengths, 2, 6, 5)
    interval = chunk
    o1, f1, c1 = _run(lib, p, 0, interval)
    o2, f2, c2 = _run(lib, p, chunk, interval)
    return float(max(rel(o2, o1), rel(f2, f1), rel(c2, c1)))


# --- I6: o and S_T are jointly linear in (V, S_0) -----------------------------------
def pin_linearity(lib):
    rng = np.random.default_rng(18)
    p1 = rand_problem(rng, [11, 4], 2, 4, 3)
    p2 = dict(p1)
    p2["v"] = rng.standard_normal(p1["v"].shape)
    p2["init_state"] = rng.standard_normal(p1["init_state"].shape)
    a, b = 0.7, -1.3
    p3 = dict(p1)
    p3["v"] = a * p1["v"] + b * p2["v"]
    p3["init_state"] = a * p1["init_state"] + b * p2["init_state"]
    o1, f1, _ = _run(lib, p1)
    o2, f2, _ = _run(lib, p2)
    o3, f3, _ = _run(lib, p3)
    return float(max(rel(o3, a * o1 + b * o2), rel(f3, a * f1 + b * f2)))


# --- I7: value columns evolve independently -----------------------------------------
def pin_column_split(lib):
    rng = np.random.default_rng(19)
    p = rand_problem(rng, [9, 6], 2, 4, 6)
    o, f, _ = _run(lib, p)
    err = 0.0
    for sl in (slice(0, 2), slice(2, 6)):
        ps = dict(p)
        ps["v"] = np.ascontiguousarray(p["v"][..., sl])
        ps["init_state"] = np.ascontiguousarray(p["init_state"][..., sl])
        os_, fs, _ = _run(lib, ps)
        err = max(err, np.abs(os_ - o[..., sl]).max(), np.abs(fs - f[..., sl]).max())
    return float(err)


# --- I8: checkpoint j is the state after j*interval tokens; resuming reproduces ------
def pin_checkpoint_resume(lib):
    rng = np.random.default_rng(20)
    L, interval = 23, 5
    p = rand_problem(rng, [L, 12], 2, 3, 4)
    o, f, ck = _run(lib, p, 0, interval)
    err = 0.0
    if ck.shape[0] != L // interval + 12 // interval:
        return float("inf")
    for j in range(1, L // interval + 1):
        n = j * interval
        pj = {key: (val[:n] if key in ("q", "k", "v", "g", "beta") else val)
              for key, val in p.items()}
        pj["init_state"] = p["init_state"][:1]
        pj["cu_seqlens"] = np.array([0, n], dtype=np.int64)
        _, fj, _ = _run(lib, pj)
        err = max(err, np.abs(ck[j - 1] - fj[0]).max())
        # resume the rest from checkpoint j
        pr = {key: (val[n:L] if key in ("q", "k", "v", "g", "beta") else val)
              for key, val in p.items()}
        pr["init_state"] = ck[j - 1][None]
        pr["cu_seqlens"] = np.array([0, L - n], dtype=np.int64)
        orr, fr, _ = _run(lib, pr)
        err = max(err, np.abs(orr - o[n:L]).max(), np.abs(fr[0] - f[0]).max())
    return float(err)


# --- I9: a packed batch equals separate calls ----------------------------------------
def pin_varlen(lib):
    rng = np.random.default_rng(21)
    lengths = [3, 8, 1, 5]
    p = rand_problem(rng, lengths, 2, 3, 2)
    o, f, _ = _run(lib, p)
    err = 0.0
    cu = p["cu_seqlens"]
    for n in range(len(lengths)):
        a, b = cu[n], cu[n + 1]
        pn = {key: (val[a:b] if key in ("q", "k", "v", "g", "beta") else val)
              for key, val in p.items()}
        pn["init_state"] = p["init_state"][n:n + 1]
        pn["cu_seqlens"] = np.array([0, b - a], dtype=np.int64)
        on, fn, _ = _run(lib, pn)
        err = max(err, np.abs(on - o[a:b]).max(), np.abs(fn[0] - f[n]).max())
    return float(err)


# --- explicit positions: the state after j tokens is the final state of the first j ---
def pin_positions(lib):
    rng = np.random.default_rng(22)
    lengths = [19, 7, 12]
    p = rand_problem(rng, lengths, 2, 3, 4)
    positions = [[1, 5, 5, 13, 19, 30], [0, 7], []]
    o, f, ck, ps = oracle.prefill(p["q"], p["k"], p["v"], p["g"], p["beta"], p["cu_seqlens"],
                                  p["init_state"], 0, 0, 2, lib, positions)
    if ps.shape[0] != sum(len(x) for x in positions):
        return float("inf")
    err, j = 0.0, 0
    cu = p["cu_seqlens"]
    for n, lst in enumerate(positions):
        for pos in lst:
            m = max(0, min(pos, lengths[n]))
            a = cu[n]
            pn = {key: (val[a:a + m] if key in ("q", "k", "v", "g", "beta") else val)
                  for key, val in p.items()}
            pn["init_state"] = p["init_state"][n:n + 1]
            pn["cu_seqlens"] = np.array([0, m], dtype=np.int64)
            _, fn, _ = _run(lib, pn)
            err = max(err, np.abs(ps[j] - fn[0]).max())
            j += 1
    return float(err)


# name -> (function, bound)
PINS = {
    "identity_tokens": (pin_identity_tokens, 1e-15),
    "delta_retrieval": (pin_delta_retrieval, 1e-12),
    "pure_decay": (pin_pure_decay, 1e-12),
    "scalar_gate": (pin_scalar_gate, 1e-12),
    "matrix_form": (pin_matrix_form, 1e-12),
    "closed_form_sum": (pin_closed_form_sum, 1e-12),
    "exact_rational": (pin_exact_rational, 1e-14),
    "gradient_step": (pin_gradient_step, 1e-12),
    "hand_example": (pin_hand_example, 1e-14),
    "chunked_16": (lambda lib: pin_chunked(lib, 16), 1e-10),
    "chunked_64": (lambda lib: pin_chunked(lib, 64), 1e-10),
    "chunked_5": (lambda lib: pin_chunked(lib, 5), 1e-10),
    "linearity": (pin_linearity, 1e-10),
    "column_split": (pin_column_split, 1e-14),
    "checkpoint_resume": (pin_checkpoint_resume, 1e-12),
    "varlen": (pin_varlen, 1e-14),
    "positions": (pin_positions, 1e-14),
}
