"""The oracle's backward pass pinned to central finite differences of its own
forward recurrence (FP64): for a loss L = sum(o * Ro) + sum(S_final * Rs) with
random weights, every gradient the backward returns must match (L(x + h) -
L(x - h)) / 2h for every element of every input.  A dropped term, a wrong sign
or a transposed operand anywhere in the reverse recurrence fails here."""
import numpy as np
import pytest

import oracle

H_STEP = 1e-6


def _case(lengths, H, Dk, Dv, seed, with_init=True, with_dfin=True):
    rng = np.random.default_rng(seed)
    T = int(sum(lengths))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    N = len(lengths)
    x = {
        "q": rng.normal(size=(T, H, Dk)),
        "k": rng.normal(size=(T, H, Dk)) * 0.7,
        "v": rng.normal(size=(T, H, Dv)),
        "g": -rng.uniform(0.05, 2.0, size=(T, H, Dk)),
        "beta": rng.uniform(0.1, 0.9, size=(T, H)),
        "init": rng.normal(size=(N, H, Dk, Dv)) * 0.3 if with_init else None,
    }
    Ro = rng.normal(size=(T, H, Dv))
    Rs = rng.normal(size=(N, H, Dk, Dv)) if with_dfin else None
    return x, cu, Ro, Rs


def _loss(x, cu, Ro, Rs):
    out, fin, _ = oracle.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], cu, x["init"], 0, 0, 1)
    val = float((out * Ro).sum())
    if Rs is not None:
        val += float((fin * Rs).sum())
    return val


@pytest.mark.parametrize("with_init,with_dfin", [(True, True), (False, False), (True, False)])
def test_backward_matches_finite_differences(with_init, with_dfin):
    x, cu, Ro, Rs = _case([4, 3, 0], 2, 3, 2, seed=7, with_init=with_init, with_dfin=with_dfin)
    grads = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], cu, Ro,
                            init_state=x["init"], d_final=Rs, nthreads=1)
    names = ("q", "k", "v", "g", "beta", "init")
    for name, grad in zip(names, grads):
        arr = x[name]
        if arr is None:
            continue
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            orig = arr[idx]
            arr[idx] = orig + H_STEP
            lp = _loss(x, cu, Ro, Rs)
            arr[idx] = orig - H_STEP
            lm = _loss(x, cu, Ro, Rs)
            arr[idx] = orig
            fd[idx] = (lp - lm) / (2 * H_STEP)
        np.testing.assert_allclose(grad, fd, rtol=1e-6, atol=1e-7, err_msg=name)


def test_backward_of_an_empty_sequence_passes_the_final_gradient_through():
    """With no tokens the state is the identity map: d_init = d_final."""
    x, cu, Ro, Rs = _case([0, 2], 1, 2, 2, seed=3)
    *_, d_init = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], cu, Ro,
                                 init_state=x["init"], d_final=Rs, nthreads=1)
    np.testing.assert_array_equal(d_init[0], Rs[0])


BACKWARD_MUTATIONS = {
    "drop_P_du_term": ("dkt[c] = a - bt * b;", "dkt[c] = a;"),
    "dq_from_previous_state": ("a += Sn[c * Dv + j] * dot[j];", "a += Sp[c * Dv + j] * dot[j];"),
    "carry_without_decay": ("dS[c * Dv + j] = alpha[c] * (dS[c * Dv + j] - bt * kt[c] * du[j]);",
                            "dS[c * Dv + j] = (dS[c * Dv + j] - bt * kt[c] * du[j]);"),
    "dbeta_sign": ("db += du[j] * (vt[j] - y[j]);", "db += du[j] * (vt[j] + y[j]);"),
    "dg_without_alpha": ("dgt[c] = alpha[c] * da;", "dgt[c] = da;"),
}


@pytest.mark.parametrize("name", sorted(BACKWARD_MUTATIONS))
def test_finite_differences_catch_backward_mutation(name, tmp_path):
    import os
    import subprocess
    src = open(os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")).read()
    old, new = BACKWARD_MUTATIONS[name]
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    path = tmp_path / "mut.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", str(so),
                           str(path), "-lm"])
    lib = oracle.load(str(so))
    x, cu, Ro, Rs = _case([4, 3], 2, 3, 2, seed=11)
    grads = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], cu, Ro,
                            init_state=x["init"], d_final=Rs, nthreads=1, lib=lib)
    worst = 0.0
    for name_i, grad in zip(("q", "k", "v", "g", "beta", "init"), grads):
        arr = x[name_i]
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            orig = arr[idx]
            arr[idx] = orig + H_STEP
            lp = _loss(x, cu, Ro, Rs)
            arr[idx] = orig - H_STEP
            lm = _loss(x, cu, Ro, Rs)
            arr[idx] = orig
            fd[idx] = (lp - lm) / (2 * H_STEP)
        worst = max(worst, float(np.max(np.abs(grad - fd)) / (np.max(np.abs(fd)) + 1e-30)))
    assert worst > 1e-4, f"finite differences did not catch {name}"
