"""Context parallelism (linear_attention_08_b200/cp.py) on CPU.

The orchestration runs with its arithmetic replaced by the FP64 oracle and
plain FP64 matrix products (OracleOps below, test-side only), so the affine
decomposition itself is checked: segments composed through (A, B), the fold
order of the incoming states, the output correction and the checkpoints must
reproduce the oracle run over the whole sequence.  The two-rank test runs the
real collective path (torch.distributed all_gather) over gloo.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
from linear_attention_08_b200 import cp  # noqa: E402


class OracleOps:
    """FP64 CPU stand-ins for the CUDA operations (tests only)."""

    def prefill(self, q, k, v, g, beta, init_state, chunk, ckpt_interval):
        T = q.shape[0]
        out, fin, ck = oracle.prefill(q, k, v, g, beta, [0, T], init_state, ckpt_interval, 0, 1)
        return torch.from_numpy(out), torch.from_numpy(fin), torch.from_numpy(ck)

    def affine_rows(self, x, M, y):
        y += torch.einsum("rhc,hcd->rhd", x.double(), M.double())
        return y

    def affine_state(self, A, S, B):
        return torch.einsum("hci,hid->hcd", A.double(), S.double()) + B.double()

    def zeros(self, shape, like):
        return torch.zeros(shape, dtype=torch.float64)

    def eye(self, H, D, like):
        return torch.eye(D, dtype=torch.float64).expand(1, H, D, D).contiguous()


def _sequence(T, H, Dk, Dv, seed):
    rng = np.random.default_rng(seed)
    k = rng.normal(size=(T, H, Dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    x = dict(q=rng.normal(size=(T, H, Dk)), k=k, v=rng.normal(size=(T, H, Dv)),
             g=-np.minimum(np.log1p(np.exp(rng.normal(size=(T, H, Dk)))), 5.0),
             beta=1.0 / (1.0 + np.exp(-rng.normal(size=(T, H)))),
             init=rng.normal(size=(1, H, Dk, Dv)) * 0.1)
    return {n: torch.from_numpy(np.ascontiguousarray(a)) for n, a in x.items()}


def _whole(x, interval):
    T = x["q"].shape[0]
    return oracle.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], [0, T], x["init"], interval, 0, 1)


def test_segments_compose_to_the_whole_sequence():
    x = _sequence(300, 2, 8, 6, seed=1)
    bounds = [0, 128, 192, 300]          # segment lengths 128, 64, 108; checkpoints every 64
    ops = OracleOps()
    segs = []
    for a, b in zip(bounds[:-1], bounds[1:]):
        sl = {n: x[n][a:b] for n in ("q", "k", "v", "g", "beta")}
        segs.append(cp.segment_pass(sl["q"], sl["k"], sl["v"], sl["g"], sl["beta"], chunk=64,
                                    ckpt_interval=64, ops=ops))
    As = [s["A"] for s in segs]
    Bs = [s["B"] for s in segs]
    outs, cks = [], []
    for r, seg in enumerate(segs):
        S_in = cp.incoming_state(As, Bs, r, x["init"][0], ops=ops)
        out, fin, ck = cp.finish_segment(seg, S_in, ops=ops)
        outs.append(out)
        cks.append(ck)
    ro, rf, rc = _whole(x, 64)
    np.testing.assert_allclose(torch.cat(outs).numpy(), ro, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(fin.numpy(), rf[0], rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(torch.cat(cks).numpy(), rc, rtol=1e-9, atol=1e-9)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, bounds, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    x = _sequence(bounds[-1], 2, 8, 6, seed=2)
    a, b = bounds[rank], bounds[rank + 1]
    out, fin, ck = cp.prefill_cp(x["q"][a:b], x["k"][a:b], x["v"][a:b], x["g"][a:b],
                                 x["beta"][a:b], init_state=x["init"], chunk=64,
                                 ckpt_interval=64, ops=OracleOps())
    q.put((rank, out.numpy(), fin.numpy(), ck.numpy()))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("bounds", [[0, 192, 250], [0, 64, 192, 250]],
                         ids=["two_ranks", "three_ranks"])
def test_prefill_cp_gloo(bounds):
    """Consecutive segments on 2 or 3 gloo ranks; the last segment is ragged
    and the three-rank case folds two incoming transitions."""
    world = len(bounds) - 1
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, bounds, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict((r, (o, f, c)) for r, o, f, c in (q.get(timeout=120) for _ in range(world)))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    x = _sequence(bounds[-1], 2, 8, 6, seed=2)
    ro, rf, rc = _whole(x, 64)
    out = np.concatenate([res[r][0] for r in range(world)])
    np.testing.assert_allclose(out, ro, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(res[world - 1][1], rf[0], rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(np.concatenate([res[r][2] for r in range(world)]), rc,
                               rtol=1e-9, atol=1e-9)



def _worker_bad_interval(rank, world, port, q):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import torch.distributed as dist
    # A long timeout: the refusal must not need one to end.
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    x = _sequence(100, 1, 4, 4, seed=3)
    a, b = (0, 50) if rank == 0 else (50, 100)
    import time
    t0 = time.monotonic()
    try:
        cp.prefill_cp(x["q"][a:b], x["k"][a:b], x["v"][a:b], x["g"][a:b], x["beta"][a:b],
                      chunk=16, ckpt_interval=16, ops=OracleOps())
        q.put((rank, "ok", time.monotonic() - t0))
    except ValueError:
        q.put((rank, "ValueError", time.monotonic() - t0))
    except Exception as e:
        q.put((rank, f"other: {e!r}", time.monotonic() - t0))
    dist.destroy_process_group()


def test_prefill_cp_rejects_unaligned_segment():
    """Checkpoint positions stay global only if every segment but the last is a
    multiple of ckpt_interval.  Rank 0's 50 tokens are not a multiple of 16: both
    ranks learn it from the gathered lengths and both raise ValueError at once,
    long before the process group's timeout, with no collective left pending."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_bad_interval, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {r: (what, dt) for r, what, dt in (q.get(timeout=120) for _ in range(2))}
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert res[0][0] == "ValueError" and res[1][0] == "ValueError", res
    assert max(res[0][1], res[1][1]) < 30.0, res
