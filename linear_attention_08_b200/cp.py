"""Context (sequence) parallelism: one long sequence split over ranks.

The pages name KDA context parallelism ("MoonshotAI/Kimi-K3 딥다이브", section
4-1) without detail.  This is the plainest split the recurrence allows.  The
recurrence is affine in the state it starts from: over a segment,
S_out = A S_in + B, where A is the state reached with v = 0 from the identity
and B the state reached from zero; token by token, the outputs from S_in are
o_t = o_t(B) + S_in^T (A_t^T q_t), and A_t^T q_t is the output of the v = 0,
identity-start run.  So every rank:

0. all-gathers the segment lengths (a refusal of misaligned segments is
   then taken by every rank alike);
1. runs its segment twice, from zero (B and the outputs o(B)) and with v = 0
   from the identity (A and the vectors A_t^T q_t): two ordinary prefill calls;
2. all-gathers (A, B) of every segment (one collective of
   H * D_k * (D_k + D_v) * 4 bytes per rank);
3. composes the state entering its segment, S_in = A_{r-1}(... (A_0 S_0 + B_0)
   ...) + B_{r-1};
4. forms its outputs, checkpoints and final state by two affine maps.

No segment runs a third time.  Checkpoints land at multiples of
``ckpt_interval`` from the sequence start, so every segment but the last must
be a multiple of it.  All arithmetic runs in the library's CUDA kernels
(``CudaOps``); the collective is ``torch.distributed.all_gather``.
"""
from __future__ import annotations

import torch

from . import kda


class CudaOps:
    """The operations a segment needs, on the library's CUDA kernels."""

    def prefill(self, q, k, v, g, beta, init_state, chunk, ckpt_interval):
        T = q.shape[0]
        cu = torch.tensor([0, T], dtype=torch.int32, device=q.device)
        return kda.kda_prefill(q, k, v, g, beta, cu, init_state=init_state, chunk=chunk,
                               ckpt_interval=ckpt_interval, cu_seqlens_host=[0, T])

    def affine_rows(self, x, M, y):
        """y += x M (per head)."""
        return kda.kda_affine_rows(x, M, y, accumulate=True)

    def affine_state(self, A, S, B):
        """A S + B (per head)."""
        return kda.kda_affine_state(A, S, B)

    def zeros(self, shape, like):
        return torch.zeros(shape, dtype=like.dtype, device=like.device)

    def eye(self, H, D, like):
        return torch.eye(D, dtype=torch.float32, device=like.device).expand(1, H, D, D).contiguous()


def segment_pass(q, k, v, g, beta, *, chunk=64, ckpt_interval=0, ops=None):
    """Step 1 for one segment: {A, B, oB, aq, ckA, ckB}.  A [H, Dk, Dk] and B
    [H, Dk, Dv] are the segment's transition, oB the outputs from zero, aq the
    vectors A_t^T q_t [T, H, Dk], ckA / ckB the two runs' checkpoints."""
    ops = ops or CudaOps()
    T, H, Dk = q.shape
    oB, B, ckB = ops.prefill(q, k, v, g, beta, None, chunk, ckpt_interval)
    aq, A, ckA = ops.prefill(q, k, ops.zeros((T, H, Dk), q), g, beta, ops.eye(H, Dk, q), chunk,
                             ckpt_interval)
    return dict(A=A[0], B=B[0], oB=oB, aq=aq, ckA=ckA, ckB=ckB)


def incoming_state(As, Bs, r, S0, ops=None):
    """Step 3: the state entering segment r from the state S0 [H, Dk, Dv] before
    segment 0 and the transitions (As[j], Bs[j]) of segments j < r."""
    ops = ops or CudaOps()
    S = S0
    for j in range(r):
        S = ops.affine_state(As[j], S, Bs[j])
    return S


def finish_segment(seg, S_in, ops=None):
    """Step 4: outputs, checkpoints and final state of a segment entered with S_in."""
    ops = ops or CudaOps()
    out = seg["oB"].clone()
    ops.affine_rows(seg["aq"], S_in, out)
    fin = ops.affine_state(seg["A"], S_in, seg["B"])
    if seg["ckA"] is None:   # no checkpoints requested
        return out, fin, None
    ck = [ops.affine_state(seg["ckA"][j], S_in, seg["ckB"][j]) for j in range(seg["ckA"].shape[0])]
    ck = torch.stack(ck) if ck else seg["ckB"]
    return out, fin, ck


def prefill_cp(q, k, v, g, beta, *, init_state=None, chunk=64, ckpt_interval=0, group=None,
               ops=None):
    """This rank's segment of one long sequence; ranks hold consecutive segments
    in rank order.  q, k, g [T_r, H, Dk], v [T_r, H, Dv], beta [T_r, H];
    init_state [1, H, Dk, Dv] (the state before the whole sequence) or None.
    Returns (out [T_r, H, Dv], final_state [H, Dk, Dv] after this segment,
    checkpoints [n, H, Dk, Dv] inside this segment)."""
    import torch.distributed as dist
    ops = ops or CudaOps()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    T, H, Dk = q.shape
    Dv = v.shape[2]
    # Every rank learns every segment's length first, so that a refusal is
    # collective: all ranks raise together and none is left in a collective.
    mine = torch.tensor([T], dtype=torch.int64, device=q.device)
    lens = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(lens, mine, group=group)
    if ckpt_interval > 0:
        bad = [r for r in range(world - 1) if int(lens[r]) % ckpt_interval != 0]
        if bad:
            raise ValueError(f"segments of ranks {bad} are not multiples of ckpt_interval="
                             f"{ckpt_interval}; every segment but the last must be")
    seg = segment_pass(q, k, v, g, beta, chunk=chunk, ckpt_interval=ckpt_interval, ops=ops)
    ab = torch.cat([seg["A"].reshape(-1), seg["B"].reshape(-1)])
    parts = [torch.empty_like(ab) for _ in range(world)]
    dist.all_gather(parts, ab, group=group)
    n_a = H * Dk * Dk
    As = [p[:n_a].view(H, Dk, Dk) for p in parts]
    Bs = [p[n_a:].view(H, Dk, Dv) for p in parts]
    S0 = init_state[0] if init_state is not None else torch.zeros_like(seg["B"])
    S_in = incoming_state(As, Bs, rank, S0, ops=ops)
    return finish_segment(seg, S_in, ops=ops)
