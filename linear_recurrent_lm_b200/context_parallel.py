"""Context parallelism: the tokens of every row split into consecutive segments, one per rank (one
process per GPU), with one exchange step each way.

Over a segment the WKV-7 recurrence is affine in the state entering it: S_end = S_in P + U, with P
the product of the segment's transitions diag(w_t) + a_t b_t^T -- the forward from s0 = I with v = 0
-- and U the forward's end state from s0 = 0 (a reset inside the segment makes P zero from there on,
as it should).  The state gradient goes back through the same P: dS_in = dS_end P^T + D, with D the
backward's ds0 from dsT = 0.  So:

forward  (rank p of R)
  1. p = 0 runs its real forward from the sequence's s0; its end state is U_0.  p >= 1 computes P_p
     and U_p (two forwards without checkpoints).
  2. all-gather of (P_q, U_q): the one exchange (NCCL over NVLink; 2 x B*H*N*N*4 bytes per rank).
  3. p >= 1 composes its entering state S_p = (...(U_0 P_1 + U_1) P_2 + ...) P_{p-1} + U_{p-1}
     (``wkv7_state_compose``) and runs its real forward from it (y, the checkpoints, its end state).
backward
  1. the last rank runs its real backward from the sequence's dsT; its ds0 is dS entering its
     segment.  Every other rank runs its backward with dsT = 0 and keeps only ds0 = D_p.
  2. all-gather of those ds0.
  3. p < R-1 composes dS leaving its segment, dS_p = (...(D_{R-1} P_{R-2}^T + D_{R-2}) ...)
     P_{p+1}^T + D_{p+1}, and runs its real backward from it.  Rank 0's ds0 is the sequence's.

Every compute step is a call into libwkv7 (``ops``, the binding module by default); this module only
moves tensors and runs the collectives.  The phases are separate functions so that a single process
can run all ranks' phases in turn (``emulate_forward`` / ``emulate_backward``), with the gathers
replaced by plain lists.  The pages have no passage on this; it is the exchange the state's
affinity allows.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence

import torch

def _binding():
    from . import wkv7
    return wkv7


@dataclasses.dataclass
class Segment:
    """One rank's tokens of every row: r..b [B, T_p, H, N] and its slice of the reset flags."""
    inputs: Sequence[torch.Tensor]
    reset: Optional[torch.Tensor] = None


@dataclasses.dataclass
class Context:
    """What a rank keeps from its forward for its backward."""
    rank: int
    world: int
    segment: Segment
    s_in: Optional[torch.Tensor]          # state entering the segment (the sequence's s0 on rank 0)
    workspace: torch.Tensor               # checkpoints of the real forward
    transitions: List[Optional[torch.Tensor]]   # P_q of every rank (None for rank 0)
    algo: str
    log_decay: bool


class DistExchange:
    """All-gather over a torch.distributed process group (NCCL on GPUs, gloo on CPU)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def all_gather(self, t: torch.Tensor) -> List[torch.Tensor]:
        out = [torch.empty_like(t) for _ in range(self.world)]
        self.dist.all_gather(out, t.contiguous(), group=self.group)
        return out


def _identity_state(ref: torch.Tensor) -> torch.Tensor:
    B, _, H, N = ref.shape
    return torch.eye(N, device=ref.device, dtype=torch.float32).expand(B, H, N, N).contiguous()


# ----------------------------------------------------------------- forward phases
def forward_local(seg: Segment, rank: int, s0=None, *, ops=None, algo="auto", log_decay=False):
    """Phase 1.  Rank 0: its real forward from s0 -> (y, s_end, workspace, P=None, U=s_end).
    Rank p >= 1: (None, None, None, P_p, U_p)."""
    ops = ops or _binding()
    r, w, k, v, a, b = seg.inputs
    if rank == 0:
        y, s_end, ws = ops.forward(r, w, k, v, a, b, s0=s0, reset=seg.reset, algo=algo, log_decay=log_decay)
        return y, s_end, ws, None, s_end
    _, P, _ = ops.forward(r, w, k, torch.zeros_like(v), a, b, s0=_identity_state(r), reset=seg.reset,
                          need_workspace=False, algo=algo, log_decay=log_decay)
    _, U, _ = ops.forward(r, w, k, v, a, b, reset=seg.reset, need_workspace=False, algo=algo, log_decay=log_decay)
    return None, None, None, P, U


def entering_state(rank: int, Ps: Sequence[torch.Tensor], Us: Sequence[torch.Tensor], *, ops=None):
    """S entering segment ``rank`` (>= 1) from the gathered (P_q, U_q): U_0 composed through
    segments 1 .. rank-1 in order."""
    ops = ops or _binding()
    S = Us[0]
    for q in range(1, rank):
        S = ops.state_compose(S, Ps[q], Us[q])
    return S


def forward_final(seg: Segment, rank: int, s_in, *, ops=None, algo="auto", log_decay=False):
    """Phase 3 (ranks >= 1): the real forward from the entering state."""
    ops = ops or _binding()
    return ops.forward(*seg.inputs, s0=s_in, reset=seg.reset, algo=algo, log_decay=log_decay)


def forward(seg: Segment, s0=None, *, exchange=None, ops=None, algo="auto", log_decay=False):
    """This rank's part of the forward over the whole sequence.  ``s0`` (the sequence's initial
    state) is read on rank 0 only.  Returns (y of the segment, the state after the segment -- the
    sequence's final state on the last rank --, Context for ``backward``)."""
    ex = exchange or DistExchange()
    rank, world = ex.rank, ex.world
    y, s_end, ws, P, U = forward_local(seg, rank, s0, ops=ops, algo=algo, log_decay=log_decay)
    Ps = ex.all_gather(P if P is not None else torch.zeros_like(U))
    Us = ex.all_gather(U)
    s_in = s0
    if rank > 0:
        s_in = entering_state(rank, Ps, Us, ops=ops)
        y, s_end, ws = forward_final(seg, rank, s_in, ops=ops, algo=algo, log_decay=log_decay)
    trans = [None] + list(Ps[1:])
    return y, s_end, Context(rank, world, seg, s_in, ws, trans, algo, log_decay)


# ----------------------------------------------------------------- backward phases
def backward_local(ctx: Context, dy, dsT=None, *, ops=None):
    """Phase 1.  The last rank: its real backward from dsT (gradients and its ds0).  Others: their
    backward with dsT = 0, of which only ds0 is kept.  Returns (grads or None, ds0)."""
    ops = ops or _binding()
    seg = ctx.segment
    last = ctx.rank == ctx.world - 1
    g = ops.backward(*seg.inputs, dy, ctx.workspace, s0=ctx.s_in, reset=seg.reset, dsT=dsT if last else None,
                     algo=ctx.algo, log_decay=ctx.log_decay)
    return (g if last else None), g["ds0"]


def leaving_gradient(ctx: Context, Ds: Sequence[torch.Tensor], *, ops=None):
    """dS leaving segment ``ctx.rank`` (< world - 1) from the gathered ds0 and the transitions."""
    ops = ops or _binding()
    last = ctx.world - 1
    D = Ds[last]
    for q in range(last - 1, ctx.rank, -1):
        D = ops.state_compose(D, ctx.transitions[q], Ds[q], transpose=True)
    return D


def backward_final(ctx: Context, dy, ds_end, *, ops=None):
    ops = ops or _binding()
    seg = ctx.segment
    return ops.backward(*seg.inputs, dy, ctx.workspace, s0=ctx.s_in, reset=seg.reset, dsT=ds_end, algo=ctx.algo,
                        log_decay=ctx.log_decay)


def backward(ctx: Context, dy, dsT=None, *, exchange=None, ops=None):
    """This rank's part of the backward: gradients of its segment's inputs ("ds0" on rank 0 is the
    gradient of the sequence's s0; elsewhere it is dS entering the segment).  ``dsT`` (the
    gradient of the sequence's final state) is read on the last rank only."""
    ex = exchange or DistExchange()
    g, D = backward_local(ctx, dy, dsT, ops=ops)
    Ds = ex.all_gather(D)
    if ctx.rank < ctx.world - 1:
        g = backward_final(ctx, dy, leaving_gradient(ctx, Ds, ops=ops), ops=ops)
    return g


# ----------------------------------------------------------------- all ranks in one process
def emulate_forward(segs: Sequence[Segment], s0=None, *, ops=None, algo="auto", log_decay=False):
    """Every rank's forward phases in turn on one device (the gathers become lists).  Returns
    ([y_p], [s_end_p], [Context_p])."""
    R = len(segs)
    loc = [forward_local(segs[p], p, s0, ops=ops, algo=algo, log_decay=log_decay) for p in range(R)]
    Us = [l[4] for l in loc]
    Ps = [l[3] if l[3] is not None else torch.zeros_like(Us[0]) for l in loc]
    ys, ends, ctxs = [], [], []
    for p in range(R):
        y, s_end, ws = loc[p][0], loc[p][1], loc[p][2]
        s_in = s0
        if p > 0:
            s_in = entering_state(p, Ps, Us, ops=ops)
            y, s_end, ws = forward_final(segs[p], p, s_in, ops=ops, algo=algo, log_decay=log_decay)
        ys.append(y)
        ends.append(s_end)
        ctxs.append(Context(p, R, segs[p], s_in, ws, [None] + Ps[1:], algo, log_decay))
    return ys, ends, ctxs


def emulate_backward(ctxs: Sequence[Context], dys: Sequence[torch.Tensor], dsT=None, *, ops=None):
    """Every rank's backward phases in turn on one device.  Returns [grads_p]."""
    R = len(ctxs)
    loc = [backward_local(ctxs[p], dys[p], dsT, ops=ops) for p in range(R)]
    Ds = [l[1] for l in loc]
    out = []
    for p in range(R):
        g = loc[p][0]
        if p < R - 1:
            g = backward_final(ctxs[p], dys[p], leaving_gradient(ctxs[p], Ds, ops=ops), ops=ops)
        out.append(g)
    return out


def split_tokens(T: int, world: int) -> List[int]:
    """Boundaries [t_0 = 0, t_1, ..., t_world = T] of world consecutive segments made of whole
    16-token chunks (the first segments take one chunk more when the chunks do not divide; the
    last one ends at T).  With T < 16 (world - 1) + 1 the last segments are empty: an empty
    segment passes the state and its gradient through unchanged."""
    if world < 1:
        raise ValueError("world must be >= 1")
    chunks = (T + 15) // 16
    per, extra = divmod(chunks, world)
    bounds = [0]
    for p in range(world):
        bounds.append(min(T, bounds[-1] + 16 * (per + (1 if p < extra else 0))))
    return bounds
