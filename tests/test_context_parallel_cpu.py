"""Context parallelism without a GPU: the tokens of each row split over 2 and 3 gloo ranks on this
host, each rank's compute steps done by the fp64 oracle (forward, backward) and an fp64 matrix
product (the state composition), so that what is tested is the module's own logic: which rank
computes which transition, the order of the two scans, the exchange, and which gradient each rank
returns.  The result must equal the oracle's single run over the whole sequence (resets, an initial
state and a final-state gradient included).  The GPU kernels of the same steps are tested on one
device in ``test_gpu_context_parallel.py``.
"""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


class OracleOps:
    """The three compute steps the module calls, in fp64 on the CPU."""

    @staticmethod
    def forward(r, w, k, v, a, b, s0=None, reset=None, need_workspace=True, algo="auto", log_decay=False, **_):
        import oracle
        f = lambda x: None if x is None else x.numpy()   # noqa: E731
        y, s, _ = oracle.forward(*(f(x) for x in (r, w, k, v, a, b)), s0=f(s0), reset=f(reset), log_decay=log_decay)
        return torch.from_numpy(y), torch.from_numpy(s), torch.zeros(1)

    @staticmethod
    def backward(r, w, k, v, a, b, dy, ws, s0=None, reset=None, dsT=None, algo="auto", log_decay=False, **_):
        import oracle
        f = lambda x: None if x is None else x.numpy()   # noqa: E731
        g, _ = oracle.backward(*(f(x) for x in (r, w, k, v, a, b)), f(dy), s0=f(s0), reset=f(reset), dsT=f(dsT),
                               log_decay=log_decay)
        return {n: torch.from_numpy(g[n]) for n in g}

    @staticmethod
    def state_compose(S, P, U, transpose=False, **_):
        PP = P.transpose(-1, -2) if transpose else P
        return (S @ PP if S is not None else 0) + (U if U is not None else 0)


def _problem(T, log_decay=False):
    from linear_recurrent_lm_b200 import inputs as I
    rng = np.random.default_rng(123 + T)
    B, H, N = 2, 2, 8
    d = I.draw_inputs(rng, (B, T, H, N), "f32", log_decay=log_decay)
    xs = [I.to_f64(d[n]) for n in I.NAMES]
    s0 = rng.standard_normal((B, H, N, N))
    dy = rng.standard_normal((B, T, H, N))
    dsT = rng.standard_normal((B, H, N, N))
    reset = np.zeros((B, T), np.uint8)
    reset[0, T // 2] = 1
    reset[1, 32] = 1                  # the first token of rank 1's segment in both splits below
    return xs, s0, dy, dsT, reset


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, T, log_decay, out):
    from linear_recurrent_lm_b200 import context_parallel as cp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        xs, s0, dy, dsT, reset = _problem(T, log_decay)
        bounds = cp.split_tokens(T, world)
        t0, t1 = bounds[rank], bounds[rank + 1]
        seg = cp.Segment([torch.from_numpy(np.ascontiguousarray(x[:, t0:t1])) for x in xs],
                         torch.from_numpy(np.ascontiguousarray(reset[:, t0:t1])))
        ex = cp.DistExchange()
        y, s_end, ctx = cp.forward(seg, torch.from_numpy(s0), exchange=ex, ops=OracleOps, log_decay=log_decay)
        g = cp.backward(ctx, torch.from_numpy(np.ascontiguousarray(dy[:, t0:t1])), torch.from_numpy(dsT),
                        exchange=ex, ops=OracleOps)
        out[rank] = (t0, t1, y.numpy(), s_end.numpy(), {n: g[n].numpy() for n in g})
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,T,log_decay", [(2, 45, False), (3, 70, False), (3, 70, True)])
def test_context_parallel_equals_one_run(world, T, log_decay):
    import oracle
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_rank_main, args=(world, port, T, log_decay, out), nprocs=world, join=True,
                       start_method="spawn")
    xs, s0, dy, dsT, reset = _problem(T, log_decay)
    y, s, _ = oracle.forward(*xs, s0=s0, reset=reset, log_decay=log_decay)
    g, _ = oracle.backward(*xs, dy, s0=s0, reset=reset, dsT=dsT, log_decay=log_decay)
    rel = lambda a, b: float(np.max(np.abs(a - b)) / np.sqrt(np.mean(b * b)))   # noqa: E731
    for p in range(world):
        t0, t1, yp, sp, gp = out[p]
        assert rel(yp, y[:, t0:t1]) < 1e-12, p
        for n in ("dr", "dw", "dk", "dv", "da", "db"):
            assert rel(gp[n], g[n][:, t0:t1]) < 1e-11, (p, n)
    assert rel(out[world - 1][3], s) < 1e-12          # the last rank ends with the sequence's state
    assert rel(out[0][4]["ds0"], g["ds0"]) < 1e-11    # rank 0 returns the sequence's ds0


def test_split_tokens():
    from linear_recurrent_lm_b200 import context_parallel as cp
    assert cp.split_tokens(4096, 4) == [0, 1024, 2048, 3072, 4096]
    assert cp.split_tokens(70, 3) == [0, 32, 64, 70]
    assert cp.split_tokens(45, 2) == [0, 32, 45]
    assert cp.split_tokens(20, 3) == [0, 16, 20, 20]
    with pytest.raises(ValueError):
        cp.split_tokens(10, 0)


def test_emulated_ranks_equal_one_run():
    """The single-process driver (every rank's phases in turn, the gathers as lists) with the same
    oracle steps: 4 segments, the last one ragged."""
    import oracle
    from linear_recurrent_lm_b200 import context_parallel as cp
    T = 61
    xs, s0, dy, dsT, reset = _problem(T)
    bounds = cp.split_tokens(T, 4)
    segs = [cp.Segment([torch.from_numpy(np.ascontiguousarray(x[:, t0:t1])) for x in xs],
                       torch.from_numpy(np.ascontiguousarray(reset[:, t0:t1])))
            for t0, t1 in zip(bounds[:-1], bounds[1:])]
    ys, ends, ctxs = cp.emulate_forward(segs, torch.from_numpy(s0), ops=OracleOps)
    gs = cp.emulate_backward(ctxs, [torch.from_numpy(np.ascontiguousarray(dy[:, t0:t1]))
                                    for t0, t1 in zip(bounds[:-1], bounds[1:])],
                             torch.from_numpy(dsT), ops=OracleOps)
    y, s, _ = oracle.forward(*xs, s0=s0, reset=reset)
    g, _ = oracle.backward(*xs, dy, s0=s0, reset=reset, dsT=dsT)
    rel = lambda a, b: float(np.max(np.abs(a - b)) / np.sqrt(np.mean(b * b)))   # noqa: E731
    assert rel(torch.cat(ys, dim=1).numpy(), y) < 1e-12
    assert rel(ends[-1].numpy(), s) < 1e-12
    for n in ("dr", "dw", "dk", "dv", "da", "db"):
        assert rel(torch.cat([gp[n] for gp in gs], dim=1).numpy(), g[n]) < 1e-11, n
    assert rel(gs[0]["ds0"].numpy(), g["ds0"]) < 1e-11


def test_segment_is_affine_in_its_entering_state():
    """The identity the split rests on, on the oracle alone: with P the end state from s0 = I and
    v = 0, and U the end state from s0 = 0, the end state from any s0 is s0 P + U (a reset inside
    the segment included); and the backward's ds0 from a final-state gradient D and dy is
    D P^T + (its ds0 from dy alone)."""
    import oracle
    xs, s0, dy, dsT, reset = _problem(37)
    B, H, N = s0.shape[0], s0.shape[1], s0.shape[2]
    eye = np.broadcast_to(np.eye(N), (B, H, N, N)).copy()
    v0 = np.zeros_like(xs[3])
    for rs in (np.zeros_like(reset), reset):
        _, P, _ = oracle.forward(xs[0], xs[1], xs[2], v0, xs[4], xs[5], s0=eye, reset=rs)
        _, U, _ = oracle.forward(*xs, reset=rs)
        _, S, _ = oracle.forward(*xs, s0=s0, reset=rs)
        np.testing.assert_allclose(S, s0 @ P + U, rtol=0, atol=1e-12 * np.abs(S).max())
        g, _ = oracle.backward(*xs, dy, s0=s0, reset=rs, dsT=dsT)
        g0, _ = oracle.backward(*xs, dy, s0=s0, reset=rs)
        ref = dsT @ np.swapaxes(P, -1, -2) + g0["ds0"]
        np.testing.assert_allclose(g["ds0"], ref, rtol=0, atol=1e-12 * np.abs(ref).max())
    assert np.abs(P).max() == 0.0        # the reset inside the segment (row 0) and at t = 32 (row 1)
