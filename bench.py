"""WKV-7 benchmark on B200: tokens/s for forward and forward+backward at H=32, N=64.

Default workload (one "step" = one forward with checkpoints + one backward over
one batch): the packed-document training batch B=8, T=4096, H=32, N=64, bf16,
geometric document lengths (mean 512) with state resets, seeded synthetic
data shaped like a 1.5B-model layer (32 heads of 64).  Its inputs (>0.9 GB)
exceed the 126 MB L2, so no flush is needed between timed steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints ONE JSON line (rank 0).  ``value`` is fwd+bwd tokens/s over all ranks
(weak scaling: every rank runs its own batch, no data-path collective);
timing is CUDA events on the launching stream, max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from linear_recurrent_lm_b200 import inputs as I   # noqa: E402

METRIC = "WKV-7 tokens/s fwd and fwd+bwd (H=32,N=64) + % of HBM roofline, 1xB200"
WORKLOAD = 3
# algorithmic bytes per token-head (bf16): inputs 6x64x2, y or dy 64x2, one fp32 64x64
# checkpoint per 16 tokens (16 KiB / 16), gradients 6x64x2
BYTES_FWD_TRAIN = 768 + 128 + 1024
BYTES_BWD = 768 + 128 + 1024 + 768
BYTES_PREFILL = 768 + 128
BYTES_DECODE = 64 * 64 * 4 * 2 + 768 + 128
BYTES_EPI_FWD = 5 * 128 + 128                # y, r, k, v, g in; out (bf16)
BYTES_EPI_BWD = 6 * 128 + 128 + 4 * 256      # y, r, k, v, g, dout in; dg, and dy, dr, dk, dv parts (fp32) out
# GDN map per value token-head at N = 128, bf16, two value heads per key head: q, k read once per key
# head (512 B / 2), g and beta (8 B), r, x, kw, a, b written (5 x 256 B).
BYTES_GDN_MAP = 512 // 2 + 8 + 5 * 256
# Token-order forward at N = 128 without checkpoints: six inputs and y, 256 B each.
BYTES_SCAN128_FWD = 7 * 256


def rank_seed(rank: int) -> int:
    """Seed of a rank's synthetic batch: every rank draws a different batch of the same workload."""
    return 1000 + WORKLOAD + rank


def rank_max(values, device, world: int):
    """Element-wise max over ranks of per-rank timings (ms); the identity on one rank."""
    import torch
    t = torch.tensor([float(v) for v in values], device=device, dtype=torch.float64)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_tokens_per_s(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput under weak scaling: all ranks' tokens over the slowest rank's step time."""
    return tokens_per_rank * world / (ms_per_step / 1e3)


NOMINAL_HBM_GBS = 8000.0   # B200 HBM3e nominal (context: the roofline uses the measured copy bandwidth)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


_KERNEL_HEADERS = ("common.cuh", "kernels.h", "mma.cuh", "tc05.cuh", "token_path.cuh")


def _strip_c_comments(text: str) -> str:
    """C/CUDA source without comments, whitespace runs collapsed (string literals kept)."""
    out, i, n = [], 0, len(text)
    while i < n:
        if text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif text[i] == '"':
            j = i + 1
            while j < n and text[j] != '"':
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            out.append(text[i])
            i += 1
    return " ".join("".join(out).split())


def kernel_code_sha256(source_file: str) -> str:
    """Hash of a kernel's code: its .cu file and the shared headers, comments and layout ignored,
    so that a profile stays attached to the kernel until the code itself changes."""
    h = hashlib.sha256()
    for rel in [source_file] + [f"linear_recurrent_lm_b200/csrc/{x}" for x in _KERNEL_HEADERS]:
        with open(os.path.join(ROOT, rel)) as f:
            h.update(_strip_c_comments(f.read()).encode())
        h.update(b"\0")
    return h.hexdigest()


def kernel_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current code."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_code = re.search(r"code_sha256:\s*([0-9a-f]{64})", text)
    m_tr = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    src = re.search(r"source_file:\s*(\S+)", text)
    if not m_code or not m_tr or not src:
        return None
    try:
        cur = kernel_code_sha256(src.group(1))
    except OSError:
        return None
    return float(m_tr.group(1)) if cur == m_code.group(1) else None


class Clocks:
    """Samples the SM clock and the clock-event (throttle) reasons through NVML every few
    milliseconds on a background thread.  Only samples taken between mark_start() and
    mark_end() -- the timed region -- are summarised; reading clocks changes nothing."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int, period_s: float = 0.002):
        self.index, self.period = index, period_s
        self.samples, self.t0, self.t1 = [], None, None
        self.handle, self.thread, self.max_mhz = None, None, None
        self._stop = False

    def _open(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(self.index).uuid)
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(self.index)
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
        get = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        return pynvml, get

    def _run(self, pynvml, get_reasons):
        while not self._stop:
            try:
                now = time.perf_counter()
                mhz = pynvml.nvmlDeviceGetClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
                self.samples.append((now, float(mhz), int(get_reasons(self.handle))))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        try:
            pynvml, get = self._open()
            self.thread = threading.Thread(target=self._run, args=(pynvml, get), daemon=True)
            self.thread.start()
        except Exception:
            self.thread = None
        return self

    def mark_start(self):
        self.t0 = time.perf_counter()

    def mark_end(self):
        self.t1 = time.perf_counter()

    def __exit__(self, *exc):
        self._stop = True
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self):
        if self.thread is None or self.t0 is None or self.t1 is None:
            return None
        rows = [(m, r) for t, m, r in list(self.samples) if self.t0 <= t <= self.t1]
        if not rows:
            return None
        reasons = sorted({name for _, r in rows for bit, name in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(m for m, _ in rows), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(rows), "source": "nvml"}


def cpu_oracle_sample(wl, budget_s: float = 10.0):
    """The CPU oracle (C, fp64, all host cores) on a bounded sample of whole (b,h) units of the
    workload, forward + backward.  Returns tokens/s scaled to the workload's H heads."""
    import oracle
    cores = os.cpu_count() or 1
    units = [(b, h) for b in range(wl.B) for h in range(wl.H)]
    rng = np.random.default_rng(0)
    rng.shuffle(units)

    def run(us):
        t0 = time.perf_counter()
        for b in sorted({u[0] for u in us}):
            hs = [u[1] for u in us if u[0] == b]
            part = {n: I.to_f64(wl.inputs[n][b:b + 1, :, hs]) for n in I.NAMES}
            reset = wl.reset[b:b + 1] if wl.reset is not None else None
            oracle.forward(*(part[n] for n in I.NAMES), reset=reset)
            oracle.backward(*(part[n] for n in I.NAMES), I.to_f64(wl.dy[b:b + 1, :, hs]), reset=reset)
        return time.perf_counter() - t0

    t_one = run(units[:1])
    n = int(min(len(units), max(1, budget_s / max(t_one, 1e-3)) * min(cores, len(units)) / 2))
    n = max(1, min(n, len(units)))
    t = run(units[:n])
    tokens = n * wl.T / wl.H          # unit-tokens expressed as tokens of the H-head layer
    return {"value": tokens / t, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} of {wl.B * wl.H} (b,h) units x T={wl.T}, fwd+bwd, fp64 C oracle, {t:.1f} s"}


def oracle_table(cores: int):
    """The fp64 C oracle on every workload: forward and forward+backward of workloads 1-3 and
    the 128 ragged decode steps of workload 4, with all host cores and with one, each on a
    bounded sample of whole (b, h) units (tokens/s scaled to the workload's H heads)."""
    import oracle
    out = {}

    def time_units(wl, units, threads, bwd, prior=False):
        src = wl.inputs
        t0 = time.perf_counter()
        by_b = {}
        for b, h in units:
            by_b.setdefault(b, []).append(h)
        for b, hs in by_b.items():
            part = [I.to_f64(src[n][b:b + 1, :, hs]) for n in I.NAMES]
            reset = wl.reset[b:b + 1] if wl.reset is not None else None
            s0 = None
            if prior:
                _, s0, _ = oracle.forward(*(I.to_f64(wl.prior[n][b:b + 1, :, hs]) for n in I.NAMES), nthreads=threads)
            oracle.forward(*part, s0=s0, reset=reset, nthreads=threads)
            if bwd:
                oracle.backward(*part, I.to_f64(wl.dy[b:b + 1, :, hs]), s0=s0, reset=reset, nthreads=threads)
        dt = time.perf_counter() - t0
        return len(units) * wl.T / wl.H / dt

    for idx, name in ((1, "c1_B2_T512_H12"), (2, "c2_prefill_B1_T1024_H32"), (3, "c3_packed_B8_T4096_H32")):
        wl = I.make_workload(idx)
        units = [(b, h) for b in range(wl.B) for h in range(wl.H)]
        for threads, n_units in ((cores, min(len(units), 2 * cores if idx == 3 else len(units))), (1, min(len(units), 2))):
            key = f"{name}_{'all_cores' if threads == cores else '1_core'}"
            entry = {"fwd_tokens_per_s": time_units(wl, units[:n_units], threads, False, prior=idx == 2),
                     "units": n_units}
            if idx != 2:
                entry["fwd_bwd_tokens_per_s"] = time_units(wl, units[:n_units], threads, True)
            out[key] = entry
    wl = I.make_workload(4)
    rows = list(range(min(wl.B, 16)))
    st = wl.state0[rows].astype(np.float64)
    t0 = time.perf_counter()
    active_tok = 0
    for s in range(len(wl.steps)):
        act = wl.active(s)[rows]
        active_tok += int(act.sum())
        _, st = oracle.step(*(I.to_f64(wl.steps[s][n][rows]) for n in I.NAMES), st, act)
    out["c4_decode_128_steps_1_core"] = {"tokens_per_s": active_tok / (time.perf_counter() - t0), "rows": len(rows)}
    return out


def run_reference(args):
    """The oracle as the reference arm: same workload/metric, bounded sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = I.make_workload(WORKLOAD)
    cores = os.cpu_count() or 1
    import oracle
    units = [(b, h) for b in range(wl.B) for h in range(wl.H)][: max(1, min(cores, 32))]
    part_b = {}
    for b, h in units:
        part_b.setdefault(b, []).append(h)

    def step():
        for b, hs in part_b.items():
            part = {n: I.to_f64(wl.inputs[n][b:b + 1, :, hs]) for n in I.NAMES}
            reset = wl.reset[b:b + 1]
            oracle.forward(*(part[n] for n in I.NAMES), reset=reset)
            oracle.backward(*(part[n] for n in I.NAMES), I.to_f64(wl.dy[b:b + 1, :, hs]), reset=reset)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / max(args.steps, 1)
    tokens = len(units) * wl.T / wl.H
    value = tokens / dt
    sample = f"{len(units)} of {wl.B * wl.H} (b,h) units x T={wl.T} per step, fwd+bwd, fp64 C oracle"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "B": wl.B, "T": wl.T, "H": wl.H, "N": wl.N},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "oracle_table": oracle_table(cores),
    }))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--algo", default="auto", choices=["auto", "scan", "chunked", "chunked_fused", "chunked_split"])
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--only", choices=["fwd", "bwd", "prefill", "step", "gdn_map"],
                    help="time one kernel alone (profiling entry point); prints its own JSON line")
    ap.add_argument("--B", type=int, default=None, help="batch override for --only")
    ap.add_argument("--step", type=int, default=0, help="--only step: which of the 128 ragged decode steps")
    ap.add_argument("--no-workspace", action="store_true",
                    help="--only prefill: no workspace (the fused chunked form instead of the split one)")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.only:
        return run_only(args)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    from linear_recurrent_lm_b200 import wkv7

    dev = torch.device("cuda", local)
    wl = I.make_workload(WORKLOAD, seed=rank_seed(rank))
    B, T, H = wl.B, wl.T, wl.H

    def d(x):
        x = np.ascontiguousarray(x)
        if x.dtype == np.uint16:
            return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(x).to(dev)

    xs = [d(wl.inputs[n]) for n in I.NAMES]
    dy = d(wl.dy)
    reset = d(wl.reset)
    y = torch.empty_like(xs[0])
    s_out = torch.empty((B, H, 64, 64), device=dev, dtype=torch.float32)
    ws = torch.empty(wkv7.workspace_bytes(B, T, H), device=dev, dtype=torch.uint8)
    grads = {n: torch.empty_like(xs[0]) for n in ("dr", "dw", "dk", "dv", "da", "db")}
    stream = torch.cuda.current_stream()

    def step(evs=None):
        if evs is not None:
            evs[0].record(stream)
        wkv7.forward(*xs, reset=reset, y=y, s_out=s_out, workspace=ws, algo=args.algo)
        if evs is not None:
            evs[1].record(stream)
        wkv7.backward(*xs, dy, ws, reset=reset, grads=grads, want_ds0=False, algo=args.algo)
        if evs is not None:
            evs[2].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    with Clocks(local) as clk:
        time.sleep(0.05)   # let the sampler take its first readings
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        clk.mark_start()
        start.record(stream)
        for s in range(args.steps):
            step(evs[s])
        end.record(stream)
        torch.cuda.synchronize()
        clk.mark_end()
    total_ms = start.elapsed_time(end)
    fwd_ms = [e[0].elapsed_time(e[1]) for e in evs]
    bwd_ms = [e[1].elapsed_time(e[2]) for e in evs]
    total_ms, fwd_avg, bwd_avg = rank_max([total_ms, statistics.mean(fwd_ms), statistics.mean(bwd_ms)], dev, world)
    ms_per_step = total_ms / args.steps
    tokens_step = B * T * world
    value = job_tokens_per_s(B * T, world, ms_per_step)

    # ---- e2e: through the public API with host buffers, copies inside the timed region.  Every step
    # copies its inputs from pinned host memory and all of its outputs (y and the six gradients) back;
    # the steps are pipelined two deep on three streams, as a training loop would run them: the H2D
    # copy of step k+1 and the D2H copy of step k-1 overlap the kernels of step k.
    host_in = [x.cpu().pin_memory() for x in xs] + [dy.cpu().pin_memory(), reset.cpu().pin_memory()]
    host_out = [torch.empty(xs[0].shape, dtype=xs[0].dtype, pin_memory=True) for _ in range(7)]
    dev_in = [[torch.empty_like(x, device=dev) for x in host_in] for _ in range(2)]
    dev_out = [[torch.empty_like(xs[0]) for _ in range(7)] for _ in range(2)]
    h2d = sum(x.numel() * x.element_size() for x in host_in)
    d2h = sum(x.numel() * x.element_size() for x in host_out)
    s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in", "comp", "out")}
    gnames = ("dr", "dw", "dk", "dv", "da", "db")

    def e2e_pipeline(n_steps, e_start=None, e_end=None):
        for k in range(n_steps):
            st = k % 2
            with torch.cuda.stream(s_h2d):
                if k == 0 and e_start is not None:
                    e_start.record(s_h2d)
                if k >= 2:
                    s_h2d.wait_event(ev["comp"][st])          # step k-2 no longer reads this input set
                for hsrc, dd in zip(host_in, dev_in[st]):
                    dd.copy_(hsrc, non_blocking=True)
                ev["in"][st].record(s_h2d)
            stream.wait_event(ev["in"][st])
            if k >= 2:
                stream.wait_event(ev["out"][st])              # step k-2's outputs have been copied out
            xin, outs = dev_in[st], dev_out[st]
            wkv7.forward(*xin[:6], reset=xin[7], y=outs[0], s_out=s_out, workspace=ws, algo=args.algo)
            wkv7.backward(*xin[:6], xin[6], ws, reset=xin[7], grads=dict(zip(gnames, outs[1:])), want_ds0=False,
                          algo=args.algo)
            ev["comp"][st].record(stream)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(ev["comp"][st])
                for o, hdst in zip(outs, host_out):
                    hdst.copy_(o, non_blocking=True)
                ev["out"][st].record(s_d2h)
                if k == n_steps - 1 and e_end is not None:
                    e_end.record(s_d2h)

    e2e_pipeline(2)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e2e_pipeline(args.e2e_steps, e0, e1)
    torch.cuda.synchronize()
    e2e_ms = rank_max([e0.elapsed_time(e1)], dev, world)[0] / args.e2e_steps
    e2e_value = job_tokens_per_s(B * T, world, e2e_ms)

    # The secondary lines are single-GPU diagnostics (about a minute of work): under torchrun the
    # other ranks would sit in the barrier below for all of it, against the process group's timeout.
    secondary = {}
    if rank == 0 and world == 1 and not args.no_secondary:
        secondary = measure_secondary(wkv7, dev, args.algo)
        if args.algo != "scan":   # the token-order scan kernels on the same batch, for comparison
            ev3 = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            f_ms, b_ms = [], []
            for rep in range(4):
                ev3[0].record(stream)
                wkv7.forward(*xs, reset=reset, y=y, s_out=s_out, workspace=ws, algo="scan")
                ev3[1].record(stream)
                wkv7.backward(*xs, dy, ws, reset=reset, grads=grads, want_ds0=False, algo="scan")
                ev3[2].record(stream)
                torch.cuda.synchronize()
                if rep:
                    f_ms.append(ev3[0].elapsed_time(ev3[1]))
                    b_ms.append(ev3[1].elapsed_time(ev3[2]))
            fm, bm = statistics.median(f_ms), statistics.median(b_ms)
            units_s = B * T * H
            peak_s, _ = measured_peaks()
            secondary[f"scan_{wl.name}"] = {
                "fwd_ms": fm, "bwd_ms": bm, "fwd_bwd_tokens_per_s": B * T / ((fm + bm) / 1e3),
                "fwd_frac": BYTES_FWD_TRAIN * units_s / (fm / 1e3) / 1e9 / peak_s,
                "bwd_frac": BYTES_BWD * units_s / (bm / 1e3) / 1e9 / peak_s}

    if world > 1:
        dist.barrier()
    if rank == 0:
        peak, peak_kind = measured_peaks()
        units = B * T * H
        fwd_gbs = BYTES_FWD_TRAIN * units / (fwd_avg / 1e3) / 1e9
        bwd_gbs = BYTES_BWD * units / (bwd_avg / 1e3) / 1e9
        dominant = ("bwd", bwd_avg, bwd_gbs, BYTES_BWD) if bwd_avg >= fwd_avg else ("fwd", fwd_avg, fwd_gbs, BYTES_FWD_TRAIN)
        kname = {"fwd": "chunk_fwd" if args.algo != "scan" else "scan_fwd",
                 "bwd": "chunk_bwd" if args.algo != "scan" else "scan_bwd"}[dominant[0]]
        traffic = kernel_traffic(kname, "packed_train_B8_T4096_H32")
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            cpu = cpu_oracle_sample(wl)
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "B": B, "T": T, "H": H, "N": 64, "algo": args.algo,
                       "l2": "inputs larger than L2 (no flush)", "parallelism": f"dp{world} (independent batches)"},
            "fwd": {"tokens_per_s": tokens_step / (fwd_avg / 1e3), "ms": fwd_avg, "achieved_gbs": fwd_gbs,
                    "frac": fwd_gbs / peak},
            "fwd_bwd": {"tokens_per_s": value, "ms": ms_per_step,
                        "achieved_gbs": (BYTES_FWD_TRAIN + BYTES_BWD) * units / (ms_per_step / 1e3) / 1e9,
                        "frac": (BYTES_FWD_TRAIN + BYTES_BWD) * units / (ms_per_step / 1e3) / 1e9 / peak},
            "roofline": {"bound": "hbm", "kernel": kname, "achieved": dominant[2], "peak": peak, "unit": "GB/s",
                         "frac": dominant[2] / peak, "peak_kind": peak_kind,
                         "frac_of_nominal_8000": dominant[2] / NOMINAL_HBM_GBS,
                         "bytes_per_launch": dominant[3] * units,
                         "traffic": traffic},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms, "steps": args.e2e_steps,
                    "pipelining": "two deep: H2D of step k+1 and D2H of step k-1 overlap step k (pinned host buffers)"},
            # per step: the forward kernel, the chunked backward and its exact re-run of flagged heads
            # (which returns at once when none is flagged); the scan algorithm launches one kernel each way
            "gpu_launches": (3 if args.algo != "scan" else 2) * args.steps,
            "clocks": clk.summary(),
            "secondary": secondary,
        }
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()


def measure_secondary(wkv7, dev, algo):
    """Stateful prefill (B=1, T=1024, H=32), the backward's exact fallback for a flagged head, the
    packed batch with the log-space decay input, the WKV epilogue, and the 128-step ragged decode
    (256 x 32 states)."""
    import torch
    out = {}
    peak, _ = measured_peaks()
    flush = torch.empty(512 * 1024 * 1024 // 4, device=dev, dtype=torch.float32)

    def d(x):
        x = np.ascontiguousarray(x)
        if x.dtype == np.uint16:
            return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(x).to(dev)

    wl = I.make_workload(2)
    prior = [d(wl.prior[n]) for n in I.NAMES]
    _, s0, _ = wkv7.forward(*prior, algo=algo, need_workspace=False)
    xs = [d(wl.inputs[n]) for n in I.NAMES]
    y = torch.empty_like(xs[0])
    s_out = torch.empty_like(s0)
    ws = torch.empty(wkv7.workspace_bytes(wl.B, wl.T, wl.H, xs[0].dtype), device=dev, dtype=torch.uint8)
    units = wl.B * wl.T * wl.H
    # With a workspace the 32 (b,h) units take the split chunked form (a chunk-parallel pass, then
    # a short sequential one per unit); without one, the fused form (one CTA per unit).
    for key, workspace in (("prefill_B1_T1024_H32", ws), ("prefill_B1_T1024_H32_no_workspace", None)):
        times = []
        for rep in range(25):
            flush.fill_(float(rep))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            wkv7.forward(*xs, s0=s0, y=y, s_out=s_out, workspace=workspace, need_workspace=False, algo=algo)
            e1.record()
            torch.cuda.synchronize()
            if rep >= 5:
                times.append(e0.elapsed_time(e1))
        ms = statistics.median(times)
        gbs = BYTES_PREFILL * units / (ms / 1e3) / 1e9
        out[key] = {"tokens_per_s": wl.B * wl.T / (ms / 1e3), "ms": ms, "achieved_gbs": gbs,
                    "frac": gbs / peak, "workspace": workspace is not None,
                    "l2": "flushed (512 MB write) before each rep"}

    # The exact fallback of the chunked backward: a head whose decay the 1/L scaling cannot take
    # (some w < 1/16 in a chunk) is marked and recomputed by the token-order scan backward.  One such
    # head among the 32 of one packed row (B=1, T=4096), timed against the same row without it.
    wl = I.make_workload(3, B=1)
    xs = [d(wl.inputs[n]) for n in I.NAMES]
    dyt, rst = d(wl.dy), d(wl.reset)
    w_flag = I.to_f64(wl.inputs["w"]).copy()
    w_flag[0, 2000, 5, :4] = 0.03
    xs_flag = list(xs)
    xs_flag[I.NAMES.index("w")] = d(I.to_storage(w_flag, "bf16"))
    for key, xx in (("bwd_B1_T4096_H32", xs), ("bwd_B1_T4096_H32_one_flagged_head", xs_flag)):
        _, _, wsb = wkv7.forward(*xx, reset=rst, algo=algo)
        times = []
        for rep in range(8):
            flush.fill_(float(rep))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            wkv7.backward(*xx, dyt, wsb, reset=rst, want_ds0=False, algo=algo)
            e1.record()
            torch.cuda.synchronize()
            if rep >= 2:
                times.append(e0.elapsed_time(e1))
        ms = statistics.median(times)
        out[key] = {"ms": ms, "tokens_per_s": wl.B * wl.T / (ms / 1e3),
                    "flagged_heads": 1 if "flagged" in key else 0,
                    "l2": "flushed (512 MB write) before each rep"}

    # The packed training batch with the log-space decay input (x in place of w, w = exp(-exp(x))
    # computed in the kernels, dL/dx out): the cost of the transform on the full step.
    wl = I.make_workload(3, log_decay=True)
    xs = [d(wl.inputs[n]) for n in I.NAMES]
    dyt, rst = d(wl.dy), d(wl.reset)
    _, _, wsl = wkv7.forward(*xs, reset=rst, algo=algo, log_decay=True)
    f_ms, b_ms = [], []
    for rep in range(6):
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record()
        wkv7.forward(*xs, reset=rst, workspace=wsl, algo=algo, log_decay=True)
        e1.record()
        wkv7.backward(*xs, dyt, wsl, reset=rst, want_ds0=False, algo=algo, log_decay=True)
        e2.record()
        torch.cuda.synchronize()
        if rep >= 2:
            f_ms.append(e0.elapsed_time(e1))
            b_ms.append(e1.elapsed_time(e2))
    fm, bm = statistics.median(f_ms), statistics.median(b_ms)
    out["packed_train_B8_T4096_H32_log_decay"] = {
        "fwd_ms": fm, "bwd_ms": bm, "fwd_bwd_tokens_per_s": wl.B * wl.T / ((fm + bm) / 1e3),
        "l2": "inputs larger than L2 (no flush)"}
    del xs, dyt, rst, wsl

    # The WKV epilogue (GroupNorm per head, bonus, gating) on the packed batch's shape, each way one
    # streaming kernel: forward reads y, r, k, v, g and writes out (768 B per token-head); backward
    # reads those and dout and writes dg and an fp32 block of dy and the bonus parts of dr, dk, dv (1920 B).
    B3, T3, H3 = 8, 4096, 32
    gen = torch.Generator(device=dev).manual_seed(5)
    tens = [torch.randn((B3, T3, H3, 64), device=dev, generator=gen).to(torch.bfloat16) for _ in range(6)]
    ln_w = 1.0 + 0.3 * torch.randn((H3, 64), device=dev, generator=gen)
    ln_b = 0.2 * torch.randn((H3, 64), device=dev, generator=gen)
    r_k = 0.5 * torch.randn((H3, 64), device=dev, generator=gen)
    yb, rb, kb, vb, gb, dob = tens
    outb = torch.empty_like(yb)
    eg = {"eg": torch.empty((4, B3, T3, H3, 64), device=dev, dtype=torch.float32), "dg": torch.empty_like(yb)}
    f_ms, b_ms = [], []
    for rep in range(12):
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record()
        wkv7.epilogue_forward(yb, rb, kb, vb, gb, ln_w, ln_b, r_k, 64e-5, out=outb)
        e1.record()
        wkv7.epilogue_backward(yb, rb, kb, vb, gb, dob, ln_w, ln_b, r_k, 64e-5, grads=eg)
        e2.record()
        torch.cuda.synchronize()
        if rep >= 2:
            f_ms.append(e0.elapsed_time(e1))
            b_ms.append(e1.elapsed_time(e2))
    fm, bm = statistics.median(f_ms), statistics.median(b_ms)
    units3 = B3 * T3 * H3
    # the forward with the epilogue fused into its y write-out (packed batch, fused chunked form)
    wl = I.make_workload(3)
    xs = [d(wl.inputs[n]) for n in I.NAMES]
    rst = d(wl.reset)
    ws3 = torch.empty(wkv7.workspace_bytes(wl.B, wl.T, wl.H, xs[0].dtype), device=dev, dtype=torch.uint8)
    fused = {}
    for key, want_y in (("with_y", True), ("out_only", False)):
        ms = []
        for rep in range(8):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            wkv7.forward_epilogue(*xs, gb, ln_w, ln_b, r_k, 64e-5, reset=rst, out=outb, y=yb if want_y else None,
                                  want_y=want_y, workspace=ws3, algo=algo)
            e1.record()
            torch.cuda.synchronize()
            if rep >= 2:
                ms.append(e0.elapsed_time(e1))
        fused[key] = statistics.median(ms)
    del xs, rst, ws3
    out["epilogue_B8_T4096_H32"] = {
        "forward_with_fused_epilogue_ms": fused["with_y"], "forward_with_fused_epilogue_out_only_ms": fused["out_only"],
        "fwd_ms": fm, "bwd_ms": bm,
        "fwd_frac": BYTES_EPI_FWD * units3 / (fm / 1e3) / 1e9 / peak,
        "bwd_frac": BYTES_EPI_BWD * units3 / (bm / 1e3) / 1e9 / peak,
        "l2": "inputs larger than L2 (no flush)"}
    del tens, yb, rb, kb, vb, gb, dob, outb, eg

    # A gated-DeltaNet layer on this recurrence (rwkv-lab page, "Highlight result -- GDN in RWKV-7"):
    # 32 value heads over 16 key heads of 128 channels, B=8, T=4096, bf16.  The map (q, k, g, beta ->
    # r, x, kw, a, b; HBM streaming) and then the token-order forward at N = 128 with the log-space
    # decay, no checkpoints (there is no N = 128 backward).
    Bg, Tg, Hg, Hkg, Ng = 8, 4096, 32, 16, 128
    gd = I.draw_gdn_inputs(np.random.default_rng(77), Bg, Tg, Hg, Hkg, Ng, "bf16")
    gq, gk, gv, gg, gb = (d(gd[n]) for n in ("q", "k", "v", "g", "beta"))
    del gd
    mo = {n: torch.empty((Bg, Tg, Hg, Ng), device=dev, dtype=torch.bfloat16) for n in ("r", "x", "kw", "a", "b")}
    yg = torch.empty_like(gv)
    sg = torch.empty((Bg, Hg, Ng, Ng), device=dev, dtype=torch.float32)
    m_ms, f_ms = [], []
    for rep in range(6):
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record()
        wkv7.gdn_map(gq, gk, gg, gb, Hg, eps=1e-6, out=mo)
        e1.record()
        wkv7.forward(mo["r"], mo["x"], mo["kw"], gv, mo["a"], mo["b"], y=yg, s_out=sg, need_workspace=False,
                     log_decay=True)
        e2.record()
        torch.cuda.synchronize()
        if rep >= 2:
            m_ms.append(e0.elapsed_time(e1))
            f_ms.append(e1.elapsed_time(e2))
    mm, fm = statistics.median(m_ms), statistics.median(f_ms)
    ug = Bg * Tg * Hg
    out["gdn_layer_B8_T4096_H32_Hk16_N128"] = {
        "map_ms": mm, "forward_ms": fm, "tokens_per_s": Bg * Tg / ((mm + fm) / 1e3),
        "map_frac": BYTES_GDN_MAP * ug / (mm / 1e3) / 1e9 / peak,
        "forward_gbs": BYTES_SCAN128_FWD * ug / (fm / 1e3) / 1e9,
        "l2": "inputs larger than L2 (no flush)"}
    del gq, gk, gv, gg, gb, mo, yg, sg

    # Context parallelism (the packed batch's rows split into R segments of T/R tokens, one per GPU),
    # emulated on this one GPU: the compute of one middle rank -- the transition P and zero-state end U
    # of its segment (two forwards), its entering state composed from R-2 gathered pairs (the most any
    # rank composes), its real forward; its backward with dsT = 0, the leaving gradient composed
    # through R-2 transitions, its real backward.  The all-gathers (2 x B*H*64*64*4 bytes per rank in
    # the forward, half that in the backward) are not timed here.
    from linear_recurrent_lm_b200 import context_parallel as cp
    wl = I.make_workload(3)
    cpo = {}
    for R in (2, 4, 8):
        bnd = cp.split_tokens(wl.T, R)
        t0, t1 = bnd[1], bnd[2]
        seg = cp.Segment([d(np.ascontiguousarray(wl.inputs[n][:, t0:t1])) for n in I.NAMES],
                         d(np.ascontiguousarray(wl.reset[:, t0:t1])))
        dys = d(np.ascontiguousarray(wl.dy[:, t0:t1]))
        gen = torch.Generator(device=dev).manual_seed(R)
        pairs = [torch.randn((wl.B, wl.H, 64, 64), device=dev, generator=gen) for _ in range(2 * R)]
        Ps, Us = pairs[:R], pairs[R:]
        ms = []
        for rep in range(5):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            cp.forward_local(seg, 1, None)
            s_in = cp.entering_state(R - 1, Ps, Us)
            _, _, ws = cp.forward_final(seg, 1, s_in)
            ctx = cp.Context(0, R, seg, s_in, ws, [None] + Ps[1:], "auto", False)
            cp.backward_local(ctx, dys, None)
            cp.backward_final(ctx, dys, cp.leaving_gradient(ctx, Us))
            e1.record()
            torch.cuda.synchronize()
            if rep >= 2:
                ms.append(e0.elapsed_time(e1))
        m = statistics.median(ms)
        cpo[f"R{R}"] = {"segment_tokens": t1 - t0, "rank_ms": m,
                        "job_tokens_per_s_without_exchange": wl.B * wl.T / (m / 1e3),
                        "exchange_bytes_per_rank": 3 * wl.B * wl.H * 64 * 64 * 4}
        del seg, dys, pairs, Ps, Us, ws, ctx
    out["context_parallel_B8_T4096_H32_emulated"] = {
        **cpo, "note": "one GPU runs one middle rank's compute; all-gathers not timed (one GPU per run)"}

    wl = I.make_workload(4)
    state = d(wl.state0)
    steps = [[d(s[n]) for n in I.NAMES] for s in wl.steps]
    acts = [d(wl.active(s)) for s in range(len(wl.steps))]
    yb = torch.empty_like(steps[0][0])
    for s in range(len(steps)):            # warm-up pass (state keeps evolving; the timing is per byte)
        wkv7.step(*steps[s], state, acts[s], y=yb)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for s in range(len(steps)):
        wkv7.step(*steps[s], state, acts[s], y=yb)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    active_tok = int(sum(int(wl.active(s).sum()) for s in range(len(wl.steps))))
    gbs = BYTES_DECODE * active_tok * wl.H / (ms / 1e3) / 1e9
    # Back to back, the states of the rows still active late in the ragged batch fit in the 126 MB L2,
    # so part of that traffic never reaches HBM.  The same 128 steps with L2 flushed before each one
    # (512 MB write, outside the timed events) read every state from HBM: that is the roofline figure.
    cold_ms = 0.0
    for s in range(len(steps)):
        flush.fill_(float(s))
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record()
        wkv7.step(*steps[s], state, acts[s], y=yb)
        c1.record()
        torch.cuda.synchronize()
        cold_ms += c0.elapsed_time(c1)
    cold_gbs = BYTES_DECODE * active_tok * wl.H / (cold_ms / 1e3) / 1e9
    out["decode_B256_H32_128steps"] = {"tokens_per_s": active_tok / (ms / 1e3), "ms_128_steps": ms,
                                       "achieved_gbs": gbs, "frac": gbs / peak, "active_tokens": active_tok,
                                       "l2": "back to back (late ragged steps partly served from L2)"}
    out["decode_B256_H32_128steps_l2_flushed"] = {
        "tokens_per_s": active_tok / (cold_ms / 1e3), "ms_128_steps": cold_ms, "achieved_gbs": cold_gbs,
        "frac": cold_gbs / peak, "active_tokens": active_tok,
        "l2": "flushed (512 MB write) before each step, outside the timed events: the HBM roofline figure"}
    return out


def run_only_gdn_map(args):
    """Warm-up + timed launches of the GDN map on the GDN layer shape (B=8 or --B, T=4096, 32 value
    heads over 16 key heads of 128, bf16)."""
    import torch
    from linear_recurrent_lm_b200 import wkv7
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    B = args.B or 8
    T, H, Hk, N = 4096, 32, 16, 128
    gd = I.draw_gdn_inputs(np.random.default_rng(77), B, T, H, Hk, N, "bf16")
    q, k = (torch.from_numpy(gd[n].view(np.int16)).view(torch.bfloat16).to(dev) for n in ("q", "k"))
    g, beta = (torch.from_numpy(gd[n]).to(dev) for n in ("g", "beta"))
    out = {n: torch.empty((B, T, H, N), device=dev, dtype=torch.bfloat16) for n in ("r", "x", "kw", "a", "b")}
    fn = lambda: wkv7.gdn_map(q, k, g, beta, H, eps=1e-6, out=out)   # noqa: E731
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / max(args.steps, 1)
    peak, _ = measured_peaks()
    gbs = BYTES_GDN_MAP * B * T * H / (ms / 1e3) / 1e9
    print(json.dumps({"only": "gdn_map", "workload": f"gdn_layer_B{B}_T{T}_H{H}_Hk{Hk}_N{N}", "ms": ms,
                      "achieved_gbs": gbs, "frac": gbs / peak}))


def run_only(args):
    """Warm-up + timed launches of a single kernel on the default workload (or a smaller batch)."""
    import torch
    from linear_recurrent_lm_b200 import wkv7
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if args.only == "gdn_map":
        return run_only_gdn_map(args)
    idx = {"fwd": 3, "bwd": 3, "prefill": 2, "step": 4}[args.only]
    wl = I.make_workload(idx, B=args.B)

    def d(x):
        x = np.ascontiguousarray(x)
        if x.dtype == np.uint16:
            return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(x).to(dev)

    if args.only == "step":
        state = d(wl.state0)
        xs = [d(wl.steps[args.step][n]) for n in I.NAMES]
        act = d(wl.active(args.step))
        fn = lambda: wkv7.step(*xs, state, act)
        units, per = int(wl.active(args.step).sum()) * wl.H, BYTES_DECODE
    else:
        xs = [d(wl.inputs[n]) for n in I.NAMES]
        reset = d(wl.reset) if wl.reset is not None else None
        # prefill: with a workspace (the split chunked form for few units) unless --no-workspace
        want_ws = args.only != "prefill" or not args.no_workspace
        y, s_out, ws = wkv7.forward(*xs, reset=reset, algo=args.algo, need_workspace=want_ws)
        units = wl.B * wl.T * wl.H
        if args.only in ("fwd", "prefill"):
            fn = lambda: wkv7.forward(*xs, reset=reset, y=y, s_out=s_out, workspace=ws, algo=args.algo,
                                      need_workspace=False)
            per = BYTES_FWD_TRAIN if args.only == "fwd" else BYTES_PREFILL
        else:
            dy = d(wl.dy)
            grads = {n: torch.empty_like(xs[0]) for n in ("dr", "dw", "dk", "dv", "da", "db")}
            fn = lambda: wkv7.backward(*xs, dy, ws, reset=reset, grads=grads, want_ds0=False, algo=args.algo)
            per = BYTES_BWD
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / max(args.steps, 1)
    peak, _ = measured_peaks()
    gbs = per * units / (ms / 1e3) / 1e9
    print(json.dumps({"only": args.only, "workload": wl.name, "B": wl.B, "algo": args.algo, "ms": ms,
                      "achieved_gbs": gbs, "frac": gbs / peak}))


if __name__ == "__main__":
    main()
