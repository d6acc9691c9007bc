"""Benchmark: ReplaySSM decode of a Mamba-2 layer at serving shape.

Workload (one GPU): batch 256, 80 heads, headdim 64, dstate 128, 1 group, bf16
inputs, fp32 master checkpoint + bf16 output copy, commit interval K = 8, the
checkpoint seeded by a 512-token eager prefill.  A step is one pass of the
decode path over the batch: append the step's inputs to the ring, compute the
outputs by output-only replay, and commit every 8th step.  The checkpoint
(335 MB bf16 + 671 MB fp32) is larger than L2, so no flush is needed between
steps.

Prints one JSON line.  `--impl reference` times the fp64 CPU oracle instead
(the reference arm: there is no runnable reference implementation).

`--k-sweep` (one GPU) measures the commit-interval trade-off instead: for
K = 4, 8, 16, 32 (ring capacity K) the same decode steps with the whole batch
committing every K-th step, and with staggered commits (sequence b commits at
the steps i with i = b mod K, through the commit mask), one JSON line per K
with throughput, per-step time percentiles and state bytes per token.
"""
import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

B, H, P, N, G, K_COMMIT, CAP, PREFILL = 256, 80, 64, 128, 1, 8, 8, 512
# Each decode step buffers one entry and every K_COMMIT-th step commits them
# all, so the ring never holds more than K_COMMIT entries: CAP = K_COMMIT.
POOL = 256          # distinct decode steps of inputs kept resident (cycled)
METRIC = "SSM-layer decode tokens/s at batch 256; achieved HBM GB/s vs B200 peak"
UNIT = "tokens/s"
WORKLOAD = "mamba2-decode-b256-h80-p64-n128-bf16copy-K8"
# DRAM bytes (read + write) of one streaming-kernel launch on this workload,
# from an ncu capture of the current kernel; None when the kernel has changed
# since the last capture.  The last one (359,565,056 read + 3,879,680 written,
# profiles/stream_outputs_mamba2_*.md) predates the consumer-team change.
TRAFFIC = None


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4096)
    ap.add_argument("--warmup", type=int, default=16)
    ap.add_argument("--impl", default="rs", choices=["rs", "reference"])
    ap.add_argument("--prefill", type=int, default=PREFILL)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-work", type=float, default=20.0)
    ap.add_argument("--k-sweep", action="store_true")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ------------------------------------------------------------- clocks ------

class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons while the
    timed region runs, with `nvidia-smi -lms` in a child process (a Python
    thread would hardly run while the main thread issues launches).  The
    first sample is awaited before the region starts."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, index=0, period_ms=20):
        self.index, self.period_ms = index, period_ms
        self.rows, self.max_mhz, self.proc = [], None, None

    def __enter__(self):
        import shutil
        import subprocess
        exe = shutil.which("nvidia-smi")
        if exe is None:
            return self
        self.proc = subprocess.Popen(
            [exe, f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
             f"-lms={self.period_ms}"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        self._reader = threading.Thread(target=self._read, daemon=True)
        self._reader.start()
        t0 = time.time()
        while not self.rows and time.time() - t0 < 10 and self.proc.poll() is None:
            time.sleep(0.005)
        self.rows.clear()   # samples from here on fall in the timed region
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) == 9:
                self.rows.append(parts)

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(2 * self.period_ms / 1000)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        mhz, reasons = [], set()
        for r in list(self.rows):
            try:
                mhz.append(float(r[1]))
                self.max_mhz = float(r[2])
            except ValueError:
                continue
            for name, flag in zip(self.NAMES, r[5:9]):
                if flag.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(mhz)}


# ------------------------------------------------------------ CPU oracle ---

class OracleSample:
    """A bounded sample of the workload for the fp64 CPU oracle: nseq
    sequences x all heads, T decode steps per call, state carried across calls."""

    def __init__(self, nseq, T, seed):
        import numpy as np
        rng = np.random.default_rng(seed)
        n = nseq * H
        self.nseq, self.T = nseq, T
        self.A = -np.exp(rng.uniform(0, math.log(16), n))
        self.D = rng.standard_normal(n)
        self.x = rng.standard_normal((n, T, P))
        self.dt = np.log1p(np.exp(rng.standard_normal((n, T)) * 0.5 - 3.0))
        self.B = rng.standard_normal((n, T, N)) / math.sqrt(N)
        self.C = rng.standard_normal((n, T, N)) / math.sqrt(N)
        self.h = rng.standard_normal((n, P, N)) * 0.1

    def run(self, cores):
        import oracle
        t0 = time.perf_counter()
        oracle.mamba2_eager_batch(self.A, self.D, self.x, self.dt, self.B, self.C, h=self.h,
                                  nthreads=cores)
        return time.perf_counter() - t0


def cpu_oracle_rate(cpu_work_s, nseq=32, T=8, seed=0):
    """Times the oracle on about `cpu_work_s` seconds of CPU work (wall time x
    threads).  Returns (tokens/s, threads, sample text)."""
    cores = os.cpu_count() or 1
    s = OracleSample(nseq, T, seed)
    s.run(cores)                                   # warm the pages
    target = max(0.5, cpu_work_s / cores)
    el, reps = 0.0, 0
    while el < target:
        el += s.run(cores)
        reps += 1
    return nseq * T * reps / el, cores, (
        f"{reps} x ({nseq} sequences x {H} heads x {T} decode steps) of the fp64 eager "
        f"recurrence ({P}x{N} state per head), {el:.2f} s wall on {cores} threads")


def reference_arm(args, rank):
    if rank != 0:
        return
    cores = os.cpu_count() or 1
    # each step: nseq sequences x all heads x 8 decode steps, nseq sized (<= 32)
    # so that the whole warm-up + timed run takes about 90 s of wall time
    probe = OracleSample(32, 8, 0)
    probe.run(cores)
    t32 = probe.run(cores)
    nseq = int(max(1, min(32, 32 * 90.0 / max((args.steps + args.warmup) * t32, 1e-9))))
    s = OracleSample(nseq, 8, 0)
    for _ in range(args.warmup):
        s.run(cores)
    el = sum(s.run(cores) for _ in range(args.steps))
    value = s.nseq * s.T * args.steps / el
    sample = (f"per step {s.nseq} sequences x {H} heads x {s.T} decode steps of the fp64 eager "
              f"recurrence; {args.steps} timed steps, {el:.2f} s wall on {cores} threads")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * B / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD, "global_batch": B,
                                            "parallelism": "none (CPU oracle)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------- rank helpers ----
# One process per GPU; every rank decodes its own batch of sequences (weak
# scaling).  The only cross-rank operations are the timing barrier and the
# maximum of the ranks' device times.

def rank_seed(rank):
    """Seed of rank `rank`'s synthetic inputs (distinct sequences per rank)."""
    return 1 + 1000 * rank


def max_over_ranks(x, world, device):
    """Maximum of a per-rank float over all ranks (the job's time)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world, batch_per_rank, steps, ms):
    """Whole-job throughput: all ranks' tokens over the slowest rank's time."""
    return world * batch_per_rank * steps / (ms * 1e-3)


# ------------------------------------------------------------- GPU arm -----

def gpu_arm(args, rank, world):
    import torch
    import torch.distributed as dist

    import rs_decode_outputs_b200 as rs
    from rs_decode_outputs_b200 import inputs as gen

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    seed = rank_seed(rank)

    A, D, dtb = gen.mamba2_params(H, seed, dev)
    src = gen.Mamba2Stream(B, H, P, N, G, torch.bfloat16, dtb, seed + 10_000, dev)
    cfg = rs.make_config(rs.RS_MAMBA2, B, H, P, N, G, cap=CAP, npos_max=1, in_dtype=rs.RS_BF16,
                         copy_dtype=rs.RS_BF16, out_dtype=rs.RS_BF16)
    sess = rs.ReplaySSM(cfg, A=A, D=D, device=dev)

    # prefill: eager fp32 steps on a state tensor, then load it as the checkpoint
    state = torch.zeros(B, H, P, N, device=dev)
    ypre = torch.empty(1, B, H, P, device=dev, dtype=torch.bfloat16)
    left = args.prefill
    while left > 0:
        n = min(64, left)
        chunk = src.next(n)
        for t in range(n):
            sess.eager_step(state, rs.RS_F32, {k: v[t:t + 1] for k, v in chunk.items()}, 1, ypre)
        left -= n
    sess.load_checkpoint(state)
    del state

    pool = src.next(POOL)
    steps_in = [{k: v[t:t + 1] for k, v in pool.items()} for t in range(POOL)]
    y = sess.new_out()
    h = sess.handle

    ins = [rs.make_inputs(d) for d in steps_in]

    def step(i, ev=None):
        # one decode step: append this token's inputs and replay the outputs
        # (prep kernel + streaming kernel), then commit every K_COMMIT steps
        rs.rs_decode_step(h, ins[i % POOL], 1, y)
        if (i + 1) % K_COMMIT == 0:
            if ev is not None:
                ev[0].record(stream)
            rs.rs_commit(h, K_COMMIT)
            if ev is not None:
                ev[1].record(stream)

    i = 0
    for _ in range(args.warmup):
        step(i)
        i += 1
    # align the timed region to commit boundaries so every K-th step commits
    while i % K_COMMIT:
        step(i)
        i += 1

    # pass 1: whole-step throughput (no per-kernel events)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    n0 = rs.rs_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            step(i)
            i += 1
        e1.record(stream)
        torch.cuda.synchronize()
    launches = rs.rs_launch_count() - n0
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    if world > 1:
        dist.barrier()

    # pass 2: per-kernel durations for the roofline (the library's own events
    # around its prep and streaming launches; events around each commit)
    nk = min(args.steps, 512)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(nk)]
    torch.cuda.synchronize()
    rs.rs_profile_start(h, nk)
    com_idx = []
    for j in range(nk):
        if (i + 1) % K_COMMIT == 0:
            com_idx.append(j)
        step(i, evs[j])
        i += 1
    torch.cuda.synchronize()
    ncalls, prep_total, stream_total = rs.rs_profile_stop(h)
    prep_ms = prep_total / ncalls
    stream_ms = stream_total / ncalls
    com_ms = [evs[j][0].elapsed_time(evs[j][1]) for j in com_idx]

    # eager read-modify-write baseline on the same shape (fp32 state and bf16 state)
    eager = {}
    for name, sdt, tdt, ebytes in (("fp32", rs.RS_F32, torch.float32, 4), ("bf16", rs.RS_BF16, torch.bfloat16, 2)):
        st = torch.zeros(B, H, P, N, device=dev, dtype=tdt)
        ye = torch.empty(1, B, H, P, device=dev, dtype=torch.bfloat16)
        for j in range(8):
            sess.eager_step(st, sdt, steps_in[j], 1, ye)
        ne = min(args.steps, 256)
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for j in range(ne):
            rs.rs_eager_step(h, st, sdt, rs.make_inputs(steps_in[j % POOL]), 1, ye)
        a1.record(stream)
        torch.cuda.synchronize()
        ems = a0.elapsed_time(a1) / ne
        eager[name] = {"tokens_per_s": B / (ems * 1e-3), "ms_per_step": ems,
                       "state_bytes_per_token": 2 * ebytes * H * P * N,
                       "achieved_gbs": 2 * ebytes * B * H * P * N / (ems * 1e-3) / 1e9}
        del st

    # end to end through rs_decode_step: every step copies its inputs from
    # pinned host memory and reads its outputs back.  The copies run on their
    # own streams with two device buffers each way, so step j's transfers
    # overlap the computation of its neighbours (the pipelining a serving
    # loop would use); events order buffer reuse.
    ne2e = min(args.steps, 512)
    nh = 16   # distinct pinned input sets, cycled
    host_in = [{k: v.cpu().pin_memory() for k, v in steps_in[j].items()} for j in range(nh)]
    dev_in = [{k: torch.empty_like(v) for k, v in steps_in[0].items()} for _ in range(2)]
    dev_ins = [rs.make_inputs(d) for d in dev_in]
    y_dev = [sess.new_out() for _ in range(2)]
    y_host = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of buffer k are on the device
    ev_used = [torch.cuda.Event() for _ in range(2)]   # step done with buffer k (inputs read, outputs written)
    ev_out = [torch.cuda.Event() for _ in range(2)]    # outputs of buffer k are on the host
    h2d = sum(v.numel() * v.element_size() for v in host_in[0].values())
    d2h = y.numel() * y.element_size()
    torch.cuda.synchronize()
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b0.record(s_in)
    for j in range(ne2e):
        k = j % 2
        if j >= 2:
            s_in.wait_event(ev_used[k])
        with torch.cuda.stream(s_in):
            for name, v in host_in[j % nh].items():
                dev_in[k][name].copy_(v, non_blocking=True)
        ev_in[k].record(s_in)
        stream.wait_event(ev_in[k])
        if j >= 2:
            stream.wait_event(ev_out[k])
        rs.rs_decode_step(h, dev_ins[k], 1, y_dev[k], stream)
        ev_used[k].record(stream)
        if (i + 1) % K_COMMIT == 0:
            rs.rs_commit(h, K_COMMIT, stream=stream)
        i += 1
        s_out.wait_event(ev_used[k])
        with torch.cuda.stream(s_out):
            y_host[k].copy_(y_dev[k], non_blocking=True)
        ev_out[k].record(s_out)
    b1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(b0.elapsed_time(b1) / ne2e, world, dev)

    status, flags = sess.get_error()
    if status != rs.RS_OK:
        raise RuntimeError(f"device error flags set: {set(flags.tolist())}")

    if rank != 0:
        return
    hbm, peak_kind = peaks()
    copy_bytes = B * H * P * N * 2
    y_bytes = B * H * P * 2
    achieved = (copy_bytes + y_bytes) / (stream_ms * 1e-3) / 1e9
    com_avg = statistics.mean(com_ms) if com_ms else float("nan")
    commit_bytes = B * H * P * N * (4 + 4 + 2)
    step_ms = ms / args.steps
    value = job_tokens_per_s(world, B, args.steps, ms)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; Mamba-2 serving-shape distributions)",
        "config": {"workload": WORKLOAD, "global_batch": B * world, "batch_per_gpu": B,
                   "nheads": H, "headdim": P, "dstate": N, "ngroups": G, "commit_interval": K_COMMIT,
                   "ring_cap": CAP, "prefill_tokens": args.prefill, "checkpoint": "fp32 master + bf16 copy",
                   "parallelism": f"dp{world} (independent sequences per GPU, no collective)",
                   "l2": "inputs larger than L2 (checkpoint copy 335 MB per step), no flush"},
        "roofline": {"bound": "hbm", "kernel": "stream_outputs_kernel (output-only replay, Mamba-2)",
                     "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": TRAFFIC, "peak_source": peak_kind,
                     "algorithmic_bytes_per_launch": copy_bytes + y_bytes,
                     "avg_launch_us": stream_ms * 1e3},
        "kernels": {"prep_us": prep_ms * 1e3, "stream_us": stream_ms * 1e3,
                    "decode_us": (prep_ms + stream_ms) * 1e3, "commit_us": com_avg * 1e3,
                    "commit_gbs": commit_bytes / (com_avg * 1e-3) / 1e9 if com_ms else None,
                    "step_state_bytes_per_token": H * P * N * (2 + 10 / K_COMMIT),
                    "step_achieved_gbs": B * H * P * N * (2 + 10 / K_COMMIT) / (step_ms * 1e-3) / 1e9},
        "eager": eager,
        "e2e": {"value": job_tokens_per_s(world, B, 1, e2e_ms), "unit": UNIT, "pipeline": "H2D, decode step, D2H on three streams, two buffers each way", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": launches,
        "clocks": clk.summary(),
    }
    if not args.no_cpu_baseline:
        v, cores, sample = cpu_oracle_rate(args.cpu_work)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": sample}
    print(json.dumps(line), flush=True)


# ------------------------------------------------ commit-interval sweep ----

def k_sweep(args):
    """Replay cost against checkpoint traffic as K varies.  A larger K moves
    fewer checkpoint bytes per token (10 / K B per state element for the
    commit) but buffers more entries: the prep reduces up to K entries per
    head and the streaming pass stages each tile's whole ring block
    (cap x P x 2 B).  Synchronous commits make every K-th step long;
    staggered ones spread the same work over all steps."""
    import torch

    import rs_decode_outputs_b200 as rs
    from rs_decode_outputs_b200 import inputs as gen

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    A, D, dtb = gen.mamba2_params(H, 1, dev)
    src = gen.Mamba2Stream(B, H, P, N, G, torch.bfloat16, dtb, 10_001, dev)
    pool = src.next(64)
    steps_in = [rs.make_inputs({k: v[t:t + 1] for k, v in pool.items()}) for t in range(64)]
    nsteps = max(256, args.steps // 8)
    for K in (4, 8, 16, 32):
        cfg = rs.make_config(rs.RS_MAMBA2, B, H, P, N, G, cap=K, npos_max=1, in_dtype=rs.RS_BF16,
                             copy_dtype=rs.RS_BF16, out_dtype=rs.RS_BF16)
        sess = rs.ReplaySSM(cfg, A=A, D=D, device=dev)
        g = torch.Generator(device=dev).manual_seed(K)
        sess.load_checkpoint(0.1 * torch.randn(B, H, P, N, device=dev, generator=g))
        h, y = sess.handle, sess.new_out()
        masks = [(torch.arange(B, device=dev) % K == ph).to(torch.int32) for ph in range(K)]
        res = {}
        for mode in ("sync", "staggered"):
            def step(i):
                rs.rs_decode_step(h, steps_in[i % 64], 1, y)
                if mode == "sync" and (i + 1) % K == 0:
                    rs.rs_commit(h, K)
                elif mode == "staggered":
                    rs.rs_commit(h, 1, masks[i % K])
            i = 0
            for _ in range(4 * K):   # warm-up; staggered lengths settle within K steps
                step(i)
                i += 1
            while i % K:
                step(i)
                i += 1
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(nsteps + 1)]
            torch.cuda.synchronize()
            ev[0].record(stream)
            for j in range(nsteps):
                step(i)
                i += 1
                ev[j + 1].record(stream)
            torch.cuda.synchronize()
            per = sorted(ev[j].elapsed_time(ev[j + 1]) * 1e3 for j in range(nsteps))
            total_us = ev[0].elapsed_time(ev[nsteps]) * 1e3
            res[mode] = {"tokens_per_s": B * nsteps / (total_us * 1e-6), "us_per_step": total_us / nsteps,
                         "p50_us": per[nsteps // 2], "p99_us": per[min(nsteps - 1, int(0.99 * nsteps))],
                         "max_us": per[-1]}
        status, flags = sess.get_error()
        if status != rs.RS_OK:
            raise RuntimeError(f"device error flags set at K={K}: {set(flags.tolist())}")
        line = {"k_sweep": True, "workload": WORKLOAD.replace("K8", f"K{K}"), "commit_interval": K, "ring_cap": K,
                "steps": nsteps, "state_bytes_per_token": H * P * N * (2 + 10 / K),
                "ring_block_bytes_per_tile": K * P * 2, **res}
        print(json.dumps(line), flush=True)
        del sess
        torch.cuda.empty_cache()


def main():
    args = parse()
    if args.k_sweep:
        k_sweep(args)
        return
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        reference_arm(args, rank)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        gpu_arm(args, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
