#!/usr/bin/env python
"""Benchmark of the block-diffusion attention hot path on B200.

One step = one bd_attn_fwd call on the training shape (B=4, Hq=32, Hkv=8,
L=2048 noisy + 2048 clean, b=32, d=128, keys x 0.5), the workload the
headline metric is quoted on.  ``value`` is TFLOP/s counting only unmasked
FLOPs, 4 d (L^2 + L b) B Hq per call, timed with CUDA events on the launching
stream, L2 flushed (256 MB write) before every step, inputs resident in HBM.
The same run also times the block-decode workloads (HBM GB/s of algorithmic
bytes) and the long-context block-size sweep, reported under ``rows``.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs the same per-GPU workload with no
data-path collective (weak scaling); the time is the max over ranks.
``--impl reference`` times the fp64 CPU oracle on the host cores instead
(rank 0 only), on a bounded row sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import bd_inputs  # noqa: E402

METRIC = ("BD-attn fwd TFLOP/s (unmasked FLOPs) & block-decode HBM GB/s, "
          "% of roofline")
L2_FLUSH_BYTES = 256 << 20
_flush_read = None


def flush_l2(flush, i):
    """Cold L2 for the next step: write a buffer twice the size of L2, then
    read a second one, so that the written (dirty) lines are written back to
    HBM here and not during the timed kernel."""
    global _flush_read
    flush.fill_(i & 0xff)
    if _flush_read is None or _flush_read.device != flush.device:
        _flush_read = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32,
                                 device=flush.device)
    torch.sum(_flush_read)
HOST_COVER_CYCLES = 400000  # ~0.2 ms GPU sleep queued before each timed step
# dram__bytes_read.sum + dram__bytes_write.sum of one launch of the dominant
# kernel, from the ncu captures summarised under profiles/
# (bd_tc_pair_kernel_fwd_training_shape.md: 201,509,376 read + 100,790,528
# written; bd_tc_persist_kernel_decode.md: 543,351,040 read + 7,544,064
# written by the denoising-decode attention kernel, whose combine launch
# moves no tile data in whole-unit mode).  Set back to None whenever the
# kernel changes after those counters were taken.
FWD_TRAFFIC_BYTES = 302299904
DECODE_TRAFFIC_BYTES = 550895104


def fwd_flops(s) -> int:
    return 4 * s.d * (s.L * s.L + s.L * s.b) * s.B * s.Hq


def decode_bytes(s, lens) -> int:
    kv = sum(s.Hkv * (int(n) + s.b) * s.d * 2 * 2 for n in lens)
    return kv + s.B * s.Hq * s.b * s.d * 2 * 2 + s.B * s.Hq * s.b * 4


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return (float(p["hbm_gbs"]), float(p["bf16_tflops"]),
                float(p["bf16_tflops_sustained"]), "measured")
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------------------
# clocks sampled during the timed region


class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.out = tempfile.TemporaryFile(mode="w+")
        self.windows = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx),
                 "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def mark(self, t0, t1):
        self.windows.append((t0, t1))

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except Exception:
            self.proc.kill()
        self.out.seek(0)
        rows = []
        for line in self.out:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0],
                                               "%Y/%m/%d %H:%M:%S"))
                rows.append((ts, float(parts[2]), float(parts[3]),
                             parts[6:10]))
            except Exception:
                continue
        inside = [r for r in rows
                  if any(a - 1 <= r[0] <= b + 1 for a, b in self.windows)]
        use = inside or rows
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = sorted({names[i] for r in use for i, v in enumerate(r[3])
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in use),
                "sm_max_mhz": max(r[2] for r in use), "reasons": reasons,
                "samples": len(use)}


# ---------------------------------------------------------------------------
# our arm


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d" % (n_gpus, world))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier_sync(world):
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The slowest rank's time: every rank runs its own replica of the
    workload, so the job finishes when the slowest one does."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job rate: all ranks' units over the slowest rank's time (per s)."""
    return world * units_per_rank / (max_ms * 1e-3)


def timed_steps(fn, steps, warmup, flush, world, sampler=None,
                cover_host=True):
    """Runs fn `warmup` times untimed, then `steps` times, each after an L2
    flush and a short GPU sleep that covers the host-side enqueue, timing each
    call with CUDA events on the current stream.  Returns the total device
    ms over the K steps, max over ranks."""
    st = torch.cuda.current_stream()
    for _ in range(warmup):
        flush_l2(flush, 1)
        fn()
    ev = [(torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier_sync(world)
    t0 = time.time()
    for i in range(steps):
        flush_l2(flush, i)
        # keep the GPU busy while the host enqueues the step, so that the
        # events bracket device time only (not host-side launch overhead)
        if cover_host:
            torch.cuda._sleep(HOST_COVER_CYCLES)
        ev[i][0].record(st)
        fn()
        ev[i][1].record(st)
    barrier_sync(world)
    t1 = time.time()
    if sampler is not None:
        sampler.mark(t0, t1)
    total = sum(a.elapsed_time(b) for a, b in ev)
    return max_over_ranks(total, world)


def run_e2e(bd, s, q, k, v, qd, kd, vd, out, lse, flush, world, steps):
    """The same call through the public API with host buffers: pinned-host
    -> device copies of q, k, v and device -> pinned-host copies of out and
    lse are inside the timed region of every step."""
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    outh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    lseh = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()

    def e2e_step():
        qd.copy_(qh, non_blocking=True)
        kd.copy_(kh, non_blocking=True)
        vd.copy_(vh, non_blocking=True)
        bd.fwd(qd, kd, vd, s.L, s.b, s.scale, out=out, lse=lse)
        outh.copy_(out, non_blocking=True)
        lseh.copy_(lse, non_blocking=True)

    # end to end: host-side launch overhead stays inside the timed region
    ms = timed_steps(e2e_step, steps, 3, flush, world, cover_host=False) / steps
    h2d = sum(t.numel() * t.element_size() for t in (q, k, v))
    d2h = out.numel() * out.element_size() + lse.numel() * lse.element_size()
    return {"value": round(world * fwd_flops(s) / (ms * 1e-3) / 1e12, 3),
            "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 4)}


def run_ours(args):
    import block_diffusion_lm_attn_b200 as bd
    world, rank, local = dist_setup(args.gpus)
    bd.load()
    hbm, tf_burst, tf_sus, peak_kind = peaks()
    dev = torch.device("cuda", local if world > 1 else 0)
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        gpu_id = str(torch.cuda.current_device())
    sampler = ClockSampler(gpu_id)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    sampler.start()
    only = args.only
    rows = {}
    n_launch = 0
    value = ms = fwd_kernel_tflops = None
    e2e = None
    s = bd_inputs.FWD_TRAIN

    # ---- headline: training shape, one bd_attn_fwd per step
    if only in ("all", "fwd"):
        q, k, v = bd_inputs.fwd_inputs_for(s)
        qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
        out = torch.empty_like(qd)
        lse = torch.empty((s.B, s.Hq, 2 * s.L), device=dev,
                          dtype=torch.float32)

        def step():
            bd.fwd(qd, kd, vd, s.L, s.b, s.scale, out=out, lse=lse)

        total_ms = timed_steps(step, args.steps, args.warmup, flush, world,
                               sampler)
        ms = total_ms / args.steps
        value = job_throughput(fwd_flops(s) * args.steps, world, total_ms) / 1e12
        fwd_kernel_tflops = fwd_flops(s) / (ms * 1e-3) / 1e12
        n_launch = args.steps  # one fwd kernel per step
        rows["fwd_train"] = {"tflops": round(fwd_kernel_tflops, 2),
                             "ms": round(ms, 4),
                             "frac_of_measured_bf16":
                                 round(fwd_kernel_tflops / tf_burst, 4)}
        if only == "all":
            e2e = run_e2e(bd, s, q, k, v, qd, kd, vd, out, lse, flush, world,
                          max(3, min(args.steps, 20)))
        del qd, kd, vd, out, lse

    # ---- long-context block-size sweep
    if only == "all" and not args.quick:
        for bb, sl in sorted(bd_inputs.FWD_LONG.items()):
            q, k, v = bd_inputs.fwd_inputs_for(sl)
            qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
            o = torch.empty_like(qd)
            ls = torch.empty((sl.B, sl.Hq, 2 * sl.L), device=dev,
                             dtype=torch.float32)
            n = max(5, args.steps // 10)
            t = timed_steps(lambda: bd.fwd(qd, kd, vd, sl.L, sl.b, sl.scale,
                                           out=o, lse=ls),
                            n, 3, flush, world, sampler) / n
            tf = fwd_flops(sl) / (t * 1e-3) / 1e12
            rows[sl.name] = {"tflops": round(tf, 2), "ms": round(t, 4),
                             "frac_of_measured_bf16": round(tf / tf_burst, 4)}
            del qd, kd, vd, o, ls

    # ---- block decode workloads (stream-K attention kernel + combine per call)
    dec_roof = None
    if only in ("all", "decode"):
        for sd in (bd_inputs.DEC_DENOISE, bd_inputs.DEC_VERIFY):
            q, kc, vc, cl = bd_inputs.decode_inputs_for(sd)
            qd, kcd, vcd, cld = q.to(dev), kc.to(dev), vc.to(dev), cl.to(dev)
            o = torch.empty_like(qd)
            ls = torch.empty((sd.B, sd.Hq, sd.b), device=dev,
                             dtype=torch.float32)
            nb = bd.workspace_bytes(sd.B, sd.Hq, sd.Hkv, sd.b, sd.d, sd.S_cap)
            ws = torch.empty(nb, dtype=torch.uint8, device=dev)
            n = max(5, args.steps // 5) if only == "all" else args.steps
            t = timed_steps(lambda: bd.decode(qd, kcd, vcd, cld, sd.mode,
                                              out=o, lse=ls, workspace=ws),
                            n, 3, flush, world, sampler) / n
            nbytes = decode_bytes(sd, cl.tolist())
            gbs = nbytes / (t * 1e-3) / 1e9
            rows[sd.name] = {"gbs": round(gbs, 1), "ms": round(t, 4),
                             "bytes": nbytes,
                             "frac_of_measured_hbm": round(gbs / hbm, 4),
                             "frac_of_8tbs": round(gbs / 8000.0, 4)}
            if sd is bd_inputs.DEC_DENOISE:
                dec_roof = {"bound": "hbm", "achieved": round(gbs, 1),
                            "peak": hbm, "unit": "GB/s",
                            "frac": round(gbs / hbm, 4),
                            "traffic": DECODE_TRAFFIC_BYTES,
                            "peak_source": peak_kind,
                            "kernels": "stream-K attention + combine"}
            del qd, kcd, vcd, o, ls, ws
    clocks = sampler.stop()

    result = None
    if rank == 0:
        result = {
            "metric": METRIC,
            "value": round(value, 3) if value is not None else None,
            "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 5) if ms is not None else None,
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16; keys x0.5)",
            "config": {"workload": "bd_attn_fwd training shape: B=4 Hq=32 "
                                   "Hkv=8 L=2048 noisy+2048 clean b=32 d=128",
                       "B": s.B, "Hq": s.Hq, "Hkv": s.Hkv, "L": s.L, "b": s.b,
                       "d": s.d, "seq_len": 2 * s.L,
                       "parallelism": "replicas" if world > 1 else "single",
                       "l2": "flushed before every step (256 MB write, then "
                             "256 MB read of another buffer)"},
            "roofline": None if fwd_kernel_tflops is None else {
                "bound": "tensor", "achieved": round(fwd_kernel_tflops, 2),
                "peak": tf_burst, "unit": "TFLOP/s",
                "frac": round(fwd_kernel_tflops / tf_burst, 4),
                "traffic": FWD_TRAFFIC_BYTES,
                "peak_source": peak_kind + " bf16 burst"},
            "roofline_decode": dec_roof,
            "e2e": e2e,
            "gpu_launches": n_launch,
            "clocks": clocks,
            "rows": rows,
        }
        if world == 1 and only == "all" and not args.no_cpu_baseline:
            result["cpu_baseline"] = cpu_baseline(s, budget_s=args.cpu_seconds)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if result is not None:
        print(json.dumps(result), flush=True)


# ---------------------------------------------------------------------------
# the oracle on the host cores


def row_flops(s, rows) -> int:
    """Unmasked FLOPs of the given flat query rows (4 d per visible key)."""
    n = 0
    for r in rows:
        r = r % (2 * s.L)
        kb = (r if r < s.L else r - s.L) // s.b
        n += (kb + 1) * s.b
    return 4 * s.d * n


def cpu_baseline(s, budget_s=15.0, rows_per_step=None, steps=1, warmup=0):
    import oracle
    q, k, v = bd_inputs.fwd_inputs_for(s)
    total = s.B * s.Hq * 2 * s.L
    if rows_per_step is None:
        probe = bd_inputs.sample_rows(total, 0, 64, seed=7)
        t0 = time.perf_counter()
        oracle.fwd(q, k, v, s.L, s.b, s.scale, rows=probe)
        dt = time.perf_counter() - t0
        rows_per_step = max(16, int(len(probe) * budget_s / max(dt, 1e-3)))
    rows = bd_inputs.sample_rows(total, 0, rows_per_step, seed=11)
    for _ in range(warmup):
        oracle.fwd(q, k, v, s.L, s.b, s.scale, rows=rows)
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle.fwd(q, k, v, s.L, s.b, s.scale, rows=rows)
    dt = (time.perf_counter() - t0) / steps
    fl = row_flops(s, rows)
    return {"value": round(fl / dt / 1e12, 6), "unit": "TFLOP/s",
            "cores": oracle.max_threads(), "kind": "oracle",
            "sample": "%d seeded query rows of the training shape (of %d), "
                      "fp64, %.2f s per pass" % (len(rows), total, dt),
            "seconds_per_step": dt}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    s = bd_inputs.FWD_TRAIN
    budget_total = 90.0
    per_step = budget_total / max(1, args.steps + args.warmup)
    cb = cpu_baseline(s, budget_s=per_step)
    rows_per_step = int(cb["sample"].split()[0])
    cb = cpu_baseline(s, rows_per_step=rows_per_step, steps=args.steps,
                      warmup=args.warmup)
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": cb["value"],
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(cb["seconds_per_step"] * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded N(0,1) bf16; keys x0.5)",
        "config": {"workload": "bd_attn_fwd training shape: B=4 Hq=32 Hkv=8 "
                               "L=2048 noisy+2048 clean b=32 d=128",
                   "B": s.B, "Hq": s.Hq, "Hkv": s.Hkv, "L": s.L, "b": s.b,
                   "d": s.d, "seq_len": 2 * s.L},
        "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "kind",
                                             "sample")},
        "e2e": {"value": cb["value"], "unit": "TFLOP/s",
                "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--quick", action="store_true",
                    help="skip the long-context sweep")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--only", choices=["all", "fwd", "decode"], default="all",
                    help="time only the training-shape fwd or only decode "
                         "(used for profiling captures)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
