"""Benchmark: verified seq-steps/s and achieved HBM GB/s of spec_verify on B200.

One step = one spec_verify call (every kernel of the path) over one batch of the
workload "c3": B=64 sequences, gamma=5, V=128256, bf16 logits (Zipf-biased
N(0,3^2) target, rho=0.9 draft, T=1).  Inputs are resident in HBM before the
timed region; calls rotate over several copies of the batch so that every call
reads logits last touched > 2x L2 (126 MB) earlier.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank verifies its own batch (sequences are
independent: no collective on the data path); value = all ranks' sequences /
the slowest rank's time.  ``--impl reference`` times the fp64 CPU oracle (the
only reference on hand) on the host cores on the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "verified seq-steps/sec and achieved HBM GB/s (% of B200 peak) for spec_verify"
WORKLOAD = "c3"
WORKLOAD_DESC = ("spec_verify B=64, gamma=5, V=128256, bf16 logits; target N(0,3^2)+Zipf(1.1) log-bias, "
                 "draft rho=0.9, T=1.0 (synthetic, seed 86)")
FALLBACK_HBM_GBS = 6650.0


def algorithmic_bytes(B, gamma, V, esz):
    """Logits read once + small inputs + outputs, per call (per the path's definition)."""
    logits = (2 * gamma + 1) * V * esz * B
    small_in = (gamma + gamma + 1 + 1) * 4 * B          # tokens, u_accept, u_resample, T
    outs = (gamma + 1 + 1) * 4 * B                      # out_tokens, n_accepted
    return logits + small_in + outs


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling in the background during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            p = [x.strip() for x in line.split(",")]
            if len(p) >= 9:
                rows.append(p)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def job_value(local_ms, world, per_rank_units, pg=None, device=None):
    """Whole-job throughput (units per second) and the job's time in ms.

    Every rank processed its own per_rank_units; the job took as long as its
    slowest rank, so the time is the max over ranks (an all-reduce over pg when
    there is more than one rank)."""
    total_ms = float(local_ms)
    if pg is not None:
        import torch
        t = torch.tensor([total_ms], dtype=torch.float64, device=device)
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
        total_ms = float(t.item())
    return world * per_rank_units / (total_ms / 1e3), total_ms


def oracle_time(w, min_seconds, n_threads=0):
    """Time the oracle on the batch, repeated until min_seconds of CPU work; seq-steps/s."""
    import oracle
    oracle.build()
    cores = n_threads or oracle.max_threads()
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.verify_workload(w, n_threads=n_threads)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    return reps * w.B / el, cores, reps, el


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    from speculative_decoding_verification_84_b200 import workloads as W
    w = W.make_workload(WORKLOAD)
    import oracle
    oracle.build()
    cores = oracle.max_threads()
    for _ in range(args.warmup):
        oracle.verify_workload(w)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.verify_workload(w)
    el = time.perf_counter() - t0
    val = args.steps * w.B / el
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "seq-steps/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD_DESC},
        "cpu_baseline": {"value": val, "unit": "seq-steps/s", "cores": cores, "kind": "oracle",
                         "sample": f"the full c3 batch ({w.B} sequences) per step, fp64 C oracle, OpenMP"},
        "e2e": {"value": val, "unit": "seq-steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        pg = dist

    from speculative_decoding_verification_84_b200 import binding, build, workloads as W
    build.build()
    lib = binding.load_library()

    w = W.make_workload(WORKLOAD)
    B, gamma, V = w.B, w.gamma, w.V
    esz = 2 if w.dtype == "bf16" else 4
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    base = binding.to_device(w, dev)
    l2_bytes = 126 * 2 ** 20
    n_copies = max(3, int(np.ceil(2 * l2_bytes / w.logits_bytes())) + 1)
    sets = [base] + [{k: v.clone() for k, v in base.items()} for _ in range(n_copies - 1)]
    out_t = torch.empty((B, gamma + 1), dtype=torch.int32, device=dev)
    out_n = torch.empty((B,), dtype=torch.int32, device=dev)
    wsz = binding.workspace_size(B, gamma, V, tdt)
    wspace = torch.zeros(wsz, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    dt_code = binding._dt_code(tdt)
    kernels_per_call = binding.kernels_per_call(B, gamma, V, tdt)
    rowbytes = V * esz
    kernel_name = ("sv_stream + sv_draw (one call; sv_stream reads every logit once)"
                   if rowbytes % 16 == 0 and rowbytes >= 4096 else "sv_reset + sv_rowpass + sv_resample (one call)")

    def call(d):
        st = lib.spec_verify(d["target"].data_ptr(), d["draft"].data_ptr(), dt_code, d["draft_tokens"].data_ptr(),
                             d["temperature"].data_ptr(), d["u_accept"].data_ptr(), d["u_resample"].data_ptr(),
                             out_t.data_ptr(), out_n.data_ptr(), B, gamma, V, wspace.data_ptr(), wsz, None, None,
                             stream.cuda_stream)
        if st != 0:
            raise RuntimeError(binding.status_string(st))

    def barrier():
        if pg is not None:
            pg.barrier()

    for i in range(max(3, args.warmup)):
        call(sets[i % n_copies])
    torch.cuda.synchronize()

    # timed region: K back-to-back calls bracketed by two events on the launching
    # stream (an event between calls would add its own gap to every call)
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    sampler.start()
    barrier()
    torch.cuda.synchronize()
    e_start.record(stream)
    for i in range(args.steps):
        call(sets[i % n_copies])
    e_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    local_ms = e_start.elapsed_time(e_end)
    value, total_ms = job_value(local_ms, ws, B * args.steps, pg, dev)
    ms_per_step = total_ms / args.steps

    # spread of single calls, from a separate untimed sample with an event pair
    # around each call
    n_spread = min(args.steps, 200)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * n_spread)]
    for i in range(n_spread):
        ev[2 * i].record(stream)
        call(sets[i % n_copies])
        ev[2 * i + 1].record(stream)
    torch.cuda.synchronize()
    per_call = [ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(n_spread)]

    alg = algorithmic_bytes(B, gamma, V, esz)
    mean_call_ms = local_ms / args.steps  # this rank's mean call over the timed region
    achieved = alg / (mean_call_ms / 1e3) / 1e9
    peak, peak_kind = peaks()

    # end to end through the public API: pinned host inputs -> device, call, outputs -> host
    host = {}
    for k, v in base.items():
        h = torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
        h.copy_(v)
        host[k] = h
    h_out_t = torch.empty((B, gamma + 1), dtype=torch.int32, pin_memory=True)
    h_out_n = torch.empty((B,), dtype=torch.int32, pin_memory=True)
    dbuf = {k: torch.empty_like(v) for k, v in base.items()}
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = h_out_t.numel() * 4 + h_out_n.numel() * 4
    e2e_steps = max(3, min(args.steps, 50))

    def e2e_step():
        for k in dbuf:
            dbuf[k].copy_(host[k], non_blocking=True)
        call(dbuf)
        h_out_t.copy_(out_t, non_blocking=True)
        h_out_n.copy_(out_n, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_value, _ = job_value(e0.elapsed_time(e1), ws, B * e2e_steps, pg, dev)

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        val, cores, reps, el = oracle_time(w, args.cpu_seconds)
        cpu = {"value": val, "unit": "seq-steps/s", "cores": cores, "kind": "oracle",
               "sample": f"{reps} passes over the full c3 batch ({w.B} sequences), {el:.1f} s, fp64 C oracle"}

    traffic = None
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tpath):
        try:
            traffic = json.load(open(tpath)).get(WORKLOAD)
        except Exception:
            traffic = None

    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": "seq-steps/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD_DESC, "global_batch": ws * B, "gamma": gamma, "V": V,
                   "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU",
                   "l2": f"inputs rotate over {n_copies} resident copies ({n_copies * w.logits_bytes() / 1e6:.0f} MB > 2x L2)"},
        "hbm_gbs": achieved, "pct_of_peak": 100.0 * achieved / peak,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "peak_source": f"{peak_kind} hbm_gbs",
                     "kernel": kernel_name,
                     "algorithmic_bytes_per_launch": alg, "mean_launch_us": 1e3 * mean_call_ms,
                     "single_call_p10_us": 1e3 * float(np.percentile(per_call, 10)),
                     "single_call_p90_us": 1e3 * float(np.percentile(per_call, 90))},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "seq-steps/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps},
        "gpu_launches": kernels_per_call * args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.impl == "reference":
        if args.steps > 200:
            args.steps = 20
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
