"""Benchmark of the gated delta-rule hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One JSON line on rank 0.  A step is one gdn_chunk_fwd over the GDN-style
scalar-gated workload (B=4, H=16, T=2048, d_k=d_v=128, chunk 64, bf16 tokens,
fp32 state), inputs resident in HBM; `value` is whole-job tokens/s (all ranks;
weak scaling: every rank runs its own copy of the workload, no collective on
the data path).  The same line carries the decode half of the metric: the
recurrent decode step over 256 sequences x 32 heads (537 MB fp32 state updated
in place), timed over 128 consecutive steps, as GB/s and fraction of HBM.

`--impl reference` times the fp64 CPU oracle (the plain token recurrence) on
the host cores on the same workload and metric; it is the reference arm of
this benchmark, a deliberately slow program, not a target.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from gated_delta_rule_94_b200 import inputs as gi  # noqa: E402

METRIC = "gated-delta fwd tokens/s & TFLOP/s (% bf16 peak); decode GB/s (% HBM)"
C = 64
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def flops_per_token_head(Dk, Dv, chunk=C):
    """Algorithmic FLOPs of the chunk method per token and head: K K^T, Q K^T
    and T (beta K_bar) at 2 C d_k each; T (beta V) and P D at 2 C d_v each;
    W h, Q_bar h and K_tilde^T D at 2 d_k d_v each."""
    return 2 * chunk * (3 * Dk + 2 * Dv) + 6 * Dk * Dv


def chunk_bytes(w: gi.Workload, final_state=True):
    """Algorithmic HBM bytes of one chunk forward: every input and output
    token tensor once, the states once each way (when present)."""
    es = 2 if w.dtype == "bf16" else 4
    ntok = w.B * w.T * w.H
    per_tok = es * (2 * w.Dk + 2 * w.Dv + 1)
    if w.gate == "scalar":
        per_tok += es
    elif w.gate == "per_dim":
        per_tok += es * w.Dk
    state = w.B * w.H * w.Dk * w.Dv * 4
    return ntok * per_tok + (state if w.s0_std is not None else 0) + (state if final_state else 0)


def decode_bytes_per_step(w: gi.Workload):
    es = 2
    nh = w.B * w.H
    per = 2 * w.Dk * w.Dv * 4 + es * (2 * w.Dk + 2 * w.Dv + 1)
    per += es if w.gate == "scalar" else (es * w.Dk if w.gate == "per_dim" else 0)
    return nh * per


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured (MEASURED_PEAKS.json)"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback (earlier measurement on this pool)"


def ncu_traffic(kernel_name):
    """DRAM bytes per launch from the committed ncu capture, valid only while
    the kernel's source is unchanged since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel_name)
    except (OSError, ValueError):
        return None
    if not rec:
        return None
    src = os.path.join(ROOT, "gated_delta_rule_94_b200", "csrc", rec["source"])
    try:
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    except OSError:
        return None
    return rec["bytes_per_launch"] if sha == rec["source_sha256"] else None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML every ~10 ms."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int):
        self.samples = []
        self.load_window = []
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # noqa: BLE001 -- no NVML: report clocks as unavailable
            self.max_mhz = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.01)

    def start(self):
        if self.ok:
            self._t.start()

    def mark(self, t0, t1):
        self.load_window.append((t0, t1))

    def stop(self):
        self._stop.set()
        if self.ok:
            self._t.join(timeout=1)
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        loaded = [s for s in self.samples if any(a <= s[0] <= b for a, b in self.load_window)]
        use = loaded or self.samples
        reasons = sorted({name for _, _, rs in use for name, bit in self.REASONS.items() if rs & bit})
        return {"sm_mhz": statistics.median(m for _, m, _ in use) if use else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples_under_load": len(loaded)}


def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl" if torch.cuda.is_available() else "gloo",
                                             timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    """Maximum of a per-rank scalar (the slowest rank's time) over all ranks."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


# ----------------------------------------------------------------- CPU oracle
def oracle_tokens_per_s(w: gi.Workload, min_seconds: float, x=None):
    """The fp64 oracle on the host cores, over whole copies of the workload,
    repeated until at least min_seconds of CPU time has run."""
    import oracle
    oracle.build()
    if x is None:
        x = gi.workload_inputs(w)
    f = gi.to_f64_numpy(x)
    cores = len(os.sched_getaffinity(0))
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.recurrent(f["q"], f["k"], f["v"], f["beta"], f["g"], f["gate_kind"], f["S0"],
                         threads=cores)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    return w.B * w.T * reps / el, cores, reps, el


def run_reference(args, world, rank):
    if rank != 0:
        return
    w = gi.WORKLOADS[1]
    import oracle
    oracle.build()
    x = gi.workload_inputs(w)
    f = gi.to_f64_numpy(x)
    cores = len(os.sched_getaffinity(0))

    def step():
        oracle.recurrent(f["q"], f["k"], f["v"], f["beta"], f["g"], f["gate_kind"], f["S0"],
                         threads=cores)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    tok_s = w.B * w.T * args.steps / el
    F = flops_per_token_head(w.Dk, w.Dv) * w.B * w.T * w.H
    line = {
        "impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "Dk": w.Dk, "Dv": w.Dv,
                   "chunk": w.chunk, "gate": w.gate, "parallelism": "none (host threads)"},
        "algorithmic_tflops": F * args.steps / el / 1e12,
        "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"whole workload per step ({w.B * w.T * w.H} token-heads), "
                                   f"{args.steps} steps"},
        "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm
def run_ours(args, world, rank, local):
    import gated_delta_rule_94_b200 as gdn
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks, peak_src = load_peaks()
    w = gi.WORKLOADS[1]
    x = gi.workload_inputs(w)
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    B, T, H, Dk, Dv = w.B, w.T, w.H, w.Dk, w.Dv
    o = torch.empty((B, T, H, Dv), dtype=d["q"].dtype, device=dev)
    S = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    kname = gdn.gdn_chunk_fwd_kernel_name(Dk, Dv, d["gate_kind"], d["q"].dtype)
    nws = gdn.gdn_chunk_fwd_workspace_bytes(B, T, H, Dk, Dv, 64, d["q"].dtype, d["gate_kind"])
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev) if nws else None

    def step():
        gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], d["gate_kind"], d["S0"], o, S,
                          workspace=ws, stream=stream)

    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    sampler.start()
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    # ---- timed region: K chunk-forward steps, L2 flushed before each
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    n0 = gdn.gdn_kernel_launch_count()
    t_wall0 = time.perf_counter()
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    t_wall1 = time.perf_counter()
    launches = gdn.gdn_kernel_launch_count() - n0
    sampler.mark(t_wall0, t_wall1)
    per_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms = max_over_ranks(sum(per_ms) / len(per_ms), world)
    tokens = B * T * world
    value = tokens / (ms * 1e-3)
    N_th = B * T * H
    F = flops_per_token_head(Dk, Dv) * N_th
    tflops = F / (ms * 1e-3) / 1e12
    nbytes = chunk_bytes(w)
    achieved_gbs = nbytes / (ms * 1e-3) / 1e9

    # ---- decode: 128 consecutive steps over the 256 x 32 state, in place
    wd = gi.WORKLOADS[4]
    xd = gi.workload_inputs(wd)
    dd = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in xd.items()}
    state = dd["S0"].clone()
    steps_d = wd.T
    toks = [tuple(dd[n][:, t].contiguous() if dd[n] is not None else None
                  for n in ("q", "k", "v", "beta", "g")) for t in range(steps_d)]
    od = torch.empty((wd.B, wd.H, wd.Dv), dtype=dd["q"].dtype, device=dev)

    def decode_all():
        for (q, k, v, b_, g) in toks:
            gdn.gdn_decode_step(q, k, v, b_, g, dd["gate_kind"], state, od, stream=stream)
    for _ in range(max(1, args.warmup // 3)):
        decode_all()
    torch.cuda.synchronize()
    dec_ms = []
    barrier(world)
    td0 = time.perf_counter()
    for _ in range(args.steps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        decode_all()
        e1.record(stream)
        e1.synchronize()
        dec_ms.append(e0.elapsed_time(e1) / steps_d)
    td1 = time.perf_counter()
    sampler.mark(td0, td1)
    dec_step_ms = max_over_ranks(sum(dec_ms) / len(dec_ms), world)
    dec_bytes = decode_bytes_per_step(wd)
    dec_gbs = dec_bytes / (dec_step_ms * 1e-3) / 1e9

    # ---- end to end through the public API: pinned host -> device, compute,
    # device -> host of o and the final state, every step
    host = {k: (v.pin_memory() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    S_h = torch.empty(S.shape, dtype=S.dtype).pin_memory()
    names = ("q", "k", "v", "beta", "g")
    h2d = sum(host[n].numel() * host[n].element_size() for n in names if host[n] is not None)
    d2h = o.numel() * o.element_size() + S.numel() * S.element_size()

    def e2e_step():
        for n in names:
            if host[n] is not None:
                d[n].copy_(host[n], non_blocking=True)
        step()
        o_h.copy_(o, non_blocking=True)
        S_h.copy_(S, non_blocking=True)
    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    ee0 = torch.cuda.Event(enable_timing=True)
    ee1 = torch.cuda.Event(enable_timing=True)
    ee0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    ee1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(ee0.elapsed_time(ee1) / args.steps, world)
    clocks = sampler.stop()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tok_s, cores, reps, el = oracle_tokens_per_s(w, args.cpu_seconds, x=x)
        cpu = {"value": tok_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"whole workload ({N_th} token-heads) x {reps} repetitions, "
                         f"{el:.1f} s wall"}

    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if kname.startswith("chunk_prep_kernel") else "f32",
        "data": "synthetic",
        "config": {"workload": w.name, "B": B, "T": T, "H": H, "Dk": Dk, "Dv": Dv,
                   "chunk": w.chunk, "gate": w.gate, "initial_state": "zero (NULL)",
                   "final_state": "written", "parallelism": f"dp{world} (whole workload per rank)",
                   "l2": f"flushed before every step ({2 * l2 >> 20} MiB write)",
                   "kernel": kname},
        "tflops": tflops,
        "pct_bf16_peak": tflops / peaks["bf16_tflops"],
        "bf16_peak_tflops": peaks["bf16_tflops"],
        # the forward's kernels overlap one another (programmatic dependent
        # launch), so the unit timed and compared with the roofline is the
        # whole forward: its algorithmic bytes over the CUDA-event time of the
        # call; traffic is the DRAM bytes of all its launches (ncu)
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved_gbs / peaks["hbm_gbs"],
                     "traffic": ncu_traffic("chunk_fwd"), "algorithmic_bytes": nbytes,
                     "kernel": kname + " (one forward: all its launches)",
                     "peak_source": peak_src + ", hbm_gbs (copy bandwidth)"},
        "decode": {"workload": wd.name, "us_per_step": dec_step_ms * 1e3,
                   "gbs": dec_gbs, "pct_hbm": dec_gbs / peaks["hbm_gbs"],
                   "tokens_per_s": wd.B * world / (dec_step_ms * 1e-3),
                   "algorithmic_bytes_per_step": dec_bytes, "steps_timed": args.steps * steps_d,
                   "roofline": {"bound": "hbm", "achieved": dec_gbs, "peak": peaks["hbm_gbs"],
                                "unit": "GB/s", "frac": dec_gbs / peaks["hbm_gbs"],
                                "kernel": "decode_step_kernel",
                                "traffic": ncu_traffic("decode_step_kernel")}},
        "e2e": {"value": B * T * world / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": launches,
        "clocks": clocks,
        "cpu_baseline": cpu,
        "gpu": torch.cuda.get_device_name(dev),
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="minimum host time of the oracle CPU baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        # host-only arm: rank 0 runs it, other ranks exit without work
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")),
                      int(os.environ.get("RANK", "0")))
        return
    world, rank, local = dist_init()
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
