"""Benchmark of the gated delta-rule hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One JSON line on rank 0.  A step is one gdn_chunk_fwd over a whole workload,
inputs resident in HBM, L2 flushed before every step.  The headline is the
largest single-GPU workload, the long-sequence scalar-gated forward (B=1,
H=32, T=65536, d_k=d_v=128, chunk 64, bf16 tokens, fp32 state); `value` is
its whole-job tokens/s.  The same line carries one record per other forward
workload (GDN B4 H16 T2048; per-dimension gate B4 H16 T4096; fp32 B1 H2 T256
d64) and the decode step (256 sequences x 32 heads, 537 MB fp32 state updated
in place, 128 consecutive steps), each with its own roofline, end-to-end
figure and CPU baseline.

With N ranks (one per GPU) the heads of every workload are split across the
ranks, no collective on the data path: total work is fixed (strong scaling).

`--impl reference` times the fp64 CPU oracle (the plain token recurrence) on
the host cores on a bounded sample of the headline workload, reported in the
same unit; it is the reference arm of this benchmark, a deliberately slow
program, not a target.
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

import torch  # noqa: E402

from gated_delta_rule_94_b200 import inputs as gi  # noqa: E402

METRIC = "gated-delta fwd tokens/s & TFLOP/s (% bf16 peak); decode GB/s (% HBM)"
C = 64
HEADLINE = 3                      # long-sequence GDN forward, the largest single-GPU workload
SUBRECORDS = (1, 2, 0)            # the other forward workloads
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# fp32 FMA peak of the CUDA-core path: 148 SMs x 128 fp32 lanes x 2 flop x 1.965 GHz
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def flops_per_token_head(Dk, Dv, chunk=C):
    """Algorithmic FLOPs of the chunk method per token and head: K K^T, Q K^T
    and T (beta K_bar) at 2 C d_k each; T (beta V) and P D at 2 C d_v each;
    W h, Q_bar h and K_tilde^T D at 2 d_k d_v each."""
    return 2 * chunk * (3 * Dk + 2 * Dv) + 6 * Dk * Dv


def chunk_bytes(w: gi.Workload, H: int | None = None, final_state=True):
    """Algorithmic HBM bytes of one chunk forward over H heads (default: all):
    every input and output token tensor once, the states once each way (when
    present)."""
    H = w.H if H is None else H
    es = 2 if w.dtype == "bf16" else 4
    ntok = w.B * w.T * H
    per_tok = es * (2 * w.Dk + 2 * w.Dv + 1)
    if w.gate == "scalar":
        per_tok += es
    elif w.gate == "per_dim":
        per_tok += es * w.Dk
    state = w.B * H * w.Dk * w.Dv * 4
    return ntok * per_tok + (state if w.s0_std is not None else 0) + (state if final_state else 0)


def decode_bytes_per_step(w: gi.Workload, H: int | None = None):
    H = w.H if H is None else H
    es = 2
    nh = w.B * H
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


def ncu_traffic(key):
    """DRAM bytes per forward (or launch) from the committed ncu capture,
    valid only while every source file it names is unchanged since."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(key)
    except (OSError, ValueError):
        return None
    if not rec:
        return None
    for src, want in rec["sources"].items():
        try:
            sha = hashlib.sha256(open(os.path.join(ROOT, src), "rb").read()).hexdigest()
        except OSError:
            return None
        if sha != want:
            return None
    return rec["bytes_per_launch"]


def shard_heads(H: int, world: int, rank: int) -> tuple[int, int]:
    """Heads [h0, h1) of rank `rank` when H heads are split over `world` ranks:
    contiguous, disjoint, covering all heads; sizes differ by at most one."""
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


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
def oracle_sample(w: gi.Workload, seconds: float):
    """The fp64 oracle on the host cores over a bounded sample of workload w:
    min(H, cores) heads of the first B=1 sequence, the sequence cut to the
    length that takes about `seconds`.  Returns (token-heads/s, cores, text)."""
    import oracle
    oracle.build()
    cores = len(os.sched_getaffinity(0))
    H = min(w.H, cores)
    T = min(w.T, 512)
    while True:   # grow the sample until one run takes a tenth of the budget
        x = gi.workload_inputs(w, B=1, T=T, H=H)
        f = gi.to_f64_numpy(x)
        t0 = time.perf_counter()
        oracle.recurrent(f["q"], f["k"], f["v"], f["beta"], f["g"], f["gate_kind"], f["S0"],
                         threads=cores)
        el = time.perf_counter() - t0
        if el >= seconds / 10 or T >= w.T:
            break
        T = min(w.T, T * 4)
    reps, total = 1, el
    while total < seconds:
        t0 = time.perf_counter()
        oracle.recurrent(f["q"], f["k"], f["v"], f["beta"], f["g"], f["gate_kind"], f["S0"],
                         threads=cores)
        total += time.perf_counter() - t0
        reps += 1
    rate = H * T * reps / total
    return rate, cores, f"{H} heads x {T} tokens of one sequence, {reps} runs, {total:.1f} s"


def oracle_decode_sample(w: gi.Workload, seconds: float):
    """The oracle's decode: min(cores, N) sequences x H heads, one token step
    from the workload's initial state, repeated for about `seconds`.
    Returns (token-heads/s, cores, text)."""
    import oracle
    oracle.build()
    cores = len(os.sched_getaffinity(0))
    n = min(w.B, cores)
    x = gi.workload_inputs(w, B=n, T=1)
    f = gi.to_f64_numpy(x)
    S0 = f["S0"]
    reps, total = 0, 0.0
    while total < seconds or reps == 0:
        t0 = time.perf_counter()
        oracle.recurrent(f["q"], f["k"], f["v"], f["beta"], f["g"], f["gate_kind"], S0,
                         threads=cores)
        total += time.perf_counter() - t0
        reps += 1
    rate = n * w.H * reps / total
    return rate, cores, f"{n} sequences x {w.H} heads x 1 step, {reps} runs, {total:.1f} s"


def run_reference(args, world, rank):
    """The reference arm: the oracle on a bounded sample of the headline
    workload per step, rank 0 only."""
    if rank != 0:
        return
    w = gi.WORKLOADS[HEADLINE]
    import oracle
    oracle.build()
    cores = len(os.sched_getaffinity(0))
    H = min(w.H, cores)
    T = 4096
    x = gi.workload_inputs(w, B=1, T=T, H=H)
    f = gi.to_f64_numpy(x)

    def step():
        oracle.recurrent(f["q"], f["k"], f["v"], f["beta"], f["g"], f["gate_kind"], f["S0"],
                         threads=cores)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    th_per_s = H * T * args.steps / el
    tok_s = th_per_s / w.H          # tokens/s of the whole workload (all its heads)
    F = flops_per_token_head(w.Dk, w.Dv)
    line = {
        "impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": w.B * w.T / tok_s * 1e3, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "Dk": w.Dk, "Dv": w.Dv,
                   "chunk": w.chunk, "gate": w.gate, "parallelism": "none (host threads)"},
        "algorithmic_tflops": th_per_s * F / 1e12,
        "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{H} heads x {T} tokens of one sequence per step, "
                                   f"{args.steps} steps; tokens/s of the whole workload = "
                                   f"token-heads/s / {w.H} heads"},
        "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm
class Ctx:
    def __init__(self, args, world, rank, local):
        import gated_delta_rule_94_b200 as gdn
        self.gdn = gdn
        self.args, self.world, self.rank = args, world, rank
        torch.cuda.set_device(local)
        self.dev = torch.device("cuda", local)
        self.peaks, self.peak_src = load_peaks()
        l2 = torch.cuda.get_device_properties(self.dev).L2_cache_size
        self.l2 = l2
        self.flush = torch.empty(2 * l2, dtype=torch.uint8, device=self.dev)
        self.stream = torch.cuda.current_stream(self.dev)
        self.sampler = ClockSampler(self.dev.index if self.dev.index is not None else 0)


def time_forward(ctx: Ctx, wid: int):
    """Times K forwards of this rank's share of workload `wid` (L2 flushed
    before each); returns the per-workload record (rank 0) and its launches."""
    gdn, args, world, rank = ctx.gdn, ctx.args, ctx.world, ctx.rank
    w = gi.WORKLOADS[wid]
    h0, h1 = shard_heads(w.H, world, rank)
    Hl = h1 - h0
    B, T, Dk, Dv = w.B, w.T, w.Dk, w.Dv
    launches, per_ms, e2e_ms = 0, [0.0], 0.0
    kname = gdn.gdn_chunk_fwd_kernel_name(Dk, Dv, w.gate_kind, w.torch_dtype)
    h2d = d2h = 0
    if Hl > 0:
        d = gi.workload_inputs(w, H=Hl, seed=w.seed + rank, device=ctx.dev)
        o = torch.empty((B, T, Hl, Dv), dtype=w.torch_dtype, device=ctx.dev)
        S = torch.empty((B, Hl, Dk, Dv), dtype=torch.float32, device=ctx.dev)
        nws = gdn.gdn_chunk_fwd_workspace_bytes(B, T, Hl, Dk, Dv, 64, w.torch_dtype, w.gate_kind)
        ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=ctx.dev) if nws else None

        def step():
            gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], w.gate_kind, d["S0"], o,
                              S, workspace=ws, stream=ctx.stream)
        for _ in range(args.warmup):
            ctx.flush.zero_()
            step()
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()
    if Hl > 0:
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        n0 = gdn.gdn_kernel_launch_count()
        for i in range(args.steps):
            ctx.flush.zero_()
            starts[i].record(ctx.stream)
            step()
            ends[i].record(ctx.stream)
        torch.cuda.synchronize()
        launches = gdn.gdn_kernel_launch_count() - n0
        per_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    barrier(world)
    ctx.sampler.mark(t_wall0, time.perf_counter())
    ms = max_over_ranks(sum(per_ms) / len(per_ms), world)
    ms_min = max_over_ranks(min(per_ms), world)

    # ---- end to end through the public API: pinned host -> device copies of
    # this step's inputs, the forward, device -> host of o and the final state
    if Hl > 0 and not args.no_e2e:
        names = ("q", "k", "v", "beta", "g")
        host = {n: d[n].cpu().pin_memory() for n in names if d[n] is not None}
        o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        S_h = torch.empty(S.shape, dtype=S.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = o.numel() * o.element_size() + S.numel() * S.element_size()

        def e2e_step():
            for n, t in host.items():
                d[n].copy_(t, non_blocking=True)
            step()
            o_h.copy_(o, non_blocking=True)
            S_h.copy_(S, non_blocking=True)
        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize()
    barrier(world)
    if Hl > 0 and not args.no_e2e:
        ee0 = torch.cuda.Event(enable_timing=True)
        ee1 = torch.cuda.Event(enable_timing=True)
        ee0.record(ctx.stream)
        for _ in range(args.steps):
            e2e_step()
        ee1.record(ctx.stream)
        torch.cuda.synchronize()
        e2e_ms = ee0.elapsed_time(ee1) / args.steps
    e2e_ms = max_over_ranks(e2e_ms, world)
    h2d_all = max_over_ranks(float(h2d), world) * world
    d2h_all = max_over_ranks(float(d2h), world) * world
    if Hl > 0:
        del d, o, S, ws
    torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, cores, sample = oracle_sample(w, args.cpu_seconds)
        cpu = {"value": rate / w.H, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": sample + f"; tokens/s of the whole workload = token-heads/s / {w.H}"}
    if rank != 0:
        return None, launches
    peaks = ctx.peaks
    tokens = B * T                       # every head of every token, over all ranks
    N_th = B * T * w.H
    F = flops_per_token_head(Dk, Dv) * N_th
    nbytes = chunk_bytes(w)
    gbs = nbytes / (ms * 1e-3) / 1e9
    tflops = F / (ms * 1e-3) / 1e12
    bf16 = w.dtype == "bf16"
    rec = {
        "workload": w.name,
        "config": {"workload": w.name, "B": B, "T": T, "H": w.H, "Dk": Dk, "Dv": Dv,
                   "chunk": w.chunk, "gate": w.gate,
                   "initial_state": "zero (NULL)" if w.s0_std is None else f"N(0, {w.s0_std})",
                   "final_state": "written", "kernel": kname},
        "dtype": "bf16" if bf16 else "f32",
        "ms_per_step": ms, "ms_min": ms_min,
        "tokens_per_s": tokens / (ms * 1e-3),
        "tflops": tflops,
        "pct_bf16_peak": tflops / peaks["bf16_tflops"] if bf16 else None,
        "algorithmic_flops": F,
        "hbm_gbs": gbs, "pct_hbm": gbs / peaks["hbm_gbs"],
        # the forward's launches overlap one another (programmatic dependent
        # launch), so the unit timed and compared with the roofline is the
        # whole forward: its algorithmic bytes (or FLOPs) over the CUDA-event
        # time of the call; traffic is the DRAM bytes of all its launches (ncu)
        "roofline": ({"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                      "frac": gbs / peaks["hbm_gbs"], "traffic": ncu_traffic(f"chunk_fwd_w{wid}"),
                      "algorithmic_bytes": nbytes,
                      "kernel": f"{kname} (one forward: all its launches)",
                      "peak_source": ctx.peak_src + ", hbm_gbs (copy bandwidth)"} if bf16 else
                     {"bound": "alu", "achieved": tflops, "peak": FP32_ALU_TFLOPS,
                      "unit": "TFLOP/s", "frac": tflops / FP32_ALU_TFLOPS,
                      "traffic": ncu_traffic(f"chunk_fwd_w{wid}"), "algorithmic_flops": F,
                      "kernel": kname,
                      "peak_source": "fp32 FMA: 148 SMs x 128 lanes x 2 flop x 1.965 GHz"}),
        "e2e": {"value": tokens / (e2e_ms * 1e-3) if e2e_ms else None, "unit": "tokens/s",
                "h2d_bytes_per_step": int(h2d_all), "d2h_bytes_per_step": int(d2h_all),
                "ms_per_step": e2e_ms or None},
        "gpu_launches": launches,
        "cpu_baseline": cpu,
    }
    return rec, launches


def time_decode(ctx: Ctx):
    """128 consecutive in-place decode steps over this rank's heads, timed as
    one block per repetition."""
    gdn, args, world, rank = ctx.gdn, ctx.args, ctx.world, ctx.rank
    wd = gi.WORKLOADS[4]
    h0, h1 = shard_heads(wd.H, world, rank)
    Hl = h1 - h0
    steps_d = wd.T
    dec_ms, launches = [0.0], 0
    if Hl > 0:
        dd = gi.workload_inputs(wd, H=Hl, seed=wd.seed + rank, device=ctx.dev)
        state = dd["S0"].clone()
        toks = [tuple(dd[n][:, t].contiguous() if dd[n] is not None else None
                      for n in ("q", "k", "v", "beta", "g")) for t in range(steps_d)]
        od = torch.empty((wd.B, Hl, wd.Dv), dtype=dd["q"].dtype, device=ctx.dev)

        def decode_all():
            for (q, k, v, b_, g) in toks:
                gdn.gdn_decode_step(q, k, v, b_, g, wd.gate_kind, state, od, stream=ctx.stream)
        for _ in range(max(1, args.warmup // 3)):
            decode_all()
        torch.cuda.synchronize()
    barrier(world)
    td0 = time.perf_counter()
    if Hl > 0:
        dec_ms = []
        n0 = gdn.gdn_kernel_launch_count()
        for _ in range(args.steps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(ctx.stream)
            decode_all()
            e1.record(ctx.stream)
            e1.synchronize()
            dec_ms.append(e0.elapsed_time(e1) / steps_d)
        launches = gdn.gdn_kernel_launch_count() - n0
    barrier(world)
    ctx.sampler.mark(td0, time.perf_counter())
    step_ms = max_over_ranks(sum(dec_ms) / len(dec_ms), world)

    # end to end: each step's tokens copied in from pinned host memory, o read
    # back, the state resident on the device (as in serving)
    e2e_ms, h2d, d2h = 0.0, 0, 0
    if Hl > 0 and not args.no_e2e:
        names = ("q", "k", "v", "beta", "g")
        host = [[t.cpu().pin_memory() if t is not None else None for t in tk] for tk in toks]
        od_h = torch.empty(od.shape, dtype=od.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host[0] if t is not None)
        d2h = od.numel() * od.element_size()

        def e2e_all():
            for tk, th in zip(toks, host):
                for dst, src in zip(tk, th):
                    if dst is not None:
                        dst.copy_(src, non_blocking=True)
                q, k, v, b_, g = tk
                gdn.gdn_decode_step(q, k, v, b_, g, wd.gate_kind, state, od, stream=ctx.stream)
                od_h.copy_(od, non_blocking=True)
        e2e_all()
        torch.cuda.synchronize()
    barrier(world)
    if Hl > 0 and not args.no_e2e:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(ctx.stream)
        e2e_all()
        e1.record(ctx.stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1) / steps_d
    e2e_ms = max_over_ranks(e2e_ms, world)
    h2d_all = max_over_ranks(float(h2d), world) * world
    d2h_all = max_over_ranks(float(d2h), world) * world
    if Hl > 0:
        del dd, state, toks, od
    torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, cores, sample = oracle_decode_sample(wd, args.cpu_seconds)
        cpu = {"value": rate / wd.H, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": sample + f"; tokens/s = token-heads/s / {wd.H} heads"}
    if rank != 0:
        return None, launches
    peaks = ctx.peaks
    nbytes = decode_bytes_per_step(wd)
    gbs = nbytes / (step_ms * 1e-3) / 1e9
    rec = {
        "workload": wd.name, "us_per_step": step_ms * 1e3,
        "gbs": gbs, "pct_hbm": gbs / peaks["hbm_gbs"],
        "tokens_per_s": wd.B / (step_ms * 1e-3),
        "algorithmic_bytes_per_step": nbytes, "steps_timed": args.steps * steps_d,
        "l2": "not flushed between the 128 consecutive steps of one repetition",
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"], "kernel": "decode_step_kernel",
                     "traffic": ncu_traffic("decode_step_kernel")},
        "e2e": {"value": wd.B / (e2e_ms * 1e-3) if e2e_ms else None, "unit": "tokens/s",
                "h2d_bytes_per_step": int(h2d_all), "d2h_bytes_per_step": int(d2h_all),
                "us_per_step": e2e_ms * 1e3 if e2e_ms else None},
        "gpu_launches": launches,
        "cpu_baseline": cpu,
    }
    return rec, launches


# ------------------------------------------------- the rows beyond the forward
def time_events(ctx: Ctx, fn, flush=True):
    """Mean and min CUDA-event time (ms) of fn over --steps calls after
    --warmup, L2 flushed before each call (outside the events)."""
    for _ in range(ctx.args.warmup):
        if flush:
            ctx.flush.zero_()
        fn()
    torch.cuda.synchronize()
    ms = []
    for _ in range(ctx.args.steps):
        if flush:
            ctx.flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(ctx.stream)
        fn()
        e1.record(ctx.stream)
        e1.synchronize()
        ms.append(e0.elapsed_time(e1))
    return sum(ms) / len(ms), min(ms)


def hbm_roofline(ctx: Ctx, nbytes, ms, kernel):
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": gbs, "peak": ctx.peaks["hbm_gbs"], "unit": "GB/s",
            "frac": gbs / ctx.peaks["hbm_gbs"], "traffic": None, "algorithmic_bytes": nbytes,
            "kernel": kernel, "peak_source": ctx.peak_src + ", hbm_gbs (copy bandwidth)"}


def retention_gate(B, T, H, seed, device):
    """Retention gate of the preconditioner scan: sigmoid(N(0,1) + 2), bf16."""
    gen = torch.Generator().manual_seed(seed)
    return torch.sigmoid(torch.randn(B, T, H, generator=gen) + 2.0).to(torch.bfloat16).to(device)


def time_osdn(ctx: Ctx):
    """The preconditioned delta rule on the GDN workload's shape (B4 H16 T2048,
    scalar gate, bf16): phase 1 (write keys by the preconditioner scan, eta 0.5,
    retention gate) and phase 2 (the chunk forward with the write keys)."""
    gdn, args = ctx.gdn, ctx.args
    w = gi.WORKLOADS[1]
    B, T, H, Dk, Dv = w.B, w.T, w.H, w.Dk, w.Dv
    d = gi.workload_inputs(w, device=ctx.dev)
    r = retention_gate(B, T, H, 7, ctx.dev)
    kw = torch.empty_like(d["k"])
    d1 = torch.empty(B, H, Dk, device=ctx.dev)
    o = torch.empty(B, T, H, Dv, dtype=torch.bfloat16, device=ctx.dev)
    S = torch.empty(B, H, Dk, Dv, device=ctx.dev)
    nws = gdn.gdn_chunk_fwd_workspace_bytes(B, T, H, Dk, Dv, 64, torch.bfloat16, w.gate_kind)
    ws = torch.empty(nws, dtype=torch.uint8, device=ctx.dev)

    ws1 = torch.empty(gdn.gdn_osdn_precondition_workspace_bytes(B, T, H, Dk), dtype=torch.uint8,
                      device=ctx.dev)

    def phase1():
        gdn.gdn_osdn_precondition(d["k"], d["beta"], r, 0.5, None, kw, d1, workspace=ws1,
                                  stream=ctx.stream)

    def both():
        phase1()
        gdn.gdn_chunk_fwd_wk(d["q"], d["k"], kw, d["v"], d["beta"], d["g"], w.gate_kind, d["S0"],
                             o, S, workspace=ws, stream=ctx.stream)
    n0 = gdn.gdn_kernel_launch_count()
    both()
    torch.cuda.synchronize()
    launches = gdn.gdn_kernel_launch_count() - n0
    ms1, _ = time_events(ctx, phase1)
    ms, ms_min = time_events(ctx, both)
    N = B * T * H
    b1 = N * (2 * Dk * 2 + 2 + 2) + B * H * Dk * 4          # k, beta, r in; k_write, d out
    b2 = chunk_bytes(w) + N * Dk * 2                          # the forward, plus k_write
    cpu = None
    if not args.no_cpu_baseline:
        import oracle
        cores = len(os.sched_getaffinity(0))
        Hs, Ts = min(H, cores), 1024
        x = gi.workload_inputs(w, B=1, T=Ts, H=Hs)
        f = gi.to_f64_numpy(x)
        rr = retention_gate(1, Ts, Hs, 7, "cpu").double().numpy()
        reps, total = 0, 0.0
        while total < args.cpu_seconds or reps == 0:
            t0 = time.perf_counter()
            kw_ref, _ = oracle.osdn_precondition(f["k"], f["beta"], 0.5, r=rr)
            oracle.recurrent_wk(f["q"], f["k"], kw_ref, f["v"], f["beta"], f["g"], f["gate_kind"],
                                f["S0"], threads=cores)
            total += time.perf_counter() - t0
            reps += 1
        cpu = {"value": Hs * Ts * reps / total / H, "unit": "tokens/s", "cores": cores,
               "kind": "oracle", "sample": f"{Hs} heads x {Ts} tokens of one sequence, both "
                                          f"phases, {reps} runs, {total:.1f} s; tokens/s = "
                                          f"token-heads/s / {H} heads"}
    del d, r, kw, d1, o, S, ws, ws1
    torch.cuda.empty_cache()
    return {
        "workload": f"preconditioned delta rule (eta 0.5, retention gate), {w.name}",
        "ms_per_step": ms, "ms_min": ms_min, "tokens_per_s": B * T / (ms * 1e-3),
        "phase1_ms": ms1,
        "phase1_roofline": hbm_roofline(ctx, b1, ms1, "osdn_block_kernel, osdn_chain_kernel, "
                                                      "osdn_write_kernel"),
        "roofline": hbm_roofline(ctx, b1 + b2, ms, "osdn_block_kernel, osdn_chain_kernel, osdn_write_kernel + chunk_prep_kernel,"
                                                   "chunk_chain_kernel (both phases)"),
        "gpu_launches_per_step": launches, "cpu_baseline": cpu,
    }


def time_segments(ctx: Ctx):
    """A few-head long sequence (B1 H4 T65536, scalar gate, bf16), where the
    segment-parallel state pass engages with the full-speed workspace; timed
    beside the largest workspace whose plan runs the plain chain."""
    gdn, args = ctx.gdn, ctx.args
    w = gi.Workload("few-head long-sequence scalar-gated chunk fwd bf16 B1 H4 T65536 d128",
                    "chunk", B=1, T=65536, H=4, Dk=128, Dv=128, chunk=64, dtype="bf16",
                    gate="scalar", gate_scale=0.1, s0_std=None)
    B, T, H, Dk, Dv = w.B, w.T, w.H, w.Dk, w.Dv
    d = gi.workload_inputs(w, device=ctx.dev)
    o = torch.empty(B, T, H, Dv, dtype=torch.bfloat16, device=ctx.dev)
    S = torch.empty(B, H, Dk, Dv, device=ctx.dev)
    full = gdn.gdn_chunk_fwd_workspace_bytes(B, T, H, Dk, Dv, 64, torch.bfloat16, w.gate_kind)
    plain = None
    for frac in [x / 20 for x in range(19, 0, -1)]:
        n = int(full * frac) // 256 * 256
        if gdn.gdn_chunk_fwd_plan(B, T, H, Dk, Dv, 64, torch.bfloat16, w.gate_kind, n)["segments"] == 1:
            plain = n
            break
    rec = {"workload": w.name}
    for name, nws in (("segmented", full), ("plain_chain", plain)):
        if nws is None:
            continue
        ws = torch.empty(nws, dtype=torch.uint8, device=ctx.dev)
        plan = gdn.gdn_chunk_fwd_plan(B, T, H, Dk, Dv, 64, torch.bfloat16, w.gate_kind, nws)

        def step():
            gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], w.gate_kind, d["S0"], o,
                              S, workspace=ws, stream=ctx.stream)
        ms, ms_min = time_events(ctx, step)
        rec[name] = {"ms_per_step": ms, "ms_min": ms_min, "tokens_per_s": B * T / (ms * 1e-3),
                     "workspace_bytes": nws, "plan": plan,
                     "roofline": hbm_roofline(ctx, chunk_bytes(w), ms,
                                              "chunk_prep_kernel,chunk_chain_kernel,"
                                              "segment_combine_kernel (one forward)")}
        del ws
    del d, o, S
    torch.cuda.empty_cache()
    return rec


def time_backward(ctx: Ctx):
    """The backward of the chunk forward on the GDN workload's shape (B4 H16
    T2048, scalar gate, bf16 tokens): fp32 dq, dk, dv, dbeta, dg and the
    initial state's gradient from dO (bf16) and the final state's gradient."""
    gdn, args = ctx.gdn, ctx.args
    w = gi.WORKLOADS[1]
    B, T, H, Dk, Dv = w.B, w.T, w.H, w.Dk, w.Dv
    d = gi.workload_inputs(w, device=ctx.dev)
    gen = torch.Generator().manual_seed(11)
    do = torch.randn(B, T, H, Dv, generator=gen).to(torch.bfloat16).to(ctx.dev)
    dS = (0.02 * torch.randn(B, H, Dk, Dv, generator=gen)).to(ctx.dev)
    g = {n: torch.empty(B, T, H, *s, device=ctx.dev) for n, s in
         (("dq", (Dk,)), ("dk", (Dk,)), ("dv", (Dv,)), ("dbeta", ()), ("dg", ()))}
    dS0 = torch.empty(B, H, Dk, Dv, device=ctx.dev)
    nws = gdn.gdn_chunk_bwd_workspace_bytes(B, T, H, Dk, Dv, 64, torch.bfloat16, w.gate_kind)
    ws = torch.empty(nws, dtype=torch.uint8, device=ctx.dev)

    def step():
        gdn.gdn_chunk_bwd(d["q"], d["k"], d["v"], d["beta"], d["g"], w.gate_kind, d["S0"], do, dS,
                          g["dq"], g["dk"], g["dv"], g["dbeta"], g["dg"], dS0, workspace=ws,
                          stream=ctx.stream)
    n0 = gdn.gdn_kernel_launch_count()
    step()
    torch.cuda.synchronize()
    launches = gdn.gdn_kernel_launch_count() - n0
    ms, ms_min = time_events(ctx, step)
    N = B * T * H
    nbytes = N * (2 * (2 * Dk + 2 * Dv + 2)) + N * 4 * (2 * Dk + Dv + 2) + 2 * B * H * Dk * Dv * 4
    cpu = None
    if not args.no_cpu_baseline:
        import oracle
        Hs, Ts = 2, 128
        x = gi.workload_inputs(w, B=1, T=Ts, H=Hs)
        f = gi.to_f64_numpy(x)
        dof = do[:1, :Ts, :Hs].double().cpu().numpy()
        reps, total = 0, 0.0
        while total < args.cpu_seconds or reps == 0:
            t0 = time.perf_counter()
            oracle.backward(f["q"], f["k"], f["v"], f["beta"], f["g"], f["gate_kind"], f["S0"], dof)
            total += time.perf_counter() - t0
            reps += 1
        cpu = {"value": Hs * Ts * reps / total / H, "unit": "tokens/s",
               "cores": torch.get_num_threads(), "kind": "oracle",
               "sample": f"{Hs} heads x {Ts} tokens of one sequence (reverse-mode autograd of the "
                         f"fp64 token loop), {reps} runs, {total:.1f} s; tokens/s = "
                         f"token-heads/s / {H} heads"}
    del d, do, dS, g, dS0, ws
    torch.cuda.empty_cache()
    return {
        "workload": f"backward, {w.name}", "ms_per_step": ms, "ms_min": ms_min,
        "tokens_per_s": B * T / (ms * 1e-3),
        "roofline": hbm_roofline(ctx, nbytes, ms, "chunk_prep_kernel,chunk_chain_kernel (forward "
                                                  "rerun), adjoint_chain_kernel, chunk_bwd_kernel"),
        "gpu_launches_per_step": launches, "cpu_baseline": cpu,
    }


def run_only(args, world, rank, local):
    """One forward workload, or one extra record, alone (for profiling): its
    record, no CPU baseline."""
    args.no_cpu_baseline = True
    ctx = Ctx(args, world, rank, local)
    ctx.sampler.start()
    if args.only_extra:
        rec = {"osdn": time_osdn, "segments": time_segments,
               "backward": time_backward}[args.only_extra](ctx)
    else:
        rec, _ = time_forward(ctx, args.only)
    ctx.sampler.stop()
    if rank == 0:
        print(json.dumps(rec), flush=True)


def run_ours(args, world, rank, local):
    if args.only is not None or args.only_extra:
        return run_only(args, world, rank, local)
    ctx = Ctx(args, world, rank, local)
    ctx.sampler.start()
    head, _ = time_forward(ctx, HEADLINE)
    subs = {}
    for wid in SUBRECORDS:
        if str(wid) in args.workloads.split(","):
            subs[str(wid)], _ = time_forward(ctx, wid)
    dec = None
    if not args.no_decode:
        dec, _ = time_decode(ctx)
    extras = {}
    if rank == 0 and world == 1 and not args.no_extras:
        t0 = time.perf_counter()
        extras = {"osdn": time_osdn(ctx), "segments": time_segments(ctx),
                  "backward": time_backward(ctx)}
        ctx.sampler.mark(t0, time.perf_counter())
    clocks = ctx.sampler.stop()
    if rank != 0:
        return
    w = gi.WORKLOADS[HEADLINE]
    line = {
        "metric": METRIC, "value": head["tokens_per_s"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": head["dtype"], "data": "synthetic",
        "config": dict(head["config"],
                       parallelism=(f"heads split over {world} ranks, no collective on the "
                                    "data path" if world > 1 else "one GPU"),
                       l2=f"flushed before every step ({2 * ctx.l2 >> 20} MiB write)",
                       inputs="drawn on the device with the workload recipe (seed 0 + rank)"),
        "tflops": head["tflops"], "pct_bf16_peak": head["pct_bf16_peak"],
        "bf16_peak_tflops": ctx.peaks["bf16_tflops"],
        "roofline": head["roofline"],
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "clocks": clocks,
        "cpu_baseline": head["cpu_baseline"],
        "workloads": subs,
        "decode": dec,
        "extras": extras,
        "gpu": torch.cuda.get_device_name(ctx.dev),
    }
    _ = w
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workloads", default="1,2,0",
                    help="forward workloads reported beside the headline (comma separated)")
    ap.add_argument("--cpu-seconds", type=float, default=3.0,
                    help="host time of each oracle CPU baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the preconditioned-rule, segment and backward records")
    ap.add_argument("--only", type=int, default=None, choices=(0, 1, 2, 3),
                    help="time one forward workload alone and print its record (profiling)")
    ap.add_argument("--only-extra", default=None, choices=("osdn", "segments", "backward"),
                    help="time one extra record alone and print it (profiling)")
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
