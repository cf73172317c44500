"""Decode-step benchmark: paged decode attention seq-steps/s and KV-read GB/s.

One step = one pass of the whole hot path on one batch of synthetic input:
copy_blocks (copy-on-write pairs, when the workload has them) ->
reshape_and_cache (one new token per sequence) -> paged_attention_decode.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload cfg2]
    python bench.py --impl reference ...     # the fp64 CPU oracle, bounded sample
    python bench.py --measure swap           # swap_blocks: HBM <-> page-locked host GB/s
    python bench.py --measure block_manager  # host block manager, decode steps/s (no GPU)
    python bench.py --measure prefill        # chunked-prefill attention, TFLOP/s

Multi-GPU (torchrun): every rank runs its own batch of the same workload
(sequences are independent; no data-path collective) -> weak scaling; the
time is the max over ranks.  Prints one JSON line on rank 0.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention seq-steps/s and KV-read HBM GB/s (% of B200 peak)"
L2_BYTES = 126 * 1024 * 1024
WORKLOADS = {"cfg1": 1, "cfg2": 2, "cfg3": 3, "cfg4": 4, "cfg5": 5,
             "short": 7}    # 2048 sequences of U[1, 64] tokens (not one of the five configurations)


# ---------------------------------------------------------------- distributed
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed_offset(rank: int) -> int:
    """Each rank draws its own batch (weak scaling): seed offset per rank."""
    return 1000 * rank


def reduce_max(value: float, world: int, device=None) -> float:
    """Max over ranks of a timing (a timing reduction, not a data-path exchange)."""
    if world <= 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------- workload
def make_workload(name: str, rank: int, num_seqs: int = 0):
    from paged_kv_cache_373_b200 import workloads as W
    cfg = WORKLOADS[name]
    kw = {}
    if num_seqs and cfg in (2, 3, 4, 7):
        kw["num_seqs"] = num_seqs
    elif num_seqs and cfg == 5:
        kw["num_prompts"] = max(1, num_seqs // 8)
    wl = W.make_config(cfg, **kw)
    if rank:
        # a different, equally shaped batch per rank
        import math
        if cfg == 5:
            wl = W.config5()
        else:
            gen = torch.Generator().manual_seed(W._seed(cfg) * 1000 + rank_seed_offset(rank))
            lens = wl.seq_lens.tolist()
            perm = torch.randperm(len(lens), generator=gen).tolist()
            lens = [lens[i] for i in perm]
            wl = W.build_decode(wl.name, lens, wl.num_heads, wl.num_kv_heads, wl.head_dim,
                                wl.block_size, wl.kv_dtype, wl.q_dtype,
                                W._seed(cfg) + rank_seed_offset(rank),
                                num_blocks=wl.num_blocks, scale=wl.scale)
    return wl


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def recorded_traffic(workload: str):
    """dram read+write bytes per attention launch from a committed ncu summary
    (profiles/traffic.json), or None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    return d.get(workload)


# ---------------------------------------------------------------- clocks
HOST_GATE_CYCLES = 6_000_000  # about 3 ms of the SM clock


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons.  Started before
    the warm-up (nvidia-smi needs a few hundred ms to start); summary() keeps
    the samples whose timestamps fall inside the timed window."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.window = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()
        self.rows = self._read()

    def _read(self):
        if not self.path or not os.path.exists(self.path):
            return []
        import datetime
        rows = []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for ln in f:
                parts = [x.strip() for x in ln.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    rows.append((ts, float(parts[2]), float(parts[3]),
                                 {n for n, v in zip(names, parts[6:10]) if v.lower() == "active"}))
                except ValueError:
                    continue
        os.unlink(self.path)
        return rows

    def summary(self, window=None):
        """Median SM clock, max clock and throttle reasons of the samples taken
        inside `window` (wall-clock (t0, t1); default: the timed region)."""
        rows = getattr(self, "rows", None) or []
        if not rows:
            return None
        t0, t1 = window or self.window or (rows[0][0], rows[-1][0])
        inside = [r for r in rows if t0 - 0.02 <= r[0] <= t1 + 0.02]
        scope = "timed region"
        if not inside:  # region shorter than the sampling period: nearest samples
            inside = sorted(rows, key=lambda r: min(abs(r[0] - t0), abs(r[0] - t1)))[:2]
            scope = "nearest to the timed region"
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": inside[0][2],
                "reasons": sorted(set().union(*[r[3] for r in inside])), "samples": len(inside),
                "scope": scope}


# ---------------------------------------------------------------- oracle leg
class OracleSample:
    """The oracle (as it stands) timed on the first k sequences of the workload,
    k chosen once so that one call costs about `budget_s` seconds."""

    def __init__(self, wl, budget_s: float, threads: int = 0):
        sys.path.insert(0, os.path.join(ROOT, "tests"))
        import oracle
        from pkv_testutil import oracle_caches
        self.oracle, self.wl = oracle, wl
        self.cores = threads or oracle.num_threads_available()
        kmax = wl.num_seqs if not wl.is_fp8 else min(wl.num_seqs, 64)
        self.kmax = kmax
        self.kc, self.vc = oracle_caches(wl, None if not wl.is_fp8 else list(range(kmax)))
        self.k = self._calibrate(budget_s, self.cores)

    def _calibrate(self, budget_s: float, threads: int) -> int:
        k = 1
        while True:
            dt = self.time(k, threads)
            if dt >= budget_s / 2 or k >= self.kmax:
                return k
            k = min(self.kmax, max(k + 1, int(k * min(8.0, budget_s / max(dt, 1e-4)))))

    def time(self, k: int, threads: int = 0) -> float:
        wl = self.wl
        t0 = time.perf_counter()
        self.oracle.paged_attention_decode(wl.query, self.kc, self.vc, wl.block_tables, wl.seq_lens,
                                           wl.scale, wl.k_scale, wl.v_scale,
                                           seq_subset=list(range(k)), num_threads=threads or self.cores)
        return time.perf_counter() - t0

    def rate(self) -> float:
        return self.k / self.time(self.k)

    def single_thread(self, budget_s: float):
        """(seq-steps/s, sequences timed) with one thread."""
        k1 = self._calibrate(budget_s, 1)
        return k1 / self.time(k1, 1), k1


def host_cores() -> dict:
    """os.cpu_count() and nproc (the cores this process may use)."""
    try:
        nproc = int(subprocess.run(["nproc"], capture_output=True, text=True).stdout.strip())
    except Exception:
        nproc = None
    return {"os_cpu_count": os.cpu_count(), "nproc": nproc}


def cpu_baseline_line(wl, budget_s: float) -> dict:
    """The oracle on the host cores: all threads (the reported value) and one thread."""
    smp = OracleSample(wl, budget_s=budget_s)
    r = smp.rate()
    r1, k1 = smp.single_thread(budget_s / 3)
    return {"value": r, "unit": "seq-steps/s", "cores": smp.cores, "kind": "oracle",
            "sample": f"first {smp.k} of {wl.num_seqs} sequences of the same workload, "
                      f"fp64 C oracle, {smp.cores} OpenMP threads",
            "single_thread": {"value": r1, "unit": "seq-steps/s", "cores": 1,
                              "sample": f"first {k1} of {wl.num_seqs} sequences, 1 thread"},
            **host_cores()}


def pool_bytes(wl) -> int:
    return wl.num_blocks * wl.block_size * wl.num_kv_heads * wl.head_dim * wl.kv_elem_bytes() * 2


def decode_config(wl, cascade: bool, world: int) -> dict:
    """The decode line's config, shared by both arms."""
    flush = pool_bytes(wl) < 2 * L2_BYTES
    return {"workload": wl.name + ("_cascade" if cascade else ""),
            "num_seqs": wl.num_seqs, "num_heads": wl.num_heads,
            "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim,
            "block_size": wl.block_size, "num_blocks": wl.num_blocks,
            "max_seq_len": wl.max_seq_len, "cow_pairs": int(wl.cow_pairs.shape[0]),
            "kv_bytes_alg": wl.algorithmic_bytes(),
            "l2": "flushed between steps" if flush else "inputs larger than L2 (126 MB)",
            "parallelism": f"replicas x{world} (independent batches)"}


def run_reference(args):
    rank, world, local = dist_env()
    if rank != 0:
        return 0
    wl = make_workload(args.workload, 0, args.num_seqs)
    # each step is a bounded sample so the whole run (warm-up included) stays
    # within a few minutes
    budget = max(0.5, min(args.ref_budget, 120.0 / max(1, args.steps + args.warmup)))
    smp = OracleSample(wl, budget_s=budget)
    for _ in range(args.warmup):
        smp.rate()
    rates = [smp.rate() for _ in range(args.steps)]
    k_used, cores = smp.k, smp.cores
    value = statistics.median(rates)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "seq-steps/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * wl.num_seqs / value, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": decode_config(wl, args.cascade, args.gpus),
        "cpu_baseline": {"value": value, "unit": "seq-steps/s", "cores": cores, "kind": "oracle",
                         "sample": f"first {k_used} of {wl.num_seqs} sequences per step, fp64 C oracle, "
                                   f"median of {args.steps} steps",
                         **host_cores()},
        "e2e": {"value": value, "unit": "seq-steps/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ---------------------------------------------------------------- GPU leg
def run_ours(args):
    import paged_kv_cache_373_b200 as pkv
    from paged_kv_cache_373_b200 import _build
    _build.build()
    rank, world, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    wl = make_workload(args.workload, rank, args.num_seqs)

    # ---- resident device state
    from paged_kv_cache_373_b200.device_inputs import decode_inputs
    g = decode_inputs(wl, dev)
    out = torch.empty_like(g["q"])
    ws = pkv.alloc_workspace(wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim,
                             args.num_ctas, device=dev)
    has_pairs = g["pairs"].numel() > 0
    stream = torch.cuda.current_stream()
    flush = pool_bytes(wl) < 2 * L2_BYTES
    scratch = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev) if flush else None

    if args.cascade:
        from paged_kv_cache_373_b200 import workloads as W
        goff, gmem, gpre, gmax = (t.to(dev) if torch.is_tensor(t) else t for t in W.cascade_groups(wl))
        cws = torch.empty(pkv.paged_attention_cascade_workspace_bytes(
            wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim, gpre.shape[0], gmax,
            args.num_ctas), dtype=torch.uint8, device=dev)

    def attend():
        if args.cascade:
            pkv.paged_attention_decode_cascade(out, g["q"], g["kc"], g["vc"], g["tables"], g["lens"],
                                               goff, gmem, gpre, gmax, wl.scale, g["ks"], g["vs"],
                                               workspace=cws, num_ctas=args.num_ctas)
        else:
            pkv.paged_attention_decode(out, g["q"], g["kc"], g["vc"], g["tables"], g["lens"], wl.scale,
                                       g["ks"], g["vs"], workspace=ws, num_ctas=args.num_ctas)

    def step(ev_a0=None, ev_a1=None):
        if has_pairs:
            pkv.copy_blocks([g["kc"]], [g["vc"]], g["pairs"])
        pkv.reshape_and_cache(g["nk"], g["nv"], g["kc"], g["vc"], g["slots"], g["ks"], g["vs"])
        if ev_a0 is not None:
            ev_a0.record(stream)
        attend()
        if ev_a1 is not None:
            ev_a1.record(stream)

    def timed_steps(n):
        """n steps, each bracketed by events (step, and attention inside it)."""
        ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(4)) for _ in range(n)]
        for i in range(n):
            if flush:
                scratch.fill_(i & 0xff)     # evict the small workload from L2 (outside the step events)
            ev[i][0].record(stream)
            step(ev[i][1], ev[i][2])
            ev[i][3].record(stream)
        return ev

    # warm-up: at least W steps and at least --spinup-ms of GPU work, so the SM
    # clock has left its idle state before the timed region
    clk = ClockSampler(dev.index).start()
    warm = 0
    t0 = time.perf_counter()
    while warm < args.warmup or (time.perf_counter() - t0) * 1000.0 < args.spinup_ms:
        step()
        warm += 1
        if warm % 8 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    if pkv.get_device_error() != 0:
        raise RuntimeError("device error during warm-up")

    # ---- the timed region: exactly K steps
    K = args.steps
    barrier(world)
    torch.cuda.synchronize()
    wall0 = time.time()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    # the GPU first spins ~3 ms (before the start event) while the host
    # enqueues all K steps, so no host-side pause can fall inside the interval
    torch.cuda._sleep(HOST_GATE_CYCLES)
    t_start.record(stream)
    ev = timed_steps(K)
    t_end.record(stream)
    torch.cuda.synchronize()
    clk.window = (wall0, time.time())
    barrier(world)
    step_ms = [a.elapsed_time(d) for a, _, _, d in ev]
    attn_ms = [b.elapsed_time(c) for _, b, c, _ in ev]
    total_ms = sum(step_ms) if flush else t_start.elapsed_time(t_end)
    total_ms = reduce_max(total_ms, world, dev)
    if pkv.get_device_error() != 0:
        raise RuntimeError("device error during the timed steps")

    # ---- the measurement protocol of the scope table, after the timed
    # region: the median of >= 50 individually timed steps spanning >= 0.5 s,
    # with the SM clock sampled over that window
    proto = None
    if not args.no_protocol:
        n_proto, proto_ms, proto_attn = 0, [], []
        wallp = time.time()
        while n_proto < 50 or time.time() - wallp < 0.5:
            evp = timed_steps(50)
            torch.cuda.synchronize()
            proto_ms += [a.elapsed_time(d) for a, _, _, d in evp]
            proto_attn += [b.elapsed_time(c) for _, b, c, _ in evp]
            n_proto += 50
        window = (wallp, time.time())
        med_attn = statistics.median(proto_attn)
        proto = {"runs": n_proto, "median_step_ms": statistics.median(proto_ms),
                 "median_attention_ms": med_attn,
                 "p10_p90_attention_ms": [sorted(proto_attn)[n_proto // 10],
                                          sorted(proto_attn)[(9 * n_proto) // 10]],
                 "kv_read_gbs_at_median": wl.algorithmic_bytes() / (med_attn / 1000.0) / 1e9,
                 "window_s": window[1] - window[0], "clocks": None}
        proto["_window"] = window
        if pkv.get_device_error() != 0:
            raise RuntimeError("device error during the protocol steps")
    clk.stop()
    if proto is not None:
        proto["clocks"] = clk.summary(proto.pop("_window"))

    ms_per_step = total_ms / K
    value = world * wl.num_seqs / (ms_per_step / 1000.0)
    attn_avg_ms = statistics.mean(attn_ms)
    b_alg = wl.algorithmic_bytes()
    peak, peak_kind = measured_peaks()
    achieved = b_alg / (attn_avg_ms / 1000.0) / 1e9
    traffic = recorded_traffic(wl.name + ("_cascade" if args.cascade else ""))

    # ---- end-to-end through the C ABI with host buffers
    casc = (W.cascade_groups(wl), cws) if args.cascade else None
    e2e = e2e_leg(pkv, wl, g, ws, args, dev, out_ref=out, cascade=casc) if not args.no_e2e else None
    e2e_pipe = reduce_max(e2e["pipelined_ms"], world, dev) if e2e else None
    # (the cascade call has no host-step entry point: pipelined mode only)
    e2e_serial = reduce_max(e2e["serial_ms"], world, dev) if e2e and e2e["serial_ms"] is not None else None
    e2e_value = None if e2e is None else (e2e_pipe if e2e_serial is None else min(e2e_pipe, e2e_serial))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_line(wl, args.ref_budget)

    # copy_blocks, reshape_and_cache, then decode + merge (cascade, batches of up to 256 sequences:
    # zeroing, setup, prefix, suffix decode, finish)
    launches_per_step = (1 if has_pairs else 0) + 1 + (5 if args.cascade else 2)
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "seq-steps/s", "n_gpus": world,
            "steps": K, "warmup": warm, "warmup_requested": args.warmup,
            "warmup_note": f"at least the requested steps and at least {args.spinup_ms:.0f} ms of GPU "
                           "work, so the SM clock has left its idle state before the timed region",
            "ms_per_step": ms_per_step,
            "timing": f"sum of {K} per-step event intervals (L2 flushed between steps)" if flush else
                      f"one event interval over {K} back-to-back steps (mean)",
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": {True: "fp8_e4m3 kv / fp32 accum", False: str(wl.kv_dtype).replace("torch.", "")
                      + " kv / fp32 accum"}[wl.is_fp8],
            "data": "synthetic",
            "config": decode_config(wl, args.cascade, world),
            "attention_ms": attn_avg_ms,
            "attention_ms_median": statistics.median(attn_ms),
            "kv_read_gbs": achieved,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_kind": f"{peak_kind} copy bandwidth",
                         "traffic": traffic,
                         "traffic_source": None if traffic is None else
                         "profiles/traffic.json: ncu dram__bytes_read.sum + dram__bytes_write.sum of one "
                         "attention call (every kernel of the call: decode + merge, or the cascade's zeroing, "
                         "setup, prefix, suffix decode and finish passes) on this workload, not measured in "
                         "this run"},
            "clocks": clk.summary(),
            "protocol": proto,
            "gpu_launches": launches_per_step * K,
            "e2e": None if e2e is None else {
                "value": world * wl.num_seqs / (e2e_value / 1000.0), "unit": "seq-steps/s",
                "mode": "pipelined" if e2e_serial is None or e2e_pipe <= e2e_serial else "serial",
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                "copies_per_step": e2e["copies"], "output_matches_device_path": e2e["matches_device_path"],
                "api": "the faster of the host-driven modes below (the cascade call: pipelined only, it "
                       "has no host-step entry point); in each, every step copies its inputs host -> device "
                       "and its output device -> host",
                "pipelined": {"value": world * wl.num_seqs / (e2e_pipe / 1000.0),
                              "api": "two steps in flight: one H2D copy of the packed inputs (pinned host "
                                     "buffer" + (", and one of the group arrays" if args.cascade else "") +
                                     ") on the step's copy stream, copy_blocks / reshape_and_cache / " +
                                     ("paged_attention_decode_cascade" if args.cascade else
                                      "paged_attention_decode") +
                                     " on one compute stream, one D2H copy of the output; step n+1's input "
                                     "copy overlaps step n's kernels"},
                "serial": None if e2e_serial is None else {
                    "value": world * wl.num_seqs / (e2e_serial / 1000.0),
                    "api": "pkv_decode_step_host, packed inputs (one H2D, one D2H, one stream sync "
                           "per step, one step at a time)"}},
            "cpu_baseline": cpu,
        }
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------- swap leg
SWAP_METRIC = "swap_blocks GB/s (KV blocks between HBM and page-locked host memory)"


def run_swap(args):
    """Preemption by swapping on cfg5-shaped blocks (16 tokens x 8 kv heads x
    128 x bf16 = 32 KB per K or V block): swap out `--swap-blocks` scattered
    device blocks to a pinned host pool, then swap them back into other
    scattered device blocks.  One step = out + in.  The peak is one
    contiguous cudaMemcpyAsync of the same bytes each way in the same run (the
    copy engines over the host link); the per-block copy loop is the
    one-DMA-call-per-block pattern, timed beside it."""
    import paged_kv_cache_373_b200 as pkv
    from paged_kv_cache_373_b200 import _build
    _build.build()
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    gen = torch.Generator().manual_seed(373)
    nb_dev, n = 16384, args.swap_blocks
    shape = (16, 8, 128)
    dk = torch.randn((nb_dev,) + shape, generator=gen, dtype=torch.float32).to(torch.bfloat16).to(dev)
    dv = torch.randn((nb_dev,) + shape, generator=gen, dtype=torch.float32).to(torch.bfloat16).to(dev)
    hk = torch.empty((n,) + shape, dtype=torch.bfloat16).pin_memory()
    hv = torch.empty((n,) + shape, dtype=torch.bfloat16).pin_memory()
    perm = torch.randperm(nb_dev, generator=gen)
    out_map = torch.stack([perm[:n], torch.arange(n)], 1).to(dev)
    in_map = torch.stack([torch.arange(n), perm[n:2 * n]], 1).to(dev)
    block_bytes = hk[0].numel() * 2
    moved = 2 * n * block_bytes                     # K and V, one direction
    stream = torch.cuda.current_stream()

    def timed(fn, k):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(k):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / k

    out_ms = timed(lambda: pkv.swap_blocks([hk], [hv], [dk], [dv], out_map), args.steps)
    in_ms = timed(lambda: pkv.swap_blocks([dk], [dv], [hk], [hv], in_map), args.steps)
    if pkv.get_device_error() != 0:
        raise RuntimeError("device error in swap_blocks")
    # peaks: one contiguous copy of the same bytes each way (K and V pools)
    dflat = dk[:n].view(-1)
    hflat = hk.view(-1)
    d2h_ms = timed(lambda: (hflat.copy_(dflat, non_blocking=True), hv.view(-1).copy_(dv[:n].view(-1), non_blocking=True)), args.steps)
    h2d_ms = timed(lambda: (dflat.copy_(hflat, non_blocking=True), dv[:n].view(-1).copy_(hv.view(-1), non_blocking=True)), args.steps)
    # one cudaMemcpyAsync per block (torch's copy_ per block row)
    idx_out = perm[:n].tolist()

    def per_block_out():
        for i, b in enumerate(idx_out[:256]):
            hk[i].copy_(dk[b], non_blocking=True)
            hv[i].copy_(dv[b], non_blocking=True)
    pb_ms = timed(per_block_out, max(3, args.steps // 10)) * n / 256
    # CPU baseline: the oracle's swap (memcpy per block) on host copies of the pools
    cpu = None
    if not args.no_cpu_baseline:
        import oracle
        sk, sv = [dk[perm[:n]].cpu()], [dv[perm[:n]].cpu()]
        ok, ov = [torch.empty_like(sk[0])], [torch.empty_like(sv[0])]
        m = torch.stack([torch.arange(n), torch.arange(n)], 1)
        t0 = time.perf_counter()
        reps = 0
        while time.perf_counter() - t0 < min(args.ref_budget, 10.0) or reps == 0:
            oracle.swap_blocks(ok, ov, sk, sv, m)
            reps += 1
        dt = (time.perf_counter() - t0) / reps
        cpu = {"value": moved / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
               "sample": f"{n} blocks x K,V host-to-host memcpy per block, {reps} reps"}
    out_gbs, in_gbs = moved / out_ms / 1e6, moved / in_ms / 1e6
    d2h_gbs, h2d_gbs = moved / d2h_ms / 1e6, moved / h2d_ms / 1e6
    value = 2 * moved / (out_ms + in_ms) / 1e6
    peak = 2 * moved / (d2h_ms + h2d_ms) / 1e6
    line = {
        "metric": SWAP_METRIC, "value": value, "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": out_ms + in_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bytes (bf16 blocks)", "data": "synthetic",
        "config": {"workload": f"swap_{n}_blocks_of_32KB_x2", "blocks": n, "block_bytes": block_bytes,
                   "device_pool_blocks": nb_dev, "bytes_per_direction": moved},
        "swap_out_gbs": out_gbs, "swap_in_gbs": in_gbs,
        "contiguous_copy_gbs": {"d2h": d2h_gbs, "h2d": h2d_gbs},
        "per_block_memcpy_out_gbs": moved / pb_ms / 1e6,
        "roofline": {"bound": "host link", "achieved": value, "peak": peak, "unit": "GB/s",
                     "frac": value / peak, "peak_kind": "contiguous cudaMemcpyAsync of the same bytes, "
                                                      "measured in this run", "traffic": None},
        "gpu_launches": 2 * args.steps, "e2e": None, "cpu_baseline": cpu,
    }
    print(json.dumps(line))
    return 0


# ---------------------------------------------------------------- prefill leg
PREFILL_METRIC = "chunked-prefill attention TFLOP/s (causal, paged KV)"


def run_prefill(args):
    """One step of chunked prefill: reshape_and_cache of the chunks' K/V, then
    paged_prefill over all chunk rows (the budget-8192 step of the
    ttlab.hopto.org experiment by default).  FLOPs = 4 * causal pairs * Hq * D;
    the dominant kernel is bound by the tensor cores (bf16 mma.sync), peak =
    the measured cuBLAS bf16 burst figure."""
    import paged_kv_cache_373_b200 as pkv
    from paged_kv_cache_373_b200 import _build, workloads as W
    _build.build()
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    wl = W.prefill_config(args.prefill_budget)
    kc, vc = wl.key_cache.to(dev), wl.value_cache.to(dev)
    q, nk, nv = wl.query.to(dev), wl.new_key.to(dev), wl.new_value.to(dev)
    slots, tables = wl.slot_mapping.to(dev), wl.block_tables.to(dev)
    lens, qs = wl.seq_lens.to(dev), wl.query_start.to(dev)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()
    scratch = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def step(e0=None, e1=None):
        pkv.reshape_and_cache(nk, nv, kc, vc, slots)
        if e0 is not None:
            e0.record(stream)
        pkv.paged_prefill(out, q, kc, vc, tables, lens, qs, wl.scale)
        if e1 is not None:
            e1.record(stream)

    clk = ClockSampler(dev.index).start()
    t0 = time.perf_counter()
    warm = 0
    while warm < args.warmup or (time.perf_counter() - t0) * 1000.0 < args.spinup_ms:
        step()
        warm += 1
    torch.cuda.synchronize()
    if pkv.get_device_error() != 0:
        raise RuntimeError("device error in prefill warm-up")
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    wall0 = time.time()
    for i in range(K):
        scratch.fill_(i & 0xff)          # cold L2 for every step (outside the step events)
        ev[i][0].record(stream)
        step(ev[i][1], ev[i][2])
        ev[i][3].record(stream)
    torch.cuda.synchronize()
    clk.window = (wall0, time.time())
    clk.stop()
    if pkv.get_device_error() != 0:
        raise RuntimeError("device error in prefill")
    step_ms = statistics.mean(a.elapsed_time(d) for a, _, _, d in ev)
    attn_ms = statistics.mean(b.elapsed_time(c) for _, b, c, _ in ev)
    flops = wl.flops()
    achieved = flops / (attn_ms / 1000.0) / 1e12
    peak, kind = 1590.0, "fallback bf16 burst"
    pp = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pp):
        with open(pp) as f:
            peak, kind = float(json.load(f)["bf16_tflops"]), "measured cuBLAS bf16 burst"
    cpu = None
    if not args.no_cpu_baseline:
        import oracle
        kc_h, vc_h = wl.key_cache.clone(), wl.value_cache.clone()
        oracle.reshape_and_cache(wl.new_key, wl.new_value, kc_h, vc_h, wl.slot_mapping)
        # the decode row and the last chunk (the oracle's bounded sample)
        qsl = wl.query_start.tolist()
        sub = [0, wl.num_seqs - 1]
        rows = torch.cat([wl.query[qsl[s]:qsl[s + 1]] for s in sub])
        qsub = torch.tensor([0] + list(torch.tensor([qsl[s + 1] - qsl[s] for s in sub]).cumsum(0).tolist()),
                            dtype=torch.int32)
        sw = W.build_prefill("sample", [int(wl.seq_lens[s]) - (qsl[s + 1] - qsl[s]) for s in sub],
                             [qsl[s + 1] - qsl[s] for s in sub], wl.num_heads, wl.num_kv_heads,
                             wl.head_dim, wl.block_size, wl.kv_dtype, 1)
        t0 = time.perf_counter()
        oracle.paged_prefill(rows, kc_h, vc_h, wl.block_tables[sub], wl.seq_lens[sub], qsub, wl.scale,
                             num_threads=oracle.num_threads_available())
        dt = time.perf_counter() - t0
        cpu = {"value": sw.flops() / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads_available(),
               "kind": "oracle", "sample": f"sequences {sub} of the step ({sw.num_tokens} chunk rows), fp64 C oracle"}
    line = {
        "metric": PREFILL_METRIC, "value": achieved, "unit": "TFLOP/s", "n_gpus": 1, "steps": K,
        "warmup": warm, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 / fp32 accum", "data": "synthetic",
        "config": {"workload": wl.name, "num_seqs": wl.num_seqs, "chunk_tokens": wl.num_tokens,
                   "seq_lens": wl.seq_lens.tolist(), "num_heads": wl.num_heads,
                   "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim, "block_size": wl.block_size,
                   "flops": flops, "l2": "flushed between steps"},
        "prefill_ms": attn_ms,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "peak_kind": kind, "traffic": recorded_traffic(wl.name)},
        "clocks": clk.summary(), "gpu_launches": 2 * K, "e2e": None, "cpu_baseline": cpu,
    }
    print(json.dumps(line))
    return 0


# ---------------------------------------------------------------- host block manager leg
BM_METRIC = "host block manager decode-step bookkeeping, seq-steps/s"


def run_block_manager(args):
    """The serving-side bookkeeping of cfg5 (16 prompts x 8 samples, 3000-token
    shared prefix, prefix caching on): admit the prompts (key chain, cache
    hits for samples forked from them), then per decode step one batched
    append for all 128 sequences (slot mapping + copy-on-write pairs) and the
    batch's block tables.  Host only; the oracle is timed on the same steps."""
    import paged_kv_cache_373_b200 as pkv
    from paged_kv_cache_373_b200 import _build
    _build.build()
    prompts, samples, prefix, bs = 16, 8, 3000, 16
    nblocks = prompts * (prefix // bs + 1) + prompts * samples * 40 + 64
    gen = torch.Generator().manual_seed(373 + 5)
    toks = torch.randint(0, 32000, (prompts, prefix), generator=gen).tolist()

    def admit(bm):
        sids = []
        for p in range(prompts):
            parent, _ = bm.add_sequence(toks[p])
            sids += [bm.fork(parent) for _ in range(samples)]
            bm.free_sequence(parent)
        return sids

    K = args.steps
    new_tok = torch.randint(0, 32000, (K + args.warmup, prompts * samples), generator=gen).tolist()
    mbps = (prefix + K + args.warmup) // bs + 2
    bm = pkv.HostBlockManager(nblocks, bs)
    t0 = time.perf_counter()
    sids = admit(bm)
    admit_s = time.perf_counter() - t0
    for i in range(args.warmup):
        bm.append_batch(sids, new_tok[i])
    t0 = time.perf_counter()
    cows = 0
    for i in range(K):
        slots, pairs = bm.append_batch(sids, new_tok[args.warmup + i])
        tables, lens = bm.batch_tables(sids, mbps)
        cows += pairs.shape[0]
    dt = time.perf_counter() - t0
    value = K * len(sids) / dt
    cpu = None
    if not args.no_cpu_baseline:
        from oracle.block_manager import OracleBlockManager
        ob = OracleBlockManager(nblocks, bs)
        sids_o = admit(_OracleAdapter(ob))
        for i in range(args.warmup):
            for s, t in zip(sids_o, new_tok[i]):
                ob.append_token(s, t)
        k_o, t0 = 0, time.perf_counter()
        while k_o < K and time.perf_counter() - t0 < min(args.ref_budget, 10.0):
            for s, t in zip(sids_o, new_tok[args.warmup + k_o]):
                ob.append_token(s, t)
            _ = [ob.block_table(s) for s in sids_o]
            k_o += 1
        cpu = {"value": k_o * len(sids_o) / (time.perf_counter() - t0), "unit": "seq-steps/s", "cores": 1,
               "kind": "oracle", "sample": f"{k_o} of {K} decode steps, pure-Python oracle"}
    line = {
        "metric": BM_METRIC, "value": value, "unit": "seq-steps/s", "n_gpus": 0, "steps": K,
        "warmup": args.warmup, "ms_per_step": 1000.0 * dt / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int32 ids / sha256 keys", "data": "synthetic",
        "config": {"workload": "cfg5_serving_bookkeeping_16x8", "num_seqs": len(sids), "block_size": bs,
                   "num_blocks": nblocks, "prefix_tokens": prefix, "prefix_cache": True},
        "admit_ms": 1000.0 * admit_s, "stats": bm.stats(), "cow_pairs_in_timed_steps": cows,
        "roofline": None, "gpu_launches": 0, "e2e": None, "cpu_baseline": cpu,
    }
    print(json.dumps(line))
    return 0


class _OracleAdapter:
    """The oracle block manager behind the native binding's method names."""

    def __init__(self, ob):
        self.ob = ob

    def add_sequence(self, tokens, extras=b""):
        return self.ob.add_sequence(tokens, extras)

    def fork(self, parent):
        return self.ob.fork(parent)

    def free_sequence(self, sid):
        self.ob.free_sequence(sid)


def e2e_leg(pkv, wl, g, ws, args, dev, out_ref=None, cascade=None):
    """decode_step_host with packed inputs: the step's inputs sit in one pinned
    host buffer (laid out by pkv_decode_step_layout) -> one H2D copy ->
    copy_blocks / reshape_and_cache / decode -> one D2H copy of the output ->
    stream sync, every step."""
    qd = pkv.dtype_code(wl.query)
    npairs = int(wl.cow_pairs.shape[0])
    lay = pkv.decode_step_layout(wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim, qd,
                                 wl.max_blocks_per_seq, npairs)
    hbuf = torch.zeros(lay.total, dtype=torch.uint8).pin_memory()

    def put(off, t):
        b = t.contiguous().view(-1).view(torch.uint8)
        hbuf[off:off + b.numel()] = b

    put(lay.query, wl.query)
    put(lay.new_key, wl.new_key.to(wl.q_dtype))
    put(lay.new_value, wl.new_value.to(wl.q_dtype))
    put(lay.slot_mapping, wl.slot_mapping)
    put(lay.block_tables, wl.block_tables)
    put(lay.seq_lens, wl.seq_lens)
    if npairs:
        put(lay.cow_pairs, wl.cow_pairs)
    if cascade is not None:
        # the cascade call: pipelined mode only, its group arrays copied in every step too
        pipe = e2e_pipelined(pkv, wl, g, ws, args, dev, lay, hbuf, out_ref, cascade)
        return {"pipelined_ms": pipe["ms"], "serial_ms": None, "h2d": int(lay.total) + pipe["extra_h2d"],
                "d2h": wl.query.numel() * wl.query.element_size(), "copies": 3,
                "matches_device_path": pipe["same"]}
    dbuf = torch.empty(max(lay.total, 16), dtype=torch.uint8, device=dev)
    h_out = torch.empty_like(wl.query).pin_memory()
    d_out = torch.empty_like(g["q"])
    a = pkv.DecodeStepArgs()
    a.num_seqs, a.num_heads, a.num_kv_heads = wl.num_seqs, wl.num_heads, wl.num_kv_heads
    a.head_dim, a.block_size, a.max_blocks_per_seq = wl.head_dim, wl.block_size, wl.max_blocks_per_seq
    a.num_blocks = wl.num_blocks
    a.q_dtype = qd
    a.cache_dtype = pkv.PKV_FP8_E4M3 if wl.is_fp8 else qd
    a.scale, a.num_ctas = wl.scale, args.num_ctas
    a.num_cow_pairs = npairs
    a.h_packed, a.d_packed = hbuf.data_ptr(), dbuf.data_ptr()
    a.h_out, a.d_out = h_out.data_ptr(), d_out.data_ptr()
    a.key_cache, a.value_cache = g["kc"].data_ptr(), g["vc"].data_ptr()
    a.k_scale = g["ks"].data_ptr() if g["ks"] is not None else None
    a.v_scale = g["vs"].data_ptr() if g["vs"] is not None else None
    a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        pkv.decode_step_host(a, stream)
    K = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(K):
        pkv.decode_step_host(a, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    same = None if out_ref is None else bool(torch.equal(h_out.view(-1).view(torch.uint8),
                                                         out_ref.cpu().view(-1).view(torch.uint8)))
    serial_ms = e0.elapsed_time(e1) / K
    pipe = e2e_pipelined(pkv, wl, g, ws, args, dev, lay, hbuf, out_ref)
    return {"pipelined_ms": pipe["ms"], "serial_ms": serial_ms, "h2d": int(lay.total),
            "d2h": h_out.numel() * h_out.element_size(), "copies": 2,
            "matches_device_path": same if pipe["same"] is None else (bool(same) and pipe["same"])}


def e2e_pipelined(pkv, wl, g, ws, args, dev, lay, hbuf, out_ref=None, cascade=None):
    """The same steps with two in flight: every step still copies its packed
    inputs host -> device (one copy) and its output device -> host (one
    copy), but step n+1's input copy runs on its own copy stream while step
    n's kernels run, and step n's output copy while step n+1's kernels run.
    Two slots of device staging alternate; the kernels of all steps stay on
    one compute stream, so consecutive steps never touch the caches at the
    same time.  Calls: the package's copy_blocks / reshape_and_cache /
    paged_attention_decode on views of the packed device buffer."""
    npairs = int(wl.cow_pairs.shape[0])
    S, Hq, Hkv, D = wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim
    qdt = wl.query.dtype
    comp = torch.cuda.current_stream()
    cps = [torch.cuda.Stream(), torch.cuda.Stream()]
    dbufs = [torch.empty(max(lay.total, 16), dtype=torch.uint8, device=dev) for _ in range(2)]
    d_outs = [torch.empty_like(g["q"]) for _ in range(2)]
    h_outs = [torch.empty_like(wl.query).pin_memory() for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_k = [torch.cuda.Event() for _ in range(2)]

    def view(buf, off, n, dtype, shape):
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        return buf[off:off + nbytes].view(dtype).view(shape)

    views = []
    for b in dbufs:
        views.append({
            "q": view(b, lay.query, S * Hq * D, qdt, (S, Hq, D)),
            "nk": view(b, lay.new_key, S * Hkv * D, qdt, (S, Hkv, D)),
            "nv": view(b, lay.new_value, S * Hkv * D, qdt, (S, Hkv, D)),
            "slots": view(b, lay.slot_mapping, S, torch.int64, (S,)),
            "tables": view(b, lay.block_tables, S * wl.max_blocks_per_seq, torch.int32,
                           (S, wl.max_blocks_per_seq)),
            "lens": view(b, lay.seq_lens, S, torch.int32, (S,)),
            "pairs": view(b, lay.cow_pairs, 2 * npairs, torch.int64, (npairs, 2)) if npairs else None,
        })

    # the cascade call's group arrays (offsets, members, prefix lengths), one
    # more pinned buffer copied in every step
    h_grp, d_grps, grp_views, gmax, cws = None, None, None, 0, None
    if cascade is not None:
        (goff, gmem, gpre, gmax), cws = cascade
        h_grp = torch.cat([goff, gmem, gpre]).to(torch.int32).pin_memory()
        d_grps = [torch.empty_like(h_grp, device=dev) for _ in range(2)]
        n0, n1 = goff.numel(), gmem.numel()
        grp_views = [(d[:n0], d[n0:n0 + n1], d[n0 + n1:]) for d in d_grps]

    def step(i):
        k = i & 1
        v = views[k]
        with torch.cuda.stream(cps[k]):
            dbufs[k][:lay.total].copy_(hbuf, non_blocking=True)
            if h_grp is not None:
                d_grps[k].copy_(h_grp, non_blocking=True)
            ev_in[k].record(cps[k])
        comp.wait_event(ev_in[k])
        if npairs:
            pkv.copy_blocks([g["kc"]], [g["vc"]], v["pairs"], stream=comp)
        pkv.reshape_and_cache(v["nk"], v["nv"], g["kc"], g["vc"], v["slots"], g["ks"], g["vs"], stream=comp)
        if cascade is not None:
            go, gm, gp = grp_views[k]
            pkv.paged_attention_decode_cascade(d_outs[k], v["q"], g["kc"], g["vc"], v["tables"], v["lens"],
                                               go, gm, gp, gmax, wl.scale, g["ks"], g["vs"], workspace=cws,
                                               num_ctas=args.num_ctas, stream=comp)
        else:
            pkv.paged_attention_decode(d_outs[k], v["q"], g["kc"], g["vc"], v["tables"], v["lens"], wl.scale,
                                       g["ks"], g["vs"], workspace=ws, num_ctas=args.num_ctas, stream=comp)
        ev_k[k].record(comp)
        cps[k].wait_event(ev_k[k])
        with torch.cuda.stream(cps[k]):
            h_outs[k].copy_(d_outs[k], non_blocking=True)

    def drain():
        comp.wait_stream(cps[0])
        comp.wait_stream(cps[1])

    for i in range(max(args.warmup, 2)):
        step(i)
    drain()
    torch.cuda.synchronize()
    K = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    for i in range(K):
        step(i)
    drain()
    e1.record(comp)
    torch.cuda.synchronize()
    same = None
    if out_ref is not None:
        ref = out_ref.cpu().view(-1).view(torch.uint8)
        same = all(bool(torch.equal(h.view(-1).view(torch.uint8), ref)) for h in h_outs)
    return {"ms": e0.elapsed_time(e1) / K, "same": same,
            "extra_h2d": 0 if h_grp is None else h_grp.numel() * h_grp.element_size()}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="cfg3", choices=sorted(WORKLOADS),
                    help="cfg3 (the largest single-GPU configuration) by default")
    ap.add_argument("--num-ctas", type=int, default=0)
    ap.add_argument("--num-seqs", type=int, default=0,
                    help="override the workload's batch (profiling a smaller case)")
    ap.add_argument("--spinup-ms", type=float, default=400.0,
                    help="minimum untimed warm-up time (clock ramp-up)")
    ap.add_argument("--ref-budget", type=float, default=15.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-protocol", action="store_true",
                    help="skip the median-of->=50-steps measurement after the timed region")
    ap.add_argument("--cascade", action="store_true",
                    help="prefix-sharing workloads: read each shared prefix once per group")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--measure", default="decode", choices=["decode", "swap", "block_manager", "prefill"],
                    help="decode (the hot path), or a widened row: swap_blocks / host block manager")
    ap.add_argument("--swap-blocks", type=int, default=4096)
    ap.add_argument("--prefill-budget", type=int, default=8192, choices=[2048, 8192])
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)   # at least 3 untimed warm-up steps
    if args.measure == "swap":
        return run_swap(args)
    if args.measure == "block_manager":
        return run_block_manager(args)
    if args.measure == "prefill":
        return run_prefill(args)
    return run_reference(args) if args.impl == "reference" else run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
