#!/usr/bin/env python
"""Benchmark of the ResidualQuant decode step on B200.

One step = one decode step of the looped model over every layer and loop
(loop 1 .. L-1 read residual codes, loop L the BF16 reference); each call
attends over the cached tokens plus the new token's own BF16 K/V of that loop,
and the step ends with the append-encode of the new token into the cache (its
L-1 non-final loops against its final loop, all layers in one call).  Workload: the Ouro-1.4B-shaped
decode (24 layers x 4 loops, batch 16, ctx 4096, 16 heads MHA, head_dim 128,
INT2 residuals with group 32), synthetic seeded data.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs its own copy of the workload (weak scaling);
the timed region is bracketed by a barrier and a device synchronize, the
elapsed time is the max over ranks.  Rank 0 prints one JSON line.

Besides the headline (the --steps timed region) the line carries:
  sustained   the same step held for --sustain-s seconds, with its own clock
              record (the 1 kW power cap lowers the SM clock in steady state)
  workloads   (N=1) the other configured workloads, timed in the same run
              with CUDA events around back-to-back launches and the SM clock
              sampled meanwhile: the mixed-precision 32K decode calls (loop 1
              INT4, loop 2 INT2, loop 4 BF16), the deep-loop grouped-query
              decode calls (INT2, BF16), the whole 32K-prefill rq_encode in one
              call, and the budgeted batch sweep's maximum batches with their
              full 24-layer caches allocated in HBM
  cpu_baseline (N=1) the oracle on this host's cores: decode on one thread
              and on every core, and the encoder's GB/s
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode attn tokens/s over residual-INT2 KV; HBM GB/s vs B200 peak"
UNIT = "tokens/s"
WORKLOAD = "ouro1.4b_decode"


# ---------------------------------------------------------------------------
# distributed helpers (also exercised by the CPU multi-rank test)
# ---------------------------------------------------------------------------

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def aggregate(elapsed_s, units, group=None):
    """(max elapsed over ranks, total units over ranks)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return elapsed_s, units
    dev = "cuda" if dist.get_backend(group) == "nccl" else "cpu"
    t = torch.tensor([elapsed_s], dtype=torch.float64, device=dev)
    u = torch.tensor([float(units)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    dist.all_reduce(u, op=dist.ReduceOp.SUM, group=group)
    return float(t.item()), float(u.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------

CLOCK_FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
                "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                "clocks_event_reasons.sw_power_cap")
REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


class ClockSampler:
    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_id), f"--query-gpu={CLOCK_FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, active = [], [], set()
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(REASONS, parts[3:7]):
                if val.lower().startswith("active"):
                    active.add(name)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(active), "samples": len(sm)}


def gpu_id_for(device_index):
    import torch
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
    except Exception:
        return device_index


# ---------------------------------------------------------------------------
# workload
# ---------------------------------------------------------------------------

from kv_cache_residual_rq_b200.step import DecodeStep, algorithmic_bytes  # noqa: E402


# the sources that make up the single-query decode kernel the roofline names
DECODE_SOURCES = ("rq_decode.cu", "rq_decode_common.cuh", "rq_device.cuh", "rq_internal.h")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_ouro1.4b_traffic.json")


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "kv_cache_residual_rq_b200", "csrc")
    for fn in DECODE_SOURCES:
        h.update(open(os.path.join(csrc, fn), "rb").read())
    return h.hexdigest()[:16]


def record_traffic(csv_path):
    """Write the traffic file from an ncu CSV (`--csv --log-file`) of the
    decode kernel with dram__bytes_read.sum and dram__bytes_write.sum, taken
    on `python -m kv_cache_residual_rq_b200.profile_decode --tail 1` (one
    layer of the bench's workload, the bench's launch shape)."""
    import csv
    rows = [r for r in csv.reader(l for l in open(csv_path) if not l.startswith("=="))]
    head = rows[0]
    ki, mi, vi = head.index("Kernel Name"), head.index("Metric Name"), head.index("Metric Value")
    ui, idi = head.index("Metric Unit"), head.index("ID")
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9,
             "B": 1, "KB": 1e3, "MB": 1e6, "GB": 1e9}
    per = {}
    for r in rows[1:]:
        if len(r) <= vi or "decode_kernel<" not in r[ki]:
            continue
        if r[mi] in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            val = float(r[vi].replace(",", "")) * scale[r[ui]]
            per.setdefault(r[idi], {})[r[mi]] = val
    launches = [v for v in per.values() if len(v) == 2]
    if not launches:
        raise SystemExit(f"no decode_kernel launches with both DRAM metrics in {csv_path}")
    rd = sum(v["dram__bytes_read.sum"] for v in launches) / len(launches)
    wr = sum(v["dram__bytes_write.sum"] for v in launches) / len(launches)
    rec = {"kernel": "decode_kernel<128, 1, 2> (residual INT2, G = 1)",
           "workload": "ouro1.4b_decode, one call: B 16, Hkv 16, T 4096 + 1 BF16 tail token",
           "command": ("ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,"
                       "gpu__time_duration.sum --clock-control none -k regex:decode_kernel "
                       "-s 1 -c 2 --csv --log-file <csv> python -m "
                       "kv_cache_residual_rq_b200.profile_decode --tail 1 --calls 3"),
           "launches": len(launches), "dram_bytes_read": rd, "dram_bytes_write": wr,
           "dram_bytes_per_launch": rd + wr, "kernel_source_hash": kernel_source_hash()}
    with open(TRAFFIC_FILE, "w") as f:
        json.dump(rec, f, indent=1)
        f.write("\n")
    print(json.dumps(rec))


def measured_traffic(kernel_hash):
    """ncu DRAM bytes per launch of the decode kernel, if taken on this source."""
    try:
        rec = json.load(open(TRAFFIC_FILE))
    except (OSError, ValueError):
        return None
    if rec.get("kernel_source_hash") != kernel_hash:
        return None
    return rec.get("dram_bytes_per_launch")


def hbm_peak():
    try:
        pk = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        return float(pk["hbm_gbs"]), "measured"
    except (OSError, ValueError, KeyError):
        return 6650.0, "fallback"


# ---------------------------------------------------------------------------
# CPU oracle timing (the reported baseline and the reference arm)
# ---------------------------------------------------------------------------

_ORACLE_INPUTS = {}
_ORACLE_CODES = {}


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def _pool_map(fn, items, threads):
    """Run fn over items on `threads` host threads (the oracle is called
    through ctypes, which releases the GIL for the duration of each call)."""
    if threads <= 1:
        return [fn(i) for i in items]
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(threads) as ex:
        return list(ex.map(fn, items))


def _oracle_inputs(w):
    """Layer-0 inputs of one sequence on the CPU, generated once."""
    if w.name not in _ORACLE_INPUTS:
        import numpy as np
        import torch
        from kv_cache_residual_rq_b200 import synth
        u16 = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
        rk = synth.reference(w, 0, 0, "cpu", batch=1)
        rv = synth.reference(w, 0, 1, "cpu", batch=1)
        xk = synth.loop_kv(w, 0, 0, 1, rk)
        xv = synth.loop_kv(w, 0, 1, 1, rv)
        q = synth.query(w, 0, 1, "cpu", batch=1)
        _ORACLE_INPUTS[w.name] = tuple(u16(t[0]) for t in (rk, rv, xk, xv, q))
    return _ORACLE_INPUTS[w.name]


def _oracle_head_codes(w, h):
    """The oracle's own encode of kv head h's loop-1 K/V (prepared, not timed)."""
    key = (w.name, h)
    if key not in _ORACLE_CODES:
        import oracle
        rk, rv, xk, xv, _ = _oracle_inputs(w)
        ck, sk, _ = oracle.encode_rows_f32(xk[h], rk[h], w.bits[0], w.group, w.seed)
        cv, sv, _ = oracle.encode_rows_f32(xv[h], rv[h], w.bits[0], w.group, w.seed)
        _ORACLE_CODES[key] = (ck, cv, sk, sv)
    return _ORACLE_CODES[key]


def oracle_head_seconds(w, n_res, n_ref, threads=1, seed_offset=0):
    """Time the oracle's decode attention on sampled heads of layer 0, run on
    `threads` host threads.

    Returns (wall seconds per residual head, wall seconds per reference
    head): each batch of heads is timed as a whole, so with several threads
    these are throughput figures.  Inputs are the workload's generator run on
    the CPU; the oracle encodes them itself beforehand (not timed)."""
    import oracle
    oracle.lib()
    rk, rv, _, _, q = _oracle_inputs(w)
    bits = w.bits[0]
    res_heads = [(i + seed_offset) % w.kv_heads for i in range(n_res)]
    ref_heads = [(i + seed_offset) % w.kv_heads for i in range(n_ref)]
    for h in set(res_heads):
        _oracle_head_codes(w, h)

    def res(h):
        ck, cv, sk, sv = _oracle_head_codes(w, h)
        oracle.decode_attention_f64(q[h * w.G:(h + 1) * w.G], rk[h], rv[h], ck, cv, sk, sv,
                                    bits, w.group, w.seed)

    def ref(h):
        oracle.decode_attention_f64(q[h * w.G:(h + 1) * w.G], rk[h], rv[h], None, None, None,
                                    None, 16, w.group, w.seed)

    t0 = time.perf_counter()
    _pool_map(res, res_heads, threads)
    t_res = time.perf_counter() - t0
    t0 = time.perf_counter()
    _pool_map(ref, ref_heads, threads)
    t_ref = time.perf_counter() - t0
    return t_res / max(n_res, 1), t_ref / max(n_ref, 1)


def oracle_step_seconds(w, s_res, s_ref):
    heads = w.batch * w.kv_heads
    n_res_calls = sum(1 for b in w.bits if b != 16) * w.layers
    n_ref_calls = (w.loops - 1 - sum(1 for b in w.bits if b != 16) + 1) * w.layers
    return heads * (n_res_calls * s_res + n_ref_calls * s_ref)


def oracle_encode_gbs(threads, rows_per_job=16384):
    """The fp32 exact-spec oracle encoder on rows of the 32K-prefill workload
    (16 heads x rows_per_job/16 tokens of layer 0's K, its 3 INT2 loops),
    one job per thread.  Returns (GB/s of algorithmic bytes, wall seconds)."""
    import numpy as np
    import torch
    import oracle
    from kv_cache_residual_rq_b200 import synth
    from kv_cache_residual_rq_b200.measure import encode_bytes
    w = synth.ENCODE
    oracle.lib()
    key = ("encode", rows_per_job)
    if key not in _ORACLE_INPUTS:
        u16 = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
        t = rows_per_job // w.kv_heads
        rk = synth.reference(w, 0, 0, "cpu", batch=1, ctx=t)
        xs = [synth.loop_kv(w, 0, 0, l, rk) for l in range(1, w.loops)]
        _ORACLE_INPUTS[key] = (u16(rk[0]).reshape(-1, w.head_dim),
                               [u16(x[0]).reshape(-1, w.head_dim) for x in xs])
    ref, xs = _ORACLE_INPUTS[key]

    def job(_):
        for x, b in zip(xs, w.bits):
            oracle.encode_rows_f32(x, ref, b, w.group, w.seed)

    t0 = time.perf_counter()
    _pool_map(job, range(threads), threads)
    wall = time.perf_counter() - t0
    return encode_bytes(w, rows_per_job) * threads / wall / 1e9, wall


def cpu_baseline(w):
    """The oracle timed on this host: decode (the bench's metric) on one
    thread and on every core, and the encoder's GB/s likewise."""
    cores = host_cores()
    t0 = time.perf_counter()
    s_res1, s_ref1 = oracle_head_seconds(w, 32, 16, threads=1)
    single = w.batch / oracle_step_seconds(w, s_res1, s_ref1)
    s_resn, s_refn = oracle_head_seconds(w, 8 * cores, 4 * cores, threads=cores)
    multi = w.batch / oracle_step_seconds(w, s_resn, s_refn)
    enc1, _ = oracle_encode_gbs(1, 65536)
    encn, _ = oracle_encode_gbs(cores, 16384)
    spent = time.perf_counter() - t0
    return {"value": multi, "unit": UNIT, "cores": cores, "kind": "oracle",
            "extrapolated": True, "nproc": os.cpu_count(), "cpu_model": cpu_model(),
            "single_thread": {"value": single, "unit": UNIT, "cores": 1},
            "encode": {"unit": "GB/s", "single_thread": enc1, "all_cores": encn,
                       "sample": ("fp32 exact-spec oracle encoder, 3 INT2 loops of layer 0's "
                                  "K of the 32K-prefill workload: 65536 rows on 1 thread, "
                                  f"16384 rows per thread on {cores} threads")},
            "sample": (f"fp64 oracle decode attention of layer-0 heads (T={w.ctx}, "
                       f"d={w.head_dim}): {8 * cores} residual-INT2 + {4 * cores} reference "
                       f"heads on {cores} threads (value), 32 + 16 heads on 1 thread "
                       f"(single_thread), scaled to the full step ({w.layers} layers x "
                       f"{w.loops} loops x {w.batch * w.kv_heads} heads); {spent:.1f} s in "
                       f"all with the encode timing; the append-encode (<0.1% of the step) "
                       f"is not included")}


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------

def config_dict(w, l2_note):
    return {"workload": (f"{w.name}: {w.layers} layers x {w.loops} loops, batch {w.batch}, "
                         f"ctx {w.ctx}, {w.q_heads} q / {w.kv_heads} kv heads, head_dim "
                         f"{w.head_dim}, loops 1-{w.loops - 1} INT{w.bits[0]} group {w.group}, "
                         f"loop {w.loops} BF16 reference"),
            "global_batch": w.batch, "seq_len": w.ctx, "layers": w.layers, "loops": w.loops,
            "l2": l2_note}


def run_reference(args, w):
    rank, _, world = dist_env()
    if rank != 0:
        return
    cores = host_cores()
    n_res, n_ref = cores, max(1, cores // 2)
    for i in range(args.warmup):
        oracle_head_seconds(w, n_res, n_ref, threads=cores, seed_offset=i)
    times, walls = [], []
    for i in range(args.steps):
        t0 = time.perf_counter()
        s_res, s_ref = oracle_head_seconds(w, n_res, n_ref, threads=cores, seed_offset=i)
        walls.append(time.perf_counter() - t0)
        times.append(oracle_step_seconds(w, s_res, s_ref))
    step = statistics.mean(times)
    value = w.batch / step
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3,
        "extrapolated": True,
        "sampled_heads_per_step": {"residual": n_res, "reference": n_ref},
        "sample_wall_ms_per_step": statistics.mean(walls) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; Ouro-1.4B-shaped KV, no model or dataset)",
        "config": config_dict(w, "n/a (CPU)"),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "nproc": os.cpu_count(), "cpu_model": cpu_model(),
                         "sample": (f"each step: fp64 oracle decode attention of {n_res} "
                                    f"residual and {n_ref} reference heads of layer 0 on "
                                    f"{cores} threads, scaled to the full step "
                                    f"(ms_per_step is that extrapolation; the sample itself "
                                    f"took sample_wall_ms_per_step)")},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def other_workloads(peak, local_rank, args):
    """The other configured workloads, timed in this run: the mixed-precision
    32K and deep-loop grouped-query decode calls, the whole 32K-prefill
    encode, and the budgeted batch sweep at its maximum batches with the full
    caches held in HBM."""
    from kv_cache_residual_rq_b200 import capacity, measure, synth
    make_sampler = lambda: ClockSampler(gpu_id_for(local_rank))
    entries = measure.bench_workloads(peak, make_sampler)
    w = synth.ENCODE
    rows, maxb = capacity.plan(w, w.ctx, synth.SWEEP_BATCHES, synth.KV_BUDGET_BYTES)
    cap = {"budget_bytes": synth.KV_BUDGET_BYTES, "ctx": w.ctx, "max_batch": maxb,
           "exceeds_budget": sorted({f"{s} {b}" for s, b, _, ok in rows if not ok}),
           "runs": []}
    for scheme in ("rq", "bf16", "rq_cr8"):
        r = capacity.run_batch(w, w.ctx, maxb[scheme], scheme, args.capacity_steps, peak,
                               synth.KV_BUDGET_BYTES)
        cap["runs"].append({k: r[k] for k in ("scheme", "batch", "cache_bytes_allocated",
                                              "device_bytes_held", "step_ms", "tokens_per_s",
                                              "frac_hbm", "workspace_status",
                                              "outputs_finite")})
    return {"entries": entries, "capacity": cap}


def run_ours(args, w):
    import torch
    import torch.distributed as dist
    import kv_cache_residual_rq_b200 as rq
    from kv_cache_residual_rq_b200 import build as rq_build

    rank, local_rank, world = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=device)
    if rank == 0:
        rq_build.build()
    barrier()
    rq.lib()

    state = DecodeStep(w, device)
    stream = torch.cuda.current_stream(device)
    torch.cuda.synchronize(device)

    # ---- device-resident timed region ----
    for _ in range(args.warmup):
        state.run(stream)
    timers = []
    clocks = ClockSampler(gpu_id_for(local_rank))
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize(device)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push(f"{w.name} timed steps")
    t_start.record(stream)
    for _ in range(args.steps):
        state.run(stream, timers)
    t_end.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize(device)
    barrier()
    clk = clocks.stop()
    elapsed = t_start.elapsed_time(t_end) / 1e3
    max_elapsed, tokens = aggregate(elapsed, w.batch * args.steps)
    value = tokens / max_elapsed

    # average launch duration = loop segment time / calls in the segment
    res_ms = [a.elapsed_time(b) / n for a, b, bits, n in timers if bits != 16]
    ref_ms = [a.elapsed_time(b) / n for a, b, bits, n in timers if bits == 16]
    avg_res_s = statistics.mean(res_ms) / 1e3
    bytes_res = algorithmic_bytes(w, w.bits[0])
    peak, peak_kind = hbm_peak()
    achieved = bytes_res / avg_res_s / 1e9
    khash = kernel_source_hash()
    traffic = measured_traffic(khash)

    # ---- end-to-end through the public API with host buffers ----
    # Like a serving loop, inputs and outputs are double-buffered: step k+1's
    # queries and new-token K/V go up on a copy stream while step k computes,
    # and step k's outputs come back while step k+1 computes.  Every step
    # still moves its own inputs and outputs between pinned host memory and
    # the device inside the timed region.
    q_host = state.q.cpu().pin_memory()
    new_kv_host = state.new_kv.cpu().pin_memory()
    out_host = [torch.empty(state.out.shape, dtype=state.out.dtype).pin_memory()
                for _ in range(2)]
    bufs = [(state.q, state.new_kv, state.out),
            (torch.empty_like(state.q), torch.empty_like(state.new_kv),
             torch.empty_like(state.out))]
    h2d = q_host.numel() * 2 + new_kv_host.numel() * 2
    d2h = out_host[0].numel() * 4
    copy = torch.cuda.Stream(device)

    def e2e_loop(n, e_start=None, e_end=None):
        up = [None] * n

        def upload(k):
            qd, kvd, _ = bufs[k % 2]
            with torch.cuda.stream(copy):
                qd.copy_(q_host, non_blocking=True)
                kvd.copy_(new_kv_host, non_blocking=True)
            up[k] = torch.cuda.Event()
            up[k].record(copy)

        if e_start is not None:
            e_start.record(copy)
        for k in range(min(2, n)):
            upload(k)
        for k in range(n):
            stream.wait_event(up[k])
            state.run(stream, bufs=bufs[k % 2])
            done = torch.cuda.Event()
            done.record(stream)
            copy.wait_event(done)
            with torch.cuda.stream(copy):
                out_host[k % 2].copy_(bufs[k % 2][2], non_blocking=True)
            if k + 2 < n:
                upload(k + 2)      # after step k's download: its buffers are free
        if e_end is not None:
            e_end.record(copy)

    e2e_loop(args.warmup)
    barrier()
    torch.cuda.synchronize(device)
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push(f"{w.name} end-to-end steps")
    e2e_loop(args.steps, e_start, e_end)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize(device)
    barrier()
    e_elapsed, e_tokens = aggregate(e_start.elapsed_time(e_end) / 1e3, w.batch * args.steps)
    status = rq.rq_workspace_status(state.ws)

    # ---- the same step held for a few seconds (power-capped steady state) ----
    sustained = None
    if args.sustain_s > 0:
        n_sus = max(args.steps, int(args.sustain_s / (max_elapsed / args.steps)))
        sus_timers = []
        clocks = ClockSampler(gpu_id_for(local_rank))
        clocks.start()
        time.sleep(0.3)
        barrier()
        torch.cuda.synchronize(device)
        s_start = torch.cuda.Event(enable_timing=True)
        s_end = torch.cuda.Event(enable_timing=True)
        torch.cuda.nvtx.range_push(f"{w.name} sustained steps")
        s_start.record(stream)
        for _ in range(n_sus):
            state.run(stream, sus_timers)
        s_end.record(stream)
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize(device)
        barrier()
        s_clk = clocks.stop()
        s_elapsed, s_tokens = aggregate(s_start.elapsed_time(s_end) / 1e3, w.batch * n_sus)
        s_res = statistics.mean(a.elapsed_time(b) / n for a, b, bits, n in sus_timers
                                if bits != 16) / 1e3
        sustained = {"steps": n_sus, "ms_per_step": s_elapsed / n_sus * 1e3,
                     "value": s_tokens / s_elapsed, "avg_launch_us": s_res * 1e6,
                     "frac": bytes_res / s_res / 1e9 / peak, "clocks": s_clk,
                     "launch_kcycles": (s_res * 1e3 * s_clk["sm_mhz"]
                                        if s_clk.get("sm_mhz") else None)}
        del sus_timers
    status = status | rq.rq_workspace_status(state.ws)

    if rank == 0:
        step_bytes = state.step_bytes()
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": max_elapsed / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded; Ouro-1.4B-shaped KV, no model or dataset)",
            "config": dict(config_dict(w, "inputs larger than L2: each call streams "
                                          f"{bytes_res / 1e6:.0f} MB"),
                           parallelism=f"replica x{world} (independent sequences per GPU)"),
            "clocks": clk,
            "e2e": {"value": e_tokens / e_elapsed, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": state.launches_per_step * args.steps,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "launch_kcycles": (avg_res_s * 1e3 * clk["sm_mhz"]
                                            if clk.get("sm_mhz") else None),
                         "kernel": f"decode_kernel<128,1,{w.bits[0]}> (residual loop)",
                         "algorithmic_bytes_per_launch": bytes_res,
                         "avg_launch_us": avg_res_s * 1e6, "peak_source": peak_kind + " hbm_gbs",
                         "launches_timed": len(res_ms) * w.layers,
                         "timing": ("CUDA events at the loop boundaries of every timed step: "
                                    "segment time / 24 back-to-back launches")},
            "step_hbm_gbs_per_gpu": step_bytes / (max_elapsed / args.steps) / 1e9,
            "ref_loop_avg_launch_us": statistics.mean(ref_ms) * 1e3 if ref_ms else None,
            "workspace_status": status,
            "kernel_source_hash": khash,
        }
        if sustained is not None:
            line["sustained"] = sustained
        if world == 1 and not args.no_workloads:
            del state, bufs
            torch.cuda.empty_cache()
            line["workloads"] = other_workloads(peak, local_rank, args)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other workloads' block (N=1 only)")
    ap.add_argument("--sustain-s", type=float, default=3.0,
                    help="seconds of a second, longer timed region (0: skip)")
    ap.add_argument("--capacity-steps", type=int, default=3)
    ap.add_argument("--record-traffic", metavar="NCU_CSV",
                    help="write the decode kernel's ncu DRAM bytes into profiles/ and exit")
    args = ap.parse_args(argv)
    if args.record_traffic:
        record_traffic(args.record_traffic)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    from kv_cache_residual_rq_b200 import synth
    w = synth.BY_NAME[WORKLOAD]
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
