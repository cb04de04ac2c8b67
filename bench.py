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

def algorithmic_bytes(w, bits):
    """HBM bytes one decode call must move: reference K/V, codes, scales, q, out."""
    heads_t = w.batch * w.kv_heads * w.ctx
    b = 2 * heads_t * w.head_dim * 2
    if bits != 16:
        b += 2 * heads_t * w.head_dim * bits // 8 + 2 * heads_t * (w.head_dim // w.group) * 2
    b += w.batch * w.q_heads * w.head_dim * (2 + 4)
    return b


class DecodeStep:
    """Device-resident cache of every layer plus the per-step inputs.

    Cache arrays are contiguous across layers, [layers][K, V][B][Hkv][T][...],
    so the step's append-encode covers every layer in one call."""

    def __init__(self, w, device):
        import torch
        import kv_cache_residual_rq_b200 as rq
        from kv_cache_residual_rq_b200 import synth
        self.w, self.rq, self.torch = w, rq, torch
        L, N, B, H, T, d = w.loops, w.layers, w.batch, w.kv_heads, w.ctx, w.head_dim
        self.shape = rq.make_shape(B, H, T, d, w.group, w.q_heads)
        cache_shape = rq.make_shape(N * 2 * B, H, T, d, w.group)
        self.ref = torch.empty((N, 2, B, H, T, d), dtype=torch.bfloat16, device=device)
        self.codes = [rq.alloc_codes(cache_shape, b, device) for b in w.bits]
        self.scales = [rq.alloc_scales(cache_shape, b, device) for b in w.bits]
        # exact bytes of one (layer, K or V) part: parts are packed back to back
        self.code_bytes = [B * H * T * d * b // 8 for b in w.bits]
        self.scale_bytes = [B * H * T * (d // w.group) * 2 for b in w.bits]
        assert all(n % 16 == 0 for n in self.code_bytes + self.scale_bytes)
        layer_shape = rq.make_shape(B, H, T, d, w.group)
        for layer in range(N):
            for kind in (0, 1):
                r = synth.reference(w, layer, kind, device)
                self.ref[layer, kind].copy_(r)
                loops = [synth.loop_kv(w, layer, kind, l, r) for l in range(1, L)]
                part = layer * 2 + kind
                rq.rq_encode(layer_shape, loops, self.ref[layer, kind], list(w.bits), w.seed,
                             [self._slice(self.codes[l], self.code_bytes[l], part)
                              for l in range(L - 1)],
                             [self._slice(self.scales[l], self.scale_bytes[l], part)
                              for l in range(L - 1)])
                del loops, r
            torch.cuda.empty_cache()
        # per-step inputs: one query per (loop, layer), and the new token's K/V
        # of every loop and layer ([loop][layer][K, V][B][Hkv][1][d])
        self.q = torch.stack([torch.stack([synth.query(w, layer, loop, device)
                                           for layer in range(N)]) for loop in range(1, L + 1)])
        g = torch.Generator(device=device)
        g.manual_seed(w.seed * 31 + 7)
        newref = torch.randn((N, 2, B, H, 1, d), generator=g, device=device)
        self.new_kv = torch.stack(
            [(newref + w.sigma[l] * torch.randn(newref.shape, generator=g, device=device))
             .to(torch.bfloat16) for l in range(L - 1)] + [newref.to(torch.bfloat16)])
        self.append_shape = rq.make_shape(N * 2 * B, H, 1, d, w.group)
        self.out = torch.empty((L, N, B, w.q_heads, d), dtype=torch.float32, device=device)
        self.ws = rq.alloc_workspace(self.shape, device)
        self.ws_bytes = self.ws.numel()
        self.launches_per_step = L * N + 1

    @staticmethod
    def _slice(buf, nbytes, part):
        return buf[part * nbytes:(part + 1) * nbytes]

    def run(self, stream, timers=None, bufs=None):
        """One decode step: every (loop, layer) attends over the cache plus the
        new token's BF16 K/V of that loop; then the new token is encoded into
        the cache (the last slot is reused every step, so T stays fixed).
        timers: list to append (start, end, bits, calls) per loop segment --
        events only at loop boundaries, so consecutive calls of a loop stay
        back to back and each launch overlaps its predecessor's tail
        (programmatic dependent launch); an event between two launches would
        serialise them.  bufs: (q, new_kv, out) tensors to use instead of the
        step's own (double-buffered end-to-end loop)."""
        rq, w, torch = self.rq, self.w, self.torch
        st = stream.cuda_stream
        q_all, kv_all, out_all = bufs if bufs is not None else (self.q, self.new_kv, self.out)
        T = w.ctx
        for li in range(w.loops):
            bits = w.bits[li] if li < w.loops - 1 else 16
            ev = None
            if timers is not None:
                ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                ev[0].record(stream)
            for layer in range(w.layers):
                ck = cv = sk = sv = None
                if bits != 16:
                    ck = self._slice(self.codes[li], self.code_bytes[li], 2 * layer)
                    cv = self._slice(self.codes[li], self.code_bytes[li], 2 * layer + 1)
                    sk = self._slice(self.scales[li], self.scale_bytes[li], 2 * layer)
                    sv = self._slice(self.scales[li], self.scale_bytes[li], 2 * layer + 1)
                rq.rq_decode_attention_tail(
                    self.shape, q_all[li, layer], self.ref[layer, 0], self.ref[layer, 1],
                    ck, cv, sk, sv, bits, w.seed, 0.0, kv_all[li, layer, 0],
                    kv_all[li, layer, 1], 1, 1, out_all[li, layer], self.ws, self.ws_bytes, st)
            if ev is not None:
                ev[1].record(stream)
                timers.append((ev[0], ev[1], bits, w.layers))
        rq.rq_encode_at(self.append_shape, 1, 0, T, T - 1, list(kv_all[:w.loops - 1]),
                        kv_all[w.loops - 1], list(w.bits), w.seed, self.codes, self.scales,
                        self.ref, st)

    def step_bytes(self):
        w = self.w
        total = 0
        for li in range(w.loops):
            bits = w.bits[li] if li < w.loops - 1 else 16
            total += w.layers * algorithmic_bytes(w, bits)
        return total


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


def oracle_head_seconds(w, n_res, n_ref, seed_offset=0):
    """Time the oracle's decode attention on sampled heads of layer 0.

    Returns (seconds per residual head, seconds per reference head).  Inputs
    are the workload's generator run on the CPU; the oracle encodes them
    itself (not timed), then its decode attention is timed."""
    import oracle
    rk, rv, xk, xv, q = _oracle_inputs(w)
    bits = w.bits[0]
    t_res = t_ref = 0.0
    for i in range(n_res):
        h = (i + seed_offset) % w.kv_heads
        ck, sk, _ = oracle.encode_rows_f32(xk[h], rk[h], bits, w.group, w.seed)
        cv, sv, _ = oracle.encode_rows_f32(xv[h], rv[h], bits, w.group, w.seed)
        qh = q[h * w.G:(h + 1) * w.G]
        t0 = time.perf_counter()
        oracle.decode_attention_f64(qh, rk[h], rv[h], ck, cv, sk, sv, bits, w.group, w.seed)
        t_res += time.perf_counter() - t0
    for i in range(n_ref):
        h = (i + seed_offset) % w.kv_heads
        qh = q[h * w.G:(h + 1) * w.G]
        t0 = time.perf_counter()
        oracle.decode_attention_f64(qh, rk[h], rv[h], None, None, None, None, 16, w.group, w.seed)
        t_ref += time.perf_counter() - t0
    return t_res / max(n_res, 1), t_ref / max(n_ref, 1)


def oracle_step_seconds(w, s_res, s_ref):
    heads = w.batch * w.kv_heads
    n_res_calls = sum(1 for b in w.bits if b != 16) * w.layers
    n_ref_calls = (w.loops - 1 - sum(1 for b in w.bits if b != 16) + 1) * w.layers
    return heads * (n_res_calls * s_res + n_ref_calls * s_ref)


def cpu_baseline(w):
    n_res, n_ref = 64, 32
    t0 = time.perf_counter()
    s_res, s_ref = oracle_head_seconds(w, n_res, n_ref)
    spent = time.perf_counter() - t0
    step = oracle_step_seconds(w, s_res, s_ref)
    return {"value": w.batch / step, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": (f"fp64 oracle decode attention of {n_res} residual-INT2 heads and {n_ref} "
                       f"reference heads (T={w.ctx}, d={w.head_dim}) of one layer, "
                       f"{spent:.1f} s single-threaded, scaled to the full step "
                       f"({w.layers} layers x {w.loops} loops x {w.batch * w.kv_heads} heads); "
                       f"the append-encode (<0.1% of the step) is not included")}


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
    for i in range(args.warmup):
        oracle_head_seconds(w, 1, 1, seed_offset=i)
    times = []
    for i in range(args.steps):
        s_res, s_ref = oracle_head_seconds(w, 1, 1, seed_offset=i)
        times.append(oracle_step_seconds(w, s_res, s_ref))
    step = statistics.mean(times)
    value = w.batch / step
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; Ouro-1.4B-shaped KV, no model or dataset)",
        "config": config_dict(w, "n/a (CPU)"),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": (f"each step: fp64 oracle decode attention of 1 residual and 1 "
                                    f"reference head of layer 0, scaled to the full step")},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


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
    t_start.record(stream)
    for _ in range(args.steps):
        state.run(stream, timers)
    t_end.record(stream)
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
    e2e_loop(args.steps, e_start, e_end)
    torch.cuda.synchronize(device)
    barrier()
    e_elapsed, e_tokens = aggregate(e_start.elapsed_time(e_end) / 1e3, w.batch * args.steps)
    status = rq.rq_workspace_status(state.ws)

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
