"""Batch sweep at 32K context under a fixed KV budget: BF16 KV vs ResidualQuant.

    python -m kv_cache_residual_rq_b200.capacity [--batches 1,2,4,...] [--steps N]

The pages' capacity claim (page "ResidualQuant: KV Cache Quantization for
Looped Transformers with 2-Bit Residuals", Abstract: a larger maximum batch
and higher throughput than a BF16 KV cache) is measured here on the shapes of
the 32K-prefill workload (24 layers, 4 loops, 16 KV heads, head_dim 128,
group 32, loops 1-3 INT2):

  bf16 : every loop's K/V kept in BF16; a decode step runs one BF16
         attention call per (loop, layer) over that loop's own K/V
  rq   : the final loop in BF16 plus INT2 residuals of loops 1-3; a step
         runs the residual call for loops 1-3 and the BF16 call for loop 4
  rq_cr8 : the same with the final loop itself stored as rotated INT8 codes
         with fp16 scales (the compressed reference), the residuals taken
         against its reconstruction; a step runs the compressed-reference
         call with loop l's residual for loops 1-3 and the reference alone
         for loop 4

For every batch of the sweep the full cache size is computed; a batch whose
cache exceeds the budget (120e9 bytes, decimal) is reported as such and not
run.  A batch within budget allocates its whole 24-layer cache in HBM, fills
it from the seeded generator (the ResidualQuant cache through the library's
encoder), and runs whole decode steps over it, loop-major like a looped
model (loop 1 over all layers, then loop 2, ...); every call also attends
over the new token's own BF16 K/V of its loop.  The step is attention only
(no append), the same for both schemes.  Time: CUDA events around whole
steps, median over --steps after 3 warm-up steps.  tokens/s = batch / step
time.

Prints one JSON line per (scheme, batch).
"""
import argparse
import dataclasses
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


SCHEMES = ("bf16", "rq", "rq_cr8")
CR_REF_BITS = 8           # reference code bits of the rq_cr8 scheme


def kv_bytes_per_sequence(w, ctx, scheme):
    """KV bytes of one sequence across all layers and loops."""
    if scheme != "rq_cr8":
        return synth_kv_bytes(w, ctx, scheme == "rq")
    per_elem_bits = CR_REF_BITS + 16.0 / w.group             # reference codes + scales
    for b in w.bits:
        per_elem_bits += b + 16.0 / w.group                  # each residual loop
    return int(2 * w.layers * w.kv_heads * ctx * w.head_dim * per_elem_bits / 8)


def synth_kv_bytes(w, ctx, quantized):
    from kv_cache_residual_rq_b200 import synth
    return synth.kv_bytes_per_sequence(w, ctx, quantized)


def step_bytes(w, ctx, batch, scheme):
    """Algorithmic bytes one decode step reads (all loops and layers)."""
    heads_t = batch * w.kv_heads * ctx
    scales = 2 * (w.head_dim // w.group)                     # fp16 scale bytes per token
    if scheme == "rq_cr8":
        ref = 2 * heads_t * (w.head_dim * CR_REF_BITS // 8 + scales)   # K + V codes, scales
    else:
        ref = 2 * heads_t * w.head_dim * 2                   # K + V, bf16
    per_layer = 0
    for li in range(w.loops):
        per_layer += ref                                     # every call reads the reference
        if scheme != "bf16" and li < w.loops - 1:
            b = w.bits[li]
            per_layer += 2 * heads_t * (w.head_dim * b // 8 + scales)
    q_out = w.loops * batch * w.q_heads * w.head_dim * 6
    return w.layers * (per_layer + q_out)


class BF16Step:
    """Every loop's K/V of every layer in BF16, [loops][layers][K, V][B][Hkv][T][d],
    with the per-step inputs of DecodeStep (queries, new-token K/V)."""

    def __init__(self, w, device):
        import torch
        import kv_cache_residual_rq_b200 as rq
        from kv_cache_residual_rq_b200 import synth
        self.w, self.rq = w, rq
        L, N, B, H, T, d = w.loops, w.layers, w.batch, w.kv_heads, w.ctx, w.head_dim
        self.shape = rq.make_shape(B, H, T, d, w.group, w.q_heads)
        self.kv = torch.empty((L, N, 2, B, H, T, d), dtype=torch.bfloat16, device=device)
        for layer in range(N):
            for kind in (0, 1):
                r = synth.reference(w, layer, kind, device)
                self.kv[L - 1, layer, kind].copy_(r)
                for l in range(1, L):
                    self.kv[l - 1, layer, kind].copy_(synth.loop_kv(w, layer, kind, l, r))
                del r
            torch.cuda.empty_cache()
        self.q = torch.stack([torch.stack([synth.query(w, layer, loop, device)
                                           for layer in range(N)]) for loop in range(1, L + 1)])
        g = torch.Generator(device=device)
        g.manual_seed(w.seed * 31 + 7)
        self.new_kv = torch.randn((L, N, 2, B, H, 1, d), generator=g,
                                  device=device).to(torch.bfloat16)
        self.out = torch.empty((L, N, B, w.q_heads, d), dtype=torch.float32, device=device)
        self.ws = rq.alloc_workspace(self.shape, device)
        self.ws_bytes = self.ws.numel()

    def cache_bytes(self):
        return self.kv.numel() * 2

    def run(self, stream, append=False):
        st = stream.cuda_stream
        for li in range(self.w.loops):
            for layer in range(self.w.layers):
                self.rq.rq_decode_attention_tail(
                    self.shape, self.q[li, layer], self.kv[li, layer, 0], self.kv[li, layer, 1],
                    None, None, None, None, 16, self.w.seed, 0.0, self.new_kv[li, layer, 0],
                    self.new_kv[li, layer, 1], 1, 1, self.out[li, layer], self.ws,
                    self.ws_bytes, st)


class CRStep:
    """The rq_cr8 cache: per (layer, K or V) the final loop as INT8 reference
    codes and scales and loops 1-3 as INT2 residuals against its
    reconstruction, all from the library's compressed-reference encoder; the
    per-step inputs as in BF16Step."""

    def __init__(self, w, device):
        import torch
        import kv_cache_residual_rq_b200 as rq
        from kv_cache_residual_rq_b200 import synth
        self.w, self.rq = w, rq
        L, N, B, H, T, d = w.loops, w.layers, w.batch, w.kv_heads, w.ctx, w.head_dim
        self.shape = rq.make_shape(B, H, T, d, w.group, w.q_heads)
        # [layer][K, V] -> ((ref codes, ref scales), [codes per loop], [scales per loop])
        self.parts = []
        for layer in range(N):
            kinds = []
            for kind in (0, 1):
                r = synth.reference(w, layer, kind, device)
                loops = [synth.loop_kv(w, layer, kind, l, r) for l in range(1, L)]
                kinds.append(rq.encode_cr(loops, r, CR_REF_BITS, list(w.bits), w.group, w.seed))
                del loops, r
            self.parts.append(kinds)
            torch.cuda.empty_cache()
        self.q = torch.stack([torch.stack([synth.query(w, layer, loop, device)
                                           for layer in range(N)]) for loop in range(1, L + 1)])
        g = torch.Generator(device=device)
        g.manual_seed(w.seed * 31 + 7)
        self.new_kv = torch.randn((L, N, 2, B, H, 1, d), generator=g,
                                  device=device).to(torch.bfloat16)
        self.out = torch.empty((L, N, B, w.q_heads, d), dtype=torch.float32, device=device)
        self.ws = rq.alloc_workspace(self.shape, device)
        self.ws_bytes = self.ws.numel()

    def cache_bytes(self):
        n = 0
        for kinds in self.parts:
            for (rc, rs), codes, scales in kinds:
                n += rc.numel() + rs.numel() + sum(c.numel() for c in codes)
                n += sum(x.numel() for x in scales)
        return n

    def run(self, stream, append=False):
        st = stream.cuda_stream
        w = self.w
        for li in range(w.loops):
            res = li < w.loops - 1
            for layer in range(w.layers):
                (rck, rsk), ck, sk = self.parts[layer][0]
                (rcv, rsv), cv, sv = self.parts[layer][1]
                self.rq.rq_decode_attention_cr(
                    self.shape, None, self.q[li, layer], rck, rcv, rsk, rsv, CR_REF_BITS,
                    ck[li] if res else None, cv[li] if res else None,
                    sk[li] if res else None, sv[li] if res else None,
                    w.bits[li] if res else 16, w.seed, 0.0, self.new_kv[li, layer, 0],
                    self.new_kv[li, layer, 1], 1, 1, self.out[li, layer], self.ws,
                    self.ws_bytes, st)


def run_batch(w, ctx, batch, scheme, steps, peak, budget):
    """Allocate and fill the full cache of `batch` sequences, check it against
    the budget, time whole decode steps.  Returns the result line."""
    import torch
    import kv_cache_residual_rq_b200 as rq
    from kv_cache_residual_rq_b200 import synth
    from kv_cache_residual_rq_b200.step import DecodeStep
    dev = torch.device("cuda", torch.cuda.current_device())
    wb = dataclasses.replace(w, batch=batch, ctx=ctx)
    torch.cuda.empty_cache()
    base = torch.cuda.memory_allocated(dev)
    state = {"rq": DecodeStep, "bf16": BF16Step, "rq_cr8": CRStep}[scheme](wb, dev)
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    held = torch.cuda.memory_allocated(dev) - base
    cache = state.cache_bytes()
    if cache > budget:
        raise RuntimeError(f"{scheme} batch {batch}: cache of {cache} bytes exceeds the budget")
    stream = torch.cuda.current_stream(dev)
    for _ in range(3):
        state.run(stream, append=False)
    times = []
    torch.cuda.nvtx.range_push(f"{w.name} capacity {scheme} batch {batch}")
    for _ in range(steps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        state.run(stream, append=False)
        b.record(stream)
        torch.cuda.synchronize(dev)
        times.append(a.elapsed_time(b) / 1e3)
    torch.cuda.nvtx.range_pop()
    status = rq.rq_workspace_status(state.ws)
    finite = bool(torch.isfinite(state.out).all().item())
    times.sort()
    t = times[len(times) // 2]
    nb = step_bytes(w, ctx, batch, scheme)
    line = {"scheme": scheme, "batch": batch, "ctx": ctx, "status": "run",
            "kv_bytes": batch * kv_bytes_per_sequence(w, ctx, scheme),
            "cache_bytes_allocated": cache, "device_bytes_held": held,
            "budget_bytes": budget, "step_ms": t * 1e3, "tokens_per_s": batch / t,
            "step_bytes": nb, "gbs": nb / t / 1e9, "frac_hbm": nb / t / 1e9 / peak,
            "calls_per_step": w.loops * w.layers, "layers_resident": w.layers,
            "workspace_status": status, "outputs_finite": finite}
    del state
    torch.cuda.empty_cache()
    return line


def plan(w, ctx, batches, budget):
    """(scheme, batch, cache bytes, fits) for the sweep, plus the max batches."""
    rows = []
    maxb = {}
    for scheme in SCHEMES:
        per_seq = kv_bytes_per_sequence(w, ctx, scheme)
        maxb[scheme] = int(budget // per_seq)
        for b in batches:
            rows.append((scheme, b, b * per_seq, b * per_seq <= budget))
    return rows, maxb


def main(argv=None):
    from kv_cache_residual_rq_b200 import synth
    from kv_cache_residual_rq_b200.measure import _peak
    ap = argparse.ArgumentParser()
    ap.add_argument("--batches", default=",".join(str(b) for b in synth.SWEEP_BATCHES))
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--budget", type=float, default=synth.KV_BUDGET_BYTES)
    args = ap.parse_args(argv)
    w = synth.ENCODE
    ctx = w.ctx
    batches = [int(x) for x in args.batches.split(",")]
    rows, maxb = plan(w, ctx, batches, args.budget)
    emit = lambda d: print(json.dumps(d), flush=True)
    emit({"workload": w.name, "ctx": ctx, "budget_bytes": args.budget,
          "kv_bytes_per_sequence": {s: kv_bytes_per_sequence(w, ctx, s) for s in SCHEMES},
          "max_batch": maxb})
    peak = _peak()
    for scheme, b, kv, fits in rows:
        if not fits:
            emit({"scheme": scheme, "batch": b, "ctx": ctx, "status": "exceeds budget",
                  "kv_bytes": kv})
            continue
        emit(run_batch(w, ctx, b, scheme, args.steps, peak, args.budget))


if __name__ == "__main__":
    main()
