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

For every batch of the sweep the full cache size is computed; a batch whose
cache exceeds the budget (120e9 bytes, decimal) is reported as such and not
run.  A batch within budget is run as a whole decode step, loop-major like a
looped model (loop 1 over all layers, then loop 2, ...), with two layers'
worth of cache resident and alternated between consecutive calls: each call
streams at least 268 MB, more than the 126 MB L2, so the bytes a step moves
are those of a full 24-layer cache.  Time: CUDA events around whole steps,
median over --steps after warm-up.  tokens/s = batch / step time.

Prints one JSON line per (scheme, batch).
"""
import argparse
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

RESIDENT_LAYERS = 2


def step_bytes(w, ctx, batch, scheme):
    """Algorithmic bytes one decode step reads (all loops and layers)."""
    heads_t = batch * w.kv_heads * ctx
    ref = 2 * heads_t * w.head_dim * 2                       # K + V, bf16
    per_layer = 0
    for li in range(w.loops):
        per_layer += ref                                     # every call reads a BF16 K/V
        if scheme == "rq" and li < w.loops - 1:
            b = w.bits[li]
            per_layer += 2 * heads_t * (w.head_dim * b // 8 + 2 * (w.head_dim // w.group))
    q_out = w.loops * batch * w.q_heads * w.head_dim * 6
    return w.layers * (per_layer + q_out)


def run_batch(w, ctx, batch, scheme, steps, emit, peak):
    import torch
    import kv_cache_residual_rq_b200 as rq
    from kv_cache_residual_rq_b200 import synth
    dev = torch.device("cuda:0")
    L = w.loops
    shape = rq.make_shape(batch, w.kv_heads, ctx, w.head_dim, w.group, w.q_heads)
    layers = []
    for layer in range(RESIDENT_LAYERS):
        ent = {}
        for kind, name in ((0, "k"), (1, "v")):
            ref = synth.reference(w, layer, kind, dev, batch=batch, ctx=ctx)
            loops = [synth.loop_kv(w, layer, kind, l, ref) for l in range(1, L)]
            if scheme == "bf16":
                ent[name] = loops + [ref]                    # loop l's own K/V
            else:
                codes, scales = rq.encode(loops, ref, list(w.bits), w.group, w.seed)
                ent[name] = ref
                ent["c" + name], ent["s" + name] = codes, scales
            del loops
        layers.append(ent)
        torch.cuda.empty_cache()
    qs = [synth.query(w, 0, li + 1, dev, batch=batch) for li in range(L)]
    out = torch.empty((batch, w.q_heads, w.head_dim), dtype=torch.float32, device=dev)
    ws = rq.alloc_workspace(shape, dev)

    def step():
        for li in range(L):
            for layer in range(w.layers):
                e = layers[layer % RESIDENT_LAYERS]
                if scheme == "bf16":
                    rq.rq_decode_attention(shape, qs[li], e["k"][li], e["v"][li], None, None,
                                           None, None, 16, w.seed, 0.0, out, ws)
                elif li < L - 1:
                    rq.rq_decode_attention(shape, qs[li], e["k"], e["v"], e["ck"][li],
                                           e["cv"][li], e["sk"][li], e["sv"][li], w.bits[li],
                                           w.seed, 0.0, out, ws)
                else:
                    rq.rq_decode_attention(shape, qs[li], e["k"], e["v"], None, None, None,
                                           None, 16, w.seed, 0.0, out, ws)

    for _ in range(3):
        step()
    times = []
    for _ in range(steps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        step()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b) / 1e3)
    assert rq.rq_workspace_status(ws) == 0
    times.sort()
    t = times[len(times) // 2]
    nb = step_bytes(w, ctx, batch, scheme)
    emit({"scheme": scheme, "batch": batch, "ctx": ctx, "status": "run",
          "kv_bytes": batch * synth.kv_bytes_per_sequence(w, ctx, scheme == "rq"),
          "step_ms": t * 1e3, "tokens_per_s": batch / t, "step_bytes": nb,
          "gbs": nb / t / 1e9, "frac_hbm": nb / t / 1e9 / peak,
          "calls_per_step": L * w.layers, "resident_layers": RESIDENT_LAYERS})
    del layers, qs, out, ws
    torch.cuda.empty_cache()


def plan(w, ctx, batches, budget):
    """(scheme, batch, cache bytes, fits) for the sweep, plus the max batches."""
    from kv_cache_residual_rq_b200 import synth
    rows = []
    maxb = {}
    for scheme in ("bf16", "rq"):
        per_seq = synth.kv_bytes_per_sequence(w, ctx, scheme == "rq")
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
          "kv_bytes_per_sequence": {s: synth.kv_bytes_per_sequence(w, ctx, s == "rq")
                                    for s in ("bf16", "rq")},
          "max_batch": maxb})
    peak = _peak()
    for scheme, b, kv, fits in rows:
        if not fits:
            emit({"scheme": scheme, "batch": b, "ctx": ctx, "status": "exceeds budget",
                  "kv_bytes": kv})
            continue
        run_batch(w, ctx, b, scheme, args.steps, emit, peak)


if __name__ == "__main__":
    main()
