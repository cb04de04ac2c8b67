"""Per-workload kernel timings (one layer each), for the measured tables.

    python -m kv_cache_residual_rq_b200.measure [--workloads a,b] [--reps N] [--gqa-variants]

For every workload: the decode call of each distinct loop kind (residual INT2,
INT4, BF16 reference) over one full layer, and rq_encode of one layer's K
(all non-final loops), timed with CUDA events on the launching stream after
warm-up, inputs larger than L2 or the L2 flushed between repetitions.
Prints one JSON line per measurement with algorithmic bytes, GB/s and the
fraction of the measured HBM copy bandwidth.
"""
import argparse
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _peak():
    try:
        return float(json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["hbm_gbs"])
    except (OSError, ValueError, KeyError):
        return 6650.0


def decode_bytes(w, bits, batch=None):
    b = w.batch if batch is None else batch
    heads_t = b * w.kv_heads * w.ctx
    n = 2 * heads_t * w.head_dim * 2
    if bits != 16:
        n += 2 * heads_t * w.head_dim * bits // 8 + 2 * heads_t * (w.head_dim // w.group) * 2
    return n + b * w.q_heads * w.head_dim * 6


def cr_decode_bytes(w, rb, bits):
    """Algorithmic bytes of one decode call over a compressed reference of rb
    bits (codes and scales of K and V) plus a residual loop of `bits` (none
    for 16), q and out."""
    heads_t = w.batch * w.kv_heads * w.ctx
    per_tok = 2 * (w.head_dim * rb // 8 + 2 * (w.head_dim // w.group))
    if bits != 16:
        per_tok += 2 * (w.head_dim * bits // 8 + 2 * (w.head_dim // w.group))
    return heads_t * per_tok + w.batch * w.q_heads * w.head_dim * 6


def encode_bytes(w, rows):
    active = [b for b in w.bits if b != 16]
    read = rows * w.head_dim * 2 * (1 + len(active))
    written = sum(rows * (w.head_dim * b // 8 + 2 * w.head_dim // w.group) for b in active)
    return read + written


def _time(fn, reps, flush):
    import torch
    for _ in range(3):
        fn()
    times = []
    for _ in range(reps):
        if flush is not None:
            flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b) / 1e3)
    times.sort()
    return times[len(times) // 2]


def _to_pool(flat, B, H, T, perm):
    """A dense [B, H, T, X] cache (flat device buffer) as a pool of 64-token
    pages [pages, H, 64, X]: page (b, j) stored at pool index perm[b * P + j]."""
    import torch
    P = T // 64
    x = flat[: B * H * T * (flat.numel() // (B * H * T))].view(B, H, P, 64, -1)
    pages = x.permute(0, 2, 1, 3, 4).reshape(B * P, H, 64, -1)
    pool = torch.empty_like(pages)
    pool[perm] = pages
    return pool


def measure_paged(w, refk, refv, ck, cv, sk, sv, q, out, peak, reps, emit):
    """The loop-1 residual call with the cache scattered over a shuffled pool
    of 64-token pages (every sequence at full length): the same bytes as the
    dense call, addressed through the page table."""
    import torch
    import kv_cache_residual_rq_b200 as rq
    dev = refk.device
    B, H, T, d = w.batch, w.kv_heads, w.ctx, w.head_dim
    P = T // 64
    g = torch.Generator(device="cpu").manual_seed(w.seed * 131 + 7)
    perm = torch.randperm(B * P, generator=g).to(dev)
    table = perm.view(B, P).to(torch.int32).contiguous()
    u8 = lambda t: t.contiguous().view(torch.uint8).view(-1)
    pk, pv = _to_pool(u8(refk), B, H, T, perm), _to_pool(u8(refv), B, H, T, perm)
    pck, pcv = _to_pool(ck, B, H, T, perm), _to_pool(cv, B, H, T, perm)
    psk, psv = _to_pool(sk, B, H, T, perm), _to_pool(sv, B, H, T, perm)
    shape = rq.make_shape(B, H, T, d, w.group, w.q_heads)
    lens = torch.full((B,), T, dtype=torch.int32, device=dev)
    ws = rq.alloc_workspace(shape, dev, varlen=True)
    b = w.bits[0]
    fn = lambda: rq.rq_decode_attention_paged(shape, lens, table, P, B * P, q, pk, pv, pck, pcv,
                                              psk, psv, b, w.seed, 0.0, None, None, 0, 0, out,
                                              ws)
    t = _time(fn, reps, None)
    nb = decode_bytes(w, b)
    emit({"workload": w.name, "kernel": f"decode paged bits={b} (shuffled 64-token pages)",
          "G": w.G, "us": t * 1e6, "bytes": nb, "gbs": nb / t / 1e9, "frac": nb / t / 1e9 / peak})
    assert rq.rq_workspace_status(ws) == 0


def measure(w, reps, peak, emit):
    import torch
    import kv_cache_residual_rq_b200 as rq
    from kv_cache_residual_rq_b200 import synth
    dev = torch.device("cuda:0")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # > L2
    refk = synth.reference(w, 0, 0, dev)
    refv = synth.reference(w, 0, 1, dev)
    q = synth.query(w, 0, 1, dev)
    xk = [synth.loop_kv(w, 0, 0, l, refk) for l in range(1, w.loops)]
    rows = refk.numel() // w.head_dim
    t = _time(lambda: rq.encode(xk, refk, list(w.bits), w.group, w.seed), reps, flush)
    nb = encode_bytes(w, rows)
    emit({"workload": w.name, "kernel": "encode", "rows": rows, "loops": len(w.bits),
          "us": t * 1e6, "bytes": nb, "gbs": nb / t / 1e9, "frac": nb / t / 1e9 / peak})
    for it in (1, 4):
        t = _time(lambda: rq.encode(xk, refk, list(w.bits), w.group, w.seed, refine_iters=it),
                  reps, flush)
        emit({"workload": w.name, "kernel": f"encode refits={it}", "rows": rows,
              "loops": len(w.bits), "us": t * 1e6, "bytes": nb, "gbs": nb / t / 1e9,
              "frac": nb / t / 1e9 / peak})
    ck, sk = rq.encode(xk, refk, list(w.bits), w.group, w.seed)
    xv = [synth.loop_kv(w, 0, 1, l, refv) for l in range(1, w.loops)]
    cv, sv = rq.encode(xv, refv, list(w.bits), w.group, w.seed)
    del xk, xv
    torch.cuda.empty_cache()
    shape = rq.make_shape(w.batch, w.kv_heads, w.ctx, w.head_dim, w.group, w.q_heads)
    ws = rq.alloc_workspace(shape, dev)
    out = torch.empty((w.batch, w.q_heads, w.head_dim), dtype=torch.float32, device=dev)
    kinds = {}
    for l, b in enumerate(w.bits):
        kinds.setdefault(b, l)
    kinds.setdefault(16, None)
    for b, l in sorted(kinds.items()):
        args = (None,) * 4 if b == 16 else (ck[l], cv[l], sk[l], sv[l])
        fn = lambda: rq.rq_decode_attention(shape, q, refk, refv, *args, b, w.seed, 0.0, out, ws)
        t = _time(fn, reps, None)
        nb = decode_bytes(w, b)
        emit({"workload": w.name, "kernel": f"decode bits={b}", "G": w.G, "us": t * 1e6,
              "bytes": nb, "gbs": nb / t / 1e9, "frac": nb / t / 1e9 / peak,
              "tokens_per_s_per_head_call": w.batch / t})
    assert rq.rq_workspace_status(ws) == 0
    if w.name in ("ouro1.4b_decode", "deep_loop_gqa"):
        measure_paged(w, refk, refv, ck[0], cv[0], sk[0], sv[0], q, out, peak, reps, emit)
        torch.cuda.empty_cache()
    if w.name in ("ouro1.4b_decode", "deep_loop_gqa"):
        # compressed reference (reference loop as rotated INT8 / INT4 codes)
        xk1 = synth.loop_kv(w, 0, 0, 1, refk)
        xv1 = synth.loop_kv(w, 0, 1, 1, refv)
        for rb in (8, 4):
            t = _time(lambda: rq.encode_cr([xk1], refk, rb, [2], w.group, w.seed), reps, flush)
            nb_e = (rows * w.head_dim * 2 * 2 + rows * (w.head_dim * (rb + 2) // 8
                                                      + 2 * 2 * (w.head_dim // w.group)))
            emit({"workload": w.name, "kernel": f"encode compressed ref INT{rb} + 1 loop INT2",
                  "us": t * 1e6, "bytes": nb_e, "gbs": nb_e / t / 1e9,
                  "frac": nb_e / t / 1e9 / peak})
            (rck, rsk), ckc, skc = rq.encode_cr([xk1], refk, rb, [2], w.group, w.seed)
            (rcv, rsv), cvc, svc = rq.encode_cr([xv1], refv, rb, [2], w.group, w.seed)
            for b in (2, 16):
                nb = cr_decode_bytes(w, rb, b)
                args = (ckc[0], cvc[0], skc[0], svc[0]) if b != 16 else (None,) * 4
                fn = lambda: rq.rq_decode_attention_cr(shape, None, q, rck, rcv, rsk, rsv, rb,
                                                       *args, b, w.seed, 0.0, None, None, 0, 0,
                                                       out, ws)
                t = _time(fn, reps, None)
                emit({"workload": w.name, "kernel": f"decode compressed ref INT{rb} bits={b}",
                      "G": w.G, "us": t * 1e6, "bytes": nb, "gbs": nb / t / 1e9,
                      "frac": nb / t / 1e9 / peak})
            assert rq.rq_workspace_status(ws) == 0
            del rck, rsk, ckc, skc, rcv, rsv, cvc, svc
        del xk1, xv1
        torch.cuda.empty_cache()
    if w.G == 1 and w.name == "ouro1.4b_decode":
        # variable-length batch: seeded lengths in [ctx/8, ctx], the cache at
        # full capacity; bytes are those of the tokens actually present
        g = torch.Generator().manual_seed(w.seed * 977 + 5)
        lens = torch.randint(w.ctx // 8, w.ctx + 1, (w.batch,), generator=g, dtype=torch.int32)
        lens_d = lens.to(dev)
        wsv = rq.alloc_workspace(shape, dev, varlen=True)
        b = w.bits[0]
        fn = lambda: rq.rq_decode_attention_varlen(shape, lens_d, q, refk, refv, ck[0], cv[0],
                                                   sk[0], sv[0], b, w.seed, 0.0, None, None, 0,
                                                   0, out, wsv)
        t = _time(fn, reps, None)
        per_tok = 4 * w.head_dim + 2 * w.head_dim * b // 8 + 4 * (w.head_dim // w.group)
        nb = int(lens.sum()) * w.kv_heads * per_tok + w.batch * w.q_heads * w.head_dim * 6
        emit({"workload": w.name, "kernel": f"decode varlen bits={b}", "G": w.G,
              "lens": lens.tolist(), "us": t * 1e6, "bytes": nb, "gbs": nb / t / 1e9,
              "frac": nb / t / 1e9 / peak})
        assert rq.rq_workspace_status(wsv) == 0


def measure_gqa_variants(reps, peak, emit):
    """Deep-loop shapes (B 32, Hkv 8, G 4, T 8192, d 128) with the residual
    formats the configured workload does not use: INT4 with 64- and 32-dim
    scale groups, INT2 with 32-dim groups (the configured call is INT2 with
    64-dim groups)."""
    import dataclasses
    import torch
    import kv_cache_residual_rq_b200 as rq
    from kv_cache_residual_rq_b200 import synth
    dev = torch.device("cuda:0")
    base = synth.DEEP
    for bits, group in ((4, 64), (4, 32), (2, 32)):
        w = dataclasses.replace(base, group=group, bits=(bits,) * (base.loops - 1))
        refk = synth.reference(w, 0, 0, dev)
        refv = synth.reference(w, 0, 1, dev)
        q = synth.query(w, 0, 1, dev)
        (ck,), (sk,) = rq.encode([synth.loop_kv(w, 0, 0, 1, refk)], refk, [bits], group, w.seed)
        (cv,), (sv,) = rq.encode([synth.loop_kv(w, 0, 1, 1, refv)], refv, [bits], group, w.seed)
        shape = rq.make_shape(w.batch, w.kv_heads, w.ctx, w.head_dim, group, w.q_heads)
        ws = rq.alloc_workspace(shape, dev)
        out = torch.empty((w.batch, w.q_heads, w.head_dim), dtype=torch.float32, device=dev)
        fn = lambda: rq.rq_decode_attention(shape, q, refk, refv, ck, cv, sk, sv, bits, w.seed,
                                            0.0, out, ws)
        t = _time(fn, reps, None)
        nb = decode_bytes(w, bits)
        emit({"workload": f"{w.name} shapes", "kernel": f"decode bits={bits} group={group}",
              "G": w.G, "us": t * 1e6, "bytes": nb, "gbs": nb / t / 1e9,
              "frac": nb / t / 1e9 / peak})
        assert rq.rq_workspace_status(ws) == 0
        del refk, refv, ck, cv, sk, sv, ws, out
        torch.cuda.empty_cache()


def measure_cr_long(reps, peak, emit, batches=(1, 4, 16)):
    """The compressed-reference decode (INT8 reference + one INT2 loop, and
    the reference alone) at the 32K-prefill workload's shapes (16 KV heads,
    32K context, one layer) for several batches: single launches (median of
    `reps`) and ten back-to-back launches (best of three)."""
    import dataclasses
    import torch
    import kv_cache_residual_rq_b200 as rq
    from kv_cache_residual_rq_b200 import synth
    dev = torch.device("cuda", torch.cuda.current_device())
    for B in batches:
        w = dataclasses.replace(synth.ENCODE, batch=B)
        refk, refv = synth.reference(w, 0, 0, dev), synth.reference(w, 0, 1, dev)
        q = synth.query(w, 0, 1, dev)
        xk, xv = synth.loop_kv(w, 0, 0, 1, refk), synth.loop_kv(w, 0, 1, 1, refv)
        (rck, rsk), ck, sk = rq.encode_cr([xk], refk, 8, [2], w.group, w.seed)
        (rcv, rsv), cv, sv = rq.encode_cr([xv], refv, 8, [2], w.group, w.seed)
        del xk, xv, refk, refv
        torch.cuda.empty_cache()
        shape = rq.make_shape(B, w.kv_heads, w.ctx, w.head_dim, w.group, w.q_heads)
        ws = rq.alloc_workspace(shape, dev)
        out = torch.empty((B, w.q_heads, w.head_dim), dtype=torch.float32, device=dev)
        for b in (2, 16):
            args = (ck[0], cv[0], sk[0], sv[0]) if b != 16 else (None,) * 4
            fn = lambda: rq.rq_decode_attention_cr(shape, None, q, rck, rcv, rsk, rsv, 8, *args,
                                                   b, w.seed, 0.0, None, None, 0, 0, out, ws)
            t_iso = _time(fn, reps, None)
            best = float("inf")
            for _ in range(3):
                a = torch.cuda.Event(enable_timing=True)
                e = torch.cuda.Event(enable_timing=True)
                a.record()
                for _ in range(10):
                    fn()
                e.record()
                torch.cuda.synchronize()
                best = min(best, a.elapsed_time(e) / 1e3 / 10)
            nb = cr_decode_bytes(w, 8, b)
            emit({"workload": f"encode_prefill_32k batch {B}",
                  "kernel": f"decode compressed ref INT8 bits={b}", "G": w.G,
                  "us": t_iso * 1e6, "us_back_to_back": best * 1e6, "bytes": nb,
                  "gbs": nb / t_iso / 1e9, "frac": nb / t_iso / 1e9 / peak,
                  "frac_back_to_back": nb / best / 1e9 / peak})
        assert rq.rq_workspace_status(ws) == 0
        del rck, rsk, rcv, rsv, ck, cv, sk, sv, ws, out
        torch.cuda.empty_cache()


def main(argv=None):
    from kv_cache_residual_rq_b200 import synth
    ap = argparse.ArgumentParser()
    ap.add_argument("--workloads", default=",".join(w.name for w in synth.WORKLOADS))
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--gqa-variants", action="store_true",
                    help="also time the deep-loop shapes with INT4 residuals (64- and 32-dim "
                         "groups) and INT2 with 32-dim groups")
    ap.add_argument("--cr-long", action="store_true",
                    help="also time the compressed-reference decode at 32K context for "
                         "batches 1, 4, 16 (isolated and back to back)")
    args = ap.parse_args(argv)
    peak = _peak()
    emit = lambda d: print(json.dumps(d), flush=True)
    for name in args.workloads.split(",") if args.workloads else []:
        measure(synth.BY_NAME[name], args.reps, peak, emit)
    if args.gqa_variants:
        measure_gqa_variants(args.reps, peak, emit)
    if args.cr_long:
        measure_cr_long(args.reps, peak, emit)


if __name__ == "__main__":
    main()


# ---------------------------------------------------------------------------
# the bench's per-workload block: back-to-back launches with sampled clocks
# ---------------------------------------------------------------------------

def _back_to_back(fn, stream, target_s, sampler, label="timed launches"):
    """Average duration of `fn` launched back to back on `stream` (CUDA events
    around n launches, n chosen so the timed region lasts about target_s),
    with the SM clock sampled during the timed region."""
    import time
    import torch
    for _ in range(3):
        fn()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(3):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    est = a.elapsed_time(b) / 3e3
    n = int(min(5000, max(10, target_s / max(est, 1e-6))))
    if sampler is not None:
        sampler.start()
        time.sleep(0.25)
    torch.cuda.nvtx.range_push(label)
    a.record(stream)
    for _ in range(n):
        fn()
    b.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    clk = sampler.stop() if sampler is not None else {}
    return a.elapsed_time(b) / 1e3 / n, n, clk


def _entry(name, t, n, clk, nbytes, peak, **extra):
    mhz = clk.get("sm_mhz")
    e = {"name": name, "us": round(t * 1e6, 2), "launches": n, "bytes": nbytes,
         "gbs": round(nbytes / t / 1e9, 1), "frac": round(nbytes / t / 1e9 / peak, 4),
         "sm_mhz": mhz, "kcycles": round(t * 1e6 * mhz / 1e3, 1) if mhz else None}
    if clk.get("reasons"):
        e["reasons"] = clk["reasons"]
    e.update(extra)
    return e


def bench_workloads(peak, make_sampler, target_s=0.4):
    """Entries for the bench's `workloads` block: the configured decode calls
    of the mixed-precision 32K workload (loop 1 INT4, loop 2 INT2, loop 4 BF16)
    and of the deep-loop grouped-query workload (INT2 loop, BF16 reference),
    one full layer each (every call streams more than 1 GB, far beyond L2);
    the compressed-reference format's call (INT8 reference + the first INT2
    loop) on the Ouro-shaped and deep-loop layers, beside the same loop over
    the BF16 reference; and rq_encode of the whole 32K prefill (24 layers x
    K/V x 4 loops in one call, 25.8 GB read).  make_sampler() returns a clock
    sampler with start()/stop()."""
    import torch
    import kv_cache_residual_rq_b200 as rq
    from kv_cache_residual_rq_b200 import synth
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    st = stream.cuda_stream
    out_entries = []

    for w, loops in ((synth.MIXED, (1, 2, None)), (synth.DEEP, (1, None))):
        refk = synth.reference(w, 0, 0, dev)
        refv = synth.reference(w, 0, 1, dev)
        shape = rq.make_shape(w.batch, w.kv_heads, w.ctx, w.head_dim, w.group, w.q_heads)
        ws = rq.alloc_workspace(shape, dev)
        out = torch.empty((w.batch, w.q_heads, w.head_dim), dtype=torch.float32, device=dev)
        per_call = {}
        for loop in loops:
            if loop is None:
                bits, args = 16, (None,) * 4
                q = synth.query(w, 0, w.loops, dev)
            else:
                bits = w.bits[loop - 1]
                (ck,), (sk,) = rq.encode([synth.loop_kv(w, 0, 0, loop, refk)], refk, [bits],
                                         w.group, w.seed)
                (cv,), (sv,) = rq.encode([synth.loop_kv(w, 0, 1, loop, refv)], refv, [bits],
                                         w.group, w.seed)
                args = (ck, cv, sk, sv)
                q = synth.query(w, 0, loop, dev)
            fn = lambda: rq.rq_decode_attention(shape, q, refk, refv, *args, bits, w.seed, 0.0,
                                                out, ws, stream=st)
            label = f"loop {loop} INT{bits}" if loop else f"loop {w.loops} BF16 reference"
            t, n, clk = _back_to_back(fn, stream, target_s, make_sampler(),
                                      f"{w.name} decode {label}")
            per_call[bits] = t
            out_entries.append(_entry(f"{w.name} decode {label}", t, n, clk,
                                      decode_bytes(w, bits), peak, G=w.G))
            del args
            torch.cuda.empty_cache()
        assert rq.rq_workspace_status(ws) == 0
        # the configured step from these per-call times: every non-final loop
        # at its bits, the final loop BF16, over all layers
        step_s = w.layers * (sum(per_call[b] for b in w.bits) + per_call[16])
        out_entries[-1]["step_tokens_per_s_from_calls"] = round(w.batch / step_s, 1)
        del refk, refv, ws, out
        torch.cuda.empty_cache()

    # the compressed-reference format (next to the BF16-reference call of the
    # same loop on the same layer)
    for w in (synth.BY_NAME["ouro1.4b_decode"], synth.DEEP):
        refk = synth.reference(w, 0, 0, dev)
        refv = synth.reference(w, 0, 1, dev)
        shape = rq.make_shape(w.batch, w.kv_heads, w.ctx, w.head_dim, w.group, w.q_heads)
        ws = rq.alloc_workspace(shape, dev)
        out = torch.empty((w.batch, w.q_heads, w.head_dim), dtype=torch.float32, device=dev)
        q = synth.query(w, 0, 1, dev)
        xk1 = synth.loop_kv(w, 0, 0, 1, refk)
        xv1 = synth.loop_kv(w, 0, 1, 1, refv)
        bits = w.bits[0]
        if w is not synth.DEEP:          # (the deep-loop BF16-reference call is above)
            (ck,), (sk,) = rq.encode([xk1], refk, [bits], w.group, w.seed)
            (cv,), (sv,) = rq.encode([xv1], refv, [bits], w.group, w.seed)
            fn = lambda: rq.rq_decode_attention(shape, q, refk, refv, ck, cv, sk, sv, bits,
                                                w.seed, 0.0, out, ws, stream=st)
            label = f"{w.name} decode loop 1 INT{bits} over the BF16 reference"
            t, n, clk = _back_to_back(fn, stream, target_s, make_sampler(), label)
            out_entries.append(_entry(label, t, n, clk, decode_bytes(w, bits), peak, G=w.G))
            del ck, cv, sk, sv
        (rck, rsk), (cck,), (csk,) = rq.encode_cr([xk1], refk, 8, [bits], w.group, w.seed)
        (rcv, rsv), (ccv,), (csv,) = rq.encode_cr([xv1], refv, 8, [bits], w.group, w.seed)
        del xk1, xv1
        fn = lambda: rq.rq_decode_attention_cr(shape, None, q, rck, rcv, rsk, rsv, 8, cck, ccv,
                                               csk, csv, bits, w.seed, 0.0, None, None, 0, 0,
                                               out, ws, stream=st)
        label = f"{w.name} decode compressed reference INT8 + loop 1 INT{bits}"
        t, n, clk = _back_to_back(fn, stream, target_s, make_sampler(), label)
        out_entries.append(_entry(label, t, n, clk, cr_decode_bytes(w, 8, bits), peak, G=w.G))
        assert rq.rq_workspace_status(ws) == 0
        del refk, refv, ws, out, rck, rsk, cck, csk, rcv, rsv, ccv, csv
        torch.cuda.empty_cache()

    # the whole 32K prefill encode in one call
    w = synth.ENCODE
    N, H, T, d = w.layers, w.kv_heads, w.ctx, w.head_dim
    rows_batch = N * 2 * w.batch
    x = torch.empty((w.loops, rows_batch, H, T, d), dtype=torch.bfloat16, device=dev)
    for layer in range(N):
        for kind in (0, 1):
            r = synth.reference(w, layer, kind, dev)
            part = slice((layer * 2 + kind) * w.batch, (layer * 2 + kind + 1) * w.batch)
            x[w.loops - 1, part].copy_(r)
            for l in range(1, w.loops):
                x[l - 1, part].copy_(synth.loop_kv(w, layer, kind, l, r))
            del r
    shape = rq.make_shape(rows_batch, H, T, d, w.group)
    codes = [rq.alloc_codes(shape, b, dev) for b in w.bits]
    scales = [rq.alloc_scales(shape, b, dev) for b in w.bits]
    fn = lambda: rq.rq_encode(shape, list(x[:w.loops - 1]), x[w.loops - 1], list(w.bits),
                              w.seed, codes, scales, st)
    t, n, clk = _back_to_back(fn, stream, target_s, make_sampler(), f"{w.name} encode")
    nb = encode_bytes(w, rows_batch * H * T)
    out_entries.append(_entry(f"{w.name} encode (24 layers x K/V x {w.loops} loops, one call)",
                              t, n, clk, nb, peak, rows=rows_batch * H * T))
    del x, codes, scales
    torch.cuda.empty_cache()
    return out_entries
