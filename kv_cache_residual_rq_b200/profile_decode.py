"""Small, self-contained decode case for profiler captures.

    python -m kv_cache_residual_rq_b200.profile_decode [--workload NAME] [--calls N] [--bits B]

Builds ONE layer of a workload on cuda:0 (for the Ouro-shaped decode: 537 MB
of reference K/V plus 84 MB of codes and scales, above the 126 MB L2),
encodes it, and runs the decode kernel `--calls` times on the same inputs,
so a profiler can capture a handful of launches of exactly the kernel the
benchmark times without holding the whole 24-layer cache on the device.
"""
import argparse
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main(argv=None):
    import torch
    import kv_cache_residual_rq_b200 as rq
    from kv_cache_residual_rq_b200 import synth

    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="ouro1.4b_decode")
    ap.add_argument("--calls", type=int, default=4)
    ap.add_argument("--bits", type=int, default=0, help="0: the workload's first loop")
    ap.add_argument("--encode", action="store_true", help="also time rq_encode of the layer")
    ap.add_argument("--tail", type=int, default=0,
                    help="BF16 tail tokens per call (1 = the benchmark's launch: cache + new token)")
    ap.add_argument("--ref-bits", type=int, default=0,
                    help="4 or 8: decode a compressed-reference cache instead")
    args = ap.parse_args(argv)
    w = synth.BY_NAME[args.workload]
    bits = args.bits or w.bits[0]
    dev = torch.device("cuda:0")
    refk = synth.reference(w, 0, 0, dev)
    refv = synth.reference(w, 0, 1, dev)
    q = synth.query(w, 0, 1, dev)
    ck = cv = sk = sv = None
    if bits != 16:
        xk = [synth.loop_kv(w, 0, 0, l, refk) for l in range(1, w.loops)]
        xv = [synth.loop_kv(w, 0, 1, l, refv) for l in range(1, w.loops)]
        bl = [bits] * (w.loops - 1)
        cks, sks = rq.encode(xk, refk, bl, w.group, w.seed)
        cvs, svs = rq.encode(xv, refv, bl, w.group, w.seed)
        if args.encode:
            for _ in range(args.calls):
                rq.encode(xk, refk, bl, w.group, w.seed)
        ck, cv, sk, sv = cks[0], cvs[0], sks[0], svs[0]
        del xk, xv
    shape = rq.make_shape(w.batch, w.kv_heads, w.ctx, w.head_dim, w.group, w.q_heads)
    ws = rq.alloc_workspace(shape, dev)
    out = torch.empty((w.batch, w.q_heads, w.head_dim), dtype=torch.float32, device=dev)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    times = []
    tail_k = tail_v = None
    if args.tail:
        g = torch.Generator(device=dev)
        g.manual_seed(w.seed * 31 + 7)
        tail_k = torch.randn((w.batch, w.kv_heads, args.tail, w.head_dim), generator=g,
                             device=dev).to(torch.bfloat16)
        tail_v = torch.randn(tail_k.shape, generator=g, device=dev).to(torch.bfloat16)
    crref = None
    if args.ref_bits:
        xk1 = synth.loop_kv(w, 0, 0, 1, refk)
        xv1 = synth.loop_kv(w, 0, 1, 1, refv)
        b1 = bits if bits != 16 else 2
        (rck, rsk), ckc, skc = rq.encode_cr([xk1], refk, args.ref_bits, [b1], w.group, w.seed)
        (rcv, rsv), cvc, svc = rq.encode_cr([xv1], refv, args.ref_bits, [b1], w.group, w.seed)
        crref = (rck, rsk, rcv, rsv, args.ref_bits)
        del xk1, xv1
    for _ in range(args.calls):
        start.record()
        if crref is not None:
            rq.decode_attention_cr(q, crref, *((ckc[0], cvc[0], skc[0], svc[0]) if bits != 16
                                              else (None,) * 4), bits, w.group, w.seed, w.ctx,
                                   out=out, workspace=ws, tail_k=tail_k, tail_v=tail_v,
                                   n_tail=args.tail, kv_heads=w.kv_heads)
        else:
            rq.decode_attention(q, refk, refv, ck, cv, sk, sv, bits, w.group, w.seed, out=out,
                                workspace=ws, tail_k=tail_k, tail_v=tail_v, n_tail=args.tail)
        end.record()
        torch.cuda.synchronize()
        times.append(start.elapsed_time(end))
    print(f"{w.name} bits={bits}: decode call ms {['%.3f' % t for t in times]}, "
          f"status {rq.rq_workspace_status(ws)}")


if __name__ == "__main__":
    main()
