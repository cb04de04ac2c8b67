"""Quality of the encoding without a model: ResidualQuant vs the rotation-only
baseline on the synthetic workloads.

    python -m kv_cache_residual_rq_b200.quality [--workloads a,b] [--heads-sample N]

The pages compare ResidualQuant with "rotation-based KV quantization" at the
same memory budget on model benchmarks (Abstract); without models, this
compares the two encodings directly on the synthetic looped-KV data:

  ResidualQuant : the final loop kept in BF16, every other loop as its
                  rotated residual against it (rq_encode with the reference)
  ResidualQuant with 4 least-squares refits (rq_encode_at_ex)
  rotation-only : every loop quantised on its own with the same rotation,
                  grid and least-squares scale (rq_encode with a zero
                  reference), at INT2 and INT4

For each non-final loop it reports the relative reconstruction error
||K_hat - K|| / ||K|| (rq_reconstruct) and the attention-output error of the
fused decode against exact attention over the BF16 loop (torch SDPA in fp32
as the measuring stick), and the stored bits per (token, head, channel)
summed over all loops.  Prints one JSON line per (workload, tensor, scheme).
"""
import argparse
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def bits_per_position(w, scheme, b=None):
    """Stored bits per (token, head, channel) over all L loops."""
    if scheme == "residualquant":
        return 16.0 + sum(16.0 if x == 16 else x + 16.0 / w.group for x in w.bits)
    return w.loops * (b + 16.0 / w.group)


def study(w, emit):
    import torch
    import torch.nn.functional as F
    import kv_cache_residual_rq_b200 as rq
    from kv_cache_residual_rq_b200 import synth
    dev = torch.device("cuda:0")
    q = synth.query(w, 0, 1, dev)
    for kind, name in ((0, "K"), (1, "V")):
        ref = synth.reference(w, 0, kind, dev)
        zero = torch.zeros_like(ref)
        for l in range(1, w.loops):
            x = synth.loop_kv(w, 0, kind, l, ref)
            xf = x.float()
            schemes = [("residualquant", w.bits[l - 1], ref, 0),
                       ("residualquant_ls4", w.bits[l - 1], ref, 4)]
            schemes += [(f"rotation_only_int{b}", b, zero, 0) for b in (2, 4)]
            for scheme, bits, base, it in schemes:
                if bits == 16:
                    continue
                (c,), (s,) = rq.encode([x], base, [bits], w.group, w.seed, refine_iters=it)
                xh = rq.reconstruct(base, c, s, bits, w.group, w.seed)
                rel = (torch.linalg.vector_norm(xh - xf) / torch.linalg.vector_norm(xf)).item()
                emit({"workload": w.name, "tensor": name, "loop": l, "scheme": scheme,
                      "bits": bits, "rel_recon_err": rel,
                      "bits_per_position_all_loops": bits_per_position(
                          w, "residualquant" if scheme.startswith("residualquant") else "rot",
                          bits)})
                del c, s, xh
            del x, xf
            torch.cuda.empty_cache()
    # compressed reference: the final loop itself as rotated INT8 / INT4 codes,
    # the other loops as residuals against its reconstruction
    for kind, name in ((0, "K"), (1, "V")):
        ref = synth.reference(w, 0, kind, dev)
        xs = [synth.loop_kv(w, 0, kind, l, ref) for l in range(1, w.loops)]
        rbits = [b if b != 16 else 2 for b in w.bits]
        for rb in (8, 4):
            (rc, rs), codes, scales = rq.encode_cr(xs, ref, rb, rbits, w.group, w.seed)
            bpp = (rb + 16.0 / w.group) + sum(b + 16.0 / w.group for b in rbits)
            xh = rq.reconstruct_cr(ref.shape, rc, rs, rb, None, None, 16, w.group, w.seed)
            rf = ref.float()
            emit({"workload": w.name, "tensor": name, "loop": w.loops,
                  "scheme": f"compressed_ref_int{rb}", "bits": rb,
                  "rel_recon_err": (torch.linalg.vector_norm(xh - rf) /
                                    torch.linalg.vector_norm(rf)).item(),
                  "bits_per_position_all_loops": bpp})
            for l in range(1, w.loops):
                xf = xs[l - 1].float()
                xh = rq.reconstruct_cr(ref.shape, rc, rs, rb, codes[l - 1], scales[l - 1],
                                       rbits[l - 1], w.group, w.seed)
                emit({"workload": w.name, "tensor": name, "loop": l,
                      "scheme": f"compressed_ref_int{rb}", "bits": rbits[l - 1],
                      "rel_recon_err": (torch.linalg.vector_norm(xh - xf) /
                                        torch.linalg.vector_norm(xf)).item(),
                      "bits_per_position_all_loops": bpp})
            del rc, rs, codes, scales, xh
        del xs
        torch.cuda.empty_cache()
    # attention output: quantise loop 1 (the most sensitive) of both K and V
    refk = synth.reference(w, 0, 0, dev)
    refv = synth.reference(w, 0, 1, dev)
    xk = synth.loop_kv(w, 0, 0, 1, refk)
    xv = synth.loop_kv(w, 0, 1, 1, refv)
    G = w.G
    exact = F.scaled_dot_product_attention(
        q.float().unsqueeze(2), xk.float().repeat_interleave(G, dim=1),
        xv.float().repeat_interleave(G, dim=1)).squeeze(2)
    for scheme, bits, use_ref, it in (("residualquant", w.bits[0], True, 0),
                                      ("residualquant_ls4", w.bits[0], True, 4),
                                      ("rotation_only_int2", 2, False, 0),
                                      ("rotation_only_int4", 4, False, 0)):
        bk = refk if use_ref else torch.zeros_like(refk)
        bv = refv if use_ref else torch.zeros_like(refv)
        (ck,), (sk,) = rq.encode([xk], bk, [bits], w.group, w.seed, refine_iters=it)
        (cv,), (sv,) = rq.encode([xv], bv, [bits], w.group, w.seed, refine_iters=it)
        out = rq.decode_attention(q, bk, bv, ck, cv, sk, sv, bits, w.group, w.seed)
        err = (torch.linalg.vector_norm(out - exact) / torch.linalg.vector_norm(exact)).item()
        emit({"workload": w.name, "tensor": "attention(loop 1)", "scheme": scheme, "bits": bits,
              "rel_output_err": err})
    for rb in (8, 4):
        b1 = w.bits[0] if w.bits[0] != 16 else 2
        (rck, rsk), ck, sk = rq.encode_cr([xk], refk, rb, [b1], w.group, w.seed)
        (rcv, rsv), cv, sv = rq.encode_cr([xv], refv, rb, [b1], w.group, w.seed)
        out = rq.decode_attention_cr(q, (rck, rsk, rcv, rsv, rb), ck[0], cv[0], sk[0], sv[0],
                                     b1, w.group, w.seed, refk.shape[2], kv_heads=w.kv_heads)
        err = (torch.linalg.vector_norm(out - exact) / torch.linalg.vector_norm(exact)).item()
        emit({"workload": w.name, "tensor": "attention(loop 1)",
              "scheme": f"compressed_ref_int{rb}", "bits": b1, "rel_output_err": err})


def main(argv=None):
    from kv_cache_residual_rq_b200 import synth
    ap = argparse.ArgumentParser()
    ap.add_argument("--workloads", default="tiny,ouro1.4b_decode,mixed_precision_32k,deep_loop_gqa")
    args = ap.parse_args(argv)
    for name in args.workloads.split(","):
        w = synth.BY_NAME[name]
        study(w, lambda d: print(json.dumps(d), flush=True))


if __name__ == "__main__":
    main()
