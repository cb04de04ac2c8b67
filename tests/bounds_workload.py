"""Every entry point of the library on small tiny/edge shapes, for the test of
the bounds-checked build (test_gpu_bounds.py).  Run in a subprocess with
RQ_LIBRARY naming the library to load:

    RQ_LIBRARY=<librq.so or librq_bounds.so> python tests/bounds_workload.py <out.pt>

Saves every output and the status words: the encoders' word (read after
every call) and each decode call's workspace word.  Inputs are seeded, so two
runs with different builds of the library can be compared result by result.
"""
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import kv_cache_residual_rq_b200 as rq          # noqa: E402
from kv_cache_residual_rq_b200 import synth     # noqa: E402

PAGE = 64


def main(out_path):
    torch.cuda.set_device(0)
    res, status = {}, {}

    def enc_status(name):
        status["enc " + name] = rq.rq_encode_take_status()

    def ws_status(name, ws):
        status["ws " + name] = rq.rq_workspace_status(ws)

    cases = [  # name, d, group, G, bits, batch, hkv, ctx
        ("tiny", 64, 32, 4, 2, 1, 2, 256),
        ("g1_int2", 128, 32, 1, 2, 2, 3, 200),
        ("g1_int4_ragged", 128, 64, 1, 4, 2, 2, 333),
        ("g2_int2_d64", 64, 64, 2, 2, 2, 2, 130),
        ("g8_int4_ragged", 128, 32, 8, 4, 1, 3, 129),
        ("g4_int2_single", 128, 64, 4, 2, 1, 1, 1),
    ]
    for name, d, group, G, bits, B, H, T in cases:
        w = synth.Workload(name, 3, 1, B, T, H * G, H, d, group, (bits, 16), (0.25, 0.1), 31)
        refk, refv = synth.reference(w, 0, 0), synth.reference(w, 0, 1)
        xk, xv = synth.loop_kv(w, 0, 0, 1, refk), synth.loop_kv(w, 0, 1, 1, refv)
        q = synth.query(w, 0, 1)
        # tensor-copy encoder, with and without refits
        (ck,), (sk,) = rq.encode([xk], refk, [bits], group, w.seed)
        (cv,), (sv,) = rq.encode([xv], refv, [bits], group, w.seed)
        enc_status(name)
        (ckr,), (skr,) = rq.encode([xk], refk, [bits], group, w.seed, refine_iters=2)
        enc_status(name + " refits")
        res[name + " codes"] = (ck.cpu(), sk.cpu(), ckr.cpu(), skr.cpu())
        # streaming encoder: the same rows into a cache of capacity T + 5 at offset 2
        cap = T + 5
        shape_a = rq.make_shape(B, H, T, d, group)
        shape_c = rq.make_shape(B, H, cap, d, group)
        ca, sa = rq.alloc_codes(shape_c, bits), rq.alloc_scales(shape_c, bits)
        ref_out = torch.zeros((B, H, cap, d), dtype=torch.bfloat16, device="cuda")
        rq.rq_encode_at(shape_a, T, 0, cap, 2, [xk], refk, [bits], w.seed, [ca], [sa], ref_out)
        enc_status(name + " append")
        res[name + " append"] = (ca.cpu(), sa.cpu(), ref_out.cpu())
        # reconstruction
        res[name + " recon"] = rq.reconstruct(refk, ck, sk, bits, group, w.seed).cpu()
        res[name + " recon bf16"] = rq.reconstruct(refk, ck, sk, bits, group, w.seed,
                                                   out_bf16=True).cpu()
        enc_status(name + " recon")
        # decode: residual loop with a BF16 tail, the reference loop
        shape = rq.make_shape(B, H, T, d, group, q_heads=H * G)
        ws = rq.alloc_workspace(shape)
        tail_k = synth.reference(w, 0, 0, batch=B, ctx=4)
        tail_v = synth.reference(w, 0, 1, batch=B, ctx=4)
        out = torch.empty((B, H * G, d), dtype=torch.float32, device="cuda")
        rq.rq_decode_attention_tail(shape, q, refk, refv, ck, cv, sk, sv, bits, w.seed, 0.0,
                                    tail_k, tail_v, 3, 4, out, ws)
        ws_status(name + " tail", ws)
        res[name + " decode tail"] = out.cpu()
        out16 = torch.empty_like(out)
        rq.rq_decode_attention(shape, q, refk, refv, None, None, None, None, 16, w.seed, 0.0,
                               out16, ws)
        ws_status(name + " ref", ws)
        res[name + " decode ref"] = out16.cpu()
        # variable lengths (one empty sequence when B > 1)
        lens = torch.tensor([max(0, T - 77 * b) if b else T for b in range(B)], dtype=torch.int32,
                            device="cuda")
        if B > 1:
            lens[1] = 0
        wsv = rq.alloc_workspace(shape, varlen=True)
        outv = torch.empty_like(out)
        rq.rq_decode_attention_varlen(shape, lens, q, refk, refv, ck, cv, sk, sv, bits, w.seed,
                                      0.0, tail_k, tail_v, 2, 4, outv, wsv)
        ws_status(name + " varlen", wsv)
        res[name + " decode varlen"] = outv.cpu()
        # paged: the same cache as a pool of 64-token pages in reversed order
        n_pg = (T + PAGE - 1) // PAGE
        tcap = n_pg * PAGE
        n_pages = B * n_pg
        table = torch.tensor([[n_pages - 1 - (b * n_pg + j) for j in range(n_pg)]
                              for b in range(B)], dtype=torch.int32, device="cuda")

        def pool(x, per_tok):
            flat = x.contiguous().view(torch.uint8)[: B * H * T * per_tok].view(B, H, T, per_tok)
            dense = torch.zeros((B, H, tcap, per_tok), dtype=torch.uint8, device="cuda")
            dense[:, :, :T] = flat
            pg = dense.view(B, H, n_pg, PAGE, per_tok).permute(0, 2, 1, 3, 4).reshape(
                n_pages, H, PAGE, per_tok)
            out_pool = torch.empty_like(pg)
            out_pool[table.view(-1).long()] = pg
            return out_pool

        cb, sbytes = d * bits // 8, 2 * d // group
        pk, pv = pool(refk, 2 * d), pool(refv, 2 * d)
        pck, pcv, psk, psv = pool(ck, cb), pool(cv, cb), pool(sk, sbytes), pool(sv, sbytes)
        shape_p = rq.make_shape(B, H, tcap, d, group, q_heads=H * G)   # ctx = the table's capacity
        wsp = rq.alloc_workspace(shape_p, varlen=True)
        outp = torch.empty_like(out)
        rq.rq_decode_attention_paged(shape_p, lens, table, n_pg, n_pages, q, pk, pv, pck, pcv,
                                     psk, psv, bits, w.seed, 0.0, None, None, 0, 0, outp, wsp)
        ws_status(name + " paged", wsp)
        res[name + " decode paged"] = outp.cpu()
        # paged append-encode of one new token per sequence
        pos = torch.tensor([min(T - 1, 5 * b) for b in range(B)], dtype=torch.int32,
                           device="cuda")
        one = rq.make_shape(B, H, 1, d, group)
        newk = synth.reference(w, 0, 0, batch=B, ctx=1)
        newx = synth.loop_kv(w, 0, 0, 1, newk)
        rq.rq_encode_paged(one, [newx], newk, [bits], w.seed, 0, pos, table, n_pg, n_pages,
                           [pck], [psk], pk)
        enc_status(name + " paged append")
        res[name + " paged append"] = (pck.cpu(), psk.cpu(), pk.cpu())
        # compressed reference, INT8 and INT4
        for rb in (8, 4):
            (rck, rsk), (cck,), (csk,) = rq.encode_cr([xk], refk, rb, [bits], group, w.seed)
            (rcv, rsv), (ccv,), (csv,) = rq.encode_cr([xv], refv, rb, [bits], group, w.seed)
            enc_status(f"{name} cr{rb}")
            outc = torch.empty_like(out)
            rq.rq_decode_attention_cr(shape, None, q, rck, rcv, rsk, rsv, rb, cck, ccv, csk, csv,
                                      bits, w.seed, 0.0, tail_k, tail_v, 2, 4, outc, ws)
            ws_status(f"{name} cr{rb}", ws)
            res[f"{name} cr{rb}"] = (rck.cpu(), rsk.cpu(), cck.cpu(), csk.cpu(), outc.cpu())
            res[f"{name} cr{rb} recon"] = rq.reconstruct_cr(refk.shape, rck, rsk, rb, cck, csk,
                                                            bits, group, w.seed).cpu()
            enc_status(f"{name} cr{rb} recon")
    torch.cuda.synchronize()
    torch.save({"res": res, "status": status, "lib": rq._abi.LIB_PATH}, out_path)
    bad = {k: v for k, v in status.items() if v}
    print(f"{len(status)} status words, non-zero: {bad}", flush=True)


if __name__ == "__main__":
    main(sys.argv[1])
