"""Decode-loop pieces: append-encode into a cache position, decode over a
cache with spare capacity, and decode with BF16 tail tokens.

A token's non-final loops can be encoded only once its final loop exists, so
a decode loop keeps recent tokens in BF16 (a window), attends over the
encoded cache plus that tail, and retires tokens into the cache.  The oracle
side is the oracle's own encode of the same bf16 rows, its fp64
reconstruction, and its fp64 attention over the concatenated key/value rows.
"""
import numpy as np
import pytest
import torch

import oracle
import kv_cache_residual_rq_b200 as rq
from kv_cache_residual_rq_b200 import synth

pytestmark = pytest.mark.gpu

OUT_TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_residual_rq_b200 import build
    build.build()
    rq.lib()


def u16(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def words_of(buf, heads, pitch, wpr):
    return buf[: heads * pitch * wpr * 4].view(torch.int32).view(heads, pitch, wpr)


def scales_of(buf, heads, pitch, ng):
    return buf[: heads * pitch * ng * 2].view(torch.int16).view(heads, pitch, ng)


def test_encode_at_writes_only_its_positions():
    w = synth.Workload("app", 4, 1, 2, 40, 4, 4, 128, 32, (2, 4, 16), (0.2, 0.1, 0.05), 31)
    B, H, d, W, cap = 2, 4, 128, 8, 100
    win_ref = synth.reference(w, 0, 0, batch=B, ctx=W)
    win_loops = [synth.loop_kv(w, 0, 0, l, win_ref) for l in range(1, 4)]
    shape_cache = rq.make_shape(B, H, cap, d, 32)
    codes = [rq.alloc_codes(shape_cache, b) for b in w.bits]
    scales = [rq.alloc_scales(shape_cache, b) for b in w.bits]
    for buf in codes[:2] + scales[:2]:
        buf.fill_(0x5A)
    ref_cache = torch.full((B, H, cap, d), 7.0, dtype=torch.bfloat16, device="cuda")
    n, src_off, pos = 3, 2, 57
    shape = rq.make_shape(B, H, n, d, 32)
    rq.rq_encode_at(shape, W, src_off, cap, pos, win_loops, win_ref, list(w.bits), w.seed,
                    codes, scales, ref_out=ref_cache)
    torch.cuda.synchronize()
    for l, bits in enumerate(w.bits):
        if bits == 16:
            continue
        wpr, ng = d * bits // 32, d // 32
        got_w = words_of(codes[l], B * H, cap, wpr).cpu().numpy().view(np.uint32)
        got_s = scales_of(scales[l], B * H, cap, ng).cpu().numpy().view(np.uint16)
        x = u16(win_loops[l]).reshape(B * H, W, d)[:, src_off:src_off + n]
        r = u16(win_ref).reshape(B * H, W, d)[:, src_off:src_off + n]
        want_w, want_s, _ = oracle.encode_rows_f32(x, r, bits, 32, w.seed)
        assert np.array_equal(got_w[:, pos:pos + n], want_w)
        s_got = np.vectorize(oracle.f16_to_f64)(got_s[:, pos:pos + n])
        s_want = np.vectorize(oracle.f16_to_f64)(want_s)
        assert np.all(np.abs(s_got - s_want) <= np.maximum(1e-3 * np.abs(s_want), 2.0 ** -24))
        # everything else untouched
        mask = np.ones(cap, dtype=bool)
        mask[pos:pos + n] = False
        assert (got_w[:, mask] == 0x5A5A5A5A).all()
        assert (got_s[:, mask] == 0x5A5A).all()
    rc = ref_cache.view(B * H, cap, d)
    assert torch.equal(rc[:, pos:pos + n], win_ref.view(B * H, W, d)[:, src_off:src_off + n])
    assert (rc[:, :pos] == 7.0).all() and (rc[:, pos + n:] == 7.0).all()


def oracle_loop_attention(w, q, refk, refv, xk, xv, bits, b, h, ctx, tail_k=None, tail_v=None,
                          n_tail=0):
    """fp64 attention of head (b, h) over the first ctx cached tokens (the
    oracle encodes and reconstructs them) plus n_tail BF16 tail tokens."""
    G, d = w.G, w.head_dim
    rk, rv = u16(refk[b, h, :ctx]), u16(refv[b, h, :ctx])
    if bits == 16:
        K = oracle.bf16_to_f32(rk).astype(np.float64)
        V = oracle.bf16_to_f32(rv).astype(np.float64)
    else:
        ck, sk, _ = oracle.encode_rows_f32(u16(xk[b, h, :ctx]), rk, bits, w.group, w.seed)
        cv, sv, _ = oracle.encode_rows_f32(u16(xv[b, h, :ctx]), rv, bits, w.group, w.seed)
        K = oracle.reconstruct_rows_f64(rk, ck, sk, bits, w.group, w.seed)
        V = oracle.reconstruct_rows_f64(rv, cv, sv, bits, w.group, w.seed)
    if n_tail:
        K = np.concatenate([K, oracle.bf16_to_f32(u16(tail_k[b, h, :n_tail])).astype(np.float64)])
        V = np.concatenate([V, oracle.bf16_to_f32(u16(tail_v[b, h, :n_tail])).astype(np.float64)])
    qh = oracle.bf16_to_f32(u16(q[b, h * G:(h + 1) * G])).astype(np.float64)
    return oracle.attention_f64(qh, K, V, 1.0 / np.sqrt(d))


@pytest.mark.parametrize("G,bits,ctx,cap,n_tail", [
    (1, 2, 700, 1000, 0), (1, 2, 700, 1000, 1), (1, 16, 300, 301, 5), (1, 4, 129, 256, 256),
    (4, 2, 700, 1000, 3), (4, 16, 64, 65, 1), (2, 4, 333, 400, 17)])
def test_decode_with_capacity_and_tail(G, bits, ctx, cap, n_tail):
    B, Hkv, d = 2, 2, 128
    group = 64 if G == 4 else 32
    bl = (bits, 16) if bits != 16 else (2, 16)
    w = synth.Workload("tail", 3, 1, B, cap, Hkv * G, Hkv, d, group, bl, (0.25, 0.1), 41)
    refk = synth.reference(w, 0, 0)
    refv = synth.reference(w, 0, 1)
    q = synth.query(w, 0, 1)
    xk = xv = None
    ck = cv = sk = sv = None
    if bits != 16:
        xk = synth.loop_kv(w, 0, 0, 1, refk)
        xv = synth.loop_kv(w, 0, 1, 1, refv)
        (ck,), (sk,) = rq.encode([xk], refk, [bits], group, w.seed)
        (cv,), (sv,) = rq.encode([xv], refv, [bits], group, w.seed)
    tw = max(n_tail, 1) + 3
    tail_k = synth.reference(w, 0, 0, batch=B, ctx=tw) if n_tail else None
    tail_v = synth.reference(w, 0, 1, batch=B, ctx=tw) if n_tail else None
    out = rq.decode_attention(q, refk, refv, ck, cv, sk, sv, bits, group, w.seed, ctx=ctx,
                              tail_k=tail_k, tail_v=tail_v, n_tail=n_tail)
    torch.cuda.synchronize()
    worst = 0.0
    for b in range(B):
        for h in range(Hkv):
            want = oracle_loop_attention(w, q, refk, refv, xk, xv, bits, b, h, ctx, tail_k, tail_v,
                                         n_tail)
            got = out[b, h * G:(h + 1) * G].double().cpu().numpy()
            worst = max(worst, float(np.abs(got - want).max()))
    assert worst <= OUT_TOL
    print(f"G{G} b{bits} ctx {ctx}/{cap} tail {n_tail}: max-abs {worst:.2e}")


def test_three_step_decode_loop_retires_tokens_into_the_cache():
    # cache of capacity T0 + 3; each step attends over the cache plus the new
    # token's BF16 K/V (tail of 1), then encodes that token into the cache
    B, Hkv, G, d, T0, steps = 1, 2, 4, 128, 200, 3
    w = synth.Workload("loop", 3, 1, B, T0 + steps, Hkv * G, Hkv, d, 64, (2, 16), (0.2, 0.1), 53)
    full_refk = synth.reference(w, 0, 0)          # final loop of all tokens
    full_refv = synth.reference(w, 0, 1)
    full_xk = synth.loop_kv(w, 0, 0, 1, full_refk)  # loop 1 of all tokens
    full_xv = synth.loop_kv(w, 0, 1, 1, full_refv)
    cap = T0 + steps
    shape_cap = rq.make_shape(B, Hkv, cap, d, 64)
    ck, cv = rq.alloc_codes(shape_cap, 2), rq.alloc_codes(shape_cap, 2)
    sk, sv = rq.alloc_scales(shape_cap, 2), rq.alloc_scales(shape_cap, 2)
    refk = torch.zeros_like(full_refk)
    refv = torch.zeros_like(full_refv)
    pre = rq.make_shape(B, Hkv, T0, d, 64)
    rq.rq_encode_at(pre, cap, 0, cap, 0, [full_xk], full_refk, [2], w.seed, [ck], [sk], refk)
    rq.rq_encode_at(pre, cap, 0, cap, 0, [full_xv], full_refv, [2], w.seed, [cv], [sv], refv)
    for s in range(steps):
        t = T0 + s
        q = synth.query(w, 0, 1, step=s)
        tail_k = full_xk[:, :, t:t + 1].contiguous()     # loop-1 K/V of the new token
        tail_v = full_xv[:, :, t:t + 1].contiguous()
        out = rq.decode_attention(q, refk, refv, ck, cv, sk, sv, 2, 64, w.seed, ctx=t,
                                  tail_k=tail_k, tail_v=tail_v, n_tail=1)
        torch.cuda.synchronize()
        for h in range(Hkv):
            want = oracle_loop_attention(w, q, full_refk, full_refv, full_xk, full_xv, 2, 0, h, t,
                                         tail_k, tail_v, 1)
            got = out[0, h * G:(h + 1) * G].double().cpu().numpy()
            assert np.abs(got - want).max() <= OUT_TOL
        # the token's final loop now exists: retire it into the cache
        one = rq.make_shape(B, Hkv, 1, d, 64)
        rq.rq_encode_at(one, cap, t, cap, t, [full_xk], full_refk, [2], w.seed, [ck], [sk], refk)
        rq.rq_encode_at(one, cap, t, cap, t, [full_xv], full_refv, [2], w.seed, [cv], [sv], refv)
    torch.cuda.synchronize()
    assert torch.equal(refk, full_refk) and torch.equal(refv, full_refv)
