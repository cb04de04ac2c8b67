"""Variable-length decode (rq_decode_attention_varlen) against the oracle.

Every sequence of the batch attends over its own number of cached tokens
(read from a device array) plus the BF16 tail.  Everything in the cache past
a sequence's length -- reference K/V, codes, scales -- is overwritten with
NaN or garbage first, so a kernel that read beyond a length would return NaN
or a wrong result.  The oracle encodes and reconstructs each sequence's
first len_b tokens itself and attends in fp64."""
import numpy as np
import pytest
import torch

import oracle
import kv_cache_residual_rq_b200 as rq
from kv_cache_residual_rq_b200 import synth

pytestmark = pytest.mark.gpu

OUT_TOL = 1e-2
BF16_NAN = 0x7FC0
F16_NAN = 0x7E00


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_residual_rq_b200 import build
    build.build()
    rq.lib()


def u16(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def oracle_head(w, q, refk, refv, xk, xv, bits, b, h, ctx, tail_k, tail_v, n_tail):
    G, d = w.G, w.head_dim
    parts_k, parts_v = [], []
    if ctx > 0:
        rk, rv = u16(refk[b, h, :ctx]), u16(refv[b, h, :ctx])
        if bits == 16:
            parts_k.append(oracle.bf16_to_f32(rk).astype(np.float64))
            parts_v.append(oracle.bf16_to_f32(rv).astype(np.float64))
        else:
            ck, sk, _ = oracle.encode_rows_f32(u16(xk[b, h, :ctx]), rk, bits, w.group, w.seed)
            cv, sv, _ = oracle.encode_rows_f32(u16(xv[b, h, :ctx]), rv, bits, w.group, w.seed)
            parts_k.append(oracle.reconstruct_rows_f64(rk, ck, sk, bits, w.group, w.seed))
            parts_v.append(oracle.reconstruct_rows_f64(rv, cv, sv, bits, w.group, w.seed))
    if n_tail:
        parts_k.append(oracle.bf16_to_f32(u16(tail_k[b, h, :n_tail])).astype(np.float64))
        parts_v.append(oracle.bf16_to_f32(u16(tail_v[b, h, :n_tail])).astype(np.float64))
    K, V = np.concatenate(parts_k), np.concatenate(parts_v)
    qh = oracle.bf16_to_f32(u16(q[b, h * G:(h + 1) * G])).astype(np.float64)
    return oracle.attention_f64(qh, K, V, 1.0 / np.sqrt(d))


def build_case(G, bits, lens, cap, n_tail, seed):
    B, Hkv, d = len(lens), 2, 128
    group = 64 if G == 4 else 32
    bl = (bits, 16) if bits != 16 else (2, 16)
    w = synth.Workload("varlen", 3, 1, B, cap, Hkv * G, Hkv, d, group, bl, (0.25, 0.1), seed)
    refk, refv = synth.reference(w, 0, 0), synth.reference(w, 0, 1)
    xk = xv = ck = cv = sk = sv = None
    if bits != 16:
        xk, xv = synth.loop_kv(w, 0, 0, 1, refk), synth.loop_kv(w, 0, 1, 1, refv)
        (ck,), (sk,) = rq.encode([xk], refk, [bits], group, w.seed)
        (cv,), (sv,) = rq.encode([xv], refv, [bits], group, w.seed)
    q = synth.query(w, 0, 1)
    tail_k = tail_v = None
    if n_tail:
        tail_k = synth.reference(w, 0, 0, batch=B, ctx=n_tail + 2)
        tail_v = synth.reference(w, 0, 1, batch=B, ctx=n_tail + 2)
    return w, refk, refv, xk, xv, ck, cv, sk, sv, q, tail_k, tail_v


@pytest.mark.parametrize("G,bits", [(1, 2), (1, 16), (1, 4), (4, 2), (4, 16), (2, 4)])
def test_varlen_matches_oracle_and_never_reads_past_a_length(G, bits):
    lens = [0, 1, 63, 130, 200]
    cap, n_tail = 200, 1
    w, refk, refv, xk, xv, ck, cv, sk, sv, q, tail_k, tail_v = build_case(G, bits, lens, cap,
                                                                          n_tail, 91 + G + bits)
    B, Hkv, d = len(lens), w.kv_heads, w.head_dim
    # the oracle reads the clean tensors; the device ones get poisoned
    refk_h, refv_h = refk.clone(), refv.clone()
    rk16, rv16 = refk.view(torch.int16), refv.view(torch.int16)
    for b, n in enumerate(lens):
        rk16[b, :, n:] = BF16_NAN
        rv16[b, :, n:] = BF16_NAN
    if bits != 16:
        for sc in (sk, sv):
            v = sc[: B * Hkv * cap * (d // w.group) * 2].view(torch.int16).view(B, Hkv, cap, -1)
            for b, n in enumerate(lens):
                v[b, :, n:] = F16_NAN
        for cc in (ck, cv):
            v = cc[: B * Hkv * cap * d * bits // 8].view(torch.int32).view(B, Hkv, cap, -1)
            for b, n in enumerate(lens):
                v[b, :, n:] = -1
    shape = rq.make_shape(B, Hkv, cap, d, w.group, q_heads=Hkv * G)
    ws = rq.alloc_workspace(shape, varlen=True)
    lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = torch.empty((B, Hkv * G, d), dtype=torch.float32, device="cuda")
    rq.rq_decode_attention_varlen(shape, lens_d, q, refk, refv, ck, cv, sk, sv, bits, w.seed,
                                  0.0, tail_k, tail_v, n_tail, tail_k.shape[2], out, ws)
    torch.cuda.synchronize()
    assert rq.rq_workspace_status(ws) == 0
    assert torch.isfinite(out).all()
    worst = 0.0
    for b in range(B):
        for h in range(Hkv):
            want = oracle_head(w, q, refk_h, refv_h, xk, xv, bits, b, h, lens[b], tail_k, tail_v,
                               n_tail)
            got = out[b, h * G:(h + 1) * G].double().cpu().numpy()
            worst = max(worst, float(np.abs(got - want).max()))
    assert worst <= OUT_TOL
    print(f"G{G} b{bits}: max-abs {worst:.2e}")


@pytest.mark.parametrize("G,bits", [(1, 2), (4, 2), (4, 16)])
def test_equal_lengths_equal_the_uniform_call(G, bits):
    lens = [150] * 3
    w, refk, refv, xk, xv, ck, cv, sk, sv, q, tail_k, tail_v = build_case(G, bits, lens, 150, 1,
                                                                          17)
    B, Hkv, d = 3, w.kv_heads, w.head_dim
    shape = rq.make_shape(B, Hkv, 150, d, w.group, q_heads=Hkv * G)
    out_u = torch.empty((B, Hkv * G, d), dtype=torch.float32, device="cuda")
    out_v = torch.empty_like(out_u)
    rq.rq_decode_attention_tail(shape, q, refk, refv, ck, cv, sk, sv, bits, w.seed, 0.0, tail_k,
                                tail_v, 1, tail_k.shape[2], out_u, rq.alloc_workspace(shape))
    lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
    rq.rq_decode_attention_varlen(shape, lens_d, q, refk, refv, ck, cv, sk, sv, bits, w.seed, 0.0,
                                  tail_k, tail_v, 1, tail_k.shape[2], out_v,
                                  rq.alloc_workspace(shape, varlen=True))
    torch.cuda.synchronize()
    assert torch.equal(out_u, out_v)


def test_lengths_past_the_capacity_are_clamped_and_flagged():
    lens = [10, 500]                       # capacity 64
    w, refk, refv, xk, xv, ck, cv, sk, sv, q, tail_k, tail_v = build_case(1, 2, lens, 64, 0, 23)
    shape = rq.make_shape(2, w.kv_heads, 64, w.head_dim, w.group, q_heads=w.kv_heads)
    ws = rq.alloc_workspace(shape, varlen=True)
    out = torch.empty((2, w.kv_heads, w.head_dim), dtype=torch.float32, device="cuda")
    lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
    rq.rq_decode_attention_varlen(shape, lens_d, q, refk, refv, ck, cv, sk, sv, 2, w.seed, 0.0,
                                  None, None, 0, 0, out, ws)
    torch.cuda.synchronize()
    assert rq.rq_workspace_status(ws) & 16
    for h in range(w.kv_heads):
        want = oracle_head(w, q, refk, refv, xk, xv, 2, 1, h, 64, None, None, 0)
        assert np.abs(out[1, h:h + 1].double().cpu().numpy() - want).max() <= OUT_TOL


@pytest.mark.parametrize("G", [1, 4])
def test_uniform_call_ignores_nan_in_spare_capacity(G):
    # a uniform call over ctx tokens of a larger cache: the spare capacity may
    # hold anything (here NaN) and must not reach the output
    ctx, cap = 100, 160
    w, refk, refv, xk, xv, ck, cv, sk, sv, q, tail_k, tail_v = build_case(G, 2, [ctx] * 2, cap, 0,
                                                                          29)
    refk_h, refv_h = refk.clone(), refv.clone()
    refk.view(torch.int16)[:, :, ctx:] = BF16_NAN
    refv.view(torch.int16)[:, :, ctx:] = BF16_NAN
    out = rq.decode_attention(q, refk, refv, ck, cv, sk, sv, 2, w.group, w.seed, ctx=ctx)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    for b in range(2):
        for h in range(w.kv_heads):
            want = oracle_head(w, q, refk_h, refv_h, xk, xv, 2, b, h, ctx, None, None, 0)
            got = out[b, h * G:(h + 1) * G].double().cpu().numpy()
            assert np.abs(got - want).max() <= OUT_TOL


@pytest.mark.parametrize("G", [1, 4])
def test_one_captured_graph_serves_changing_lengths(G):
    # capture a variable-length call once; new lengths written on the device
    # between replays change the work each replay does
    cap, bits = 200, 2
    w, refk, refv, xk, xv, ck, cv, sk, sv, q, tail_k, tail_v = build_case(G, bits, [cap] * 3, cap,
                                                                          1, 61 + G)
    B, Hkv, d = 3, w.kv_heads, w.head_dim
    shape = rq.make_shape(B, Hkv, cap, d, w.group, q_heads=Hkv * G)
    ws = rq.alloc_workspace(shape, varlen=True)
    lens_d = torch.tensor([cap] * B, dtype=torch.int32, device="cuda")
    out = torch.empty((B, Hkv * G, d), dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    call = lambda: rq.rq_decode_attention_varlen(shape, lens_d, q, refk, refv, ck, cv, sk, sv,
                                                 bits, w.seed, 0.0, tail_k, tail_v, 1,
                                                 tail_k.shape[2], out, ws,
                                                 stream=torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call()                                       # warm-up outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        call()
    torch.cuda.synchronize()
    for lens in ([5, 200, 64], [130, 1, 0], [200, 200, 200]):
        lens_d.copy_(torch.tensor(lens, dtype=torch.int32))
        g.replay()
        torch.cuda.synchronize()
        got = out.clone()
        want = torch.empty_like(out)
        rq.rq_decode_attention_varlen(shape, lens_d, q, refk, refv, ck, cv, sk, sv, bits, w.seed,
                                      0.0, tail_k, tail_v, 1, tail_k.shape[2], want,
                                      rq.alloc_workspace(shape, varlen=True))
        torch.cuda.synchronize()
        assert torch.equal(got, want), lens
    assert rq.rq_workspace_status(ws) == 0
