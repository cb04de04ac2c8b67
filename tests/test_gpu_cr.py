"""Compressed-reference format: encoder, reconstruction and decode attention
against the oracle.

The reference loop is stored as rotated INT4/INT8 codes and the other loops
as residuals against its reconstruction in the rotated domain; every scale's
least-squares sum has a fixed order, so codes AND scales are compared bit for
bit.  Decode outputs are compared with fp64 attention over the oracle's own
reconstruction of its own encode."""
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


def words(buf, rows, d, bits):
    return buf[: rows * d * bits // 8].view(torch.int32).view(rows, d * bits // 32)


def halves(buf, rows, d, group):
    return buf[: rows * (d // group) * 2].view(torch.int16).view(rows, d // group)


def as_u32(t):
    return t.cpu().numpy().view(np.uint32)


def as_u16(t):
    return t.cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("ref_bits", [4, 8])
@pytest.mark.parametrize("d,group", [(128, 32), (128, 64), (64, 32), (64, 64)])
def test_cr_encode_bit_exact(ref_bits, d, group):
    B, H, T = 1, 3, 133                     # 399 rows: several tiles, ragged
    w = synth.Workload("cr", 3, 1, B, T, H, H, d, group, (2, 4), (0.3, 0.1), 101)
    ref = synth.reference(w, 0, 0)
    loops = [synth.loop_kv(w, 0, 0, l, ref) for l in (1, 2)]
    (rc, rs), codes, scales = rq.encode_cr(loops, ref, ref_bits, list(w.bits), group, w.seed)
    torch.cuda.synchronize()
    assert rq.rq_encode_take_status() == 0
    rows = B * H * T
    r_np = u16(ref).reshape(rows, d)
    for l, bits in enumerate(w.bits):
        want_rw, want_rs, want_w, want_s = oracle.encode_rows_cr_f32(
            u16(loops[l]).reshape(rows, d), r_np, ref_bits, bits, group, w.seed)
        if l == 0:
            assert np.array_equal(as_u32(words(rc, rows, d, ref_bits)), want_rw), "ref codes"
            assert np.array_equal(as_u16(halves(rs, rows, d, group)), want_rs), "ref scales"
        assert np.array_equal(as_u32(words(codes[l], rows, d, bits)), want_w), f"codes {bits}"
        assert np.array_equal(as_u16(halves(scales[l], rows, d, group)), want_s), "scales"


def test_cr_encode_into_a_cache_position():
    B, H, d, n, cap, pos = 2, 2, 128, 3, 50, 20
    w = synth.Workload("crpos", 2, 1, B, n, H, H, d, 32, (2,), (0.2,), 102)
    ref = synth.reference(w, 0, 1)
    x = synth.loop_kv(w, 0, 1, 1, ref)
    cshape = rq.make_shape(B, H, cap, d, 32)
    rc, rs = rq.alloc_codes(cshape, 8), rq.alloc_scales(cshape, 8)
    c, s = rq.alloc_codes(cshape, 2), rq.alloc_scales(cshape, 2)
    for buf in (rc, rs, c, s):
        buf.fill_(0x5A)
    rq.rq_encode_cr_at(rq.make_shape(B, H, n, d, 32), cap, pos, [x], ref, 8, [2], w.seed, rc, rs,
                       [c], [s])
    torch.cuda.synchronize()
    want_rw, want_rs, want_w, want_s = oracle.encode_rows_cr_f32(
        u16(x).reshape(-1, d), u16(ref).reshape(-1, d), 8, 2, 32, w.seed)
    got_rw = as_u32(words(rc, B * H * cap, d, 8)).reshape(B * H, cap, -1)
    got_w = as_u32(words(c, B * H * cap, d, 2)).reshape(B * H, cap, -1)
    assert np.array_equal(got_rw[:, pos:pos + n].reshape(-1, got_rw.shape[-1]), want_rw)
    assert np.array_equal(got_w[:, pos:pos + n].reshape(-1, got_w.shape[-1]), want_w)
    mask = np.ones(cap, dtype=bool)
    mask[pos:pos + n] = False
    assert (got_rw[:, mask] == 0x5A5A5A5A).all() and (got_w[:, mask] == 0x5A5A5A5A).all()


@pytest.mark.parametrize("ref_bits,bits", [(8, 2), (4, 4), (8, 16), (4, 16)])
def test_cr_reconstruct_matches_oracle(ref_bits, bits):
    B, H, T, d, g = 1, 2, 100, 128, 32
    w = synth.Workload("crrec", 2, 1, B, T, H, H, d, g, (2,), (0.2,), 103)
    ref = synth.reference(w, 0, 0)
    x = synth.loop_kv(w, 0, 0, 1, ref)
    (rc, rs), codes, scales = rq.encode_cr([x], ref, ref_bits, [bits if bits != 16 else 2], g,
                                           w.seed)
    c0, s0 = (codes[0], scales[0]) if bits != 16 else (None, None)
    got = rq.reconstruct_cr(ref.shape, rc, rs, ref_bits, c0, s0, bits, g, w.seed)
    torch.cuda.synchronize()
    rows = B * H * T
    rw, rsc, ww, ws = oracle.encode_rows_cr_f32(u16(x).reshape(rows, d), u16(ref).reshape(rows, d),
                                                ref_bits, bits if bits != 16 else 2, g, w.seed)
    want = oracle.reconstruct_rows_cr_f64(rw, rsc, ww if bits != 16 else None,
                                          ws if bits != 16 else None, ref_bits,
                                          bits if bits != 16 else 2, g, w.seed, d)
    g32 = got.reshape(rows, d).double().cpu().numpy()
    assert np.abs(g32 - want).max() <= 2e-5 * (1 + np.abs(want).max())


def oracle_cr_head(xk, xv, refk, refv, ref_bits, bits, g, seed, q, b, h, ctx, tail_k, tail_v,
                   n_tail):
    d = refk.shape[-1]
    parts_k, parts_v = [], []
    if ctx > 0:
        for src_x, src_r, parts in ((xk, refk, parts_k), (xv, refv, parts_v)):
            r = u16(src_r[b, h, :ctx])
            xx = u16(src_x[b, h, :ctx])
            rw, rs, ww, ws = oracle.encode_rows_cr_f32(xx, r, ref_bits, bits if bits != 16 else 2,
                                                       g, seed)
            parts.append(oracle.reconstruct_rows_cr_f64(
                rw, rs, ww if bits != 16 else None, ws if bits != 16 else None, ref_bits,
                bits if bits != 16 else 2, g, seed, d))
    if n_tail:
        parts_k.append(oracle.bf16_to_f32(u16(tail_k[b, h, :n_tail])).astype(np.float64))
        parts_v.append(oracle.bf16_to_f32(u16(tail_v[b, h, :n_tail])).astype(np.float64))
    qh = oracle.bf16_to_f32(u16(q[b, h:h + 1])).astype(np.float64)
    return oracle.attention_f64(qh, np.concatenate(parts_k), np.concatenate(parts_v),
                                1.0 / np.sqrt(d))


@pytest.mark.parametrize("ref_bits,bits", [(8, 2), (8, 4), (4, 2), (8, 16), (4, 16)])
@pytest.mark.parametrize("varlen", [False, True])
def test_cr_decode_matches_oracle(ref_bits, bits, varlen):
    lens = [0, 1, 65, 200] if varlen else [150, 150, 150]
    B, Hkv, d, g, cap, n_tail = len(lens), 2, 128, 32, 200, 1
    w = synth.Workload("crdec", 2, 1, B, cap, Hkv, Hkv, d, g, (2,), (0.25,), 104 + ref_bits)
    refk, refv = synth.reference(w, 0, 0), synth.reference(w, 0, 1)
    xk, xv = synth.loop_kv(w, 0, 0, 1, refk), synth.loop_kv(w, 0, 1, 1, refv)
    rb = bits if bits != 16 else 2
    (rck, rsk), ck, sk = rq.encode_cr([xk], refk, ref_bits, [rb], g, w.seed)
    (rcv, rsv), cv, sv = rq.encode_cr([xv], refv, ref_bits, [rb], g, w.seed)
    q = synth.query(w, 0, 1)
    tail_k = synth.reference(w, 0, 0, batch=B, ctx=n_tail + 2)
    tail_v = synth.reference(w, 0, 1, batch=B, ctx=n_tail + 2)
    if varlen:
        # garbage past every length: NaN scales, all-ones codes
        for buf, nb, ratio in ((rsk, 2, None), (rsv, 2, None), (sk[0], 2, None), (sv[0], 2, None)):
            v = buf[: B * Hkv * cap * (d // g) * 2].view(torch.int16).view(B, Hkv, cap, -1)
            for bi, n in enumerate(lens):
                v[bi, :, n:] = F16_NAN
        for buf, bb in ((rck, ref_bits), (rcv, ref_bits), (ck[0], rb), (cv[0], rb)):
            v = buf[: B * Hkv * cap * d * bb // 8].view(torch.int32).view(B, Hkv, cap, -1)
            for bi, n in enumerate(lens):
                v[bi, :, n:] = -1
    ctx_lens = torch.tensor(lens, dtype=torch.int32, device="cuda") if varlen else None
    out = rq.decode_attention_cr(q, (rck, rsk, rcv, rsv, ref_bits),
                                 None if bits == 16 else ck[0], None if bits == 16 else cv[0],
                                 None if bits == 16 else sk[0], None if bits == 16 else sv[0],
                                 bits, g, w.seed, cap, ctx=None if varlen else lens[0],
                                 ctx_lens=ctx_lens, tail_k=tail_k, tail_v=tail_v, n_tail=n_tail)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    worst = 0.0
    for b in range(B):
        for h in range(Hkv):
            want = oracle_cr_head(xk, xv, refk, refv, ref_bits, bits, g, w.seed, q, b, h, lens[b],
                                  tail_k, tail_v, n_tail)
            got = out[b, h:h + 1].double().cpu().numpy()
            worst = max(worst, float(np.abs(got - want).max()))
    assert worst <= OUT_TOL
    print(f"ref INT{ref_bits} bits {bits} varlen {varlen}: max-abs {worst:.2e}")


@pytest.mark.parametrize("ref_bits,bits,d,g", [
    (8, 2, 64, 32), (8, 2, 64, 64), (8, 2, 128, 64), (8, 4, 64, 32), (8, 4, 128, 64),
    (8, 16, 64, 64), (4, 2, 64, 32), (4, 2, 128, 64), (4, 4, 64, 64), (4, 4, 128, 32),
    (4, 16, 64, 32)])
def test_cr_decode_single_query_shapes(ref_bits, bits, d, g):
    """One query row per kv head on the tensor-core kernel at every head size
    and scale group: head_dim 64 uses two of the four 32-dim slices (the
    score MMAs' k positions and B columns of the other two are zero), and
    64-dim groups share one scale between two slices.  Ragged contexts (a
    partial last tile, one token past a tile) and a BF16 tail token."""
    lens = [193, 65]
    B, Hkv, cap, n_tail = len(lens), 2, 200, 1
    w = synth.Workload("crsq", 2, 1, B, cap, Hkv, Hkv, d, g, (2,), (0.25,),
                       300 + ref_bits + bits + d + g)
    refk, refv = synth.reference(w, 0, 0), synth.reference(w, 0, 1)
    xk, xv = synth.loop_kv(w, 0, 0, 1, refk), synth.loop_kv(w, 0, 1, 1, refv)
    rb = bits if bits != 16 else 2
    (rck, rsk), ck, sk = rq.encode_cr([xk], refk, ref_bits, [rb], g, w.seed)
    (rcv, rsv), cv, sv = rq.encode_cr([xv], refv, ref_bits, [rb], g, w.seed)
    q = synth.query(w, 0, 1)
    tail_k = synth.reference(w, 0, 0, batch=B, ctx=n_tail + 2)
    tail_v = synth.reference(w, 0, 1, batch=B, ctx=n_tail + 2)
    ctx_lens = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = rq.decode_attention_cr(q, (rck, rsk, rcv, rsv, ref_bits),
                                 None if bits == 16 else ck[0], None if bits == 16 else cv[0],
                                 None if bits == 16 else sk[0], None if bits == 16 else sv[0],
                                 bits, g, w.seed, cap, ctx_lens=ctx_lens, tail_k=tail_k,
                                 tail_v=tail_v, n_tail=n_tail)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    worst = 0.0
    for b in range(B):
        for h in range(Hkv):
            want = oracle_cr_head(xk, xv, refk, refv, ref_bits, bits, g, w.seed, q, b, h, lens[b],
                                  tail_k, tail_v, n_tail)
            got = out[b, h:h + 1].double().cpu().numpy()
            worst = max(worst, float(np.abs(got - want).max()))
    assert worst <= OUT_TOL
    print(f"single query ref INT{ref_bits} bits {bits} d {d} group {g}: max-abs {worst:.2e}")


@pytest.mark.parametrize("ref_bits,bits,hkv,ctx", [(8, 2, 1, 20000), (4, 2, 8, 3000)])
def test_cr_decode_many_records_per_head(ref_bits, bits, hkv, ctx):
    """Few heads over a long context: one head spread over every CTA of the
    single-query kernel (more records than one merge chunk), or a few dozen
    records per head (above the one-batch merge, within one chunk)."""
    B, d, g = 1, 128, 32
    w = synth.Workload("crlong", 2, 1, B, ctx, hkv, hkv, d, g, (2,), (0.25,), 410 + hkv)
    refk, refv = synth.reference(w, 0, 0), synth.reference(w, 0, 1)
    xk, xv = synth.loop_kv(w, 0, 0, 1, refk), synth.loop_kv(w, 0, 1, 1, refv)
    (rck, rsk), ck, sk = rq.encode_cr([xk], refk, ref_bits, [bits], g, w.seed)
    (rcv, rsv), cv, sv = rq.encode_cr([xv], refv, ref_bits, [bits], g, w.seed)
    q = synth.query(w, 0, 1)
    out = rq.decode_attention_cr(q, (rck, rsk, rcv, rsv, ref_bits), ck[0], cv[0], sk[0], sv[0],
                                 bits, g, w.seed, ctx, kv_heads=hkv)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    worst = 0.0
    for h in range(hkv):
        want = oracle_cr_head(xk, xv, refk, refv, ref_bits, bits, g, w.seed, q, 0, h, ctx,
                              None, None, 0)
        got = out[0, h:h + 1].double().cpu().numpy()
        worst = max(worst, float(np.abs(got - want).max()))
    assert worst <= OUT_TOL
    print(f"ref INT{ref_bits} bits {bits} Hkv {hkv} T {ctx}: max-abs {worst:.2e}")


def oracle_cr_kv(xk, xv, refk, refv, ref_bits, bits, g, seed, b, h, ctx):
    """fp64 K_hat, V_hat of (sequence b, kv head h) from the oracle's own encode."""
    d = refk.shape[-1]
    out = []
    for src_x, src_r in ((xk, refk), (xv, refv)):
        rw, rs, ww, ws = oracle.encode_rows_cr_f32(u16(src_x[b, h, :ctx]), u16(src_r[b, h, :ctx]),
                                                   ref_bits, bits if bits != 16 else 2, g, seed)
        out.append(oracle.reconstruct_rows_cr_f64(
            rw, rs, ww if bits != 16 else None, ws if bits != 16 else None, ref_bits,
            bits if bits != 16 else 2, g, seed, d))
    return out


@pytest.mark.parametrize("ref_bits,G,d,g,bits,varlen", [
    (8, 2, 128, 32, 2, False), (8, 4, 128, 32, 4, True), (8, 8, 128, 64, 2, True),
    (8, 8, 128, 32, 16, False), (8, 4, 64, 32, 2, False), (8, 2, 64, 64, 4, True),
    (8, 8, 64, 32, 2, False), (8, 4, 128, 64, 16, True),
    (4, 4, 128, 32, 2, False), (4, 2, 128, 64, 4, True), (4, 8, 64, 32, 2, True),
    (4, 4, 64, 64, 16, False), (4, 8, 128, 32, 16, True),
    # INT2 residuals with 64-dim groups (ldmatrix code words) at d 64
    (8, 4, 64, 64, 2, True), (4, 2, 64, 64, 2, False)])
def test_cr_decode_grouped_queries(ref_bits, G, d, g, bits, varlen):
    """Grouped queries over an INT8 or INT4 compressed reference (the
    tensor-core kernel): G query rows per kv head, several tiles, ragged and
    empty lengths, one tail token."""
    lens = [0, 1, 130, 200] if varlen else [177, 177]
    B, Hkv, cap, n_tail = len(lens), 2, 200, 1
    w = synth.Workload("crgqa", 2, 1, B, cap, Hkv * G, Hkv, d, g, (2,), (0.25,), 140 + G + d)
    refk, refv = synth.reference(w, 0, 0), synth.reference(w, 0, 1)
    xk, xv = synth.loop_kv(w, 0, 0, 1, refk), synth.loop_kv(w, 0, 1, 1, refv)
    rb = bits if bits != 16 else 2
    (rck, rsk), ck, sk = rq.encode_cr([xk], refk, ref_bits, [rb], g, w.seed)
    (rcv, rsv), cv, sv = rq.encode_cr([xv], refv, ref_bits, [rb], g, w.seed)
    q = synth.query(w, 0, 1)
    tail_k = synth.reference(w, 0, 0, batch=B, ctx=n_tail + 2)
    tail_v = synth.reference(w, 0, 1, batch=B, ctx=n_tail + 2)
    if varlen:
        # garbage past every length: NaN scales, all-ones codes
        for buf in (rsk, rsv, sk[0], sv[0]):
            v = buf[: B * Hkv * cap * (d // g) * 2].view(torch.int16).view(B, Hkv, cap, -1)
            for bi, n in enumerate(lens):
                v[bi, :, n:] = F16_NAN
        for buf, bb in ((rck, ref_bits), (rcv, ref_bits), (ck[0], rb), (cv[0], rb)):
            v = buf[: B * Hkv * cap * d * bb // 8].view(torch.int32).view(B, Hkv, cap, -1)
            for bi, n in enumerate(lens):
                v[bi, :, n:] = -1
    ctx_lens = torch.tensor(lens, dtype=torch.int32, device="cuda") if varlen else None
    out = rq.decode_attention_cr(q, (rck, rsk, rcv, rsv, ref_bits),
                                 None if bits == 16 else ck[0], None if bits == 16 else cv[0],
                                 None if bits == 16 else sk[0], None if bits == 16 else sv[0],
                                 bits, g, w.seed, cap, ctx=None if varlen else lens[0],
                                 ctx_lens=ctx_lens, tail_k=tail_k, tail_v=tail_v, n_tail=n_tail,
                                 kv_heads=Hkv)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    worst = 0.0
    for b in range(B):
        for h in range(Hkv):
            parts_k, parts_v = [], []
            if lens[b] > 0:
                kh, vh = oracle_cr_kv(xk, xv, refk, refv, ref_bits, bits, g, w.seed, b, h, lens[b])
                parts_k.append(kh)
                parts_v.append(vh)
            parts_k.append(oracle.bf16_to_f32(u16(tail_k[b, h, :n_tail])).astype(np.float64))
            parts_v.append(oracle.bf16_to_f32(u16(tail_v[b, h, :n_tail])).astype(np.float64))
            qh = oracle.bf16_to_f32(u16(q[b, h * G:(h + 1) * G])).astype(np.float64)
            want = oracle.attention_f64(qh, np.concatenate(parts_k), np.concatenate(parts_v),
                                        1.0 / np.sqrt(d))
            got = out[b, h * G:(h + 1) * G].double().cpu().numpy()
            worst = max(worst, float(np.abs(got - want).max()))
    assert worst <= OUT_TOL
    print(f"ref INT{ref_bits} G {G} d {d} group {g} bits {bits} varlen {varlen}: "
          f"max-abs {worst:.2e}")



def test_cr_grouped_peaky_scores_long_context():
    """Scores spread wide over many tiles: the lazy softmax lets weights grow
    to 2^8 before the running max moves, which the INT8 reference's f16 value
    weights must absorb without overflow."""
    G, d, g, bits, B, Hkv, T = 4, 128, 32, 2, 2, 2, 1500
    w = synth.Workload("crpeak", 2, 1, B, T, Hkv * G, Hkv, d, g, (bits,), (0.25,), 177)
    refk, refv = synth.reference(w, 0, 0), synth.reference(w, 0, 1)
    xk, xv = synth.loop_kv(w, 0, 0, 1, refk), synth.loop_kv(w, 0, 1, 1, refv)
    (rck, rsk), ck, sk = rq.encode_cr([xk], refk, 8, [bits], g, w.seed)
    (rcv, rsv), cv, sv = rq.encode_cr([xv], refv, 8, [bits], g, w.seed)
    q = (synth.query(w, 0, 1).float() * 8.0).to(torch.bfloat16)
    shape = rq.make_shape(B, Hkv, T, d, g, q_heads=Hkv * G)
    ws = rq.alloc_workspace(shape, q.device)
    out = rq.decode_attention_cr(q, (rck, rsk, rcv, rsv, 8), ck[0], cv[0], sk[0], sv[0], bits, g,
                                 w.seed, T, workspace=ws, kv_heads=Hkv)
    torch.cuda.synchronize()
    assert rq.rq_workspace_status(ws) == 0
    assert torch.isfinite(out).all()
    worst = 0.0
    for b in range(B):
        for h in range(Hkv):
            kh, vh = oracle_cr_kv(xk, xv, refk, refv, 8, bits, g, w.seed, b, h, T)
            qh = oracle.bf16_to_f32(u16(q[b, h * G:(h + 1) * G])).astype(np.float64)
            want = oracle.attention_f64(qh, kh, vh, 1.0 / np.sqrt(d))
            worst = max(worst, float(np.abs(out[b, h * G:(h + 1) * G].double().cpu().numpy()
                                            - want).max()))
    assert worst <= OUT_TOL
    print(f"peaky G {G}: max-abs {worst:.2e}")


@pytest.mark.parametrize("name", ["ouro1.4b_decode", "deep_loop_gqa"])
def test_cr_decode_full_size_sampled(name):
    """The compressed-reference call at full size, in the shape the bench's
    workloads block times (INT8 reference + the first INT2 loop of one layer:
    the single-query kernel on the Ouro-shaped call, the grouped-query kernel
    with shared value accumulators on the deep-loop call), checked on sampled
    heads against fp64 attention over the oracle's own encode."""
    w = synth.BY_NAME[name]
    G, d, g = w.G, w.head_dim, w.group
    refk, refv = synth.reference(w, 0, 0), synth.reference(w, 0, 1)
    xk, xv = synth.loop_kv(w, 0, 0, 1, refk), synth.loop_kv(w, 0, 1, 1, refv)
    (rck, rsk), ck, sk = rq.encode_cr([xk], refk, 8, [2], g, w.seed)
    (rcv, rsv), cv, sv = rq.encode_cr([xv], refv, 8, [2], g, w.seed)
    q = synth.query(w, 0, 1)
    shape = rq.make_shape(w.batch, w.kv_heads, w.ctx, d, g, w.q_heads)
    ws = rq.alloc_workspace(shape, q.device)
    out = rq.decode_attention_cr(q, (rck, rsk, rcv, rsv, 8), ck[0], cv[0], sk[0], sv[0], 2, g,
                                 w.seed, w.ctx, workspace=ws, kv_heads=w.kv_heads)
    torch.cuda.synchronize()
    assert rq.rq_workspace_status(ws) == 0
    rng = np.random.default_rng(5)
    heads = {(0, 0), (w.batch - 1, w.kv_heads - 1)}
    heads |= {(int(rng.integers(w.batch)), int(rng.integers(w.kv_heads))) for _ in range(2)}
    worst = 0.0
    for b, h in sorted(heads):
        kh, vh = oracle_cr_kv(xk, xv, refk, refv, 8, 2, g, w.seed, b, h, w.ctx)
        qh = oracle.bf16_to_f32(u16(q[b, h * G:(h + 1) * G])).astype(np.float64)
        want = oracle.attention_f64(qh, kh, vh, 1.0 / np.sqrt(d))
        got = out[b, h * G:(h + 1) * G].double().cpu().numpy()
        worst = max(worst, float(np.abs(got - want).max()))
    assert worst <= OUT_TOL
    print(f"{name} compressed reference INT8 + INT2: {len(heads)} heads, max-abs {worst:.2e}")


def test_cr_single_query_large_value_scales():
    """One query row per kv head: the value weights p s 2^Ev are f16 after a
    lazily updated warp-wide power of two, so reference value scales at the
    fp16 maximum decode without overflow (status 0) and match the oracle's
    attention over the same scales.  A NaN scale of a cached token makes the
    weights non-finite, which raises workspace status bit 64."""
    d, g, B, H, T = 128, 32, 2, 2, 2000
    w = synth.Workload("crbig", 2, 1, B, T, H, H, d, g, (2,), (0.25,), 178)
    refk, refv = synth.reference(w, 0, 0), synth.reference(w, 0, 1)
    xk, xv = synth.loop_kv(w, 0, 0, 1, refk), synth.loop_kv(w, 0, 1, 1, refv)
    (rck, rsk), ck, sk = rq.encode_cr([xk], refk, 8, [2], g, w.seed)
    (rcv, rsv), cv, sv = rq.encode_cr([xv], refv, 8, [2], g, w.seed)
    big = 0x7BFF                                                 # fp16 65504
    rsv.view(torch.int16)[: B * H * T * (d // g)] = big
    q = (synth.query(w, 0, 1).float() * 4.0).to(torch.bfloat16)
    shape = rq.make_shape(B, H, T, d, g)
    ws = rq.alloc_workspace(shape, q.device)
    out = rq.decode_attention_cr(q, (rck, rsk, rcv, rsv, 8), ck[0], cv[0], sk[0], sv[0], 2, g,
                                 w.seed, T, workspace=ws)
    torch.cuda.synchronize()
    assert rq.rq_workspace_status(ws) == 0
    assert torch.isfinite(out).all()
    worst, top = 0.0, 0.0
    for b in range(B):
        for h in range(H):
            parts = []
            for src_x, src_r, v in ((xk, refk, False), (xv, refv, True)):
                rw, rs, ww, wsc = oracle.encode_rows_cr_f32(u16(src_x[b, h, :T]),
                                                            u16(src_r[b, h, :T]), 8, 2, g, w.seed)
                if v:
                    rs = np.full_like(rs, big)
                parts.append(oracle.reconstruct_rows_cr_f64(rw, rs, ww, wsc, 8, 2, g, w.seed, d))
            qh = oracle.bf16_to_f32(u16(q[b, h:h + 1])).astype(np.float64)
            want = oracle.attention_f64(qh, parts[0], parts[1], 1.0 / np.sqrt(d))
            worst = max(worst, float(np.abs(out[b, h:h + 1].double().cpu().numpy() - want).max()))
            top = max(top, float(np.abs(want).max()))
    print(f"value scales 65504: max-abs {worst:.3e} of max |out| {top:.3e}")
    assert worst <= 1e-4 * top
    rsv.view(torch.int16)[5 * (d // g) + 1] = F16_NAN           # token 5 of head (0, 0)
    rq.decode_attention_cr(q, (rck, rsk, rcv, rsv, 8), ck[0], cv[0], sk[0], sv[0], 2, g, w.seed,
                           T, workspace=ws)
    torch.cuda.synchronize()
    assert rq.rq_workspace_status(ws) & 64
