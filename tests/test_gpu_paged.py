"""Paged caches: pools of 64-token pages addressed through a page table.

Pools are assembled from a dense cache by a random page permutation; pages
no sequence uses, and table entries past each sequence's length, hold NaN
or out-of-range ids, so any read they were not meant to get would show.  The
paged call must equal the dense variable-length call bit for bit (same work
split, same data) and the oracle within 1e-2."""
import numpy as np
import pytest
import torch

import oracle
import kv_cache_residual_rq_b200 as rq
from kv_cache_residual_rq_b200 import synth

pytestmark = pytest.mark.gpu

OUT_TOL = 1e-2
BF16_NAN = 0x7FC0
PAGE = 64


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_residual_rq_b200 import build
    build.build()
    rq.lib()


def u16(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def to_pool(dense, table, lens, n_pages, fill):
    """dense [B, H, cap, ...] -> pool [n_pages, H, 64, ...] per the table."""
    B, H = dense.shape[:2]
    pool = torch.empty((n_pages, H, PAGE) + tuple(dense.shape[3:]), dtype=dense.dtype,
                       device=dense.device)
    pool.view(torch.int16 if dense.element_size() == 2 else torch.int32).fill_(fill)
    for b in range(B):
        for j in range((lens[b] + PAGE - 1) // PAGE):
            pool[table[b][j]] = dense[b, :, j * PAGE:(j + 1) * PAGE]
    return pool


def build_paged_case(G, bits, lens, max_pages, n_pages, seed):
    B, Hkv, d = len(lens), 2, 128
    group = 64 if G == 4 else 32
    cap = max_pages * PAGE
    bl = (bits, 16) if bits != 16 else (2, 16)
    w = synth.Workload("paged", 3, 1, B, cap, Hkv * G, Hkv, d, group, bl, (0.25, 0.1), seed)
    refk, refv = synth.reference(w, 0, 0), synth.reference(w, 0, 1)
    xk = xv = ck = cv = sk = sv = None
    if bits != 16:
        xk, xv = synth.loop_kv(w, 0, 0, 1, refk), synth.loop_kv(w, 0, 1, 1, refv)
        (ck,), (sk,) = rq.encode([xk], refk, [bits], group, w.seed)
        (cv,), (sv,) = rq.encode([xv], refv, [bits], group, w.seed)
    rng = np.random.default_rng(seed)
    perm = rng.permutation(n_pages)
    table = np.full((B, max_pages), -7, dtype=np.int32)   # past-length entries: invalid ids
    k = 0
    for b in range(B):
        for j in range((lens[b] + PAGE - 1) // PAGE):
            table[b, j] = perm[k]
            k += 1
    return w, refk, refv, xk, xv, ck, cv, sk, sv, table, group


@pytest.mark.parametrize("G,bits", [(1, 2), (1, 16), (4, 2), (4, 16), (2, 4)])
def test_paged_equals_dense_varlen_and_oracle(G, bits):
    lens, max_pages, n_pages = [0, 70, 200, 129], 4, 13
    w, refk, refv, xk, xv, ck, cv, sk, sv, table, group = build_paged_case(G, bits, lens,
                                                                           max_pages, n_pages,
                                                                           70 + G + bits)
    B, Hkv, d = len(lens), w.kv_heads, w.head_dim
    cap = max_pages * PAGE
    q = synth.query(w, 0, 1)
    tail_k = synth.reference(w, 0, 0, batch=B, ctx=3)
    tail_v = synth.reference(w, 0, 1, batch=B, ctx=3)
    pk = to_pool(refk, table, lens, n_pages, BF16_NAN)
    pv = to_pool(refv, table, lens, n_pages, BF16_NAN)
    pck = pcv = psk = psv = None
    if bits != 16:
        wpr, ng = d * bits // 32, d // group
        as_words = lambda buf: buf[: B * Hkv * cap * wpr * 4].view(torch.int32).view(B, Hkv, cap, wpr)
        as_halves = lambda buf: buf[: B * Hkv * cap * ng * 2].view(torch.int16).view(B, Hkv, cap, ng)
        pck = to_pool(as_words(ck), table, lens, n_pages, -1)
        pcv = to_pool(as_words(cv), table, lens, n_pages, -1)
        psk = to_pool(as_halves(sk), table, lens, n_pages, 0x7E00)
        psv = to_pool(as_halves(sv), table, lens, n_pages, 0x7E00)
    shape = rq.make_shape(B, Hkv, cap, d, group, q_heads=Hkv * G)
    lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
    table_d = torch.tensor(table, dtype=torch.int32, device="cuda")
    out_p = torch.empty((B, Hkv * G, d), dtype=torch.float32, device="cuda")
    out_d = torch.empty_like(out_p)
    ws_p = rq.alloc_workspace(shape, varlen=True)
    rq.rq_decode_attention_paged(shape, lens_d, table_d, max_pages, n_pages, q, pk, pv, pck, pcv,
                                 psk, psv, bits, w.seed, 0.0, tail_k, tail_v, 1, 3, out_p, ws_p)
    rq.rq_decode_attention_varlen(shape, lens_d, q, refk, refv, ck, cv, sk, sv, bits, w.seed, 0.0,
                                  tail_k, tail_v, 1, 3, out_d, rq.alloc_workspace(shape, varlen=True))
    torch.cuda.synchronize()
    assert rq.rq_workspace_status(ws_p) == 0
    assert torch.equal(out_p, out_d)
    # oracle for two heads
    for b, h in ((1, 0), (2, 1)):
        n = lens[b]
        rk, rv = u16(refk[b, h, :n]), u16(refv[b, h, :n])
        if bits == 16:
            K = oracle.bf16_to_f32(rk).astype(np.float64)
            V = oracle.bf16_to_f32(rv).astype(np.float64)
        else:
            cwk, csk, _ = oracle.encode_rows_f32(u16(xk[b, h, :n]), rk, bits, group, w.seed)
            cwv, csv, _ = oracle.encode_rows_f32(u16(xv[b, h, :n]), rv, bits, group, w.seed)
            K = oracle.reconstruct_rows_f64(rk, cwk, csk, bits, group, w.seed)
            V = oracle.reconstruct_rows_f64(rv, cwv, csv, bits, group, w.seed)
        K = np.concatenate([K, oracle.bf16_to_f32(u16(tail_k[b, h, :1])).astype(np.float64)])
        V = np.concatenate([V, oracle.bf16_to_f32(u16(tail_v[b, h, :1])).astype(np.float64)])
        qh = oracle.bf16_to_f32(u16(q[b, h * G:(h + 1) * G])).astype(np.float64)
        want = oracle.attention_f64(qh, K, V, 1.0 / np.sqrt(d))
        assert np.abs(out_p[b, h * G:(h + 1) * G].double().cpu().numpy() - want).max() <= OUT_TOL


def test_bad_page_inside_a_length_is_flagged_and_read_as_empty():
    lens, max_pages, n_pages = [130, 64], 3, 6
    w, refk, refv, xk, xv, ck, cv, sk, sv, table, group = build_paged_case(1, 16, lens, max_pages,
                                                                           n_pages, 5)
    B, Hkv, d = len(lens), w.kv_heads, w.head_dim
    table[0, 1] = 999                      # inside sequence 0's length, outside the pool
    pk = to_pool(refk, np.where(table < 0, 0, np.minimum(table, n_pages - 1)), [64, 64],
                 n_pages, 0)
    pv = pk.clone()
    shape = rq.make_shape(B, Hkv, max_pages * PAGE, d, group)
    ws = rq.alloc_workspace(shape, varlen=True)
    out = torch.empty((B, Hkv, d), dtype=torch.float32, device="cuda")
    q = synth.query(w, 0, 1)
    rq.rq_decode_attention_paged(shape, torch.tensor(lens, dtype=torch.int32, device="cuda"),
                                 torch.tensor(table, dtype=torch.int32, device="cuda"), max_pages,
                                 n_pages, q, pk, pv, None, None, None, None, 16, w.seed, 0.0,
                                 None, None, 0, 0, out, ws)
    torch.cuda.synchronize()
    assert rq.rq_workspace_status(ws) & 32
    assert torch.isfinite(out).all()


@pytest.mark.parametrize("refits", [0, 2])
def test_paged_encode_writes_its_pool_rows_only(refits):
    B, Hkv, d, group, n_tok = 3, 2, 128, 32, 70
    max_pages, n_pages = 4, 12
    w = synth.Workload("pgenc", 3, 1, B, n_tok, Hkv, Hkv, d, group, (2, 4), (0.2, 0.1), 33)
    ref = synth.reference(w, 0, 0)
    loops = [synth.loop_kv(w, 0, 0, l, ref) for l in (1, 2)]
    rng = np.random.default_rng(3)
    table = rng.permutation(n_pages)[:B * max_pages].reshape(B, max_pages).astype(np.int32)
    pos = np.array([0, 60, 130], dtype=np.int32)           # spans page boundaries
    pool_shape = rq.make_shape(n_pages, Hkv, PAGE, d, group)
    codes = [rq.alloc_codes(pool_shape, b) for b in w.bits]
    scales = [rq.alloc_scales(pool_shape, b) for b in w.bits]
    ref_pool = torch.full((n_pages, Hkv, PAGE, d), 3.0, dtype=torch.bfloat16, device="cuda")
    for buf in codes + scales:
        buf.fill_(0x5A)
    rq.rq_encode_paged(rq.make_shape(B, Hkv, n_tok, d, group), loops, ref, list(w.bits), w.seed,
                       refits, torch.tensor(pos, device="cuda"),
                       torch.tensor(table, device="cuda"), max_pages, n_pages, codes, scales,
                       ref_out=ref_pool)
    torch.cuda.synchronize()
    written = np.zeros((n_pages, Hkv, PAGE), dtype=bool)
    for l, bits in enumerate(w.bits):
        wpr = d * bits // 32
        pool_w = codes[l][: n_pages * Hkv * PAGE * wpr * 4].view(torch.int32)
        pool_w = pool_w.view(n_pages, Hkv, PAGE, wpr).cpu().numpy().view(np.uint32)
        src_x = u16(loops[l]).reshape(B, Hkv, n_tok, d)
        src_r = u16(ref).reshape(B, Hkv, n_tok, d)
        for b in range(B):
            if refits:
                want, _ = oracle.encode_rows_refined_f32(src_x[b].reshape(-1, d),
                                                         src_r[b].reshape(-1, d), bits, group,
                                                         w.seed, refits)
            else:
                want, _, _ = oracle.encode_rows_f32(src_x[b].reshape(-1, d),
                                                    src_r[b].reshape(-1, d), bits, group, w.seed)
            want = want.reshape(Hkv, n_tok, wpr)
            for t in range(n_tok):
                p_ = pos[b] + t
                page, off = table[b, p_ // PAGE], p_ % PAGE
                assert np.array_equal(pool_w[page, :, off], want[:, t])
                written[page, :, off] = True
                assert torch.equal(ref_pool[page, :, off], ref[b, :, t])
        assert (pool_w[~written] == 0x5A5A5A5A).all()
    assert (ref_pool.view(torch.int16).cpu().numpy()[~written] == u16(torch.tensor(3.0,
            dtype=torch.bfloat16))[()]).all()
