"""Least-squares refinement in both encoder kernels against the oracle.

With refits the binary32 order of <y,l> is part of the specification, so
codes AND scales must equal the oracle's fp32 refinement bit for bit (the
tensor-copy kernel through rq_encode_at_ex with contiguous sources, the
streaming kernel through a token pitch larger than ctx)."""
import numpy as np
import pytest
import torch

import oracle
import kv_cache_residual_rq_b200 as rq
from kv_cache_residual_rq_b200 import synth

pytestmark = pytest.mark.gpu


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


@pytest.mark.parametrize("d,group", [(128, 32), (128, 64), (64, 32), (64, 64)])
@pytest.mark.parametrize("iters", [1, 3])
def test_refined_codes_and_scales_bit_exact(d, group, iters):
    B, H, T = 1, 3, 173                     # 519 rows: several tiles, ragged
    w = synth.Workload("refine", 3, 1, B, T, H, H, d, group, (2, 4), (0.3, 0.15), 81)
    ref = synth.reference(w, 0, 1)
    loops = [synth.loop_kv(w, 0, 1, l, ref) for l in (1, 2)]
    rows = B * H * T
    shape = rq.make_shape(B, H, T, d, group)
    P = T + 3
    shape_p = rq.make_shape(B, H, P, d, group)
    pad = lambda x: torch.nn.functional.pad(x, (0, 0, 0, 3)).contiguous()
    ca = [rq.alloc_codes(shape, b) for b in w.bits]
    sa = [rq.alloc_scales(shape, b) for b in w.bits]
    cb = [rq.alloc_codes(shape_p, b) for b in w.bits]
    sb = [rq.alloc_scales(shape_p, b) for b in w.bits]
    rq.rq_encode_at_ex(shape, T, 0, T, 0, loops, ref, list(w.bits), w.seed, iters, ca, sa)
    rq.rq_encode_at_ex(shape, P, 0, P, 0, [pad(x) for x in loops], pad(ref), list(w.bits),
                       w.seed, iters, cb, sb)
    torch.cuda.synchronize()
    assert rq.rq_encode_take_status() == 0
    r_np = u16(ref).reshape(rows, d)
    for l, bits in enumerate(w.bits):
        want_w, want_s = oracle.encode_rows_refined_f32(u16(loops[l]).reshape(rows, d), r_np,
                                                        bits, group, w.seed, iters)
        got_wa = words(ca[l], rows, d, bits).cpu().numpy().view(np.uint32)
        got_sa = halves(sa[l], rows, d, group).cpu().numpy().view(np.uint16)
        got_wb = words(cb[l], B * H * P, d, bits).view(B * H, P, -1)[:, :T].reshape(rows, -1)
        got_sb = halves(sb[l], B * H * P, d, group).view(B * H, P, -1)[:, :T].reshape(rows, -1)
        assert np.array_equal(got_wa, want_w), f"tensor-copy codes, bits {bits}"
        assert np.array_equal(got_sa, want_s), f"tensor-copy scales, bits {bits}"
        assert np.array_equal(got_wb.cpu().numpy().view(np.uint32), want_w), "streaming codes"
        assert np.array_equal(got_sb.cpu().numpy().view(np.uint16), want_s), "streaming scales"


def test_zero_refits_is_the_plain_encoder():
    w = synth.OURO
    ref = synth.reference(w, 0, 0, batch=2, ctx=300)
    x = synth.loop_kv(w, 0, 0, 1, ref)
    (c0,), (s0,) = rq.encode([x], ref, [2], w.group, w.seed)
    (c1,), (s1,) = rq.encode([x], ref, [2], w.group, w.seed, refine_iters=0)
    shape = rq.make_shape(2, w.kv_heads, 300, w.head_dim, w.group)
    c2, s2 = rq.alloc_codes(shape, 2), rq.alloc_scales(shape, 2)
    rq.rq_encode_at_ex(shape, 300, 0, 300, 0, [x], ref, [2], w.seed, 0, [c2], [s2])
    torch.cuda.synchronize()
    assert torch.equal(c0, c1) and torch.equal(c0, c2)
    assert torch.equal(s0, s1) and torch.equal(s0, s2)


def test_refits_lower_the_reconstruction_error():
    w = synth.OURO
    ref = synth.reference(w, 0, 0, batch=2, ctx=512)
    x = synth.loop_kv(w, 0, 0, 1, ref)
    errs = []
    for it in (0, 1, 4):
        (c,), (s,) = rq.encode([x], ref, [2], w.group, w.seed, refine_iters=it)
        xh = rq.reconstruct(ref, c, s, 2, w.group, w.seed)
        errs.append(torch.linalg.vector_norm(xh - x.float()).item())
    assert errs[1] < errs[0] and errs[2] <= errs[1] * (1 + 1e-3)
    print("relative reconstruction error, refits 0/1/4:",
          [e / torch.linalg.vector_norm(x.float()).item() for e in errs])
