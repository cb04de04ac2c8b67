"""The two encoder kernels against the oracle and against each other.

rq_encode of contiguous sources runs the kernel fed by tensor copies (tiles
of 120 rows at head_dim 128, 240 at 64); rq_encode_at with a token pitch
larger than ctx runs the streaming kernel.  Both must give the oracle's codes
bit for bit, over several tiles with a ragged last tile, for every
(head_dim, group, bits) the library builds."""
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


def f16(a):
    return np.vectorize(oracle.f16_to_f64)(a)


@pytest.mark.parametrize("d,group", [(128, 32), (128, 64), (64, 32), (64, 64)])
def test_tensor_copy_and_streaming_encoders_match_oracle(d, group):
    B, H, T = 1, 3, 247                     # 741 rows: 7 tiles of 120 (4 of 240), ragged
    w = synth.Workload("paths", 4, 1, B, T, H, H, d, group, (2, 4, 16), (0.3, 0.2, 0.1), 71)
    ref = synth.reference(w, 0, 0)
    loops = [synth.loop_kv(w, 0, 0, l, ref) for l in range(1, 4)]
    rows = B * H * T
    codes, scales = rq.encode(loops, ref, list(w.bits), group, w.seed)       # tensor copies
    # streaming kernel: the same tokens, read from and written to arrays of pitch T + 5
    P = T + 5
    pad = lambda x: torch.nn.functional.pad(x, (0, 0, 0, 5)).contiguous()
    shape_p = rq.make_shape(B, H, T, d, group, ctx_cap=P)
    c2 = [rq.alloc_codes(rq.make_shape(B, H, P, d, group), b) for b in w.bits]
    s2 = [rq.alloc_scales(rq.make_shape(B, H, P, d, group), b) for b in w.bits]
    ref_copy = torch.zeros((B, H, P, d), dtype=torch.bfloat16, device="cuda")
    rq.rq_encode_at(rq.make_shape(B, H, T, d, group), P, 0, P, 0, [pad(x) for x in loops],
                    pad(ref), list(w.bits), w.seed, c2, s2, ref_out=ref_copy)
    torch.cuda.synchronize()
    assert rq.rq_encode_take_status() == 0
    assert torch.equal(ref_copy[:, :, :T], ref)
    r_np = u16(ref).reshape(rows, d)
    for l, bits in enumerate(w.bits):
        if bits == 16:
            continue
        want_w, want_s, _ = oracle.encode_rows_f32(u16(loops[l]).reshape(rows, d), r_np, bits,
                                                   group, w.seed)
        got_a = words(codes[l], rows, d, bits).cpu().numpy().view(np.uint32)
        got_b = words(c2[l], B * H * P, d, bits).view(B * H, P, -1)[:, :T].reshape(rows, -1)
        got_b = got_b.cpu().numpy().view(np.uint32)
        assert np.array_equal(got_a, want_w), f"tensor-copy kernel, loop {l + 1}"
        assert np.array_equal(got_b, want_w), f"streaming kernel, loop {l + 1}"
        sa = f16(halves(scales[l], rows, d, group).cpu().numpy().view(np.uint16))
        sb = halves(s2[l], B * H * P, d, group).view(B * H, P, -1)[:, :T].reshape(rows, -1)
        sb = f16(sb.cpu().numpy().view(np.uint16))
        sw = f16(want_s)
        tol = np.maximum(1e-3 * np.abs(sw), 2.0 ** -24)
        assert np.all(np.abs(sa - sw) <= tol) and np.all(np.abs(sb - sw) <= tol)


def test_tensor_copy_encoder_copies_the_reference_rows():
    B, H, T, d = 2, 2, 130, 128
    w = synth.Workload("refout", 3, 1, B, T, H, H, d, 32, (2, 16), (0.2, 0.1), 72)
    ref = synth.reference(w, 0, 1)
    x = synth.loop_kv(w, 0, 1, 1, ref)
    shape = rq.make_shape(B, H, T, d, 32)
    codes = [rq.alloc_codes(shape, 2), None]
    scales = [rq.alloc_scales(shape, 2), None]
    out = torch.full_like(ref, 5.0)
    rq.rq_encode_at(shape, T, 0, T, 0, [x, None], ref, [2, 16], w.seed, codes, scales,
                    ref_out=out)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    (c1,), _ = rq.encode([x], ref, [2], 32, w.seed)
    assert torch.equal(codes[0][: c1.numel()], c1)
