"""rq_decode_attention_noalloc: decode attention for callers that cannot
allocate device memory (their host application owns every allocation, or
their path must not call cudaMalloc).  It uses the library's fixed scratch
array instead of a caller workspace.

Checked through the C ABI against rq_decode_attention with a caller
workspace, on two calls in a row (the second sees the scratch the first left
behind).  Both run the same kernel with the same split of the context over
the same CTAs, and the final merge visits the partial records in a fixed
order, so the outputs must be bit-identical.  This file is collected last on
purpose.
"""
import numpy as np
import pytest
import torch

import kv_cache_residual_rq_b200 as rq
from kv_cache_residual_rq_b200 import synth

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 8 << 20  # RQ_NOALLOC_SCRATCH_BYTES in include/rq.h


@pytest.fixture(scope="module")
def cuda_lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_residual_rq_b200 import build
    build.build()
    return rq.lib()


def _inputs(w, batch, ctx, loop):
    refk = synth.reference(w, 0, 0, batch=batch, ctx=ctx)
    refv = synth.reference(w, 0, 1, batch=batch, ctx=ctx)
    xk = synth.loop_kv(w, 0, 0, loop, refk)
    xv = synth.loop_kv(w, 0, 1, loop, refv)
    q = synth.query(w, 0, loop, batch=batch)
    bits = w.bits[loop - 1]
    (ck,), (sk,) = rq.encode([xk], refk, [bits], w.group, w.seed)
    (cv,), (sv,) = rq.encode([xv], refv, [bits], w.group, w.seed)
    return q, refk, refv, ck, cv, sk, sv, bits


@pytest.mark.parametrize("name,batch,ctx,loop", [("ouro1.4b_decode", 4, 1500, 1),
                                                 ("deep_loop_gqa", 3, 777, 2),
                                                 ("tiny", 1, 256, 3)])
def test_noalloc_matches_workspace_call_twice(cuda_lib, name, batch, ctx, loop):
    w = synth.BY_NAME[name]
    q, refk, refv, ck, cv, sk, sv, bits = _inputs(w, batch, ctx, loop)
    want = rq.decode_attention(q, refk, refv, ck, cv, sk, sv, bits, w.group, w.seed)
    shape = rq.make_shape(batch, w.kv_heads, ctx, w.head_dim, w.group, q_heads=w.q_heads)
    outs = []
    for _ in range(2):
        out = torch.full_like(want, float("nan"))
        rq.rq_decode_attention_noalloc(shape, q, refk, refv, ck, cv, sk, sv, bits, w.seed, 0.0,
                                       out)
        outs.append(out)
    torch.cuda.synchronize()
    for out in outs:
        assert torch.isfinite(out).all()
        assert torch.equal(out, want)
    # the reference loop through the same entry point
    ref_want = rq.decode_attention(q, refk, refv, None, None, None, None, 16, w.group, w.seed)
    ref_out = torch.empty_like(ref_want)
    rq.rq_decode_attention_noalloc(shape, q, refk, refv, None, None, None, None, 16, w.seed, 0.0,
                                   ref_out)
    torch.cuda.synchronize()
    assert torch.equal(ref_out, ref_want)


def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_lib):
    # 64 sequences x 16 heads x 32768 tokens needs more scratch than it has
    big = rq.make_shape(256, 16, 32768, 128, 32, q_heads=128)
    assert rq.rq_decode_workspace_bytes(big) > SCRATCH_BYTES
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    st = rq.rq_decode_attention_noalloc(big, dummy, dummy, dummy, dummy, dummy, dummy, dummy, 2,
                                        1, 0.0, dummy, check=False)
    assert st == rq.RQ_ERR_WORKSPACE
    # invalid arguments get rq_decode_attention's statuses, nothing enqueued
    ok = rq.make_shape(1, 2, 64, 128, 32, q_heads=2)
    assert rq.rq_decode_attention_noalloc(ok, None, dummy, dummy, dummy, dummy, dummy, dummy, 2,
                                          1, 0.0, dummy, check=False) == rq.RQ_ERR_INVALID_ARG
    assert rq.rq_decode_attention_noalloc(ok, dummy, dummy, dummy, dummy, dummy, dummy, dummy, 3,
                                          1, 0.0, dummy, check=False) == rq.RQ_ERR_UNSUPPORTED
