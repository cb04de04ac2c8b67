"""rq_reconstruct (the storage format's decoder) against the oracle's fp64
reconstruction of the same rows.  The oracle encodes the rows itself."""
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


@pytest.mark.parametrize("d,group,bits,ctx", [(128, 32, 2, 300), (128, 64, 4, 65), (64, 32, 2, 7),
                                              (64, 64, 4, 130), (128, 32, 16, 50)])
def test_reconstruct_matches_oracle(d, group, bits, ctx):
    bl = (bits, 16) if bits != 16 else (2, 16)
    w = synth.Workload("rec", 3, 1, 2, ctx, 3, 3, d, group, bl, (0.3, 0.1), 61)
    ref = synth.reference(w, 0, 0)
    x = synth.loop_kv(w, 0, 0, 1, ref)
    rows = ref.numel() // d
    if bits == 16:
        codes = scales = None
        want = oracle.bf16_to_f32(u16(ref)).astype(np.float64).reshape(rows, d)
    else:
        (codes,), (scales,) = rq.encode([x], ref, [bits], group, w.seed)
        wo, so, _ = oracle.encode_rows_f32(u16(x).reshape(rows, d), u16(ref).reshape(rows, d),
                                           bits, group, w.seed)
        want = oracle.reconstruct_rows_f64(u16(ref).reshape(rows, d), wo, so, bits, group, w.seed)
    got32 = rq.reconstruct(ref, codes, scales, bits, group, w.seed).reshape(rows, d)
    got16 = rq.reconstruct(ref, codes, scales, bits, group, w.seed, out_bf16=True).reshape(rows, d)
    torch.cuda.synchronize()
    g32 = got32.double().cpu().numpy()
    assert np.abs(g32 - want).max() <= 2e-5 * (1 + np.abs(want).max())
    # bf16 output: the same fp32 value rounded to nearest-even once, so it is
    # exactly the host's rounding of the fp32 output, and within half a bf16
    # step (2^-8 relative) plus the fp32 tolerance of the oracle's value
    assert torch.equal(got16.cpu(), got32.cpu().to(torch.bfloat16))
    g16 = got16.float().cpu().numpy().astype(np.float64)
    tol32 = 2e-5 * (1 + np.abs(want).max())
    assert np.all(np.abs(g16 - want) <= (np.abs(want) + tol32) * 2.0 ** -8 + tol32)


def test_reconstruct_with_capacity_writes_only_ctx_tokens():
    w = synth.Workload("cap", 3, 1, 1, 40, 2, 2, 128, 32, (2, 16), (0.2, 0.1), 62)
    ref = synth.reference(w, 0, 0)
    x = synth.loop_kv(w, 0, 0, 1, ref)
    (codes,), (scales,) = rq.encode([x], ref, [2], 32, w.seed)
    shape = rq.make_shape(1, 2, 25, 128, 32, ctx_cap=40)
    out = torch.full((1, 2, 40, 128), 3.0, dtype=torch.float32, device="cuda")
    rq.rq_reconstruct(shape, ref, codes, scales, 2, w.seed, out)
    full = rq.reconstruct(ref, codes, scales, 2, 32, w.seed)
    torch.cuda.synchronize()
    assert torch.equal(out[:, :, :25], full[:, :, :25])
    assert (out[:, :, 25:] == 3.0).all()
