"""Host-side checks of librq.so that need no GPU.

The library loads, exports every entry point include/rq.h declares, answers
its size queries, and rejects bad arguments with the documented status
before touching the device.  None of these calls reaches a kernel launch.
"""
import ctypes
import os
import re

import pytest

import kv_cache_residual_rq_b200 as rq
from kv_cache_residual_rq_b200 import build as rq_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

FAKE = 0x100000          # an aligned, never-dereferenced address
MISALIGNED = 0x100008


@pytest.fixture(scope="module", autouse=True)
def built():
    rq_build.build()


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(rq_\w+)\s*\(", text, re.M))
    return sorted(names)


def test_header_declares_the_abi():
    names = declared_functions()
    for want in ("rq_encode", "rq_decode_attention", "rq_codes_bytes", "rq_scales_bytes",
                 "rq_decode_workspace_bytes", "rq_status_string", "rq_version",
                 "rq_workspace_status"):
        assert want in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(rq_build.LIB)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_bounds_checked_library_exports_every_declared_symbol():
    # librq_bounds.so: the same ABI, built with every computed index checked
    if rq_build._stale(rq_build.LIB_BOUNDS):
        pytest.skip("librq_bounds.so not built from the current sources")
    lib = ctypes.CDLL(rq_build.LIB_BOUNDS)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_version_and_status_strings():
    assert rq.rq_version() >= 100
    for s in range(6):
        assert rq.rq_status_string(s)
    assert rq.rq_status_string(99) == "unknown status"


def test_size_queries():
    s = rq.make_shape(16, 16, 4096, 128, 32)
    assert rq.rq_codes_bytes(s, 2) == 16 * 16 * 4096 * 128 * 2 // 8
    assert rq.rq_codes_bytes(s, 4) == 16 * 16 * 4096 * 128 * 4 // 8
    assert rq.rq_codes_bytes(s, 16) == 0
    assert rq.rq_scales_bytes(s, 2) == 16 * 16 * 4096 * 4 * 2
    # rounded up to 16 bytes
    odd = rq.make_shape(1, 1, 3, 128, 64)
    assert rq.rq_scales_bytes(odd, 2) == 16
    assert rq.rq_codes_bytes(rq.make_shape(1, 1, 0, 64, 32), 2) == 0
    # unsupported shapes answer 0
    assert rq.rq_codes_bytes(rq.make_shape(1, 1, 8, 96, 32), 2) == 0
    assert rq.rq_scales_bytes(rq.make_shape(1, 1, 8, 128, 16), 2) == 0
    ws = rq.rq_decode_workspace_bytes(rq.make_shape(16, 16, 4096, 128, 32))
    assert ws > 16 and ws % 16 == 0
    assert rq.rq_decode_workspace_bytes(rq.make_shape(1, 3, 64, 128, 32, q_heads=4)) == 0
    assert rq.rq_decode_workspace_bytes(rq.make_shape(1, 1, 0, 128, 32)) == 0


def _decode(shape, bits=2, q=FAKE, rk=FAKE, rv=FAKE, ck=FAKE, cv=FAKE, sk=FAKE, sv=FAKE,
            out=FAKE, ws=FAKE, ws_bytes=None, scale=0.0):
    if ws_bytes is None:
        ws_bytes = rq.rq_decode_workspace_bytes(shape) or 1 << 30
    return rq.rq_decode_attention(shape, q, rk, rv, ck, cv, sk, sv, bits, 1, scale, out, ws,
                                  ws_bytes, stream=0, check=False)



def _decode_cr(shape, ref_bits=8, rck=FAKE, rsv=FAKE, bits=16, q=FAKE):
    ws_bytes = rq.rq_decode_workspace_bytes(shape) or 1 << 30
    return rq.rq_decode_attention_cr(shape, None, q, rck, FAKE, FAKE, rsv, ref_bits, None, None,
                                      None, None, bits, 1, 0.0, None, None, 0, 0, FAKE, FAKE,
                                      ws_bytes, stream=0, check=False)


def test_cr_decode_rejects_bad_arguments_before_launch():
    E = rq
    gqa = rq.make_shape(2, 2, 100, 128, 32, q_heads=8)
    assert _decode_cr(gqa, ref_bits=3) == E.RQ_ERR_UNSUPPORTED
    assert _decode_cr(rq.make_shape(2, 2, 100, 128, 32), ref_bits=16) == E.RQ_ERR_UNSUPPORTED
    # past the format checks, INT8 and INT4 with grouped queries reach the
    # pointer checks
    assert _decode_cr(gqa, rck=None) == E.RQ_ERR_INVALID_ARG
    assert _decode_cr(gqa, ref_bits=4, rck=None) == E.RQ_ERR_INVALID_ARG
    assert _decode_cr(gqa, ref_bits=4, rsv=MISALIGNED) == E.RQ_ERR_ALIGNMENT
    assert _decode_cr(gqa, rsv=MISALIGNED) == E.RQ_ERR_ALIGNMENT
    assert _decode_cr(gqa, q=MISALIGNED) == E.RQ_ERR_ALIGNMENT
    assert _decode_cr(rq.make_shape(2, 1, 100, 128, 32, q_heads=16)) == E.RQ_ERR_UNSUPPORTED

def test_decode_rejects_bad_arguments_before_launch():
    good = rq.make_shape(2, 2, 100, 128, 32, q_heads=8)
    E = rq
    assert _decode(good, q=None) == E.RQ_ERR_INVALID_ARG
    assert _decode(good, out=None) == E.RQ_ERR_INVALID_ARG
    assert _decode(good, ck=None) == E.RQ_ERR_INVALID_ARG
    assert _decode(good, bits=3) == E.RQ_ERR_UNSUPPORTED
    assert _decode(good, rk=MISALIGNED) == E.RQ_ERR_ALIGNMENT
    assert _decode(good, sv=MISALIGNED) == E.RQ_ERR_ALIGNMENT
    assert _decode(good, ws=None) == E.RQ_ERR_WORKSPACE
    assert _decode(good, ws_bytes=rq.rq_decode_workspace_bytes(good) - 16) == E.RQ_ERR_WORKSPACE
    assert _decode(good, ws=MISALIGNED) == E.RQ_ERR_ALIGNMENT
    assert _decode(good, scale=float("nan")) == E.RQ_ERR_INVALID_ARG
    assert _decode(rq.make_shape(2, 3, 100, 128, 32, q_heads=8)) == E.RQ_ERR_INVALID_ARG
    assert _decode(rq.make_shape(2, 2, 0, 128, 32, q_heads=8)) == E.RQ_ERR_INVALID_ARG
    assert _decode(rq.make_shape(0, 2, 10, 128, 32, q_heads=8)) == E.RQ_ERR_INVALID_ARG
    assert _decode(rq.make_shape(2, 2, 10, 96, 32, q_heads=8)) == E.RQ_ERR_UNSUPPORTED
    assert _decode(rq.make_shape(2, 2, 10, 128, 48, q_heads=8)) == E.RQ_ERR_UNSUPPORTED
    assert _decode(rq.make_shape(2, 1, 10, 128, 32, q_heads=3)) == E.RQ_ERR_UNSUPPORTED
    assert _decode(rq.make_shape(2, 1, 10, 128, 32, q_heads=16)) == E.RQ_ERR_UNSUPPORTED
    # bits 16 needs no codes or scales, but still checks the rest
    assert _decode(good, bits=16, ck=None, cv=None, sk=None, sv=None, q=MISALIGNED) == \
        E.RQ_ERR_ALIGNMENT
    assert rq.rq_decode_attention(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 1, 0.0,
                                  FAKE, FAKE, 1 << 20, stream=0, check=False) == \
        E.RQ_ERR_INVALID_ARG


def _encode(shape, bits=(2, 2, 2), x=FAKE, ref=FAKE, codes=FAKE, scales=FAKE):
    n = len(bits)
    return rq.rq_encode(shape, [x] * n, ref, list(bits), 0, [codes] * n, [scales] * n,
                        stream=0, check=False)


def test_encode_rejects_bad_arguments_before_launch():
    good = rq.make_shape(2, 2, 100, 128, 32)
    E = rq
    assert _encode(good, ref=None) == E.RQ_ERR_INVALID_ARG
    assert _encode(good, x=None) == E.RQ_ERR_INVALID_ARG
    assert _encode(good, codes=None) == E.RQ_ERR_INVALID_ARG
    assert _encode(good, bits=(2, 3)) == E.RQ_ERR_UNSUPPORTED
    assert _encode(good, bits=()) == E.RQ_ERR_INVALID_ARG
    assert _encode(good, bits=(2,) * 17) == E.RQ_ERR_INVALID_ARG
    assert _encode(good, x=MISALIGNED) == E.RQ_ERR_ALIGNMENT
    assert _encode(good, scales=MISALIGNED) == E.RQ_ERR_ALIGNMENT
    assert _encode(rq.make_shape(2, 2, 100, 80, 32)) == E.RQ_ERR_UNSUPPORTED
    assert _encode(rq.make_shape(2, 2, 100, 64, 128)) == E.RQ_ERR_UNSUPPORTED
    assert _encode(rq.make_shape(-1, 2, 100, 64, 32)) == E.RQ_ERR_INVALID_ARG
    # nothing to do: empty context, or every loop kept in BF16
    assert _encode(rq.make_shape(2, 2, 0, 128, 32)) == E.RQ_OK
    assert _encode(good, bits=(16, 16), x=None, codes=None, scales=None) == E.RQ_OK


def plan(batch, kv_heads, ctx, num_sms, tile=64, per_sm=2, max_ctas=1024):
    """Host restatement of the decode work split, for checking its bounds."""
    heads = batch * kv_heads
    nt = (ctx + tile - 1) // tile
    n_tiles = heads * nt
    P = max(1, min(num_sms * per_sm, max_ctas, n_tiles))
    max_contrib = min(nt, max_ctas // heads + 2)
    return heads, nt, n_tiles, P, max_contrib


@pytest.mark.parametrize("batch,kv_heads,ctx", [
    (1, 2, 256), (16, 16, 4096), (8, 16, 32768), (32, 8, 8192), (1, 1, 1), (3, 5, 1000),
    (64, 16, 32768), (1, 1, 64 * 2000 + 1), (7, 3, 65), (1, 16, 32768)])
@pytest.mark.parametrize("num_sms", [1, 148, 132, 512])
def test_decode_split_covers_each_head_within_its_record_budget(batch, kv_heads, ctx, num_sms):
    heads, nt, n_tiles, P, max_contrib = plan(batch, kv_heads, ctx, num_sms)
    start = [c * n_tiles // P for c in range(P + 1)]
    assert all(start[c + 1] > start[c] for c in range(P))        # no idle CTA
    sizes = [start[c + 1] - start[c] for c in range(P)]
    assert max(sizes) - min(sizes) <= 1                          # balanced
    for hd in {0, heads // 2, heads - 1}:
        f, e = hd * nt, hd * nt + nt - 1
        c_first = ((f + 1) * P - 1) // n_tiles
        c_last = ((e + 1) * P - 1) // n_tiles
        assert start[c_first] <= f < start[c_first + 1]
        assert start[c_last] <= e < start[c_last + 1]
        assert c_last - c_first + 1 <= max_contrib


def test_capacity_and_window_arguments_are_checked():
    E = rq
    # ctx_cap below ctx is rejected; size queries follow the capacity
    bad = rq.make_shape(2, 2, 100, 128, 32, q_heads=2, ctx_cap=50)
    assert rq.rq_codes_bytes(bad, 2) == 0
    assert _decode(bad) == E.RQ_ERR_INVALID_ARG
    grown = rq.make_shape(2, 2, 100, 128, 32, ctx_cap=300)
    assert rq.rq_codes_bytes(grown, 2) == 2 * 2 * 300 * 128 * 2 // 8
    assert rq.rq_scales_bytes(grown, 2) == 2 * 2 * 300 * 4 * 2
    # encode_at: ranges must fit their pitches
    s = rq.make_shape(2, 2, 5, 128, 32)
    enc = lambda sp, so, dp, do, ref_out=None: rq.rq_encode_at(
        s, sp, so, dp, do, [FAKE], FAKE, [2], 0, [FAKE], [FAKE], ref_out, stream=0, check=False)
    assert enc(4, 0, 10, 0) == E.RQ_ERR_INVALID_ARG
    assert enc(10, 6, 10, 0) == E.RQ_ERR_INVALID_ARG
    assert enc(10, 0, 10, 6) == E.RQ_ERR_INVALID_ARG
    assert enc(10, -1, 10, 0) == E.RQ_ERR_INVALID_ARG
    assert enc(10, 0, 10, 0, ref_out=MISALIGNED) == E.RQ_ERR_ALIGNMENT
    # decode with a tail: count, pointers, pitch, alignment
    good = rq.make_shape(2, 2, 100, 128, 32, q_heads=8)
    ws = rq.rq_decode_workspace_bytes(good)
    tail = lambda tk, tv, n, pitch: rq.rq_decode_attention_tail(
        good, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 1, 0.0, tk, tv, n, pitch, FAKE, FAKE,
        ws, stream=0, check=False)
    assert tail(FAKE, FAKE, 257, 300) == E.RQ_ERR_INVALID_ARG
    assert tail(FAKE, FAKE, -1, 300) == E.RQ_ERR_INVALID_ARG
    assert tail(None, FAKE, 3, 4) == E.RQ_ERR_INVALID_ARG
    assert tail(FAKE, FAKE, 3, 2) == E.RQ_ERR_INVALID_ARG
    assert tail(FAKE, MISALIGNED, 3, 4) == E.RQ_ERR_ALIGNMENT


def test_reconstruct_rejects_bad_arguments_before_launch():
    E = rq
    s = rq.make_shape(2, 2, 10, 128, 32)
    rec = lambda shape=s, bits=2, ref=FAKE, codes=FAKE, scales=FAKE, out=FAKE: rq.rq_reconstruct(
        shape, ref, codes, scales, bits, 0, out, stream=0, check=False)
    assert rec(ref=None) == E.RQ_ERR_INVALID_ARG
    assert rec(out=None) == E.RQ_ERR_INVALID_ARG
    assert rec(codes=None) == E.RQ_ERR_INVALID_ARG
    assert rec(bits=3) == E.RQ_ERR_UNSUPPORTED
    assert rec(shape=rq.make_shape(2, 2, 10, 96, 32)) == E.RQ_ERR_UNSUPPORTED
    assert rec(shape=rq.make_shape(2, 2, 10, 128, 32, ctx_cap=5)) == E.RQ_ERR_INVALID_ARG
    assert rec(scales=MISALIGNED) == E.RQ_ERR_ALIGNMENT
    assert rec(shape=rq.make_shape(2, 2, 0, 128, 32)) == E.RQ_OK      # nothing to rebuild


def test_encode_at_ex_rejects_refits_out_of_range():
    s = rq.make_shape(1, 2, 10, 128, 32)
    call = lambda it: rq.rq_encode_at_ex(s, 10, 0, 10, 0, [FAKE], FAKE, [2], 0, it, [FAKE],
                                         [FAKE], stream=0, check=False)
    assert call(-1) == rq.RQ_ERR_INVALID_ARG
    assert call(rq.RQ_MAX_REFINE + 1) == rq.RQ_ERR_INVALID_ARG
    # in range but nothing to do (ctx 0) is fine without a device
    z = rq.make_shape(1, 2, 0, 128, 32)
    assert rq.rq_encode_at_ex(z, 1, 0, 1, 0, [FAKE], FAKE, [2], 0, rq.RQ_MAX_REFINE, [FAKE],
                              [FAKE], stream=0, check=False) == rq.RQ_OK


def test_varlen_decode_rejects_bad_arguments_before_launch():
    s = rq.make_shape(4, 2, 100, 128, 32, q_heads=8)
    call = lambda shape=s, lens=FAKE: rq.rq_decode_attention_varlen(
        shape, lens, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 0, 0.0, None, None, 0, 0, FAKE,
        FAKE, 1 << 30, stream=0, check=False)
    assert call(lens=None) == rq.RQ_ERR_INVALID_ARG
    assert call(lens=FAKE + 2) == rq.RQ_ERR_ALIGNMENT
    big = rq.make_shape(rq.RQ_MAX_VARLEN_BATCH + 1, 2, 100, 128, 32, q_heads=8)
    assert call(shape=big) == rq.RQ_ERR_INVALID_ARG
    assert rq.rq_decode_workspace_bytes_varlen(big) == 0
    # the workspace bound covers any lengths up to the capacity
    cap = rq.make_shape(4, 2, 64, 128, 32, q_heads=8, ctx_cap=640)
    assert rq.rq_decode_workspace_bytes_varlen(cap) >= rq.rq_decode_workspace_bytes(
        rq.make_shape(4, 2, 640, 128, 32, q_heads=8))
    small_ws = rq.rq_decode_attention_varlen(
        cap, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 0, 0.0, None, None, 0, 0, FAKE,
        FAKE, 64, stream=0, check=False)
    assert small_ws == rq.RQ_ERR_WORKSPACE


def test_paged_entry_points_validate_before_launch():
    s = rq.make_shape(2, 2, 4 * 64, 128, 32)
    dec = lambda shape=s, lens=FAKE, table=FAKE, mp=4, npg=10: rq.rq_decode_attention_paged(
        shape, lens, table, mp, npg, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 0, 0.0, None,
        None, 0, 0, FAKE, FAKE, 1 << 30, stream=0, check=False)
    assert dec(lens=None) == rq.RQ_ERR_INVALID_ARG
    assert dec(table=None) == rq.RQ_ERR_INVALID_ARG
    assert dec(mp=3) == rq.RQ_ERR_INVALID_ARG          # ctx must be max_pages * 64
    assert dec(npg=0) == rq.RQ_ERR_INVALID_ARG
    assert dec(table=FAKE + 2) == rq.RQ_ERR_ALIGNMENT
    enc = lambda pos=FAKE, table=FAKE, it=0: rq.rq_encode_paged(
        rq.make_shape(2, 2, 1, 128, 32), [FAKE], FAKE, [2], 0, it, pos, table, 4, 10, [FAKE],
        [FAKE], stream=0, check=False)
    assert enc(pos=None) == rq.RQ_ERR_INVALID_ARG
    assert enc(table=None) == rq.RQ_ERR_INVALID_ARG
    assert enc(it=rq.RQ_MAX_REFINE + 1) == rq.RQ_ERR_INVALID_ARG
    assert enc(pos=FAKE + 1) == rq.RQ_ERR_ALIGNMENT
