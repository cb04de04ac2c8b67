"""ResidualQuant KV cache for looped Transformers on B200 (sm_100a).

The compute path is librq.so (hand-written CUDA, C ABI in include/rq.h);
this package is its Python binding.  torch is used for device memory and
streams only: the helpers below allocate buffers with the sizes the library
reports and pass pointers through.

    from kv_cache_residual_rq_b200 import make_shape, encode, decode_attention
"""
from ._abi import (RQ_ERR_ALIGNMENT, RQ_ERR_CUDA, RQ_ERR_INVALID_ARG, RQ_ERR_UNSUPPORTED,
                   RQ_ERR_WORKSPACE, RQ_MAX_LOOPS, RQ_OK, RqError, lib, make_shape,
                   rq_codes_bytes, rq_decode_attention, rq_decode_attention_noalloc,
                   rq_decode_attention_tail, rq_decode_workspace_bytes, rq_encode, rq_encode_at,
                   rq_encode_at_ex, rq_encode_take_status, rq_reconstruct, RQ_MAX_REFINE,
                   RQ_MAX_VARLEN_BATCH, rq_decode_attention_varlen,
                   rq_decode_workspace_bytes_varlen, rq_encode_cr_at, rq_reconstruct_cr,
                   rq_decode_attention_cr, rq_decode_attention_paged, rq_encode_paged,
                   rq_scales_bytes, rq_shape, rq_status_string, rq_version,
                   rq_workspace_status)

__all__ = [
    "RQ_OK", "RQ_ERR_INVALID_ARG", "RQ_ERR_UNSUPPORTED", "RQ_ERR_ALIGNMENT", "RQ_ERR_WORKSPACE",
    "RQ_ERR_CUDA", "RQ_MAX_LOOPS", "RqError", "lib", "rq_shape", "make_shape", "rq_version",
    "rq_status_string", "rq_codes_bytes", "rq_scales_bytes", "rq_decode_workspace_bytes",
    "rq_encode", "rq_encode_at", "rq_encode_at_ex", "RQ_MAX_REFINE", "rq_decode_attention", "rq_decode_attention_tail",
    "rq_decode_attention_noalloc", "rq_decode_attention_varlen", "rq_decode_workspace_bytes_varlen",
    "RQ_MAX_VARLEN_BATCH", "rq_reconstruct", "rq_encode_cr_at", "rq_reconstruct_cr",
    "rq_decode_attention_cr", "encode_cr", "reconstruct_cr", "decode_attention_cr",
    "rq_decode_attention_paged", "rq_encode_paged", "rq_workspace_status", "rq_encode_take_status",
    "alloc_codes", "alloc_scales", "alloc_workspace", "encode", "decode_attention", "reconstruct",
]


def alloc_codes(shape, bits, device="cuda"):
    """uint8 device buffer of rq_codes_bytes(shape, bits) bytes (None for bits 16)."""
    import torch
    n = rq_codes_bytes(shape, bits)
    return torch.empty(n, dtype=torch.uint8, device=device) if n else None


def alloc_scales(shape, bits, device="cuda"):
    import torch
    n = rq_scales_bytes(shape, bits)
    return torch.empty(n, dtype=torch.uint8, device=device) if n else None


def alloc_workspace(shape, device="cuda", varlen=False):
    """Zero-filled decode workspace, as rq_decode_attention (or, with
    varlen, rq_decode_attention_varlen) requires."""
    import torch
    n = rq_decode_workspace_bytes_varlen(shape) if varlen else rq_decode_workspace_bytes(shape)
    if n == 0:
        raise RqError(RQ_ERR_INVALID_ARG, "rq_decode_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def encode(kv_loops, ref, bits_per_loop, group, seed, stream=None, refine_iters=0):
    """Encode non-final loops (bf16 tensors [rows, Hkv, T, d]) against `ref`,
    with `refine_iters` least-squares refits per group.

    Returns (codes, scales): per loop a uint8 device buffer, or None for a
    loop kept in BF16 (bits 16)."""
    rows, hkv, t, d = ref.shape
    shape = make_shape(rows, hkv, t, d, group)
    codes = [alloc_codes(shape, b, ref.device) for b in bits_per_loop]
    scales = [alloc_scales(shape, b, ref.device) for b in bits_per_loop]
    if refine_iters:
        rq_encode_at_ex(shape, t, 0, t, 0, kv_loops, ref, bits_per_loop, seed, refine_iters,
                        codes, scales, stream=stream)
    else:
        rq_encode(shape, kv_loops, ref, bits_per_loop, seed, codes, scales, stream)
    return codes, scales


def reconstruct(ref, codes, scales, bits, group, seed, out_bf16=False, stream=None):
    """Rebuild a loop's rows [rows, Hkv, T, d] from ref (bf16) and its codes/scales
    (as returned by encode; None for bits 16).  Returns fp32 (or bf16) rows."""
    import torch
    rows, hkv, t, d = ref.shape
    shape = make_shape(rows, hkv, t, d, group)
    out = torch.empty(ref.shape, dtype=torch.bfloat16 if out_bf16 else torch.float32,
                      device=ref.device)
    rq_reconstruct(shape, ref, codes, scales, bits, seed, out, out_bf16, stream)
    return out


def decode_attention(q, ref_k, ref_v, codes_k, codes_v, scales_k, scales_v, bits, group, seed,
                     softmax_scale=0.0, out=None, workspace=None, stream=None, ctx=None,
                     tail_k=None, tail_v=None, n_tail=0):
    """Decode attention of one loop.  q [B, Hq, d] bf16; ref_k/ref_v
    [B, Hkv, T_cap, d] bf16 of which the first `ctx` tokens (default T_cap) are
    attended; codes/scales as returned by encode (None for bits 16); optional
    BF16 tail tokens tail_k/tail_v [B, Hkv, W, d], the first n_tail attended
    too.  Returns out [B, Hq, d] fp32."""
    import torch
    b, hq, d = q.shape
    _, hkv, t_cap, _ = ref_k.shape
    t = t_cap if ctx is None else ctx
    shape = make_shape(b, hkv, t, d, group, q_heads=hq, ctx_cap=t_cap)
    if out is None:
        out = torch.empty((b, hq, d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(shape, q.device)
    if n_tail:
        rq_decode_attention_tail(shape, q, ref_k, ref_v, codes_k, codes_v, scales_k, scales_v,
                                 bits, seed, softmax_scale, tail_k, tail_v, n_tail,
                                 tail_k.shape[2], out, workspace, stream=stream)
    else:
        rq_decode_attention(shape, q, ref_k, ref_v, codes_k, codes_v, scales_k, scales_v, bits,
                            seed, softmax_scale, out, workspace, stream=stream)
    return out


def encode_cr(kv_loops, ref, ref_bits, bits_per_loop, group, seed, stream=None):
    """Compressed-reference encode of contiguous [rows, Hkv, T, d] bf16 tensors.
    Returns ((ref_codes, ref_scales), codes, scales)."""
    rows, hkv, t, d = ref.shape
    shape = make_shape(rows, hkv, t, d, group)
    rc, rs = alloc_codes(shape, ref_bits, ref.device), alloc_scales(shape, ref_bits, ref.device)
    codes = [alloc_codes(shape, b, ref.device) for b in bits_per_loop]
    scales = [alloc_scales(shape, b, ref.device) for b in bits_per_loop]
    rq_encode_cr_at(shape, t, 0, kv_loops, ref, ref_bits, bits_per_loop, seed, rc, rs, codes,
                    scales, stream=stream)
    return (rc, rs), codes, scales


def reconstruct_cr(shape4, ref_codes, ref_scales, ref_bits, codes, scales, bits, group, seed,
                   device="cuda", out_bf16=False, stream=None):
    """Rows [rows, Hkv, T, d] of a compressed-reference loop (bits 16: the reference)."""
    import torch
    rows, hkv, t, d = shape4
    shape = make_shape(rows, hkv, t, d, group)
    out = torch.empty(shape4, dtype=torch.bfloat16 if out_bf16 else torch.float32,
                      device=device)
    rq_reconstruct_cr(shape, ref_codes, ref_scales, ref_bits, codes, scales, bits, seed, out,
                      out_bf16, stream)
    return out


def decode_attention_cr(q, ref, codes_k, codes_v, scales_k, scales_v, bits, group, seed, ctx_cap,
                        ctx=None, ctx_lens=None, tail_k=None, tail_v=None, n_tail=0,
                        softmax_scale=0.0, out=None, workspace=None, stream=None, kv_heads=None):
    """Decode attention over a compressed-reference cache.  ref = (ref_codes_k,
    ref_scales_k, ref_codes_v, ref_scales_v, ref_bits); q [B, Hq, d]; the
    cache has kv_heads heads (default Hq)."""
    import torch
    rck, rsk, rcv, rsv, ref_bits = ref
    b, h, d = q.shape
    hkv = h if kv_heads is None else kv_heads
    shape = make_shape(b, hkv, ctx if ctx is not None else ctx_cap, d, group, q_heads=h,
                       ctx_cap=ctx_cap)
    if out is None:
        out = torch.empty((b, h, d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(shape, q.device, varlen=ctx_lens is not None)
    rq_decode_attention_cr(shape, ctx_lens, q, rck, rcv, rsk, rsv, ref_bits, codes_k, codes_v,
                           scales_k, scales_v, bits, seed, softmax_scale, tail_k, tail_v, n_tail,
                           tail_k.shape[2] if n_tail else 0, out, workspace, stream=stream)
    return out
