"""ctypes binding of librq.so: the C ABI of include/rq.h, names unchanged.

Argument marshalling only.  Each function takes what the C function takes;
a torch tensor may stand in for a device pointer (its data_ptr() is passed)
and `stream=None` means torch's current CUDA stream.  A non-zero rq_status
raises RqError.  There is no fallback: if librq.so is missing or fails to
load, every call raises.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# RQ_LIBRARY selects another build of the same library (the bounds-checked
# librq_bounds.so); default: the in-tree librq.so
LIB_PATH = os.environ.get("RQ_LIBRARY") or os.path.join(HERE, "librq.so")

RQ_OK = 0
RQ_ERR_INVALID_ARG = 1
RQ_ERR_UNSUPPORTED = 2
RQ_ERR_ALIGNMENT = 3
RQ_ERR_WORKSPACE = 4
RQ_ERR_CUDA = 5
RQ_MAX_LOOPS = 16
RQ_MAX_REFINE = 8
RQ_MAX_VARLEN_BATCH = 1024


class RqError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: rq_status {status} ({rq_status_string(status)})")


class rq_shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("kv_heads", ctypes.c_int32),
                ("q_heads", ctypes.c_int32), ("ctx", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("group", ctypes.c_int32),
                ("ctx_cap", ctypes.c_int32)]

    def __repr__(self):
        return ("rq_shape(batch=%d, kv_heads=%d, q_heads=%d, ctx=%d, head_dim=%d, group=%d, "
                "ctx_cap=%d)" % (self.batch, self.kv_heads, self.q_heads, self.ctx, self.head_dim,
                                 self.group, self.ctx_cap))


def make_shape(batch, kv_heads, ctx, head_dim, group, q_heads=None, ctx_cap=0):
    return rq_shape(batch, kv_heads, kv_heads if q_heads is None else q_heads, ctx, head_dim,
                    group, ctx_cap)


_lib = None


def lib():
    """Load librq.so once; raise if it is absent (no CPU fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run `python -m kv_cache_residual_rq_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        c = ctypes
        sp = c.POINTER(rq_shape)
        L.rq_version.argtypes = []
        L.rq_version.restype = c.c_int
        L.rq_status_string.argtypes = [c.c_int]
        L.rq_status_string.restype = c.c_char_p
        L.rq_codes_bytes.argtypes = [sp, c.c_int]
        L.rq_codes_bytes.restype = c.c_size_t
        L.rq_scales_bytes.argtypes = [sp, c.c_int]
        L.rq_scales_bytes.restype = c.c_size_t
        L.rq_decode_workspace_bytes.argtypes = [sp]
        L.rq_decode_workspace_bytes.restype = c.c_size_t
        L.rq_encode.argtypes = [sp, c.POINTER(c.c_void_p), c.c_int, c.c_void_p,
                                c.POINTER(c.c_uint8), c.c_uint64, c.POINTER(c.c_void_p),
                                c.POINTER(c.c_void_p), c.c_void_p]
        L.rq_encode.restype = c.c_int
        L.rq_decode_attention.argtypes = [sp, c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p,
                                          c.c_void_p, c.c_void_p, c.c_void_p, c.c_int, c.c_uint64,
                                          c.c_float, c.c_void_p, c.c_void_p, c.c_size_t, c.c_void_p]
        L.rq_decode_attention.restype = c.c_int
        L.rq_encode_at.argtypes = [sp, c.c_int, c.c_int, c.c_int, c.c_int,
                                   c.POINTER(c.c_void_p), c.c_int, c.c_void_p,
                                   c.POINTER(c.c_uint8), c.c_uint64, c.POINTER(c.c_void_p),
                                   c.POINTER(c.c_void_p), c.c_void_p, c.c_void_p]
        L.rq_encode_at.restype = c.c_int
        L.rq_encode_at_ex.argtypes = [sp, c.c_int, c.c_int, c.c_int, c.c_int,
                                      c.POINTER(c.c_void_p), c.c_int, c.c_void_p,
                                      c.POINTER(c.c_uint8), c.c_uint64, c.c_int,
                                      c.POINTER(c.c_void_p), c.POINTER(c.c_void_p), c.c_void_p,
                                      c.c_void_p]
        L.rq_encode_at_ex.restype = c.c_int
        L.rq_decode_attention_varlen.argtypes = [sp, c.c_void_p, c.c_void_p, c.c_void_p,
                                                 c.c_void_p, c.c_void_p, c.c_void_p,
                                                 c.c_void_p, c.c_void_p, c.c_int, c.c_uint64,
                                                 c.c_float, c.c_void_p, c.c_void_p, c.c_int,
                                                 c.c_int, c.c_void_p, c.c_void_p, c.c_size_t,
                                                 c.c_void_p]
        L.rq_decode_attention_varlen.restype = c.c_int
        L.rq_decode_workspace_bytes_varlen.argtypes = [sp]
        L.rq_decode_workspace_bytes_varlen.restype = c.c_size_t
        L.rq_encode_cr_at.argtypes = [sp, c.c_int, c.c_int, c.POINTER(c.c_void_p), c.c_int,
                                      c.c_void_p, c.c_int, c.POINTER(c.c_uint8), c.c_uint64,
                                      c.c_void_p, c.c_void_p, c.POINTER(c.c_void_p),
                                      c.POINTER(c.c_void_p), c.c_void_p]
        L.rq_encode_cr_at.restype = c.c_int
        L.rq_reconstruct_cr.argtypes = [sp, c.c_void_p, c.c_void_p, c.c_int, c.c_void_p,
                                        c.c_void_p, c.c_int, c.c_uint64, c.c_void_p, c.c_int,
                                        c.c_void_p]
        L.rq_reconstruct_cr.restype = c.c_int
        L.rq_decode_attention_cr.argtypes = [sp, c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p,
                                             c.c_void_p, c.c_void_p, c.c_int, c.c_void_p,
                                             c.c_void_p, c.c_void_p, c.c_void_p, c.c_int,
                                             c.c_uint64, c.c_float, c.c_void_p, c.c_void_p,
                                             c.c_int, c.c_int, c.c_void_p, c.c_void_p,
                                             c.c_size_t, c.c_void_p]
        L.rq_decode_attention_cr.restype = c.c_int
        L.rq_decode_attention_paged.argtypes = [sp, c.c_void_p, c.c_void_p, c.c_int, c.c_int,
                                                c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p,
                                                c.c_void_p, c.c_void_p, c.c_void_p, c.c_int,
                                                c.c_uint64, c.c_float, c.c_void_p, c.c_void_p,
                                                c.c_int, c.c_int, c.c_void_p, c.c_void_p,
                                                c.c_size_t, c.c_void_p]
        L.rq_decode_attention_paged.restype = c.c_int
        L.rq_encode_paged.argtypes = [sp, c.POINTER(c.c_void_p), c.c_int, c.c_void_p,
                                      c.POINTER(c.c_uint8), c.c_uint64, c.c_int, c.c_void_p,
                                      c.c_void_p, c.c_int, c.c_int, c.POINTER(c.c_void_p),
                                      c.POINTER(c.c_void_p), c.c_void_p, c.c_void_p]
        L.rq_encode_paged.restype = c.c_int
        L.rq_decode_attention_tail.argtypes = [sp, c.c_void_p, c.c_void_p, c.c_void_p,
                                               c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p,
                                               c.c_int, c.c_uint64, c.c_float, c.c_void_p,
                                               c.c_void_p, c.c_int, c.c_int, c.c_void_p,
                                               c.c_void_p, c.c_size_t, c.c_void_p]
        L.rq_decode_attention_tail.restype = c.c_int
        L.rq_decode_attention_noalloc.argtypes = [sp, c.c_void_p, c.c_void_p, c.c_void_p,
                                                  c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p,
                                                  c.c_int, c.c_uint64, c.c_float, c.c_void_p,
                                                  c.c_void_p]
        L.rq_decode_attention_noalloc.restype = c.c_int
        L.rq_reconstruct.argtypes = [sp, c.c_void_p, c.c_void_p, c.c_void_p, c.c_int,
                                     c.c_uint64, c.c_void_p, c.c_int, c.c_void_p]
        L.rq_reconstruct.restype = c.c_int
        L.rq_workspace_status.argtypes = [c.c_void_p, c.c_size_t, c.POINTER(c.c_uint32), c.c_void_p]
        L.rq_workspace_status.restype = c.c_int
        L.rq_encode_take_status.argtypes = [c.POINTER(c.c_uint32)]
        L.rq_encode_take_status.restype = c.c_int
        _lib = L
    return _lib


def _ptr(x):
    """Device pointer of a tensor, an int, or None (NULL)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _shp(shape):
    return None if shape is None else ctypes.byref(shape)


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status, what):
    if status != RQ_OK:
        raise RqError(status, what)


# ---- the C ABI, one function per entry point ---------------------------------

def rq_version():
    return lib().rq_version()


def rq_status_string(status):
    return lib().rq_status_string(int(status)).decode()


def rq_codes_bytes(shape, bits):
    return lib().rq_codes_bytes(_shp(shape), int(bits))


def rq_scales_bytes(shape, bits):
    return lib().rq_scales_bytes(_shp(shape), int(bits))


def rq_decode_workspace_bytes(shape):
    return lib().rq_decode_workspace_bytes(_shp(shape))


def rq_encode(shape, kv_loops, ref, bits_per_loop, seed, codes_out, scales_out, stream=None,
              check=True):
    """kv_loops / codes_out / scales_out: sequences (one entry per non-final
    loop) of tensors, ints or None.  Returns the rq_status."""
    n = len(bits_per_loop)
    ptrs = lambda seq: (ctypes.c_void_p * max(n, 1))(*[_ptr(v) for v in seq])
    bits = (ctypes.c_uint8 * max(n, 1))(*[int(b) for b in bits_per_loop])
    st = lib().rq_encode(_shp(shape), ptrs(kv_loops), n, _ptr(ref), bits,
                         ctypes.c_uint64(seed), ptrs(codes_out), ptrs(scales_out),
                         _stream(stream))
    if check:
        _check(st, "rq_encode")
    return st


def rq_encode_at(shape, src_pitch, src_offset, dst_pitch, dst_offset, kv_loops, ref,
                 bits_per_loop, seed, codes_out, scales_out, ref_out=None, stream=None,
                 check=True):
    n = len(bits_per_loop)
    ptrs = lambda seq: (ctypes.c_void_p * max(n, 1))(*[_ptr(v) for v in seq])
    bits = (ctypes.c_uint8 * max(n, 1))(*[int(b) for b in bits_per_loop])
    st = lib().rq_encode_at(_shp(shape), int(src_pitch), int(src_offset), int(dst_pitch),
                            int(dst_offset), ptrs(kv_loops), n, _ptr(ref), bits,
                            ctypes.c_uint64(seed), ptrs(codes_out), ptrs(scales_out),
                            _ptr(ref_out), _stream(stream))
    if check:
        _check(st, "rq_encode_at")
    return st


def rq_encode_at_ex(shape, src_pitch, src_offset, dst_pitch, dst_offset, kv_loops, ref,
                    bits_per_loop, seed, refine_iters, codes_out, scales_out, ref_out=None,
                    stream=None, check=True):
    n = len(bits_per_loop)
    ptrs = lambda seq: (ctypes.c_void_p * max(n, 1))(*[_ptr(v) for v in seq])
    bits = (ctypes.c_uint8 * max(n, 1))(*[int(b) for b in bits_per_loop])
    st = lib().rq_encode_at_ex(_shp(shape), int(src_pitch), int(src_offset), int(dst_pitch),
                               int(dst_offset), ptrs(kv_loops), n, _ptr(ref), bits,
                               ctypes.c_uint64(seed), int(refine_iters), ptrs(codes_out),
                               ptrs(scales_out), _ptr(ref_out), _stream(stream))
    if check:
        _check(st, "rq_encode_at_ex")
    return st


def rq_decode_workspace_bytes_varlen(shape):
    return lib().rq_decode_workspace_bytes_varlen(_shp(shape))


def rq_decode_attention_varlen(shape, ctx_lens, q, ref_k, ref_v, codes_k, codes_v, scales_k,
                               scales_v, bits, seed, softmax_scale, tail_k, tail_v, n_tail,
                               tail_pitch, out, workspace, workspace_bytes=None, stream=None,
                               check=True):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    st = lib().rq_decode_attention_varlen(
        _shp(shape), _ptr(ctx_lens), _ptr(q), _ptr(ref_k), _ptr(ref_v), _ptr(codes_k),
        _ptr(codes_v), _ptr(scales_k), _ptr(scales_v), int(bits), ctypes.c_uint64(seed),
        float(softmax_scale), _ptr(tail_k), _ptr(tail_v), int(n_tail), int(tail_pitch), _ptr(out),
        _ptr(workspace), int(workspace_bytes), _stream(stream))
    if check:
        _check(st, "rq_decode_attention_varlen")
    return st


def rq_decode_attention_tail(shape, q, ref_k, ref_v, codes_k, codes_v, scales_k, scales_v,
                             bits, seed, softmax_scale, tail_k, tail_v, n_tail, tail_pitch, out,
                             workspace, workspace_bytes=None, stream=None, check=True):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    st = lib().rq_decode_attention_tail(
        _shp(shape), _ptr(q), _ptr(ref_k), _ptr(ref_v), _ptr(codes_k), _ptr(codes_v),
        _ptr(scales_k), _ptr(scales_v), int(bits), ctypes.c_uint64(seed), float(softmax_scale),
        _ptr(tail_k), _ptr(tail_v), int(n_tail), int(tail_pitch), _ptr(out), _ptr(workspace),
        int(workspace_bytes), _stream(stream))
    if check:
        _check(st, "rq_decode_attention_tail")
    return st


def rq_decode_attention(shape, q, ref_k, ref_v, codes_k, codes_v, scales_k, scales_v, bits,
                        seed, softmax_scale, out, workspace, workspace_bytes=None, stream=None,
                        check=True):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    st = lib().rq_decode_attention(_shp(shape), _ptr(q), _ptr(ref_k), _ptr(ref_v),
                                   _ptr(codes_k), _ptr(codes_v), _ptr(scales_k), _ptr(scales_v),
                                   int(bits), ctypes.c_uint64(seed), float(softmax_scale),
                                   _ptr(out), _ptr(workspace), int(workspace_bytes),
                                   _stream(stream))
    if check:
        _check(st, "rq_decode_attention")
    return st


def rq_decode_attention_noalloc(shape, q, ref_k, ref_v, codes_k, codes_v, scales_k, scales_v,
                                bits, seed, softmax_scale, out, stream=None, check=True):
    """rq_decode_attention with the library's fixed scratch instead of a
    caller workspace (for callers that cannot allocate)."""
    st = lib().rq_decode_attention_noalloc(_shp(shape), _ptr(q), _ptr(ref_k), _ptr(ref_v),
                                           _ptr(codes_k), _ptr(codes_v), _ptr(scales_k),
                                           _ptr(scales_v), int(bits), ctypes.c_uint64(seed),
                                           float(softmax_scale), _ptr(out), _stream(stream))
    if check:
        _check(st, "rq_decode_attention_noalloc")
    return st


def rq_reconstruct(shape, ref, codes, scales, bits, seed, out, out_bf16=False, stream=None,
                   check=True):
    st = lib().rq_reconstruct(_shp(shape), _ptr(ref), _ptr(codes), _ptr(scales), int(bits),
                              ctypes.c_uint64(seed), _ptr(out), 1 if out_bf16 else 0,
                              _stream(stream))
    if check:
        _check(st, "rq_reconstruct")
    return st


def rq_workspace_status(workspace, workspace_bytes=None, stream=None):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    v = ctypes.c_uint32(0)
    _check(lib().rq_workspace_status(_ptr(workspace), int(workspace_bytes), ctypes.byref(v),
                                     _stream(stream)), "rq_workspace_status")
    return v.value


def rq_encode_take_status():
    """Read and clear the encoders' sticky status word of the current device."""
    v = ctypes.c_uint32(0)
    _check(lib().rq_encode_take_status(ctypes.byref(v)), "rq_encode_take_status")
    return v.value


def rq_encode_cr_at(shape, dst_pitch, dst_offset, kv_loops, ref, ref_bits, bits_per_loop, seed,
                    ref_codes_out, ref_scales_out, codes_out, scales_out, stream=None,
                    check=True):
    n = len(bits_per_loop)
    ptrs = lambda seq: (ctypes.c_void_p * max(n, 1))(*[_ptr(v) for v in seq])
    bits = (ctypes.c_uint8 * max(n, 1))(*[int(b) for b in bits_per_loop])
    st = lib().rq_encode_cr_at(_shp(shape), int(dst_pitch), int(dst_offset), ptrs(kv_loops), n,
                               _ptr(ref), int(ref_bits), bits, ctypes.c_uint64(seed),
                               _ptr(ref_codes_out), _ptr(ref_scales_out), ptrs(codes_out),
                               ptrs(scales_out), _stream(stream))
    if check:
        _check(st, "rq_encode_cr_at")
    return st


def rq_reconstruct_cr(shape, ref_codes, ref_scales, ref_bits, codes, scales, bits, seed, out,
                      out_bf16=False, stream=None, check=True):
    st = lib().rq_reconstruct_cr(_shp(shape), _ptr(ref_codes), _ptr(ref_scales), int(ref_bits),
                                 _ptr(codes), _ptr(scales), int(bits), ctypes.c_uint64(seed),
                                 _ptr(out), 1 if out_bf16 else 0, _stream(stream))
    if check:
        _check(st, "rq_reconstruct_cr")
    return st


def rq_decode_attention_cr(shape, ctx_lens, q, ref_codes_k, ref_codes_v, ref_scales_k,
                           ref_scales_v, ref_bits, codes_k, codes_v, scales_k, scales_v, bits,
                           seed, softmax_scale, tail_k, tail_v, n_tail, tail_pitch, out,
                           workspace, workspace_bytes=None, stream=None, check=True):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    st = lib().rq_decode_attention_cr(
        _shp(shape), _ptr(ctx_lens), _ptr(q), _ptr(ref_codes_k), _ptr(ref_codes_v),
        _ptr(ref_scales_k), _ptr(ref_scales_v), int(ref_bits), _ptr(codes_k), _ptr(codes_v),
        _ptr(scales_k), _ptr(scales_v), int(bits), ctypes.c_uint64(seed), float(softmax_scale),
        _ptr(tail_k), _ptr(tail_v), int(n_tail), int(tail_pitch), _ptr(out), _ptr(workspace),
        int(workspace_bytes), _stream(stream))
    if check:
        _check(st, "rq_decode_attention_cr")
    return st


def rq_decode_attention_paged(shape, ctx_lens, page_table, max_pages, n_pages, q, ref_k, ref_v,
                              codes_k, codes_v, scales_k, scales_v, bits, seed, softmax_scale,
                              tail_k, tail_v, n_tail, tail_pitch, out, workspace,
                              workspace_bytes=None, stream=None, check=True):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    st = lib().rq_decode_attention_paged(
        _shp(shape), _ptr(ctx_lens), _ptr(page_table), int(max_pages), int(n_pages), _ptr(q),
        _ptr(ref_k), _ptr(ref_v), _ptr(codes_k), _ptr(codes_v), _ptr(scales_k), _ptr(scales_v),
        int(bits), ctypes.c_uint64(seed), float(softmax_scale), _ptr(tail_k), _ptr(tail_v),
        int(n_tail), int(tail_pitch), _ptr(out), _ptr(workspace), int(workspace_bytes),
        _stream(stream))
    if check:
        _check(st, "rq_decode_attention_paged")
    return st


def rq_encode_paged(shape, kv_loops, ref, bits_per_loop, seed, refine_iters, dst_pos, page_table,
                    max_pages, n_pages, codes_out, scales_out, ref_out=None, stream=None,
                    check=True):
    n = len(bits_per_loop)
    ptrs = lambda seq: (ctypes.c_void_p * max(n, 1))(*[_ptr(v) for v in seq])
    bits = (ctypes.c_uint8 * max(n, 1))(*[int(b) for b in bits_per_loop])
    st = lib().rq_encode_paged(_shp(shape), ptrs(kv_loops), n, _ptr(ref), bits,
                               ctypes.c_uint64(seed), int(refine_iters), _ptr(dst_pos),
                               _ptr(page_table), int(max_pages), int(n_pages), ptrs(codes_out),
                               ptrs(scales_out), _ptr(ref_out), _stream(stream))
    if check:
        _check(st, "rq_encode_paged")
    return st
