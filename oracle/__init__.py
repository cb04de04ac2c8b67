"""Python face of the CPU oracle (test infrastructure only).

Thin ctypes wrappers around liboracle.so (rq_oracle.c), taking and returning
numpy arrays.  Only the test-suite, the smoke check and the benchmark's
CPU-baseline leg import this package; the CUDA library never does.

bf16 and fp16 values travel as their raw uint16 bit patterns.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        u16p = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
        u32p = np.ctypeslib.ndpointer(np.uint32, flags="C_CONTIGUOUS")
        u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
        i8p = np.ctypeslib.ndpointer(np.int8, flags="C_CONTIGUOUS")
        f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
        f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
        c = ctypes
        L.orq_bf16_to_f32.argtypes = [c.c_uint16]
        L.orq_bf16_to_f32.restype = c.c_float
        L.orq_f16_to_f64.argtypes = [c.c_uint16]
        L.orq_f16_to_f64.restype = c.c_double
        L.orq_f64_to_f16.argtypes = [c.c_double]
        L.orq_f64_to_f16.restype = c.c_uint16
        L.orq_splitmix64.argtypes = [c.c_uint64, c.c_uint64]
        L.orq_splitmix64.restype = c.c_uint64
        L.orq_signs.argtypes = [c.c_uint64, c.c_int, i8p]
        L.orq_signs.restype = None
        L.orq_cd_f32.argtypes = [c.c_int]
        L.orq_cd_f32.restype = c.c_float
        L.orq_hadamard_entry.argtypes = [c.c_int, c.c_int]
        L.orq_hadamard_entry.restype = c.c_int
        L.orq_rotation_matrix_f64.argtypes = [c.c_int, i8p, f64p]
        L.orq_rotation_matrix_f64.restype = None
        L.orq_rotate_f32.argtypes = [c.c_int, i8p, f32p, f32p]
        L.orq_rotate_f32.restype = None
        L.orq_fwht_f64.argtypes = [c.c_int, f64p]
        L.orq_fwht_f64.restype = None
        L.orq_quantize_group_f32.argtypes = [c.c_int, c.c_int, f32p, u8p,
                                             c.POINTER(c.c_double), c.POINTER(c.c_uint16),
                                             c.POINTER(c.c_int)]
        L.orq_quantize_group_f32.restype = None
        L.orq_pack_codes.argtypes = [c.c_int, c.c_int, u8p, u32p]
        L.orq_pack_codes.restype = None
        L.orq_unpack_codes.argtypes = [c.c_int, c.c_int, u32p, u8p]
        L.orq_unpack_codes.restype = None
        L.orq_encode_rows_f32.argtypes = [c.c_long, c.c_int, c.c_int, c.c_int, c.c_uint64,
                                          u16p, u16p, u32p, u16p]
        L.orq_encode_rows_f32.restype = c.c_long
        L.orq_encode_row_f64.argtypes = [c.c_int, c.c_int, c.c_int, i8p, u16p, u16p,
                                         u8p, f64p, f64p]
        L.orq_encode_row_f64.restype = None
        L.orq_reconstruct_row_f64.argtypes = [c.c_int, c.c_int, c.c_int, i8p, u16p,
                                              u32p, u16p, f64p]
        L.orq_reconstruct_row_f64.restype = None
        L.orq_attention_f64.argtypes = [c.c_int, c.c_int, c.c_int, f64p, f64p, f64p,
                                        c.c_double, f64p]
        L.orq_attention_f64.restype = None
        L.orq_decode_attention_f64.argtypes = [c.c_int, c.c_int, c.c_int, c.c_int, c.c_int,
                                               c.c_uint64, c.c_double, u16p, u16p, u16p,
                                               c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p,
                                               f64p]
        L.orq_decode_attention_f64.restype = c.c_int
        i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
        L.orq_ls_dot_f32.argtypes = [c.c_int, f32p, i32p]
        L.orq_ls_dot_f32.restype = c.c_float
        L.orq_quantize_group_refined_f32.argtypes = [c.c_int, c.c_int, f32p, c.c_int, u8p,
                                                     c.POINTER(c.c_float),
                                                     c.POINTER(c.c_uint16)]
        L.orq_quantize_group_refined_f32.restype = None
        L.orq_encode_rows_refined_f32.argtypes = [c.c_long, c.c_int, c.c_int, c.c_int,
                                                  c.c_uint64, c.c_int, u16p, u16p, u32p, u16p]
        L.orq_encode_rows_refined_f32.restype = None
        L.orq_quantize_group_refined_f64.argtypes = [c.c_int, c.c_int, f64p, c.c_int, u8p,
                                                     c.POINTER(c.c_double), f64p]
        L.orq_quantize_group_refined_f64.restype = c.c_int
        L.orq_encode_rows_cr_f32.argtypes = [c.c_long, c.c_int, c.c_int, c.c_int, c.c_int,
                                             c.c_uint64, u16p, c.c_void_p, u32p, u16p,
                                             c.c_void_p, c.c_void_p]
        L.orq_encode_rows_cr_f32.restype = None
        L.orq_reconstruct_row_cr_f64.argtypes = [c.c_int, c.c_int, c.c_int, c.c_int, i8p, u32p,
                                                 u16p, c.c_void_p, c.c_void_p, f64p]
        L.orq_reconstruct_row_cr_f64.restype = None
        _lib = L
    return _lib


def _u16(a):
    return np.ascontiguousarray(a, dtype=np.uint16)


# ---- scalar formats ---------------------------------------------------------

def bf16_to_f32(bits):
    bits = _u16(bits)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def f16_to_f64(h):
    return lib().orq_f16_to_f64(int(h))


def f64_to_f16(x):
    return int(lib().orq_f64_to_f16(float(x)))


# ---- signs and rotation -----------------------------------------------------

def splitmix64(seed, i):
    return int(lib().orq_splitmix64(seed, i))


def signs(seed, d):
    D = np.empty(d, dtype=np.int8)
    lib().orq_signs(seed, d, D)
    return D


def cd_f32(d):
    return np.float32(lib().orq_cd_f32(d))


def hadamard_entry(i, j):
    return int(lib().orq_hadamard_entry(i, j))


def rotation_matrix_f64(d, seed):
    R = np.empty((d, d), dtype=np.float64)
    lib().orq_rotation_matrix_f64(d, signs(seed, d), R)
    return R


def rotate_f32(r, seed):
    r = np.ascontiguousarray(r, dtype=np.float32)
    d = r.shape[-1]
    y = np.empty_like(r)
    D = signs(seed, d)
    for idx in np.ndindex(r.shape[:-1]):
        out = np.empty(d, dtype=np.float32)
        lib().orq_rotate_f32(d, D, np.ascontiguousarray(r[idx]), out)
        y[idx] = out
    return y


def fwht_f64(v):
    v = np.array(v, dtype=np.float64, copy=True)
    lib().orq_fwht_f64(v.shape[0], v)
    return v


# ---- quantiser ----------------------------------------------------------------

def quantize_group_f32(y, bits):
    """Returns (codes uint8[g], s_exact float, s_f16 bits int, ties int)."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    c = np.empty(y.shape[0], dtype=np.uint8)
    s = ctypes.c_double()
    h = ctypes.c_uint16()
    t = ctypes.c_int(0)
    lib().orq_quantize_group_f32(y.shape[0], bits, y, c, ctypes.byref(s), ctypes.byref(h),
                                 ctypes.byref(t))
    return c, s.value, int(h.value), t.value


def pack_codes(codes, bits):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    d = codes.shape[-1]
    w = np.empty(codes.shape[:-1] + ((d * bits + 31) // 32,), dtype=np.uint32)
    for idx in np.ndindex(codes.shape[:-1]):
        out = np.empty((d * bits + 31) // 32, dtype=np.uint32)
        lib().orq_pack_codes(d, bits, np.ascontiguousarray(codes[idx]), out)
        w[idx] = out
    return w


def unpack_codes(words, bits, d):
    words = np.ascontiguousarray(words, dtype=np.uint32)
    c = np.empty(words.shape[:-1] + (d,), dtype=np.uint8)
    for idx in np.ndindex(words.shape[:-1]):
        out = np.empty(d, dtype=np.uint8)
        lib().orq_unpack_codes(d, bits, np.ascontiguousarray(words[idx]), out)
        c[idx] = out
    return c


# ---- encoder --------------------------------------------------------------------

def encode_rows_f32(x, ref, bits, group, seed):
    """fp32 exact-spec encode of rows [..., d] (bf16 bits).

    Returns (words uint32[..., d*bits/32], scales uint16[..., d/group], ties)."""
    x = _u16(x)
    ref = _u16(ref)
    assert x.shape == ref.shape
    d = x.shape[-1]
    n = int(np.prod(x.shape[:-1])) if x.ndim > 1 else 1
    words = np.empty(x.shape[:-1] + ((d * bits + 31) // 32,), dtype=np.uint32)
    scales = np.empty(x.shape[:-1] + (d // group,), dtype=np.uint16)
    ties = lib().orq_encode_rows_f32(n, d, group, bits, seed, x, ref, words, scales)
    return words, scales, int(ties)


def ls_dot_f32(y, lvl):
    """<y, l> in the refinement's fixed binary32 order."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    lvl = np.ascontiguousarray(lvl, dtype=np.int32)
    return float(lib().orq_ls_dot_f32(y.size, y, lvl))


def quantize_group_refined_f32(y, bits, iters):
    """Alternating refits of one group (fp32 spec).  Returns (codes, s_f32, s_f16)."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    codes = np.empty(y.size, dtype=np.uint8)
    sv = ctypes.c_float(0.0)
    h = ctypes.c_uint16(0)
    lib().orq_quantize_group_refined_f32(y.size, bits, y, iters, codes, ctypes.byref(sv),
                                         ctypes.byref(h))
    return codes, sv.value, h.value


def quantize_group_refined_f64(y, bits, iters):
    """The refits in double.  Returns (codes, s, err[0..done], done)."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    codes = np.empty(y.size, dtype=np.uint8)
    sv = ctypes.c_double(0.0)
    err = np.zeros(iters + 1, dtype=np.float64)
    done = lib().orq_quantize_group_refined_f64(y.size, bits, y, iters, codes,
                                                ctypes.byref(sv), err)
    return codes, sv.value, err[:done + 1], done


def encode_rows_refined_f32(x, ref, bits, group, seed, iters):
    """fp32 spec encode with `iters` least-squares refits per group.
    Returns (words, scales)."""
    x = _u16(x)
    ref = _u16(ref)
    assert x.shape == ref.shape
    d = x.shape[-1]
    n = int(np.prod(x.shape[:-1])) if x.ndim > 1 else 1
    words = np.empty(x.shape[:-1] + ((d * bits + 31) // 32,), dtype=np.uint32)
    scales = np.empty(x.shape[:-1] + (d // group,), dtype=np.uint16)
    lib().orq_encode_rows_refined_f32(n, d, group, bits, seed, iters, x, ref, words, scales)
    return words, scales


def encode_rows_cr_f32(x, ref, ref_bits, bits, group, seed):
    """Compressed-reference encode of rows [..., d] (bf16 bits); x None
    encodes only the reference.  Returns (ref_words, ref_scales, words,
    scales), the last two None without x."""
    ref = _u16(ref)
    d = ref.shape[-1]
    n = int(np.prod(ref.shape[:-1])) if ref.ndim > 1 else 1
    lead = ref.shape[:-1]
    rw = np.empty(lead + ((d * ref_bits + 31) // 32,), dtype=np.uint32)
    rs = np.empty(lead + (d // group,), dtype=np.uint16)
    w = s = None
    xp = wp = sp = None
    if x is not None:
        x = _u16(x)
        assert x.shape == ref.shape
        w = np.empty(lead + ((d * bits + 31) // 32,), dtype=np.uint32)
        s = np.empty(lead + (d // group,), dtype=np.uint16)
        xp, wp, sp = x.ctypes.data, w.ctypes.data, s.ctypes.data
    lib().orq_encode_rows_cr_f32(n, d, group, ref_bits, bits, seed, ref, xp, rw, rs, wp, sp)
    return rw, rs, w, s


def reconstruct_rows_cr_f64(ref_words, ref_scales, words, scales, ref_bits, bits, group, seed,
                            d):
    """fp64 rows of a compressed-reference loop (words None: the reference)."""
    rw = np.ascontiguousarray(ref_words, dtype=np.uint32).reshape(-1, (d * ref_bits + 31) // 32)
    rs = np.ascontiguousarray(ref_scales, dtype=np.uint16).reshape(-1, d // group)
    n = rw.shape[0]
    if words is not None:
        w = np.ascontiguousarray(words, dtype=np.uint32).reshape(n, -1)
        sc = np.ascontiguousarray(scales, dtype=np.uint16).reshape(n, -1)
    out = np.empty((n, d), dtype=np.float64)
    D = signs(seed, d)
    for i in range(n):
        row = out[i]
        lib().orq_reconstruct_row_cr_f64(
            d, group, ref_bits, bits, D, np.ascontiguousarray(rw[i]), np.ascontiguousarray(rs[i]),
            None if words is None else w[i].ctypes.data,
            None if words is None else sc[i].ctypes.data, row)
    return out


def encode_row_f64(x, ref, bits, group, seed):
    """fp64 definitional encode of one row.  Returns (codes, scales, bdist)."""
    x = _u16(x)
    ref = _u16(ref)
    d = x.shape[0]
    codes = np.empty(d, dtype=np.uint8)
    scales = np.empty(d // group, dtype=np.float64)
    bdist = np.empty(d, dtype=np.float64)
    lib().orq_encode_row_f64(d, group, bits, signs(seed, d), x, ref, codes, scales, bdist)
    return codes, scales, bdist


def reconstruct_rows_f64(ref, words, scales, bits, group, seed):
    ref = _u16(ref)
    d = ref.shape[-1]
    out = np.empty(ref.shape, dtype=np.float64)
    D = signs(seed, d)
    for idx in np.ndindex(ref.shape[:-1]):
        o = np.empty(d, dtype=np.float64)
        if bits == 16:
            w = np.zeros(1, dtype=np.uint32)
            s = np.zeros(1, dtype=np.uint16)
        else:
            w = np.ascontiguousarray(words[idx], dtype=np.uint32)
            s = np.ascontiguousarray(scales[idx], dtype=np.uint16)
        lib().orq_reconstruct_row_f64(d, group, bits, D, np.ascontiguousarray(ref[idx]), w, s, o)
        out[idx] = o
    return out


def attention_f64(q, K, V, scale):
    q = np.ascontiguousarray(q, dtype=np.float64)
    K = np.ascontiguousarray(K, dtype=np.float64)
    V = np.ascontiguousarray(V, dtype=np.float64)
    G, d = q.shape
    T = K.shape[0]
    out = np.empty((G, d), dtype=np.float64)
    lib().orq_attention_f64(T, d, G, q, K, V, float(scale), out)
    return out


def decode_attention_f64(q, ref_k, ref_v, codes_k, codes_v, scales_k, scales_v,
                         bits, group, seed, scale=0.0):
    """Decode attention of one (batch, kv-head): q [G, d] bf16 bits,
    ref_k/ref_v [T, d] bf16 bits, codes [T, d*bits/32], scales [T, d/group]."""
    q = _u16(q)
    ref_k = _u16(ref_k)
    ref_v = _u16(ref_v)
    G, d = q.shape
    T = ref_k.shape[0]
    out = np.empty((G, d), dtype=np.float64)
    keep = []

    def ptr(a, dt):
        if bits == 16 or a is None:
            return None
        a = np.ascontiguousarray(a, dtype=dt)
        keep.append(a)
        return a.ctypes.data

    rc = lib().orq_decode_attention_f64(
        T, d, group, G, bits, seed, float(scale), q, ref_k, ref_v,
        ptr(codes_k, np.uint32), ptr(codes_v, np.uint32),
        ptr(scales_k, np.uint16), ptr(scales_v, np.uint16), out)
    if rc != 0:
        raise ValueError(f"oracle decode attention rejected its arguments (rc={rc})")
    return out
