"""ctypes wrapper of the CPU oracle (test infrastructure only).

Only tests/, the smoke check and bench.py's CPU-baseline leg may import this
package.  The CUDA product path never does.  Arrays are numpy, host memory.
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

F16, BF16 = 0, 1
STOP_GROUP, STOP_TENSOR, STOP_NONE = 0, 1, 2

_lib = None


def lib(path: str = None):
    """Load (building first if needed) the oracle library."""
    global _lib
    if path is not None:
        return _bind(C.CDLL(path))
    if _lib is None:
        # HQQ_ORACLE_LIB points the pin tests at a deliberately broken copy
        # (the mutation test); otherwise the library is built from source.
        override = os.environ.get("HQQ_ORACLE_LIB")
        _lib = _bind(C.CDLL(override if override else _build.build()))
    return _lib


def _bind(L):
    P = C.c_void_p
    i64, i32, f32 = C.c_int64, C.c_int, C.c_float
    L.oracle_shrink.restype = f32
    L.oracle_shrink.argtypes = [f32, f32, f32]
    L.oracle_quantize.restype = i32
    L.oracle_quantize.argtypes = [P, i64, i64, i32, i32, i32, i32, f32, f32, f32, i32, i32, i32,
                                  P, P, P, P, P, P, P, i32]
    L.oracle_dequantize.restype = i32
    L.oracle_dequantize.argtypes = [P, P, P, P, i64, i64, i32, i32, i32, i32, i32, P]
    L.oracle_dequantize_s8.restype = i32
    L.oracle_dequantize_s8.argtypes = [P, P, P, i32, P, P, i64, i64, i32, i32, i32, i32, i32, P]
    L.oracle_gemv.restype = i32
    L.oracle_gemv.argtypes = [P, P, P, P, i64, i64, i32, i32, i32, P, i32, i32, P]
    L.oracle_gemm.restype = i32
    L.oracle_gemm.argtypes = [P, P, P, P, i64, i64, i32, i32, i32, P, i32, i32, P, P]
    L.oracle_quantize_scale8.restype = i32
    L.oracle_quantize_scale8.argtypes = [P, i64, i32, P, P]
    L.oracle_trace_group.restype = i32
    L.oracle_trace_group.argtypes = [P, i32, i32, f32, f32, f32, i32, P, P, P, P]
    L.oracle_pack_levels.restype = None
    L.oracle_pack_levels.argtypes = [P, i64, i64, i32, i32, P]
    L.oracle_unpack_levels.restype = None
    L.oracle_unpack_levels.argtypes = [P, i64, i64, i32, i32, P]
    L.oracle_group_codes.restype = None
    L.oracle_group_codes.argtypes = [P, i32, i32, f32, f32, P]
    L.oracle_update_zero.restype = f32
    L.oracle_update_zero.argtypes = [P, P, P, i32, f32, f32, f32]
    L.oracle_quantize_half.restype = i32
    L.oracle_quantize_half.argtypes = [P, i64, i64, i32, i32, i32, i32, f32, f32, f32, i32, i32, i32,
                                       P, P, P, P, P, P, P, i32]
    L.oracle_trace_group_half.restype = i32
    L.oracle_trace_group_half.argtypes = [P, i32, i32, f32, f32, f32, i32, P, P, P, P]
    L.oracle_group_codes_half.restype = None
    L.oracle_group_codes_half.argtypes = [P, i32, i32, f32, f32, P]
    L.oracle_quantize_groups.restype = i32
    L.oracle_quantize_groups.argtypes = [P, i64, i64, i32, i32, i32, i32, f32, f32, f32, i32, i32,
                                         P, i64, P, P, P, P, P, i32]
    return L


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _bits16(W):
    """Return (uint16 view, dtype code) of a float16 numpy array or bf16 bits."""
    if W.dtype == np.float16:
        return np.ascontiguousarray(W).view(np.uint16), F16
    raise TypeError("pass float16 arrays, or use quantize(..., dtype=BF16) with uint16 bf16 bits")


def num_groups(rows, cols, g):
    return rows * cols // g


def quantize(W, nbits, group_size, axis=1, p=0.7, beta=1.0, kappa=1.01, iters=20, stop_mode=STOP_GROUP,
             zero_nbits=16, dtype=None, nthreads=0, L=None):
    """Quantise W ([rows, cols] float16, or uint16 bf16 bits with dtype=BF16).

    Returns a dict with packed, scale (fp16 bits as float16), zero (float16 or
    uint8), zero_meta (fp32[2] or None), best_iter, best_err, zero_f32.
    """
    L = L or lib()
    if dtype is None:
        bits, dtype = _bits16(W)
    else:
        bits = np.ascontiguousarray(W).view(np.uint16)
    rows, cols = bits.shape
    G = num_groups(rows, cols, group_size)
    packed = np.zeros(rows * cols * nbits // 8, np.uint8)
    scale = np.zeros(G, np.float16)
    zero = np.zeros(G, np.float16 if zero_nbits == 16 else np.uint8)
    meta = np.zeros(2, np.float32) if zero_nbits == 8 else None
    bi = np.zeros(G, np.int32)
    be = np.zeros(G, np.float32)
    zf = np.zeros(G, np.float32)
    rc = L.oracle_quantize(_p(bits), rows, cols, dtype, nbits, group_size, axis, p, beta, kappa, iters, stop_mode,
                           zero_nbits, _p(packed), _p(scale), _p(zero), _p(meta), _p(bi), _p(be), _p(zf), nthreads)
    if rc != 0:
        raise ValueError(f"oracle_quantize failed with code {rc}")
    return dict(packed=packed, scale=scale, zero=zero, zero_meta=meta, best_iter=bi, best_err=be, zero_f32=zf)


def dequantize(packed, scale, zero, zero_meta, rows, cols, nbits, group_size, axis=1, zero_nbits=16,
               out_dtype=F16, L=None):
    """Returns float16 array (out_dtype F16) or uint16 bf16 bits (BF16)."""
    L = L or lib()
    out = np.zeros((rows, cols), np.uint16)
    rc = L.oracle_dequantize(_p(np.ascontiguousarray(packed)), _p(np.ascontiguousarray(scale)),
                             _p(np.ascontiguousarray(zero)), _p(zero_meta), rows, cols, nbits, group_size, axis,
                             zero_nbits, out_dtype, _p(out))
    if rc != 0:
        raise ValueError(f"oracle_dequantize failed with code {rc}")
    return out.view(np.float16) if out_dtype == F16 else out


def quantize_scale8(scale, scale_group=128, L=None):
    """8-bit quantisation of fp16 scales in runs of scale_group (reading R15).
    Returns (codes uint8[G], meta fp32[ceil(G/scale_group), 2] = (1/sc, zc))."""
    L = L or lib()
    scale = np.ascontiguousarray(scale, np.float16)
    G = scale.size
    codes = np.zeros(G, np.uint8)
    meta = np.zeros((max(1, -(-G // scale_group)), 2), np.float32)
    if L.oracle_quantize_scale8(_p(scale), G, scale_group, _p(codes), _p(meta)) != 0:
        raise ValueError("oracle_quantize_scale8 failed")
    return codes, meta


def dequantize_s8(packed, scale_q, scale_meta, scale_group, zero, zero_meta, rows, cols, nbits, group_size, axis=1,
                  zero_nbits=16, out_dtype=F16, L=None):
    """dequantize() with 8-bit scales (codes + per-run meta from quantize_scale8)."""
    L = L or lib()
    out = np.zeros((rows, cols), np.uint16)
    rc = L.oracle_dequantize_s8(_p(np.ascontiguousarray(packed)), _p(np.ascontiguousarray(scale_q)),
                                _p(np.ascontiguousarray(scale_meta, np.float32)), scale_group,
                                _p(np.ascontiguousarray(zero)), _p(zero_meta), rows, cols, nbits, group_size, axis,
                                zero_nbits, out_dtype, _p(out))
    if rc != 0:
        raise ValueError(f"oracle_dequantize_s8 failed with code {rc}")
    return out.view(np.float16) if out_dtype == F16 else out


def gemv(packed, scale, zero, zero_meta, rows, cols, nbits, group_size, zero_nbits, x, x_dtype=F16, L=None):
    """y[b] = W_r @ x[b] in fp64 with W_r = (W_q - zero) * scale in fp32 (axis 1).
    x: [batch, cols] float16 array (x_dtype F16) or uint16 bf16 bits (BF16)."""
    L = L or lib()
    x = np.ascontiguousarray(x)
    x2 = x.reshape(-1, cols)
    y = np.zeros((x2.shape[0], rows), np.float64)
    rc = L.oracle_gemv(_p(np.ascontiguousarray(packed)), _p(np.ascontiguousarray(scale)),
                       _p(np.ascontiguousarray(zero)), _p(zero_meta), rows, cols, nbits, group_size, zero_nbits,
                       _p(x2.view(np.uint16)), x_dtype, x2.shape[0], _p(y))
    if rc != 0:
        raise ValueError(f"oracle_gemv failed with code {rc}")
    return y


def gemm(packed, scale, zero, zero_meta, rows, cols, nbits, group_size, zero_nbits, x, x_dtype=F16, L=None):
    """(y, yabs): y[b] = round16(W_r) @ x[b] in fp64, W_r = (W_q - zero) * scale in
    fp32 rounded to x's 16-bit type (axis 1); yabs[b][r] = sum |w16 * x|.
    x: [batch, cols] float16 array (x_dtype F16) or uint16 bf16 bits (BF16)."""
    L = L or lib()
    x = np.ascontiguousarray(x)
    x2 = x.reshape(-1, cols)
    y = np.zeros((x2.shape[0], rows), np.float64)
    yabs = np.zeros((x2.shape[0], rows), np.float64)
    rc = L.oracle_gemm(_p(np.ascontiguousarray(packed)), _p(np.ascontiguousarray(scale)),
                       _p(np.ascontiguousarray(zero)), _p(zero_meta), rows, cols, nbits, group_size, zero_nbits,
                       _p(x2.view(np.uint16)), x_dtype, x2.shape[0], _p(y), _p(yabs))
    if rc != 0:
        raise ValueError(f"oracle_gemm failed with code {rc}")
    return y, yabs


def shrink(x, p, beta, L=None):
    L = L or lib()
    return L.oracle_shrink(float(x), float(p), float(beta))


def trace_group(w, nbits, p=0.7, beta=1.0, kappa=1.01, iters=20, L=None):
    """Run one fp32 group through `iters` iterations without early stop.

    Returns (s, z[iters], e[iters], beta[iters]).
    """
    L = L or lib()
    w = np.ascontiguousarray(w, np.float32)
    s = np.zeros(1, np.float32)
    z = np.zeros(iters, np.float32)
    e = np.zeros(iters, np.float64)
    b = np.zeros(iters, np.float32)
    rc = L.oracle_trace_group(_p(w), w.size, nbits, p, beta, kappa, iters, _p(s), _p(z), _p(e), _p(b))
    if rc != 0:
        raise ValueError("oracle_trace_group failed")
    return float(s[0]), z, e, b


def group_codes(w, nbits, s, z, L=None):
    L = L or lib()
    w = np.ascontiguousarray(w, np.float32)
    out = np.zeros(w.size, np.uint8)
    L.oracle_group_codes(_p(w), w.size, nbits, float(s), float(z), _p(out))
    return out


def update_zero(w, q, d, s, p, beta, L=None):
    L = L or lib()
    w, q, d = (np.ascontiguousarray(a, np.float32) for a in (w, q, d))
    return L.oracle_update_zero(_p(w), _p(q), _p(d), w.size, float(s), float(p), float(beta))


def pack_levels(levels, nbits, axis, L=None):
    L = L or lib()
    levels = np.ascontiguousarray(levels, np.uint8)
    rows, cols = levels.shape
    out = np.zeros(rows * cols * nbits // 8, np.uint8)
    L.oracle_pack_levels(_p(levels), rows, cols, nbits, axis, _p(out))
    return out


def unpack_levels(packed, rows, cols, nbits, axis, L=None):
    L = L or lib()
    out = np.zeros((rows, cols), np.uint8)
    L.oracle_unpack_levels(_p(np.ascontiguousarray(packed, np.uint8)), rows, cols, nbits, axis, _p(out))
    return out


def quantize_groups(W, group_ids, nbits, group_size, axis=1, p=0.7, beta=1.0, kappa=1.01, iters=20,
                    stop_mode=STOP_GROUP, dtype=None, nthreads=0, L=None):
    """Solve only the listed groups (group mode / no early stop)."""
    L = L or lib()
    if dtype is None:
        bits, dtype = _bits16(W)
    else:
        bits = np.ascontiguousarray(W).view(np.uint16)
    rows, cols = bits.shape
    ids = np.ascontiguousarray(group_ids, np.int64)
    n = ids.size
    levels = np.zeros(n * group_size, np.uint8)
    s = np.zeros(n, np.float32)
    zb = np.zeros(n, np.float32)
    bi = np.zeros(n, np.int32)
    be = np.zeros(n, np.float32)
    rc = L.oracle_quantize_groups(_p(bits), rows, cols, dtype, nbits, group_size, axis, p, beta, kappa, iters,
                                  stop_mode, _p(ids), n, _p(levels), _p(s), _p(zb), _p(bi), _p(be), nthreads)
    if rc != 0:
        raise ValueError("oracle_quantize_groups failed")
    return dict(levels=levels.reshape(n, group_size), s=s, zbest=zb, best_iter=bi, best_err=be)


# ---------------------------------------------- half-precision variant ----

def quantize_half(W, nbits, group_size, axis=1, p=0.7, beta=1.0, kappa=1.01, iters=20, stop_mode=STOP_GROUP,
                  zero_nbits=16, nthreads=0, L=None):
    """The half-precision solver variant (reading H) on a float16 array; the
    same output dict as quantize() (zero_f32 holds the fp16 zero-points)."""
    L = L or lib()
    bits, dtype = _bits16(W)
    rows, cols = bits.shape
    G = num_groups(rows, cols, group_size)
    packed = np.zeros(rows * cols * nbits // 8, np.uint8)
    scale = np.zeros(G, np.float16)
    zero = np.zeros(G, np.float16 if zero_nbits == 16 else np.uint8)
    meta = np.zeros(2, np.float32) if zero_nbits == 8 else None
    bi = np.zeros(G, np.int32)
    be = np.zeros(G, np.float32)
    zf = np.zeros(G, np.float32)
    rc = L.oracle_quantize_half(_p(bits), rows, cols, dtype, nbits, group_size, axis, p, beta, kappa, iters,
                                stop_mode, zero_nbits, _p(packed), _p(scale), _p(zero), _p(meta), _p(bi), _p(be),
                                _p(zf), nthreads)
    if rc != 0:
        raise ValueError(f"oracle_quantize_half failed with code {rc}")
    return dict(packed=packed, scale=scale, zero=zero, zero_meta=meta, best_iter=bi, best_err=be, zero_f32=zf)


def trace_group_half(w, nbits, p=0.7, beta=1.0, kappa=1.01, iters=20, L=None):
    """One fp16 group (values as float32) through `iters` iterations of the
    half-precision variant without early stop: (s, z[iters], e[iters], beta[iters])."""
    L = L or lib()
    w = np.ascontiguousarray(w, np.float32)
    s = np.zeros(1, np.float32)
    z = np.zeros(iters, np.float32)
    e = np.zeros(iters, np.float64)
    b = np.zeros(iters, np.float32)
    if L.oracle_trace_group_half(_p(w), w.size, nbits, p, beta, kappa, iters, _p(s), _p(z), _p(e), _p(b)) != 0:
        raise ValueError("oracle_trace_group_half failed")
    return float(s[0]), z, e, b


def group_codes_half(w, nbits, s, z, L=None):
    L = L or lib()
    w = np.ascontiguousarray(w, np.float32)
    out = np.zeros(w.size, np.uint8)
    L.oracle_group_codes_half(_p(w), w.size, nbits, float(s), float(z), _p(out))
    return out
