"""Thin ctypes binding of libhqq_b200.so (include/hqq.h), same names as the C ABI.

Argument marshalling only: every step of the quantiser runs in the library's
CUDA kernels.  torch provides device memory and streams.  If the library is
missing the import fails loudly; there is no CPU fallback.
"""
import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhqq_b200.so")

HQQ_OK, HQQ_ERR_INVALID_ARG, HQQ_ERR_SHAPE, HQQ_ERR_DTYPE, HQQ_ERR_ALIGN = 0, 1, 2, 3, 4
HQQ_ERR_CUDA, HQQ_ERR_TIMEOUT, HQQ_ERR_COOP_UNSUPPORTED, HQQ_ERR_WORKSPACE = 5, 6, 7, 8
HQQ_F16, HQQ_BF16 = 0, 1
HQQ_STOP_GROUP, HQQ_STOP_TENSOR, HQQ_STOP_NONE = 0, 1, 2

EXPORTED = ("hqq_packed_bytes", "hqq_num_groups", "hqq_workspace_bytes", "hqq_quantize", "hqq_dequantize",
            "hqq_get_status", "hqq_status_string", "hqq_quantize_noalloc", "hqq_quantize_scale8",
            "hqq_dequantize_s8", "hqq_stream_device_bytes", "hqq_quantize_stream", "hqq_gemv",
            "hqq_stream_jobs_device_bytes", "hqq_quantize_stream_jobs", "hqq_gemm", "hqq_gemm_get_status",
            "hqq_gemm_wait_selftest", "hqq_gemm_workspace_bytes", "hqq_quantize_half", "hqq_tensor_resident",
            "hqq_set_tensor_resident", "hqq_quantize_wait_selftest")


class hqq_host_matrix(C.Structure):
    """struct hqq_host_matrix of include/hqq.h (host pointers)."""
    _fields_ = [("W", C.c_void_p), ("rows", C.c_int64), ("cols", C.c_int64), ("W_q_packed", C.c_void_p),
                ("scale", C.c_void_p), ("zero", C.c_void_p), ("zero_meta", C.c_void_p)]


class hqq_stream_job(C.Structure):
    """struct hqq_stream_job of include/hqq.h: a host matrix and its settings."""
    _fields_ = [("m", hqq_host_matrix), ("nbits", C.c_int), ("group_size", C.c_int), ("axis", C.c_int),
                ("stop_mode", C.c_int), ("zero_nbits", C.c_int)]


hqq_stream_done_fn = C.CFUNCTYPE(None, C.c_int, C.c_void_p)
HQQ_NOALLOC_SCRATCH_BYTES = 16 << 20


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with calibration_free_weight_b200/build.py "
                          "(there is no CPU fallback)")
    L = C.CDLL(LIB_PATH)
    P, i64, i32, f32, sz = C.c_void_p, C.c_int64, C.c_int, C.c_float, C.c_size_t
    L.hqq_packed_bytes.restype = sz
    L.hqq_packed_bytes.argtypes = [i64, i64, i32, i32, i32]
    L.hqq_num_groups.restype = i64
    L.hqq_num_groups.argtypes = [i64, i64, i32, i32]
    L.hqq_workspace_bytes.restype = sz
    L.hqq_workspace_bytes.argtypes = [i64, i64, i32, i32, i32, i32]
    L.hqq_quantize.restype = i32
    L.hqq_quantize.argtypes = [P, i64, i64, i32, i32, i32, i32, f32, f32, f32, i32, i32, i32,
                               P, P, P, P, P, sz, P, P, P, P]
    L.hqq_quantize_half.restype = i32
    L.hqq_quantize_half.argtypes = L.hqq_quantize.argtypes
    L.hqq_dequantize.restype = i32
    L.hqq_dequantize.argtypes = [P, P, P, P, i64, i64, i32, i32, i32, i32, i32, P, P]
    L.hqq_get_status.restype = i32
    L.hqq_get_status.argtypes = [P, P]
    L.hqq_status_string.restype = C.c_char_p
    L.hqq_status_string.argtypes = [i32]
    L.hqq_quantize_scale8.restype = i32
    L.hqq_quantize_scale8.argtypes = [P, i64, i32, P, P, P]
    L.hqq_dequantize_s8.restype = i32
    L.hqq_dequantize_s8.argtypes = [P, P, P, i32, P, P, i64, i64, i32, i32, i32, i32, i32, P, P]
    L.hqq_gemv.restype = i32
    L.hqq_gemv.argtypes = [P, P, P, P, i64, i64, i32, i32, i32, P, i32, i32, P, P]
    L.hqq_gemm.restype = i32
    L.hqq_gemm.argtypes = [P, P, P, P, i64, i64, i32, i32, i32, P, i32, i32, P, P, sz, P]
    L.hqq_gemm_workspace_bytes.restype = sz
    L.hqq_gemm_workspace_bytes.argtypes = [i64, i64, i32]
    L.hqq_gemm_get_status.restype = i32
    L.hqq_gemm_get_status.argtypes = [P]
    L.hqq_gemm_wait_selftest.restype = i32
    L.hqq_gemm_wait_selftest.argtypes = [i64, P]
    L.hqq_tensor_resident.restype = i32
    L.hqq_tensor_resident.argtypes = [i64, i64, i32, i32, i32, i32]
    L.hqq_set_tensor_resident.restype = i32
    L.hqq_set_tensor_resident.argtypes = [i32]
    L.hqq_quantize_wait_selftest.restype = i32
    L.hqq_quantize_wait_selftest.argtypes = [P, sz, i64, P]
    HM = C.POINTER(hqq_host_matrix)
    L.hqq_stream_device_bytes.restype = sz
    L.hqq_stream_device_bytes.argtypes = [HM, i32, i32, i32, i32, i32, i32]
    L.hqq_quantize_stream.restype = i32
    L.hqq_quantize_stream.argtypes = [HM, i32, i32, i32, i32, i32, f32, f32, f32, i32, i32, i32, P, sz, P]
    SJ = C.POINTER(hqq_stream_job)
    L.hqq_stream_jobs_device_bytes.restype = sz
    L.hqq_stream_jobs_device_bytes.argtypes = [SJ, i32]
    L.hqq_quantize_stream_jobs.restype = i32
    L.hqq_quantize_stream_jobs.argtypes = [SJ, i32, i32, f32, f32, f32, i32, P, sz, hqq_stream_done_fn, P,
                                           C.POINTER(i32), P]
    L.hqq_quantize_noalloc.restype = i32
    L.hqq_quantize_noalloc.argtypes = [P, i64, i64, i32, i32, i32, i32, f32, f32, f32, i32, i32, i32,
                                       P, P, P, P, P, P, P, P]
    return L


lib = _load()


class HQQError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {hqq_status_string(code)} (code {code})")
        self.code = code


def _ptr(t):
    if t is None:
        return None
    return C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


# -------------------------------------------------------- C ABI, same names --

def hqq_packed_bytes(rows, cols, nbits, group_size, axis=1):
    return lib.hqq_packed_bytes(rows, cols, nbits, group_size, axis)


def hqq_num_groups(rows, cols, group_size, axis=1):
    return lib.hqq_num_groups(rows, cols, group_size, axis)


def hqq_workspace_bytes(rows, cols, group_size, axis=1, stop_mode=HQQ_STOP_GROUP, zero_nbits=16):
    return lib.hqq_workspace_bytes(rows, cols, group_size, axis, stop_mode, zero_nbits)


def hqq_quantize(W, rows, cols, dtype, nbits, group_size, axis, p, beta, kappa, iters, stop_mode, zero_nbits,
                 W_q_packed, scale, zero, zero_meta, workspace, workspace_bytes, debug_best_iter=None,
                 debug_best_err=None, debug_zero_f32=None, stream=None):
    """Raw call: tensors are passed by device address; returns the status code."""
    return lib.hqq_quantize(_ptr(W), rows, cols, dtype, nbits, group_size, axis, p, beta, kappa, iters, stop_mode,
                            zero_nbits, _ptr(W_q_packed), _ptr(scale), _ptr(zero), _ptr(zero_meta), _ptr(workspace),
                            workspace_bytes, _ptr(debug_best_iter), _ptr(debug_best_err), _ptr(debug_zero_f32),
                            _stream(stream))


def hqq_quantize_half(W, rows, cols, dtype, nbits, group_size, axis, p, beta, kappa, iters, stop_mode, zero_nbits,
                      W_q_packed, scale, zero, zero_meta, workspace, workspace_bytes, debug_best_iter=None,
                      debug_best_err=None, debug_zero_f32=None, stream=None):
    """Raw call of the half-precision solver variant; returns the status code."""
    return lib.hqq_quantize_half(_ptr(W), rows, cols, dtype, nbits, group_size, axis, p, beta, kappa, iters,
                                 stop_mode, zero_nbits, _ptr(W_q_packed), _ptr(scale), _ptr(zero), _ptr(zero_meta),
                                 _ptr(workspace), workspace_bytes, _ptr(debug_best_iter), _ptr(debug_best_err),
                                 _ptr(debug_zero_f32), _stream(stream))


def hqq_quantize_noalloc(W, rows, cols, dtype, nbits, group_size, axis, p, beta, kappa, iters, stop_mode,
                         zero_nbits, W_q_packed, scale, zero, zero_meta, debug_best_iter=None, debug_best_err=None,
                         debug_zero_f32=None, stream=None):
    """hqq_quantize without a workspace argument: the library's own static
    device scratch is used (for callers that cannot allocate)."""
    return lib.hqq_quantize_noalloc(_ptr(W), rows, cols, dtype, nbits, group_size, axis, p, beta, kappa, iters,
                                    stop_mode, zero_nbits, _ptr(W_q_packed), _ptr(scale), _ptr(zero), _ptr(zero_meta),
                                    _ptr(debug_best_iter), _ptr(debug_best_err), _ptr(debug_zero_f32),
                                    _stream(stream))


def hqq_dequantize(W_q_packed, scale, zero, zero_meta, rows, cols, nbits, group_size, axis, zero_nbits, out_dtype,
                   W_out, stream=None):
    return lib.hqq_dequantize(_ptr(W_q_packed), _ptr(scale), _ptr(zero), _ptr(zero_meta), rows, cols, nbits,
                              group_size, axis, zero_nbits, out_dtype, _ptr(W_out), _stream(stream))


def hqq_quantize_scale8(scale, num_groups, scale_group, scale_q, scale_meta, stream=None):
    return lib.hqq_quantize_scale8(_ptr(scale), num_groups, scale_group, _ptr(scale_q), _ptr(scale_meta),
                                   _stream(stream))


def hqq_dequantize_s8(W_q_packed, scale_q, scale_meta, scale_group, zero, zero_meta, rows, cols, nbits, group_size,
                      axis, zero_nbits, out_dtype, W_out, stream=None):
    return lib.hqq_dequantize_s8(_ptr(W_q_packed), _ptr(scale_q), _ptr(scale_meta), scale_group, _ptr(zero),
                                 _ptr(zero_meta), rows, cols, nbits, group_size, axis, zero_nbits, out_dtype,
                                 _ptr(W_out), _stream(stream))


def hqq_stream_device_bytes(mats, n, nbits, group_size, axis=1, stop_mode=HQQ_STOP_GROUP, zero_nbits=16):
    return lib.hqq_stream_device_bytes(mats, n, nbits, group_size, axis, stop_mode, zero_nbits)


def hqq_quantize_stream(mats, n, dtype, nbits, group_size, axis, p, beta, kappa, iters, stop_mode, zero_nbits,
                        device_buffer, device_bytes, stream=None):
    return lib.hqq_quantize_stream(mats, n, dtype, nbits, group_size, axis, p, beta, kappa, iters, stop_mode,
                                   zero_nbits, _ptr(device_buffer), device_bytes, _stream(stream))


def hqq_gemm(W_q_packed, scale, zero, zero_meta, rows, cols, nbits, group_size, zero_nbits, x, x_dtype, batch, y,
             workspace=None, workspace_bytes=0, stream=None):
    return lib.hqq_gemm(_ptr(W_q_packed), _ptr(scale), _ptr(zero), _ptr(zero_meta), rows, cols, nbits, group_size,
                        zero_nbits, _ptr(x), x_dtype, batch, _ptr(y), _ptr(workspace), workspace_bytes,
                        _stream(stream))


def hqq_gemm_workspace_bytes(rows, cols, batch):
    return lib.hqq_gemm_workspace_bytes(rows, cols, batch)


def hqq_gemm_get_status(stream=None):
    return lib.hqq_gemm_get_status(_stream(stream))


def hqq_gemm_wait_selftest(limit_us, stream=None):
    return lib.hqq_gemm_wait_selftest(limit_us, _stream(stream))


def hqq_tensor_resident(rows, cols, dtype, group_size, axis=1, iters=20):
    return lib.hqq_tensor_resident(rows, cols, dtype, group_size, axis, iters)


def hqq_set_tensor_resident(mode):
    return lib.hqq_set_tensor_resident(int(mode))


def hqq_quantize_wait_selftest(workspace, workspace_bytes, limit_us, stream=None):
    return lib.hqq_quantize_wait_selftest(_ptr(workspace), workspace_bytes, limit_us, _stream(stream))


def hqq_stream_jobs_device_bytes(jobs, n):
    return lib.hqq_stream_jobs_device_bytes(jobs, n)


def hqq_quantize_stream_jobs(jobs, n, dtype, p, beta, kappa, iters, device_buffer, device_bytes, on_done=None,
                             user=None, jobs_done=None, stream=None):
    cb = on_done if on_done is not None else hqq_stream_done_fn()
    return lib.hqq_quantize_stream_jobs(jobs, n, dtype, p, beta, kappa, iters, _ptr(device_buffer), device_bytes, cb,
                                        user, jobs_done, _stream(stream))


def hqq_gemv(W_q_packed, scale, zero, zero_meta, rows, cols, nbits, group_size, zero_nbits, x, x_dtype, batch, y,
             stream=None):
    return lib.hqq_gemv(_ptr(W_q_packed), _ptr(scale), _ptr(zero), _ptr(zero_meta), rows, cols, nbits, group_size,
                        zero_nbits, _ptr(x), x_dtype, batch, _ptr(y), _stream(stream))


def hqq_get_status(workspace, stream=None):
    return lib.hqq_get_status(_ptr(workspace), _stream(stream))


def hqq_status_string(code):
    return lib.hqq_status_string(code).decode()


# ------------------------------------------------------ allocating helpers --

_DT = {torch.float16: HQQ_F16, torch.bfloat16: HQQ_BF16}


def alloc_outputs(rows, cols, nbits, group_size, axis=1, stop_mode=HQQ_STOP_GROUP, zero_nbits=16, debug=False,
                  device="cuda"):
    """torch-allocated output and workspace buffers for one hqq_quantize call."""
    G = hqq_num_groups(rows, cols, group_size, axis)
    if G < 0:
        raise HQQError(HQQ_ERR_SHAPE, "hqq_num_groups")
    nb = hqq_packed_bytes(rows, cols, nbits, group_size, axis)
    wsb = hqq_workspace_bytes(rows, cols, group_size, axis, stop_mode, zero_nbits)
    u8 = torch.uint8
    out = dict(
        packed=torch.empty(max(nb, 16), dtype=u8, device=device)[:nb],
        scale=torch.empty(G, dtype=torch.float16, device=device),
        zero=torch.empty(G, dtype=torch.float16 if zero_nbits == 16 else u8, device=device),
        zero_meta=torch.empty(2, dtype=torch.float32, device=device) if zero_nbits == 8 else None,
        workspace=torch.empty(wsb, dtype=u8, device=device),
    )
    if debug:
        out.update(best_iter=torch.empty(G, dtype=torch.int32, device=device),
                   best_err=torch.empty(G, dtype=torch.float32, device=device),
                   zero_f32=torch.empty(G, dtype=torch.float32, device=device))
    return out


def quantize(W, nbits=4, group_size=64, axis=1, p=0.7, beta=1.0, kappa=1.01, iters=20, stop_mode=HQQ_STOP_GROUP,
             zero_nbits=16, debug=False, out=None, stream=None):
    """Quantise a CUDA fp16/bf16 [rows, cols] tensor; returns the output dict."""
    if W.dtype not in _DT or not W.is_cuda or W.dim() != 2 or not W.is_contiguous():
        raise HQQError(HQQ_ERR_INVALID_ARG, "quantize expects a contiguous 2-D CUDA fp16/bf16 tensor")
    rows, cols = W.shape
    if out is None:
        out = alloc_outputs(rows, cols, nbits, group_size, axis, stop_mode, zero_nbits, debug, W.device)
    rc = hqq_quantize(W, rows, cols, _DT[W.dtype], nbits, group_size, axis, p, beta, kappa, iters, stop_mode,
                      zero_nbits, out["packed"], out["scale"], out["zero"], out["zero_meta"], out["workspace"],
                      out["workspace"].numel(), out.get("best_iter"), out.get("best_err"), out.get("zero_f32"),
                      stream)
    if rc != HQQ_OK:
        raise HQQError(rc, "hqq_quantize")
    return out


def quantize_half(W, nbits=4, group_size=64, p=0.7, beta=1.0, kappa=1.01, iters=20, stop_mode=HQQ_STOP_GROUP,
                  zero_nbits=16, debug=False, out=None, stream=None):
    """The half-precision solver variant on a CUDA fp16 [rows, cols] tensor
    (axis 1, group or no stop); returns the output dict."""
    if W.dtype != torch.float16 or not W.is_cuda or W.dim() != 2 or not W.is_contiguous():
        raise HQQError(HQQ_ERR_INVALID_ARG, "quantize_half expects a contiguous 2-D CUDA fp16 tensor")
    rows, cols = W.shape
    if out is None:
        out = alloc_outputs(rows, cols, nbits, group_size, 1, stop_mode, zero_nbits, debug, W.device)
    rc = hqq_quantize_half(W, rows, cols, HQQ_F16, nbits, group_size, 1, p, beta, kappa, iters, stop_mode,
                           zero_nbits, out["packed"], out["scale"], out["zero"], out["zero_meta"], out["workspace"],
                           out["workspace"].numel(), out.get("best_iter"), out.get("best_err"), out.get("zero_f32"),
                           stream)
    if rc != HQQ_OK:
        raise HQQError(rc, "hqq_quantize_half")
    return out


def host_outputs(rows, cols, nbits, group_size, axis=1, zero_nbits=16, pin=True):
    """Pinned host output buffers for one matrix of quantize_stream()."""
    G = hqq_num_groups(rows, cols, group_size, axis)
    nb = hqq_packed_bytes(rows, cols, nbits, group_size, axis)
    mk = (lambda t: t.pin_memory()) if pin else (lambda t: t)
    return dict(packed=mk(torch.empty(nb, dtype=torch.uint8)), scale=mk(torch.empty(G, dtype=torch.float16)),
                zero=mk(torch.empty(G, dtype=torch.float16 if zero_nbits == 16 else torch.uint8)),
                zero_meta=mk(torch.empty(2, dtype=torch.float32)) if zero_nbits == 8 else None)


def quantize_stream(Ws, outs, nbits=4, group_size=64, axis=1, p=0.7, beta=1.0, kappa=1.01, iters=20,
                    stop_mode=HQQ_STOP_GROUP, zero_nbits=16, device_buffer=None, stream=None):
    """Quantise host fp16/bf16 matrices (pinned for overlap) into host output
    dicts (host_outputs()), streaming them through the GPU.  Returns the
    device buffer used (reusable for another call with the same sizes)."""
    if not Ws or len(Ws) != len(outs):
        raise HQQError(HQQ_ERR_INVALID_ARG, "quantize_stream needs one output dict per matrix")
    dt = Ws[0].dtype
    if dt not in _DT or any(w.dtype != dt or w.is_cuda or w.dim() != 2 or not w.is_contiguous() for w in Ws):
        raise HQQError(HQQ_ERR_INVALID_ARG, "quantize_stream expects contiguous 2-D host tensors of one dtype")
    arr = (hqq_host_matrix * len(Ws))()
    for a, w, o in zip(arr, Ws, outs):
        a.W, a.rows, a.cols = w.data_ptr(), w.shape[0], w.shape[1]
        a.W_q_packed, a.scale, a.zero = o["packed"].data_ptr(), o["scale"].data_ptr(), o["zero"].data_ptr()
        a.zero_meta = o["zero_meta"].data_ptr() if o.get("zero_meta") is not None else None
    need = hqq_stream_device_bytes(arr, len(Ws), nbits, group_size, axis, stop_mode, zero_nbits)
    if need == 0:
        raise HQQError(HQQ_ERR_INVALID_ARG, "hqq_stream_device_bytes")
    if device_buffer is None or device_buffer.numel() < need:
        device_buffer = torch.empty(need, dtype=torch.uint8, device="cuda")
    rc = hqq_quantize_stream(arr, len(Ws), _DT[dt], nbits, group_size, axis, p, beta, kappa, iters, stop_mode,
                             zero_nbits, device_buffer, device_buffer.numel(), stream)
    if rc != HQQ_OK:
        raise HQQError(rc, "hqq_quantize_stream")
    return device_buffer


def gemm(q, x, rows, cols, nbits, group_size, zero_nbits=16, out=None, workspace=None, split=True, stream=None):
    """y = round16(dequant(W)) @ x.T on the tensor cores for the outputs of
    quantize() (axis 1, cols a multiple of 64) and a CUDA [batch, cols]
    fp16/bf16 tensor x; returns fp32 [batch, rows].  With split (default) a
    workspace is allocated when the shape is split along K (or the one given
    is used)."""
    if x.dtype not in _DT or not x.is_cuda or x.dim() != 2 or not x.is_contiguous():
        raise HQQError(HQQ_ERR_INVALID_ARG, "gemm expects a contiguous 2-D CUDA fp16/bf16 x")
    if out is None:
        out = torch.empty(x.shape[0], rows, dtype=torch.float32, device=x.device)
    need = hqq_gemm_workspace_bytes(rows, cols, x.shape[0]) if split else 0
    if need and (workspace is None or workspace.numel() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    if not need:
        workspace = None
    rc = hqq_gemm(q["packed"], q["scale"], q["zero"], q.get("zero_meta"), rows, cols, nbits, group_size, zero_nbits,
                  x, _DT[x.dtype], x.shape[0], out, workspace, workspace.numel() if workspace is not None else 0,
                  stream)
    if rc != HQQ_OK:
        raise HQQError(rc, "hqq_gemm")
    return out


SETTING_KEYS = ("nbits", "group_size", "axis", "stop_mode", "zero_nbits")


def settings_for(name, base, dynamic=None):
    """Settings of the matrix `name` (e.g. "layers.3.self_attn.q_proj"): `base`
    (a dict of SETTING_KEYS) overridden by the first entry of `dynamic` whose
    key occurs in the name, as in a per-layer-type config
    {"attn": {"nbits": 4, "group_size": 64}, "mlp": {"nbits": 2, "group_size": 32}}."""
    out = {k: base[k] for k in SETTING_KEYS if k in base}
    for key, over in (dynamic or {}).items():
        if key in name:
            unknown = set(over) - set(SETTING_KEYS)
            if unknown:
                raise HQQError(HQQ_ERR_INVALID_ARG, f"unknown settings {sorted(unknown)} for {key!r}")
            out.update(over)
            break
    defaults = dict(axis=1, stop_mode=HQQ_STOP_GROUP, zero_nbits=16)
    return {k: out.get(k, defaults.get(k)) for k in SETTING_KEYS}


def quantize_stream_jobs(Ws, settings, outs, p=0.7, beta=1.0, kappa=1.01, iters=20, on_done=None,
                         device_buffer=None, stream=None):
    """quantize_stream with settings per matrix: settings[i] is a dict of
    SETTING_KEYS (see settings_for), outs[i] from host_outputs() with the same
    settings.  on_done(i) runs on this thread as soon as matrix i's outputs are
    in host memory, in order (persist them there to make a run resumable: pass
    only the matrices not yet persisted next time).  Returns (device buffer,
    number of leading matrices completed)."""
    n = len(Ws)
    if n == 0 or len(settings) != n or len(outs) != n:
        raise HQQError(HQQ_ERR_INVALID_ARG, "quantize_stream_jobs needs one settings dict and one output dict "
                       "per matrix")
    dt = Ws[0].dtype
    if dt not in _DT or any(w.dtype != dt or w.is_cuda or w.dim() != 2 or not w.is_contiguous() for w in Ws):
        raise HQQError(HQQ_ERR_INVALID_ARG, "quantize_stream_jobs expects contiguous 2-D host tensors of one dtype")
    arr = (hqq_stream_job * n)()
    for a, w, st, o in zip(arr, Ws, settings, outs):
        a.m.W, a.m.rows, a.m.cols = w.data_ptr(), w.shape[0], w.shape[1]
        a.m.W_q_packed, a.m.scale, a.m.zero = o["packed"].data_ptr(), o["scale"].data_ptr(), o["zero"].data_ptr()
        a.m.zero_meta = o["zero_meta"].data_ptr() if o.get("zero_meta") is not None else None
        for k in SETTING_KEYS:
            setattr(a, k, int(st[k]))
    need = hqq_stream_jobs_device_bytes(arr, n)
    if need == 0:
        raise HQQError(HQQ_ERR_INVALID_ARG, "hqq_stream_jobs_device_bytes")
    if device_buffer is None or device_buffer.numel() < need:
        device_buffer = torch.empty(need, dtype=torch.uint8, device="cuda")
    errors = []

    def report(i, _user):
        try:
            if on_done is not None:
                on_done(i)
        except BaseException as e:  # a ctypes callback cannot raise into C: keep it for after the call
            errors.append(e)

    cb = hqq_stream_done_fn(report)
    done = C.c_int(0)
    rc = hqq_quantize_stream_jobs(arr, n, _DT[dt], p, beta, kappa, iters, device_buffer, device_buffer.numel(), cb,
                                  None, C.byref(done), stream)
    if errors:
        raise errors[0]
    if rc != HQQ_OK:
        raise HQQError(rc, f"hqq_quantize_stream_jobs ({done.value} of {n} matrices completed)")
    return device_buffer, done.value


def gemv(q, x, rows, cols, nbits, group_size, zero_nbits=16, out=None, stream=None):
    """y = dequant(W) @ x.T for the outputs of quantize() (axis 1) and a CUDA
    [batch, cols] fp16/bf16 tensor x (batch <= 8); returns fp32 [batch, rows]."""
    if x.dtype not in _DT or not x.is_cuda or x.dim() != 2 or not x.is_contiguous():
        raise HQQError(HQQ_ERR_INVALID_ARG, "gemv expects a contiguous 2-D CUDA fp16/bf16 x")
    if out is None:
        out = torch.empty(x.shape[0], rows, dtype=torch.float32, device=x.device)
    rc = hqq_gemv(q["packed"], q["scale"], q["zero"], q.get("zero_meta"), rows, cols, nbits, group_size, zero_nbits,
                  x, _DT[x.dtype], x.shape[0], out, stream)
    if rc != HQQ_OK:
        raise HQQError(rc, "hqq_gemv")
    return out


def quantize_scale8(q, scale_group=128, stream=None):
    """8-bit scales (the "_s*" variant) for the outputs of quantize(): adds
    q["scale_q"] (uint8[G]) and q["scale_meta"] (fp32[ceil(G/S), 2])."""
    G = q["scale"].numel()
    dev = q["scale"].device
    q["scale_q"] = torch.empty(G, dtype=torch.uint8, device=dev)
    q["scale_meta"] = torch.empty(max(1, -(-G // scale_group)), 2, dtype=torch.float32, device=dev)
    q["scale_group"] = scale_group
    rc = hqq_quantize_scale8(q["scale"], G, scale_group, q["scale_q"], q["scale_meta"], stream)
    if rc != HQQ_OK:
        raise HQQError(rc, "hqq_quantize_scale8")
    return q


def dequantize_s8(q, rows, cols, nbits, group_size, axis=1, zero_nbits=16, out_dtype=torch.float16, out=None,
                  stream=None):
    """dequantize() with the 8-bit scales of quantize_scale8()."""
    if out is None:
        out = torch.empty(rows, cols, dtype=out_dtype, device=q["scale"].device)
    rc = hqq_dequantize_s8(q["packed"], q["scale_q"], q["scale_meta"], q["scale_group"], q["zero"], q["zero_meta"],
                           rows, cols, nbits, group_size, axis, zero_nbits, _DT[out_dtype], out, stream)
    if rc != HQQ_OK:
        raise HQQError(rc, "hqq_dequantize_s8")
    return out


def dequantize(q, rows, cols, nbits, group_size, axis=1, zero_nbits=16, out_dtype=torch.float16, out=None,
               stream=None):
    """Dequantise the outputs of quantize() into a [rows, cols] tensor."""
    if out is None:
        out = torch.empty(rows, cols, dtype=out_dtype, device=q["scale"].device)
    rc = hqq_dequantize(q["packed"], q["scale"], q["zero"], q["zero_meta"], rows, cols, nbits, group_size, axis,
                        zero_nbits, _DT[out_dtype], out, stream)
    if rc != HQQ_OK:
        raise HQQError(rc, "hqq_dequantize")
    return out
