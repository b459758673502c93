"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
function include/hqq.h declares, answers the size queries, and rejects bad
arguments on the host before anything is launched."""
import ctypes as C
import os
import re
import subprocess

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def hq():
    from calibration_free_weight_b200 import build
    build.build()
    from calibration_free_weight_b200 import hqq
    return hqq


def _declared():
    src = open(os.path.join(ROOT, "include", "hqq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hqq_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported(hq):
    names = _declared()
    assert "hqq_quantize" in names and "hqq_dequantize" in names
    for n in names:
        assert hasattr(hq.lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", hq.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (hqq_\w+)", out))
    assert set(names) <= exported
    assert set(hq.EXPORTED) == set(names)


@pytest.mark.parametrize("rows,cols,nbits,g,axis", [(4096, 4096, 4, 64, 1), (11008, 4096, 3, 64, 1),
                                                    (128, 48, 2, 16, 0), (8, 24, 1, 8, 1), (0, 64, 4, 64, 1)])
def test_size_queries(hq, rows, cols, nbits, g, axis):
    assert hq.hqq_packed_bytes(rows, cols, nbits, g, axis) == rows * cols * nbits // 8
    assert hq.hqq_num_groups(rows, cols, g, axis) == rows * cols // g
    for stop in (0, 1, 2):
        for zb in (8, 16):
            ws = hq.hqq_workspace_bytes(rows, cols, g, axis, stop, zb)
            G = rows * cols // g
            assert ws >= 256
            if zb == 8:
                assert ws >= 4 * G
            if stop == 1:
                assert ws >= 28 * G


@pytest.mark.parametrize("args", [(64, 100, 4, 64, 1), (100, 64, 4, 64, 0), (64, 64, 4, 48, 1), (64, 64, 4, 4, 1),
                                  (64, 64, 4, 2048, 1), (-1, 64, 4, 64, 1), (64, 64, 4, 64, 2)])
def test_size_queries_reject_bad_shapes(hq, args):
    rows, cols, nbits, g, axis = args
    assert hq.hqq_packed_bytes(rows, cols, nbits, g, axis) == 0
    assert hq.hqq_num_groups(rows, cols, g, axis) == -1


def test_bad_nbits_rejected(hq):
    for b in (0, 5, 6, 7, 9, 16):
        assert hq.hqq_packed_bytes(64, 64, b, 64, 1) == 0


def _call(hq, **kw):
    a = dict(W=None, rows=64, cols=64, dtype=0, nbits=4, g=64, axis=1, p=0.7, beta=1.0, kappa=1.01, iters=20,
             stop=0, zb=16, ws_bytes=0)
    a.update(kw)
    return hq.lib.hqq_quantize(None, a["rows"], a["cols"], a["dtype"], a["nbits"], a["g"], a["axis"], a["p"],
                               a["beta"], a["kappa"], a["iters"], a["stop"], a["zb"], None, None, None, None, None,
                               a["ws_bytes"], None, None, None, None)


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=2), 3), (dict(nbits=5), 1), (dict(g=48), 2), (dict(cols=96), 2), (dict(axis=0, rows=96), 2),
    (dict(axis=3), 1), (dict(p=0.0), 1), (dict(p=2.0), 1), (dict(p=float("nan")), 1), (dict(beta=0.0), 1),
    (dict(beta=float("inf")), 1), (dict(kappa=0.99), 1), (dict(iters=-1), 1), (dict(iters=1001), 1),
    (dict(stop=3), 1), (dict(zb=4), 1), (dict(), 8),
])
def test_quantize_rejects_on_host(hq, kw, code):
    assert _call(hq, **kw) == code


def test_dequantize_rejects_on_host(hq):
    L = hq.lib
    assert L.hqq_dequantize(None, None, None, None, 64, 64, 4, 64, 1, 16, 7, None, None) == 3
    assert L.hqq_dequantize(None, None, None, None, 64, 64, 5, 64, 1, 16, 0, None, None) == 1
    assert L.hqq_dequantize(None, None, None, None, 64, 96, 4, 64, 1, 16, 0, None, None) == 2
    assert L.hqq_dequantize(None, None, None, None, 64, 64, 4, 64, 1, 12, 0, None, None) == 1
    assert L.hqq_dequantize(None, None, None, None, 0, 64, 4, 64, 1, 16, 0, None, None) == 0


def test_scale8_entry_points_reject_on_host(hq):
    L = hq.lib
    # run length below 1, negative count: rejected before any pointer is looked at
    assert L.hqq_quantize_scale8(None, 10, 0, None, None, None) == hq.HQQ_ERR_INVALID_ARG
    assert L.hqq_quantize_scale8(None, -1, 128, None, None, None) == hq.HQQ_ERR_INVALID_ARG
    # nothing to do
    assert L.hqq_quantize_scale8(None, 0, 128, None, None, None) == hq.HQQ_OK
    # host (non-device) pointers
    buf = C.create_string_buffer(64)
    p = C.cast(buf, C.c_void_p).value
    assert L.hqq_quantize_scale8(p, 8, 128, p, p, None) == hq.HQQ_ERR_INVALID_ARG
    # dequantize with 8-bit scales: bad run length, bad dtype, bad shape, empty
    args = (None, None, None)
    assert L.hqq_dequantize_s8(*args, 0, None, None, 64, 64, 4, 64, 1, 16, 0, None, None) == hq.HQQ_ERR_INVALID_ARG
    assert L.hqq_dequantize_s8(*args, 128, None, None, 64, 64, 4, 64, 1, 16, 7, None, None) == hq.HQQ_ERR_DTYPE
    assert L.hqq_dequantize_s8(*args, 128, None, None, 64, 96, 4, 64, 1, 16, 0, None, None) == hq.HQQ_ERR_SHAPE
    assert L.hqq_dequantize_s8(*args, 128, None, None, 0, 64, 4, 64, 1, 16, 0, None, None) == hq.HQQ_OK


def test_stream_size_query_and_rejections(hq):
    L = hq.lib
    arr = (hq.hqq_host_matrix * 3)()
    for a, (r, c) in zip(arr, [(4096, 1024), (256, 2048), (1024, 512)]):
        a.rows, a.cols = r, c
    one = hq.hqq_stream_device_bytes(arr, 1, 4, 64)
    three = hq.hqq_stream_device_bytes(arr, 3, 4, 64)
    assert one > 2 * 4096 * 1024 * 2 and three == one  # two slots sized by the largest matrix
    arr[2].cols = 100  # not a multiple of the group size
    assert hq.hqq_stream_device_bytes(arr, 3, 4, 64) == 0
    assert hq.hqq_stream_device_bytes(arr, 0, 4, 64) == 0
    assert L.hqq_quantize_stream(None, 1, 0, 4, 64, 1, 0.7, 1.0, 1.01, 20, 0, 16, None, 0, None) == \
        hq.HQQ_ERR_INVALID_ARG
    assert L.hqq_quantize_stream(arr, 0, 0, 4, 64, 1, 0.7, 1.0, 1.01, 20, 0, 16, None, 0, None) == hq.HQQ_OK
    arr[2].cols = 512  # host buffers missing
    assert L.hqq_quantize_stream(arr, 3, 0, 4, 64, 1, 0.7, 1.0, 1.01, 20, 0, 16, None, 0, None) == \
        hq.HQQ_ERR_INVALID_ARG


def _jobs(hq, specs):
    arr = (hq.hqq_stream_job * len(specs))()
    for a, (r, c, nb, g, axis, stop, zb) in zip(arr, specs):
        a.m.rows, a.m.cols = r, c
        a.nbits, a.group_size, a.axis, a.stop_mode, a.zero_nbits = nb, g, axis, stop, zb
    return arr


def test_stream_jobs_size_query(hq):
    """Two slots, each buffer kind sized for the largest job (256-byte parts)."""
    specs = [(5120, 5120, 4, 64, 1, 1, 16), (13824, 5120, 2, 32, 1, 1, 16), (5120, 13824, 2, 32, 1, 1, 16),
             (1024, 8192, 8, 128, 0, 0, 8)]
    arr = _jobs(hq, specs)
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    mx = dict(W=0, packed=0, scale=0, zero=0, ws=0)
    for r, c, nb, g, axis, stop, zb in specs:
        G = hq.hqq_num_groups(r, c, g, axis)
        mx["W"] = max(mx["W"], 2 * r * c)
        mx["packed"] = max(mx["packed"], hq.hqq_packed_bytes(r, c, nb, g, axis))
        mx["scale"] = max(mx["scale"], 2 * G)
        mx["zero"] = max(mx["zero"], G * (2 if zb == 16 else 1))
        mx["ws"] = max(mx["ws"], hq.hqq_workspace_bytes(r, c, g, axis, stop, zb))
    slot = up(mx["W"]) + up(mx["packed"]) + up(mx["scale"]) + up(mx["zero"]) + up(8) + up(mx["ws"])
    assert hq.hqq_stream_jobs_device_bytes(arr, 4) == 2 * slot
    # the uniform-settings query is the same computation
    mats = (hq.hqq_host_matrix * 1)()
    mats[0].rows, mats[0].cols = 5120, 5120
    assert hq.hqq_stream_device_bytes(mats, 1, 4, 64, 1, 1, 16) == hq.hqq_stream_jobs_device_bytes(arr, 1)
    assert hq.hqq_stream_jobs_device_bytes(arr, 0) == 0
    assert hq.hqq_stream_jobs_device_bytes(None, 1) == 0


@pytest.mark.parametrize("bad,status", [((4096, 1024, 5, 64, 1, 0, 16), "HQQ_ERR_INVALID_ARG"),
                                        ((4096, 1000, 4, 64, 1, 0, 16), "HQQ_ERR_SHAPE"),
                                        ((4096, 1024, 4, 48, 1, 0, 16), "HQQ_ERR_SHAPE"),
                                        ((4096, 1024, 4, 64, 2, 0, 16), "HQQ_ERR_INVALID_ARG"),
                                        ((4096, 1024, 4, 64, 1, 3, 16), "HQQ_ERR_INVALID_ARG"),
                                        ((4096, 1024, 4, 64, 1, 0, 4), "HQQ_ERR_INVALID_ARG")])
def test_stream_jobs_rejects_a_bad_job_before_anything_runs(hq, bad, status):
    """One bad job anywhere in the list: its hqq_quantize status, no copy,
    no launch, no callback, zero jobs done (checked on a box with no GPU)."""
    good = (1024, 1024, 4, 64, 1, 0, 16)
    arr = _jobs(hq, [good, bad, good])
    assert hq.hqq_stream_jobs_device_bytes(arr, 3) == 0
    calls = []
    cb = hq.hqq_stream_done_fn(lambda i, u: calls.append(i))
    done = C.c_int(-1)
    rc = hq.lib.hqq_quantize_stream_jobs(arr, 3, 0, 0.7, 1.0, 1.01, 20, None, 0, cb, None, C.byref(done), None)
    assert rc == getattr(hq, status) and calls == [] and done.value == 0
    # the call's own solver parameters are checked the same way
    arr = _jobs(hq, [good])
    assert hq.lib.hqq_quantize_stream_jobs(arr, 1, 0, 2.5, 1.0, 1.01, 20, None, 0, cb, None, None, None) == \
        hq.HQQ_ERR_INVALID_ARG
    assert hq.lib.hqq_quantize_stream_jobs(arr, 1, 9, 0.7, 1.0, 1.01, 20, None, 0, cb, None, None, None) == \
        hq.HQQ_ERR_DTYPE
    # host buffers missing, then no device buffer
    assert hq.lib.hqq_quantize_stream_jobs(arr, 1, 0, 0.7, 1.0, 1.01, 20, None, 0, cb, None, None, None) == \
        hq.HQQ_ERR_INVALID_ARG
    assert hq.lib.hqq_quantize_stream_jobs(arr, 0, 0, 0.7, 1.0, 1.01, 20, None, 0, cb, None, None, None) == \
        hq.HQQ_OK


def test_settings_for_per_layer_types(hq):
    """A per-layer-type config: attention 4-bit g64, MLP 2-bit g32 tensor stop."""
    base = dict(nbits=4, group_size=64)
    dyn = {"attn": dict(nbits=4, group_size=64), "mlp": dict(nbits=2, group_size=32, stop_mode=1)}
    a = hq.settings_for("model.layers.7.self_attn.o_proj", base, dyn)
    m = hq.settings_for("model.layers.7.mlp.down_proj", base, dyn)
    o = hq.settings_for("lm_head", dict(base, zero_nbits=8), dyn)
    assert a == dict(nbits=4, group_size=64, axis=1, stop_mode=0, zero_nbits=16)
    assert m == dict(nbits=2, group_size=32, axis=1, stop_mode=1, zero_nbits=16)
    assert o == dict(nbits=4, group_size=64, axis=1, stop_mode=0, zero_nbits=8)
    with pytest.raises(hq.HQQError):
        hq.settings_for("x.mlp", base, {"mlp": dict(bits=2)})


def test_gemm_rejections(hq):
    """hqq_gemm argument checks, all on the host before any launch."""
    L = hq.lib
    a = (None, None, None, None)
    assert L.hqq_gemm(*a, 128, 128, 4, 64, 16, None, 7, 4, None, None, 0, None) == hq.HQQ_ERR_DTYPE
    assert L.hqq_gemm(*a, 128, 128, 5, 64, 16, None, 1, 4, None, None, 0, None) == hq.HQQ_ERR_INVALID_ARG
    assert L.hqq_gemm(*a, 128, 128, 4, 64, 16, None, 1, 0, None, None, 0, None) == hq.HQQ_ERR_INVALID_ARG
    assert L.hqq_gemm(*a, 128, 128, 4, 64, 16, None, 1, 65537, None, None, 0, None) == hq.HQQ_ERR_INVALID_ARG
    assert L.hqq_gemm(*a, 128, 96, 4, 32, 16, None, 1, 4, None, None, 0, None) == hq.HQQ_ERR_SHAPE  # cols % 64
    assert L.hqq_gemm(*a, 128, 128, 4, 48, 16, None, 1, 4, None, None, 0, None) == hq.HQQ_ERR_SHAPE
    assert L.hqq_gemm(*a, 128, 128, 4, 64, 12, None, 1, 4, None, None, 0, None) == hq.HQQ_ERR_INVALID_ARG
    assert L.hqq_gemm(*a, 0, 128, 4, 64, 16, None, 1, 4, None, None, 0, None) == hq.HQQ_OK
    buf = C.create_string_buffer(4096)
    p = C.cast(buf, C.c_void_p).value
    assert L.hqq_gemm(p, p, p, None, 128, 128, 4, 64, 16, p, 1, 4, p, None, 0, None) == hq.HQQ_ERR_INVALID_ARG


def test_gemm_workspace_query(hq):
    """Split products need tickets and partial tiles; the query is 0 for
    shapes whose tiles already fill the GPU and for invalid sizes."""
    assert hq.hqq_gemm_workspace_bytes(28672, 8192, 256) == 0  # 224 tiles
    w = hq.hqq_gemm_workspace_bytes(4096, 11008, 256)          # 32 tiles, 172 K tiles: split
    assert w > 0 and w >= 4096 * 256 * 4 * 2
    assert hq.hqq_gemm_workspace_bytes(4096, 4096, 256) == 0   # 64 K tiles: too short to split
    assert hq.hqq_gemm_workspace_bytes(4096, 4096, 16) > 0     # narrow batch tile: split
    assert hq.hqq_gemm_workspace_bytes(4096, 100, 16) == 0     # cols not a multiple of 64
    assert hq.hqq_gemm_workspace_bytes(4096, 4096, 0) == 0


def _gemm_ws_expected(rows, cols, batch, sms=148):
    """The split policy and workspace size of hqq_gemm, restated: batch tiles
    of at most 256 rows (equal, multiples of 16); a grid under 3/4 of the SMs
    splits K into sms // ctas parts, each at least 8 K tiles (40 for batch
    tiles >= 128); tickets (rounded to 256 bytes) then fp32 partial tiles."""
    nt = (batch + 255) // 256
    ntile = ((batch + nt - 1) // nt + 15) // 16 * 16
    ctas = ((rows + 127) // 128) * nt
    ktot = cols // 64
    sp = 1 if ctas >= sms * 3 // 4 else sms // ctas
    sp = min(sp, ktot // (40 if ntile >= 128 else 8))
    if sp <= 1:
        return 0
    kps = (ktot + sp - 1) // sp
    splits = (ktot + kps - 1) // kps
    tiles = ((rows + 127) // 128) * nt
    return (tiles * 4 + 255) // 256 * 256 + tiles * splits * ntile * 128 * 4


@pytest.mark.parametrize("rows,cols,batch", [(4096, 11008, 256), (4096, 4096, 16), (512, 4096, 16), (1000, 8192, 40),
                                             (4096, 4096, 256), (11008, 4096, 256), (256, 1024, 1), (128, 64, 1),
                                             (4096, 28672, 512), (8192, 8192, 300)])
def test_gemm_split_policy(hq, rows, cols, batch):
    """With no GPU the library assumes the B200's 148 SMs, so the policy is
    checked here against its restatement."""
    assert hq.hqq_gemm_workspace_bytes(rows, cols, batch) == _gemm_ws_expected(rows, cols, batch)


def test_gemm_wait_selftest_rejects_bad_limits(hq):
    assert hq.lib.hqq_gemm_wait_selftest(0, None) == hq.HQQ_ERR_INVALID_ARG
    assert hq.lib.hqq_gemm_wait_selftest(1000001, None) == hq.HQQ_ERR_INVALID_ARG


def test_status_strings(hq):
    for code in range(9):
        s = hq.hqq_status_string(code)
        assert s and s != "unknown status"
    assert hq.hqq_status_string(99) == "unknown status"


def test_binding_fails_loudly_without_library(tmp_path):
    """Importing the binding with the library missing raises; nothing falls back to the CPU."""
    import shutil
    import sys
    pkg = tmp_path / "calibration_free_weight_b200"
    shutil.copytree(os.path.join(ROOT, "calibration_free_weight_b200"), pkg,
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    code = "import calibration_free_weight_b200.hqq"
    r = subprocess.run([sys.executable, "-c", code], cwd=tmp_path, capture_output=True, text=True)
    assert r.returncode != 0 and "missing" in r.stderr


@pytest.mark.parametrize("axis", [1, 0])
def test_noalloc_zero8_limit_is_exact(hq, axis):
    """hqq_quantize_noalloc with an 8-bit zero.  Axis 1 needs only the kept
    zeros (4 bytes each) beside a 256-byte header: 4,194,240 groups fill the
    16 MiB scratch.  Axis 0 also needs one slice of 4,096 entries of running
    state: 4,149,184 groups fill it.  At the limit the size check passes;
    one group more is refused with HQQ_ERR_WORKSPACE before anything else
    happens.  The accepted call then fails on its missing buffers (or, with
    no GPU, on the device query), never on the size."""
    def call(rows, cols):
        return hq.lib.hqq_quantize_noalloc(None, rows, cols, hq.HQQ_F16, 2, 16, axis, 0.7, 1.0, 1.01, 20,
                                           hq.HQQ_STOP_GROUP, 8, None, None, None, None, None, None, None, None)
    if axis == 1:
        fit, over = (4_194_240, 16), (4_194_241, 16)
    else:
        fit, over = (1024, 64831), (80, 829837)
    assert fit[0] * fit[1] // 16 == (4_194_240 if axis == 1 else 4_149_184)
    assert over[0] * over[1] // 16 == fit[0] * fit[1] // 16 + 1
    assert call(*fit) not in (hq.HQQ_ERR_WORKSPACE, hq.HQQ_OK)
    assert call(*over) == hq.HQQ_ERR_WORKSPACE


def test_half_variant_rejects_on_host(hq):
    """hqq_quantize_half takes fp16 input, axis 1, group or no stop; the other
    cases are refused before anything is touched."""
    def call(dtype=0, axis=1, stop=0):
        return hq.lib.hqq_quantize_half(None, 64, 64, dtype, 4, 64, axis, 0.7, 1.0, 1.01, 20, stop, 16, None, None,
                                        None, None, None, 0, None, None, None, None)
    assert call(dtype=1) == 3
    assert call(axis=0) == 1
    assert call(stop=1) == 1
    assert call() == 8  # every argument valid: only the missing workspace is left


def test_tensor_resident_switch_and_query(hq):
    """The process-wide switch returns the previous setting; the query answers 0
    for invalid arguments and, without a device, for any problem; the wait
    self-test rejects bad limits and host memory before launching."""
    assert hq.lib.hqq_set_tensor_resident(0) == 1
    assert hq.lib.hqq_set_tensor_resident(2) == 0
    assert hq.lib.hqq_set_tensor_resident(3) == -1 and hq.lib.hqq_set_tensor_resident(-1) == -1
    assert hq.lib.hqq_set_tensor_resident(1) == 2
    assert hq.lib.hqq_set_tensor_resident(1) == 1
    assert hq.lib.hqq_tensor_resident(4096, 4096, 0, 48, 1, 20) == 0
    assert hq.lib.hqq_tensor_resident(4096, 4096, 5, 64, 1, 20) == 0
    assert hq.lib.hqq_tensor_resident(4096, 4096, 0, 64, 1, -1) == 0
    if not torch.cuda.is_available():
        assert hq.lib.hqq_tensor_resident(4096, 4096, 0, 64, 1, 20) == 0
    buf = (C.c_uint8 * 512)()
    assert hq.lib.hqq_quantize_wait_selftest(C.cast(buf, C.c_void_p), 512, 0, None) == hq.HQQ_ERR_INVALID_ARG
    assert hq.lib.hqq_quantize_wait_selftest(C.cast(buf, C.c_void_p), 512, 1000001, None) == hq.HQQ_ERR_INVALID_ARG
    assert hq.lib.hqq_quantize_wait_selftest(C.cast(buf, C.c_void_p), 512, 1000, None) == hq.HQQ_ERR_INVALID_ARG


def test_header_is_plain_c(tmp_path):
    """include/hqq.h is a C header: a C99 translation unit that includes it and
    names every declared entry point compiles with -pedantic -Werror."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    header = open(os.path.join(root, "include", "hqq.h")).read()
    names = sorted(set(re.findall(r"^(?:int|size_t|int64_t|const char\*)\s+(hqq_\w+)\(", header, re.M)))
    assert len(names) >= 20
    src = tmp_path / "use_header.c"
    src.write_text('#include "hqq.h"\nint hqq_header_declares = (int)(' + " + ".join(f"sizeof(&{n})" for n in names)
                   + ");\n")
    r = subprocess.run(["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
                        "-I", os.path.join(root, "include"), "-c", str(src), "-o", str(tmp_path / "u.o")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
