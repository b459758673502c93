"""hqq_quantize_noalloc: the quantiser for callers that cannot allocate device
memory (a plugin inside a host runtime that owns every allocation, or a loop
that must not pay for cudaMalloc and the synchronisation it can cause).

It takes no workspace and uses the library's own 16 MiB device scratch buffer.
The test calls it through the C ABI twice in a row -- on different matrices
and settings, so the second call runs on scratch the first call left behind --
and compares each result with hqq_quantize on a caller-allocated workspace,
within the parity tolerances the other GPU tests use.  It lives in a file of
its own, collected last, and passes alone in a fresh process too.
"""
import numpy as np
import pytest
import torch

from calibration_free_weight_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from calibration_free_weight_b200 import hqq
    return hqq


def _levels(packed, n, nbits):
    bits = np.unpackbits(packed, bitorder="little").reshape(n, nbits)
    return (bits * (1 << np.arange(nbits))).sum(1)


def _compare(ref, got, rows, cols, nbits, zero_nbits):
    r = {k: v.cpu().numpy() for k, v in ref.items() if isinstance(v, torch.Tensor) and k != "workspace"}
    g = {k: v.cpu().numpy() for k, v in got.items() if isinstance(v, torch.Tensor)}
    lr, lg = _levels(r["packed"], rows * cols, nbits), _levels(g["packed"], rows * cols, nbits)
    d = lr.astype(np.int64) - lg.astype(np.int64)
    assert np.all(np.abs(d) <= 1) and np.count_nonzero(d) <= 1e-4 * d.size + 1
    sr, sg = r["scale"].astype(np.float64), g["scale"].astype(np.float64)
    assert np.all(np.abs(sr - sg) <= 1e-3 * np.abs(sr))
    zr, zg = r["zero_f32"].astype(np.float64), g["zero_f32"].astype(np.float64)
    assert np.all(np.abs(zr - zg) <= 1e-3 * np.maximum(np.abs(zr), 1.0))
    if zero_nbits == 8:
        dz = r["zero"].astype(np.int64) - g["zero"].astype(np.int64)
        assert np.all(np.abs(dz) <= 1) and np.count_nonzero(dz) <= 1e-4 * dz.size + 1
        assert np.allclose(r["zero_meta"], g["zero_meta"], rtol=1e-5, atol=1e-6)
    else:
        z16r, z16g = r["zero"].astype(np.float64), g["zero"].astype(np.float64)
        assert np.all(np.abs(z16r - z16g) <= 1e-3 * np.maximum(np.abs(z16r), 1.0))
    assert np.array_equal(r["best_iter"], g["best_iter"])


def _noalloc(hq, W, nbits, g, stop, zero_nbits, axis=1):
    rows, cols = W.shape
    G = rows * cols // g
    dev = W.device
    out = dict(packed=torch.empty(rows * cols * nbits // 8, dtype=torch.uint8, device=dev),
               scale=torch.empty(G, dtype=torch.float16, device=dev),
               zero=torch.empty(G, dtype=torch.float16 if zero_nbits == 16 else torch.uint8, device=dev),
               zero_meta=torch.empty(2, dtype=torch.float32, device=dev) if zero_nbits == 8 else None,
               best_iter=torch.empty(G, dtype=torch.int32, device=dev),
               best_err=torch.empty(G, dtype=torch.float32, device=dev),
               zero_f32=torch.empty(G, dtype=torch.float32, device=dev))
    dt = hq.HQQ_F16 if W.dtype == torch.float16 else hq.HQQ_BF16
    rc = hq.hqq_quantize_noalloc(W, rows, cols, dt, nbits, g, axis, 0.7, 1.0, 1.01, 20, stop, zero_nbits,
                                 out["packed"], out["scale"], out["zero"], out["zero_meta"], out["best_iter"],
                                 out["best_err"], out["zero_f32"])
    assert rc == hq.HQQ_OK, hq.hqq_status_string(rc)
    return out


def test_noalloc_matches_workspace_entry_point_twice(hq):
    cases = [  # second call: other shape, dtype, group size and stop rule on the same scratch
        (synth.weight(4096, 4096, seed=0, dtype=torch.float16), 4, 64, hq.HQQ_STOP_GROUP, 8),
        (synth.weight(11008, 4096, seed=4, dtype=torch.bfloat16), 2, 16, hq.HQQ_STOP_NONE, 8),
        (synth.weight(11008, 4096, seed=5, dtype=torch.bfloat16), 4, 64, hq.HQQ_STOP_GROUP, 16),
    ]
    for W_cpu, nbits, g, stop, zb in cases:
        W = W_cpu.cuda()
        got = _noalloc(hq, W, nbits, g, stop, zb)
        ref = hq.quantize(W, nbits, g, stop_mode=stop, zero_nbits=zb, debug=True)
        torch.cuda.synchronize()
        _compare(ref, got, *W.shape, nbits, zb)


def _levels_axis0(packed, rows, cols, nbits):
    """Codes of an axis-0 stream ([rows*nbits/8, cols], one LSB-first stream per column) as [rows, cols]."""
    col = packed.reshape(rows * nbits // 8, cols).T  # [cols, rows*nbits/8]
    return np.stack([_levels(np.ascontiguousarray(c), rows, nbits) for c in col], axis=1)


def test_noalloc_axis0_runs_in_slices(hq):
    """Axis 0 keeps per-group running state; its full workspace (31 MB here)
    exceeds the scratch, so the call runs in slices of groups, one after
    another on the stream, and must equal the workspace entry point."""
    W = synth.weight(4096, 11008, seed=7, dtype=torch.bfloat16).cuda()
    assert hq.hqq_workspace_bytes(4096, 11008, 64, 0, 0, 16) > hq.HQQ_NOALLOC_SCRATCH_BYTES
    for _ in range(2):
        got = _noalloc(hq, W, 4, 64, hq.HQQ_STOP_GROUP, 16, axis=0)
        ref = hq.quantize(W, 4, 64, axis=0, stop_mode=hq.HQQ_STOP_GROUP, zero_nbits=16, debug=True)
        torch.cuda.synchronize()
        lr = _levels_axis0(ref["packed"].cpu().numpy(), 4096, 11008, 4)
        lg = _levels_axis0(got["packed"].cpu().numpy(), 4096, 11008, 4)
        d = lr.astype(np.int64) - lg.astype(np.int64)
        assert np.all(np.abs(d) <= 1) and np.count_nonzero(d) <= 1e-4 * d.size + 1
        assert np.array_equal(ref["best_iter"].cpu().numpy(), got["best_iter"].cpu().numpy())
        zr, zg = ref["zero_f32"].cpu().numpy(), got["zero_f32"].cpu().numpy()
        assert np.all(np.abs(zr - zg) <= 1e-3 * np.maximum(np.abs(zr), 1.0))


def test_noalloc_rejects_what_does_not_fit(hq):
    W = torch.empty(8192, 8192, dtype=torch.float16, device="cuda")  # 4,194,304 groups at g16: above 4,194,240
    G = W.numel() // 16
    assert hq.hqq_workspace_bytes(8192, 8192, 16, 1, 0, 8) > hq.HQQ_NOALLOC_SCRATCH_BYTES
    out = [torch.empty(W.numel() * 2 // 8, dtype=torch.uint8, device="cuda"),
           torch.empty(G, dtype=torch.float16, device="cuda"), torch.empty(G, dtype=torch.uint8, device="cuda"),
           torch.empty(2, dtype=torch.float32, device="cuda")]
    rc = hq.hqq_quantize_noalloc(W, 8192, 8192, hq.HQQ_F16, 2, 16, 1, 0.7, 1.0, 1.01, 20, 0, 8, *out)
    assert rc == hq.HQQ_ERR_WORKSPACE
    rc = hq.hqq_quantize_noalloc(W, 8192, 8192, hq.HQQ_F16, 2, 16, 1, 0.7, 1.0, 1.01, 20, hq.HQQ_STOP_TENSOR, 16,
                                 *out[:2], torch.empty(G, dtype=torch.float16, device="cuda"), None)
    assert rc == hq.HQQ_ERR_INVALID_ARG
