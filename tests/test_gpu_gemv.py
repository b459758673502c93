"""GPU parity of the fused dequantisation + matrix-vector product (hqq_gemv)
against the oracle's fp64 product of the dequantised weights.

Both sides run on the oracle's own quantisation outputs (uploaded to the GPU),
so no oracle input comes from the CUDA path.  The GPU computes in fp32, per
8-column piece s * (sum q x - z * sum x); the bound below is derived from that
order of operations: with u = 2^-24 and n the longest chain of roundings one
thread performs (at most cols / 1024 + 1 piece or chunk additions, an
in-chunk chain of up to 32 fused multiply-adds, and up to 8 reduction
levels), |y_gpu - y_ref| <= u * (n + 25) * sum_c s (|q| + |z|) |x|, where the
extra terms cover the oracle's own fp32 rounding of each W_r.
"""
import numpy as np
import pytest
import torch

import oracle
from calibration_free_weight_b200 import synth

pytestmark = pytest.mark.gpu
U = 2.0 ** -24


@pytest.fixture(scope="module")
def hq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from calibration_free_weight_b200 import hqq
    return hqq


def _magnitude(o, rows, cols, nbits, g, zb, X):
    lv = oracle.unpack_levels(o["packed"], rows, cols, nbits, 1).reshape(rows, cols).astype(np.float64)
    G = rows * cols // g
    s = o["scale"].astype(np.float64).reshape(rows, cols // g)
    if zb == 16:
        z = o["zero"].astype(np.float64)
    else:
        m = o["zero_meta"].astype(np.float32)
        z = ((o["zero"].astype(np.float32) - m[1]) * m[0]).astype(np.float64)
    z = z.reshape(rows, cols // g)
    sw = np.repeat(s, g, axis=1)
    aw = np.repeat(np.abs(z), g, axis=1)
    Xf = X.astype(np.float64) if X.dtype == np.float16 else (X.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return (sw * (np.abs(lv) + aw)) @ np.abs(Xf).T  # [rows, batch]


def _case(hq, rows, cols, nbits, g, zb, batch, xdt, seed):
    W = synth.weight(rows, cols, seed=seed, dtype=torch.float16)
    o = oracle.quantize(W.numpy(), nbits, g, 1, 0.7, 1.0, 1.01, 20, oracle.STOP_GROUP, zb)
    xs = synth.weight(batch, cols, seed=seed + 1, dtype=torch.float32) * 50.0
    X = xs.to(torch.float16 if xdt == oracle.F16 else torch.bfloat16)
    Xn = X.numpy() if xdt == oracle.F16 else X.view(torch.int16).numpy().view(np.uint16)
    ref = oracle.gemv(o["packed"], o["scale"], o["zero"], o["zero_meta"], rows, cols, nbits, g, zb, Xn, xdt)
    dev = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in o.items()
           if k in ("packed", "scale", "zero", "zero_meta") and v is not None}
    y = hq.gemv(dev, X.cuda(), rows, cols, nbits, g, zero_nbits=zb)
    torch.cuda.synchronize()
    got = y.cpu().numpy().astype(np.float64)
    n = cols // 1024 + 1 + 32 + 8
    bound = U * (n + 25) * _magnitude(o, rows, cols, nbits, g, zb, Xn).T
    err = np.abs(got - ref)
    assert np.all(err <= bound), f"max err/bound {np.max(err / np.maximum(bound, 1e-300))}"
    return float(np.max(err / np.maximum(bound, 1e-300)))


@pytest.mark.parametrize("nbits,g", [(1, 16), (2, 16), (3, 64), (4, 64), (8, 128), (4, 8), (2, 1024), (3, 16),
                                     (1, 32), (8, 16)])
@pytest.mark.parametrize("zb", [16, 8])
def test_gemv_settings(hq, nbits, g, zb):
    _case(hq, 99, 2048, nbits, g, zb, 1, oracle.F16, seed=nbits * 7 + g)


@pytest.mark.parametrize("batch", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("xdt", [oracle.F16, oracle.BF16])
def test_gemv_batches_and_dtypes(hq, batch, xdt):
    _case(hq, 130, 1024, 4, 64, 16, batch, xdt, seed=batch)


@pytest.mark.parametrize("rows,cols", [(1, 8 * 16), (3, 1024), (4096, 4096), (1024, 8192), (4096, 11008),
                                       (40000, 1024)])  # the last: 4 rows per warp
def test_gemv_shapes(hq, rows, cols):
    _case(hq, rows, cols, 4, 64 if cols % 64 == 0 else 16, 8, 1, oracle.F16, seed=rows + cols)


def test_gemv_rejects(hq):
    x = torch.zeros(9, 64, dtype=torch.float16, device="cuda")
    y = torch.zeros(9, 16, dtype=torch.float32, device="cuda")
    q = hq.quantize(torch.zeros(16, 64, dtype=torch.float16, device="cuda"), 4, 64)
    rc = hq.hqq_gemv(q["packed"], q["scale"], q["zero"], None, 16, 64, 4, 64, 16, x, hq.HQQ_F16, 9, y)
    assert rc == hq.HQQ_ERR_INVALID_ARG  # batch above 8
    rc = hq.hqq_gemv(q["packed"], q["scale"], q["zero"], None, 16, 64, 4, 64, 16, x, hq.HQQ_F16, 1, y)
    assert rc == hq.HQQ_OK
