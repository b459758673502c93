"""hqq_gemm (tcgen05 tensor cores) against the oracle's tensor-core product.

Inputs: seeded random codes packed by the oracle, seeded synthetic fp16
scales (the spread of 0.02-std weights' dequantisation multipliers) and
zeros, seeded activations; nothing comes from the CUDA path.  The oracle
rounds the fp32 W_r to the activations' type exactly as the kernel must and
sums in fp64; the kernel sums in fp32 in an unspecified order, so the bound
is the textbook one for n-term fp32 summation of exact products:
|y - y_exact| <= cols * 2^-23 * sum |w16 x| (a wrong element, index, swizzle
or scale gives errors of the order of |y| itself, far above it).
"""
import numpy as np
import pytest
import torch

import oracle
from calibration_free_weight_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from calibration_free_weight_b200 import hqq
    return hqq


def make_q(rows, cols, nbits, g, zb, seed):
    """Random codes, synthetic scales, zeros in [0, L] (fp16) or 8-bit with a meta pair."""
    r = np.random.default_rng(seed)
    L = (1 << nbits) - 1
    lv = r.integers(0, L + 1, (rows, cols)).astype(np.uint8)
    packed = np.zeros(rows * cols * nbits // 8, np.uint8)
    oracle.lib().oracle_pack_levels(lv.ctypes.data, rows, cols, nbits, 1, packed.ctypes.data)
    G = rows * cols // g
    scale = synth.scales(G, seed).numpy()
    if zb == 16:
        zero = (r.random(G) * L).astype(np.float16)
        meta = None
    else:
        zero = r.integers(0, 256, G).astype(np.uint8)
        meta = np.array([L / 255.0, 3.0], np.float32)  # (1/sz, zz)
    return dict(packed=packed, scale=scale, zero=zero, zero_meta=meta)


def make_x(batch, cols, dtype, seed):
    x = synth.weight(batch, cols, seed=seed, dtype=torch.float32, std=1.0).to(dtype)
    if dtype == torch.bfloat16:
        return x, x.view(torch.int16).numpy().view(np.uint16), oracle.BF16
    return x, x.numpy(), oracle.F16


def run(hq, q, x, rows, cols, nbits, g, zb):
    d = {k: (torch.from_numpy(v).cuda() if v is not None else None) for k, v in q.items()}
    y = hq.gemm(d, x.cuda(), rows, cols, nbits, g, zb)
    assert hq.hqq_gemm_get_status() == hq.HQQ_OK
    return y.cpu().numpy().astype(np.float64)


def check(y, yo, ya, cols):
    bound = cols * 2.0 ** -23 * ya + 1e-30
    err = np.abs(y - yo)
    assert np.all(err <= bound), f"max excess {np.max(err - bound)}, max err {err.max()}"
    return float(np.max(err / np.maximum(ya, 1e-30)))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("nbits,g,zb", [(4, 64, 16), (8, 128, 8), (3, 64, 16), (2, 16, 8), (1, 8, 16), (4, 32, 8)])
@pytest.mark.parametrize("rows,cols,batch", [(256, 512, 16), (200, 256, 7), (128, 64, 1), (384, 1024, 33)])
def test_gemm_matches_oracle(hq, dtype, nbits, g, zb, rows, cols, batch):
    if cols % g:
        pytest.skip("the group size must divide cols")
    q = make_q(rows, cols, nbits, g, zb, seed=rows + cols + nbits)
    x, xo, xdt = make_x(batch, cols, dtype, seed=batch + 17)
    y = run(hq, q, x, rows, cols, nbits, g, zb)
    yo, ya = oracle.gemm(q["packed"], q["scale"], q["zero"], q["zero_meta"], rows, cols, nbits, g, zb, xo, xdt)
    check(y, yo, ya, cols)


@pytest.mark.parametrize("batch", [16, 48, 100, 128, 200, 256, 300, 777])
def test_gemm_batch_tiles(hq, batch):
    """One MMA N tile up to 256 rows of x, then equal tiles (a multiple of 16)."""
    rows, cols, nbits, g, zb = 256, 1024, 4, 64, 16
    q = make_q(rows, cols, nbits, g, zb, seed=batch)
    x, xo, xdt = make_x(batch, cols, torch.bfloat16, seed=batch)
    y = run(hq, q, x, rows, cols, nbits, g, zb)
    yo, ya = oracle.gemm(q["packed"], q["scale"], q["zero"], q["zero_meta"], rows, cols, nbits, g, zb, xo, xdt)
    check(y, yo, ya, cols)


@pytest.mark.parametrize("rows,cols,nbits,g,batch", [(11008, 4096, 4, 64, 128), (4096, 11008, 2, 16, 16),
                                                     (28672, 8192, 4, 128, 256)])
def test_gemm_full_size_sampled_rows(hq, rows, cols, nbits, g, batch):
    """Llama-2 MLP shapes in the benchmark's launch configuration; the oracle
    checks a sample of rows (rows are independent along axis 1)."""
    zb = 8 if g == 16 else 16
    q = make_q(rows, cols, nbits, g, zb, seed=rows % 97)
    x, xo, xdt = make_x(batch, cols, torch.bfloat16, seed=3)
    y = run(hq, q, x, rows, cols, nbits, g, zb)
    rng = np.random.default_rng(1)
    sample = np.unique(np.concatenate([[0, 127, 128, rows - 1], rng.choice(rows, 60, replace=False)]))
    bpr = cols * nbits // 8
    gpr = cols // g
    for r0 in sample:
        sub = dict(packed=q["packed"][r0 * bpr:(r0 + 1) * bpr], scale=q["scale"][r0 * gpr:(r0 + 1) * gpr],
                   zero=q["zero"][r0 * gpr:(r0 + 1) * gpr], zero_meta=q["zero_meta"])
        yo, ya = oracle.gemm(sub["packed"], sub["scale"], sub["zero"], sub["zero_meta"], 1, cols, nbits, g, zb, xo,
                             xdt)
        check(y[:, r0:r0 + 1], yo, ya, cols)


def test_gemm_unit_vectors_are_the_dequantiser_columns(hq):
    """x = e_c: y is column c of the dequantised matrix in x's type, exactly
    (one non-zero product per sum), against the GPU dequantiser's output."""
    rows, cols, nbits, g, zb = 256, 256, 4, 64, 16
    q = make_q(rows, cols, nbits, g, zb, seed=5)
    d = {k: (torch.from_numpy(v).cuda() if v is not None else None) for k, v in q.items()}
    cs = [0, 1, 63, 64, 127, 200, 255]
    for dtype in (torch.bfloat16, torch.float16):
        X = torch.zeros(len(cs), cols, dtype=dtype)
        for i, c in enumerate(cs):
            X[i, c] = 1.0
        y = hq.gemm(d, X.cuda(), rows, cols, nbits, g, zb)
        deq = hq.dequantize(d, rows, cols, nbits, g, 1, zb, dtype)
        torch.cuda.synchronize()
        for i, c in enumerate(cs):
            assert torch.equal(y[i].cpu(), deq[:, c].float().cpu()), (dtype, c)


def test_gemm_repeated_calls_are_deterministic(hq):
    rows, cols, nbits, g, zb = 512, 2048, 3, 64, 16
    q = make_q(rows, cols, nbits, g, zb, seed=8)
    x, _, _ = make_x(64, cols, torch.float16, seed=2)
    a = run(hq, q, x, rows, cols, nbits, g, zb)
    b = run(hq, q, x, rows, cols, nbits, g, zb)
    assert np.array_equal(a, b)


def test_gemm_bounded_wait_gives_up_and_reports(hq):
    """The product's mbarrier wait, run on a barrier nothing arrives on with a
    5 ms limit, gives up, the status reads HQQ_ERR_TIMEOUT once (then it is
    cleared), and the context stays usable: a product right after is correct."""
    assert hq.hqq_gemm_get_status() == hq.HQQ_OK
    assert hq.hqq_gemm_wait_selftest(5000) == hq.HQQ_OK
    assert hq.hqq_gemm_get_status() == hq.HQQ_ERR_TIMEOUT
    assert hq.hqq_gemm_get_status() == hq.HQQ_OK
    rows, cols, nbits, g, zb = 256, 512, 4, 64, 16
    q = make_q(rows, cols, nbits, g, zb, seed=11)
    x, xo, xdt = make_x(16, cols, torch.bfloat16, seed=11)
    y = run(hq, q, x, rows, cols, nbits, g, zb)
    yo, ya = oracle.gemm(q["packed"], q["scale"], q["zero"], q["zero_meta"], rows, cols, nbits, g, zb, xo, xdt)
    check(y, yo, ya, cols)


@pytest.mark.parametrize("rows,cols,batch", [(512, 4096, 16), (4096, 11008, 256), (1000, 8192, 40), (4096, 4096, 16)])
def test_gemm_split_k(hq, rows, cols, batch):
    """Grids too small for the GPU split K across CTAs; the last split of each
    tile sums the partials in split order: within the bound of the oracle,
    within twice the bound of the unsplit product, and bit-identical on
    repeated calls."""
    nbits, g, zb = 4, 64, 8
    assert hq.hqq_gemm_workspace_bytes(rows, cols, batch) > 0
    q = make_q(rows, cols, nbits, g, zb, seed=rows + batch)
    x, xo, xdt = make_x(batch, cols, torch.bfloat16, seed=batch)
    d = {k: (torch.from_numpy(v).cuda() if v is not None else None) for k, v in q.items()}
    xc = x.cuda()
    ys = hq.gemm(d, xc, rows, cols, nbits, g, zb)
    ys2 = hq.gemm(d, xc, rows, cols, nbits, g, zb)
    yu = hq.gemm(d, xc, rows, cols, nbits, g, zb, split=False)
    assert hq.hqq_gemm_get_status() == hq.HQQ_OK
    assert torch.equal(ys, ys2)
    ys, yu = ys.cpu().numpy().astype(np.float64), yu.cpu().numpy().astype(np.float64)
    sample = np.unique(np.r_[0, rows - 1, np.random.default_rng(2).choice(rows, 24, replace=False)])
    bpr, gpr = cols * nbits // 8, cols // g
    for r0 in sample:
        yo, ya = oracle.gemm(q["packed"][r0 * bpr:(r0 + 1) * bpr], q["scale"][r0 * gpr:(r0 + 1) * gpr],
                             q["zero"][r0 * gpr:(r0 + 1) * gpr], q["zero_meta"], 1, cols, nbits, g, zb, xo, xdt)
        check(ys[:, r0:r0 + 1], yo, ya, cols)
        check(yu[:, r0:r0 + 1], yo, ya, cols)
        assert np.all(np.abs(ys[:, r0:r0 + 1] - yu[:, r0:r0 + 1]) <= 2 * cols * 2.0 ** -23 * ya + 1e-30)
