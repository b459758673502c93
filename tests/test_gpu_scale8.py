"""GPU parity of the 8-bit scales (the "_s*" variant of the Llama-2 table:
the scale is also quantised to 8 bit, group size 128) against the oracle.

Codes and meta pairs are integer decisions taken from fp32 arithmetic that
both sides perform in the same order, so they must agree bit for bit.  The
dequantiser with 8-bit scales must agree bit for bit on the same inputs.
"""
import numpy as np
import pytest
import torch

import oracle
from calibration_free_weight_b200 import synth

from . import parity_check as pc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from calibration_free_weight_b200 import hqq
    return hqq


def _gpu_scale8(hq, sc16, S):
    G = sc16.numel()
    q = {"scale": sc16.cuda()}
    hq.quantize_scale8(q, S)
    torch.cuda.synchronize()
    return q["scale_q"].cpu().numpy(), q["scale_meta"].cpu().numpy()


@pytest.mark.parametrize("G,S", [(1000, 128), (128, 128), (129, 128), (5, 128), (300, 7), (257, 1), (4096, 4096),
                                 (70000, 128)])
def test_scale8_matches_oracle(hq, G, S):
    sc = synth.scales(G, seed=G + S)
    c, m = _gpu_scale8(hq, sc, S)
    oc, om = oracle.quantize_scale8(sc.numpy(), S)
    assert np.array_equal(c, oc)
    assert np.array_equal(m.view(np.uint32), om.view(np.uint32))


def test_scale8_full_size_70b_gate_g16(hq):
    """28672x8192 at g16: 14.68 M scales, 114,688 runs of 128."""
    G = 28672 * 8192 // 16
    sc = synth.scales(G, seed=70)
    c, m = _gpu_scale8(hq, sc, 128)
    oc, om = oracle.quantize_scale8(sc.numpy(), 128)
    assert np.array_equal(c, oc)
    assert np.array_equal(m.view(np.uint32), om.view(np.uint32))


def test_scale8_empty(hq):
    q = {"scale": torch.empty(0, dtype=torch.float16, device="cuda")}
    hq.quantize_scale8(q, 128)
    torch.cuda.synchronize()
    assert q["scale_q"].numel() == 0


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("nbits,g,zb", [(2, 16, 8), (4, 64, 16), (3, 32, 8)])
def test_pipeline_with_8bit_scales(hq, dtype, nbits, g, zb):
    """quantize -> 8-bit scales -> dequantize, GPU against oracle on the same W."""
    rows, cols = 333, 1024
    W = synth.weight(rows, cols, seed=nbits * 10 + g, dtype=dtype)
    out = hq.quantize(W.cuda(), nbits, g, zero_nbits=zb, debug=True)
    hq.quantize_scale8(out, 128)
    d8 = {dt: hq.dequantize_s8(out, rows, cols, nbits, g, zero_nbits=zb, out_dtype=dt)
          for dt in (torch.float16, torch.bfloat16)}
    torch.cuda.synchronize()
    gpu = pc.gpu_to_numpy(out)
    Wo, dt = pc.w_for_oracle(W)
    orc = oracle.quantize(Wo, nbits, g, 1, 0.7, 1.0, 1.01, 20, 0, zb, dtype=dt)
    pc.check(W, dict(nbits=nbits, group_size=g, axis=1, p=0.7, beta=1.0, kappa=1.01, iters=20, stop_mode=0,
                     zero_nbits=zb), gpu, orc)
    # scales are computed by identical fp32 steps on both sides: the 8-bit scales agree exactly
    oc, om = oracle.quantize_scale8(orc["scale"], 128)
    assert np.array_equal(gpu["scale_q"], oc) and np.array_equal(gpu["scale_meta"], om)
    # dequantiser with 8-bit scales: bit-exact against the oracle on the oracle's own outputs
    run = pc.gpu_dequantizer(hq)
    for code in (oracle.F16, oracle.BF16):
        ref = oracle.dequantize_s8(orc["packed"], oc, om, 128, orc["zero"], orc["zero_meta"], rows, cols, nbits, g, 1,
                                   zb, code)
        got = run(dict(packed=orc["packed"], scale_q=oc, scale_meta=om, zero=orc["zero"], zero_meta=orc["zero_meta"]),
                  rows, cols, nbits, g, 1, zb, code, scale8=128)
        assert np.array_equal(ref.view(np.uint16), got)
    # the GPU's own pipeline: same tensor lp error as the oracle's
    Wf = pc.w_float(W).astype(np.float64)
    for out_dt, d in d8.items():
        code = oracle.F16 if out_dt == torch.float16 else oracle.BF16
        od = oracle.dequantize_s8(orc["packed"], oc, om, 128, orc["zero"], orc["zero_meta"], rows, cols, nbits, g, 1,
                                  zb, code)
        got = d.cpu()
        got = got.numpy().astype(np.float64) if out_dt == torch.float16 else \
            got.float().numpy().astype(np.float64)
        odf = od.astype(np.float64) if code == oracle.F16 else \
            (od.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        eg, eo = np.mean(np.abs(Wf - got) ** 0.7), np.mean(np.abs(Wf - odf) ** 0.7)
        assert abs(eg - eo) <= 1e-3 * eo
