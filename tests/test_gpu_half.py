"""GPU parity of the half-precision solver variant (hqq_quantize_half)
against its oracle (oracle.quantize_half): the arithmetic of both sides is
the same fp16 rounding sequence except the error terms, so outputs are
bit-identical except at near-tie stop decisions, which must be explained on
the oracle's own trajectory (parity_check.check_half).

Method: techreport.ngo, "Weight-only quantization without the calibration
tax", sections "Speed: from hours to minutes" (the solver in half precision)
and "Outlier-aware optimization without gradients" (the steps)."""
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


def _run(hq, W_cpu, nbits, g, stop=0, zb=16, iters=20, beta=1.0, kappa=1.01):
    prm = dict(nbits=nbits, group_size=g, axis=1, p=0.7, beta=beta, kappa=kappa, iters=iters, stop_mode=stop,
               zero_nbits=zb)
    out = hq.quantize_half(W_cpu.cuda(), nbits, g, 0.7, beta, kappa, iters, stop, zb, debug=True)
    torch.cuda.synchronize()
    assert hq.hqq_get_status(out["workspace"]) == hq.HQQ_OK
    gpu = pc.gpu_to_numpy(out)
    orc = oracle.quantize_half(W_cpu.numpy(), nbits, g, 1, 0.7, beta, kappa, iters, stop, zb)
    rep = pc.check_half(W_cpu, prm, gpu, orc)
    if zb == 8:
        z = gpu["zero_f32"]
        mn, mx = z.min(), z.max()
        sz = min(np.float32(255.0) / np.float32(mx - mn), np.float32(2e4)) if mx > mn else np.float32(2e4)
        zz = np.float32(-mn * sz)
        assert gpu["zero_meta"][0] == np.float32(np.float32(1.0) / sz) and gpu["zero_meta"][1] == zz
        assert np.array_equal(np.clip(np.rint(np.float32(z * sz) + zz), 0, 255).astype(np.uint8), gpu["zero"])
    return rep


@pytest.mark.parametrize("nbits", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("g", [8, 16, 32, 64, 128, 1024])
def test_half_group_mode(hq, nbits, g):
    W = synth.weight(67, 2048, seed=nbits * 10 + g, dtype=torch.float16)
    rep = _run(hq, W, nbits, g)
    assert rep["tie_frac"] < 0.05, rep


@pytest.mark.parametrize("iters", [0, 1, 2, 20, 50])
@pytest.mark.parametrize("stop", [0, 2])
def test_half_iterations_and_modes(hq, iters, stop):
    W = synth.weight(300, 512, seed=iters + 7 * stop, dtype=torch.float16)
    _run(hq, W, 2, 32, stop=stop, iters=iters)


def test_half_proximal_path(hq):
    """Large weights and beta = 4 make the proximal step non-zero (the slow path)."""
    W = (synth.weight(128, 256, seed=5, dtype=torch.float32) * 200.0).to(torch.float16)
    for nbits in (1, 2):
        _run(hq, W, nbits, 64, beta=4.0)


@pytest.mark.parametrize("nbits,g", [(2, 16), (4, 128)])
def test_half_llama2_70b_gate_zero8(hq, nbits, g):
    """The 70B gate shape (28672x8192) at the model's two settings, 8-bit zero,
    every group against the oracle."""
    W = synth.weight(28672, 8192, seed=synth.seed_for(2, "gate"), dtype=torch.float16)
    rep = _run(hq, W, nbits, g, zb=8)
    assert rep["tie_frac"] < 0.05, rep


def test_half_rejects(hq):
    W = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(hq.HQQError):
        hq.quantize_half(W, 4, 64)
    W16 = torch.zeros(64, 64, dtype=torch.float16, device="cuda")
    with pytest.raises(hq.HQQError):
        hq.quantize_half(W16, 4, 64, stop_mode=hq.HQQ_STOP_TENSOR)
