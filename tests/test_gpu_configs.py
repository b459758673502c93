"""GPU parity at the full sizes of the other benchmark configurations.

The benchmark line times the Llama-2-7B MLP sweep (tests/test_gpu_parity.py
covers it in full).  The other configurations are checked here, each with the
launch configuration the library picks for that size:

* Llama-2-7B weight set, b4 g128, 8-bit zero, group stop: one decoder layer
  (q, k, v, o 4096x4096; gate, up 11008x4096; down 4096x11008; fp16, that
  layer's seeds), sampled groups against the oracle;
* Llama-2-13B mixed precision, tensor stop: attention 5120x5120 at b4 g64 and
  MLP 13824x5120 / 5120x13824 at b2 g32, every group against the full oracle
  (the stop is tensor-wide);
* Llama-2-70B shapes, b2 g16 and b4 g128, 8-bit zero, group stop: q 8192x8192,
  k 1024x8192, gate 28672x8192, down 8192x28672, sampled groups.

Sampled runs check the 8-bit zero by a property that holds at any size: the
meta pair and every code follow from the GPU's own fp32 kept zeros by the
quantiser's definition (one RTN pair from their min/max).
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


def _params(nbits, g, stop=0, zb=16):
    return dict(nbits=nbits, group_size=g, axis=1, p=0.7, beta=1.0, kappa=1.01, iters=20, stop_mode=stop,
                zero_nbits=zb)


def _zero8_property(gpu):
    z = gpu["zero_f32"].astype(np.float32)
    mn, mx = z.min(), z.max()
    sz = np.float32(2e4)
    if mx > mn:
        sz = min(np.float32(255.0) / np.float32(mx - mn), np.float32(2e4))
    zz = np.float32(-mn * sz)
    meta = gpu["zero_meta"]
    assert meta[0] == np.float32(np.float32(1.0) / sz) and meta[1] == zz, (meta, sz, zz)
    codes = np.clip(np.rint(np.float32(z * sz) + zz), 0, 255).astype(np.uint8)
    assert np.array_equal(codes, gpu["zero"])


def _sampled(hq, W_cpu, prm, n=4000, seed=0):
    rows, cols = W_cpu.shape
    G = rows * cols // prm["group_size"]
    out = hq.quantize(W_cpu.cuda(), prm["nbits"], prm["group_size"], prm["axis"], prm["p"], prm["beta"],
                      prm["kappa"], prm["iters"], prm["stop_mode"], prm["zero_nbits"], debug=True)
    torch.cuda.synchronize()
    assert hq.hqq_get_status(out["workspace"]) == hq.HQQ_OK
    gpu = pc.gpu_to_numpy(out)
    ids = np.sort(np.random.default_rng(seed).choice(G, size=min(n, G), replace=False))
    ids[0], ids[-1] = 0, G - 1
    rep = pc.check(W_cpu, prm, gpu, sample=np.unique(ids))
    if prm["zero_nbits"] == 8:
        _zero8_property(gpu)
    del out
    torch.cuda.empty_cache()
    return rep


LLAMA7B = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
           ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]


@pytest.mark.parametrize("name,rows,cols", LLAMA7B)
def test_llama2_7b_layer_b4_g128_zero8(hq, name, rows, cols):
    W = synth.weight(rows, cols, seed=synth.seed_for(31, name), dtype=torch.float16)
    _sampled(hq, W, _params(4, 128, zb=8))


@pytest.mark.parametrize("rows,cols,nbits,g", [(5120, 5120, 4, 64), (13824, 5120, 2, 32), (5120, 13824, 2, 32)])
def test_llama2_13b_mixed_tensor_stop(hq, rows, cols, nbits, g):
    W = synth.weight(rows, cols, seed=rows + 7 * cols, dtype=torch.float16)
    prm = _params(nbits, g, stop=1)
    out = hq.quantize(W.cuda(), nbits, g, stop_mode=1, debug=True)
    torch.cuda.synchronize()
    gpu = pc.gpu_to_numpy(out)
    Wo, dt = pc.w_for_oracle(W)
    orc = oracle.quantize(Wo, nbits, g, 1, 0.7, 1.0, 1.01, 20, 1, 16, dtype=dt)
    pc.check(W, prm, gpu, orc)
    assert np.all(gpu["best_iter"] == orc["best_iter"][0])


@pytest.mark.parametrize("rows,cols", [(8192, 8192), (1024, 8192), (28672, 8192), (8192, 28672)])
@pytest.mark.parametrize("nbits,g", [(2, 16), (4, 128)])
def test_llama2_70b_shapes_zero8(hq, rows, cols, nbits, g):
    W = synth.weight(rows, cols, seed=rows // 1024 + cols // 1024, dtype=torch.float16)
    _sampled(hq, W, _params(nbits, g, zb=8))


def test_llama2_7b_every_layer_first_matrix(hq):
    """Full-model configuration, sampled: the first matrix (q) of every one of
    the 32 layers, each with that layer's seed, 1000 random groups per layer."""
    for layer in range(32):
        W = synth.weight(4096, 4096, seed=synth.seed_for(layer, "q"), dtype=torch.float16)
        _sampled(hq, W, _params(4, 128, zb=8), n=1000, seed=layer)
