"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Inputs are seeded synthetic weights with the pages' weight statistics
(0.02 * N(0,1), 0.1% outliers x10) plus degenerate cases.  Small shapes span
several tiles and a ragged tail; the Llama-2 shapes the benchmark quantises
are checked in full, in the same launch configuration.
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


def _params(nbits, g, axis=1, p=0.7, beta=1.0, kappa=1.01, iters=20, stop=0, zb=16):
    return dict(nbits=nbits, group_size=g, axis=axis, p=p, beta=beta, kappa=kappa, iters=iters, stop_mode=stop,
                zero_nbits=zb)


def _run(hq, W_cpu, prm, check_recon=True, tie_cap=None):
    W = W_cpu.cuda()
    out = hq.quantize(W, prm["nbits"], prm["group_size"], prm["axis"], prm["p"], prm["beta"], prm["kappa"],
                      prm["iters"], prm["stop_mode"], prm["zero_nbits"], debug=True)
    torch.cuda.synchronize()
    st = hq.hqq_get_status(out["workspace"])
    assert st == hq.HQQ_OK, hq.hqq_status_string(st)
    gpu = pc.gpu_to_numpy(out)
    Wo, dt = pc.w_for_oracle(W_cpu)
    orc = oracle.quantize(Wo, prm["nbits"], prm["group_size"], prm["axis"], prm["p"], prm["beta"], prm["kappa"],
                          prm["iters"], prm["stop_mode"], prm["zero_nbits"], dtype=dt)
    rep = pc.check(W_cpu, prm, gpu, orc, tie_cap=tie_cap)
    if prm["zero_nbits"] == 8:
        pc.check_zero8(gpu, orc)
    if check_recon:
        rows, cols = W_cpu.shape
        for out_dt in (torch.float16, torch.bfloat16):
            deq = hq.dequantize(out, rows, cols, prm["nbits"], prm["group_size"], prm["axis"], prm["zero_nbits"],
                                out_dt)
            d = deq.cpu()
            d = d.numpy() if out_dt == torch.float16 else d.view(torch.int16).numpy().view(np.uint16)
            pc.check_reconstruction(W_cpu, prm, d, orc, pc.gpu_dequantizer(hq))
    return rep, gpu, orc


# ------------------------------------------------------------- group mode --

@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("nbits", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("g", [8, 16, 32, 64, 128, 256, 512, 1024])
def test_group_mode_axis1(hq, dtype, nbits, g):
    rows = max(8, 40960 // 512)  # several tiles for small g, ragged tails for large g
    W = synth.weight(rows + 3, 1024, seed=nbits * 100 + g, dtype=dtype)
    _run(hq, W, _params(nbits, g), check_recon=(g in (16, 64)))


@pytest.mark.parametrize("rows,cols,g", [(37, 192, 64), (1000, 320, 64), (777, 64, 16), (5, 1024, 1024),
                                         (301, 1536, 512), (2049, 40, 8)])
def test_ragged_tiles(hq, rows, cols, g):
    W = synth.weight(rows, cols, seed=rows + cols, dtype=torch.float16)
    _run(hq, W, _params(4, g))


@pytest.mark.parametrize("rows,cols,g", [(256, 200, 64), (128, 37, 32), (1024, 520, 16), (2048, 24, 1024),
                                         (64, 1000, 8)])
@pytest.mark.parametrize("nbits", [3, 4])
def test_axis0(hq, rows, cols, g, nbits):
    W = synth.weight(rows, cols, seed=7 * rows + cols, dtype=torch.bfloat16)
    _run(hq, W, _params(nbits, g, axis=0))


@pytest.mark.parametrize("iters", [0, 1, 2, 5, 11, 20, 50])  # 11, 20: tensor-stop tail chunks merged (g = 32)
@pytest.mark.parametrize("stop", [0, 1, 2])
def test_iteration_counts_and_modes(hq, iters, stop):
    W = synth.weight(300, 512, seed=iters * 3 + stop, dtype=torch.float16)
    _run(hq, W, _params(2, 32, iters=iters, stop=stop))


@pytest.mark.parametrize("nbits,g,stop", [(2, 128, 0), (2, 16, 0), (4, 32, 0), (2, 128, 2)])
def test_long_group_runs(hq, nbits, g, stop):
    """Groups that keep improving for hundreds of iterations (p = 1.9, beta 20,
    no annealing; on the oracle the kept iterates average 116, 74 and 63 at
    g128, g16 and g32, up to 543): the one-pass solver's groups pass through
    many survivor rounds of its shared-memory pool; group stop and no stop,
    1000 iterations, against the oracle.  Here a group's error flattens for
    hundreds of iterations, so successive errors differ by less than the tie
    margin (reading T1: the hardware lg2/ex2 and the summation order move a
    sum by up to ~5e-6 relative) and nearly every group's stop is a near tie
    (2,007 of 2,048 at g128): the cap of 1e-4 of the groups, made for the
    benchmark's regime, is lifted, and every group whose kept iterate differs
    must still be explained by near ties on the oracle's own trajectory and
    match the oracle's iterate at the GPU's index (zero and codes), which is
    what a corrupted pool record would fail."""
    W = synth.weight(256, 1024, seed=17, dtype=torch.float16)
    _run(hq, W, _params(nbits, g, p=1.9, beta=20.0, kappa=1.0, iters=1000, stop=stop), check_recon=False,
         tie_cap=256 * 1024 // g)


@pytest.mark.parametrize("p,beta,kappa", [(0.5, 1.0, 1.01), (1.2, 1.0, 1.01), (0.7, 10.0, 1.05), (0.7, 1.0, 1.0)])
def test_solver_parameters(hq, p, beta, kappa):
    W = synth.weight(256, 512, seed=int(p * 100), dtype=torch.float16)
    for stop in (0, 1):
        _run(hq, W, _params(4, 64, p=p, beta=beta, kappa=kappa, stop=stop), check_recon=False)


@pytest.mark.parametrize("stop", [0, 1, 2])
def test_shrink_active(hq, stop):
    """Large weights make |W - W_r| exceed the shrink threshold: W_e != 0 path."""
    W = (synth.weight(128, 256, seed=5, dtype=torch.float32) * 200.0).to(torch.float16)
    for nbits in (1, 2):
        _run(hq, W, _params(nbits, 64, beta=4.0, stop=stop), check_recon=False)


def test_constant_and_zero_groups(hq):
    W = synth.weight(64, 512, seed=9, dtype=torch.float16)
    W[0:8] = 0.0
    W[8:16, :] = 0.015625
    W[16, :256] = -0.5
    for zb in (16, 8):
        _run(hq, W, _params(4, 64, zb=zb))


@pytest.mark.parametrize("stop", [0, 1])
@pytest.mark.parametrize("nbits,g", [(4, 128), (2, 16)])
def test_zero_8bit(hq, stop, nbits, g):
    W = synth.weight(512, 1024, seed=11, dtype=torch.float16)
    _run(hq, W, _params(nbits, g, stop=stop, zb=8))


def test_empty_input(hq):
    W = torch.empty(0, 64, dtype=torch.float16, device="cuda")
    out = hq.quantize(W, 4, 64, zero_nbits=8)
    torch.cuda.synchronize()
    meta = out["zero_meta"].cpu().numpy()
    assert meta[0] == np.float32(1.0 / np.float32(2e4)) and meta[1] == 0.0
    out = hq.quantize(W, 4, 64, zero_nbits=16)
    torch.cuda.synchronize()
    assert hq.hqq_get_status(out["workspace"]) == hq.HQQ_OK


def test_repeated_calls_reuse_outputs(hq):
    """The same buffers and workspace serve consecutive calls (workspace needs no
    initialisation by the caller)."""
    W = synth.weight(512, 512, seed=12, dtype=torch.float16)
    prm = _params(4, 64, stop=1, zb=8)
    out = hq.quantize(W.cuda(), 4, 64, stop_mode=1, zero_nbits=8, debug=True)
    first = pc.gpu_to_numpy(out)
    out = hq.quantize(W.cuda(), 4, 64, stop_mode=1, zero_nbits=8, debug=True, out=out)
    second = pc.gpu_to_numpy(out)
    for k in ("packed", "scale", "zero", "zero_meta", "best_iter", "zero_f32"):
        assert np.array_equal(first[k], second[k]), k
    pc.check(W, prm, second)


# ---------------------------------------------------------- error paths ----

def test_host_pointer_rejected(hq):
    W = synth.weight(64, 64, seed=1, dtype=torch.float16)  # CPU tensor
    out = hq.alloc_outputs(64, 64, 4, 64)
    rc = hq.hqq_quantize(W, 64, 64, hq.HQQ_F16, 4, 64, 1, 0.7, 1.0, 1.01, 20, 0, 16, out["packed"], out["scale"],
                         out["zero"], None, out["workspace"], out["workspace"].numel())
    assert rc == hq.HQQ_ERR_INVALID_ARG


def test_small_workspace_rejected(hq):
    W = synth.weight(64, 64, seed=1, dtype=torch.float16).cuda()
    out = hq.alloc_outputs(64, 64, 4, 64, stop_mode=1)
    rc = hq.hqq_quantize(W, 64, 64, hq.HQQ_F16, 4, 64, 1, 0.7, 1.0, 1.01, 20, 1, 16, out["packed"], out["scale"],
                         out["zero"], None, out["workspace"], out["workspace"].numel() - 1)
    assert rc == hq.HQQ_ERR_WORKSPACE


def test_misaligned_input_rejected(hq):
    W = synth.weight(64, 72, seed=1, dtype=torch.float16).cuda().reshape(-1)[8:8 + 64 * 64].view(64, 64)
    base = synth.weight(64, 65, seed=1, dtype=torch.float16).cuda().reshape(-1)[1:1 + 64 * 64].view(64, 64)
    out = hq.alloc_outputs(64, 64, 4, 64)
    rc = hq.hqq_quantize(base, 64, 64, hq.HQQ_F16, 4, 64, 1, 0.7, 1.0, 1.01, 20, 0, 16, out["packed"], out["scale"],
                         out["zero"], None, out["workspace"], out["workspace"].numel())
    assert rc == hq.HQQ_ERR_ALIGN
    rc = hq.hqq_quantize(W, 64, 64, hq.HQQ_F16, 4, 64, 1, 0.7, 1.0, 1.01, 20, 0, 16, out["packed"], out["scale"],
                         out["zero"], None, out["workspace"], out["workspace"].numel())
    assert rc == hq.HQQ_OK


# ------------------------------------------------- full sizes, sampled -----

def _sampled(hq, W_cpu, prm, n=6000, seed=0):
    rows, cols = W_cpu.shape
    G = rows * cols // prm["group_size"]
    W = W_cpu.cuda()
    out = hq.quantize(W, prm["nbits"], prm["group_size"], prm["axis"], prm["p"], prm["beta"], prm["kappa"],
                      prm["iters"], prm["stop_mode"], prm["zero_nbits"], debug=True)
    torch.cuda.synchronize()
    assert hq.hqq_get_status(out["workspace"]) == hq.HQQ_OK
    gpu = pc.gpu_to_numpy(out)
    ids = np.sort(np.random.default_rng(seed).choice(G, size=min(n, G), replace=False))
    ids[0], ids[-1] = 0, G - 1  # first and last group always
    rep = pc.check(W_cpu, prm, gpu, sample=np.unique(ids))
    return rep, gpu


def test_llama_square_4096_fp16_b4_g64(hq):
    """Single 4096x4096 fp16 weight, b4 g64, group stop, fp16 zero: full tensor."""
    W = synth.weight(4096, 4096, seed=0, dtype=torch.float16)
    rep, _, _ = _run(hq, W, _params(4, 64))
    assert rep["tie_groups"] <= 1e-4 * (4096 * 4096 // 64) + 1


SWEEP = [(8, 128), (4, 64), (3, 64), (2, 16), (1, 16)]


@pytest.mark.parametrize("nbits,g", SWEEP)
@pytest.mark.parametrize("shape", [(11008, 4096), (4096, 11008)])
def test_llama_mlp_group_mode(hq, nbits, g, shape):
    """Llama-2-7B MLP shapes (gate/up and down), bf16, group stop: full tensors."""
    W = synth.weight(*shape, seed=4 if shape[0] == 11008 else 6, dtype=torch.bfloat16)
    _run(hq, W, _params(nbits, g), check_recon=(nbits == 4))


@pytest.mark.parametrize("nbits,g", SWEEP)
def test_llama_mlp_tensor_mode(hq, nbits, g):
    """Llama-2-7B gate shape, bf16, tensor stop: full tensor against the full oracle."""
    W = synth.weight(11008, 4096, seed=4, dtype=torch.bfloat16)
    rep, gpu, orc = _run(hq, W, _params(nbits, g, stop=1), check_recon=(nbits == 2))
    assert np.all(gpu["best_iter"] == orc["best_iter"][0])


@pytest.mark.parametrize("nbits,g,zb,iters", [(4, 64, 16, 20), (8, 128, 8, 20), (2, 16, 8, 20), (1, 16, 16, 20),
                                              (3, 64, 16, 11), (4, 32, 8, 1), (2, 64, 16, 2)])
def test_tensor_outputs_without_debug(hq, nbits, g, zb, iters):
    """Tensor stop without debug outputs writes its outputs in a separate
    streaming pass (axis 1); they must equal the debug run's, which the other
    tests check against the oracle."""
    W = synth.weight(1000, 1024, seed=nbits * 31 + g, dtype=torch.bfloat16).cuda()
    ref = hq.quantize(W, nbits, g, iters=iters, stop_mode=1, zero_nbits=zb, debug=True)
    got = hq.quantize(W, nbits, g, iters=iters, stop_mode=1, zero_nbits=zb)
    torch.cuda.synchronize()
    for k in ("packed", "scale", "zero", "zero_meta"):
        if ref[k] is None:
            continue
        assert torch.equal(ref[k].view(torch.uint8), got[k].view(torch.uint8)), k
    # and the debug run against the oracle
    _run(hq, W.cpu(), _params(nbits, g, stop=1, zb=zb, iters=iters), check_recon=False)


def _nodebug_equals_debug(hq, W, nbits, g, zb, iters):
    ref = hq.quantize(W, nbits, g, iters=iters, stop_mode=1, zero_nbits=zb, debug=True)
    got = hq.quantize(W, nbits, g, iters=iters, stop_mode=1, zero_nbits=zb)
    torch.cuda.synchronize()
    assert hq.hqq_get_status(got["workspace"]) == hq.HQQ_OK
    for k in ("packed", "scale", "zero", "zero_meta"):
        if ref[k] is None:
            continue
        assert torch.equal(ref[k].view(torch.uint8), got[k].view(torch.uint8)), k


@pytest.mark.parametrize("nbits,g,zb", [(4, 64, 16), (2, 64, 8), (1, 32, 16), (8, 128, 8), (3, 256, 16)])
@pytest.mark.parametrize("place", ["last", "rise_last", "rise_in_last_chunk", "rise_before_last_chunk"])
def test_tensor_outputs_kept_iterate_placement(hq, nbits, g, zb, place):
    """Without debug outputs the last chunk writes the outputs of its last
    iterate, and the output pass rewrites them when a tensor error rose.  The
    iteration count is set from the oracle's own tensor trajectory (kept
    iterate kb at 100 iterations, its error rising at kb + 1) so that the
    rise falls after the last iteration, at it, inside the last chunk, or
    before the last chunk; the outputs must equal the debug run's, and the
    debug run must match the oracle."""
    W_cpu = synth.weight(600, 1024, seed=nbits * 53 + g, dtype=torch.bfloat16)
    Wo, dt = pc.w_for_oracle(W_cpu)
    kb = int(oracle.quantize(Wo, nbits, g, 1, 0.7, 1.0, 1.01, 100, 1, zb, dtype=dt)["best_iter"][0])
    assert 4 <= kb < 90, kb
    iters = {"last": kb + 1, "rise_last": kb + 2, "rise_in_last_chunk": kb + 4,
             "rise_before_last_chunk": kb + 30}[place]
    _nodebug_equals_debug(hq, W_cpu.cuda(), nbits, g, zb, iters)
    _run(hq, W_cpu, _params(nbits, g, stop=1, zb=zb, iters=iters), check_recon=False)


@pytest.mark.parametrize("nbits,g", SWEEP)
def test_llama_mlp_down_tensor_mode(hq, nbits, g):
    """Llama-2-7B down shape (4096x11008, bf16, the layer's seed), tensor
    stop, every setting of the sweep: full tensor against the full oracle, and
    the launch configuration without debug outputs gives the same bytes."""
    W = synth.weight(4096, 11008, seed=6, dtype=torch.bfloat16)
    rep, gpu, orc = _run(hq, W, _params(nbits, g, stop=1), check_recon=(nbits == 3))
    if "tensor_tie" not in rep:
        assert np.all(gpu["best_iter"] == orc["best_iter"][0])
    _nodebug_equals_debug(hq, W.cuda(), nbits, g, 16, 20)


@pytest.mark.parametrize("nbits,g", SWEEP)
@pytest.mark.parametrize("zb", [16, 8])
def test_llama_mlp_tensor_mode_outputs_without_debug(hq, nbits, g, zb):
    """The benchmark's launch configuration (tensor stop, no debug outputs) on
    the Llama-2-7B gate shape: the same bytes as the debug run, which
    test_llama_mlp_tensor_mode checks against the oracle."""
    W = synth.weight(11008, 4096, seed=4, dtype=torch.bfloat16).cuda()
    _nodebug_equals_debug(hq, W, nbits, g, zb, 20)
