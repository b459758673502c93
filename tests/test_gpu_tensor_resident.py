"""GPU parity of tensor stop on one cooperative launch (W kept on chip).

Tensor stop decides on the mean lp error over the whole tensor
(techreport.ngo, "Weight-only quantization without the calibration tax",
section "Outlier-aware optimization without gradients").  On axis 1, when W
fits in half the L2 and the per-group state in shared memory, the library
runs every iteration in one cooperative launch: warps publish per-iteration
error partials, the last one to arrive sums them and publishes the stop
decision, and a warp runs at most three iterations ahead of the published
decisions (five zero-points per group are kept for that).  These tests check
that launch against the oracle: every bit width and group size in both 16-bit
types, every position of the kept iterate relative to the lookahead (no
rise, a rise at each of the last iterations, a rise found inside the loop),
ragged and degenerate shapes, the 8-bit zero, an active proximal step, the
Llama-2-7B attention shape and its launch without debug outputs.  They also
check that the chunked launches (hqq_set_tensor_resident(0)) give
the same outputs, that a workspace passes between the two, and the bounded
wait's timeout status.
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
    """The binding, with the resident launch taken wherever it fits (mode 2:
    also below g = 32, where the default leaves it to the chunks)."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from calibration_free_weight_b200 import hqq
    prev = hqq.hqq_set_tensor_resident(2)
    yield hqq
    hqq.hqq_set_tensor_resident(prev)


@pytest.fixture
def chunked(hq):
    prev = hq.hqq_set_tensor_resident(0)
    yield
    hq.hqq_set_tensor_resident(prev)


def _params(nbits, g, p=0.7, beta=1.0, kappa=1.01, iters=20, zb=16):
    return dict(nbits=nbits, group_size=g, axis=1, p=p, beta=beta, kappa=kappa, iters=iters, stop_mode=1,
                zero_nbits=zb)


def _dt(W):
    return 0 if W.dtype == torch.float16 else 1


def _resident(hq, W, g, iters=20):
    return hq.hqq_tensor_resident(W.shape[0], W.shape[1], _dt(W), g, 1, iters) == 1


def _run(hq, W_cpu, prm):
    W = W_cpu.cuda()
    out = hq.quantize(W, prm["nbits"], prm["group_size"], 1, prm["p"], prm["beta"], prm["kappa"], prm["iters"], 1,
                      prm["zero_nbits"], debug=True)
    torch.cuda.synchronize()
    st = hq.hqq_get_status(out["workspace"])
    assert st == hq.HQQ_OK, hq.hqq_status_string(st)
    gpu = pc.gpu_to_numpy(out)
    Wo, dt = pc.w_for_oracle(W_cpu)
    orc = oracle.quantize(Wo, prm["nbits"], prm["group_size"], 1, prm["p"], prm["beta"], prm["kappa"], prm["iters"],
                          1, prm["zero_nbits"], dtype=dt)
    rep = pc.check(W_cpu, prm, gpu, orc)
    if prm["zero_nbits"] == 8:
        pc.check_zero8(gpu, orc)
    return rep, gpu, orc


def _outputs(hq, W, prm, debug):
    out = hq.quantize(W, prm["nbits"], prm["group_size"], 1, prm["p"], prm["beta"], prm["kappa"], prm["iters"], 1,
                      prm["zero_nbits"], debug=debug)
    torch.cuda.synchronize()
    assert hq.hqq_get_status(out["workspace"]) == hq.HQQ_OK
    return {k: out[k].view(torch.uint8).cpu() for k in ("packed", "scale", "zero", "zero_meta")
            if out[k] is not None}


def _same(a, b):
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_path_selection(hq):
    f16, bf16 = torch.float16, torch.bfloat16
    prev = hq.hqq_set_tensor_resident(1)  # the default: g >= 32 only
    try:
        assert _resident(hq, torch.empty(4096, 4096, dtype=f16), 32)
        assert not _resident(hq, torch.empty(1000, 1024, dtype=bf16), 16)
    finally:
        hq.hqq_set_tensor_resident(prev)
    assert _resident(hq, torch.empty(4096, 4096, dtype=f16), 64)      # Llama-2-7B attention, b4 g64
    assert _resident(hq, torch.empty(5120, 5120, dtype=f16), 64)      # Llama-2-13B attention, b4 g64
    assert _resident(hq, torch.empty(1000, 1024, dtype=bf16), 16)
    assert not _resident(hq, torch.empty(11008, 4096, dtype=bf16), 64)  # W above half the L2
    assert not _resident(hq, torch.empty(4096, 4096, dtype=f16), 16)    # state above the shared memory
    assert not _resident(hq, torch.empty(4096, 4096, dtype=f16), 64, iters=0)
    assert hq.hqq_tensor_resident(4096, 4096, 0, 64, 0, 20) == 0         # axis 0: chunked
    assert hq.hqq_tensor_resident(4096, 4096, 0, 48, 1, 20) == 0         # invalid group size


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("nbits", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("g", [8, 16, 32, 64, 128, 256, 512, 1024])
def test_every_width_and_group(hq, dtype, nbits, g):
    W = synth.weight(384, 2048, seed=nbits * 97 + g, dtype=dtype)
    assert _resident(hq, W, g)
    _run(hq, W, _params(nbits, g))


@pytest.mark.parametrize("nbits,g,zb", [(4, 64, 16), (2, 64, 8), (1, 32, 16), (8, 128, 8), (3, 256, 16), (1, 16, 8)])
@pytest.mark.parametrize("delta", [1, 2, 3, 4, 5, 6, 30])
def test_kept_iterate_positions(hq, nbits, g, zb, delta):
    """iters = kb + delta, with kb the oracle's kept iterate at 100 iterations
    (its error rises at kb + 1): delta 1 no rise, 2-4 a rise among the last
    three iterations (found after the loop), 5 and more a rise found at the
    start of an iteration inside the loop, the kept zero-point then being the
    oldest of the five kept per group."""
    W_cpu = synth.weight(600, 1024, seed=nbits * 53 + g, dtype=torch.bfloat16)
    Wo, dt = pc.w_for_oracle(W_cpu)
    kb = int(oracle.quantize(Wo, nbits, g, 1, 0.7, 1.0, 1.01, 100, 1, zb, dtype=dt)["best_iter"][0])
    assert 4 <= kb < 70, kb
    prm = _params(nbits, g, iters=kb + delta, zb=zb)
    rep, gpu, orc = _run(hq, W_cpu, prm)
    if "tensor_tie" not in rep:
        assert np.all(gpu["best_iter"] == kb)
    _same(_outputs(hq, W_cpu.cuda(), prm, False), _outputs(hq, W_cpu.cuda(), prm, True))


@pytest.mark.parametrize("iters", [1, 2, 3, 4, 5, 6, 7, 8, 50])
@pytest.mark.parametrize("nbits,g", [(4, 64), (2, 16)])
def test_iteration_counts(hq, iters, nbits, g):
    W = synth.weight(512, 1024, seed=iters, dtype=torch.float16)
    _run(hq, W, _params(nbits, g, iters=iters))


@pytest.mark.parametrize("rows,cols,g", [(37, 192, 64), (5, 1024, 1024), (777, 64, 16), (3, 8, 8), (1, 1024, 512),
                                         (1000, 320, 32), (33, 4096, 128)])
def test_ragged_and_tiny(hq, rows, cols, g):
    W = synth.weight(rows, cols, seed=rows + cols, dtype=torch.bfloat16)
    assert _resident(hq, W, g)
    _run(hq, W, _params(4, g))
    _run(hq, W, _params(3 if g % 8 == 0 else 2, g, zb=8))


@pytest.mark.parametrize("p,beta,kappa", [(0.5, 1.0, 1.01), (1.2, 1.0, 1.01), (0.7, 10.0, 1.05), (0.7, 1.0, 1.0)])
def test_solver_parameters(hq, p, beta, kappa):
    W = synth.weight(256, 1024, seed=11, dtype=torch.float16)
    _run(hq, W, _params(4, 64, p=p, beta=beta, kappa=kappa))


@pytest.mark.parametrize("nbits", [1, 2])
def test_shrink_active(hq, nbits):
    """Large weights make |W - W_r| exceed the shrink threshold (beta 4), so the
    proximal step is non-zero and the slow path re-reads W from memory."""
    W = (synth.weight(128, 256, seed=5, dtype=torch.float32) * 200.0).to(torch.float16)
    assert _resident(hq, W, 64)
    _run(hq, W, _params(nbits, 64, beta=4.0))


def test_constant_and_zero_groups(hq):
    W = synth.weight(64, 1024, seed=5, dtype=torch.float16)
    W[3] = 0.0
    W[7, :512] = 0.125
    W[9, 64:128] = -3.0
    _run(hq, W, _params(4, 64))
    _run(hq, W, _params(2, 16, zb=8))


@pytest.mark.parametrize("p,beta,kappa,nbits,g", [(1.9, 20.0, 1.0, 2, 128), (1.0, 20.0, 1.05, 2, 64)])
@pytest.mark.parametrize("mode", [2, 0])
def test_long_runs(hq, p, beta, kappa, nbits, g, mode):
    """Tensor errors that keep falling for hundreds of iterations (p near 2 or
    1, a large beta; the oracle keeps iterates 543 and 321 of 1000): the
    resident launch's rounds wrap its decision ring, its zero-point ring and
    its arrival counters many times, and the chunked launches (mode 0) run
    over a hundred chunks against their fixed error history; outputs against
    the oracle."""
    W = synth.weight(256, 1024, seed=17, dtype=torch.float16)
    prev = hq.hqq_set_tensor_resident(mode)
    try:
        assert _resident(hq, W, g, iters=1000) == (mode == 2)
        rep, gpu, orc = _run(hq, W, _params(nbits, g, p=p, beta=beta, kappa=kappa, iters=1000))
    finally:
        hq.hqq_set_tensor_resident(prev)
    assert int(orc["best_iter"][0]) > 300


def test_llama2_7b_attention_b4_g64(hq):
    """The Llama-2-7B attention shape (4096x4096, fp16, seed 0) with tensor
    stop: every group against the full oracle, and the launch without debug
    outputs gives the same bytes."""
    W = synth.weight(4096, 4096, seed=0, dtype=torch.float16)
    assert _resident(hq, W, 64)
    prm = _params(4, 64)
    rep, gpu, orc = _run(hq, W, prm)
    if "tensor_tie" not in rep:
        assert np.all(gpu["best_iter"] == orc["best_iter"][0])
    _same(_outputs(hq, W.cuda(), prm, False), _outputs(hq, W.cuda(), prm, True))


@pytest.mark.parametrize("nbits,g,zb", [(4, 64, 16), (2, 32, 8), (8, 128, 16), (1, 16, 8)])
def test_resident_equals_chunked(hq, nbits, g, zb):
    """Both launches solve the same problem; their tensor errors are summed in
    different orders, so they agree unless a decision is a near tie, which the
    oracle's trajectory would show (none at these inputs)."""
    W = synth.weight(1024, 2048, seed=nbits + g, dtype=torch.bfloat16).cuda()
    prm = _params(nbits, g, zb=zb)
    assert _resident(hq, W, g)
    res = _outputs(hq, W, prm, True)
    prev = hq.hqq_set_tensor_resident(0)
    try:
        assert not _resident(hq, W, g)
        chk = _outputs(hq, W, prm, True)
    finally:
        hq.hqq_set_tensor_resident(prev)
    _same(res, chk)


@pytest.mark.parametrize("iters", [1, 11, 20])
def test_chunked_path_still_matches_oracle(hq, chunked, iters):
    W = synth.weight(600, 1024, seed=3, dtype=torch.float16)
    _run(hq, W, _params(4, 64, iters=iters))
    _run(hq, W, _params(2, 16, iters=iters, zb=8))


def test_workspace_passes_between_paths(hq):
    """The chunked launches leave their own words in the workspace header and
    partial rows; a resident call on the same workspace (and the reverse)
    starts from a zeroed header and gives the outputs of a fresh workspace."""
    W = synth.weight(512, 1024, seed=21, dtype=torch.float16).cuda()
    prm = _params(4, 64)
    fresh = _outputs(hq, W, prm, False)
    out = hq.quantize(W, 4, 64, stop_mode=1)
    for resident in (0, 2, 0, 2):
        prev = hq.hqq_set_tensor_resident(resident)
        try:
            out = hq.quantize(W, 4, 64, stop_mode=1, out=out)
            torch.cuda.synchronize()
        finally:
            hq.hqq_set_tensor_resident(prev)
        assert hq.hqq_get_status(out["workspace"]) == hq.HQQ_OK
        _same({k: out[k].view(torch.uint8).cpu() for k in fresh}, fresh)


def test_bounded_wait_times_out(hq):
    """The solver's bounded wait, on a decision that nothing publishes, gives up
    after the limit and leaves HQQ_ERR_TIMEOUT in the workspace's status word;
    the next call on that workspace starts from a zeroed status word."""
    out = hq.quantize(synth.weight(64, 1024, seed=1, dtype=torch.float16).cuda(), 4, 64, stop_mode=1)
    ws = out["workspace"]
    assert hq.hqq_quantize_wait_selftest(ws, ws.numel(), 2000) == hq.HQQ_OK
    assert hq.hqq_get_status(ws) == hq.HQQ_ERR_TIMEOUT
    assert hq.hqq_quantize_wait_selftest(ws, 128, 2000) == hq.HQQ_ERR_INVALID_ARG
    assert hq.hqq_quantize_wait_selftest(ws, ws.numel(), 0) == hq.HQQ_ERR_INVALID_ARG
    out = hq.quantize(synth.weight(64, 1024, seed=1, dtype=torch.float16).cuda(), 4, 64, stop_mode=1, out=out)
    assert hq.hqq_get_status(out["workspace"]) == hq.HQQ_OK
