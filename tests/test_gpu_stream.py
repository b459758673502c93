"""hqq_quantize_stream: host-resident matrices streamed through one GPU (two
device slots, copies overlapping the solver).  The same kernels run as in
hqq_quantize, so every output must equal the per-matrix call on
device-resident inputs bit for bit, whatever the order, the shapes mixed in
one list, the host buffers (pinned or pageable) and the list length."""
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


SHAPES = [(4096, 1024), (256, 2048), (1024, 1024), (8, 64), (3000, 512)]


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("nbits,g,zb,stop", [(4, 64, 16, 0), (2, 16, 8, 0), (3, 64, 8, 2)])
@pytest.mark.parametrize("n,pin", [(5, True), (1, True), (4, False)])
def test_stream_equals_per_matrix_calls(hq, dtype, nbits, g, zb, stop, n, pin):
    Ws = [synth.weight(r, c, seed=10 * i + r % 7, dtype=dtype) for i, (r, c) in enumerate(SHAPES[:n])]
    if pin:
        Ws = [w.pin_memory() for w in Ws]
    outs = [hq.host_outputs(*w.shape, nbits, g, zero_nbits=zb, pin=pin) for w in Ws]
    hq.quantize_stream(Ws, outs, nbits, g, stop_mode=stop, zero_nbits=zb)
    for w, o in zip(Ws, outs):
        ref = hq.quantize(w.cuda(), nbits, g, stop_mode=stop, zero_nbits=zb)
        torch.cuda.synchronize()
        for k in ("packed", "scale", "zero", "zero_meta"):
            if o.get(k) is None:
                continue
            assert np.array_equal(o[k].numpy().view(np.uint8), ref[k].cpu().numpy().view(np.uint8)), k


def test_stream_reuses_slots_many_times(hq):
    """Eleven matrices through two slots: each slot is refilled five times."""
    Ws = [synth.weight(512 * (1 + i % 3), 1024, seed=i, dtype=torch.bfloat16).pin_memory() for i in range(11)]
    outs = [hq.host_outputs(*w.shape, 4, 64) for w in Ws]
    buf = hq.quantize_stream(Ws, outs, 4, 64)
    outs2 = [hq.host_outputs(*w.shape, 4, 64) for w in Ws]
    hq.quantize_stream(Ws[::-1], outs2[::-1], 4, 64, device_buffer=buf)  # reversed order, same buffer
    for a, b in zip(outs, outs2):
        for k in ("packed", "scale", "zero"):
            assert torch.equal(a[k], b[k]), k


def test_stream_rejects_small_buffer(hq):
    W = synth.weight(256, 256, seed=1, dtype=torch.float16).pin_memory()
    o = hq.host_outputs(256, 256, 4, 64)
    arr = (hq.hqq_host_matrix * 1)()
    arr[0].W, arr[0].rows, arr[0].cols = W.data_ptr(), 256, 256
    arr[0].W_q_packed, arr[0].scale, arr[0].zero = o["packed"].data_ptr(), o["scale"].data_ptr(), o["zero"].data_ptr()
    need = hq.hqq_stream_device_bytes(arr, 1, 4, 64)
    buf = torch.empty(need, dtype=torch.uint8, device="cuda")
    rc = hq.hqq_quantize_stream(arr, 1, hq.HQQ_F16, 4, 64, 1, 0.7, 1.0, 1.01, 20, 0, 16, buf, need - 256)
    assert rc == hq.HQQ_ERR_WORKSPACE
    rc = hq.hqq_quantize_stream(arr, 1, hq.HQQ_F16, 4, 64, 1, 0.7, 1.0, 1.01, 20, 0, 16, buf, need)
    assert rc == hq.HQQ_OK


MIXED = [  # (rows, cols, settings): per-layer-type configs, both axes, all stop modes, both zero widths
    (1024, 1024, dict(nbits=4, group_size=64, axis=1, stop_mode=0, zero_nbits=16)),
    (2048, 1024, dict(nbits=2, group_size=32, axis=1, stop_mode=1, zero_nbits=16)),
    (1024, 2048, dict(nbits=2, group_size=32, axis=1, stop_mode=1, zero_nbits=8)),
    (512, 768, dict(nbits=3, group_size=64, axis=0, stop_mode=0, zero_nbits=8)),
    (4096, 512, dict(nbits=8, group_size=128, axis=1, stop_mode=2, zero_nbits=16)),
    (256, 4096, dict(nbits=1, group_size=16, axis=1, stop_mode=1, zero_nbits=8)),
    (768, 1024, dict(nbits=4, group_size=64, axis=1, stop_mode=0, zero_nbits=16)),
]


def _mixed(hq, dtype=torch.float16, pin=True):
    Ws = [synth.weight(r, c, seed=31 * i + 5, dtype=dtype) for i, (r, c, _) in enumerate(MIXED)]
    if pin:
        Ws = [w.pin_memory() for w in Ws]
    sets = [st for _, _, st in MIXED]
    outs = [hq.host_outputs(r, c, st["nbits"], st["group_size"], st["axis"], st["zero_nbits"], pin=pin)
            for r, c, st in MIXED]
    return Ws, sets, outs


def _expect(hq, w, st):
    ref = hq.quantize(w.cuda(), st["nbits"], st["group_size"], st["axis"], stop_mode=st["stop_mode"],
                      zero_nbits=st["zero_nbits"])
    torch.cuda.synchronize()
    return ref


def _same(o, ref):
    for k in ("packed", "scale", "zero", "zero_meta"):
        if o.get(k) is None:
            continue
        assert np.array_equal(o[k].numpy().view(np.uint8), ref[k].cpu().numpy().view(np.uint8)), k


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_stream_jobs_per_matrix_settings(hq, dtype):
    """Every matrix with its own settings: each output equals hqq_quantize
    with those settings on the device-resident matrix, bit for bit; the done
    callback comes once per matrix, in order, when that matrix's host outputs
    are already complete."""
    Ws, sets, outs = _mixed(hq, dtype)
    refs = [_expect(hq, w, st) for w, st in zip(Ws, sets)]
    seen = []

    def on_done(i):
        _same(outs[i], refs[i])  # complete when reported
        seen.append(i)

    _, done = hq.quantize_stream_jobs(Ws, sets, outs, on_done=on_done)
    assert seen == list(range(len(MIXED))) and done == len(MIXED)
    for o, ref in zip(outs, refs):
        _same(o, ref)


def test_stream_jobs_resume(hq):
    """A run resumed from the first matrix not yet persisted (a new call with
    the remaining matrices) gives the same outputs as one uninterrupted run
    (pageable host memory here)."""
    Ws, sets, outs = _mixed(hq, torch.bfloat16, pin=False)
    _, done = hq.quantize_stream_jobs(Ws, sets, outs)
    assert done == len(MIXED)
    outs2 = [hq.host_outputs(r, c, st["nbits"], st["group_size"], st["axis"], st["zero_nbits"], pin=False)
             for r, c, st in MIXED]
    buf, done = hq.quantize_stream_jobs(Ws[:3], sets[:3], outs2[:3])
    assert done == 3
    _, done = hq.quantize_stream_jobs(Ws[3:], sets[3:], outs2[3:], device_buffer=buf)
    assert done == len(MIXED) - 3
    for a, b in zip(outs, outs2):
        _same(a, b)


def test_stream_jobs_callback_error_surfaces_after_the_call(hq):
    """An exception in on_done cannot unwind through the C call: every matrix
    is still reported and finished, and the first exception is raised after."""
    Ws, sets, outs = _mixed(hq)
    seen = []

    def on_done(i):
        seen.append(i)
        if i == 2:
            raise KeyError("persist failed")

    with pytest.raises(KeyError):
        hq.quantize_stream_jobs(Ws, sets, outs, on_done=on_done)
    assert seen == list(range(len(MIXED)))
    for w, st, o in zip(Ws, sets, outs):
        _same(o, _expect(hq, w, st))


# ------------------------------------------------- against the oracle ------

from . import parity_check as pc  # noqa: E402


def _np(o):
    return {k: (v.numpy() if v is not None else None) for k, v in o.items() if k in ("packed", "scale", "zero",
                                                                                     "zero_meta")}


def _prm(st):
    return dict(st, p=0.7, beta=1.0, kappa=1.01, iters=20)


def test_stream_jobs_outputs_against_oracle(hq):
    """Per-matrix settings (both axes, every stop rule, both zero widths)
    streamed from host memory: each matrix's stored outputs against the full
    oracle run with that matrix's settings."""
    Ws, sets, outs = _mixed(hq)
    hq.quantize_stream_jobs(Ws, sets, outs)
    for w, st, o in zip(Ws, sets, outs):
        pc.check_stored(w, _prm(st), _np(o))


def test_stream_llama2_13b_mixed_layer_against_oracle(hq):
    """One Llama-2-13B-shaped layer with per-layer-type settings (attention b4
    g64, MLP b2 g32, tensor stop, fp16 zero) streamed through
    quantize_stream_jobs, as the 13B streamed workload runs it: q, gate and
    down against the full oracle (the stop is tensor-wide)."""
    base = dict(nbits=4, group_size=64, stop_mode=1)
    dyn = {"attn": dict(nbits=4, group_size=64, stop_mode=1), "mlp": dict(nbits=2, group_size=32, stop_mode=1)}
    names = {"q": "self_attn.q_proj", "gate": "mlp.gate_proj", "down": "mlp.down_proj"}
    mats = [(n, r, c) for n, r, c in synth.LLAMA2_13B.matrices() if n in names]
    Ws = [synth.weight(r, c, seed=synth.seed_for(3, n), dtype=torch.float16).pin_memory() for n, r, c in mats]
    sets = [hq.settings_for(f"model.layers.3.{names[n]}", base, dyn) for n, _, _ in mats]
    outs = [hq.host_outputs(r, c, st["nbits"], st["group_size"], st["axis"], st["zero_nbits"])
            for (_, r, c), st in zip(mats, sets)]
    _, done = hq.quantize_stream_jobs(Ws, sets, outs)
    assert done == len(mats)
    for w, st, o in zip(Ws, sets, outs):
        pc.check_stored(w, _prm(st), _np(o))


@pytest.mark.parametrize("nbits,g", [(2, 16), (4, 128)])
def test_stream_llama2_70b_shapes_against_oracle(hq, nbits, g):
    """The Llama-2-70B settings (8-bit zero, group stop) streamed from host
    memory on the model's four matrix shapes (q 8192x8192, k 1024x8192, gate
    28672x8192, down 8192x28672; layer 5's seeds): sampled groups of each
    against the oracle."""
    mats = [("q", 8192, 8192), ("k", 1024, 8192), ("gate", 28672, 8192), ("down", 8192, 28672)]
    Ws = [synth.weight(r, c, seed=synth.seed_for(5, n), dtype=torch.float16).pin_memory() for n, r, c in mats]
    st = dict(nbits=nbits, group_size=g, axis=1, stop_mode=0, zero_nbits=8)
    outs = [hq.host_outputs(r, c, nbits, g, zero_nbits=8) for _, r, c in mats]
    _, done = hq.quantize_stream_jobs(Ws, [st] * len(mats), outs)
    assert done == len(mats)
    for i, (w, o) in enumerate(zip(Ws, outs)):
        G = w.numel() // g
        ids = np.unique(np.concatenate([[0, G - 1], np.random.default_rng(i).choice(G, 3000, replace=False)]))
        pc.check_stored(w, _prm(st), _np(o), sample=ids)


def test_stream_jobs_reuse_a_repeated_matrix(hq):
    """Consecutive jobs on the same host matrix (one weight at several
    settings) share one device copy of it; every output still equals the
    per-matrix call with that job's settings, whatever the interleaving."""
    A = synth.weight(2048, 1024, seed=71, dtype=torch.float16).pin_memory()
    B = synth.weight(1024, 2048, seed=72, dtype=torch.float16).pin_memory()
    C = synth.weight(512, 512, seed=73, dtype=torch.float16).pin_memory()
    s1 = dict(nbits=2, group_size=16, axis=1, stop_mode=0, zero_nbits=8)
    s2 = dict(nbits=4, group_size=128, axis=1, stop_mode=0, zero_nbits=8)
    s3 = dict(nbits=3, group_size=64, axis=1, stop_mode=1, zero_nbits=16)
    s4 = dict(nbits=4, group_size=64, axis=0, stop_mode=2, zero_nbits=16)
    order = [(A, s1), (A, s2), (B, s1), (B, s2), (B, s3), (C, s4), (A, s3), (A, s4), (C, s1)]
    Ws = [w for w, _ in order]
    sets = [st for _, st in order]
    outs = [hq.host_outputs(*w.shape, st["nbits"], st["group_size"], st["axis"], st["zero_nbits"]) for w, st in order]
    _, done = hq.quantize_stream_jobs(Ws, sets, outs)
    assert done == len(order)
    for w, st, o in zip(Ws, sets, outs):
        _same(o, _expect(hq, w, st))
