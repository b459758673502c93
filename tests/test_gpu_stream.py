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
