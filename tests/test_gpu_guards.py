"""No kernel writes outside its output buffers.

compute-sanitizer is not available on this machine, so every device output is
allocated with 256 guard bytes on each side, filled with a pattern, and the
pattern is checked after the call.  Shapes are ragged (partial warp tiles,
last group of a slice, rows not a multiple of the GEMV's rows per warp) and
cover every entry point that writes device memory."""
import numpy as np
import pytest
import torch

from calibration_free_weight_b200 import synth

pytestmark = pytest.mark.gpu
GUARD = 256
PATTERN = 0xA5


@pytest.fixture(scope="module")
def hq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from calibration_free_weight_b200 import hqq
    return hqq


class Guarded:
    """A device buffer of `nbytes` with guard bytes on both sides."""

    def __init__(self, nbytes, dtype=torch.uint8):
        esz = torch.empty(0, dtype=dtype).element_size()
        self.raw = torch.full((nbytes + 2 * GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + nbytes].view(dtype)
        assert nbytes % esz == 0

    def intact(self):
        r = self.raw.cpu().numpy()
        return np.all(r[:GUARD] == PATTERN) and np.all(r[-GUARD:] == PATTERN)


def _quantize_guarded(hq, W, nbits, g, axis, stop, zb):
    rows, cols = W.shape
    G = hq.hqq_num_groups(rows, cols, g, axis)
    bufs = dict(packed=Guarded(hq.hqq_packed_bytes(rows, cols, nbits, g, axis)), scale=Guarded(2 * G, torch.float16),
                zero=Guarded(G * (2 if zb == 16 else 1), torch.float16 if zb == 16 else torch.uint8),
                meta=Guarded(8, torch.float32), bi=Guarded(4 * G, torch.int32), be=Guarded(4 * G, torch.float32),
                zf=Guarded(4 * G, torch.float32))
    wsb = hq.hqq_workspace_bytes(rows, cols, g, axis, stop, zb)
    ws = Guarded(wsb)
    dt = hq.HQQ_F16 if W.dtype == torch.float16 else hq.HQQ_BF16
    for debug in (False, True):
        rc = hq.hqq_quantize(W, rows, cols, dt, nbits, g, axis, 0.7, 1.0, 1.01, 20, stop, zb, bufs["packed"].t,
                             bufs["scale"].t, bufs["zero"].t, bufs["meta"].t if zb == 8 else None, ws.t, wsb,
                             bufs["bi"].t if debug else None, bufs["be"].t if debug else None,
                             bufs["zf"].t if debug else None)
        assert rc == hq.HQQ_OK
        torch.cuda.synchronize()
        assert ws.intact()
        for k, b in bufs.items():
            assert b.intact(), k
    return bufs


@pytest.mark.parametrize("rows,cols,g,axis", [(37, 192, 64, 1), (129, 48, 16, 1), (3, 1024, 1024, 1),
                                               (64, 40, 32, 0), (24, 72, 8, 0), (1001, 64, 64, 1)])
@pytest.mark.parametrize("nbits", [1, 3, 4, 8])
@pytest.mark.parametrize("stop,zb", [(0, 16), (1, 8), (2, 8)])
def test_quantize_writes_stay_inside(hq, rows, cols, g, axis, nbits, stop, zb):
    W = synth.weight(rows, cols, seed=rows + cols + nbits, dtype=torch.bfloat16).cuda()
    _quantize_guarded(hq, W, nbits, g, axis, stop, zb)


@pytest.mark.parametrize("rows,cols,g", [(37, 192, 64), (5, 96, 32), (130, 1024, 16), (41, 128, 8)])
def test_dequant_gemv_scale8_writes_stay_inside(hq, rows, cols, g):
    W = synth.weight(rows, cols, seed=3, dtype=torch.float16).cuda()
    q = hq.quantize(W, 4, g, zero_nbits=8)
    G = rows * cols // g
    out = Guarded(rows * cols * 2, torch.float16)
    assert hq.hqq_dequantize(q["packed"], q["scale"], q["zero"], q["zero_meta"], rows, cols, 4, g, 1, 8, hq.HQQ_F16,
                             out.t) == hq.HQQ_OK
    sq, sm = Guarded(G), Guarded(8 * (-(-G // 7)), torch.float32)
    assert hq.hqq_quantize_scale8(q["scale"], G, 7, sq.t, sm.t) == hq.HQQ_OK
    out8 = Guarded(rows * cols * 2, torch.float16)
    assert hq.hqq_dequantize_s8(q["packed"], sq.t, sm.t, 7, q["zero"], q["zero_meta"], rows, cols, 4, g, 1, 8,
                                hq.HQQ_F16, out8.t) == hq.HQQ_OK
    for batch in (1, 2, 3):
        x = Guarded(batch * cols * 2, torch.float16)
        x.t.copy_(torch.ones(batch * cols, dtype=torch.float16, device="cuda"))
        y = Guarded(batch * rows * 4, torch.float32)
        assert hq.hqq_gemv(q["packed"], q["scale"], q["zero"], q["zero_meta"], rows, cols, 4, g, 8, x.t,
                           hq.HQQ_F16, batch, y.t) == hq.HQQ_OK
        torch.cuda.synchronize()
        assert x.intact() and y.intact()
    torch.cuda.synchronize()
    for b in (out, sq, sm, out8):
        assert b.intact()
