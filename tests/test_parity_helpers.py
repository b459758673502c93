"""The stored-output parity checker (used on streamed runs, which return no
debug outputs) accepts the oracle's own outputs and rejects planted mistakes:
one code moved by two levels, a zero off by a level, a swapped scale.  CPU only."""
import numpy as np
import pytest
import torch

import oracle
from calibration_free_weight_b200 import synth

from . import parity_check as pc


def _prm(nbits, g, stop, zb, axis=1):
    return dict(nbits=nbits, group_size=g, axis=axis, p=0.7, beta=1.0, kappa=1.01, iters=20, stop_mode=stop,
                zero_nbits=zb)


@pytest.mark.parametrize("nbits,g,stop,zb,axis", [(4, 64, 0, 16, 1), (2, 16, 0, 8, 1), (3, 64, 1, 16, 1),
                                                   (2, 32, 1, 8, 1), (4, 32, 2, 16, 0)])
def test_checker_accepts_oracle_and_rejects_mistakes(nbits, g, stop, zb, axis):
    W = synth.weight(256, 512, seed=nbits + g, dtype=torch.float16)
    Wo, dt = pc.w_for_oracle(W)
    prm = _prm(nbits, g, stop, zb, axis)
    orc = oracle.quantize(Wo, nbits, g, axis, 0.7, 1.0, 1.01, 20, stop, zb, dtype=dt)
    out = {k: orc[k] for k in ("packed", "scale", "zero", "zero_meta")}
    rep = pc.check_stored(W, prm, out, orc)
    assert rep.get("tie_groups", 0) == 0
    if stop != 1:
        pc.check_stored(W, prm, out, sample=np.array([0, 5, 17, 256 * 512 // g - 1]))
    rows, cols = W.shape
    L = (1 << nbits) - 1
    lv = oracle.unpack_levels(orc["packed"], rows, cols, nbits, axis)
    bad = lv.copy()
    bad[3, 7] = (bad[3, 7] + 2) % (L + 1) if L >= 2 else 1 - bad[3, 7]
    if L >= 2:
        with pytest.raises(AssertionError):
            pc.check_stored(W, prm, dict(out, packed=oracle.pack_levels(bad, nbits, axis)), orc)
    z2 = orc["zero"].copy()
    z2[9] = z2[9] + (np.float16(1.0) if zb == 16 else np.uint8(40))
    with pytest.raises(AssertionError):
        pc.check_stored(W, prm, dict(out, zero=z2), orc)
    s2 = orc["scale"].copy()
    s2[[2, 3]] = s2[[3, 2]] * np.float16(1.5)
    with pytest.raises(AssertionError):
        pc.check_stored(W, prm, dict(out, scale=s2), orc)
