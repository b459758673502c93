"""The solver's fast path skips the proximal step (sub-problem 1) for a whole
group when it can prove that every W_e of the group is zero.  This checks the
two facts that proof rests on, with fp32 arithmetic emulated in numpy and the
oracle's own shrink operator as the judge of "zero":

1. every residual obeys |W - W_r| * s = |r| <= max(0.5, |z - z0|) + slack,
   slack = 1e-3 * (1 + L + |z|), where r = fl(fl(W*s) + z) - W_q;
2. when that bound is below 0.99 * thr * s, thr = beta^(-1/(2-p)) (the
   threshold at and below which the generalised soft-threshold is exactly
   zero), the oracle's shrink of every d = r / s is zero.

Method: techreport.ngo, "Weight-only quantization without the calibration
tax", section "Outlier-aware optimization without gradients" (the proximal
operator of the lp term, p < 1).  Groups are random and adversarial: scales
chosen so that 0.5 / s lands on either side of thr, residuals placed at exact
rounding ties (|r| = 0.5), and zero-points far from z0 so that codes clamp.
"""
import numpy as np
import pytest

F = np.float32
NBITS = [1, 2, 3, 4, 8]


def _scale_zero(w, L):
    mn, mx = F(w.min()), F(w.max())
    s = F(2e4) if not mx > mn else min(F(L) / F(mx - mn), F(2e4))
    return F(s), F(-mn * F(s))


def _residuals(w, s, z, L):
    v = (w * s).astype(F) + F(z)
    q = np.clip(np.rint(v), 0, L).astype(F)
    return (v - q).astype(F)


def _bound(z, z0, L):
    return max(F(0.5), F(abs(F(z - z0)))) + F(1e-3) * (F(1) + F(L) + F(abs(z)))


def _groups(rng, L, thr_list):
    """Random groups at several spreads, and tie-laden groups whose 0.5/s sits
    just below, at and just above each threshold."""
    out = []
    for std in (0.02, 0.3, 1.0, 3.0, 30.0):
        for g in (8, 16, 64):
            w = rng.standard_normal(g) * std
            w[rng.random(g) < 0.05] *= 10
            out.append(w.astype(F))
    for thr in thr_list:
        for f in (0.9, 0.93, 0.95, 0.97, 0.99, 1.0, 1.01, 1.03):
            s_t = 0.5 / (thr * f)
            if not 1e-3 < s_t < 1e4:
                continue
            j = np.arange(max(L, 1), dtype=np.float64)
            w = np.concatenate([[-1.0], -1.0 + (j + 0.5) / s_t, [-1.0 + L / s_t]])
            out.append(w.astype(F))
    return out


@pytest.mark.parametrize("nbits", NBITS)
@pytest.mark.parametrize("p", [0.5, 0.7, 1.0, 1.5])
def test_fast_path_gate(orc, nbits, p):
    rng = np.random.default_rng(100 + nbits)
    L = (1 << nbits) - 1
    betas = []
    for b0, kappa in ((1.0, 1.01), (1.0, 1.5), (0.25, 1.2), (4.0, 1.01)):
        b = F(b0)
        for _ in range(20):
            betas.append(b)
            b = F(b * F(kappa))
    thrs = sorted({float(np.float64(b) ** (-1.0 / (2.0 - p))) for b in betas})
    n_closed = n_checked = n_near = 0
    for w in _groups(rng, L, thrs[::7]):
        s, z0 = _scale_zero(w, L)
        zs = [z0 + F(dz) for dz in (0.0, 0.3, -0.49, 0.5, 1.0, -1.0, 2.5, -7.0, 0.5 * L + 3)]
        for z in zs:
            r = _residuals(w, s, z, L)
            bound = _bound(z, z0, L)
            assert float(np.abs(r).max()) <= bound, (nbits, p, s, z, z0)
            d = (r / s).astype(F)
            for beta in betas[::3]:
                thr = np.float64(beta) ** (-1.0 / (2.0 - p))
                # the kernel's threshold is a hardware approximation: a relative
                # error of 1e-5 either way must not change the decision
                for t in (thr * (1 - 1e-5), thr * (1 + 1e-5)):
                    if bound >= 0.99 * t * s:
                        continue  # gate open: the full proximal step runs
                    n_closed += 1
                    n_near += bound >= 0.9 * 0.99 * t * s
                    for x in d:
                        n_checked += 1
                        assert orc.shrink(float(x), p, float(beta)) == 0.0, (nbits, p, float(x), float(beta))
    # some closed decisions sit within 10 % of the gate's edge
    assert n_closed > 0 and n_checked > 0 and n_near > 0, (n_closed, n_near)


def test_gate_opens_on_tie_groups_at_the_threshold(orc):
    """Residuals of exactly 0.5 with 0.5/s just above thr give a non-zero
    W_e: the gate must be open for them (the bound's 0.5 term)."""
    p, beta, L = 0.7, F(1.0), 15
    thr = 1.0
    s_t = 0.5 / (thr * 1.05)
    j = np.arange(L, dtype=np.float64)
    w = np.concatenate([[-1.0], -1.0 + (j + 0.5) / s_t, [-1.0 + L / s_t]]).astype(F)
    s, z0 = _scale_zero(w, L)
    r = _residuals(w, s, z0, L)
    d = (r / s).astype(F)
    assert any(orc.shrink(float(x), p, float(beta)) != 0.0 for x in d)
    assert _bound(z0, z0, L) >= 0.99 * thr * s
