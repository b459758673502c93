"""Pins of the CPU oracle to facts fixed outside the oracle itself.

Each test checks the oracle against a hand value, a closed form, an
invariant, a special case that reduces to a textbook rule, or brute force on
a tiny input -- chosen so that a dropped term, a flipped sign, a wrong index
or a transposed operand in the oracle fails at least one of them.

Method source: techreport.ngo, "Weight-only quantization without the
calibration tax" (Half-Quadratic Quantization of Large Machine Learning
Models), sections "Outlier-aware optimization without gradients" and
"Benchmark results" / "Llama-2".
"""
import math
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
NBITS = [1, 2, 3, 4, 8]


def _rng(seed):
    return np.random.default_rng(seed)


def _synth_f16(rows, cols, seed, std=0.02):
    r = _rng(seed)
    w = r.standard_normal((rows, cols)) * std
    m = r.random((rows, cols)) < 1e-2
    w = np.where(m, w * 10, w)
    return w.astype(np.float16)


def _lp_err(w, q, s, z, p):
    """mean |w - (q - z)/s|^p in fp64 (the error measure the stop rule uses)."""
    w = np.asarray(w, np.float64)
    wr = (np.asarray(q, np.float64) - float(z)) / float(s)
    return float(np.mean(np.abs(w - wr) ** p))


# ---------------------------------------------------------------- shrink ----

def _shrink_rows():
    rows = []
    with open(os.path.join(GOLDEN, "shrink_hand_values.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                x, p, b, ex = (float(t) for t in line.split())
                rows.append((x, p, b, ex))
    return rows


@pytest.mark.parametrize("x,p,beta,expected", _shrink_rows())
def test_shrink_hand_values(orc, x, p, beta, expected):
    got = orc.shrink(x, p, beta)
    assert got == pytest.approx(expected, rel=2e-6, abs=1e-7)


def test_shrink_p1_is_soft_threshold(orc):
    xs = _rng(1).standard_normal(2000) * 3
    for beta in (0.5, 1.0, 2.0, 7.0):
        for x in xs:
            x = float(np.float32(x))
            expect = math.copysign(max(abs(x) - 1.0 / beta, 0.0), x)
            assert orc.shrink(x, 1.0, beta) == pytest.approx(expect, abs=2e-6)


@pytest.mark.parametrize("p", [0.3, 0.7, 1.0, 1.4])
@pytest.mark.parametrize("beta", [0.5, 1.0, 1.01 ** 19, 4.0])
def test_shrink_zero_iff_below_threshold(orc, p, beta):
    thr = beta ** (-1.0 / (2.0 - p))
    for a in np.concatenate([np.linspace(0, 3 * thr, 301), thr * (1 + np.array([-1e-3, 1e-3]))]):
        a = float(a)
        for x in (a, -a):
            got = orc.shrink(x, p, beta)
            if a < thr * (1 - 1e-4):
                assert got == 0.0
            elif a > thr * (1 + 1e-4):
                assert got != 0.0 and math.copysign(1, got) == math.copysign(1, x) and abs(got) < a


def test_shrink_zero_input_is_zero_even_without_threshold(orc):
    # |0|^(p-1) is infinite for p < 1 and 1/beta can be 0: shrink(0) must stay 0 (no NaN).
    assert orc.shrink(0.0, 0.7, 1e30) == 0.0
    assert orc.shrink(-0.0, 0.7, 1.0) == 0.0


# ------------------------------------------------------------ worked groups --

def _worked_rows():
    rows = []
    with open(os.path.join(GOLDEN, "worked_groups.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            cols = [c.strip() for c in line.split("|")]
            rid = cols[0]
            nb, p, beta, kappa = cols[1].split()
            vals = np.array([float(t) for t in cols[2].split()], np.float32)
            ev = lambda s: float(eval(s, {"__builtins__": {}}))  # closed-form expressions
            rows.append(dict(id=rid, nbits=int(nb), p=float(p), beta=float(beta), kappa=float(kappa), w=vals,
                             s=ev(cols[3]), z0=ev(cols[4]), codes=[int(t) for t in cols[5].split()],
                             e0=ev(cols[6]), z1=ev(cols[7]), e1=ev(cols[8]), best_iter=int(cols[9]),
                             zbest=ev(cols[10])))
    return rows


@pytest.mark.parametrize("row", _worked_rows(), ids=lambda r: r["id"])
def test_worked_groups(orc, row):
    s, z, e, b = orc.trace_group(row["w"], row["nbits"], row["p"], row["beta"], row["kappa"], iters=4)
    assert s == row["s"]
    assert z[0] == row["z0"]
    assert list(orc.group_codes(row["w"], row["nbits"], s, z[0])) == row["codes"]
    assert e[0] == pytest.approx(row["e0"], rel=1e-6, abs=1e-12)
    assert z[1] == pytest.approx(row["z1"], rel=1e-7, abs=1e-9)
    assert e[1] == pytest.approx(row["e1"], rel=1e-6, abs=1e-12)
    # group mode through the full quantiser: kept iterate and zero-point
    W = row["w"].astype(np.float16).reshape(1, -1)
    assert np.array_equal(W.astype(np.float32), row["w"].reshape(1, -1))
    out = orc.quantize(W, row["nbits"], W.shape[1], axis=1, p=row["p"], beta=row["beta"], kappa=row["kappa"],
                       iters=20)
    assert out["best_iter"][0] == row["best_iter"]
    assert out["zero_f32"][0] == pytest.approx(row["zbest"], abs=1e-9)


# ------------------------------------------------------------------ packing --

@pytest.mark.parametrize("nbits", NBITS)
@pytest.mark.parametrize("axis", [0, 1])
def test_pack_roundtrip_exhaustive(orc, nbits, axis):
    """Every level at every bit phase survives pack -> unpack; the byte layout is
    the documented LSB-first stream (checked with numpy's own bit unpacking)."""
    L = (1 << nbits) - 1
    rows, cols = 8 * 3, 2 * (L + 1) if axis == 1 else 8
    if axis == 0:
        rows, cols = 8 * (L + 1), 3
    r = _rng(nbits * 10 + axis)
    levels = r.integers(0, L + 1, (rows, cols)).astype(np.uint8)
    # make sure every level appears at every position modulo 8 along the stream
    along = levels.reshape(-1) if axis == 1 else levels.T.reshape(-1)
    along[: 8 * (L + 1)] = np.repeat(np.arange(L + 1), 8)[: along[: 8 * (L + 1)].size]
    levels = along.reshape(rows, cols) if axis == 1 else along.reshape(cols, rows).T.copy()
    packed = orc.pack_levels(levels, nbits, axis)
    assert packed.size == rows * cols * nbits // 8
    assert np.array_equal(orc.unpack_levels(packed, rows, cols, nbits, axis), levels)
    # independent bit reader: numpy unpackbits, little bit order
    if axis == 1:
        bits = np.unpackbits(packed, bitorder="little").reshape(-1, nbits)
        got = (bits * (1 << np.arange(nbits))).sum(1).reshape(rows, cols)
    else:
        colstreams = packed.reshape(rows * nbits // 8, cols).T  # [cols, bytes]
        bits = np.unpackbits(np.ascontiguousarray(colstreams), axis=1, bitorder="little")
        got = (bits.reshape(cols, rows, nbits) * (1 << np.arange(nbits))).sum(2).T
    assert np.array_equal(got, levels)


# ---------------------------------------------------- init / RTN properties --

@pytest.mark.parametrize("nbits", NBITS)
@pytest.mark.parametrize("g", [8, 64])
def test_rtn_properties(orc, nbits, g):
    """iters = 0 is plain min/max round-to-nearest: each group's min maps to code
    0, its max to L, and every element is reconstructed within half a step."""
    W = _synth_f16(16, 256, seed=nbits + g)
    out = orc.quantize(W, nbits, g, axis=1, iters=0)
    L = (1 << nbits) - 1
    levels = orc.unpack_levels(out["packed"], 16, 256, nbits, 1).reshape(-1, g)
    wg = W.astype(np.float64).reshape(-1, g)
    for j in range(wg.shape[0]):
        lo, hi = wg[j].argmin(), wg[j].argmax()
        assert levels[j, lo] == 0
        if L / (wg[j, hi] - wg[j, lo]) < 2e4 * (1 - 1e-6):  # scale cap (R1) not active
            assert levels[j, hi] == L
        else:
            assert levels[j, hi] == round(float(np.float32(wg[j, hi] - wg[j, lo]) * np.float32(2e4)))
    deq = orc.dequantize(out["packed"], out["scale"], out["zero"], None, 16, 256, nbits, g).astype(np.float64)
    scale = out["scale"].astype(np.float64)[:, None]
    z = out["zero"].astype(np.float64)[:, None]
    err = np.abs(deq.reshape(-1, g) - wg)
    # half a quantisation step, plus fp16 storage of scale, zero and the output
    bound = scale * (0.5 + 1e-3 * (np.abs(z) + L)) + np.abs(wg) * 2.0 ** -10 + 1e-7
    assert np.all(err <= bound)


@pytest.mark.parametrize("nbits", NBITS)
def test_one_iteration_equals_rtn(orc, nbits):
    W = _synth_f16(32, 128, seed=7 + nbits)
    a = orc.quantize(W, nbits, 32, iters=0)
    b = orc.quantize(W, nbits, 32, iters=1)
    for k in ("packed", "scale", "zero", "zero_f32"):
        assert np.array_equal(a[k], b[k]), k
    assert np.all(b["best_iter"] == 0)


@pytest.mark.parametrize("nbits", [2, 4])
def test_huge_beta_keeps_z0(orc, nbits):
    """beta -> inf makes W_e = W - W_r, so z = mean(W_q - W_r*s) = z: z stays at
    z0 (within fp32 rounding) and the codes equal round-to-nearest."""
    W = _synth_f16(16, 256, seed=11)
    rtn = orc.quantize(W, nbits, 64, iters=0)
    out = orc.quantize(W, nbits, 64, beta=1e30, iters=20, stop_mode=orc.STOP_NONE)
    z0, zb = rtn["zero_f32"], out["zero_f32"]
    assert np.all(np.abs(zb - z0) <= 1e-5 * np.maximum(np.abs(z0), 1))
    la = orc.unpack_levels(rtn["packed"], 16, 256, nbits, 1)
    lb = orc.unpack_levels(out["packed"], 16, 256, nbits, 1)
    assert np.mean(la != lb) <= 1e-3


@pytest.mark.parametrize("c", [0.0, 0.015625, -0.75, 1e-4])
@pytest.mark.parametrize("nbits", [1, 4, 8])
def test_constant_group_fixed_point(orc, c, nbits):
    """A constant group: codes 0, z = -c*s, zero error, and the second evaluation
    repeats the first so the solver stops with best_iter 0."""
    W = np.full((2, 64), c, np.float16)
    out = orc.quantize(W, nbits, 64, iters=20)
    cf = float(np.float16(c))
    assert np.all(orc.unpack_levels(out["packed"], 2, 64, nbits, 1) == 0)
    s = np.float32(2e4)
    assert np.all(out["zero_f32"] == np.float32(-np.float32(cf) * s))
    assert np.all(out["best_iter"] == 0)
    assert np.all(out["best_err"] <= 1e-6)


# ------------------------------------------------- the stop rule and best z --

@pytest.mark.parametrize("nbits,g", [(1, 8), (2, 8), (2, 16), (3, 8), (4, 16)])
def test_kept_error_between_optimum_and_rtn(orc, nbits, g):
    """Brute force on tiny groups: the kept zero-point's lp error is no worse than
    round-to-nearest (iterate 0) and no better than the best z on a fine scan."""
    r = _rng(100 + nbits * g)
    for t in range(40):
        w = (r.standard_normal(g) * 0.02).astype(np.float16)
        if t % 4 == 0:
            w[r.integers(g)] *= 10  # an outlier
        W = w.reshape(1, g)
        out = orc.quantize(W, nbits, g, iters=20)
        rtn = orc.quantize(W, nbits, g, iters=0)
        w32 = w.astype(np.float32)
        s, z, e, _ = orc.trace_group(w32, nbits, iters=1)
        lv = orc.unpack_levels(out["packed"], 1, g, nbits, 1)[0]
        lv0 = orc.unpack_levels(rtn["packed"], 1, g, nbits, 1)[0]
        e_kept = _lp_err(w32, lv, s, out["zero_f32"][0], 0.7)
        e_rtn = _lp_err(w32, lv0, s, rtn["zero_f32"][0], 0.7)
        assert e_kept <= e_rtn * (1 + 1e-9) + 1e-15
        # Exact global minimum over z: between code changes each term |.|^p is
        # concave in z, so the minimum sits at a kink (some d_i = 0, z = k - w_i s)
        # or next to a code change (z = k + 1/2 - w_i s); evaluate all of them.
        L = (1 << nbits) - 1
        ws = w32.astype(np.float64) * s
        k = np.arange(L + 1, dtype=np.float64)
        kinks = (k[:, None] - ws[None, :]).ravel()
        brk = (k[:, None] + 0.5 - ws[None, :]).ravel()
        zs = np.concatenate([kinks, brk - 1e-9, brk + 1e-9, np.linspace(-L - 1, 2 * L + 1, 2001)])
        q = np.clip(np.rint(ws[None, :] + zs[:, None]), 0, L)
        e_scan = np.mean(np.abs(w32[None, :] - (q - zs[:, None]) / s) ** 0.7, axis=1).min()
        assert e_kept >= e_scan * (1 - 1e-6)


def test_group_mode_stops_at_first_rise(orc):
    """The kept iterate is the last one before the first non-improvement."""
    W = _synth_f16(64, 256, seed=5)
    out = orc.quantize(W, 4, 64, iters=20)
    wg = W.astype(np.float32).reshape(-1, 64)
    for j in range(wg.shape[0]):
        s, z, e, _ = orc.trace_group(wg[j], 4, iters=20)
        k = 0
        while k + 1 < 20 and e[k + 1] < e[k]:
            k += 1
        assert out["best_iter"][j] == k
        assert out["zero_f32"][j] == z[k]
        assert out["best_err"][j] == np.float32(e[k])


def test_no_stop_mode_keeps_global_best(orc):
    W = _synth_f16(32, 128, seed=6)
    out = orc.quantize(W, 3, 64, iters=20, stop_mode=orc.STOP_NONE)
    grp = orc.quantize(W, 3, 64, iters=20)
    wg = W.astype(np.float32).reshape(-1, 64)
    for j in range(wg.shape[0]):
        s, z, e, _ = orc.trace_group(wg[j], 3, iters=20)
        k = int(np.argmin(e))  # first occurrence of the minimum
        assert out["best_iter"][j] == k and out["zero_f32"][j] == z[k]
        assert out["best_err"][j] <= grp["best_err"][j]


def test_beta_schedule(orc):
    w = _synth_f16(1, 64, seed=9).astype(np.float32)[0]
    _, _, _, b = orc.trace_group(w, 4, beta=1.0, kappa=1.01, iters=20)
    assert b[0] == 1.0
    assert np.allclose(b, 1.01 ** np.arange(20), rtol=1e-6)
    _, _, _, b2 = orc.trace_group(w, 4, beta=2.0, kappa=1.0, iters=5)
    assert np.all(b2 == 2.0)


def test_beta_schedule_changes_shrink_path(orc):
    """Wide groups (|W - W_r| > 1) make the shrink active, so kappa matters."""
    w = (_rng(3).standard_normal(64) * 40).astype(np.float32)
    _, za, _, _ = orc.trace_group(w, 1, kappa=1.0, iters=6)
    _, zb, _, _ = orc.trace_group(w, 1, kappa=1.5, iters=6)
    assert za[1] == zb[1]  # first update uses beta0 in both
    assert not np.allclose(za[2:], zb[2:])


# ------------------------------------------------------ the z update (LS) --

@pytest.mark.parametrize("beta", [1.0, 50.0])
def test_z_update_is_least_squares_minimiser(orc, beta):
    """Sub-problem 2: the average minimises sum (W_q - (W - W_e)*s - z)^2."""
    r = _rng(21)
    for _ in range(20):
        w = (r.standard_normal(32) * 3).astype(np.float32)
        s = np.float32(1.5)
        q = np.clip(np.rint(w * s + 4), 0, 15).astype(np.float32)
        d = (w - (q - 4) / s).astype(np.float32)
        z = orc.update_zero(w, q, d, s, 0.7, beta)
        we = np.array([orc.shrink(float(x), 0.7, beta) for x in d], np.float64)
        t = q.astype(np.float64) - (w.astype(np.float64) - we) * float(s)
        zs = np.linspace(t.min(), t.max(), 200001)
        obj = ((t[None, :] - zs[:, None]) ** 2).sum(1)
        zbf = zs[obj.argmin()]
        assert abs(z - zbf) <= (t.max() - t.min()) / 200000 + 1e-5
        if beta > 1:  # threshold beta^(-1/(2-p)) < 0.05 here: the shrink is active and must move z
            assert abs(z - np.mean(q - w * s)) > 1e-3


# ------------------------------------------------------------- invariances --

def test_translation_equivariance(orc):
    """Adding c to a group leaves the codes and the error unchanged and shifts z
    by -c*s (exactly representable shifts; fp32 rounding only)."""
    r = _rng(31)
    base = np.round(r.standard_normal((8, 64)) * 64) / 1024  # multiples of 2^-10
    for c in (0.25, -0.5, 0.125):
        W0, W1 = base.astype(np.float16), (base + c).astype(np.float16)
        assert np.array_equal(W1.astype(np.float64) - W0.astype(np.float64), np.full(base.shape, c))
        a, b = orc.quantize(W0, 4, 64), orc.quantize(W1, 4, 64)
        la = orc.unpack_levels(a["packed"], 8, 64, 4, 1)
        lb = orc.unpack_levels(b["packed"], 8, 64, 4, 1)
        assert np.mean(la != lb) <= 2 / la.size
        s = 1.0 / a["scale"].astype(np.float64)
        assert np.allclose(b["zero_f32"], a["zero_f32"] - c * s, rtol=2e-3, atol=2e-3)
        assert np.allclose(a["best_err"], b["best_err"], rtol=1e-3)


def test_permutation_within_group(orc):
    W = _synth_f16(4, 64, seed=41)
    perm = _rng(4).permutation(64)
    a, b = orc.quantize(W, 3, 64), orc.quantize(W[:, perm], 3, 64)
    la = orc.unpack_levels(a["packed"], 4, 64, 3, 1)
    lb = orc.unpack_levels(b["packed"], 4, 64, 3, 1)
    assert np.array_equal(la[:, perm], lb)
    assert np.array_equal(a["best_iter"], b["best_iter"])
    assert np.allclose(a["zero_f32"], b["zero_f32"], rtol=1e-6)


def test_groups_are_independent(orc):
    W = _synth_f16(16, 128, seed=42)
    perm = _rng(5).permutation(16)
    a, b = orc.quantize(W, 2, 32), orc.quantize(W[perm], 2, 32)
    ga = a["zero_f32"].reshape(16, 4)[perm]
    assert np.array_equal(ga, b["zero_f32"].reshape(16, 4))
    la = orc.unpack_levels(a["packed"], 16, 128, 2, 1)[perm]
    assert np.array_equal(la, orc.unpack_levels(b["packed"], 16, 128, 2, 1))


@pytest.mark.parametrize("nbits", [3, 4])
def test_axis0_is_axis1_of_transpose(orc, nbits):
    W = _synth_f16(128, 48, seed=43)
    a = orc.quantize(W, nbits, 32, axis=0)
    b = orc.quantize(np.ascontiguousarray(W.T), nbits, 32, axis=1)
    # scale/zero: axis 0 is [rows/g, cols]; axis 1 of W^T is [cols, rows/g]
    assert np.array_equal(a["zero_f32"].reshape(4, 48), b["zero_f32"].reshape(48, 4).T)
    assert np.array_equal(a["scale"].reshape(4, 48), b["scale"].reshape(48, 4).T)
    la = orc.unpack_levels(a["packed"], 128, 48, nbits, 0)
    lb = orc.unpack_levels(b["packed"], 48, 128, nbits, 1)
    assert np.array_equal(la, lb.T)
    # packed axis-0 bytes are the transpose of the axis-1 bytes of W^T
    assert np.array_equal(a["packed"].reshape(128 * nbits // 8, 48), b["packed"].reshape(48, 128 * nbits // 8).T)


def test_bf16_and_f16_agree_on_shared_values(orc):
    r = _rng(44)
    vals = np.clip(np.round(r.standard_normal((8, 64)) * 64), -255, 255) / 4096  # <= 8 significant bits: exact in both
    f16 = vals.astype(np.float16)
    bf = (vals.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(f16.astype(np.float32), (bf.astype(np.uint32) << 16).view(np.float32))
    a = orc.quantize(f16, 4, 64)
    b = orc.quantize(bf, 4, 64, dtype=orc.BF16)
    for k in ("packed", "scale", "zero", "zero_f32", "best_iter"):
        assert np.array_equal(a[k], b[k]), k


# ------------------------------------------------------------- tensor mode --

def test_tensor_mode_single_group_equals_group_mode(orc):
    for seed in range(6):
        W = _synth_f16(1, 64, seed=50 + seed)
        a = orc.quantize(W, 3, 64, stop_mode=orc.STOP_GROUP)
        b = orc.quantize(W, 3, 64, stop_mode=orc.STOP_TENSOR)
        for k in ("packed", "zero_f32", "best_iter"):
            assert np.array_equal(a[k], b[k]), k


def test_tensor_mode_identical_groups_equals_group_mode(orc):
    row = _synth_f16(1, 64, seed=60)
    W = np.repeat(row, 8, axis=0)
    a = orc.quantize(W, 4, 64, stop_mode=orc.STOP_GROUP)
    b = orc.quantize(W, 4, 64, stop_mode=orc.STOP_TENSOR)
    assert np.array_equal(a["zero_f32"], b["zero_f32"])
    assert np.array_equal(a["best_iter"], b["best_iter"])


def test_tensor_mode_uses_tensor_mean(orc):
    """The tensor stop follows the mean of all per-group errors."""
    W = _synth_f16(16, 256, seed=61)
    out = orc.quantize(W, 2, 16, stop_mode=orc.STOP_TENSOR, iters=20)
    wg = W.astype(np.float32).reshape(-1, 16)
    traces = [orc.trace_group(wg[j], 2, iters=20) for j in range(wg.shape[0])]
    E = np.mean([t[2] for t in traces], axis=0)
    k = 0
    while k + 1 < 20 and E[k + 1] < E[k]:
        k += 1
    assert np.all(out["best_iter"] == k)
    assert np.array_equal(out["zero_f32"], np.array([t[1][k] for t in traces], np.float32))


# ------------------------------------------------------------- zero 8-bit --

@pytest.mark.parametrize("nbits", [2, 4])
def test_zero_8bit_roundtrip(orc, nbits):
    W = _synth_f16(64, 256, seed=70)
    out = orc.quantize(W, nbits, 64, zero_nbits=8)
    z = out["zero_f32"].astype(np.float64)
    inv_sz, zz = out["zero_meta"].astype(np.float64)
    zdeq = (out["zero"].astype(np.float64) - zz) * inv_sz
    span = z.max() - z.min()
    assert out["zero"].min() == 0 and out["zero"].max() == 255
    assert np.all(np.abs(zdeq - z) <= span / 510 * (1 + 1e-5) + 1e-6 * np.abs(z).max())
    # the codes are those of the fp32 zero-point (zero quantisation does not re-solve W_q)
    ref = orc.quantize(W, nbits, 64, zero_nbits=16)
    assert np.array_equal(ref["packed"], out["packed"])


def test_zero_8bit_all_equal(orc):
    W = np.repeat(_synth_f16(1, 64, seed=71), 4, axis=0)
    out = orc.quantize(W, 4, 64, zero_nbits=8)
    inv_sz, zz = out["zero_meta"].astype(np.float64)
    zdeq = (out["zero"].astype(np.float64) - zz) * inv_sz
    assert np.all(out["zero"] == 0)
    assert np.allclose(zdeq, out["zero_f32"], rtol=1e-6)


def test_dequant_with_8bit_zero_close_to_16bit(orc):
    W = _synth_f16(32, 256, seed=72)
    a = orc.quantize(W, 4, 64, zero_nbits=16)
    b = orc.quantize(W, 4, 64, zero_nbits=8)
    da = orc.dequantize(a["packed"], a["scale"], a["zero"], None, 32, 256, 4, 64).astype(np.float64)
    db = orc.dequantize(b["packed"], b["scale"], b["zero"], b["zero_meta"], 32, 256, 4, 64,
                        zero_nbits=8).astype(np.float64)
    span = a["zero_f32"].max() - a["zero_f32"].min()
    step = np.repeat(a["scale"].astype(np.float64), 64).reshape(32, 256)
    assert np.all(np.abs(da - db) <= step * (span / 510 + 0.01) + 1e-6)


def test_dequant_bf16_output(orc):
    W = _synth_f16(8, 64, seed=73)
    a = orc.quantize(W, 4, 64)
    h = orc.dequantize(a["packed"], a["scale"], a["zero"], None, 8, 64, 4, 64, out_dtype=orc.F16)
    b = orc.dequantize(a["packed"], a["scale"], a["zero"], None, 8, 64, 4, 64, out_dtype=orc.BF16)
    bf = (b.astype(np.uint32) << 16).view(np.float32)
    assert np.allclose(bf, h.astype(np.float32), rtol=2 ** -8, atol=1e-6)


# ------------------------------------------- 8-bit scales ("_s*" variant) ---

def _scale8_rows():
    rows = []
    for line in open(os.path.join(GOLDEN, "scale8_hand_values.txt")):
        if line.startswith("#") or not line.strip():
            continue
        S, scales, codes, meta = [f.strip() for f in line.split("|")]
        rows.append((int(S), [float(x) for x in scales.split()], [int(x) for x in codes.split()],
                     [tuple(float(v) for v in m.split(",")) for m in meta.split(";")]))
    return rows


@pytest.mark.parametrize("row", _scale8_rows())
def test_scale8_hand_values(orc, row):
    S, scales, codes, meta = row
    c, m = orc.quantize_scale8(np.array(scales, np.float16), S)
    assert c.tolist() == codes
    assert np.allclose(m, np.array(meta, np.float32), rtol=1e-7, atol=0)


@pytest.mark.parametrize("G,S", [(1000, 128), (128, 128), (129, 128), (5, 128), (300, 7)])
def test_scale8_roundtrip_bound_and_extremes(orc, G, S):
    rng = np.random.default_rng(G + S)
    sc = (np.abs(rng.normal(0.004, 0.002, G)) + 1e-4).astype(np.float16)
    c, m = orc.quantize_scale8(sc, S)
    assert m.shape == (-(-G // S), 2)
    v = sc.astype(np.float32)
    for k in range(m.shape[0]):
        run = slice(k * S, min(G, (k + 1) * S))
        x, q = v[run], c[run]
        rebuilt = (q.astype(np.float32) - m[k, 1]) * m[k, 0]
        span = float(x.max() - x.min())
        # round to nearest: within half a step of 255 levels over the run's range
        assert np.all(np.abs(rebuilt - x) <= span / 510 * (1 + 1e-5) + 1e-9)
        if span > 0:
            assert q[np.argmin(x)] == 0 and q[np.argmax(x)] == 255
        else:
            assert np.all(q == 0) and np.all(rebuilt == x)


def test_scale8_runs_are_independent(orc):
    rng = np.random.default_rng(3)
    sc = (np.abs(rng.normal(0.004, 0.002, 512)) + 1e-4).astype(np.float16)
    c0, m0 = orc.quantize_scale8(sc, 128)
    sc2 = sc.copy()
    sc2[128:256] *= np.float16(3)  # only run 1 changes
    c1, m1 = orc.quantize_scale8(sc2, 128)
    for k in (0, 2, 3):
        assert np.array_equal(c0[k * 128:(k + 1) * 128], c1[k * 128:(k + 1) * 128]) and np.array_equal(m0[k], m1[k])
    assert not np.array_equal(m0[1], m1[1])


def test_dequant_with_8bit_scale(orc):
    """dequantize_s8 rebuilds each group's scale from its code and run pair, and
    otherwise equals dequantize with those rebuilt scales stored in fp16
    wherever the rebuilt scale is exact in fp16."""
    W = (np.random.default_rng(4).normal(0, 0.02, (64, 256))).astype(np.float16)
    o = orc.quantize(W, 4, 32, 1, 0.7, 1.0, 1.01, 20, orc.STOP_GROUP, 16)
    c, m = orc.quantize_scale8(o["scale"], 16)
    d8 = orc.dequantize_s8(o["packed"], c, m, 16, o["zero"], None, 64, 256, 4, 32)
    rebuilt = np.array([(np.float32(c[j]) - m[j // 16, 1]) * m[j // 16, 0] for j in range(c.size)], np.float32)
    # a worked element: group 0, element 0
    q = orc.unpack_levels(o["packed"], 64, 256, 4, 1).reshape(64, 256)
    v = np.float32(np.float32(q[0, 0]) - np.float32(o["zero"][0])) * rebuilt[0]
    assert d8[0, 0] == np.float16(v)
    # close to the fp16-scale dequantisation: the scale moved by at most half a step of its run
    d16 = orc.dequantize(o["packed"], o["scale"], o["zero"], None, 64, 256, 4, 32).astype(np.float32)
    assert np.max(np.abs(d8.astype(np.float32) - d16)) < 0.02 * np.abs(d16).max()


# ------------------------------------- fused dequantise + matrix-vector ---

def _gemv_case():
    d = {}
    for line in open(os.path.join(GOLDEN, "gemv_hand_values.txt")):
        if line.startswith("#") or not line.strip():
            continue
        k, *v = line.split()
        d[k] = v
    return d


def test_gemv_hand_values(orc):
    d = _gemv_case()
    rows, cols, nb, g = (int(d[k][0]) for k in ("rows", "cols", "nbits", "group"))
    lv = np.array([int(v) for v in d["levels"]], np.uint8).reshape(rows, cols)
    packed = np.zeros(rows * cols * nb // 8, np.uint8)
    orc.lib().oracle_pack_levels(lv.ctypes.data, rows, cols, nb, 1, packed.ctypes.data)
    sc = np.array([float(v) for v in d["scale"]], np.float16)
    z = np.array([float(v) for v in d["zero"]], np.float16)
    x = np.array([float(v) for v in d["x"]], np.float16)
    y = orc.gemv(packed, sc, z, None, rows, cols, nb, g, 16, x)
    assert y[0].tolist() == [float(v) for v in d["y"]]


@pytest.mark.parametrize("nbits,g,zb", [(4, 64, 16), (2, 16, 8), (3, 32, 16), (8, 128, 8), (1, 8, 16)])
def test_gemv_unit_vectors_give_dequantised_columns(orc, nbits, g, zb):
    W = _synth_f16(24, 256, seed=nbits + g)
    o = orc.quantize(W, nbits, g, 1, 0.7, 1.0, 1.01, 20, orc.STOP_GROUP, zb)
    deq = orc.dequantize(o["packed"], o["scale"], o["zero"], o["zero_meta"], 24, 256, nbits, g, 1, zb)
    cols = [0, 1, g - 1, g, 255]
    X = np.zeros((len(cols), 256), np.float16)
    for i, c in enumerate(cols):
        X[i, c] = 1.0
    Y = orc.gemv(o["packed"], o["scale"], o["zero"], o["zero_meta"], 24, 256, nbits, g, zb, X)
    for i, c in enumerate(cols):
        # the fp32 W_r of column c, rounded to fp16, is the dequantiser's output
        assert np.array_equal(Y[i].astype(np.float32).astype(np.float16), deq[:, c])


def test_gemv_is_linear_and_batched(orc):
    W = _synth_f16(40, 512, seed=11)
    o = orc.quantize(W, 4, 64, 1, 0.7, 1.0, 1.01, 20, orc.STOP_GROUP, 16)
    r = np.random.default_rng(5)
    # multiples of 1/8 below 2: sums exact in fp16, values exact in bf16
    x1 = (r.integers(-8, 8, 512) / 8).astype(np.float16)
    x2 = (r.integers(-8, 8, 512) / 8).astype(np.float16)
    args = (o["packed"], o["scale"], o["zero"], None, 40, 512, 4, 64, 16)
    y1, y2 = orc.gemv(*args, x1)[0], orc.gemv(*args, x2)[0]
    y12 = orc.gemv(*args, (x1 + x2).astype(np.float16))[0]
    assert np.allclose(y12, y1 + y2, rtol=1e-12, atol=1e-12)
    Y = orc.gemv(*args, np.stack([x1, x2, x1]))
    assert np.array_equal(Y[0], y1) and np.array_equal(Y[1], y2) and np.array_equal(Y[2], y1)
    xb = (x1.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(orc.gemv(*args, xb, x_dtype=orc.BF16)[0], y1)


# ------------------------------- tensor-core product (16-bit weights) ---

def _golden(name):
    d = {}
    for line in open(os.path.join(GOLDEN, name)):
        if line.startswith("#") or not line.strip():
            continue
        k, *v = line.split()
        d[k] = v
    return d


def _bf16_bits(a):
    """fp32 values exact in bf16 -> their bf16 bit patterns."""
    u = np.asarray(a, np.float32).view(np.uint32)
    assert np.all(u & 0xFFFF == 0)
    return (u >> 16).astype(np.uint16)


@pytest.mark.parametrize("xdt", ["bf16", "f16"])
def test_gemm_hand_values(orc, xdt):
    """Hand-worked values, including a tie that rounds to even in bf16."""
    d = _golden("gemm_hand_values.txt")
    rows, cols, nb, g = (int(d[k][0]) for k in ("rows", "cols", "nbits", "group"))
    lv = np.array([int(v) for v in d["levels"]], np.uint8).reshape(rows, cols)
    packed = np.zeros(rows * cols * nb // 8, np.uint8)
    orc.lib().oracle_pack_levels(lv.ctypes.data, rows, cols, nb, 1, packed.ctypes.data)
    sc = np.array([float(v) for v in d["scale"]], np.float16)
    z = np.array([float(v) for v in d["zero"]], np.float16)
    xf = np.array([float(v) for v in d["x"]], np.float32)
    if xdt == "bf16":
        y, ya = orc.gemm(packed, sc, z, None, rows, cols, nb, g, 16, _bf16_bits(xf), orc.BF16)
    else:
        y, ya = orc.gemm(packed, sc, z, None, rows, cols, nb, g, 16, xf.astype(np.float16), orc.F16)
    assert y[0].tolist() == [float(v) for v in d["y_" + xdt]]
    assert ya[0].tolist() == [float(v) for v in d["yabs_" + xdt]]


@pytest.mark.parametrize("nbits,g,zb", [(4, 64, 16), (2, 16, 8), (3, 32, 16), (8, 128, 8)])
def test_gemm_unit_vectors_give_dequantised_columns(orc, nbits, g, zb):
    """x = e_c picks column c of W_r rounded to x's type: the dequantiser's
    output in that type, for fp16 and bf16."""
    W = _synth_f16(24, 256, seed=3 * nbits + g)
    o = orc.quantize(W, nbits, g, 1, 0.7, 1.0, 1.01, 20, orc.STOP_GROUP, zb)
    cols = [0, 1, g - 1, g, 255]
    X = np.zeros((len(cols), 256), np.float32)
    for i, c in enumerate(cols):
        X[i, c] = 1.0
    for dt, xs in ((orc.F16, X.astype(np.float16)), (orc.BF16, _bf16_bits(X))):
        deq = orc.dequantize(o["packed"], o["scale"], o["zero"], o["zero_meta"], 24, 256, nbits, g, 1, zb,
                             out_dtype=dt)
        Y, Ya = orc.gemm(o["packed"], o["scale"], o["zero"], o["zero_meta"], 24, 256, nbits, g, zb, xs, dt)
        for i, c in enumerate(cols):
            col = deq[:, c].astype(np.float32) if dt == orc.F16 else \
                (deq[:, c].astype(np.uint32) << 16).view(np.float32)
            assert np.array_equal(Y[i], col.astype(np.float64))
            assert np.array_equal(Ya[i], np.abs(col).astype(np.float64))


def test_gemm_equals_gemv_when_weights_are_16_bit_exact(orc):
    """Codes at 2 bit, zero a multiple of 2^-4 below 3, scale a power of two:
    q - z has at most 6 significant bits, so every W_r is exact in bf16, the
    rounding is the identity and the product is the fp32-weight product of
    the matrix-vector oracle."""
    r = np.random.default_rng(9)
    rows, cols, nb, g = 16, 128, 2, 32
    lv = r.integers(0, 4, (rows, cols)).astype(np.uint8)
    packed = np.zeros(rows * cols * nb // 8, np.uint8)
    orc.lib().oracle_pack_levels(lv.ctypes.data, rows, cols, nb, 1, packed.ctypes.data)
    G = rows * cols // g
    sc = (2.0 ** -r.integers(0, 5, G)).astype(np.float16)
    z = (r.integers(0, 48, G) / 16).astype(np.float16)
    x = (r.integers(-64, 64, (3, cols)) / 32).astype(np.float32)
    y16, _ = orc.gemm(packed, sc, z, None, rows, cols, nb, g, 16, _bf16_bits(x), orc.BF16)
    y32 = orc.gemv(packed, sc, z, None, rows, cols, nb, g, 16, _bf16_bits(x), orc.BF16)
    assert np.array_equal(y16, y32)


# ------------------------------------------------- sampled-group solver ----

@pytest.mark.parametrize("axis", [0, 1])
@pytest.mark.parametrize("g,nbits", [(8, 4), (1024, 2)])
@pytest.mark.parametrize("mode", [0, 2])
def test_quantize_groups_equals_whole_tensor(orc, axis, g, nbits, mode):
    """oracle_quantize_groups (the checker of every sampled full-size GPU case)
    returns, for each listed group, exactly what the whole-tensor oracle
    returns for it: codes, scale, kept zero, kept iterate and its error.  The
    list holds the first and last group, is unsorted and repeats ids."""
    long_, short = (2048, 6) if g == 1024 else (40, 24)
    rows, cols = (short, long_) if axis == 1 else (long_, short)
    W = _synth_f16(rows, cols, seed=70 + g + axis + mode)
    full = orc.quantize(W, nbits, g, axis=axis, stop_mode=mode)
    G = rows * cols // g
    ids = np.array([G - 1, 0, 5, 5, 3, G - 1, 1, G // 2], np.int64)
    part = orc.quantize_groups(W, ids, nbits, g, axis=axis, stop_mode=mode)
    levels = orc.unpack_levels(full["packed"], rows, cols, nbits, axis)
    for k, j in enumerate(ids):
        if axis == 1:
            want = levels.reshape(-1)[j * g:(j + 1) * g]
        else:
            rb, c = divmod(int(j), cols)
            want = levels[rb * g:(rb + 1) * g, c]
        assert np.array_equal(part["levels"][k], want), f"codes of group {j}"
        assert np.float16(1.0 / part["s"][k]) == full["scale"][j], f"scale of group {j}"
        assert part["zbest"][k] == full["zero_f32"][j]
        assert part["best_iter"][k] == full["best_iter"][j]
        assert part["best_err"][k] == full["best_err"][j]


# --------------------------------------------- half-precision variant ------

def _half_rows():
    rows = []
    with open(os.path.join(GOLDEN, "half_worked_groups.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            head, w = line.split(";")
            name, nb, s, z0, z1, codes = head.split()
            rows.append((name, int(nb), float(s), float(z0), float(z1), [int(c) for c in codes.split(",")],
                         np.array([float(x) for x in w.split()], np.float32)))
    return rows


@pytest.mark.parametrize("name,nbits,s,z0,z1,codes,w", _half_rows())
def test_half_worked_groups(orc, name, nbits, s, z0, z1, codes, w):
    """Hand-worked fp16 steps (tests/golden/half_worked_groups.txt): the scale,
    z0, the codes at z0 (group B has a code that the fp16 rounding of w*s
    decides) and z1 (group A's mean is not an fp16 number)."""
    assert np.array_equal(w.astype(np.float16).astype(np.float32), w)
    ss, zt, et, _ = orc.trace_group_half(w, nbits, iters=2)
    assert ss == s and zt[0] == z0 and zt[1] == z1
    assert list(orc.group_codes_half(w, nbits, ss, zt[0])) == codes


@pytest.mark.parametrize("nbits", NBITS)
def test_half_values_are_fp16(orc, nbits):
    """Every scale and zero-point of the variant is an fp16 number, and so are
    the stored zeros; the kept error is the lowest of the trajectory."""
    rng = _rng(200 + nbits)
    for g in (8, 16, 64):
        for _ in range(20):
            w = (rng.standard_normal(g) * rng.choice([0.02, 0.3, 3.0])).astype(np.float16).astype(np.float32)
            s, zt, et, _ = orc.trace_group_half(w, nbits, iters=12)
            assert np.float32(np.float16(s)) == s
            assert np.array_equal(zt.astype(np.float16).astype(np.float32), zt)
            assert np.all(np.isfinite(et)) and np.all(et >= 0)
    W = _synth_f16(32, 256, seed=nbits)
    out = orc.quantize_half(W, nbits, 32, stop_mode=2)
    zf = out["zero_f32"]
    assert np.array_equal(zf.astype(np.float16).astype(np.float32), zf)
    assert np.array_equal(out["zero"].astype(np.float32), zf)


@pytest.mark.parametrize("nbits", [1, 2, 3, 4])
def test_half_trajectory_equals_fp32_when_exact(orc, nbits):
    """On groups whose every intermediate value is exact in fp16 (values m/256,
    range (2^b - 1)/16 so that s = 16, g = 8), no fp16 rounding happens: the
    variant's zero-points and codes follow the fp32 oracle's exactly, and its
    errors agree within the fp16 rounding of the terms (2^-11 relative each)."""
    rng = _rng(300 + nbits)
    L = (1 << nbits) - 1
    for _ in range(30):
        lo = int(rng.integers(-64, 64))
        m = rng.integers(lo, lo + 16 * L + 1, size=8)
        m[0], m[1] = lo, lo + 16 * L
        w = (m / 256.0).astype(np.float32)
        assert np.array_equal(w.astype(np.float16).astype(np.float32), w)
        s16, zh, eh, _ = orc.trace_group_half(w, nbits, iters=6)
        s32, z32, e32, _ = orc.trace_group(w, nbits, iters=6)
        assert s16 == s32 == 16.0
        if np.all(np.abs(z32) < 16):
            assert np.array_equal(zh, z32), (zh, z32)
            for z in zh:
                assert np.array_equal(orc.group_codes_half(w, nbits, s16, z), orc.group_codes(w, nbits, s32, z))
            assert np.all(np.abs(eh - e32) <= 2.0 ** -10 * e32 + 1e-30)


def test_half_quantize_matches_its_trace(orc):
    """The whole-tensor variant keeps, per group, the first iterate of lowest
    error along its own trace (group stop: up to the first rise) and stores
    fp16(1/s) and the codes of that iterate."""
    W = _synth_f16(16, 512, seed=9)
    for stop in (0, 2):
        out = orc.quantize_half(W, 4, 64, stop_mode=stop, iters=20)
        levels = orc.unpack_levels(out["packed"], 16, 512, 4, 1).reshape(-1, 64)
        for j in range(0, 16 * 512 // 64, 7):
            w = W.reshape(-1, 64)[j].astype(np.float32)
            s, zt, et, _ = orc.trace_group_half(w, 4, iters=20)
            if stop == 0:
                k = 0
                while k + 1 < 20 and et[k + 1] < et[k]:
                    k += 1
            else:
                k = int(np.argmin(et))
            assert out["best_iter"][j] == k and out["zero_f32"][j] == zt[k]
            assert out["scale"][j] == np.float16(np.float32(1.0) / np.float32(s))
            assert np.array_equal(levels[j], orc.group_codes_half(w, 4, s, zt[k]))
