"""GPU-vs-oracle comparison used by the GPU tests and the smoke check.

Bar (per group unless stated):
  * scale within 1e-3 relative (it is computed by identical fp32 steps, so it
    is expected to match exactly);
  * the kept zero-point z* within 1e-3 * max(|z*|, 1);
  * codes identical except a fraction <= 1e-4 of elements, each within one
    level (rounding ties: the two sides' z* may differ in the last bits);
  * the tensor's reconstruction lp error mean|W - dequant|^p within 1e-3
    relative;
  * the GPU dequantiser reproduces the oracle's dequantisation of the same
    codes bit for bit.
Stop decisions compare two sums of |r|^p; the GPU evaluates |r|^p with the
hardware base-2 log/exp and sums in another order, so a decision whose two
errors differ by less than TIE_TOL (relative) may go either way.  A group
whose kept iterate differs from the oracle's is accepted only if every
decision on which the two paths disagree is such a near tie, and then its
outputs are checked against the oracle's own iterate at the GPU's index.
The number of such tie groups is reported and must stay <= 1e-4 of groups
(+1 for small tensors).
"""
import numpy as np
import torch

import oracle

TIE_TOL = 2e-5
Z_TOL = 1e-3
CODE_FRAC = 1e-4
ERR_TOL = 1e-3


def w_for_oracle(W_cpu):
    """(array, dtype code) for the oracle from a CPU fp16/bf16 tensor."""
    if W_cpu.dtype == torch.float16:
        return W_cpu.numpy(), oracle.F16
    return W_cpu.view(torch.int16).numpy().view(np.uint16), oracle.BF16


def w_float(W_cpu):
    return W_cpu.float().numpy()


def gpu_to_numpy(out):
    return {k: (v.cpu().numpy() if isinstance(v, torch.Tensor) else v) for k, v in out.items()}


def group_values(Wf, j, g, axis):
    rows, cols = Wf.shape
    if axis == 1:
        return Wf.reshape(-1)[j * g:(j + 1) * g]
    rb, c = divmod(j, cols)
    return Wf[rb * g:(rb + 1) * g, c]


def group_levels(levels, j, g, axis):
    rows, cols = levels.shape
    if axis == 1:
        return levels.reshape(-1)[j * g:(j + 1) * g]
    rb, c = divmod(j, cols)
    return levels[rb * g:(rb + 1) * g, c]


def all_groups(arr, g, axis):
    """[G, g] view of a [rows, cols] array, groups in index order."""
    rows, cols = arr.shape
    if axis == 1:
        return arr.reshape(-1, g)
    return arr.reshape(rows // g, g, cols).transpose(0, 2, 1).reshape(-1, g)


def _path_ok(e, k_gpu, k_orc, iters, mode):
    """Is the GPU's kept index k_gpu explainable by near ties on the oracle's
    error trajectory e (group-mode or tensor-mode first-non-improvement rule,
    or argmin for no-stop mode)?"""
    if mode == oracle.STOP_NONE:
        return e[k_gpu] <= e[k_orc] * (1 + TIE_TOL) + 1e-30
    # decisions the GPU took: improve at 1..k_gpu, stop at k_gpu+1 (if any)
    for i in range(1, k_gpu + 1):
        if not e[i] < e[i - 1] and (e[i] - e[i - 1]) > TIE_TOL * e[i - 1]:
            return False
    if k_gpu + 1 < iters:
        nxt = k_gpu + 1
        if e[nxt] < e[k_gpu] and (e[k_gpu] - e[nxt]) > TIE_TOL * e[k_gpu]:
            return False
    return True


def check(W_cpu, params, gpu, orc=None, sample=None, report=None, tie_cap=None):
    """Compare GPU outputs (numpy dict, from quantize(..., debug=True)) with the oracle.

    params: dict(nbits, group_size, axis, p, beta, kappa, iters, stop_mode, zero_nbits).
    sample: optional array of group ids (group mode / no stop only): the oracle
    solves just those groups.  Otherwise `orc` is the oracle's full output
    (computed here when None).  tie_cap: the number of near-tie groups allowed
    (default 1e-4 of the groups, + 1); each one is explained and checked either
    way.  Returns a report dict; raises AssertionError.
    """
    nb, g, axis = params["nbits"], params["group_size"], params["axis"]
    p, beta, kappa, iters = params["p"], params["beta"], params["kappa"], params["iters"]
    mode, zb = params["stop_mode"], params["zero_nbits"]
    rows, cols = W_cpu.shape
    G = rows * cols // g
    Wo, dt = w_for_oracle(W_cpu)
    Wf = w_float(W_cpu)
    rep = report if report is not None else {}
    gl = oracle.unpack_levels(gpu["packed"], rows, cols, nb, axis)

    if sample is not None:
        assert mode != oracle.STOP_TENSOR
        ids = np.asarray(sample, np.int64)
        o = oracle.quantize_groups(Wo, ids, nb, g, axis, p, beta, kappa, iters, mode, dtype=dt)
        o_levels = o["levels"]
        o_z, o_s, o_bi, o_err = o["zbest"], o["s"], o["best_iter"], o["best_err"]
        o_scale = (1.0 / o_s).astype(np.float16)
    else:
        if orc is None:
            orc = oracle.quantize(Wo, nb, g, axis, p, beta, kappa, iters, mode, zb, dtype=dt)
        ids = np.arange(G)
        ol = oracle.unpack_levels(orc["packed"], rows, cols, nb, axis)
        o_levels = all_groups(ol, g, axis)
        o_z, o_bi, o_err, o_scale = orc["zero_f32"], orc["best_iter"], orc["best_err"], orc["scale"]
    g_levels = all_groups(gl, g, axis)[ids]

    # scale: identical fp32 steps on both sides
    gs = gpu["scale"][ids].astype(np.float64)
    os_ = o_scale.astype(np.float64)
    assert np.all(np.abs(gs - os_) <= 1e-3 * np.abs(os_)), "scale mismatch"
    rep["scale_exact_frac"] = float(np.mean(gpu["scale"][ids].view(np.uint16) == o_scale.view(np.uint16))) if len(
        ids) else 1.0

    g_z = gpu["zero_f32"][ids]
    g_bi = gpu["best_iter"][ids]
    tie = np.nonzero(g_bi != o_bi)[0]
    if mode == oracle.STOP_TENSOR and len(tie):
        # one decision for the whole tensor: check it on the oracle's tensor trajectory
        traces = [oracle.trace_group(group_values(Wf, j, g, axis), nb, p, beta, kappa, max(iters, 1)) for j in ids]
        E = np.mean([t[2] for t in traces], axis=0)
        kg, ko = int(g_bi[0]), int(o_bi[0])
        assert _path_ok(E, kg, ko, iters, mode), f"tensor stop {kg} vs oracle {ko} is not a near tie: {E}"
        exp_z = np.array([t[1][kg] for t in traces], np.float32)
        exp_lv = np.stack([oracle.group_codes(group_values(Wf, j, g, axis), nb, t[0], t[1][kg])
                           for j, t in zip(ids, traces)])
        o_z, o_levels = exp_z, exp_lv
        rep["tensor_tie"] = (kg, ko)
        tie = np.zeros(0, np.int64)
    elif len(tie):
        for t in tie:
            j = ids[t]
            w = group_values(Wf, j, g, axis)
            s, zt, et, _ = oracle.trace_group(w, nb, p, beta, kappa, max(iters, 1))
            kg = int(g_bi[t])
            assert _path_ok(et, kg, int(o_bi[t]), iters, mode), (
                f"group {j}: kept iterate {kg} vs oracle {o_bi[t]} is not a near tie: {et[:max(kg, o_bi[t]) + 2]}")
            o_z = o_z.copy()
            o_levels = o_levels.copy()
            o_z[t] = zt[kg]
            o_levels[t] = oracle.group_codes(w, nb, s, zt[kg])
        cap = CODE_FRAC * len(ids) + 1 if tie_cap is None else tie_cap
        assert len(tie) <= cap, f"{len(tie)} tie groups of {len(ids)}"
    rep["tie_groups"] = int(len(tie))

    dz = np.abs(g_z.astype(np.float64) - o_z.astype(np.float64))
    assert np.all(dz <= Z_TOL * np.maximum(np.abs(o_z), 1.0)), f"zero mismatch, max {dz.max()}"
    rep["z_max_abs_diff"] = float(dz.max()) if dz.size else 0.0

    diff = g_levels.astype(np.int32) - o_levels.astype(np.int32)
    nd = int(np.count_nonzero(diff))
    assert np.all(np.abs(diff) <= 1), "a code differs by more than one level"
    assert nd <= CODE_FRAC * diff.size + 1, f"{nd} differing codes of {diff.size}"
    rep["code_mismatch"] = nd

    # debug error of the kept zero-point (non-tie groups)
    keep = np.ones(len(ids), bool)
    keep[tie] = False
    ge, oe = gpu["best_err"][ids][keep].astype(np.float64), o_err[keep].astype(np.float64)
    if mode != oracle.STOP_TENSOR or "tensor_tie" not in rep:
        assert np.all(np.abs(ge - oe) <= ERR_TOL * np.maximum(oe, 1e-30) + 1e-12), "best_err mismatch"
    return rep


def gpu_dequantizer(hq):
    """A function running the GPU dequantiser (through the C ABI) on given
    numpy arrays -- used with the oracle's own outputs, so that no oracle input
    comes from the CUDA path."""
    import torch

    def run(q, rows, cols, nbits, g, axis, zero_nbits, out_code, scale8=None):
        dev = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in q.items() if v is not None}
        out_dt = torch.float16 if out_code == oracle.F16 else torch.bfloat16
        out = torch.empty(rows, cols, dtype=out_dt, device="cuda")
        if scale8 is None:
            rc = hq.hqq_dequantize(dev["packed"], dev["scale"], dev["zero"], dev.get("zero_meta"), rows, cols, nbits,
                                   g, axis, zero_nbits, hq.HQQ_F16 if out_code == oracle.F16 else hq.HQQ_BF16, out)
        else:
            rc = hq.hqq_dequantize_s8(dev["packed"], dev["scale_q"], dev["scale_meta"], scale8, dev["zero"],
                                      dev.get("zero_meta"), rows, cols, nbits, g, axis, zero_nbits,
                                      hq.HQQ_F16 if out_code == oracle.F16 else hq.HQQ_BF16, out)
        assert rc == hq.HQQ_OK, hq.hqq_status_string(rc)
        torch.cuda.synchronize()
        o = out.cpu()
        return (o.numpy() if out_dt == torch.float16 else o.view(torch.int16).numpy()).view(np.uint16)
    return run


def check_reconstruction(W_cpu, params, gpu_deq, orc, gpu_dequant):
    """The GPU dequantiser bit-exact against the oracle's dequantisation, both
    run on the oracle's outputs; and the tensor lp error of the GPU's
    dequantised weights (its own codes) against the oracle's."""
    nb, g, axis, zb, p = params["nbits"], params["group_size"], params["axis"], params["zero_nbits"], params["p"]
    rows, cols = W_cpu.shape
    out_dt = oracle.F16 if gpu_deq.dtype == np.float16 else oracle.BF16
    od = oracle.dequantize(orc["packed"], orc["scale"], orc["zero"], orc["zero_meta"], rows, cols, nb, g, axis, zb,
                           out_dt)
    got = gpu_dequant(dict(packed=orc["packed"], scale=orc["scale"], zero=orc["zero"], zero_meta=orc["zero_meta"]),
                      rows, cols, nb, g, axis, zb, out_dt)
    assert np.array_equal(od.view(np.uint16), got), "dequantiser differs from the oracle's"
    Wf = w_float(W_cpu).astype(np.float64)

    def tofloat(a):
        if a.dtype == np.float16:
            return a.astype(np.float64)
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)

    eg = float(np.mean(np.abs(Wf - tofloat(gpu_deq)) ** p)) if Wf.size else 0.0
    eo = float(np.mean(np.abs(Wf - tofloat(od)) ** p)) if Wf.size else 0.0
    assert abs(eg - eo) <= ERR_TOL * max(eo, 1e-30) + 1e-30, f"reconstruction error {eg} vs oracle {eo}"
    return eg, eo


def check_zero8(gpu, orc):
    """8-bit zero path: codes within one level (fp32 z* may differ in the last
    bits), meta pair within 1e-5, dequantised zeros within the zero tolerance."""
    gz, oz = gpu["zero"].astype(np.int32), orc["zero"].astype(np.int32)
    d = gz - oz
    assert np.all(np.abs(d) <= 1)
    assert np.count_nonzero(d) <= CODE_FRAC * d.size + 1
    gm, om = gpu["zero_meta"].astype(np.float64), orc["zero_meta"].astype(np.float64)
    assert np.allclose(gm, om, rtol=1e-5, atol=1e-6), (gm, om)
    zg = (gz - gm[1]) * gm[0]
    zo = (oz - om[1]) * om[0]
    assert np.all(np.abs(zg - zo) <= Z_TOL * np.maximum(np.abs(zo), 1.0) + gm[0] * 1.0001)


def check_stored(W_cpu, params, out, orc=None, sample=None):
    """Compare stored outputs only -- codes, scale, zero and zero_meta, what a
    streamed run returns (numpy dict, no debug outputs) -- with the oracle.

    Bars as in check(): scale within 1e-3 relative; a 16-bit zero within
    1e-3 * max(|z*|, 1) plus half its fp16 step; an 8-bit zero, dequantised with
    the stored pair, within half a quantiser step (plus 1e-3) of the oracle's
    z*; codes identical except <= 1e-4 of elements, each within one level.  A
    group that misses these bars is accepted only as a near tie: some iterate
    k that the oracle's own error trajectory allows (near ties, TIE_TOL) must
    reproduce its codes and zero; such groups stay <= 1e-4 of groups (+1).
    With sample= (group / no stop) only those groups are solved by the oracle.
    Returns a report dict; raises AssertionError."""
    nb, g, axis = params["nbits"], params["group_size"], params["axis"]
    p, beta, kappa, iters = params["p"], params["beta"], params["kappa"], params["iters"]
    mode, zb = params["stop_mode"], params["zero_nbits"]
    rows, cols = W_cpu.shape
    G = rows * cols // g
    Wo, dt = w_for_oracle(W_cpu)
    Wf = w_float(W_cpu)
    gl = oracle.unpack_levels(out["packed"], rows, cols, nb, axis)
    if sample is not None:
        assert mode != oracle.STOP_TENSOR
        ids = np.asarray(sample, np.int64)
        o = oracle.quantize_groups(Wo, ids, nb, g, axis, p, beta, kappa, iters, mode, dtype=dt)
        o_levels, o_z, o_bi = o["levels"], o["zbest"], o["best_iter"]
        o_scale = (1.0 / o["s"]).astype(np.float16)
    else:
        if orc is None:
            orc = oracle.quantize(Wo, nb, g, axis, p, beta, kappa, iters, mode, zb, dtype=dt)
        ids = np.arange(G)
        o_levels = all_groups(oracle.unpack_levels(orc["packed"], rows, cols, nb, axis), g, axis)
        o_z, o_bi, o_scale = orc["zero_f32"], orc["best_iter"], orc["scale"]
    g_levels = all_groups(gl, g, axis)[ids]

    gs, os_ = out["scale"][ids].astype(np.float64), o_scale.astype(np.float64)
    assert np.all(np.abs(gs - os_) <= 1e-3 * np.abs(os_)), "scale mismatch"

    if zb == 16:
        gz = out["zero"][ids].astype(np.float64)
        ztol = Z_TOL * np.maximum(np.abs(o_z), 1.0) + np.abs(o_z) * 2.0 ** -11

        def zero_ok(zg, zo):
            return np.abs(zg - zo) <= Z_TOL * max(abs(zo), 1.0) + abs(zo) * 2.0 ** -11
    else:
        meta = out["zero_meta"].astype(np.float64)
        gz = (out["zero"][ids].astype(np.float64) - meta[1]) * meta[0]
        ztol = 0.5 * meta[0] * (1 + 1e-6) + Z_TOL * np.maximum(np.abs(o_z), 1.0)

        def zero_ok(zg, zo):
            return np.abs(zg - zo) <= 0.5 * meta[0] * (1 + 1e-6) + Z_TOL * max(abs(zo), 1.0)
    zbad = np.abs(gz - o_z.astype(np.float64)) > ztol
    diff = g_levels.astype(np.int32) - o_levels.astype(np.int32)
    bad = zbad | (np.abs(diff) > 1).any(axis=1)
    nbad = np.nonzero(bad)[0]
    rep = {"groups": int(len(ids))}

    def explain(t, allowed):
        """An iterate k allowed by the trajectory's near ties that reproduces group t."""
        j = ids[t]
        w = group_values(Wf, j, g, axis)
        s, zt, et, _ = oracle.trace_group(w, nb, p, beta, kappa, max(iters, 1))
        for k in allowed(et):
            lv = oracle.group_codes(w, nb, s, zt[k]).astype(np.int32)
            if zero_ok(gz[t], zt[k]) and np.all(np.abs(lv - g_levels[t]) <= 1) and \
                    np.count_nonzero(lv - g_levels[t]) <= max(1, CODE_FRAC * g):
                return True
        return False

    if mode == oracle.STOP_TENSOR and len(nbad) > CODE_FRAC * len(ids) + 1:
        # the tensor-wide decision itself went the other way: every group at one other iterate
        traces = [oracle.trace_group(group_values(Wf, j, g, axis), nb, p, beta, kappa, max(iters, 1)) for j in ids]
        E = np.mean([t[2] for t in traces], axis=0)
        ko = int(o_bi[0])
        ks = [k for k in range(max(iters, 1)) if _path_ok(E, k, ko, iters, mode)]
        ok = False
        for k in ks:
            lv = np.stack([oracle.group_codes(group_values(Wf, j, g, axis), nb, t[0], t[1][k])
                           for j, t in zip(ids, traces)]).astype(np.int32)
            zk = np.array([t[1][k] for t in traces], np.float64)
            d = lv - g_levels.astype(np.int32)
            if np.all(np.abs(d) <= 1) and np.count_nonzero(d) <= CODE_FRAC * d.size + 1 and \
                    np.all(np.abs(gz - zk) <= ztol):
                ok = True
                rep["tensor_tie"] = (k, ko)
                break
        assert ok, f"tensor stop: {len(nbad)} groups differ and no near-tie iterate explains them ({ks})"
        return rep
    for t in nbad:
        allowed = (lambda et, t=t: [k for k in range(max(iters, 1)) if _path_ok(et, k, int(o_bi[t]), iters, mode)])
        assert explain(t, allowed), f"group {ids[t]}: outputs differ from the oracle's and no near tie explains it"
    assert len(nbad) <= CODE_FRAC * len(ids) + 1, f"{len(nbad)} tie groups of {len(ids)}"
    good = np.ones(len(ids), bool)
    good[nbad] = False
    nd = int(np.count_nonzero(diff[good]))
    assert nd <= CODE_FRAC * diff[good].size + 1, f"{nd} differing codes of {diff[good].size}"
    rep["tie_groups"] = int(len(nbad))
    rep["code_mismatch"] = nd
    return rep


# ------------------------------------------- half-precision variant -------

# The variant's error terms are |r|^p rounded to fp16; the GPU forms |r|^p
# with the hardware base-2 log and exponential in fp32 before that rounding,
# so a term can land one fp16 step (at most 2^-10 relative) from the oracle's
# exactly rounded one, and a sum of such terms can move by up to 2^-10
# relative.  A decision can therefore flip when the oracle's two sums differ
# by less than twice that.
TIE_TOL_HALF = 2.0 ** -9


def _path_ok_tol(e, k_gpu, k_orc, iters, mode, tol):
    if mode == oracle.STOP_NONE:
        return e[k_gpu] <= e[k_orc] * (1 + tol) + 1e-30
    for i in range(1, k_gpu + 1):
        if not e[i] < e[i - 1] and (e[i] - e[i - 1]) > tol * e[i - 1]:
            return False
    if k_gpu + 1 < iters:
        nxt = k_gpu + 1
        if e[nxt] < e[k_gpu] and (e[k_gpu] - e[nxt]) > tol * e[k_gpu]:
            return False
    return True


def check_half(W_cpu, params, gpu, orc):
    """The half-precision variant (GPU outputs with debug, numpy) against its
    oracle.  The arithmetic is the same on both sides except the error terms,
    so every group whose kept iterate matches has bit-identical scale, kept
    zero and codes; a group whose kept iterate differs must be explained by
    decisions within TIE_TOL_HALF on the oracle's own trajectory and must then
    match the oracle's iterate at the GPU's index exactly.  Returns a report."""
    nb, g = params["nbits"], params["group_size"]
    p, beta, kappa, iters, mode = params["p"], params["beta"], params["kappa"], params["iters"], params["stop_mode"]
    rows, cols = W_cpu.shape
    G = rows * cols // g
    Wf = W_cpu.float().numpy()
    assert np.array_equal(gpu["scale"].view(np.uint16), orc["scale"].view(np.uint16)), "scale"
    gl = all_groups(oracle.unpack_levels(gpu["packed"], rows, cols, nb, 1), g, 1)
    ol = all_groups(oracle.unpack_levels(orc["packed"], rows, cols, nb, 1), g, 1)
    differ = np.nonzero(gpu["best_iter"] != orc["best_iter"])[0]
    same = np.ones(G, bool)
    same[differ] = False
    assert np.array_equal(gpu["zero_f32"][same], orc["zero_f32"][same]), "kept zero"
    assert np.array_equal(gl[same], ol[same]), "codes"
    for j in differ:
        w = group_values(Wf, j, g, 1)
        s, zt, et, _ = oracle.trace_group_half(w, nb, p, beta, kappa, max(iters, 1))
        kg = int(gpu["best_iter"][j])
        assert _path_ok_tol(et, kg, int(orc["best_iter"][j]), iters, mode, TIE_TOL_HALF), (
            f"group {j}: kept iterate {kg} vs oracle {orc['best_iter'][j]} is not a near tie: {et[:kg + 3]}")
        assert gpu["zero_f32"][j] == zt[kg], (j, gpu["zero_f32"][j], zt[kg])
        assert np.array_equal(gl[j], oracle.group_codes_half(w, nb, s, zt[kg])), j
    if params["zero_nbits"] == 16:
        assert np.array_equal(gpu["zero"].astype(np.float32), gpu["zero_f32"])
    return {"groups": G, "tie_groups": int(len(differ)), "tie_frac": float(len(differ)) / max(G, 1)}
