"""Pins of the fp64 oracle against what the paper and the mathematics fix.

Each test names the passage of "Pretraining Transformers with Quantized
Softmax in Attention" (paperlayer.ai abstract page) it pins.  None of them
retypes the oracle's formulas: they use finite differences, closed forms,
invariants, bounds, a second (linear-scan) forward, and numpy contractions.
"""
import math
import os

import numpy as np
import pytest

import oracle as ref

HERE = os.path.dirname(os.path.abspath(__file__))

CALS = [ref.CAL_MINMAX, ref.CAL_FWM, ref.CAL_FIXED]
MODES = [ref.GRAD_FULL, ref.GRAD_DETACH, ref.GRAD_MAX_ONLY, ref.GRAD_MIN_ONLY, ref.GRAD_PROJECT]
RECSTE = [(ref.REC_LERP, ref.STE_WEIGHT), (ref.REC_NEAREST, ref.STE_WEIGHT),
          (ref.REC_NEAREST, ref.STE_PROB)]


def _rows(rng, n, L, span_lo=3.0, span_hi=30.0):
    """Random score rows with spans in [span_lo, span_hi] nats, all keys visible."""
    S = rng.standard_normal((n, L))
    S -= S.min(axis=1, keepdims=True)
    S /= S.max(axis=1, keepdims=True)
    spans = rng.uniform(span_lo, span_hi, size=(n, 1))
    S = S * spans - rng.uniform(0, 5, size=(n, 1))
    return S


def _loss(S, L, cfg, dP, fm=None, fn=None):
    out = ref.rows(S, L, cfg, frozen_m=fm, frozen_n=fn)
    return (out["P"] * dP).sum(axis=1)


def _near_kink(S, L, cfg, tol):
    """Rows where some key sits within tol (in u units) of a node, of the FWM
    edge, or where the top-2 / bottom-2 scores are within tol*h."""
    st = ref.rows(S, L, cfg)["stats"]
    bad = np.zeros(S.shape[0], bool)
    for i in range(S.shape[0]):
        s = S[i, :L[i]]
        h = st[i, ref.ST_H]
        with np.errstate(invalid="ignore", divide="ignore"):
            u = (st[i, ref.ST_M] - s) / h
        frac = np.abs(u - np.round(u))
        if cfg.cal == ref.CAL_FWM:
            frac = np.where(u > cfg.K + 0.5, 1.0, frac)
        # the extrema sit on nodes 0 and K by construction and move the grid
        # with them, so they are not kinks
        frac[int(st[i, ref.ST_AM])] = 1.0
        if cfg.cal == ref.CAL_MINMAX:
            frac[int(st[i, ref.ST_AN])] = 1.0
        ss = np.sort(s)
        gap = min(ss[-1] - ss[-2], ss[1] - ss[0]) if len(ss) > 2 else 1.0
        bad[i] = frac.min() < tol or gap < tol * h
    return bad


# ---------------------------------------------------------------- golden

def _golden():
    vals = {}
    with open(os.path.join(HERE, "golden", "page_constants.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, val = line.split()[:2]
            vals[name] = float(val)
    return vals


def test_page_constants_fwm_width_and_minmax_quarter_span():
    """Appendix A: FWM at K=4 uses h = 1.5; MinMax at K=4 uses a quarter of the span."""
    g = _golden()
    rng = np.random.default_rng(0)
    S = _rows(rng, 16, 40)
    L = np.full(16, 40)
    st = ref.rows(S, L, ref.RefConfig(K=4, cal=ref.CAL_FWM, tau=g["fwm_tau"]))["stats"]
    assert np.all(st[:, ref.ST_H] == g["fwm_K4_h"])
    st = ref.rows(S, L, ref.RefConfig(K=4, cal=ref.CAL_MINMAX))["stats"]
    span = S.max(1) - S.min(1)
    np.testing.assert_allclose(st[:, ref.ST_H], g["minmax_K4_h_over_span"] * span, rtol=1e-15)


def test_grid_has_k_plus_one_distinct_nearest_values():
    """Section 1: K+1 grid values.  Nearest weights on a dense row take exactly
    K+1 distinct values e^{-kh}, k = 0..K (MinMax: the row min sits on node K)."""
    K = 5
    S = np.linspace(0.0, -10.0, 2001)[None, :]
    out = ref.rows(S, [2001], ref.RefConfig(K=K, cal=ref.CAL_MINMAX, rec=ref.REC_NEAREST))
    w = out["P"][0] * out["stats"][0, ref.ST_WN]
    vals = np.unique(w)
    assert len(vals) == K + 1
    np.testing.assert_allclose(np.sort(vals)[::-1], np.exp(-np.arange(K + 1) * 2.0), rtol=1e-13)


# ------------------------------------------------------ finite differences

@pytest.mark.parametrize("cal", CALS)
def test_lerp_full_gradient_matches_central_differences(cal):
    """Section 3 / Appendix B: for LERP the full calibration gradient is the
    exact derivative of the loss (checked to < 1e-9 against autograd there)."""
    rng = np.random.default_rng(1 + cal)
    n, L = 24, 12
    S = _rows(rng, n, L)
    Ls = np.full(n, L)
    cfg = ref.RefConfig(K=4, cal=cal, rec=ref.REC_LERP, grad=ref.GRAD_FULL)
    dP = rng.standard_normal((n, L))
    ok = ~_near_kink(S, Ls, cfg, 1e-3)
    assert ok.sum() >= n // 2
    dS = ref.rows(S, Ls, cfg, dP=dP)["dS"]
    eps = 1e-6
    fd = np.zeros_like(S)
    for j in range(L):
        Sp, Sm = S.copy(), S.copy()
        Sp[:, j] += eps
        Sm[:, j] -= eps
        fd[:, j] = (_loss(Sp, Ls, cfg, dP) - _loss(Sm, Ls, cfg, dP)) / (2 * eps)
    err = np.abs(fd - dS)[ok].max()
    assert err < 1e-8, err


@pytest.mark.parametrize("cal", CALS)
@pytest.mark.parametrize("mode", [ref.GRAD_DETACH, ref.GRAD_MAX_ONLY, ref.GRAD_MIN_ONLY])
def test_partial_modes_are_derivatives_of_frozen_statistics(cal, mode):
    """Detach = derivative with (m, n) frozen; max-only = n frozen; min-only =
    m frozen (first page, section 5.1 and Appendix B: dropping the extremum
    terms; keeping only the maximum- or minimum-dependent term)."""
    rng = np.random.default_rng(7 + cal + 3 * mode)
    n, L = 24, 10
    S = _rows(rng, n, L)
    Ls = np.full(n, L)
    cfg = ref.RefConfig(K=4, cal=cal, rec=ref.REC_LERP, grad=mode)
    dP = rng.standard_normal((n, L))
    ok = ~_near_kink(S, Ls, cfg, 1e-3)
    dS = ref.rows(S, Ls, cfg, dP=dP)["dS"]
    m0, n0 = S.max(1), S.min(1)
    fm = m0 if mode in (ref.GRAD_DETACH, ref.GRAD_MIN_ONLY) else None
    fn = n0 if mode in (ref.GRAD_DETACH, ref.GRAD_MAX_ONLY) else None
    eps = 1e-6
    fd = np.zeros_like(S)
    for j in range(L):
        Sp, Sm = S.copy(), S.copy()
        Sp[:, j] += eps
        Sm[:, j] -= eps
        fd[:, j] = (_loss(Sp, Ls, cfg, dP, fm, fn) - _loss(Sm, Ls, cfg, dP, fm, fn)) / (2 * eps)
    err = np.abs(fd - dS)[ok].max()
    assert err < 1e-8, err


def test_mode_identities_full_equals_max_plus_min_minus_detach():
    """Linearity of the two calibration channels (Appendix B); under FWM the
    minimum plays no role, so max-only = full and min-only = detach."""
    rng = np.random.default_rng(11)
    S = _rows(rng, 32, 20)
    Ls = rng.integers(1, 21, size=32)
    dP = rng.standard_normal(S.shape)
    for rec, ste in RECSTE:
        base = ref.RefConfig(K=4, cal=ref.CAL_MINMAX, rec=rec, ste=ste)
        g = {m: ref.rows(S, Ls, base.replace(grad=m), dP=dP)["dS"] for m in MODES[:4]}
        np.testing.assert_allclose(g[0], g[2] + g[3] - g[1], atol=1e-12)
        base = base.replace(cal=ref.CAL_FWM)
        g = {m: ref.rows(S, Ls, base.replace(grad=m), dP=dP)["dS"] for m in MODES[:4]}
        np.testing.assert_array_equal(g[ref.GRAD_MAX_ONLY], g[ref.GRAD_FULL])
        np.testing.assert_array_equal(g[ref.GRAD_MIN_ONLY], g[ref.GRAD_DETACH])


# --------------------------------------------------------------- zero sum

@pytest.mark.parametrize("cal", CALS)
@pytest.mark.parametrize("rec,ste", RECSTE)
def test_zero_sum_full_and_projection_and_detach_breaks_it(cal, rec, ste):
    """Section 3 / Appendix B: the full calibration gradient gives a zero-sum
    row gradient (shift invariance); detach violates it; projection removes
    exactly the common mode."""
    rng = np.random.default_rng(20 + cal + 2 * rec + 4 * ste)
    S = _rows(rng, 64, 48)
    Ls = rng.integers(2, 49, size=64)
    dP = rng.standard_normal(S.shape)
    base = ref.RefConfig(K=4, cal=cal, rec=rec, ste=ste)
    for mode in (ref.GRAD_FULL, ref.GRAD_PROJECT):
        dS = ref.rows(S, Ls, base.replace(grad=mode), dP=dP)["dS"]
        norms = np.linalg.norm(dS, axis=1)
        assert np.all(np.abs(dS.sum(1)) <= 1e-12 * np.maximum(norms, 1e-300) + 1e-300)
    det = ref.rows(S, Ls, base.replace(grad=ref.GRAD_DETACH), dP=dP)
    sums = np.abs(det["dS"].sum(1))
    nrm = np.linalg.norm(det["dS"], axis=1)
    assert np.median(sums[nrm > 0] / nrm[nrm > 0]) > 1e-4
    proj = ref.rows(S, Ls, base.replace(grad=ref.GRAD_PROJECT), dP=dP)["dS"]
    for i in range(S.shape[0]):
        L = Ls[i]
        np.testing.assert_allclose(proj[i, :L], det["dS"][i, :L] - det["dS"][i, :L].mean(),
                                   atol=1e-13)
    # A (row sum of dw * a) equals -h * (row sum of the detached gradient)
    st = det["stats"]
    np.testing.assert_allclose(-st[:, ref.ST_A] / st[:, ref.ST_H], det["dS"].sum(1), atol=1e-11)


# ------------------------------------------------------- same forward

def test_forward_identical_across_modes_and_surrogates():
    """First page and section 5.1: detach and projection leave the forward
    bitwise unchanged; Appendix B: both STEs share the hard forward."""
    rng = np.random.default_rng(3)
    S = _rows(rng, 40, 33)
    Ls = rng.integers(1, 34, size=40)
    for cal in CALS:
        for rec in (ref.REC_LERP, ref.REC_NEAREST):
            Ps = [ref.rows(S, Ls, ref.RefConfig(K=4, cal=cal, rec=rec, ste=ste, grad=g))["P"]
                  for g in MODES for ste in (ref.STE_WEIGHT, ref.STE_PROB)]
            for P in Ps[1:]:
                np.testing.assert_array_equal(P, Ps[0])


def test_ste_coincidence_when_scores_sit_on_nodes():
    """Figure 1 / section 3: the two STE rules coincide when the hard and
    interpolated weights agree (every score on a grid node)."""
    rng = np.random.default_rng(4)
    K = 4
    for cal, h in ((ref.CAL_FWM, 1.5), (ref.CAL_MINMAX, 1.25)):
        r = rng.integers(0, K + 1, size=(30, 16))
        r[:, 0] = 0
        r[:, 1] = K
        S = -h * r.astype(float)
        Ls = np.full(30, 16)
        dP = rng.standard_normal(S.shape)
        base = ref.RefConfig(K=K, cal=cal, tau=6.0)
        for mode in MODES:
            a = ref.rows(S, Ls, base.replace(rec=ref.REC_LERP, grad=mode), dP=dP)
            b = ref.rows(S, Ls, base.replace(rec=ref.REC_NEAREST, ste=ref.STE_WEIGHT, grad=mode), dP=dP)
            c = ref.rows(S, Ls, base.replace(rec=ref.REC_NEAREST, ste=ref.STE_PROB, grad=mode), dP=dP)
            np.testing.assert_allclose(a["P"], b["P"], atol=1e-14)
            np.testing.assert_allclose(b["dS"], c["dS"], atol=1e-12)
            np.testing.assert_allclose(a["dS"], b["dS"], atol=1e-12)


def test_ste_rules_differ_off_nodes():
    """Appendix B: the centering distributions and normalisation factors of
    the two STE rules differ in general."""
    rng = np.random.default_rng(5)
    S = _rows(rng, 20, 30)
    Ls = np.full(20, 30)
    dP = rng.standard_normal(S.shape)
    b = ref.rows(S, Ls, ref.RefConfig(K=4, rec=ref.REC_NEAREST, ste=ref.STE_WEIGHT), dP=dP)
    c = ref.rows(S, Ls, ref.RefConfig(K=4, rec=ref.REC_NEAREST, ste=ref.STE_PROB), dP=dP)
    np.testing.assert_array_equal(b["P"], c["P"])
    assert np.abs(b["dS"] - c["dS"]).max() > 1e-3


# --------------------------------------------------------- softmax limit

def test_lerp_chord_lies_above_exponential_and_bounds():
    """Convexity of e^z: the LERP chord is >= e^{s-m} with equality at nodes,
    and within the chord's worst-case ratio; Nearest is within e^{h/2}."""
    rng = np.random.default_rng(6)
    S = _rows(rng, 30, 64)
    Ls = np.full(30, 64)
    for K in (2, 4, 16):
        cfg = ref.RefConfig(K=K, cal=ref.CAL_MINMAX)
        out = ref.rows(S, Ls, cfg)
        st = out["stats"]
        z = S - st[:, [ref.ST_M]]
        wL = out["P_L"] * st[:, [ref.ST_WL]]
        wN = out["P_N"] * st[:, [ref.ST_WN]]
        e = np.exp(z)
        assert np.all(wL >= e * (1 - 1e-14))
        h = st[:, [ref.ST_H]]
        tt = np.linspace(0, 1, 2001)[None, :]
        worst = ((1 - tt) + tt * np.exp(-h)) * np.exp(tt * h)
        bound = worst.max(1, keepdims=True) - 1
        assert np.all(np.abs(wL / e - 1) <= bound * (1 + 1e-12) + 1e-14)
        assert np.all(np.abs(wN / e - 1) <= (np.exp(h / 2) - 1) * (1 + 1e-12) + 1e-14)


def test_lerp_approaches_softmax_as_K_grows():
    """Section 5.3 (LERP gap closes with K) made exact: the probability error
    shrinks ~K^-2 and the full gradient approaches softmax's ~K^-1."""
    rng = np.random.default_rng(8)
    S = _rows(rng, 20, 50, 5, 20)
    Ls = np.full(20, 50)
    dP = rng.standard_normal(S.shape)
    sm = ref.rows(S, Ls, ref.RefConfig(softmax=True), dP=dP)
    errs, gerrs = [], []
    for K in (4, 16, 64, 256):
        o = ref.rows(S, Ls, ref.RefConfig(K=K, cal=ref.CAL_MINMAX), dP=dP)
        errs.append(np.abs(o["P"] - sm["P"]).max())
        gerrs.append(np.abs(o["dS"] - sm["dS"]).max())
    r = np.array(errs[:-1]) / np.array(errs[1:])
    assert np.all((r > 8) & (r < 24)), r
    g = np.array(gerrs[:-1]) / np.array(gerrs[1:])
    assert np.all(g > 1.5) and gerrs[0] / gerrs[-1] > 30, g
    assert errs[-1] < 1e-3


def test_softmax_row_matches_numpy_softmax():
    """Appendix G: softmax runs use softmax itself and its own backward."""
    rng = np.random.default_rng(9)
    S = rng.standard_normal((10, 17)) * 3
    Ls = np.full(10, 17)
    dP = rng.standard_normal(S.shape)
    o = ref.rows(S, Ls, ref.RefConfig(softmax=True), dP=dP)
    e = np.exp(S - S.max(1, keepdims=True))
    P = e / e.sum(1, keepdims=True)
    np.testing.assert_allclose(o["P"], P, rtol=1e-14)
    J = np.einsum("ij,jk->ijk", P, np.eye(17)) - np.einsum("ij,ik->ijk", P, P)
    np.testing.assert_allclose(o["dS"], np.einsum("ijk,ij->ik", J, dP), atol=1e-14)


# ------------------------------------------------------------ closed forms

def test_K1_minmax_lerp_is_linear_in_the_score():
    """Section 2 (LERP at K = 1): with one interval the weight is the chord
    1 - (1 - e^{-span}) (m - s)/span."""
    rng = np.random.default_rng(10)
    S = _rows(rng, 10, 25, 0.5, 5.0)
    Ls = np.full(10, 25)
    o = ref.rows(S, Ls, ref.RefConfig(K=1, cal=ref.CAL_MINMAX))
    m, n = S.max(1, keepdims=True), S.min(1, keepdims=True)
    span = m - n
    w = 1 - (1 - np.exp(-span)) * (m - S) / span
    np.testing.assert_allclose(o["P"], w / w.sum(1, keepdims=True), rtol=1e-13)


def test_hand_worked_fwm_row():
    """FWM, K = 4, tau = 6 (h = 1.5): scores 0, -1.5, -3, -0.75, -10 give
    u = 0, 1, 2, 1/2 and a tail key; LERP weights 1, e^-1.5, e^-3,
    (1 + e^-1.5)/2, 0; Nearest rounds u = 1/2 up to node 1."""
    S = np.array([[0.0, -1.5, -3.0, -0.75, -10.0]])
    e1, e2 = math.exp(-1.5), math.exp(-3.0)
    wl = np.array([1.0, e1, e2, (1 + e1) / 2, 0.0])
    wn = np.array([1.0, e1, e2, e1, 0.0])
    o = ref.rows(S, [5], ref.RefConfig(K=4, cal=ref.CAL_FWM, tau=6.0, rec=ref.REC_LERP))
    np.testing.assert_allclose(o["P"][0], wl / wl.sum(), rtol=1e-15)
    o = ref.rows(S, [5], ref.RefConfig(K=4, cal=ref.CAL_FWM, tau=6.0, rec=ref.REC_NEAREST))
    np.testing.assert_allclose(o["P"][0], wn / wn.sum(), rtol=1e-15)


def test_hand_worked_fixed_step_row():
    """The same row under the untruncated fixed step (Appendix D.4): the key
    FWM drops (s = -10, u = 6 2/3) keeps the LERP weight between nodes 6 and
    7, (1/3) e^-9 + (2/3) e^-10.5, and Nearest rounds it to node 7; the
    in-window keys keep FWM's weights."""
    S = np.array([[0.0, -1.5, -3.0, -0.75, -10.0]])
    e1, e2 = math.exp(-1.5), math.exp(-3.0)
    tail_l = math.exp(-9.0) / 3 + 2 * math.exp(-10.5) / 3
    wl = np.array([1.0, e1, e2, (1 + e1) / 2, tail_l])
    wn = np.array([1.0, e1, e2, e1, math.exp(-10.5)])
    o = ref.rows(S, [5], ref.RefConfig(K=4, cal=ref.CAL_FIXED, tau=6.0, rec=ref.REC_LERP))
    np.testing.assert_allclose(o["P"][0], wl / wl.sum(), rtol=1e-14)
    o = ref.rows(S, [5], ref.RefConfig(K=4, cal=ref.CAL_FIXED, tau=6.0, rec=ref.REC_NEAREST))
    np.testing.assert_allclose(o["P"][0], wn / wn.sum(), rtol=1e-14)


def _linear_scan_forward(s, K, cal, tau, rec):
    """Second forward: find the bracketing nodes by scanning node scores
    m - k h from the top, no floor()."""
    m, n = s.max(), s.min()
    h = (m - n) / K if cal == ref.CAL_MINMAX else tau / K
    # the untruncated fixed step (Appendix D.4) continues the grid down to n
    Kn = max(K, math.ceil((m - n) / h)) if cal == ref.CAL_FIXED else K
    nodes = m - h * np.arange(Kn + 1)
    w = np.zeros_like(s)
    for j, x in enumerate(s):
        if cal == ref.CAL_FWM and x < nodes[K] - 1e-15 * max(1, abs(x)):
            continue
        k = 0
        while k < Kn - 1 and x < nodes[k + 1]:
            k += 1
        lo, hi = nodes[k], nodes[k + 1]
        t = (lo - x) / (lo - hi)
        ga, gb = math.exp(nodes[k] - m), math.exp(nodes[k + 1] - m)
        if rec == ref.REC_LERP:
            w[j] = ga + t * (gb - ga)
        else:
            w[j] = gb if t >= 0.5 else ga
    return w / w.sum()


@pytest.mark.parametrize("cal", CALS)
@pytest.mark.parametrize("rec", [ref.REC_LERP, ref.REC_NEAREST])
def test_brute_force_linear_scan_forward(cal, rec):
    """Tiny rows (T <= 8) through an independent node scan."""
    rng = np.random.default_rng(12 + cal + 2 * rec)
    for L in range(2, 9):
        S = _rows(rng, 20, L, 1.0, 12.0)
        o = ref.rows(S, np.full(20, L), ref.RefConfig(K=3, cal=cal, tau=6.0, rec=rec))
        ok = ~_near_kink(S, np.full(20, L), ref.RefConfig(K=3, cal=cal, tau=6.0, rec=rec), 1e-6)
        for i in np.nonzero(ok)[0]:
            np.testing.assert_allclose(o["P"][i], _linear_scan_forward(S[i], 3, cal, 6.0, rec),
                                       rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("mode", MODES)
def test_brute_force_jacobian_composition(mode):
    """Tiny rows: dS = J_w^T (dw), with J_w the finite-difference Jacobian of
    the LERP weights (statistics frozen per mode) and dw the normalisation
    Jacobian at the surrogate's point (Appendix B), for all three
    reconstruction/surrogate placements."""
    rng = np.random.default_rng(30 + mode)
    L = 6
    S = _rows(rng, 8, L, 2.0, 10.0)
    Ls = np.full(8, L)
    dP = rng.standard_normal(S.shape)
    for cal in CALS:
        for rec, ste in RECSTE:
            cfg = ref.RefConfig(K=3, cal=cal, rec=rec, ste=ste, grad=mode)
            ok = ~_near_kink(S, Ls, cfg, 1e-3)
            out = ref.rows(S, Ls, cfg, dP=dP)
            st = out["stats"]
            lcfg = cfg.replace(rec=ref.REC_LERP)
            m0, n0 = S.max(1), S.min(1)
            live_m = mode in (ref.GRAD_FULL, ref.GRAD_MAX_ONLY)
            live_n = mode in (ref.GRAD_FULL, ref.GRAD_MIN_ONLY)
            fm = None if live_m else m0
            fn = None if live_n else n0

            def wl(SS):
                o = ref.rows(SS, Ls, lcfg, frozen_m=fm, frozen_n=fn)
                return o["P_L"] * o["stats"][:, [ref.ST_WL]]
            eps = 1e-6
            J = np.zeros((8, L, L))   # J[i, j, k] = d w_k / d s_j
            for j in range(L):
                Sp, Sm = S.copy(), S.copy()
                Sp[:, j] += eps
                Sm[:, j] -= eps
                J[:, j, :] = (wl(Sp) - wl(Sm)) / (2 * eps)
            if rec == ref.REC_LERP or ste == ref.STE_PROB:
                Pb, Wb = out["P_L"], st[:, [ref.ST_WL]]
            else:
                Pb, Wb = out["P_N"], st[:, [ref.ST_WN]]
            D = (Pb * dP).sum(1, keepdims=True)
            dw = (dP - D) / Wb
            dS = np.einsum("ijk,ik->ij", J, dw)
            if mode == ref.GRAD_PROJECT:
                dS = dS - dS.mean(1, keepdims=True)
            err = np.abs(dS - out["dS"])[ok]
            assert err.size == 0 or err.max() < 1e-7, (cal, rec, ste, err.max())


# ------------------------------------------------------------ degenerate

def test_degenerate_and_edge_rows_are_finite():
    """Appendix A / Table S1: spans below eps = 1e-12 take a separate branch;
    forward and backward stay finite.  Degenerate rows are uniform and get
    the softmax Jacobian at uniform P, (dP - mean dP)/|J|, in every mode."""
    g = _golden()
    eps = g["eps_span"]
    rows = [
        np.array([0.3]),
        np.full(7, -2.0),
        np.array([1.0, 1.0 + 0.5 * eps, 1.0]),
        np.array([0.0, 2 * eps, 0.0, eps]),
        np.array([5.0, -5.0, 5.0, -5.0]),
        np.array([0.0, -1e3, -1e4]),
    ]
    L = max(len(r) for r in rows)
    S = np.zeros((len(rows), L))
    Ls = np.array([len(r) for r in rows])
    for i, r in enumerate(rows):
        S[i, :len(r)] = r
    rng = np.random.default_rng(13)
    dP = rng.standard_normal(S.shape)
    for cal in CALS:
        for rec, ste in RECSTE:
            for mode in MODES:
                o = ref.rows(S, Ls, ref.RefConfig(K=4, cal=cal, rec=rec, ste=ste, grad=mode), dP=dP)
                assert np.all(np.isfinite(o["P"])) and np.all(np.isfinite(o["dS"]))
                np.testing.assert_allclose(o["P"].sum(1), 1.0, rtol=1e-14)
                if cal == ref.CAL_MINMAX:
                    for i in (0, 1, 2):
                        Li = Ls[i]
                        np.testing.assert_allclose(o["P"][i, :Li], 1.0 / Li, rtol=1e-15)
                        exp = (dP[i, :Li] - dP[i, :Li].mean()) / Li
                        np.testing.assert_allclose(o["dS"][i, :Li], exp, atol=1e-15)
                    # span 2e-12 is above eps: not degenerate
                    assert o["stats"][3, ref.ST_DEGEN] == 0


def test_fwm_tail_has_zero_weight_and_zero_gradient():
    """Section 3 / Appendix B: FWM gives keys below m - tau zero weight and
    zero gradient through the mask and clamp."""
    rng = np.random.default_rng(14)
    S = _rows(rng, 30, 40, 10, 40)
    Ls = np.full(30, 40)
    dP = rng.standard_normal(S.shape)
    for rec, ste in RECSTE:
        for mode in MODES[:4]:
            o = ref.rows(S, Ls, ref.RefConfig(K=4, cal=ref.CAL_FWM, tau=6.0, rec=rec, ste=ste,
                                               grad=mode), dP=dP)
            tail = S < S.max(1, keepdims=True) - 6.0
            assert tail.sum() > 100
            assert np.all(o["P"][tail] == 0.0)
            assert np.all(o["dS"][tail] == 0.0)


# ------------------------------------------- attention-level composition

@pytest.mark.parametrize("causal", [True, False])
def test_attention_composes_rows_with_numpy_contractions(causal):
    """Appendix A: S = Q K^T per causal row, O = P V; the backward takes
    dP = dO V^T, dQ = dS K, dK = dS^T Q, dV = P^T dO."""
    rng = np.random.default_rng(15)
    B, H, T, d = 1, 2, 24, 8
    Q = (rng.standard_normal((B, H, T, d)) * 0.7).astype(np.float32)
    K = rng.standard_normal((B, H, T, d)).astype(np.float32)
    V = rng.standard_normal((B, H, T, d)).astype(np.float32)
    dO = rng.standard_normal((B, H, T, d)).astype(np.float32)
    for cal in CALS:
        for rec, ste in RECSTE:
            cfg = ref.RefConfig(K=4, cal=cal, rec=rec, ste=ste, causal=causal)
            out = ref.attention(Q, K, V, dO, cfg, dump=True)
            for b in range(B):
                for hh in range(H):
                    q, k, v, g = (x[b, hh].astype(np.float64) for x in (Q, K, V, dO))
                    S = q @ k.T
                    Ls = np.arange(1, T + 1) if causal else np.full(T, T)
                    dP = g @ v.T
                    r = ref.rows(S, Ls, cfg, dP=dP)
                    np.testing.assert_allclose(out["P"][b, hh], r["P"], atol=1e-14)
                    np.testing.assert_allclose(out["O"][b, hh], r["P"] @ v, atol=1e-12)
                    np.testing.assert_allclose(out["dS"][b, hh], r["dS"], atol=1e-12)
                    np.testing.assert_allclose(out["dQ"][b, hh], r["dS"] @ k, atol=1e-11)
                    np.testing.assert_allclose(out["dK"][b, hh], r["dS"].T @ q, atol=1e-11)
                    np.testing.assert_allclose(out["dV"][b, hh], r["P"].T @ g, atol=1e-11)


def test_attention_operand_rounding_rules():
    """TF32 emulation: operands keep 10 mantissa bits; truncation, ties-away
    and ties-to-even differ exactly on the crafted values."""
    T, d = 1, 1
    one = np.ones((1, 1, T, d), np.float32)
    cases = {
        # value: (trunc, rna, rne)
        1.0 + 2.0 ** -11: (1.0, 1.0 + 2.0 ** -10, 1.0),
        1.0 + 3 * 2.0 ** -11: (1.0 + 2.0 ** -10, 1.0 + 2.0 ** -9, 1.0 + 2.0 ** -9),
        1.0 + 2.0 ** -12: (1.0, 1.0, 1.0),
        -(1.0 + 2.0 ** -11 + 2.0 ** -20): (-1.0, -(1.0 + 2.0 ** -10), -(1.0 + 2.0 ** -10)),
    }
    for x, exp in cases.items():
        q = np.full((1, 1, T, d), x, np.float32)
        for mode, e in zip((ref.ROUND_TRUNC, ref.ROUND_RNA, ref.ROUND_RNE), exp):
            st = ref.attention(q, one, one, one, ref.RefConfig(rounding=mode))["stats"]
            assert st[0, 0, 0, ref.ST_M] == e, (x, mode)


# ------------------------------------------------- fp32 weight stage

def test_own_exp_matches_libm_to_the_last_fp32_bit():
    """The fp32 grid G_k = RN32(e^{-k h}): the oracle's own fp64 exponential,
    rounded to fp32, equals libm's exp rounded to fp32."""
    rng = np.random.default_rng(16)
    xs = np.concatenate([-rng.uniform(0, 104, 20000), -np.arange(0, 104, 0.125),
                         -rng.uniform(0, 1e-6, 200)])
    for x in xs:
        a = np.float32(ref.own_exp(x))
        b = np.float32(math.exp(x))
        assert a == b, x
        assert abs(ref.own_exp(x) - math.exp(x)) <= 4e-16 * math.exp(x) + 1e-300
    assert np.float32(ref.own_exp(-200.0)) == 0.0


@pytest.mark.parametrize("cal", CALS)
@pytest.mark.parametrize("rec", [ref.REC_LERP, ref.REC_NEAREST])
def test_fp32_weight_stage_tracks_fp64(cal, rec):
    """The fp32 weight stage agrees with the fp64 method on the same scores
    (bins equal away from boundaries; weights to fp32 precision)."""
    rng = np.random.default_rng(17 + cal + 2 * rec)
    S = _rows(rng, 64, 200, 2, 60).astype(np.float32)
    Ls = rng.integers(1, 201, size=64).astype(np.int32)
    for K in (1, 4, 16, 64):
        cfg = ref.RefConfig(K=K, cal=cal, rec=rec, tau=6.0)
        f = ref.weights_fp32(S, Ls, cfg)
        o = ref.rows(S.astype(np.float64), Ls, cfg)
        st = o["stats"]
        w64 = (o["P_L"] if rec == ref.REC_LERP else o["P_N"]) * (
            st[:, [ref.ST_WL]] if rec == ref.REC_LERP else st[:, [ref.ST_WN]])
        np.testing.assert_array_equal(f["m"], S.max(1, where=np.arange(200)[None] < Ls[:, None],
                                                    initial=-np.inf))
        h = st[:, [ref.ST_H]]
        u = (st[:, [ref.ST_M]] - S) / h
        near = np.abs(u - np.round(u * 2) / 2) < 1e-3
        mask = (np.arange(200)[None] < Ls[:, None]) & ~near
        err = np.abs(f["w"] - w64)[mask]
        assert err.max() <= 2e-6 * max(1.0, K / 4), (K, err.max())
        if rec == ref.REC_NEAREST:
            assert np.all(f["w"][mask] == w64[mask].astype(np.float32)) or err.max() < 1e-7


# --------------------------------------- fixed-upstream decomposition

def _decomp_inputs(seed, B=1, H=2, T=20, d=8):
    rng = np.random.default_rng(seed)
    Q = (rng.standard_normal((B, H, T, d)) * 1.5).astype(np.float32)
    K = rng.standard_normal((B, H, T, d)).astype(np.float32)
    V = rng.standard_normal((B, H, T, d)).astype(np.float32)
    dO = rng.standard_normal((B, H, T, d)).astype(np.float32)
    return Q, K, V, dO


@pytest.mark.parametrize("causal", [True, False])
def test_decomposition_max_and_min_terms_are_extremum_derivatives(causal):
    """Appendix F, fixed-upstream decomposition (Table S24): at a fixed
    upstream dP = dO V^T the maximum-dependent term is the derivative of the
    row loss sum_j P_ij dP_ij with respect to the row maximum m_i (minimum
    frozen), the minimum-dependent term the derivative with respect to n_i;
    both checked by central differences of the LERP forward with the other
    extremum frozen."""
    Q, K, V, dO = _decomp_inputs(21)
    T = Q.shape[2]
    for cal in CALS:
        cfg = ref.RefConfig(K=4, cal=cal, rec=ref.REC_LERP, causal=causal)
        dec = ref.grad_decomposition(Q, K, V, dO, cfg)
        for hh in range(Q.shape[1]):
            q, k, v, g = (x[0, hh].astype(np.float64) for x in (Q, K, V, dO))
            S, dP = q @ k.T, g @ v.T
            Ls = np.arange(1, T + 1) if causal else np.full(T, T)
            Sm = np.where(np.arange(T)[None, :] < Ls[:, None], S, -np.inf)
            Sn = np.where(np.arange(T)[None, :] < Ls[:, None], S, np.inf)
            m0, n0 = Sm.max(1), Sn.min(1)
            ok = ~_near_kink(S, Ls, cfg, 1e-3) & (Ls >= 3)
            assert ok.sum() >= T // 2
            eps = 1e-6
            d_m = (_loss(S, Ls, cfg, dP, m0 + eps, n0) - _loss(S, Ls, cfg, dP, m0 - eps, n0)) / (2 * eps)
            d_n = (_loss(S, Ls, cfg, dP, m0, n0 + eps) - _loss(S, Ls, cfg, dP, m0, n0 - eps)) / (2 * eps)
            np.testing.assert_allclose(dec[hh, :, 1][ok], (d_m ** 2)[ok], rtol=1e-6, atol=1e-12)
            np.testing.assert_allclose(dec[hh, :, 2][ok], (d_n ** 2)[ok], rtol=1e-6, atol=1e-12)
            if cal == ref.CAL_FWM:
                assert np.all(dec[hh, :, 2] == 0.0)


@pytest.mark.parametrize("rec,ste", RECSTE)
def test_decomposition_modes_split_the_full_terms(rec, ste):
    """The terms a partial mode keeps are the full mode's own (Appendix B:
    max-only keeps the maximum-dependent term, min-only the minimum one,
    detach neither), ||dS||^2 is the squared norm of the mode's dump, and
    under the zero-sum projection the maximum slot holds |J_i| c_i^2 with
    c_i minus the mean of the detached row (the dump's rows then sum to zero)."""
    Q, K, V, dO = _decomp_inputs(22)
    for cal in CALS:
        base = ref.RefConfig(K=4, cal=cal, rec=rec, ste=ste)
        dec = {m: ref.grad_decomposition(Q, K, V, dO, base.replace(grad=m)) for m in MODES}
        full = dec[ref.GRAD_FULL]
        np.testing.assert_array_equal(dec[ref.GRAD_MAX_ONLY][..., 1], full[..., 1])
        np.testing.assert_array_equal(dec[ref.GRAD_MAX_ONLY][..., 2], 0.0)
        np.testing.assert_array_equal(dec[ref.GRAD_MIN_ONLY][..., 2], full[..., 2])
        np.testing.assert_array_equal(dec[ref.GRAD_MIN_ONLY][..., 1], 0.0)
        np.testing.assert_array_equal(dec[ref.GRAD_DETACH][..., 1:], 0.0)
        T = Q.shape[2]
        for m in MODES:
            dS = ref.attention(Q, K, V, dO, base.replace(grad=m), dump=True)["dS"][0]
            np.testing.assert_allclose(dec[m][..., 0], np.einsum("htj,htj->ht", dS, dS),
                                       rtol=1e-12)
        det = ref.attention(Q, K, V, dO, base.replace(grad=ref.GRAD_DETACH), dump=True)["dS"][0]
        Ls = np.arange(1, T + 1)
        c = -det.sum(-1) / Ls
        np.testing.assert_allclose(dec[ref.GRAD_PROJECT][..., 1], c * c * Ls, rtol=1e-10,
                                   atol=1e-30)
        np.testing.assert_array_equal(dec[ref.GRAD_PROJECT][..., 2], 0.0)
        # a full-mode row's calibration norm splits into its two extremum terms
        dfull = ref.attention(Q, K, V, dO, base, dump=True)["dS"][0]
        diff = dfull - det
        np.testing.assert_allclose(full[..., 1] + full[..., 2], np.sum(diff * diff, -1),
                                   rtol=1e-10, atol=1e-30)


def test_decomposition_closed_forms_from_row_statistics():
    """Appendix B closed forms: MinMax g_m = A/h + C/K, g_n = -C/K; FWM
    g_m = A/h, g_n = 0, with A, C the row sums the backward records."""
    Q, K, V, dO = _decomp_inputs(23)
    for cal in CALS:
        for rec, ste in RECSTE:
            cfg = ref.RefConfig(K=4, cal=cal, rec=rec, ste=ste)
            dec = ref.grad_decomposition(Q, K, V, dO, cfg)
            st = ref.attention(Q, K, V, dO, cfg)["stats"][0]
            live = st[..., ref.ST_DEGEN] == 0
            A, C, h = st[..., ref.ST_A], st[..., ref.ST_C], st[..., ref.ST_H]
            hs = np.where(live, h, 1.0)
            if cal == ref.CAL_MINMAX:
                gm, gn = A / hs + C / cfg.K, -C / cfg.K
            else:
                gm, gn = A / hs, np.zeros_like(A)
            np.testing.assert_allclose(dec[..., 1][live], (gm * gm)[live], rtol=1e-9, atol=1e-28)
            np.testing.assert_allclose(dec[..., 2][live], (gn * gn)[live], rtol=1e-9, atol=1e-28)
            np.testing.assert_array_equal(dec[..., 1:][~live], 0.0)


# ------------------------------------------ untruncated fixed step

@pytest.mark.parametrize("rec,ste", RECSTE)
@pytest.mark.parametrize("mode", MODES)
def test_fixed_step_is_fwm_with_a_window_covering_the_span(rec, ste, mode):
    """Appendix D.4: the untruncated fixed-step operator keeps FWM's step
    h = tau / K but drops the tail cut, so it equals FWM with K' = 64 K
    intervals over a window tau' = 64 tau (the same h) wide enough to hold
    every row's span; on rows whose span is within tau it equals FWM itself."""
    rng = np.random.default_rng(31 + 5 * mode + rec + ste)
    S = _rows(rng, 40, 24, 1.0, 60.0)
    Ls = rng.integers(1, 25, 40)
    dP = rng.standard_normal(S.shape)
    fixed = ref.rows(S, Ls, ref.RefConfig(K=4, cal=ref.CAL_FIXED, tau=6.0, rec=rec, ste=ste,
                                          grad=mode), dP=dP)
    wide = ref.rows(S, Ls, ref.RefConfig(K=256, cal=ref.CAL_FWM, tau=384.0, rec=rec, ste=ste,
                                         grad=mode), dP=dP)
    np.testing.assert_allclose(fixed["P"], wide["P"], rtol=1e-13, atol=1e-300)
    np.testing.assert_allclose(fixed["dS"], wide["dS"], rtol=1e-12, atol=1e-14)
    fwm = ref.rows(S, Ls, ref.RefConfig(K=4, cal=ref.CAL_FWM, tau=6.0, rec=rec, ste=ste,
                                        grad=mode), dP=dP)
    span = fixed["stats"][:, ref.ST_M] - fixed["stats"][:, ref.ST_N]
    inside = span < 6.0 - 1e-9
    assert inside.any() and (~inside).any()
    np.testing.assert_array_equal(fixed["P"][inside], fwm["P"][inside])
    np.testing.assert_array_equal(fixed["dS"][inside], fwm["dS"][inside])
    # past the window FWM puts no mass, the fixed step keeps e^{-k h}-scale weight
    out = ~inside
    assert np.all(fixed["P"][out].sum(1) == pytest.approx(1.0))
    tail = (S[out] < (fixed["stats"][out, ref.ST_M] - 6.0 - 1e-9)[:, None]) & \
        (np.arange(24)[None] < Ls[out][:, None])
    assert np.all(fixed["P"][out][tail] > 0) and np.all(fwm["P"][out][tail] == 0)
