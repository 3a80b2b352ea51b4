"""Pins of the oracle's geometry probe ("Pretraining Transformers with
Quantized Softmax in Attention", section 4 geometry probe, section 5.4,
Appendix D.6 / Figure S4): closed forms on rows small enough to work by hand,
bounds that total variation and entropy must respect, page constants, and an
independent fp64 computation from the row operator."""
import math
import os

import numpy as np
import pytest

import oracle as ref

HERE = os.path.dirname(os.path.abspath(__file__))
CALS = [ref.CAL_MINMAX, ref.CAL_FWM]
RECS = [ref.REC_LERP, ref.REC_NEAREST]


def _page(name):
    with open(os.path.join(HERE, "golden", "page_constants.txt")) as f:
        for line in f:
            if line.startswith(name + " "):
                return float(line.split()[1])
    raise KeyError(name)


def _binary_entropy(p):
    return -(p * math.log(p) + (1 - p) * math.log(1 - p))


@pytest.mark.parametrize("K", [1, 4, 16])
@pytest.mark.parametrize("rec", RECS)
def test_two_key_row_closed_form(K, rec):
    """MinMax on s = (0, -x): the two keys sit on nodes 0 and K, so the
    operator row is (1, G_K) / (1 + G_K) with G_K = e^{-x} rounded to fp32;
    softmax is (1, e^{-x}) / (1 + e^{-x}); only key 0 is in the top bucket.
    LERP reaches node K as G_{K-1} + 1 * (G_K - G_{K-1}) in fp32, one rounding
    away from G_K, hence its looser bound."""
    x = 3.0
    S = np.array([[0.0, -x]], np.float32)
    g = ref.geometry(S, [2], ref.RefConfig(K=K, cal=ref.CAL_MINMAX, rec=rec))[0]
    GK = float(np.float32(math.exp(-x)))
    ps = 1.0 / (1.0 + math.exp(-x))
    po = 1.0 / (1.0 + GK)
    assert g[ref.GEO_SPAN] == x
    assert g[ref.GEO_H] == pytest.approx(x / K, rel=1e-15)
    assert g[ref.GEO_ENT_SOFTMAX] == pytest.approx(_binary_entropy(ps), rel=1e-13)
    assert g[ref.GEO_ENT_OP] == pytest.approx(_binary_entropy(po), rel=1e-6)
    tol = 1e-15 if rec == ref.REC_NEAREST else 1e-7
    assert g[ref.GEO_TV] == pytest.approx(abs(po - ps), abs=tol)
    assert g[ref.GEO_TV] < 1e-7
    assert g[ref.GEO_TOP_SOFTMAX] == pytest.approx(ps, rel=1e-15)
    assert g[ref.GEO_TOP_OP] == pytest.approx(po, rel=tol)


@pytest.mark.parametrize("cal", CALS)
@pytest.mark.parametrize("rec", RECS)
def test_constant_row_is_uniform(cal, rec):
    """All-equal scores: both distributions uniform, entropy log L, no
    variation, the whole row in the top bucket; MinMax takes the degenerate
    branch (h = 0)."""
    L = 7
    S = np.full((1, 9), -2.5, np.float32)
    g = ref.geometry(S, [L], ref.RefConfig(K=4, cal=cal, rec=rec))[0]
    assert g[ref.GEO_SPAN] == 0.0
    assert g[ref.GEO_H] == (0.0 if cal == ref.CAL_MINMAX else 1.5)
    for f in (ref.GEO_ENT_SOFTMAX, ref.GEO_ENT_OP):
        assert g[f] == pytest.approx(math.log(L), rel=1e-14)
    assert g[ref.GEO_TV] == pytest.approx(0.0, abs=1e-15)
    assert g[ref.GEO_TOP_SOFTMAX] == pytest.approx(1.0, rel=1e-14)
    assert g[ref.GEO_TOP_OP] == pytest.approx(1.0, rel=1e-14)


def test_native_width_page_constants():
    """Appendix A: at K = 4 FWM uses h = 1.5 nats; MinMax a quarter of the
    row span."""
    rng = np.random.default_rng(3)
    S = (rng.standard_normal((16, 40)) * rng.uniform(1, 20, (16, 1))).astype(np.float32)
    Ls = rng.integers(2, 41, 16)
    fwm = ref.geometry(S, Ls, ref.RefConfig(K=4, cal=ref.CAL_FWM, tau=_page("fwm_tau")))
    np.testing.assert_array_equal(fwm[:, ref.GEO_H], _page("fwm_K4_h"))
    mm = ref.geometry(S, Ls, ref.RefConfig(K=4, cal=ref.CAL_MINMAX))
    np.testing.assert_allclose(mm[:, ref.GEO_H], _page("minmax_K4_h_over_span") * mm[:, ref.GEO_SPAN],
                               rtol=1e-15)
    S64 = S.astype(np.float64)
    span = np.array([S64[i, :Ls[i]].max() - S64[i, :Ls[i]].min() for i in range(16)])
    np.testing.assert_array_equal(mm[:, ref.GEO_SPAN], span)


@pytest.mark.parametrize("cal", CALS)
@pytest.mark.parametrize("rec", RECS)
def test_bounds_and_independent_fp64_recomputation(cal, rec):
    """0 <= TV <= 1, 0 <= entropy <= log L, masses in [0, 1], the top bucket
    holds the row maximum; the softmax entropy equals scipy's on numpy's
    softmax, TV and the operator entropy match the fp64 row operator to the
    fp32 weight stage's rounding, and under FWM TV is at least the softmax
    mass the window drops (a set on which the operator puts no mass)."""
    from scipy.special import softmax
    from scipy.stats import entropy

    rng = np.random.default_rng(5 + cal + 2 * rec)
    rows, cols = 48, 64
    S = (rng.standard_normal((rows, cols)) * rng.uniform(0.5, 12, (rows, 1))).astype(np.float32)
    Ls = rng.integers(1, cols + 1, rows)
    cfg = ref.RefConfig(K=4, cal=cal, rec=rec)
    g = ref.geometry(S, Ls, cfg)
    assert np.all(g[:, ref.GEO_TV] >= 0) and np.all(g[:, ref.GEO_TV] <= 1)
    for f in (ref.GEO_ENT_SOFTMAX, ref.GEO_ENT_OP):
        assert np.all(g[:, f] >= -1e-15) and np.all(g[:, f] <= np.log(Ls) + 1e-12)
    for f in (ref.GEO_TOP_SOFTMAX, ref.GEO_TOP_OP):
        assert np.all(g[:, f] > 0) and np.all(g[:, f] <= 1 + 1e-12)
    P64 = ref.rows(S.astype(np.float64), Ls, cfg)["P"]
    for i in range(rows):
        s = S[i, :Ls[i]].astype(np.float64)
        psm = softmax(s)
        assert g[i, ref.GEO_ENT_SOFTMAX] == pytest.approx(entropy(psm), rel=1e-12, abs=1e-14)
        pop = P64[i, :Ls[i]]
        assert g[i, ref.GEO_TV] == pytest.approx(0.5 * np.abs(pop - psm).sum(), abs=2e-6)
        assert g[i, ref.GEO_ENT_OP] == pytest.approx(entropy(pop), abs=2e-5)
        if cal == ref.CAL_FWM:
            u = (s.max() - s) / (cfg.tau / cfg.K)
            dropped = psm[u > cfg.K + 1e-5].sum()
            assert g[i, ref.GEO_TV] >= dropped - 1e-12


@pytest.mark.parametrize("cal", CALS)
def test_top_bucket_is_within_half_a_width_of_the_maximum(cal):
    """The top rounding bucket is the set of keys with u = (m - s)/h < 1/2,
    i.e. s > m - h/2: count it directly on rows whose scores stay clear of
    that boundary."""
    rng = np.random.default_rng(9 + cal)
    rows, cols = 64, 32
    S = (rng.standard_normal((rows, cols)) * 3).astype(np.float32)
    Ls = np.full(rows, cols)
    cfg = ref.RefConfig(K=4, cal=cal, rec=ref.REC_NEAREST)
    g = ref.geometry(S, Ls, cfg)
    checked = 0
    for i in range(rows):
        s = S[i].astype(np.float64)
        m = s.max()
        h = (m - s.min()) / 4 if cal == ref.CAL_MINMAX else 1.5
        u = (m - s) / h
        if np.min(np.abs(u - 0.5)) < 1e-4:
            continue
        e = np.exp(s - m)
        want = e[u < 0.5].sum() / e.sum()
        assert g[i, ref.GEO_TOP_SOFTMAX] == pytest.approx(want, rel=1e-12)
        checked += 1
    assert checked > rows // 2


def test_qnorm_and_lerp_tv_shrinks_with_K():
    """||q_i||_2 of the given queries; LERP's distortion of softmax falls as
    K grows (section 2: the chord error shrinks with the interval width)."""
    rng = np.random.default_rng(11)
    S = (rng.standard_normal((32, 50)) * 6).astype(np.float32)
    Q = rng.standard_normal((32, 16)).astype(np.float32)
    Ls = np.full(32, 50)
    tv = []
    for K in (2, 4, 8, 16, 32):
        g = ref.geometry(S, Ls, ref.RefConfig(K=K, rec=ref.REC_LERP), Q=Q)
        np.testing.assert_allclose(g[:, ref.GEO_QNORM],
                                   np.sqrt((Q.astype(np.float64) ** 2).sum(1)), rtol=1e-15)
        tv.append(g[:, ref.GEO_TV].mean())
    assert all(a > b for a, b in zip(tv, tv[1:])), tv
    assert tv[-1] < tv[0] / 50
