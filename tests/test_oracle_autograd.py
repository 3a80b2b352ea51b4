"""Independent restatement of the operator in PyTorch fp64 autograd (CPU).

Appendix B of "Pretraining Transformers with Quantized Softmax in Attention"
reports that its closed-form gradients agree with automatic differentiation
to < 1e-9.  This test repeats that check on the oracle: the forward below is
written from the section 3 / Appendix A description with the statistics
detached per gradient mode and the straight-through estimators placed as the
paper describes (Weight-STE before normalisation, Prob-STE after); autograd
supplies the derivative.  It shares nothing with the oracle's C code.
"""
import numpy as np
import pytest
import torch

import oracle as ref

MODES = [ref.GRAD_FULL, ref.GRAD_DETACH, ref.GRAD_MAX_ONLY, ref.GRAD_MIN_ONLY, ref.GRAD_PROJECT]


def autograd_row(s_np, dP_np, K, cal, tau, rec, ste, mode):
    s = torch.tensor(s_np, dtype=torch.float64, requires_grad=True)
    dP = torch.tensor(dP_np, dtype=torch.float64)
    m = s.max()
    n = s.min()
    if mode in (ref.GRAD_DETACH, ref.GRAD_MIN_ONLY, ref.GRAD_PROJECT):
        m = m.detach()
    if mode in (ref.GRAD_DETACH, ref.GRAD_MAX_ONLY, ref.GRAD_PROJECT):
        n = n.detach()
    h = (m - n) / K if cal == ref.CAL_MINMAX else torch.tensor(tau / K, dtype=torch.float64)
    u = (m - s) / h
    # the untruncated fixed step (Appendix D.4) keeps counting nodes past K
    k_hi = float("inf") if cal == ref.CAL_FIXED else K - 1
    k = torch.clamp(torch.floor(u.detach()), min=0, max=k_hi)
    t = u - k
    g_lo = torch.exp(-k * h)
    g_hi = torch.exp(-(k + 1) * h)
    w_lerp = g_lo + t * (g_hi - g_lo)
    w_near = torch.where(t.detach() >= 0.5, g_hi, g_lo).detach()
    if cal == ref.CAL_FWM:
        keep = (u.detach() <= K).to(torch.float64)
        w_lerp = w_lerp * keep
        w_near = w_near * keep
    if rec == ref.REC_LERP:
        P = w_lerp / w_lerp.sum()
    elif ste == ref.STE_WEIGHT:
        w = w_lerp + (w_near - w_lerp).detach()
        P = w / w.sum()
    else:
        P_l = w_lerp / w_lerp.sum()
        P_n = w_near / w_near.sum()
        P = P_l + (P_n - P_l).detach()
    (P * dP).sum().backward()
    g = s.grad.numpy().copy()
    if mode == ref.GRAD_PROJECT:
        g = g - g.mean()
    return P.detach().numpy(), g


@pytest.mark.parametrize("cal", [ref.CAL_MINMAX, ref.CAL_FWM, ref.CAL_FIXED])
@pytest.mark.parametrize("rec,ste", [(ref.REC_LERP, ref.STE_WEIGHT),
                                     (ref.REC_NEAREST, ref.STE_WEIGHT),
                                     (ref.REC_NEAREST, ref.STE_PROB)])
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("K", [1, 4, 32])
def test_closed_form_matches_autograd(cal, rec, ste, mode, K):
    rng = np.random.default_rng(100 + 7 * cal + 3 * rec + ste + 11 * mode + K)
    n, L = 12, 37
    S = rng.standard_normal((n, L)) * rng.uniform(0.5, 8.0, size=(n, 1))
    Ls = rng.integers(2, L + 1, size=n)
    dP = rng.standard_normal((n, L))
    cfg = ref.RefConfig(K=K, cal=cal, tau=6.0, rec=rec, ste=ste, grad=mode)
    out = ref.rows(S, Ls, cfg, dP=dP)
    for i in range(n):
        Li = Ls[i]
        P, g = autograd_row(S[i, :Li], dP[i, :Li], K, cal, 6.0, rec, ste, mode)
        np.testing.assert_allclose(out["P"][i, :Li], P, rtol=1e-13, atol=1e-15)
        scale = max(1.0, np.abs(g).max())
        assert np.abs(out["dS"][i, :Li] - g).max() < 1e-9 * scale
