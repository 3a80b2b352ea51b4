"""Pins of the oracle's reduced-precision exponential baselines
("Pretraining Transformers with Quantized Softmax in Attention", Appendix
D.5, Table S11): softmax whose numerator e^{s-m} is rounded to bfloat16 or
FP8 E4M3.  The rounding is checked against hand-worked values and against
torch's own dtype conversions; the forward and the straight-through backward
against an independent PyTorch fp64 autograd restatement."""
import math
import os

import numpy as np
import pytest
import torch

import oracle as ref

HERE = os.path.dirname(os.path.abspath(__file__))
FORMATS = {"bf16": (ref.EXP_BF16, torch.bfloat16), "fp8": (ref.EXP_FP8, torch.float8_e4m3fn)}


def _golden():
    rows = []
    with open(os.path.join(HERE, "golden", "reduced_exp_rounding.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            fmt, x, want = line.split()[:3]
            rows.append((fmt, float(x), float(want)))
    return rows


def test_rounding_hand_worked_values():
    for fmt, x, want in _golden():
        got = ref.round_exp_format(float(np.float32(x)), FORMATS[fmt][0])
        assert got == want, (fmt, x, got, want)


@pytest.mark.parametrize("fmt", sorted(FORMATS))
def test_rounding_matches_torch_dtype_conversion(fmt):
    """Nearest-even rounding to the format equals torch's conversion to it on
    random fp32 values of the numerator's range (0, 1], their exact midpoints
    and fp32 subnormals."""
    mode, dt = FORMATS[fmt]
    rng = np.random.default_rng(7)
    x = np.exp(-rng.uniform(0, 110, 20000)).astype(np.float32)
    grid = np.unique(torch.linspace(0, 1, 4097).to(dt).to(torch.float64).numpy())
    mids = ((grid[1:] + grid[:-1]) / 2).astype(np.float32)
    x = np.concatenate([x, mids[np.float64(mids) == (grid[1:] + grid[:-1]) / 2],
                        np.array([1.0, 0.0, 1e-45, 2e-40], np.float32)])
    want = torch.from_numpy(x).to(dt).to(torch.float32).numpy()
    got = np.array([ref.round_exp_format(float(v), mode) for v in x], np.float32)
    np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32))


def _autograd_row(s_np, dP_np, dt):
    """P = R(e) / sum R(e) with e = e^{s - m}, R the rounding to dt taken
    straight through (identity in the backward) and m held fixed."""
    s = torch.tensor(s_np, dtype=torch.float64, requires_grad=True)
    m = s.detach().max()
    e = torch.exp(s - m)
    r = e.detach().to(torch.float32).to(dt).to(torch.float64)
    w = e + (r - e).detach()
    P = w / w.sum()
    (P * torch.tensor(dP_np, dtype=torch.float64)).sum().backward()
    return P.detach().numpy(), s.grad.numpy()


@pytest.mark.parametrize("fmt", sorted(FORMATS))
def test_forward_and_straight_through_backward_match_autograd(fmt):
    mode, dt = FORMATS[fmt]
    rng = np.random.default_rng(11 + mode)
    n, L = 24, 40
    S = rng.standard_normal((n, L)) * rng.uniform(0.5, 6.0, (n, 1))
    Ls = rng.integers(1, L + 1, n)
    dP = rng.standard_normal((n, L))
    out = ref.rows(S, Ls, ref.RefConfig(softmax=True, exp_round=mode), dP=dP)
    for i in range(n):
        P, g = _autograd_row(S[i, :Ls[i]], dP[i, :Ls[i]], dt)
        np.testing.assert_allclose(out["P"][i, :Ls[i]], P, rtol=1e-13, atol=1e-300)
        np.testing.assert_allclose(out["dS"][i, :Ls[i]], g, rtol=1e-11, atol=1e-13)


def test_hand_worked_row():
    """s = (0, -ln 3, -8): numerators (1, 1/3, e^-8) become (1, 0.333984375,
    RN_bf16(e^-8)) and (1, 0.34375, 0) -- FP8 drops keys more than ~6.93
    nats (2^-10) below the maximum."""
    S = np.array([[0.0, -math.log(3.0), -8.0]])
    Pb = ref.rows(S, [3], ref.RefConfig(softmax=True, exp_round=ref.EXP_BF16))["P"][0]
    e8 = float(torch.tensor(math.exp(-8.0), dtype=torch.float32).to(torch.bfloat16).float())
    w = np.array([1.0, 0.333984375, e8])
    np.testing.assert_allclose(Pb, w / w.sum(), rtol=1e-15)
    Pf = ref.rows(S, [3], ref.RefConfig(softmax=True, exp_round=ref.EXP_FP8))["P"][0]
    np.testing.assert_allclose(Pf, np.array([1.0, 0.34375, 0.0]) / 1.34375, rtol=1e-15)


def test_exact_mode_is_softmax_and_rounding_breaks_zero_sum_only_slightly():
    """exp_round = 0 is numpy's softmax with the softmax Jacobian (rows of dS
    sum to zero); the rounded baselines' straight-through rows sum to
    sum_j (e_j - R(e_j)) (dP_j - D) / W, small against ||dS||."""
    rng = np.random.default_rng(3)
    S = rng.standard_normal((16, 30)) * 3
    Ls = np.full(16, 30)
    dP = rng.standard_normal(S.shape)
    ex = ref.rows(S, Ls, ref.RefConfig(softmax=True), dP=dP)
    P = np.exp(S - S.max(1, keepdims=True))
    P /= P.sum(1, keepdims=True)
    np.testing.assert_allclose(ex["P"], P, rtol=1e-14)
    D = (P * dP).sum(1, keepdims=True)
    np.testing.assert_allclose(ex["dS"], P * (dP - D), atol=1e-15)
    for mode, rel in ((ref.EXP_BF16, 2e-2), (ref.EXP_FP8, 0.3)):
        o = ref.rows(S, Ls, ref.RefConfig(softmax=True, exp_round=mode), dP=dP)
        sums = np.abs(o["dS"].sum(1))
        assert np.all(sums <= rel * np.linalg.norm(o["dS"], axis=1))
        assert np.any(sums > 1e-12)
