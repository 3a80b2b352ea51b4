"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Sizes span several 128-row tiles and a ragged tail; tolerances are the ones
the operator's checking protocol fixes: bit-exact weight stage on the same
scores, relative L2 <= 1e-5 in exact-fp32 mode and <= 2e-3 in TF32 mode,
per-row |sum_j dS_j| <= 1e-5 ||dS_i|| for the zero-sum gradient modes.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle as ref

pytestmark = pytest.mark.gpu

K = pytest.importorskip("quantized_softmax_attention_b200.kiattn")
from parity_util import compare, flag_rows, oracle_scores, rel_l2  # noqa: E402

RECSTE = [(K.REC_LERP, K.STE_WEIGHT), (K.REC_NEAREST, K.STE_WEIGHT), (K.REC_NEAREST, K.STE_PROB)]
MODES = [K.GRAD_FULL, K.GRAD_DETACH, K.GRAD_MAX_ONLY, K.GRAD_MIN_ONLY, K.GRAD_PROJECT]
# operand rounding of the tcgen05 kind::tf32 MMA, measured by
# test_tc_scores_operand_rounding below
TF32_RULE = ref.ROUND_TRUNC


def _inputs(B, H, T, d, seed, qscale=None, kscale=1.0):
    g = torch.Generator().manual_seed(seed)
    sh = (B, H, T, d)
    q = torch.randn(sh, generator=g) * (qscale if qscale is not None else d ** -0.5)
    k = torch.randn(sh, generator=g) * kscale
    v = torch.randn(sh, generator=g)
    do = torch.randn(sh, generator=g)
    return [x.numpy().astype(np.float32) for x in (q, k, v, do)]


# ------------------------------------------------------------ weight stage

def _weight_rows(rng, rows, cols):
    S = rng.standard_normal((rows, cols)).astype(np.float32) * rng.uniform(0.5, 12, (rows, 1)).astype(np.float32)
    L = rng.integers(1, cols + 1, rows).astype(np.int32)
    # crafted rows: constant (degenerate), two values, scores on grid nodes,
    # a huge span (subnormal / zero grid values), a near-degenerate span
    S[0] = 1.25
    S[1, :] = 0.0
    S[1, ::2] = -3.0
    S[2] = -1.5 * rng.integers(0, 5, cols).astype(np.float32)
    S[3] = np.linspace(0, -400, cols).astype(np.float32)
    S[4] = (1.0 + rng.integers(0, 2, cols) * 1e-6).astype(np.float32)
    L[:5] = cols
    return S, L


@pytest.mark.parametrize("cal", [K.CAL_MINMAX, K.CAL_FWM, K.CAL_FIXED])
@pytest.mark.parametrize("rec", [K.REC_LERP, K.REC_NEAREST])
@pytest.mark.parametrize("Kint", [1, 2, 4, 16, 64])
def test_weight_stage_bit_exact(cal, rec, Kint):
    """Bin indices, t, row extrema and weights equal the oracle's fp32
    definition bit for bit on the same scores.  The fixed-step grid ends
    where its values underflow to zero; past that point both sides give
    weight 0 and only the weights are compared (the library reports the
    keys there as tail, the definition keeps counting nodes)."""
    rng = np.random.default_rng(1000 + 10 * cal + rec + Kint)
    S, L = _weight_rows(rng, 300, 517)
    cfg = K.Config(K=Kint, cal=cal, rec=rec, tau=6.0)
    exp = ref.weights_fp32(S, L, ref.RefConfig(K=Kint, cal=cal, rec=rec, tau=6.0))
    dev = "cuda"
    s = torch.from_numpy(S).to(dev)
    l = torch.from_numpy(L).to(dev)
    w = torch.empty_like(s)
    t = torch.empty_like(s)
    b = torch.empty(S.shape, dtype=torch.int32, device=dev)
    m = torch.empty(S.shape[0], device=dev)
    n = torch.empty(S.shape[0], device=dev)
    if cal == K.CAL_FIXED and Kint == 64:
        # 104.5 nats / (6/64) nats is beyond the fixed-step grid's limit
        with pytest.raises(K.KiattnError) as e:
            K.kiattn_weights_from_S(s, l, cfg, w, b, t, m, n)
        assert e.value.code == -2
        return
    K.kiattn_weights_from_S(s, l, cfg, w, b, t, m, n)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(m.cpu().numpy().view(np.uint32), exp["m"].view(np.uint32))
    np.testing.assert_array_equal(n.cpu().numpy().view(np.uint32), exp["n"].view(np.uint32))
    np.testing.assert_array_equal(w.cpu().numpy().view(np.uint32), exp["w"].view(np.uint32))
    keep = np.ones(S.shape, bool) if cal != K.CAL_FIXED else exp["w"] != 0
    if cal == K.CAL_FIXED:
        assert keep.sum() > keep.size // 4
    np.testing.assert_array_equal(b.cpu().numpy()[keep], exp["bin"][keep])
    np.testing.assert_array_equal(t.cpu().numpy()[keep].view(np.uint32),
                                  exp["t"][keep].view(np.uint32))


# ------------------------------------------------------------------ scores

@pytest.mark.parametrize("d", [64, 128])
def test_fp32_scores_exact(d):
    Q, Kt, _, _ = _inputs(1, 2, 200, d, 5)
    cfg = K.Config(gemm=K.GEMM_FP32)
    q, k = torch.from_numpy(Q).cuda(), torch.from_numpy(Kt).cuda()
    S = torch.empty((1, 2, 200, 200), device="cuda")
    K.kiattn_scores(q, k, S, cfg)
    exp = np.tril(oracle_scores(Q, Kt, ref.ROUND_NONE))
    assert rel_l2(S.cpu().numpy(), exp) < 1e-6


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [128, 300])
def test_tc_scores_operand_rounding(d, T):
    """The tcgen05 TF32 scores match the oracle's S with operands rounded by
    TF32_RULE to fp32 accumulation accuracy (and the other rules do not)."""
    Q, Kt, _, _ = _inputs(2, 2, T, d, 6, qscale=1.0)
    q, k = torch.from_numpy(Q).cuda(), torch.from_numpy(Kt).cuda()
    S = torch.empty((2, 2, T, T), device="cuda")
    for causal in (True, False):
        K.kiattn_scores(q, k, S, K.Config(causal=causal))
        got = S.cpu().numpy()
        errs = {}
        for rule in (ref.ROUND_TRUNC, ref.ROUND_RNA, ref.ROUND_RNE, ref.ROUND_NONE):
            exp = oracle_scores(Q, Kt, rule)
            if causal:
                exp = np.tril(exp)
            errs[rule] = rel_l2(got, exp)
        print("tf32 rounding rule errors", errs)
        assert errs[TF32_RULE] < 2e-6, errs
        assert min(v for r, v in errs.items() if r != TF32_RULE) > 10 * errs[TF32_RULE], errs


# ------------------------------------------------- exact-fp32 operator path

SMALL = [(1, 2, 128, 64), (1, 2, 200, 64), (1, 1, 160, 128)]


@pytest.mark.parametrize("shape", SMALL)
@pytest.mark.parametrize("cal", [K.CAL_MINMAX, K.CAL_FWM, K.CAL_FIXED])
@pytest.mark.parametrize("rec,ste", RECSTE)
def test_fp32_path_matches_oracle_all_modes(shape, cal, rec, ste):
    B, H, T, d = shape
    Q, Kt, V, dO = _inputs(B, H, T, d, 7 + T + d + cal, qscale=0.5)
    for grad in MODES:
        cfg = K.Config(K=4, cal=cal, rec=rec, ste=ste, grad=grad, gemm=K.GEMM_FP32)
        errs, gpu, _ = compare(Q, Kt, V, dO, cfg, ref.ROUND_NONE, 1e-5, 1e-4)
        for name in ("O", "dQ", "dK", "dV", "dS"):
            assert errs[name] < 1e-5, (grad, errs)
        if grad in (K.GRAD_FULL, K.GRAD_PROJECT):
            assert errs["zero_sum"] < 1e-5, errs


def test_fp32_path_softmax_and_noncausal():
    Q, Kt, V, dO = _inputs(1, 2, 192, 64, 11)
    for causal, op in itertools.product((True, False), (K.OP_SOFTMAX, K.OP_KINTERVAL)):
        cfg = K.Config(K=16, cal=K.CAL_MINMAX, rec=K.REC_LERP, causal=causal, op=op,
                       gemm=K.GEMM_FP32)
        errs, _, _ = compare(Q, Kt, V, dO, cfg, ref.ROUND_NONE, 1e-5, 1e-4)
        for name in ("O", "dQ", "dK", "dV", "dS"):
            assert errs[name] < 1e-5, (causal, op, errs)


def test_fp32_forward_bitwise_identical_across_modes_and_surrogates():
    Q, Kt, V, dO = _inputs(1, 2, 256, 64, 12, qscale=0.7)
    from parity_util import run_gpu
    for cal in (K.CAL_MINMAX, K.CAL_FWM):
        outs = []
        for grad, ste in itertools.product(MODES, (K.STE_WEIGHT, K.STE_PROB)):
            cfg = K.Config(K=4, cal=cal, rec=K.REC_NEAREST, ste=ste, grad=grad, gemm=K.GEMM_FP32)
            outs.append(run_gpu(Q, Kt, V, dO, cfg, bwd=False)["O"])
        for o in outs[1:]:
            np.testing.assert_array_equal(o.view(np.uint32), outs[0].view(np.uint32))


# ------------------------------------------------- tensor-core (TF32) path

TC_SHAPES = [(1, 2, 128, 64), (1, 2, 200, 64), (2, 1, 384, 64)]


@pytest.mark.parametrize("shape", TC_SHAPES)
@pytest.mark.parametrize("cal", [K.CAL_MINMAX, K.CAL_FWM, K.CAL_FIXED])
@pytest.mark.parametrize("rec,ste", RECSTE)
def test_tc_path_matches_oracle_all_modes(shape, cal, rec, ste):
    """tcgen05 TF32 forward + backward against the oracle with TF32 operand
    rounding, every gradient mode, tolerance 2e-3 relative L2."""
    B, H, T, d = shape
    Q, Kt, V, dO = _inputs(B, H, T, d, 21 + T + cal, qscale=0.5)
    for grad in MODES:
        cfg = K.Config(K=4, cal=cal, rec=rec, ste=ste, grad=grad)
        errs, _, _ = compare(Q, Kt, V, dO, cfg, TF32_RULE, 2e-3, 1e-4)
        for name in ("O", "dQ", "dK", "dV", "dS"):
            assert errs[name] < 2e-3, (grad, errs)
        if grad in (K.GRAD_FULL, K.GRAD_PROJECT):
            assert errs["zero_sum"] < 1e-5, errs


TC128_SHAPES = [(1, 2, 200, 128), (1, 1, 320, 128)]


@pytest.mark.parametrize("shape", TC128_SHAPES)
@pytest.mark.parametrize("cal", [K.CAL_MINMAX, K.CAL_FWM])
@pytest.mark.parametrize("rec,ste", RECSTE)
@pytest.mark.parametrize("Kint", [4, 24])
def test_tc_path_d128_matches_oracle_all_modes(shape, cal, rec, ste, Kint):
    """The d = 128 tcgen05 passes against the oracle at ragged lengths (200:
    a half unit of 32 rows cut by the sequence end), every gradient mode.
    They keep the item's stationary operands in tensor memory and run each
    unit as two halves of 32 rows; under MinMax the key pass holds the
    queries' grids in two half-unit slots, and the forward holds the rows'
    grids in their own region at K = 4 and over its epilogue's staging block
    at K = 24."""
    B, H, T, d = shape
    Q, Kt, V, dO = _inputs(B, H, T, d, 41 + T + cal + Kint, qscale=0.5)
    for grad in MODES:
        cfg = K.Config(K=Kint, cal=cal, rec=rec, ste=ste, grad=grad)
        errs, _, orc = compare(Q, Kt, V, dO, cfg, TF32_RULE, 2e-3, 1e-4)
        for name in ("O", "dQ", "dK", "dV", "dS"):
            assert errs[name] < 2e-3, (grad, errs)
        if grad in (K.GRAD_FULL, K.GRAD_PROJECT):
            # A row's gradient sums to zero in exact arithmetic (Appendix B);
            # in floating point the residual follows the row's conditioning,
            # which the fp64 oracle's own residual measures (at d = 128 and
            # K = 24 MinMax some rows cancel a few hundred times worse than at
            # K = 4): fp32 gets that residual scaled by its coarser epsilon.
            ds = orc["dS"].astype(np.float64)
            norms = np.linalg.norm(ds, axis=-1)
            live = norms > 1e-12 * max(np.linalg.norm(ds), 1e-300)
            r_orc = float(np.where(live, np.abs(ds.sum(-1)) / np.maximum(norms, 1e-300), 0.0).max())
            scale = np.finfo(np.float32).eps / np.finfo(np.float64).eps
            assert errs["zero_sum"] < 1e-5 + 2.0 * scale * r_orc, (errs, r_orc)


@pytest.mark.parametrize("Kint", [1, 2, 16, 32, 64])
@pytest.mark.parametrize("cal", [K.CAL_MINMAX, K.CAL_FWM])
def test_tc_path_interval_counts(Kint, cal):
    Q, Kt, V, dO = _inputs(1, 2, 256, 64, 31 + Kint, qscale=0.5)
    for rec, ste in RECSTE:
        cfg = K.Config(K=Kint, cal=cal, rec=rec, ste=ste)
        errs, _, _ = compare(Q, Kt, V, dO, cfg, TF32_RULE, 2e-3, 1e-4)
        for name in ("O", "dQ", "dK", "dV", "dS"):
            assert errs[name] < 2e-3, (rec, ste, errs)


def test_tc_path_softmax_and_noncausal():
    Q, Kt, V, dO = _inputs(1, 2, 320, 64, 41)
    for causal, op in itertools.product((True, False), (K.OP_SOFTMAX, K.OP_KINTERVAL)):
        cfg = K.Config(K=16, cal=K.CAL_MINMAX, rec=K.REC_LERP, causal=causal, op=op)
        errs, _, _ = compare(Q, Kt, V, dO, cfg, TF32_RULE, 2e-3, 1e-4)
        for name in ("O", "dQ", "dK", "dV", "dS"):
            assert errs[name] < 2e-3, (causal, op, errs)


REDUCED_EXP = [K.OP_SOFTMAX_BF16EXP, K.OP_SOFTMAX_FP8EXP]


@pytest.mark.parametrize("op", REDUCED_EXP)
@pytest.mark.parametrize("shape", [(1, 2, 200, 64), (2, 1, 384, 64)])
def test_tc_reduced_precision_exp_baselines(op, shape):
    """Appendix D.5 baselines on the tcgen05 path: softmax with a bfloat16-
    or FP8-rounded numerator, straight-through backward; TF32 tolerance."""
    B, H, T, d = shape
    Q, Kt, V, dO = _inputs(B, H, T, d, 71 + op + T, qscale=0.5)
    for causal in (True, False):
        cfg = K.Config(op=op, causal=causal)
        errs, _, _ = compare(Q, Kt, V, dO, cfg, TF32_RULE, 2e-3, 1e-4)
        for name in ("O", "dQ", "dK", "dV", "dS"):
            assert errs[name] < 2e-3, (op, causal, errs)


@pytest.mark.parametrize("op", REDUCED_EXP)
@pytest.mark.parametrize("shape", [(1, 2, 200, 64), (1, 1, 160, 128)])
def test_fp32_reduced_precision_exp_baselines(op, shape):
    B, H, T, d = shape
    Q, Kt, V, dO = _inputs(B, H, T, d, 81 + op + T, qscale=0.5)
    for causal in (True, False):
        cfg = K.Config(op=op, causal=causal, gemm=K.GEMM_FP32)
        errs, _, _ = compare(Q, Kt, V, dO, cfg, ref.ROUND_NONE, 1e-5, 1e-4)
        for name in ("O", "dQ", "dK", "dV", "dS"):
            assert errs[name] < 1e-5, (op, causal, errs)


def test_tc_forward_bitwise_identical_across_modes_and_surrogates():
    Q, Kt, V, dO = _inputs(2, 2, 256, 64, 42, qscale=0.7)
    from parity_util import run_gpu
    for cal in (K.CAL_MINMAX, K.CAL_FWM):
        outs = []
        for grad, ste in itertools.product(MODES, (K.STE_WEIGHT, K.STE_PROB)):
            cfg = K.Config(K=4, cal=cal, rec=K.REC_NEAREST, ste=ste, grad=grad)
            outs.append(run_gpu(Q, Kt, V, dO, cfg, bwd=False)["O"])
        for o in outs[1:]:
            np.testing.assert_array_equal(o.view(np.uint32), outs[0].view(np.uint32))


@pytest.mark.parametrize("T", [256, 200])
def test_tc_d128_forward_and_backward(T):
    """d = 128 on the tensor cores, forward and both backward passes: every
    calibration x reconstruction x surrogate, every gradient mode, a ragged
    tail; per-row zero sums for the zero-sum modes."""
    Q, Kt, V, dO = _inputs(1, 2, T, 128, 43)
    for cal, (rec, ste), grad in itertools.product((K.CAL_MINMAX, K.CAL_FWM, K.CAL_FIXED), RECSTE, MODES):
        cfg = K.Config(K=32 if cal != K.CAL_FIXED else 4, cal=cal, rec=rec, ste=ste, grad=grad)
        errs, _, _ = compare(Q, Kt, V, dO, cfg, TF32_RULE, 2e-3, 1e-4)
        for name in ("O", "dQ", "dK", "dV", "dS"):
            assert errs[name] < 2e-3, (cal, rec, ste, grad, errs)
        if grad in (K.GRAD_FULL, K.GRAD_PROJECT):
            assert errs["zero_sum"] < 1e-5, errs


# ---------------------------------------- fixed-upstream decomposition

@pytest.mark.parametrize("gemm,rule,tol", [(K.GEMM_TF32, TF32_RULE, 5e-3),
                                           (K.GEMM_FP32, ref.ROUND_NONE, 5e-5)])
@pytest.mark.parametrize("cal", [K.CAL_MINMAX, K.CAL_FWM])
def test_grad_decomposition_matches_oracle(gemm, rule, tol, cal):
    """Per-row ||dS||^2 and squared maximum- / minimum-side calibration terms
    from kiattn_grad_decomposition (after a kiattn_bwd that dumped dS) against
    the oracle's mode-minus-detach decomposition, every gradient mode.  The
    quantities are squares, so the bound is about twice the operator's."""
    from parity_util import ref_cfg
    B, H, T, d = 1, 2, 200, 64
    Q, Kt, V, dO = _inputs(B, H, T, d, 61 + cal, qscale=0.5)
    for rec, ste in RECSTE:
        for grad in MODES:
            cfg = K.Config(K=4, cal=cal, rec=rec, ste=ste, grad=grad, gemm=gemm)
            flags = flag_rows(Q, Kt, cfg, rule, 1e-4)
            dO2 = dO.copy()
            dO2[flags] = 0.0
            q, k, v, g = (torch.from_numpy(np.ascontiguousarray(x)).cuda() for x in (Q, Kt, V, dO2))
            bufs = K.Buffers(B, H, T, d, cfg)
            dS = torch.empty((B, H, T, T), dtype=torch.float32, device="cuda")
            out = torch.full((B, H, T, 3), float("nan"), dtype=torch.float64, device="cuda")
            K.kiattn_fwd(q, k, v, bufs.O, bufs.stats, cfg)
            K.kiattn_bwd(q, k, v, bufs.O, g, bufs.stats, bufs.dQ, bufs.dK, bufs.dV, bufs.work, cfg,
                         dS_dbg=dS)
            K.kiattn_grad_decomposition(dS, bufs.work, out, cfg)
            torch.cuda.synchronize()
            assert K.kiattn_device_error(True) == 0
            got = out.cpu().numpy().reshape(B * H, T, 3)
            want = ref.grad_decomposition(Q, Kt, V, dO2, ref_cfg(cfg, rule))
            assert np.isfinite(got).all()
            for c in range(3):
                err = rel_l2(got[..., c], want[..., c])
                assert err < tol, (rec, ste, grad, c, err)
            if grad in (K.GRAD_DETACH,):
                assert np.all(got[..., 1:] == 0.0)
            if grad == K.GRAD_MAX_ONLY or grad == K.GRAD_PROJECT or cal == K.CAL_FWM:
                assert np.all(got[..., 2] == 0.0)
            if grad == K.GRAD_MIN_ONLY:
                assert np.all(got[..., 1] == 0.0)
            # the appendix's norm ratios
            for c in (1, 2):
                rg = np.sqrt(got[..., c].sum() / got[..., 0].sum())
                rw = np.sqrt(want[..., c].sum() / want[..., 0].sum())
                assert abs(rg - rw) <= tol * max(rw, 1e-3), (grad, c, rg, rw)


def test_grad_decomposition_rejects_bad_arguments():
    cfg = K.Config()
    dS = torch.zeros((1, 1, 128, 128), device="cuda")
    out = torch.zeros((1, 1, 128, 3), dtype=torch.float64, device="cuda")
    bufs = K.Buffers(1, 1, 128, 64, cfg)
    with pytest.raises(RuntimeError):
        K.kiattn_grad_decomposition(dS, None, out, cfg)
    with pytest.raises((RuntimeError, ValueError)):
        K.kiattn_grad_decomposition(dS[:, :, :0], bufs.work, out, cfg)
    with pytest.raises(ValueError):   # the binding checks the output's type
        K.kiattn_grad_decomposition(dS, bufs.work, out.float(), cfg)
