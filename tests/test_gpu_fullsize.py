"""Parity at the full workload sizes, in the launch configuration the
benchmark times, on sampled (batch, head) pairs the oracle recomputes.

Every (batch, head) pair is an independent problem, so the oracle runs on
the sampled heads alone and is compared with the same heads of the full-size
GPU run.  Rows near a discontinuity of the forward (see parity_util) get a
zero upstream gradient on both sides.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle as ref

pytestmark = pytest.mark.gpu

K = pytest.importorskip("quantized_softmax_attention_b200.kiattn")
from quantized_softmax_attention_b200 import workloads as W  # noqa: E402
from parity_util import check_flags, flag_budget, flag_rows, ref_cfg, rel_l2  # noqa: E402

TF32 = ref.ROUND_TRUNC
MODES = [K.GRAD_FULL, K.GRAD_DETACH, K.GRAD_MAX_ONLY, K.GRAD_MIN_ONLY, K.GRAD_PROJECT]


def _cfg(w, **kw):
    c = K.Config(K=w.K, cal=w.cal, tau=w.tau, rec=w.rec, ste=w.ste, grad=w.grad, causal=w.causal)
    return c.replace(**kw)


def _run_full(q, k, v, g, cfg, grads=(None,)):
    dev = [torch.from_numpy(x).cuda() for x in (q, k, v, g)]
    B, H, T, d = q.shape
    bufs = K.Buffers(B, H, T, d, cfg)
    K.kiattn_fwd(dev[0], dev[1], dev[2], bufs.O, bufs.stats, cfg)
    out = {"O": bufs.O.cpu().numpy()}
    for gm in grads:
        c = cfg if gm is None else cfg.replace(grad=gm)
        K.kiattn_bwd(dev[0], dev[1], dev[2], bufs.O, dev[3], bufs.stats, bufs.dQ, bufs.dK, bufs.dV,
                     bufs.work, c)
        torch.cuda.synchronize()
        out[gm] = {n: t.cpu().numpy() for n, t in (("dQ", bufs.dQ), ("dK", bufs.dK),
                                                    ("dV", bufs.dV))}
    assert K.kiattn_device_error(True) == 0
    return out


def _check_heads(q, k, v, g, cfg, heads, grads, tol=2e-3):
    """Zero dO on flagged rows of the sampled heads, run the full-size GPU
    operator, compare the sampled heads with the oracle."""
    B, H, T, d = q.shape
    g = g.copy()
    sel = [(bb, hh) for bb, hh in heads]
    qs = np.stack([q[bb, hh] for bb, hh in sel])[None]
    ks = np.stack([k[bb, hh] for bb, hh in sel])[None]
    flags = flag_rows(qs, ks, cfg, TF32, 1e-4)[0]
    check_flags(flags, flag_budget(qs, ks, cfg, TF32, 1e-4), f"{q.shape} {cfg} heads {sel}")
    for n, (bb, hh) in enumerate(sel):
        g[bb, hh][flags[n]] = 0.0
    gs = np.stack([g[bb, hh] for bb, hh in sel])[None]
    vs = np.stack([v[bb, hh] for bb, hh in sel])[None]
    got = _run_full(q, k, v, g, cfg, grads)
    keep = ~flags
    for gm in grads:
        c = cfg if gm is None else cfg.replace(grad=gm)
        orc = ref.attention(qs, ks, vs, gs, ref_cfg(c, TF32))
        o_gpu = np.stack([got["O"][bb, hh] for bb, hh in sel])[None]
        assert rel_l2(o_gpu, orc["O"], keep[None]) < tol
        for name in ("dQ", "dK", "dV"):
            a = np.stack([got[gm][name][bb, hh] for bb, hh in sel])[None]
            err = rel_l2(a, orc[name])
            assert err < tol, (gm, name, err)
    return flags


def test_gpt2_124M_fwm_nearest_probste_full_size():
    """The benchmark's workload: B8 H12 T1024 d64, FWM tau=6, Nearest +
    Prob-STE, K=4, full gradients (heads with the smallest and largest span)."""
    w = W.gpt2_fwm()
    q, k, v, g = (x.numpy() for x in W.make_inputs(w))
    _check_heads(q, k, v, g, _cfg(w), [(0, 0), (3, 11), (7, 5)], (None,))


@pytest.mark.parametrize("grad", [K.GRAD_FULL, K.GRAD_PROJECT])
def test_gpt2_124M_zero_sum_rows_full_size(grad):
    """The benchmark's workload at full size with the score gradient dumped:
    every row of the full and projection modes sums to zero (shift
    invariance, section 3 / Appendix B) to 1e-5 of its norm, on every (b, h),
    and sampled heads' dS match the oracle's."""
    w = W.gpt2_fwm()
    q, k, v, g = (x.numpy() for x in W.make_inputs(w))
    cfg = _cfg(w, grad=grad)
    heads = [(0, 0), (7, 11)]
    qs = np.stack([q[bb, hh] for bb, hh in heads])[None]
    ks = np.stack([k[bb, hh] for bb, hh in heads])[None]
    flags = flag_rows(qs, ks, cfg, TF32, 1e-4)[0]
    check_flags(flags, flag_budget(qs, ks, cfg, TF32, 1e-4), f"zero-sum {cfg}")
    g = g.copy()
    for n, (bb, hh) in enumerate(heads):
        g[bb, hh][flags[n]] = 0.0
    dev = [torch.from_numpy(x).cuda() for x in (q, k, v, g)]
    B, H, T, d = q.shape
    bufs = K.Buffers(B, H, T, d, cfg)
    dS = torch.empty((B, H, T, T), dtype=torch.float32, device="cuda")
    K.kiattn_fwd(dev[0], dev[1], dev[2], bufs.O, bufs.stats, cfg)
    K.kiattn_bwd(dev[0], dev[1], dev[2], bufs.O, dev[3], bufs.stats, bufs.dQ, bufs.dK, bufs.dV,
                 bufs.work, cfg, dS_dbg=dS)
    torch.cuda.synchronize()
    assert K.kiattn_device_error(True) == 0
    # per-row sums and norms in fp64 on the device, every (b, h)
    ds = dS.double()
    sums = ds.sum(-1).abs()
    norms = ds.norm(dim=-1)
    live = norms > 0
    ratio = torch.where(live, sums / norms.clamp_min(1e-300), torch.zeros_like(sums))
    assert int(live.sum()) > 0.9 * B * H * (T - 1)
    assert float(ratio.max()) < 1e-5, float(ratio.max())
    vs = np.stack([v[bb, hh] for bb, hh in heads])[None]
    gs = np.stack([g[bb, hh] for bb, hh in heads])[None]
    orc = ref.attention(qs, ks, vs, gs, ref_cfg(cfg, TF32), dump=True)
    got = np.stack([dS[bb, hh].cpu().numpy() for bb, hh in heads])[None]
    assert rel_l2(got, orc["dS"]) < 2e-3


def test_gpt2_124M_fixed_step_full_size():
    """The same workload under the untruncated fixed-step operator (Appendix
    D.4): heads whose spans reach past the FWM window, all five modes."""
    w = W.gpt2_fixed()
    q, k, v, g = (x.numpy() for x in W.make_inputs(w))
    _check_heads(q, k, v, g, _cfg(w), [(2, 11), (6, 4)], tuple(MODES))


def test_gpt2_124M_minmax_heavy_tail_full_size():
    """MinMax + Nearest + Weight-STE with heavy-tailed head scales; head 0
    reaches a span about seven times the softmax span (grid values at or
    below the fp32 subnormal range)."""
    w = W.gpt2_heavy()
    q, k, v, g = (x.numpy() for x in W.make_inputs(w))
    s0 = np.einsum("td,sd->ts", q[0, 0].astype(np.float64), k[0, 0].astype(np.float64))
    spans = [np.ptp(s0[i, :i + 1]) for i in range(256, 1024, 97)]
    assert max(spans) > 120.0
    _check_heads(q, k, v, g, _cfg(w), [(0, 0), (5, 3)], (None,))


def test_1B_shape_five_gradient_modes_from_one_forward():
    """B4 H16 T2048 d128, LERP K=32, FWM and MinMax: one forward, the five
    backward modes; the forward does not depend on the gradient mode."""
    for cal in (K.CAL_FWM, K.CAL_MINMAX):
        w = W.one_b(cal=cal)
        q, k, v, g = (x.numpy() for x in W.make_inputs(w))
        cfg = _cfg(w)
        _check_heads(q, k, v, g, cfg, [(1, 7)], tuple(MODES))
        # bitwise-equal forward when re-run under another gradient mode
        dev = [torch.from_numpy(x).cuda() for x in (q, k, v)]
        outs = []
        for gm in (K.GRAD_FULL, K.GRAD_PROJECT):
            c = cfg.replace(grad=gm)
            bufs = K.Buffers(w.B, w.H, w.T, w.d, c)
            K.kiattn_fwd(dev[0], dev[1], dev[2], bufs.O, bufs.stats, c)
            outs.append(bufs.O.cpu().numpy())
        np.testing.assert_array_equal(outs[0].view(np.uint32), outs[1].view(np.uint32))


@pytest.mark.parametrize("T,Kint,cal,rec,ste", [
    (1024, 2, K.CAL_MINMAX, K.REC_LERP, K.STE_WEIGHT),
    (1024, 64, K.CAL_FWM, K.REC_NEAREST, K.STE_PROB),
    (2048, 16, K.CAL_MINMAX, K.REC_NEAREST, K.STE_WEIGHT),
    (4096, 32, K.CAL_FWM, K.REC_LERP, K.STE_WEIGHT),
    # MinMax grids kept in shared memory with one ring slot fewer
    (1024, 64, K.CAL_MINMAX, K.REC_NEAREST, K.STE_PROB),
    (2048, 32, K.CAL_MINMAX, K.REC_LERP, K.STE_WEIGHT),
])
def test_throughput_sweep_shapes(T, Kint, cal, rec, ste):
    """Points of the B16 H12 d64 sweep (T up to 4096, K from 2 to 64)."""
    w = W.sweep(T, Kint, cal, rec, ste)
    q, k, v, g = (x.numpy() for x in W.make_inputs(w))
    _check_heads(q, k, v, g, _cfg(w), [(15, 11)], (None,))


def test_exact_softmax_reference_row_full_size():
    w = W.sweep(1024, 4, K.CAL_MINMAX, K.REC_LERP, K.STE_WEIGHT)
    q, k, v, g = (x.numpy() for x in W.make_inputs(w))
    _check_heads(q, k, v, g, _cfg(w, op=K.OP_SOFTMAX), [(0, 0), (9, 4)], (None,))


@pytest.mark.parametrize("op", [K.OP_SOFTMAX_BF16EXP, K.OP_SOFTMAX_FP8EXP])
def test_reduced_precision_exp_baselines_full_size(op):
    """Appendix D.5 baselines at the bench shape B8 H12 T1024 d64."""
    w = W.gpt2_fwm()
    q, k, v, g = (x.numpy() for x in W.make_inputs(w))
    _check_heads(q, k, v, g, _cfg(w, op=op), [(1, 2), (6, 10)], (None,))


# ----------------------------------------------------------------- edges

@pytest.mark.parametrize("T", [1, 2, 5, 127, 129])
def test_tiny_and_ragged_lengths(T):
    g = torch.Generator().manual_seed(T)
    q, k, v, do = (torch.randn((2, 3, T, 64), generator=g).numpy() for _ in range(4))
    q *= 0.3
    for cal, (rec, ste) in itertools.product((K.CAL_MINMAX, K.CAL_FWM),
                                             [(K.REC_LERP, 0), (K.REC_NEAREST, 1)]):
        cfg = K.Config(K=4, cal=cal, rec=rec, ste=ste)
        _check_heads(q, k, v, do, cfg, [(bb, hh) for bb in range(2) for hh in range(3)], (None,))


def test_degenerate_rows_everywhere():
    """Q = 0 makes every score row constant: MinMax takes its degenerate
    branch on every row (uniform P, finite gradients)."""
    T = 200
    g = torch.Generator().manual_seed(9)
    k, v, do = (torch.randn((1, 2, T, 64), generator=g).numpy() for _ in range(3))
    q = np.zeros_like(k)
    for rec, ste in [(K.REC_LERP, 0), (K.REC_NEAREST, 1)]:
        cfg = K.Config(K=4, cal=K.CAL_MINMAX, rec=rec, ste=ste)
        got = _run_full(q, k, v, do, cfg)
        assert np.all(np.isfinite(got["O"]))
        for name in ("dQ", "dK", "dV"):
            assert np.all(np.isfinite(got[None][name]))
        # uniform P: O_i = mean of v_0..v_i
        cum = np.cumsum(v.astype(np.float64), axis=2) / np.arange(1, T + 1)[None, None, :, None]
        assert rel_l2(got["O"], cum) < 2e-3
        _check_heads(q, k, v, do, cfg, [(0, 0), (0, 1)], tuple(MODES))
