"""GPU parity of the geometry probe (kiattn_geometry) against the oracle on
the same host-computed fp32 scores: span, width and query norm to fp32
rounding, entropies, total variation and top-bucket masses to fp32 sum
accuracy.  Covers the register path (rows of at most 1024 keys, T a
multiple of 4), the unaligned-T path and the long-row path, causal and
non-causal, every calibration and reconstruction, and the full-size
GPT-2-124M shape on sampled rows."""
import numpy as np
import pytest
import torch

import oracle as ref
from quantized_softmax_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu

K = pytest.importorskip("quantized_softmax_attention_b200.kiattn")

# span, h, ||q|| are single fp32 operations on exact values: relative bound;
# entropies, TV and masses are fp32 sums over up to T terms: absolute bound
REL_FIELDS = (ref.GEO_SPAN, ref.GEO_H, ref.GEO_QNORM)
ABS_FIELDS = (ref.GEO_ENT_SOFTMAX, ref.GEO_ENT_OP, ref.GEO_TV, ref.GEO_TOP_SOFTMAX,
              ref.GEO_TOP_OP)
REL_TOL, ABS_TOL = 2e-6, 3e-5


def _scores(Q, Kt):
    """fp32 scores computed on the host (fp64 products, rounded once)."""
    S = np.einsum("bhid,bhjd->bhij", Q.astype(np.float64), Kt.astype(np.float64))
    return np.ascontiguousarray(S.astype(np.float32))


def _run(S, Q, cfg):
    B, H, T, _ = S.shape
    s = torch.from_numpy(S).cuda()
    q = torch.from_numpy(np.ascontiguousarray(Q)).cuda() if Q is not None else None
    out = torch.full((B, H, T, K.GEO_FIELD_COUNT), float("nan"), device="cuda")
    K.kiattn_geometry(s, out, cfg, Q=q)
    torch.cuda.synchronize()
    return out.cpu().numpy().reshape(B * H * T, -1)


def _check(got, want):
    assert np.isfinite(got).all()
    for f in REL_FIELDS:
        np.testing.assert_allclose(got[:, f], want[:, f], rtol=REL_TOL, atol=1e-30,
                                   err_msg=K.GEO_FIELDS[f])
    for f in ABS_FIELDS:
        np.testing.assert_allclose(got[:, f], want[:, f], rtol=0, atol=ABS_TOL,
                                   err_msg=K.GEO_FIELDS[f])


def _row_len(T, causal, BH):
    return np.tile(np.arange(1, T + 1) if causal else np.full(T, T), BH)


@pytest.mark.parametrize("T", [200, 203, 1024, 1100])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("cal", [K.CAL_MINMAX, K.CAL_FWM, K.CAL_FIXED])
@pytest.mark.parametrize("rec", [K.REC_LERP, K.REC_NEAREST])
def test_geometry_matches_oracle(T, causal, cal, rec):
    wl = W.gpt2_heavy() if cal == K.CAL_MINMAX else W.gpt2_fwm()
    Q, Kt, _, _ = (x.numpy() for x in W.make_inputs(wl, B=1, H=3, T=T))
    S = _scores(Q, Kt)
    cfg = K.Config(K=4, cal=cal, rec=rec, causal=causal)
    got = _run(S, Q, cfg)
    want = ref.geometry(S.reshape(-1, T), _row_len(T, causal, 3),
                        ref.RefConfig(K=4, cal=cal, rec=rec, causal=causal), Q=Q.reshape(-1, 64))
    _check(got, want)


@pytest.mark.parametrize("Kint", [1, 16, 64])
def test_geometry_interval_counts_and_degenerate_rows(Kint):
    """K from 1 to the maximum; the first rows of every head are constant
    (degenerate MinMax rows); no queries given (norm field 0)."""
    wl = W.gpt2_heavy()
    Q, Kt, _, _ = (x.numpy() for x in W.make_inputs(wl, B=1, H=2, T=256))
    S = _scores(Q, Kt)
    S[:, :, :5, :] = -1.25
    for cal in (K.CAL_MINMAX, K.CAL_FWM):
        cfg = K.Config(K=Kint, cal=cal, rec=K.REC_NEAREST)
        got = _run(S, None, cfg)
        want = ref.geometry(S.reshape(-1, 256), _row_len(256, True, 2),
                            ref.RefConfig(K=Kint, cal=cal, rec=K.REC_NEAREST))
        _check(got, want)
        assert np.all(got[:, ref.GEO_QNORM] == 0.0)


def test_geometry_rejects_bad_arguments():
    S = torch.zeros((1, 1, 8, 8), device="cuda")
    out = torch.zeros((1, 1, 8, 8), device="cuda")
    with pytest.raises(RuntimeError):
        K.kiattn_geometry(S, out, K.Config(op=K.OP_SOFTMAX))
    with pytest.raises((RuntimeError, ValueError)):
        K.kiattn_geometry(S[:, :, :0], out, K.Config())
    with pytest.raises(ValueError):   # the binding checks the output's size
        K.kiattn_geometry(S, out[..., :4].contiguous(), K.Config())


def test_geometry_full_size_sampled_rows():
    """GPT-2-124M shape B8 H12 T1024 (the benchmark's workload and launch
    configuration), all rows on the GPU; the oracle recomputes 3 sampled
    (b, h) pairs in full."""
    wl = W.gpt2_fwm()
    Q, Kt, _, _ = (x.numpy() for x in W.make_inputs(wl))
    B, H, T, d = Q.shape
    S = _scores(Q, Kt)
    cfg = K.Config(K=wl.K, cal=wl.cal, rec=wl.rec, ste=wl.ste, tau=wl.tau)
    got = _run(S, Q, cfg).reshape(B * H, T, -1)
    rcfg = ref.RefConfig(K=wl.K, cal=wl.cal, rec=wl.rec, ste=wl.ste, tau=wl.tau)
    rng = np.random.default_rng(0)
    for bh in rng.choice(B * H, 3, replace=False):
        b, h = divmod(int(bh), H)
        want = ref.geometry(S[b, h], np.arange(1, T + 1), rcfg, Q=Q[b, h])
        _check(got[bh], want)
