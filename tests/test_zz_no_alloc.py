"""The fixed-scratch backward (kiattn_bwd_noalloc) against the ordinary one.

kiattn_bwd_noalloc serves callers that cannot allocate device memory (an
engine that owns all device memory, a loop that must not synchronise on an
allocation): it runs the same backward on a scratch array the library
declares itself.  Only the scratch's address differs from kiattn_bwd, so
wherever the backward runs no global atomics (the tensor-core passes at
d = 64 and d = 128, the projection's scans, the exact path's detach mode)
the gradients must be
bit-identical; the exact path's calibration scatter adds into dK with
atomics, whose order varies, so that case is held to the exact path's 1e-5
instead.  Each configuration is called twice in a row, after other
configurations, so that every call finds earlier leftovers in the shared
scratch.  This file is collected last so that a run stopping at the first
failure has already run every other test; it also passes on its own in a
fresh process.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu

K = pytest.importorskip("quantized_softmax_attention_b200.kiattn")


def _rel(a, b):
    a = a.double().cpu()
    b = b.double().cpu()
    return float((a - b).norm() / b.norm())


def _inputs(B, H, T, d, seed):
    g = torch.Generator().manual_seed(seed)
    q, k, v, do = (torch.randn((B, H, T, d), generator=g) for _ in range(4))
    q *= 0.4
    return [x.cuda() for x in (q, k, v, do)]


# (config, d, bitwise): bitwise wherever the backward has no global atomics
CASES = [
    (K.Config(K=4, cal=K.CAL_FWM, rec=K.REC_NEAREST, ste=K.STE_PROB), 64, True),
    (K.Config(K=16, cal=K.CAL_MINMAX, rec=K.REC_LERP, grad=K.GRAD_PROJECT), 64, True),
    (K.Config(K=4, cal=K.CAL_MINMAX, rec=K.REC_NEAREST, grad=K.GRAD_DETACH,
              gemm=K.GEMM_FP32), 64, True),
    (K.Config(K=4, cal=K.CAL_MINMAX, rec=K.REC_LERP, gemm=K.GEMM_FP32), 64, False),
    (K.Config(K=32, cal=K.CAL_FWM, rec=K.REC_LERP, grad=K.GRAD_DETACH), 128, True),
    (K.Config(K=8, cal=K.CAL_MINMAX, rec=K.REC_NEAREST, ste=K.STE_WEIGHT), 128, True),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_noalloc_backward_matches_workspace_backward_twice(case):
    cfg, d, bitwise = CASES[case]
    B, H, T = 2, 3, 320 if d == 64 else 200
    q, k, v, do = _inputs(B, H, T, d, 77 + case)
    bufs = K.forward(q, k, v, cfg)
    K.backward(q, k, v, do, cfg, bufs)
    torch.cuda.synchronize()
    assert K.kiattn_device_error(True) == 0
    ref = [t.clone() for t in (bufs.dQ, bufs.dK, bufs.dV)]
    for _ in range(2):
        out = [torch.full_like(t, float("nan")) for t in ref]
        K.kiattn_bwd_noalloc(q, k, v, bufs.O, do, bufs.stats, *out, cfg)
        torch.cuda.synchronize()
        assert K.kiattn_device_error(True) == 0
        for a, b in zip(out, ref):
            assert torch.isfinite(a).all()
            if bitwise:
                assert torch.equal(a, b)
            else:
                assert _rel(a, b) < 1e-5


def test_noalloc_capacity_boundary():
    """Exactly KIA_NOALLOC_MAX_ROWS rows run (bit-identical to kiattn_bwd);
    one row more is refused with KIA_ERR_CAPACITY before any launch."""
    cfg = K.Config(K=4, cal=K.CAL_FWM, rec=K.REC_NEAREST, ste=K.STE_PROB)
    B, H, T, d = K.NOALLOC_MAX_ROWS // 64, 1, 64, 64
    q, k, v, do = _inputs(B, H, T, d, 5)
    bufs = K.forward(q, k, v, cfg)
    K.backward(q, k, v, do, cfg, bufs)
    ref = [t.clone() for t in (bufs.dQ, bufs.dK, bufs.dV)]
    out = [torch.full_like(t, float("nan")) for t in ref]
    K.kiattn_bwd_noalloc(q, k, v, bufs.O, do, bufs.stats, *out, cfg)
    torch.cuda.synchronize()
    assert K.kiattn_device_error(True) == 0
    for a, b in zip(out, ref):
        assert torch.equal(a, b)
    del q, k, v, do, bufs, ref, out
    # one row more: refused before anything is read or written
    x = torch.empty((1, 1, K.NOALLOC_MAX_ROWS + 1, 64), device="cuda")
    st = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(K.KiattnError) as e:
        K.kiattn_bwd_noalloc(x, x, x, x, x, st, x, x, x, cfg)
    assert e.value.code == -6
