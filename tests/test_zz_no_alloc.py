"""The fixed-scratch backward (kiattn_bwd_noalloc) against the ordinary one.

kiattn_bwd_noalloc serves callers that cannot allocate device memory (an
engine that owns all device memory, a loop that must not synchronise on an
allocation): it runs the same backward on a scratch array the library
declares itself.  Here it must reproduce kiattn_bwd's gradients, within the
TF32 tolerance used by the parity tests, on two calls in a row (the second
call finds the first call's leftovers in the shared scratch).  This file is
collected last so that a run stopping at the first failure has already run
every other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

K = pytest.importorskip("quantized_softmax_attention_b200.kiattn")


def _rel(a, b):
    a = a.double().cpu()
    b = b.double().cpu()
    return float((a - b).norm() / b.norm())


def test_noalloc_backward_matches_workspace_backward_twice():
    g = torch.Generator().manual_seed(77)
    B, H, T, d = 2, 3, 320, 64
    q, k, v, do = (torch.randn((B, H, T, d), generator=g) for _ in range(4))
    q *= 0.4
    dev = [x.cuda() for x in (q, k, v, do)]
    for cfg in (K.Config(K=4, cal=K.CAL_FWM, rec=K.REC_NEAREST, ste=K.STE_PROB),
                K.Config(K=16, cal=K.CAL_MINMAX, rec=K.REC_LERP, grad=K.GRAD_PROJECT)):
        bufs = K.forward(dev[0], dev[1], dev[2], cfg)
        K.backward(dev[0], dev[1], dev[2], dev[3], cfg, bufs)
        ref = [t.clone() for t in (bufs.dQ, bufs.dK, bufs.dV)]
        for _ in range(2):
            out = [torch.full_like(t, float("nan")) for t in ref]
            K.kiattn_bwd_noalloc(dev[0], dev[1], dev[2], bufs.O, dev[3], bufs.stats, *out, cfg)
            torch.cuda.synchronize()
            assert K.kiattn_device_error(True) == 0
            for a, b in zip(out, ref):
                assert torch.isfinite(a).all()
                assert _rel(a, b) < 2e-3


def test_noalloc_rejects_sizes_beyond_capacity():
    cfg = K.Config()
    T = K.NOALLOC_MAX_ROWS // 2 + 128
    x = torch.empty((1, 2, T, 64), device="cuda")   # 2 * T rows > capacity
    st = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(K.KiattnError) as e:
        K.kiattn_bwd_noalloc(x, x, x, x, x, st, x, x, x, cfg)
    assert e.value.code == -6
