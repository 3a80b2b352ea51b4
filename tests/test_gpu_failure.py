"""Failure handling on the GPU without a fault: every wait inside the
tensor-core kernels is bounded, and a wait that runs out sets
KIA_ERR_TIMEOUT in the library's error word, lets what is in flight land,
frees tensor memory and returns, so the context stays usable.

The test makes one wait run out with the library's hook: the forward's first
CTA withholds its first Q tile (no copy and no expected-bytes arrival are
issued, so nothing is in flight for it), under a 20 ms wait limit.  A normal
call afterwards must reproduce an earlier run bit for bit.
"""
import time

import pytest
import torch

pytestmark = pytest.mark.gpu

K = pytest.importorskip("quantized_softmax_attention_b200.kiattn")

ERR_TIMEOUT = -4


def test_withheld_copy_times_out_and_context_stays_usable():
    g = torch.Generator().manual_seed(3)
    B, H, T, d = 1, 4, 512, 64
    q, k, v, do = (torch.randn((B, H, T, d), generator=g).cuda() for _ in range(4))
    q *= 0.3
    cfg = K.Config(K=4, cal=K.CAL_FWM, rec=K.REC_NEAREST, ste=K.STE_PROB)
    ref = K.forward(q, k, v, cfg)
    K.backward(q, k, v, do, cfg, ref)
    torch.cuda.synchronize()
    assert K.kiattn_device_error(True) == 0
    K.kiattn_debug_bounded_wait(1, 20_000_000)
    try:
        bufs = K.Buffers(B, H, T, d, cfg)
        t0 = time.perf_counter()
        K.kiattn_fwd(q, k, v, bufs.O, bufs.stats, cfg)
        torch.cuda.synchronize()
        el = time.perf_counter() - t0
        assert K.kiattn_device_error(True) == ERR_TIMEOUT
    finally:
        K.kiattn_debug_bounded_wait(0, 0)
    # the withheld wait gave up after about the shortened limit
    assert 0.015 < el < 1.5, el
    # the context is usable and the results are those of the earlier run
    bufs = K.forward(q, k, v, cfg)
    K.backward(q, k, v, do, cfg, bufs)
    torch.cuda.synchronize()
    assert K.kiattn_device_error(True) == 0
    for a, b in ((bufs.O, ref.O), (bufs.dQ, ref.dQ), (bufs.dK, ref.dK), (bufs.dV, ref.dV)):
        assert torch.equal(a, b)
