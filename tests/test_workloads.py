"""The synthetic input recipes realise the score geometry they are meant to
stand in for ("Pretraining Transformers with Quantized Softmax in
Attention": softmax-like row spans of 25-32 nats, a MinMax collapse about
seven times wider, section 5.4 and Appendix D.6): measured on the host."""
import numpy as np

from quantized_softmax_attention_b200 import workloads as W


def _spans(w, rows=(255, 383, 511, 639, 767, 895, 1023)):
    q, k, _, _ = (x.numpy().astype(np.float64) for x in W.make_inputs(w, B=1))
    out = np.zeros((q.shape[1], len(rows)))
    for h in range(q.shape[1]):
        for n, i in enumerate(rows):
            s = q[0, h, i] @ k[0, h, :i + 1].T
            out[h, n] = s.max() - s.min()
    return out


def test_span_ladder_runs_from_8_to_40_nats():
    """Per-head mean span over late rows within a factor 1.5 of the target
    8 * 5^{h/11} nats (a row's span also depends on its query's norm), and
    the ladder rising about five-fold from the first head to the last."""
    sp = _spans(W.gpt2_fwm()).mean(1)
    target = 8.0 * 5.0 ** (np.arange(12) / 11)
    assert np.all(np.abs(np.log(sp / target)) < np.log(1.5)), (sp, target)
    assert 3.0 < sp[-1] / sp[0] < 8.0


def test_heavy_tail_reaches_seven_times_the_softmax_span():
    sp = _spans(W.gpt2_heavy())
    typical = np.median(sp[1:])
    assert 12.0 < typical < 60.0
    assert sp[0].max() > 5.0 * 28.0     # head 0 pinned near 7 x the softmax span


def test_inputs_are_seeded_and_identical_across_calls():
    a = W.make_inputs(W.tiny())
    b = W.make_inputs(W.tiny())
    for x, y in zip(a, b):
        assert (x == y).all() and x.dtype == y.dtype
