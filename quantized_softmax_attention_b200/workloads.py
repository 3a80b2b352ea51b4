"""Seeded synthetic workloads for K-interval attention.

Input generators only: this module holds none of the operator's arithmetic,
so both the CUDA path's tests/benchmark and the fp64 CPU oracle can be fed
from it.  Shapes and score geometry follow the paper's settings
("Pretraining Transformers with Quantized Softmax in Attention"): GPT-2-124M
attention heads (12 heads, d = 64, context 1024), a ~1B model (16 heads,
d = 128, context 2048), softmax-like row spans of 25-32 nats and a MinMax
collapse whose span grows about seven-fold (section 5.4, Appendix D.6).
Tensors are fp32, [B, H, T, d], generated on the CPU with a seeded
torch.Generator so every consumer sees identical bits.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

CAL_MINMAX, CAL_FWM, CAL_FIXED = 0, 1, 2
REC_LERP, REC_NEAREST = 0, 1
STE_WEIGHT, STE_PROB = 0, 1
GRAD_FULL, GRAD_DETACH, GRAD_MAX_ONLY, GRAD_MIN_ONLY, GRAD_PROJECT = 0, 1, 2, 3, 4


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    d: int
    K: int
    cal: int
    rec: int
    ste: int
    grad: int = GRAD_FULL
    tau: float = 6.0
    causal: bool = True
    seed: int = 0
    scores: str = "iid"          # iid | span_ladder | heavy
    operator: int = 0            # 0 K-interval, 1 softmax, 2 / 3 bf16- / FP8-rounded exp softmax
    extra: dict = field(default_factory=dict, compare=False)

    def op(self) -> dict:
        return dict(K=self.K, cal=self.cal, tau=self.tau, rec=self.rec, ste=self.ste,
                    grad=self.grad, causal=self.causal)


def tiny() -> Workload:
    """B1 H2 T128 d64, MinMax + LERP, K = 4, full gradients; seed 0."""
    return Workload("tiny_B1H2T128d64_minmax_lerp_K4", 1, 2, 128, 64, 4, CAL_MINMAX, REC_LERP,
                    STE_WEIGHT, seed=0)


def gpt2_fwm() -> Workload:
    """GPT-2-124M attention shape B8 H12 T1024 d64, FWM tau = 6 (h = 1.5),
    Nearest + Prob-STE, K = 4; per-head score scale so that row spans run
    from 8 to 40 nats; seed 1."""
    return Workload("gpt2_124M_B8H12T1024d64_fwm_nearest_probste_K4", 8, 12, 1024, 64, 4,
                    CAL_FWM, REC_NEAREST, STE_PROB, seed=1, scores="span_ladder")


def gpt2_fixed() -> Workload:
    """The gpt2_fwm workload under the untruncated fixed-step operator
    (Appendix D.4): h = tau / K = 1.5 without the tail cut; seed 1."""
    return Workload("gpt2_124M_B8H12T1024d64_fixedstep_nearest_probste_K4", 8, 12, 1024, 64, 4,
                    CAL_FIXED, REC_NEAREST, STE_PROB, seed=1, scores="span_ladder")


def gpt2_rounded_exp(fp8: bool) -> Workload:
    """The gpt2_fwm inputs under a reduced-precision exponential baseline
    (Appendix D.5): softmax with its numerator rounded to bfloat16 or FP8."""
    tag = "fp8exp" if fp8 else "bf16exp"
    return Workload(f"gpt2_124M_B8H12T1024d64_softmax_{tag}", 8, 12, 1024, 64, 4, CAL_MINMAX,
                    REC_LERP, STE_WEIGHT, seed=1, scores="span_ladder",
                    operator=3 if fp8 else 2)


def gpt2_heavy() -> Workload:
    """Same shape, MinMax + Nearest + Weight-STE, K = 4, with heavy-tailed
    per-head score scales (one head at about seven times the softmax span)."""
    return Workload("gpt2_124M_B8H12T1024d64_minmax_nearest_weightste_K4_heavy", 8, 12, 1024,
                    64, 4, CAL_MINMAX, REC_NEAREST, STE_WEIGHT, seed=2, scores="heavy")


def one_b(cal: int = CAL_FWM, grad: int = GRAD_FULL) -> Workload:
    """1B-style shape B4 H16 T2048 d128, LERP K = 32; seed 3."""
    return Workload(f"1B_B4H16T2048d128_{'fwm' if cal else 'minmax'}_lerp_K32", 4, 16, 2048, 128,
                    32, cal, REC_LERP, STE_WEIGHT, grad=grad, seed=3)


def sweep(T: int, K: int, cal: int, rec: int, ste: int) -> Workload:
    """Throughput sweep B16 H12 T d64 with iid N(0,1) inputs, Q / 8; seed 4."""
    tag = {(REC_LERP, STE_WEIGHT): "lerp", (REC_NEAREST, STE_WEIGHT): "nearest_weightste",
           (REC_NEAREST, STE_PROB): "nearest_probste"}[(rec, ste)]
    return Workload(f"sweep_B16H12T{T}d64_{'fwm' if cal else 'minmax'}_{tag}_K{K}", 16, 12, T,
                    64, K, cal, rec, ste, seed=4)


def make_inputs(w: Workload, B: int | None = None, H: int | None = None, T: int | None = None):
    """Q, K, V, dO as fp32 CPU tensors [B, H, T, d].  B/H/T override the
    workload's sizes (same recipe, smaller case)."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    T = w.T if T is None else T
    d = w.d
    g = torch.Generator().manual_seed(w.seed)
    shape = (B, H, T, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    do = torch.randn(shape, generator=g, dtype=torch.float32)
    if w.scores == "iid":
        q *= 1.0 / math.sqrt(d)
    elif w.scores == "span_ladder":
        # target row span S_h = 8 * 5^{h/(H-1)} nats; a row of ~T normal
        # scores spans about 6.5 standard deviations and the score standard
        # deviation is sigma^2 sqrt(d) when Q, K ~ N(0, sigma^2)
        for h in range(H):
            span = 8.0 * 5.0 ** (h / max(H - 1, 1))
            sigma = math.sqrt(span / (6.5 * math.sqrt(d)))
            q[:, h] *= sigma
            k[:, h] *= sigma
    elif w.scores == "heavy":
        # base score std ~4.3 (span ~28, the softmax span); per-head scale
        # c_h = exp(0.8 z_h), head 0 pinned to sqrt(7) so its span reaches ~7x
        q *= 0.54
        z = torch.randn((H,), generator=g, dtype=torch.float32)
        c = torch.exp(0.8 * z)
        c[0] = math.sqrt(7.0)
        for h in range(H):
            q[:, h] *= c[h]
            k[:, h] *= c[h]
    else:
        raise ValueError(w.scores)
    return q.contiguous(), k.contiguous(), v.contiguous(), do.contiguous()
