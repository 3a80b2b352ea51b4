"""Helpers for GPU-vs-oracle parity tests.

Comparison protocol for the fused operator (O, dQ, dK, dV):
  * the oracle runs in fp64 on the same fp32 inputs; in TF32 mode it first
    rounds every product operand the way the tensor cores do;
  * rows whose scores sit within `delta` (in grid units u) of a
    discontinuity of the forward -- a Nearest rounding boundary, the FWM
    window edge, or a near-tie of the row max / min -- are flagged from the
    oracle's own fp64 scores.  Their upstream gradient dO is set to zero on
    both sides (so they contribute nothing to any gradient) and their O rows
    are left out of the O comparison.  Both sides then make the same
    discrete decisions on every remaining row;
  * relative L2 error per tensor, plus per-row zero sums of dS in fp64.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as ref
from quantized_softmax_attention_b200 import kiattn as K


def tf32_round(x: np.ndarray, rule: int) -> np.ndarray:
    """Round fp32 values to 10 explicit mantissa bits (test-side copy)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if rule == ref.ROUND_NONE:
        return x.astype(np.float64)
    b = x.view(np.uint32).copy()
    special = (b & 0x7F800000) == 0x7F800000
    if rule == ref.ROUND_TRUNC:
        r = b & np.uint32(0xFFFFE000)
    elif rule == ref.ROUND_RNA:
        r = (b + np.uint32(0x1000)) & np.uint32(0xFFFFE000)
    else:
        lsb = (b >> np.uint32(13)) & np.uint32(1)
        r = (b + np.uint32(0xFFF) + lsb) & np.uint32(0xFFFFE000)
    r = np.where(special, b, r)
    return r.view(np.float32).astype(np.float64)


def ref_cfg(cfg: K.Config, rounding: int) -> ref.RefConfig:
    return ref.RefConfig(K=cfg.K, cal=cfg.cal, tau=float(np.float32(cfg.tau)), rec=cfg.rec,
                         ste=cfg.ste, grad=cfg.grad, causal=bool(cfg.causal),
                         softmax=cfg.op != K.OP_KINTERVAL, rounding=rounding,
                         exp_round={K.OP_SOFTMAX_BF16EXP: ref.EXP_BF16,
                                    K.OP_SOFTMAX_FP8EXP: ref.EXP_FP8}.get(cfg.op, ref.EXP_EXACT))


def oracle_scores(Q, Kt, rule):
    q = tf32_round(Q, rule)
    k = tf32_round(Kt, rule)
    return np.einsum("bhid,bhjd->bhij", q, k)


def _round_format(x: np.ndarray, op: int) -> np.ndarray:
    """Nearest-even rounding of fp32 values to bfloat16 or FP8 E4M3 by torch's
    own dtype conversions (test-side)."""
    t = torch.from_numpy(np.ascontiguousarray(x, np.float32))
    dt = torch.bfloat16 if op == K.OP_SOFTMAX_BF16EXP else torch.float8_e4m3fn
    return t.to(dt).to(torch.float32).numpy()


def _rounding_flags(S, cfg: K.Config) -> np.ndarray:
    """Rows with a numerator e^{s-m} >= 1e-6 whose rounding to the baseline's
    format would change under a relative perturbation of the exponential's
    error size (the kernels' fast exponential and the oracle's fp64 one may
    land on either side of a rounding boundary there)."""
    B, H, T, _ = S.shape
    flags = np.zeros((B, H, T), bool)
    for i in range(T):
        L = i + 1 if cfg.causal else T
        x = S[:, :, i, :L] - S[:, :, i, :L].max(-1, keepdims=True)
        e = np.exp(x)
        rel = 2.0 ** -21 + np.abs(x) * 2.0 ** -22
        lo = _round_format((e * (1 - rel)).astype(np.float32), cfg.op)
        hi = _round_format((e * (1 + rel)).astype(np.float32), cfg.op)
        flags[:, :, i] = np.any((lo != hi) & (e >= 1e-6), -1)
    return flags


def flag_rows(Q, Kt, cfg: K.Config, rule: int, delta: float) -> np.ndarray:
    """[B, H, T] bool: rows near a discontinuity of the forward."""
    S = oracle_scores(Q, Kt, rule)
    B, H, T, _ = Q.shape
    flags = np.zeros((B, H, T), bool)
    if cfg.op == K.OP_SOFTMAX:
        return flags
    if cfg.op in (K.OP_SOFTMAX_BF16EXP, K.OP_SOFTMAX_FP8EXP):
        return _rounding_flags(S, cfg)
    tau = float(np.float32(cfg.tau))
    for i in range(T):
        L = i + 1 if cfg.causal else T
        s = S[:, :, i, :L]
        m = s.max(-1, keepdims=True)
        n = s.min(-1, keepdims=True)
        h = (m - n) / cfg.K if cfg.cal == K.CAL_MINMAX else np.full_like(m, tau / cfg.K)
        hs = np.where(h > 0, h, 1.0)
        u = (m - s) / hs
        bad = np.zeros((B, H), bool)
        if cfg.rec == K.REC_NEAREST:
            inw = (u <= cfg.K + delta) if cfg.cal == K.CAL_FWM else np.ones_like(u, bool)
            frac = np.abs(u - np.floor(u) - 0.5)
            bad |= np.any(inw & (frac < delta), -1)
        if cfg.cal == K.CAL_FWM:
            bad |= np.any(np.abs(u - cfg.K) < delta, -1)
        if L >= 2:
            srt = np.sort(s, -1)
            bad |= (srt[..., -1] - srt[..., -2]) < delta * hs[..., 0]
            if cfg.cal == K.CAL_MINMAX:
                bad |= (srt[..., 1] - srt[..., 0]) < delta * hs[..., 0]
                span = (m - n)[..., 0]
                near = np.abs(span - 1e-12) < 1e-13
                # a row clearly in the degenerate branch has uniform P and no
                # calibration term: neither its bins nor its arg-extrema matter
                bad = np.where(span < 0.5e-12, near, bad | near)
        flags[:, :, i] = bad
    return flags


def flag_budget(Q, Kt, cfg: K.Config, rule: int, delta: float) -> float:
    """Expected fraction of flagged rows for scores spread continuously: per
    row, a union bound over the discontinuities flag_rows looks for (for the
    reduced-precision exponential baselines, the rounding boundaries its
    numerators may straddle) -- each
    in-window key lies within delta of a Nearest rounding boundary with
    probability 2 delta (its position inside the interval is spread evenly),
    within delta of the FWM edge with probability 2 delta times the keys per
    unit of u around the edge, and the top (bottom) two scores come within
    delta h of each other with probability delta times the keys per unit of u
    next to the maximum (minimum)."""
    if cfg.op == K.OP_SOFTMAX:
        return 0.0
    S = oracle_scores(Q, Kt, rule)
    B, H, T, _ = Q.shape
    p = np.zeros((B, H, T))
    if cfg.op in (K.OP_SOFTMAX_BF16EXP, K.OP_SOFTMAX_FP8EXP):
        # _rounding_flags: a numerator e moved by a relative rel straddles a
        # rounding boundary of the format with probability 2 rel e / ulp(e)
        mbits, emin = (7, -126) if cfg.op == K.OP_SOFTMAX_BF16EXP else (3, -6)
        for i in range(T):
            L = i + 1 if cfg.causal else T
            x = S[:, :, i, :L] - S[:, :, i, :L].max(-1, keepdims=True)
            e = np.exp(x)
            rel = 2.0 ** -21 + np.abs(x) * 2.0 ** -22
            ex = np.maximum(np.floor(np.log2(np.maximum(e, 1e-300))), emin)
            ulp = 2.0 ** (ex - mbits)
            q = np.where(e >= 1e-6, 2 * rel * e / ulp, 0.0).sum(-1)
            p[:, :, i] = np.minimum(q, 1.0)
        return float(p.mean())
    tau = float(np.float32(cfg.tau))
    for i in range(T):
        L = i + 1 if cfg.causal else T
        s = S[:, :, i, :L]
        m = s.max(-1, keepdims=True)
        n = s.min(-1, keepdims=True)
        h = (m - n) / cfg.K if cfg.cal == K.CAL_MINMAX else np.full_like(m, tau / cfg.K)
        u = (m - s) / np.where(h > 0, h, 1.0)
        q = np.zeros((B, H))
        if cfg.rec == K.REC_NEAREST:
            inw = (u <= cfg.K + delta) if cfg.cal == K.CAL_FWM else np.ones_like(u, bool)
            q += 2 * delta * inw.sum(-1)
        if cfg.cal == K.CAL_FWM:
            q += 2 * delta * (np.abs(u - cfg.K) < 0.5).sum(-1)
        if L >= 2:
            q += delta * (u < 1).sum(-1)
            if cfg.cal == K.CAL_MINMAX:
                q += delta * (u > cfg.K - 1).sum(-1)
        if cfg.cal == K.CAL_MINMAX:
            q = np.where((m - n)[..., 0] < 0.5e-12, 0.0, q)
        p[:, :, i] = np.minimum(q, 1.0)
    return float(p.mean())


# every comparison's flagged fraction and budget, reported at the end of the run
FLAG_LOG: list = []


def check_flags(flags: np.ndarray, budget: float, label: str = ""):
    """The flagged rows must stay within what the discontinuities predict:
    at most twice the expected fraction plus three rows of slack."""
    frac = float(flags.mean())
    FLAG_LOG.append((label, frac, budget, int(flags.size)))
    assert frac <= 2.0 * budget + 3.0 / flags.size, (label, frac, budget)
    return frac


def rel_l2(a, b, mask=None) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    if mask is not None:
        a, b = a[mask], b[mask]
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def run_gpu(Q, Kt, V, dO, cfg: K.Config, want_dS=False, bwd=True):
    dev = "cuda"
    q, k, v, g = (torch.from_numpy(np.ascontiguousarray(x)).to(dev) for x in (Q, Kt, V, dO))
    B, H, T, d = q.shape
    bufs = K.Buffers(B, H, T, d, cfg)
    K.kiattn_fwd(q, k, v, bufs.O, bufs.stats, cfg)
    out = {"O": bufs.O}
    dS = None
    if bwd:
        if want_dS:
            dS = torch.empty((B, H, T, T), dtype=torch.float32, device=dev)
        K.kiattn_bwd(q, k, v, bufs.O, g, bufs.stats, bufs.dQ, bufs.dK, bufs.dV, bufs.work, cfg,
                     dS_dbg=dS)
        out.update(dQ=bufs.dQ, dK=bufs.dK, dV=bufs.dV)
        if dS is not None:
            out["dS"] = dS
    torch.cuda.synchronize()
    err = K.kiattn_device_error(True)
    assert err == 0, f"device error word {err}"
    res = {kk: vv.cpu().numpy() for kk, vv in out.items()}
    res["_bufs"] = bufs
    return res


def compare(Q, Kt, V, dO, cfg: K.Config, rule: int, tol: float, delta: float, want_dS=True,
            bwd=True):
    """Run GPU and oracle; return dict of errors and the flag mask."""
    flags = flag_rows(Q, Kt, cfg, rule, delta)
    dO2 = dO.copy()
    dO2[flags] = 0.0
    gpu = run_gpu(Q, Kt, V, dO2, cfg, want_dS=want_dS, bwd=bwd)
    orc = ref.attention(Q, Kt, V, dO2, ref_cfg(cfg, rule), want_bwd=bwd, dump=want_dS and bwd)
    keep = ~flags
    errs = {"O": rel_l2(gpu["O"], orc["O"], keep), "flagged": int(flags.sum()),
            "rows": int(flags.size),
            "flag_frac": check_flags(flags, flag_budget(Q, Kt, cfg, rule, delta),
                                     f"{Q.shape} {cfg}")}
    if bwd:
        for name in ("dQ", "dK", "dV"):
            errs[name] = rel_l2(gpu[name], orc[name])
        if want_dS:
            errs["dS"] = rel_l2(gpu["dS"], orc["dS"])
            ds = gpu["dS"].astype(np.float64)
            sums = np.abs(ds.sum(-1))
            norms = np.linalg.norm(ds, axis=-1)
            # rows whose exact gradient vanishes (one visible key, zeroed
            # upstream) carry no zero-sum information
            live = np.linalg.norm(orc["dS"], axis=-1) > 1e-12 * max(np.linalg.norm(orc["dS"]), 1e-300)
            r = np.where(live, sums / np.maximum(norms, 1e-30), 0.0)
            errs["zero_sum"] = float(r.max())
    return errs, gpu, orc
