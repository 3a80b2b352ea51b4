"""fp64 CPU oracle for K-interval attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import this package.  The product path (the CUDA
library and its Python binding) never imports it, and it imports nothing from
the product: the two share no code.

The arithmetic lives in ``kiattn_ref.c`` (plain loops, fp64, OpenMP over rows
or (batch, head) pairs); this module compiles it with gcc and marshals numpy
arrays through ctypes.  Every function cites the passage of "Pretraining
Transformers with Quantized Softmax in Attention" it follows in the C source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kiattn_ref.c")
_LIB = os.path.join(_HERE, "libkiattn_ref.so")

CAL_MINMAX, CAL_FWM, CAL_FIXED = 0, 1, 2
EXP_EXACT, EXP_BF16, EXP_FP8 = 0, 1, 2
REC_LERP, REC_NEAREST = 0, 1
STE_WEIGHT, STE_PROB = 0, 1
GRAD_FULL, GRAD_DETACH, GRAD_MAX_ONLY, GRAD_MIN_ONLY, GRAD_PROJECT = 0, 1, 2, 3, 4
ROUND_NONE, ROUND_TRUNC, ROUND_RNA, ROUND_RNE = 0, 1, 2, 3

# per-row statistics columns, same order as the C enum
ST_M, ST_N, ST_AM, ST_AN, ST_H, ST_WFWD, ST_WL, ST_WN, ST_A, ST_C, ST_DEGEN = range(11)
ST_COUNT = 11


class _Cfg(ctypes.Structure):
    _fields_ = [
        ("K", ctypes.c_int),
        ("cal", ctypes.c_int),
        ("tau", ctypes.c_double),
        ("rec", ctypes.c_int),
        ("ste", ctypes.c_int),
        ("grad", ctypes.c_int),
        ("causal", ctypes.c_int),
        ("softmax", ctypes.c_int),
        ("rounding", ctypes.c_int),
        ("exp_round", ctypes.c_int),
    ]


@dataclass(frozen=True)
class RefConfig:
    """Operator configuration: the paper's three axes plus K, tau, gradient mode."""

    K: int = 4
    cal: int = CAL_MINMAX
    tau: float = 6.0
    rec: int = REC_LERP
    ste: int = STE_WEIGHT
    grad: int = GRAD_FULL
    causal: bool = True
    softmax: bool = False
    rounding: int = ROUND_NONE
    exp_round: int = EXP_EXACT   # softmax numerator: exact, bfloat16 or FP8 E4M3 (App. D.5)

    def c(self) -> _Cfg:
        return _Cfg(int(self.K), int(self.cal), float(self.tau), int(self.rec), int(self.ste),
                    int(self.grad), int(bool(self.causal)), int(bool(self.softmax)),
                    int(self.rounding), int(self.exp_round))

    def replace(self, **kw) -> "RefConfig":
        d = dict(self.__dict__)
        d.update(kw)
        return RefConfig(**d)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        fp = ctypes.POINTER(ctypes.c_float)
        ip = ctypes.POINTER(ctypes.c_int)
        cp = ctypes.POINTER(_Cfg)
        _lib.kiattn_ref_rows.argtypes = [dp, ip, ctypes.c_int, ctypes.c_int, dp, cp, dp, dp,
                                         dp, dp, dp, dp, dp]
        _lib.kiattn_ref_attention.argtypes = [fp, fp, fp, fp, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, cp, ctypes.c_int, ctypes.c_int,
                                              dp, dp, dp, dp, dp, dp, dp, dp]
        _lib.kiattn_ref_weights_fp32.argtypes = [fp, ctypes.c_int, ctypes.c_int, ip, cp, fp, ip,
                                                 fp, fp, fp]
        _lib.kiattn_ref_round_exp_format.argtypes = [ctypes.c_float, ctypes.c_int]
        _lib.kiattn_ref_round_exp_format.restype = ctypes.c_float
        _lib.kiattn_ref_own_exp.argtypes = [ctypes.c_double]
        _lib.kiattn_ref_own_exp.restype = ctypes.c_double
    return _lib


def _ptr(a, ct):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ct))


def rows(S, row_len, cfg: RefConfig, dP=None, frozen_m=None, frozen_n=None):
    """Row-level operator on fp64 scores (section 3 / Appendices A-B).

    Returns dict with P (forward probabilities), P_L, P_N, dS (if dP given)
    and stats [rows, ST_COUNT]."""
    S = np.ascontiguousarray(S, dtype=np.float64)
    rws, cols = S.shape
    row_len = np.ascontiguousarray(row_len, dtype=np.int32)
    out = {
        "P": np.zeros((rws, cols)),
        "P_L": np.zeros((rws, cols)),
        "P_N": np.zeros((rws, cols)),
        "stats": np.zeros((rws, ST_COUNT)),
    }
    dS = None
    if dP is not None:
        dP = np.ascontiguousarray(dP, dtype=np.float64)
        dS = np.zeros((rws, cols))
    fm = None if frozen_m is None else np.ascontiguousarray(frozen_m, dtype=np.float64)
    fn = None if frozen_n is None else np.ascontiguousarray(frozen_n, dtype=np.float64)
    c = cfg.c()
    rc = lib().kiattn_ref_rows(_ptr(S, ctypes.c_double), _ptr(row_len, ctypes.c_int), rws, cols,
                               _ptr(dP, ctypes.c_double), ctypes.byref(c),
                               _ptr(fm, ctypes.c_double), _ptr(fn, ctypes.c_double),
                               _ptr(out["P"], ctypes.c_double), _ptr(dS, ctypes.c_double),
                               _ptr(out["P_L"], ctypes.c_double),
                               _ptr(out["P_N"], ctypes.c_double),
                               _ptr(out["stats"], ctypes.c_double))
    if rc != 0:
        raise ValueError("kiattn_ref_rows: bad arguments")
    if dS is not None:
        out["dS"] = dS
    return out


def attention(Q, K, V, dO, cfg: RefConfig, bh_range=None, want_bwd=True, dump=False):
    """Full operator on fp32 [B, H, T, d] (or [BH, T, d]) arrays, fp64 arithmetic.

    Returns dict with O, O_bar, stats and, when want_bwd, dQ, dK, dV; with
    dump also P [BH,T,T] and dS [BH,T,T].  bh_range=(b0, b1) restricts the
    computation to flattened (batch, head) indices b0..b1-1 (other entries
    stay zero)."""
    shape = Q.shape
    T, d = shape[-2], shape[-1]
    BH = int(np.prod(shape[:-2]))
    f = lambda a: np.ascontiguousarray(np.asarray(a, dtype=np.float32).reshape(BH, T, d))
    Q, K, V = f(Q), f(K), f(V)
    dO = f(dO) if (dO is not None and want_bwd) else None
    b0, b1 = (0, BH) if bh_range is None else bh_range
    O = np.zeros((BH, T, d))
    Ob = np.zeros((BH, T, d))
    stats = np.zeros((BH, T, ST_COUNT))
    dQ = dK = dV = None
    if dO is not None:
        dQ, dK, dV = np.zeros((BH, T, d)), np.zeros((BH, T, d)), np.zeros((BH, T, d))
    P = dS = None
    if dump:
        P = np.zeros((BH, T, T))
        if dO is not None:
            dS = np.zeros((BH, T, T))
    c = cfg.c()
    rc = lib().kiattn_ref_attention(
        _ptr(Q, ctypes.c_float), _ptr(K, ctypes.c_float), _ptr(V, ctypes.c_float),
        _ptr(dO, ctypes.c_float), BH, T, d, ctypes.byref(c), b0, b1,
        _ptr(O, ctypes.c_double), _ptr(Ob, ctypes.c_double), _ptr(dQ, ctypes.c_double),
        _ptr(dK, ctypes.c_double), _ptr(dV, ctypes.c_double), _ptr(stats, ctypes.c_double),
        _ptr(P, ctypes.c_double), _ptr(dS, ctypes.c_double))
    if rc != 0:
        raise ValueError("kiattn_ref_attention: bad arguments")
    out = {"O": O.reshape(shape), "O_bar": Ob.reshape(shape),
           "stats": stats.reshape(shape[:-1] + (ST_COUNT,))}
    if dO is not None:
        out.update(dQ=dQ.reshape(shape), dK=dK.reshape(shape), dV=dV.reshape(shape))
    if dump:
        out["P"] = P.reshape(shape[:-1] + (T,))
        if dS is not None:
            out["dS"] = dS.reshape(shape[:-1] + (T,))
    return out


def grad_decomposition(Q, K, V, dO, cfg: RefConfig, bh_range=None):
    """Fixed-upstream decomposition of the score gradient (Appendix F, "The
    detached-gradient record and its replication"; Table S24), fp64, by
    definition: the calibration terms of a mode are what it adds to the
    detached gradient at the same upstream, dS_mode - dS_detach; the
    maximum-dependent term is that difference at the row's argmax key (under
    the zero-sum projection the whole common-mode shift), the
    minimum-dependent term the difference at the argmin key.  Returns
    [BH, T, 3]: ||dS_mode,i||^2, ||max term||^2, ||min term||^2 per row."""
    mode = attention(Q, K, V, dO, cfg, bh_range=bh_range, dump=True)
    det = attention(Q, K, V, dO, cfg.replace(grad=GRAD_DETACH), bh_range=bh_range,
                    dump=True)
    dS, diff = mode["dS"], mode["dS"] - det["dS"]
    T = dS.shape[-1]
    dS = dS.reshape(-1, T, T)
    diff = diff.reshape(-1, T, T)
    st = mode["stats"].reshape(-1, T, ST_COUNT)
    out = np.zeros((dS.shape[0], T, 3))
    out[..., 0] = np.sum(dS * dS, axis=-1)
    am = st[..., ST_AM].astype(np.int64)
    an = st[..., ST_AN].astype(np.int64)
    at_m = np.take_along_axis(diff, am[..., None], axis=-1)[..., 0]
    at_n = np.take_along_axis(diff, an[..., None], axis=-1)[..., 0]
    if cfg.grad == GRAD_PROJECT:
        out[..., 1] = np.sum(diff * diff, axis=-1)
    else:
        out[..., 1] = at_m * at_m
        out[..., 2] = np.where(an != am, at_n * at_n, 0.0)
    return out


def weights_fp32(S, row_len, cfg: RefConfig):
    """The fp32 weight stage as a fixed sequence of fp32 operations (the
    bit-exact contract of the CUDA weight stage).  Returns w, bin, t, m, n."""
    S = np.ascontiguousarray(S, dtype=np.float32)
    rws, cols = S.shape
    row_len = np.ascontiguousarray(row_len, dtype=np.int32)
    w = np.zeros((rws, cols), np.float32)
    b = np.zeros((rws, cols), np.int32)
    t = np.zeros((rws, cols), np.float32)
    m = np.zeros(rws, np.float32)
    n = np.zeros(rws, np.float32)
    c = cfg.c()
    rc = lib().kiattn_ref_weights_fp32(_ptr(S, ctypes.c_float), rws, cols,
                                       _ptr(row_len, ctypes.c_int), ctypes.byref(c),
                                       _ptr(w, ctypes.c_float), _ptr(b, ctypes.c_int),
                                       _ptr(t, ctypes.c_float), _ptr(m, ctypes.c_float),
                                       _ptr(n, ctypes.c_float))
    if rc != 0:
        raise ValueError("kiattn_ref_weights_fp32: bad arguments")
    return {"w": w, "bin": b, "t": t, "m": m, "n": n}


GEO_SPAN, GEO_H, GEO_QNORM, GEO_ENT_SOFTMAX, GEO_ENT_OP, GEO_TV, GEO_TOP_SOFTMAX, GEO_TOP_OP = range(8)
GEO_FIELDS = 8


def geometry(S, row_len, cfg: RefConfig, Q=None):
    """Geometry probe per row ("Pretraining Transformers with Quantized Softmax
    in Attention", section 4 geometry probe, section 5.4, Appendix D.6 and
    Figure S4): span m - n, native width h, ||q_i||, entropy of softmax(s_i)
    and of the operator's forward probabilities, their total variation, and
    the softmax and operator mass on the keys whose nearest grid node is
    node 0 (the top rounding bucket).  The grid decisions (node, tail) and
    the operator weights are those of the fp32 weight stage, so that both
    sides take them in the same precision; everything else is fp64.
    S: [rows, cols] scores (rounded to fp32), row_len: visible keys per row;
    Q: [rows, d] or None.  Returns [rows, GEO_FIELDS]."""
    S32 = np.ascontiguousarray(S, dtype=np.float32)
    rws, cols = S32.shape
    row_len = np.asarray(row_len, dtype=np.int64)
    ws = weights_fp32(S32, row_len, cfg)
    vis = np.arange(cols)[None, :] < row_len[:, None]
    m = ws["m"].astype(np.float64)
    n = ws["n"].astype(np.float64)
    out = np.zeros((rws, GEO_FIELDS))
    out[:, GEO_SPAN] = m - n
    if cfg.cal == CAL_MINMAX:
        out[:, GEO_H] = np.where(m - n < 1e-12, 0.0, (m - n) / cfg.K)
    else:
        out[:, GEO_H] = float(np.float32(cfg.tau)) / cfg.K
    if Q is not None:
        out[:, GEO_QNORM] = np.linalg.norm(np.asarray(Q, np.float64).reshape(rws, -1), axis=1)
    x = np.where(vis, S32.astype(np.float64) - m[:, None], -np.inf)
    e = np.exp(x)
    Psm = e / e.sum(axis=1, keepdims=True)
    w = np.where(vis, ws["w"].astype(np.float64), 0.0)
    Pop = w / w.sum(axis=1, keepdims=True)

    def entropy(P):
        with np.errstate(divide="ignore", invalid="ignore"):
            return -np.sum(np.where(P > 0, P * np.log(P), 0.0), axis=1)

    out[:, GEO_ENT_SOFTMAX] = entropy(Psm)
    out[:, GEO_ENT_OP] = entropy(Pop)
    out[:, GEO_TV] = 0.5 * np.abs(Pop - Psm).sum(axis=1)
    node = ws["bin"].astype(np.int64)
    if cfg.rec == REC_LERP:   # the stage records k and t; the nearest node is k + [t >= 1/2]
        node = np.where(node >= 0, node + (ws["t"] >= np.float32(0.5)), node)
    top = vis & (node == 0)
    out[:, GEO_TOP_SOFTMAX] = np.where(top, Psm, 0.0).sum(axis=1)
    out[:, GEO_TOP_OP] = np.where(top, Pop, 0.0).sum(axis=1)
    return out


def round_exp_format(x: float, mode: int) -> float:
    """The oracle's rounding of an fp32 value to bfloat16 (mode 1) or FP8
    E4M3 (mode 2), nearest-even (Appendix D.5 baselines)."""
    return lib().kiattn_ref_round_exp_format(float(x), int(mode))


def own_exp(x: float) -> float:
    """The oracle's fp64 exponential (Cody-Waite reduction + Taylor series)."""
    return lib().kiattn_ref_own_exp(float(x))
