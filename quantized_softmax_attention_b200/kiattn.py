"""Python binding of the kiattn C ABI (argument marshalling only).

Every function here has the name of a C entry point in ``include/kiattn.h``
and forwards torch CUDA tensors' device pointers plus the current CUDA
stream.  All arithmetic runs in the CUDA library ``libkiattn.so``; there is
no Python, PyTorch or CPU implementation of the operator behind these calls.
If the library is missing the import fails loudly.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkiattn.so")

CAL_MINMAX, CAL_FWM, CAL_FIXED = 0, 1, 2
REC_LERP, REC_NEAREST = 0, 1
STE_WEIGHT, STE_PROB = 0, 1
GRAD_FULL, GRAD_DETACH, GRAD_MAX_ONLY, GRAD_MIN_ONLY, GRAD_PROJECT = 0, 1, 2, 3, 4
GEMM_TF32, GEMM_FP32 = 0, 1
OP_KINTERVAL, OP_SOFTMAX, OP_SOFTMAX_BF16EXP, OP_SOFTMAX_FP8EXP = 0, 1, 2, 3

ERRORS = {0: "ok", -1: "invalid argument", -2: "unsupported", -3: "CUDA error", -4: "timeout",
          -5: "stats mismatch", -6: "capacity exceeded"}

SYMBOLS = ("kiattn_stats_bytes", "kiattn_workspace_bytes", "kiattn_fwd", "kiattn_bwd",
           "kiattn_weights_from_S", "kiattn_scores", "kiattn_strerror", "kiattn_version",
           "kiattn_device_error", "kiattn_profile_enable", "kiattn_profile_read",
           "kiattn_bwd_noalloc", "kiattn_grad_decomposition", "kiattn_geometry",
           "kiattn_debug_bounded_wait")
NOALLOC_MAX_ROWS = 1 << 20
PHASES = ("fwd", "bwd_prep", "bwd_query_pass", "bwd_key_pass", "bwd_calibration")


class KiattnError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {code} ({ERRORS.get(code, 'unknown')})")
        self.code = code


class kia_config(ctypes.Structure):
    _fields_ = [("n_intervals", ctypes.c_int), ("cal", ctypes.c_int), ("tau", ctypes.c_float),
                ("rec", ctypes.c_int), ("ste", ctypes.c_int), ("grad", ctypes.c_int),
                ("causal", ctypes.c_int), ("gemm", ctypes.c_int), ("op", ctypes.c_int)]


@dataclass(frozen=True)
class Config:
    """The operator's axes (section 3): K, calibration, reconstruction,
    surrogate, gradient mode; plus causal mask, contraction arithmetic and
    operator (K-interval or exact softmax)."""

    K: int = 4
    cal: int = CAL_MINMAX
    tau: float = 6.0
    rec: int = REC_LERP
    ste: int = STE_WEIGHT
    grad: int = GRAD_FULL
    causal: bool = True
    gemm: int = GEMM_TF32
    op: int = OP_KINTERVAL

    def c(self) -> kia_config:
        return kia_config(int(self.K), int(self.cal), float(self.tau), int(self.rec),
                          int(self.ste), int(self.grad), int(bool(self.causal)), int(self.gemm),
                          int(self.op))

    def replace(self, **kw) -> "Config":
        d = dict(self.__dict__)
        d.update(kw)
        return Config(**d)


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"kiattn CUDA library not built: {LIB_PATH} is missing "
                          "(run python -m quantized_softmax_attention_b200.build)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, cp, i = ctypes.c_void_p, ctypes.POINTER(kia_config), ctypes.c_int
    lib.kiattn_stats_bytes.argtypes = [i, i, i, i, cp]
    lib.kiattn_stats_bytes.restype = ctypes.c_size_t
    lib.kiattn_workspace_bytes.argtypes = [i, i, i, i, cp]
    lib.kiattn_workspace_bytes.restype = ctypes.c_size_t
    lib.kiattn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, cp, vp]
    lib.kiattn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, cp, vp, vp]
    lib.kiattn_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, cp,
                                       vp]
    lib.kiattn_bwd_noalloc.restype = i
    lib.kiattn_weights_from_S.argtypes = [vp, i, i, vp, cp, vp, vp, vp, vp, vp, vp]
    lib.kiattn_scores.argtypes = [vp, vp, vp, i, i, i, i, cp, vp]
    lib.kiattn_grad_decomposition.argtypes = [vp, vp, i, i, i, cp, vp, vp]
    lib.kiattn_grad_decomposition.restype = i
    lib.kiattn_geometry.argtypes = [vp, vp, i, i, i, i, cp, vp, vp]
    lib.kiattn_geometry.restype = i
    lib.kiattn_debug_bounded_wait.argtypes = [i, ctypes.c_ulonglong]
    lib.kiattn_debug_bounded_wait.restype = i
    lib.kiattn_strerror.argtypes = [i]
    lib.kiattn_strerror.restype = ctypes.c_char_p
    lib.kiattn_version.restype = i
    lib.kiattn_device_error.argtypes = [i]
    lib.kiattn_profile_enable.argtypes = [i]
    lib.kiattn_profile_enable.restype = i
    lib.kiattn_profile_read.argtypes = [ctypes.POINTER(ctypes.c_float), i]
    lib.kiattn_profile_read.restype = i
    for name in ("kiattn_fwd", "kiattn_bwd", "kiattn_weights_from_S", "kiattn_scores",
                 "kiattn_device_error"):
        getattr(lib, name).restype = i
    return lib


_lib = _load()


def lib():
    return _lib


def _p(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("kiattn takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("kiattn takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _need(fn, name, t, numel=None, nbytes=None, dtype=None):
    """Size and type checks of one argument, before any pointer is passed:
    the library cannot see buffer sizes, so a short buffer is caught here."""
    if t is None:
        return
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{fn}: {name} must be {dtype}, got {t.dtype}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{fn}: {name} has {t.numel()} elements, needs {numel}")
    if nbytes is not None and t.numel() * t.element_size() < nbytes:
        raise ValueError(f"{fn}: {name} holds {t.numel() * t.element_size()} bytes, needs {nbytes}")


def _need_qkv(fn, Q, rest, cfg, stats=None, workspace=None, dS=None):
    f32 = torch.float32
    if Q.dim() != 4:
        raise ValueError(f"{fn}: Q must be [B, H, T, d], got {tuple(Q.shape)}")
    B, H, T, d = Q.shape
    _need(fn, "Q", Q, dtype=f32)
    for name, t in rest.items():
        _need(fn, name, t, numel=Q.numel(), dtype=f32)
    if stats is not None:
        sb = kiattn_stats_bytes(B, H, T, d, cfg)
        _need(fn, "stats", stats, nbytes=sb if sb else None)
    if workspace is not None:
        wb = kiattn_workspace_bytes(B, H, T, d, cfg)
        _need(fn, "workspace", workspace, nbytes=wb if wb else None)
    _need(fn, "dS_dbg", dS, numel=B * H * T * T, dtype=f32)
    return B, H, T, d


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn, rc):
    if rc != 0:
        raise KiattnError(fn, rc)


def kiattn_stats_bytes(B, H, T, d, cfg: Config) -> int:
    return int(_lib.kiattn_stats_bytes(B, H, T, d, ctypes.byref(cfg.c())))


def kiattn_workspace_bytes(B, H, T, d, cfg: Config) -> int:
    return int(_lib.kiattn_workspace_bytes(B, H, T, d, ctypes.byref(cfg.c())))


def kiattn_fwd(Q, K, V, O, stats, cfg: Config, stream=None):
    B, H, T, d = _need_qkv("kiattn_fwd", Q, {"K": K, "V": V, "O": O}, cfg, stats=stats)
    _check("kiattn_fwd", _lib.kiattn_fwd(_p(Q), _p(K), _p(V), _p(O), _p(stats), B, H, T, d,
                                         ctypes.byref(cfg.c()), _stream(stream)))


def kiattn_bwd(Q, K, V, O, dO, stats, dQ, dK, dV, workspace, cfg: Config, dS_dbg=None,
               stream=None):
    B, H, T, d = _need_qkv("kiattn_bwd", Q, {"K": K, "V": V, "O": O, "dO": dO, "dQ": dQ,
                                             "dK": dK, "dV": dV}, cfg, stats=stats,
                           workspace=workspace, dS=dS_dbg)
    _check("kiattn_bwd", _lib.kiattn_bwd(_p(Q), _p(K), _p(V), _p(O), _p(dO), _p(stats), _p(dQ),
                                         _p(dK), _p(dV), _p(dS_dbg), B, H, T, d,
                                         ctypes.byref(cfg.c()), _p(workspace), _stream(stream)))


def kiattn_bwd_noalloc(Q, K, V, O, dO, stats, dQ, dK, dV, cfg: Config, dS_dbg=None,
                       stream=None):
    """Backward with the library's own fixed scratch (no workspace argument),
    for callers that cannot allocate device memory; B*H*T <= NOALLOC_MAX_ROWS."""
    B, H, T, d = Q.shape
    if B * H * T <= NOALLOC_MAX_ROWS:   # beyond it the library refuses before any access
        _need_qkv("kiattn_bwd_noalloc", Q, {"K": K, "V": V, "O": O, "dO": dO, "dQ": dQ, "dK": dK,
                                            "dV": dV}, cfg, stats=stats, dS=dS_dbg)
    _check("kiattn_bwd_noalloc",
           _lib.kiattn_bwd_noalloc(_p(Q), _p(K), _p(V), _p(O), _p(dO), _p(stats), _p(dQ), _p(dK),
                                   _p(dV), _p(dS_dbg), B, H, T, d, ctypes.byref(cfg.c()),
                                   _stream(stream)))


def kiattn_weights_from_S(S, row_len, cfg: Config, w, bin=None, t=None, row_m=None, row_n=None,
                          stream=None):
    fn, f32, i32 = "kiattn_weights_from_S", torch.float32, torch.int32
    if S.dim() != 2:
        raise ValueError(f"{fn}: S must be [rows, cols], got {tuple(S.shape)}")
    rows, cols = S.shape
    _need(fn, "S", S, dtype=f32)
    _need(fn, "row_len", row_len, numel=rows, dtype=i32)
    for name, x, dt in (("w", w, f32), ("bin", bin, i32), ("t", t, f32)):
        _need(fn, name, x, numel=rows * cols, dtype=dt)
    _need(fn, "row_m", row_m, numel=rows, dtype=f32)
    _need(fn, "row_n", row_n, numel=rows, dtype=f32)
    _check("kiattn_weights_from_S",
           _lib.kiattn_weights_from_S(_p(S), rows, cols, _p(row_len), ctypes.byref(cfg.c()), _p(w),
                                      _p(bin), _p(t), _p(row_m), _p(row_n), _stream(stream)))


def kiattn_grad_decomposition(dS, workspace, out, cfg: Config, stream=None):
    """Per-row ||dS_i||^2 and the squared norms of the maximum- and
    minimum-side calibration terms (out: device fp64 [B, H, T, 3]) from the
    dS_dbg and workspace of one kiattn_bwd call with the same cfg."""
    fn = "kiattn_grad_decomposition"
    if dS.dim() != 4 or dS.shape[2] != dS.shape[3]:
        raise ValueError(f"{fn}: dS must be [B, H, T, T], got {tuple(dS.shape)}")
    B, H, T, _ = dS.shape
    _need(fn, "dS", dS, dtype=torch.float32)
    wb = kiattn_workspace_bytes(B, H, T, 64, cfg)
    _need(fn, "workspace", workspace, nbytes=wb if wb else None)
    _need(fn, "out", out, numel=B * H * T * 3, dtype=torch.float64)
    _check("kiattn_grad_decomposition",
           _lib.kiattn_grad_decomposition(_p(dS), _p(workspace), B, H, T, ctypes.byref(cfg.c()),
                                          _p(out), _stream(stream)))


GEO_FIELDS = ("span", "h", "q_norm", "entropy_softmax", "entropy_op", "tv", "top_softmax",
              "top_op")
GEO_FIELD_COUNT = len(GEO_FIELDS)


def kiattn_geometry(S, out, cfg: Config, Q=None, stream=None):
    """Per-row geometry probe of scores S [B, H, T, T] against cfg's grid;
    out: device fp32 [B, H, T, 8] in the order of GEO_FIELDS."""
    fn = "kiattn_geometry"
    if S.dim() != 4 or S.shape[2] != S.shape[3]:
        raise ValueError(f"{fn}: S must be [B, H, T, T], got {tuple(S.shape)}")
    B, H, T, _ = S.shape
    d = Q.shape[-1] if Q is not None else 0
    _need(fn, "S", S, dtype=torch.float32)
    _need(fn, "out", out, numel=B * H * T * GEO_FIELD_COUNT, dtype=torch.float32)
    _need(fn, "Q", Q, numel=B * H * T * d, dtype=torch.float32)
    _check("kiattn_geometry", _lib.kiattn_geometry(_p(S), _p(Q), B, H, T, d,
                                                   ctypes.byref(cfg.c()), _p(out),
                                                   _stream(stream)))


def kiattn_scores(Q, K, S, cfg: Config, stream=None):
    B, H, T, d = _need_qkv("kiattn_scores", Q, {"K": K}, cfg)
    _need("kiattn_scores", "S", S, numel=B * H * T * T, dtype=torch.float32)
    _check("kiattn_scores", _lib.kiattn_scores(_p(Q), _p(K), _p(S), B, H, T, d,
                                               ctypes.byref(cfg.c()), _stream(stream)))


def kiattn_strerror(code: int) -> str:
    return _lib.kiattn_strerror(code).decode()


def kiattn_version() -> int:
    return int(_lib.kiattn_version())


def kiattn_device_error(reset: bool = True) -> int:
    return int(_lib.kiattn_device_error(1 if reset else 0))


def kiattn_debug_bounded_wait(what: int, wait_limit_ns: int = 0):
    """Test hook of the bounded device-side waits: what = 1 makes the
    following tensor-core forwards withhold one operand copy so that their
    waits run out (KIA_ERR_TIMEOUT in kiattn_device_error); wait_limit_ns > 0
    shortens every wait's limit.  kiattn_debug_bounded_wait(0, 0) restores
    the defaults."""
    _check("kiattn_debug_bounded_wait", _lib.kiattn_debug_bounded_wait(int(what), int(wait_limit_ns)))


def kiattn_profile_enable(on: bool = True):
    _check("kiattn_profile_enable", _lib.kiattn_profile_enable(1 if on else 0))


def kiattn_profile_read() -> dict:
    buf = (ctypes.c_float * len(PHASES))()
    n = _lib.kiattn_profile_read(buf, len(PHASES))
    if n < 0:
        raise KiattnError("kiattn_profile_read", n)
    return {PHASES[i]: float(buf[i]) for i in range(n)}


# ------------------------------------------------------------ conveniences

class Buffers:
    """Device buffers for one shape/config: outputs, stats and workspace,
    allocated once with torch (the library itself allocates nothing)."""

    def __init__(self, B, H, T, d, cfg: Config, device="cuda"):
        self.shape = (B, H, T, d)
        f = dict(dtype=torch.float32, device=device)
        self.O = torch.empty(self.shape, **f)
        self.dQ = torch.empty(self.shape, **f)
        self.dK = torch.empty(self.shape, **f)
        self.dV = torch.empty(self.shape, **f)
        sb = kiattn_stats_bytes(B, H, T, d, cfg)
        wb = kiattn_workspace_bytes(B, H, T, d, cfg)
        if sb == 0 or wb == 0:
            raise KiattnError("kiattn_stats_bytes", -1)
        self.stats = torch.empty(sb, dtype=torch.uint8, device=device)
        self.work = torch.empty(wb, dtype=torch.uint8, device=device)


def forward(Q, K, V, cfg: Config, bufs: Buffers | None = None, stream=None):
    bufs = bufs or Buffers(*Q.shape, cfg, device=Q.device)
    kiattn_fwd(Q, K, V, bufs.O, bufs.stats, cfg, stream)
    return bufs


def backward(Q, K, V, dO, cfg: Config, bufs: Buffers, dS_dbg=None, stream=None):
    kiattn_bwd(Q, K, V, bufs.O, dO, bufs.stats, bufs.dQ, bufs.dK, bufs.dV, bufs.work, cfg,
               dS_dbg=dS_dbg, stream=stream)
    return bufs
