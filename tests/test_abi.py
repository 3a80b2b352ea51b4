"""Host-side checks of the C ABI (no GPU needed): the library builds for
sm_100a, loads, exports every entry point that include/kiattn.h declares,
sizes its buffers, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def K():
    from quantized_softmax_attention_b200 import build
    build.build()
    from quantized_softmax_attention_b200 import kiattn
    return kiattn


def _declared():
    src = open(os.path.join(ROOT, "include", "kiattn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kiattn_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol(K):
    lib = ctypes.CDLL(K.LIB_PATH)
    names = _declared()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(K.SYMBOLS)


def test_version_and_strerror(K):
    assert K.kiattn_version() >= 10000
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert K.kiattn_strerror(code) != "unknown error"
    assert K.kiattn_strerror(-99) == "unknown error"


def test_buffer_sizes(K):
    cfg = K.Config(K=4, cal=K.CAL_MINMAX)
    B, H, T, d = 2, 3, 300, 64
    rows = B * H * T
    sb = K.kiattn_stats_bytes(B, H, T, d, cfg)
    # 8 per-row words + per-row grid of K+1 values, plus header and padding
    assert sb >= rows * (8 + 5) * 4
    assert sb < rows * (8 + 5) * 4 + 64 * 1024
    fwm = K.kiattn_stats_bytes(B, H, T, d, cfg.replace(cal=K.CAL_FWM))
    assert fwm < sb
    prob = K.kiattn_stats_bytes(B, H, T, d, cfg.replace(rec=K.REC_NEAREST, ste=K.STE_PROB))
    assert prob >= sb + rows * d * 4          # O_L for Prob-STE
    wb = K.kiattn_workspace_bytes(B, H, T, d, cfg)
    assert rows * 7 * 4 <= wb < rows * 7 * 4 + 4096
    assert K.kiattn_stats_bytes(B, H, T, 96, cfg) == 0      # d unsupported
    assert K.kiattn_stats_bytes(B, H, T, d, cfg.replace(K=0)) == 0
    assert K.kiattn_stats_bytes(B, H, T, d, cfg.replace(K=65)) == 0
    assert K.kiattn_stats_bytes(B, H, T, d, cfg.replace(cal=K.CAL_FWM, tau=0.0)) == 0


def test_bad_arguments_rejected_without_launch(K):
    lib = K.lib()
    c = K.Config().c()
    fake = ctypes.c_void_p(1 << 20)          # never dereferenced: checks fail first
    # null pointers
    assert lib.kiattn_fwd(None, fake, fake, fake, fake, 1, 1, 128, 64, ctypes.byref(c), None) == -1
    # unsupported head size
    assert lib.kiattn_fwd(fake, fake, fake, fake, fake, 1, 1, 128, 96, ctypes.byref(c), None) == -2
    # misaligned pointer
    odd = ctypes.c_void_p((1 << 20) + 4)
    assert lib.kiattn_fwd(odd, fake, fake, fake, fake, 1, 1, 128, 64, ctypes.byref(c), None) == -1
    # bad enum / K
    bad = K.Config(grad=7).c()
    assert lib.kiattn_fwd(fake, fake, fake, fake, fake, 1, 1, 128, 64, ctypes.byref(bad), None) == -1
    bad = K.Config(K=100).c()
    assert lib.kiattn_fwd(fake, fake, fake, fake, fake, 1, 1, 128, 64, ctypes.byref(bad), None) == -2
    # empty shapes
    assert lib.kiattn_fwd(fake, fake, fake, fake, fake, 1, 1, 0, 64, ctypes.byref(c), None) == -1
    assert lib.kiattn_bwd(fake, fake, fake, fake, fake, fake, fake, fake, fake, None, 0, 1, 16, 64,
                          ctypes.byref(c), fake, None) == -1
    assert lib.kiattn_bwd(fake, fake, fake, fake, None, fake, fake, fake, fake, None, 1, 1, 16, 64,
                          ctypes.byref(c), fake, None) == -1
    assert lib.kiattn_weights_from_S(fake, 0, 8, fake, ctypes.byref(c), fake, None, None, None,
                                     None, None) == -1
    assert lib.kiattn_scores(fake, fake, None, 1, 1, 8, 64, ctypes.byref(c), None) == -1
    assert lib.kiattn_fwd(fake, fake, fake, fake, fake, 1, 1, 128, 64, None, None) == -1


def test_product_path_does_not_import_the_oracle():
    """The binding and the CUDA sources never reference the oracle."""
    pkg = os.path.join(ROOT, "quantized_softmax_attention_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "kiattn_ref" not in txt, f


def test_binding_checks_buffer_sizes_before_passing_pointers():
    """The library cannot see buffer sizes, so the binding checks them (and
    the dtypes) before any pointer is formed; correctly sized host tensors
    pass the checks and are then refused as not being CUDA tensors."""
    import torch
    K = pytest.importorskip("quantized_softmax_attention_b200.kiattn")
    cfg = K.Config()
    B, H, T, d = 1, 2, 128, 64
    x = torch.zeros((B, H, T, d))
    sb = K.kiattn_stats_bytes(B, H, T, d, cfg)
    wb = K.kiattn_workspace_bytes(B, H, T, d, cfg)
    st, wk = torch.zeros(sb, dtype=torch.uint8), torch.zeros(wb, dtype=torch.uint8)

    def refused(fn, *a, **kw):
        with pytest.raises(ValueError) as e:
            fn(*a, **kw)
        return str(e.value)

    assert "CUDA" in refused(K.kiattn_fwd, x, x, x, x, st, cfg)
    assert "needs" in refused(K.kiattn_fwd, x, x[:, :1], x, x, st, cfg)
    assert "bytes" in refused(K.kiattn_fwd, x, x, x, x, st[:-1], cfg)
    assert "float32" in refused(K.kiattn_fwd, x, x.double(), x, x, st, cfg)
    assert "CUDA" in refused(K.kiattn_bwd, x, x, x, x, x, st, x, x, x, wk, cfg)
    assert "bytes" in refused(K.kiattn_bwd, x, x, x, x, x, st, x, x, x, wk[:8], cfg)
    assert "needs" in refused(K.kiattn_bwd, x, x, x, x, x, st, x, x, x, wk, cfg,
                              dS_dbg=torch.zeros((B, H, T, T - 1)))
    S = torch.zeros((B, H, T, T))
    assert "CUDA" in refused(K.kiattn_scores, x, x, S, cfg)
    assert "needs" in refused(K.kiattn_scores, x, x, S[..., :-1], cfg)
    assert "CUDA" in refused(K.kiattn_geometry, S, torch.zeros((B, H, T, 8)), cfg, Q=x)
    assert "needs" in refused(K.kiattn_geometry, S, torch.zeros((B, H, T, 7)), cfg)
    assert "CUDA" in refused(K.kiattn_grad_decomposition, S, wk,
                             torch.zeros((B, H, T, 3), dtype=torch.float64), cfg)
    assert "float64" in refused(K.kiattn_grad_decomposition, S, wk, torch.zeros((B, H, T, 3)), cfg)
    rows, cols = 4, 9
    Sw = torch.zeros((rows, cols))
    L = torch.full((rows,), cols, dtype=torch.int32)
    assert "CUDA" in refused(K.kiattn_weights_from_S, Sw, L, cfg, torch.zeros((rows, cols)))
    assert "int32" in refused(K.kiattn_weights_from_S, Sw, L.long(), cfg, torch.zeros((rows, cols)))


def test_fixed_step_and_rounded_exp_configs(K):
    """The untruncated fixed step is accepted while its grid's extent,
    ceil(104.5 K / tau) nodes, fits the library's 400-node limit (tau = 6:
    K <= 22), and keeps its FWM-sized stats; the rounded-exponential softmax
    operators are accepted and sized like softmax; unknown calibration or
    operator codes are invalid arguments."""
    B, H, T, d = 1, 2, 256, 64
    fixed = K.Config(K=4, cal=K.CAL_FIXED, tau=6.0)
    fwm = K.Config(K=4, cal=K.CAL_FWM, tau=6.0)
    assert K.kiattn_stats_bytes(B, H, T, d, fixed) > 0
    assert K.kiattn_stats_bytes(B, H, T, d, fixed.replace(K=22)) > 0
    assert K.kiattn_stats_bytes(B, H, T, d, fixed.replace(K=23)) == 0
    assert K.kiattn_stats_bytes(B, H, T, d, fixed.replace(K=64, tau=60.0)) > 0
    # FWM keeps one grid; the fixed step's grid has ~70 nodes instead of 5
    assert 0 < K.kiattn_stats_bytes(B, H, T, d, fixed) - K.kiattn_stats_bytes(B, H, T, d, fwm) < 4096
    sm = K.kiattn_stats_bytes(B, H, T, d, K.Config(op=K.OP_SOFTMAX))
    for op in (K.OP_SOFTMAX_BF16EXP, K.OP_SOFTMAX_FP8EXP):
        assert K.kiattn_stats_bytes(B, H, T, d, K.Config(op=op)) == sm
    assert K.kiattn_stats_bytes(B, H, T, d, K.Config(op=4)) == 0
    assert K.kiattn_stats_bytes(B, H, T, d, K.Config(cal=3)) == 0
    assert K.kiattn_stats_bytes(B, H, T, d, fixed.replace(tau=0.0)) == 0
    lib = K.lib()
    fake = ctypes.c_void_p(1 << 20)
    c = fixed.replace(K=23).c()
    assert lib.kiattn_fwd(fake, fake, fake, fake, fake, 1, 1, 128, 64, ctypes.byref(c), None) == -2


def test_bounded_wait_hook_rejects_bad_arguments(K):
    # checked before any CUDA call, so this runs without a GPU
    with pytest.raises(K.KiattnError) as e:
        K.kiattn_debug_bounded_wait(2, 0)
    assert e.value.code == -1
    with pytest.raises(K.KiattnError):
        K.kiattn_debug_bounded_wait(-1, 5)
