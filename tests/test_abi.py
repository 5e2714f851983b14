"""CPU checks of the C ABI boundary: the library loads, exports every function
``include/bitnet.h`` declares, and rejects bad arguments on the host before
touching any device (no GPU is needed for any of these calls)."""
import ctypes
import os
import re

import pytest

import ternary_weight_token_b200 as bn
from ternary_weight_token_b200 import _binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitnet.h")


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^BITNET_API\s+[\w\s\*]*?\b(bitnet_\w+)\s*\(", src, re.M)))


def test_header_declares_the_four_calls():
    names = declared_functions()
    for n in ("bitnet_pack_weights", "bitnet_quant_act", "bitnet_linear", "bitnet_ffn"):
        assert n in names
    assert len(names) >= 12


def test_library_exports_every_declared_symbol():
    lib = bn.library()
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} is declared in bitnet.h but not exported"


def test_library_is_sm100a_native():
    assert "sm_100a" in bn.bitnet_version()


def test_packed_row_bytes():
    assert bn.bitnet_packed_row_bytes(16) == 16
    assert bn.bitnet_packed_row_bytes(64) == 16
    assert bn.bitnet_packed_row_bytes(80) == 32
    assert bn.bitnet_packed_row_bytes(2560) == 640
    assert bn.bitnet_packed_row_bytes(6912) == 1728
    assert bn.bitnet_packed_row_bytes(0) == 0


def test_workspace_sizes():
    assert bn.bitnet_pack_workspace_size(6912, 2560) >= 8
    need = bn.bitnet_ffn_workspace_size(2048, 2560, 6912)
    # codes of x, fp32 hidden activation and its codes, plus per-token vectors
    assert need >= 2048 * 2560 + 2048 * 6912 * 5
    assert bn.bitnet_ffn_workspace_size(-1, 2560, 6912) == 0
    # decode sizes (M <= 16) also hold the up projection's fp32 output
    for M in (1, 4, 16):
        glu = bn.bitnet_ffn_workspace_size(M, 2560, 6912, bn.BITNET_FFN_RELU2_GLU)
        had = bn.bitnet_ffn_workspace_size(M, 2560, 6912, bn.BITNET_FFN_HADAMARD_SILU)
        assert glu >= had + M * 6912 * 4
    assert (bn.bitnet_ffn_workspace_size(17, 2560, 6912, bn.BITNET_FFN_RELU2_GLU)
            == bn.bitnet_ffn_workspace_size(17, 2560, 6912, bn.BITNET_FFN_HADAMARD_SILU))


# Raw ctypes calls with fake, aligned pointers: validation must reject them
# before any launch, so no device memory is ever touched.
FAKE = ctypes.c_void_p(0x10000)
FAKE2 = ctypes.c_void_p(0x20000)
MISALIGNED = ctypes.c_void_p(0x10008)


def _lin(**kw):
    a = dict(Xq=FAKE, xs=FAKE, xrs=FAKE, W=FAKE, g=FAKE, M=4, N=8, K=64, Y=FAKE2, epi=0,
             res=None)
    a.update(kw)
    return bn.library().bitnet_linear(a["Xq"], a["xs"], a["xrs"], a["W"], a["g"], a["M"],
                                      a["N"], a["K"], a["Y"], a["epi"], a["res"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(K=17), bn.BITNET_ERR_INVALID_ARG),
    (dict(K=0), bn.BITNET_ERR_INVALID_ARG),
    (dict(K=16400), bn.BITNET_ERR_INVALID_ARG),
    (dict(M=-1), bn.BITNET_ERR_INVALID_ARG),
    (dict(Xq=None), bn.BITNET_ERR_INVALID_ARG),
    (dict(xrs=None), bn.BITNET_ERR_INVALID_ARG),
    (dict(g=None), bn.BITNET_ERR_INVALID_ARG),
    (dict(Y=MISALIGNED), bn.BITNET_ERR_INVALID_ARG),
    (dict(epi=7), bn.BITNET_ERR_INVALID_ARG),
    (dict(epi=0x40), bn.BITNET_ERR_INVALID_ARG),
    (dict(epi=bn.BITNET_I32 | bn.BITNET_EPI_SILU), bn.BITNET_ERR_UNSUPPORTED),
    (dict(epi=bn.BITNET_EPI_RESIDUAL), bn.BITNET_ERR_INVALID_ARG),
    (dict(res=FAKE), bn.BITNET_ERR_INVALID_ARG),
])
def test_linear_rejects_bad_arguments(kw, code):
    assert _lin(**kw) == code
    assert bn.bitnet_last_error() != ""


def test_linear_empty_shapes_are_noops():
    assert _lin(M=0) == bn.BITNET_OK
    assert _lin(N=0, Xq=None) == bn.BITNET_OK


def test_quant_rejects_bad_arguments():
    q = bn.library().bitnet_quant_act
    assert q(FAKE, 0, 4, 24, 2, None, 1e-5, FAKE, FAKE, None, None) == bn.BITNET_ERR_INVALID_ARG
    assert q(FAKE, 0, 4, 96, 2, None, 1e-5, FAKE, FAKE, None, None) == bn.BITNET_ERR_INVALID_ARG
    assert q(FAKE, 0, 4, 64, 9, None, 1e-5, FAKE, FAKE, None, None) == bn.BITNET_ERR_INVALID_ARG
    assert q(FAKE, 5, 4, 64, 0, None, 1e-5, FAKE, FAKE, None, None) == bn.BITNET_ERR_INVALID_ARG
    assert q(FAKE, 0, 4, 64, 0, FAKE, 1e-5, FAKE, FAKE, None, None) == bn.BITNET_ERR_INVALID_ARG
    assert q(FAKE, 0, 4, 64, 1, None, -1.0, FAKE, FAKE, None, None) == bn.BITNET_ERR_INVALID_ARG
    assert q(FAKE, 0, 4, 64, 0, None, 1e-5, None, FAKE, None, None) == bn.BITNET_ERR_INVALID_ARG
    assert q(MISALIGNED, 0, 4, 64, 0, None, 1e-5, FAKE, FAKE, None, None) == \
        bn.BITNET_ERR_INVALID_ARG
    assert q(FAKE, 0, 0, 64, 0, None, 1e-5, None, None, None, None) == bn.BITNET_OK


def test_pack_rejects_bad_arguments():
    p = bn.library().bitnet_pack_weights
    ws = bn.bitnet_pack_workspace_size(8, 64)
    assert p(FAKE, 0, 8, 60, FAKE, FAKE, FAKE2, ws, None) == bn.BITNET_ERR_INVALID_ARG
    assert p(FAKE, 2, 8, 64, FAKE, FAKE, FAKE2, ws, None) == bn.BITNET_ERR_INVALID_ARG
    assert p(FAKE, 0, 8, 64, None, FAKE, FAKE2, ws, None) == bn.BITNET_ERR_INVALID_ARG
    assert p(FAKE, 0, 8, 64, FAKE, FAKE, FAKE2, ws - 1, None) == bn.BITNET_ERR_WORKSPACE
    assert p(FAKE, 0, 8, 64, FAKE, FAKE, None, ws, None) == bn.BITNET_ERR_WORKSPACE


def test_tw2_conversions_reject_bad_arguments():
    for fn in (bn.library().bitnet_export_tw2, bn.library().bitnet_import_tw2):
        assert fn(FAKE, 8, 60, FAKE2, None) == bn.BITNET_ERR_INVALID_ARG      # K % 16
        assert fn(FAKE, 8, 32768, FAKE2, None) == bn.BITNET_ERR_INVALID_ARG   # K too large
        assert fn(None, 8, 64, FAKE2, None) == bn.BITNET_ERR_INVALID_ARG
        assert fn(FAKE, 8, 64, None, None) == bn.BITNET_ERR_INVALID_ARG
        assert fn(MISALIGNED, 8, 64, FAKE2, None) == bn.BITNET_ERR_INVALID_ARG
        assert fn(FAKE, -1, 64, FAKE2, None) == bn.BITNET_ERR_INVALID_ARG
        assert fn(FAKE, 0, 64, FAKE2, None) == bn.BITNET_OK                   # no-op


def test_linear_multi_rejects_bad_arguments():
    import ctypes
    f = bn.library().bitnet_linear_multi
    arr = lambda *v: (ctypes.c_void_p * len(v))(*v)
    ns = lambda *v: (ctypes.c_int * len(v))(*v)
    P = arr(FAKE, FAKE2)
    G = arr(FAKE, FAKE)
    Ys = arr(FAKE2, FAKE2)
    ok = f(FAKE, FAKE, FAKE, 2, P, G, ns(64, 32), 0, 64, Ys, bn.BITNET_F32, None)
    assert ok == bn.BITNET_OK                                         # M = 0: validated no-op
    assert f(FAKE, FAKE, FAKE, 0, P, G, ns(64, 32), 4, 64, Ys, bn.BITNET_F32, None) == \
        bn.BITNET_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 5, P, G, ns(64, 32), 4, 64, Ys, bn.BITNET_F32, None) == \
        bn.BITNET_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 2, None, G, ns(64, 32), 4, 64, Ys, bn.BITNET_F32, None) == \
        bn.BITNET_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 2, P, G, ns(64, 0), 4, 64, Ys, bn.BITNET_F32, None) == \
        bn.BITNET_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 2, arr(FAKE, None), G, ns(64, 32), 4, 64, Ys, bn.BITNET_F32,
             None) == bn.BITNET_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 2, P, G, ns(64, 32), 4, 60, Ys, bn.BITNET_F32, None) == \
        bn.BITNET_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 2, P, G, ns(64, 32), 4, 64, Ys,
             bn.BITNET_F32 | bn.BITNET_EPI_RESIDUAL, None) == bn.BITNET_ERR_UNSUPPORTED


def test_ffn_rejects_bad_arguments():
    f = bn.library().bitnet_ffn
    ws = bn.bitnet_ffn_workspace_size(4, 64, 128, 0)

    def call(variant=0, xd=1, yd=1, H=64, I=128, up=FAKE, gup=FAKE, wsb=ws, pre=None):
        return f(FAKE, xd, 4, H, I, FAKE, FAKE, up, gup, FAKE, FAKE, pre, None, 1e-5, variant,
                 FAKE2, yd, FAKE, wsb, None)
    assert call(variant=3) == bn.BITNET_ERR_INVALID_ARG
    assert call(xd=0, yd=1) == bn.BITNET_ERR_UNSUPPORTED
    assert call(up=None) == bn.BITNET_ERR_INVALID_ARG
    assert call(wsb=ws - 1) == bn.BITNET_ERR_WORKSPACE
    assert call(variant=1, H=96) == bn.BITNET_ERR_INVALID_ARG            # not a power of two
    assert call(variant=1) == bn.BITNET_ERR_INVALID_ARG                  # up given to H-FFN
    assert call(variant=1, up=None, gup=None, pre=FAKE) == bn.BITNET_ERR_INVALID_ARG
    assert call(H=60) == bn.BITNET_ERR_INVALID_ARG


def test_binding_refuses_host_tensors():
    import torch
    W = torch.zeros((4, 64))
    with pytest.raises(ValueError):
        bn.bitnet_pack_weights(W, W, W, W)


def test_debug_timeout_validates_its_limit():
    assert bn.library().bitnet_debug_wait_timeout(0, None) == bn.BITNET_ERR_INVALID_ARG
    assert bn.library().bitnet_debug_wait_timeout(2000000, None) == bn.BITNET_ERR_INVALID_ARG


def test_package_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_binding, "_lib", None)
    monkeypatch.setattr(_binding, "library_path", lambda: str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        _binding.library()
