"""CPU oracle for the BitNet b1.58 BitLinear (W1.58A8) path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product (``ternary_weight_token_b200``) never imports it, and it never imports
the product: the two share no code.

The arithmetic lives in ``bitnet_oracle.c`` (plain loops, fp64 where the
definition is a real number, IEEE fp32 where the kernel's precision decides an
integer code).  This module only marshals numpy arrays through ctypes.

Sources, cited per function in the C file:
  * nnterp encyclopedia "bitnet", "The projections quantize their inputs and
    weights": per-token ``round(x * 127 / max|x|)``, weights rounded to
    ``{-1, 0, 1} * mean|W|``, "stored ternary, four to a byte, with a
    weight_scale", and the output equals "the linear map of the rounded input
    by the ternarized weight exactly".
  * same page, "The block, in order" and "The MLP gates with a squared ReLU":
    the FFN composition.
  * "BitNet b1.58 2B4T" (Azure AI catalog), "Model Details": absmean ternary
    weights, absmax per-token int8 activations.
  * "bitnetv2-model" README, "Special Features" / "Architecture Overview":
    H-BitLinear (Hadamard transform on power-of-two widths), 512->2048->512
    FFN with SiLU.
"""
import ctypes
import os

import numpy as np

from . import build as _build

PRELUDE_NONE, PRELUDE_RMSNORM, PRELUDE_FWHT = 0, 1, 2

_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    path = _build.build()
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i32, i64, f32 = ctypes.c_int, ctypes.c_int64, ctypes.c_float
    sig = {
        "orc_absmean": (f32, [P, i64]),
        "orc_ternarize": (None, [P, i64, f32, P]),
        "orc_packed_row_bytes": (i64, [i32]),
        "orc_pack": (None, [P, i32, i32, P]),
        "orc_unpack": (i32, [P, i32, i32, P]),
        "orc_pack_tw2": (None, [P, i32, i32, P]),
        "orc_unpack_tw2": (i32, [P, i32, i32, P]),
        "orc_rmsnorm": (None, [P, i32, i32, P, f32, P]),
        "orc_fwht": (i32, [P, i32, i32, P]),
        "orc_quant_act": (i32, [P, i32, i32, i32, P, f32, P, P, P]),
        "orc_contract": (i32, [P, P, i32, i32, i32, P]),
        "orc_dequant": (None, [P, P, f32, i32, i32, P]),
        "orc_round_bf16_array": (None, [P, i64, P]),
        "orc_relu2_glu_array": (None, [P, P, i64, P]),
        "orc_silu_array": (None, [P, i64, P]),
        "orc_bitlinear": (i32, [P, i32, i32, i32, P, f32, P, f32, i32, P, P]),
        "orc_ffn_relu2": (i32, [P, i32, i32, i32, P, f32, P, f32, P, f32, P, P, f32, i32,
                                P, P, P, P]),
        "orc_hffn": (i32, [P, i32, i32, i32, P, f32, P, f32, P, P]),
        "orc_block_tail": (i32, [P, P, i32, i32, i32, P, f32, P, f32, P, f32, P, f32, P, P, P,
                                 f32, P, P]),
        "orc_set_threads": (None, [i32]),
        "orc_get_threads": (i32, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _i8(a):
    return np.ascontiguousarray(a, dtype=np.int8)


class OracleError(RuntimeError):
    pass


def _check(code, what):
    if code != 0:
        raise OracleError(f"oracle {what} failed with code {code}")


# ------------------------------------------------------------------ weights

def absmean(W):
    """gamma = mean|W| (fp64 sum, one rounding to fp32)."""
    W = _f32(W)
    return np.float32(_load().orc_absmean(_p(W), W.size))


def ternarize(W, gamma):
    """t = clamp(rint(W / gamma), -1, 1) as int8, same shape as W."""
    W = _f32(W)
    t = np.empty(W.shape, dtype=np.int8)
    _load().orc_ternarize(_p(W), W.size, ctypes.c_float(float(gamma)), _p(t))
    return t


def packed_row_bytes(K):
    return int(_load().orc_packed_row_bytes(int(K)))


def pack(T):
    """Ternary codes [N][K] -> packed uint8 [N][packed_row_bytes(K)]."""
    T = _i8(T)
    N, K = T.shape
    out = np.empty((N, packed_row_bytes(K)), dtype=np.uint8)
    _load().orc_pack(_p(T), N, K, _p(out))
    return out


def unpack(P, K):
    P = np.ascontiguousarray(P, dtype=np.uint8)
    N = P.shape[0]
    t = np.empty((N, K), dtype=np.int8)
    _check(_load().orc_unpack(_p(P), N, int(K), _p(t)), "unpack")
    return t


def pack_tw2(T):
    """Ternary codes [N][K] -> the canonical exchange layout TW2, uint8
    [N][K/4]: code t + 1 of weight k at bits 2 (k mod 4) of byte k / 4."""
    T = _i8(T)
    N, K = T.shape
    if K % 4:
        raise OracleError("TW2 needs K to be a multiple of 4")
    out = np.empty((N, K // 4), dtype=np.uint8)
    _load().orc_pack_tw2(_p(T), N, K, _p(out))
    return out


def unpack_tw2(P, K):
    P = np.ascontiguousarray(P, dtype=np.uint8)
    N = P.shape[0]
    t = np.empty((N, K), dtype=np.int8)
    _check(_load().orc_unpack_tw2(_p(P), N, int(K), _p(t)), "unpack_tw2")
    return t


def quantize_weights(W):
    """(gamma, ternary codes, packed bytes) of a weight matrix [N][K]."""
    g = absmean(W)
    t = ternarize(W, g)
    return g, t, pack(t)


# --------------------------------------------------------- activation side

def rmsnorm(X, gain=None, eps=1e-5):
    X = _f32(X)
    M, K = X.shape
    g = None if gain is None else _f32(gain)
    out = np.empty_like(X)
    _load().orc_rmsnorm(_p(X), M, K, _p(g), ctypes.c_float(eps), _p(out))
    return out


def fwht(X):
    X = _f32(X)
    M, n = X.shape
    out = np.empty_like(X)
    _check(_load().orc_fwht(_p(X), M, n, _p(out)), "fwht")
    return out


def quant_act(X, prelude=PRELUDE_NONE, gain=None, eps=1e-5):
    """(int8 codes [M][K], fp32 scale s [M], int32 sum of codes [M])."""
    X = _f32(X)
    M, K = X.shape
    g = None if gain is None else _f32(gain)
    q = np.empty((M, K), dtype=np.int8)
    s = np.empty(M, dtype=np.float32)
    rs = np.empty(M, dtype=np.int32)
    _check(_load().orc_quant_act(_p(X), M, K, int(prelude), _p(g), ctypes.c_float(eps),
                                 _p(q), _p(s), _p(rs)), "quant_act")
    return q, s, rs


def contract(q, T):
    """acc[m, n] = sum_k q[m, k] * t[n, k] (int64 loops, checked into int32)."""
    q, T = _i8(q), _i8(T)
    M, K = q.shape
    N = T.shape[0]
    acc = np.empty((M, N), dtype=np.int32)
    _check(_load().orc_contract(_p(q), _p(T), M, N, K, _p(acc)), "contract (int32 overflow)")
    return acc


def dequant(acc, s, gamma):
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    s = _f32(s)
    M, N = acc.shape
    Y = np.empty((M, N), dtype=np.float32)
    _load().orc_dequant(_p(acc), _p(s), ctypes.c_float(float(gamma)), M, N, _p(Y))
    return Y


def round_bf16(x):
    """fp32 -> nearest bf16 (ties to even), returned widened to fp32."""
    x = _f32(x)
    out = np.empty_like(x)
    _load().orc_round_bf16_array(_p(x), x.size, _p(out))
    return out


def relu2_glu(g, u):
    g, u = _f32(g), _f32(u)
    out = np.empty_like(g)
    _load().orc_relu2_glu_array(_p(g), _p(u), g.size, _p(out))
    return out


def silu(y):
    y = _f32(y)
    out = np.empty_like(y)
    _load().orc_silu_array(_p(y), y.size, _p(out))
    return out


# ------------------------------------------------------------- compositions

def bitlinear(X, T, gamma, prelude=PRELUDE_NONE, gain=None, eps=1e-5, residual=None):
    """prelude -> per-token int8 quant -> ternary contraction -> dequant (+ residual)."""
    X, T = _f32(X), _i8(T)
    M, K = X.shape
    N = T.shape[0]
    g = None if gain is None else _f32(gain)
    r = None if residual is None else _f32(residual)
    Y = np.empty((M, N), dtype=np.float32)
    _check(_load().orc_bitlinear(_p(X), M, K, int(prelude), _p(g), ctypes.c_float(eps),
                                 _p(T), ctypes.c_float(float(gamma)), N, _p(r), _p(Y)),
           "bitlinear")
    return Y


def ffn_relu2(x, Tg, gg, Tu, gu, Td, gd, pre_gain=None, sub_gain=None, eps=1e-5,
              residual=True, keep=False):
    """W1.58A8 FFN half-block: x + down(ffn_sub_norm(relu(gate(z))^2 * up(z))),
    z = RMSNorm(x).  Returns fp32 out (before any bf16 rounding), plus the
    intermediates (m, codes of m, scales of m) when ``keep``."""
    x = _f32(x)
    M, H = x.shape
    I = Tg.shape[0]
    Tg, Tu, Td = _i8(Tg), _i8(Tu), _i8(Td)
    pg = None if pre_gain is None else _f32(pre_gain)
    sg = None if sub_gain is None else _f32(sub_gain)
    out = np.empty((M, H), dtype=np.float32)
    m = np.empty((M, I), dtype=np.float32) if keep else None
    qm = np.empty((M, I), dtype=np.int8) if keep else None
    sm = np.empty(M, dtype=np.float32) if keep else None
    _check(_load().orc_ffn_relu2(_p(x), M, H, I, _p(Tg), ctypes.c_float(float(gg)),
                                 _p(Tu), ctypes.c_float(float(gu)), _p(Td),
                                 ctypes.c_float(float(gd)), _p(pg), _p(sg), ctypes.c_float(eps),
                                 1 if residual else 0, _p(out), _p(m), _p(qm), _p(sm)),
           "ffn_relu2")
    if keep:
        return out, m, qm, sm
    return out


def block_tail(a, x, To, go, Tg, gg, Tu, gu, Td, gd, attn_gain=None, post_gain=None,
               sub_gain=None, eps=1e-5, keep=False):
    """The block after attention: h = x + o_proj(attn_sub_norm(a)), then the
    W1.58A8 FFN with residual on h.  Returns fp32 out (and h when ``keep``)."""
    a, x = _f32(a), _f32(x)
    M, H = x.shape
    I = Tg.shape[0]
    To, Tg, Tu, Td = _i8(To), _i8(Tg), _i8(Tu), _i8(Td)
    gains = [None if g is None else _f32(g) for g in (attn_gain, post_gain, sub_gain)]
    out = np.empty((M, H), dtype=np.float32)
    h = np.empty((M, H), dtype=np.float32) if keep else None
    f = ctypes.c_float
    _check(_load().orc_block_tail(_p(a), _p(x), M, H, I, _p(To), f(float(go)), _p(Tg),
                                  f(float(gg)), _p(Tu), f(float(gu)), _p(Td), f(float(gd)),
                                  _p(gains[0]), _p(gains[1]), _p(gains[2]), f(eps), _p(h),
                                  _p(out)), "block_tail")
    return (out, h) if keep else out


def hffn(x, T1, g1, T2, g2, keep=False):
    """H-BitLinear FFN: W2 . silu(W1 . x), each with an FWHT prelude."""
    x = _f32(x)
    M, D = x.shape
    F = T1.shape[0]
    T1, T2 = _i8(T1), _i8(T2)
    out = np.empty((M, D), dtype=np.float32)
    h = np.empty((M, F), dtype=np.float32) if keep else None
    _check(_load().orc_hffn(_p(x), M, D, F, _p(T1), ctypes.c_float(float(g1)), _p(T2),
                            ctypes.c_float(float(g2)), _p(out), _p(h)), "hffn")
    if keep:
        return out, h
    return out


# ------------------------------------------------------------- data helpers

def bf16_bits_to_f32(u16):
    """Widen raw bf16 bit patterns (uint16) to fp32 exactly."""
    u16 = np.ascontiguousarray(u16, dtype=np.uint16)
    return (u16.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(x):
    """Round fp32 to bf16 (ties to even) and return the uint16 bit patterns."""
    r = round_bf16(x)
    return (r.view(np.uint32) >> 16).astype(np.uint16)


def num_threads():
    """Threads the OpenMP parts of the oracle use."""
    return int(_load().orc_get_threads())


def set_threads(n):
    """Set the threads of the OpenMP parts of the oracle (plumbing, no
    arithmetic); returns the previous count."""
    prev = num_threads()
    _load().orc_set_threads(int(n))
    return prev
