"""Helpers for the GPU parity tests: move numpy inputs to the device, call the
product through its binding, and compare against the oracle with the
tolerances the method's definition allows."""
import numpy as np
import torch

import ternary_weight_token_b200 as bn


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def bf16_dev(bits_u16):
    """A bf16 device tensor from raw uint16 bit patterns."""
    return dev(np.ascontiguousarray(bits_u16).view(np.int16)).view(torch.bfloat16)


def gpu_pack(W, dtype=torch.float32):
    """Pack an fp32 numpy weight through the product; returns (packed, gamma) numpy."""
    N, K = W.shape
    Wd = dev(W).to(dtype) if dtype != torch.float32 else dev(W)
    packed, gamma, ws = bn.alloc_packed(N, K)
    bn.bitnet_pack_weights(Wd, packed, gamma, ws)
    torch.cuda.synchronize()
    return packed.cpu().numpy(), gamma.cpu().numpy()[0]


def gpu_quant(X, prelude=bn.BITNET_PRELUDE_NONE, gain=None, eps=1e-5, x_dev=None):
    M, K = X.shape
    Xd = x_dev if x_dev is not None else dev(X)
    q, s, rs = bn.alloc_quant(M, K)
    g = None if gain is None else dev(gain)
    bn.bitnet_quant_act(Xd, q, s, rs, prelude=prelude, norm_gain=g, eps=eps)
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy(), rs.cpu().numpy()


def gpu_linear(q, s, rs, packed, gamma, K, N, out=torch.float32, flags=0, residual=None):
    """Contraction + epilogue on device from oracle-side codes (numpy)."""
    M = q.shape[0]
    Y = torch.empty((M, N), dtype=out, device="cuda")
    code = {torch.float32: bn.BITNET_F32, torch.bfloat16: bn.BITNET_BF16,
            torch.int32: bn.BITNET_I32}[out]
    res = None
    if residual is not None:
        res = residual if isinstance(residual, torch.Tensor) else dev(residual).to(out)
    bn.bitnet_linear(dev(q), dev(s), dev(rs), dev(packed), dev(np.array([gamma], np.float32)),
                     K, Y, epilogue=code | flags, residual=res)
    torch.cuda.synchronize()
    return Y.float().cpu().numpy() if out == torch.bfloat16 else Y.cpu().numpy()


# ----------------------------------------------------------------- checks

def assert_f32_close(got, want, rtol=1e-5, what=""):
    """Elementwise relative error <= rtol; exact zeros must stay exact zeros."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    err = np.abs(got - want)
    bad = err > rtol * np.abs(want)
    assert not np.any(bad), (f"{what}: {int(bad.sum())} of {bad.size} elements off by more than "
                             f"{rtol} relative; worst {err[bad].max() if bad.any() else 0}")


def bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (normal range)."""
    x = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(x, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def assert_bf16_matches(got_f32, want_f32, rtol=1e-5, what=""):
    """got (bf16 widened) equals round-to-nearest-even of the oracle's fp32, or
    differs by the rounding of a value the fp32 tolerance moves across a bf16
    midpoint: |got - want| <= 0.5 ulp_bf16 + rtol |want|."""
    got = np.asarray(got_f32, np.float64)
    want = np.asarray(want_f32, np.float64)
    err = np.abs(got - want)
    lim = 0.5 * bf16_ulp(want) + rtol * np.abs(want)
    bad = err > lim
    assert not np.any(bad), f"{what}: {int(bad.sum())} bf16 outputs off; worst {err[bad].max()}"
    zero = want == 0
    assert np.all(got[zero] == 0), f"{what}: exact zeros not kept"


def code_mismatch_stats(got, want):
    d = got.astype(np.int32) - want.astype(np.int32)
    return int(np.count_nonzero(d)), int(np.abs(d).max()) if d.size else 0


def assert_codes_chain(got, want, what=""):
    """Chain tolerance: at most 0.1 % of codes differ, each by +-1 only."""
    n, worst = code_mismatch_stats(got, want)
    assert worst <= 1, f"{what}: a code differs by {worst}"
    assert n <= 0.001 * got.size, f"{what}: {n} of {got.size} codes differ"
