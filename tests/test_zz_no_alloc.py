"""bitnet_ffn_noalloc: the FFN entry point that takes no workspace.

Some callers cannot call cudaMalloc: code that runs while a CUDA stream
capture is open in a mode that forbids allocation, or a plugin whose host
application owns all device memory and gives the library no allocator.  For
them the library keeps one fixed device array of scratch (8 MiB) and
bitnet_ffn_noalloc runs the FFN on it.  These tests call it through the C ABI
(the ctypes binding) and check, on two calls in a row, that it returns what
bitnet_ffn with a caller workspace returns, within the tolerance the FFN parity
tests use; and that a request larger than the built-in scratch is refused
before anything is launched.

This file is collected last on purpose, and it passes both alone in a fresh
process and after the rest of the suite.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
import ternary_weight_token_b200 as bn
from tests.gpu_util import assert_bf16_matches, assert_f32_close, bf16_dev, dev

pytestmark = pytest.mark.gpu


def _pack(W):
    P, g, ws = bn.alloc_packed(*W.shape)
    bn.bitnet_pack_weights(dev(W), P, g, ws)
    return P, g


def test_noalloc_ffn_matches_the_workspace_entry_point_twice():
    M, H, I = 48, 512, 1024
    inp = synthetic.ffn_inputs(M, H, I, seed=5)
    (Pg, gg), (Pu, gu), (Pd, gd) = (_pack(inp[k]) for k in ("Wg", "Wu", "Wd"))
    X = bf16_dev(inp["x_bf16"])
    pre = dev(np.random.default_rng(1).uniform(0.5, 1.5, H).astype(np.float32))
    sub = dev(np.random.default_rng(2).uniform(0.5, 1.5, I).astype(np.float32))
    ref = torch.empty((M, H), dtype=torch.bfloat16, device="cuda")
    ws = bn.alloc_ffn_workspace(M, H, I)
    bn.bitnet_ffn(X, Pg, gg, Pu, gu, Pd, gd, ref, ws, pre_norm_gain=pre, sub_norm_gain=sub)
    torch.cuda.synchronize()
    ref_np = ref.float().cpu().numpy()
    for call in range(2):                      # the shared scratch keeps the last call's data
        Y = torch.full((M, H), float("nan"), dtype=torch.bfloat16, device="cuda")
        bn.bitnet_ffn_noalloc(X, Pg, gg, Pu, gu, Pd, gd, Y, pre_norm_gain=pre,
                              sub_norm_gain=sub)
        torch.cuda.synchronize()
        assert_bf16_matches(Y.float().cpu().numpy(), ref_np, what=f"noalloc call {call}")
    assert bn.bitnet_check_device_error() == bn.BITNET_OK


@pytest.mark.parametrize("M", [1, 16])
def test_noalloc_decode_ffn_matches_twice(M):
    """At decode sizes (M <= 16) the GLU FFN runs gate and up as two
    projections of one decode launch and keeps the up projection's fp32
    output in a second piece of the scratch; that path too must match the
    workspace entry point, twice in a row."""
    H, I = 2560, 6912
    inp = synthetic.ffn_inputs(M, H, I, seed=9)
    (Pg, gg), (Pu, gu), (Pd, gd) = (_pack(inp[k]) for k in ("Wg", "Wu", "Wd"))
    X = bf16_dev(inp["x_bf16"])
    ref = torch.empty((M, H), dtype=torch.bfloat16, device="cuda")
    ws = bn.alloc_ffn_workspace(M, H, I)
    bn.bitnet_ffn(X, Pg, gg, Pu, gu, Pd, gd, ref, ws)
    torch.cuda.synchronize()
    ref_np = ref.float().cpu().numpy()
    for call in range(2):
        Y = torch.full((M, H), float("nan"), dtype=torch.bfloat16, device="cuda")
        bn.bitnet_ffn_noalloc(X, Pg, gg, Pu, gu, Pd, gd, Y)
        torch.cuda.synchronize()
        assert_bf16_matches(Y.float().cpu().numpy(), ref_np, what=f"noalloc decode M={M} {call}")
    assert bn.bitnet_check_device_error() == bn.BITNET_OK


def test_noalloc_hadamard_ffn_matches_twice():
    M, D, F = 16, 512, 2048
    inp = synthetic.hffn_inputs(M, D, F, seed=6)
    (P1, g1), (P2, g2) = _pack(inp["W1"]), _pack(inp["W2"])
    X = dev(inp["X"])
    ref = torch.empty((M, D), device="cuda")
    ws = bn.alloc_ffn_workspace(M, D, F, bn.BITNET_FFN_HADAMARD_SILU)
    bn.bitnet_ffn(X, P1, g1, None, None, P2, g2, ref, ws, variant=bn.BITNET_FFN_HADAMARD_SILU)
    torch.cuda.synchronize()
    for call in range(2):
        Y = torch.full((M, D), float("nan"), device="cuda")
        bn.bitnet_ffn_noalloc(X, P1, g1, None, None, P2, g2, Y,
                              variant=bn.BITNET_FFN_HADAMARD_SILU)
        torch.cuda.synchronize()
        assert_f32_close(Y.cpu().numpy(), ref.cpu().numpy(), what=f"noalloc hffn call {call}")


def test_noalloc_refuses_requests_beyond_its_scratch():
    H, I = 2560, 6912
    per_token = H + 5 * I                       # codes of x, fp32 hidden, its codes
    M = bn.BITNET_FFN_NOALLOC_SCRATCH_BYTES // per_token + 16
    assert bn.bitnet_ffn_workspace_size(M, H, I) > bn.BITNET_FFN_NOALLOC_SCRATCH_BYTES
    X = torch.zeros((M, H), dtype=torch.bfloat16, device="cuda")
    Y = torch.full((M, H), 3.0, dtype=torch.bfloat16, device="cuda")
    Pg = torch.zeros((I, bn.bitnet_packed_row_bytes(H)), dtype=torch.uint8, device="cuda")
    Pd = torch.zeros((H, bn.bitnet_packed_row_bytes(I)), dtype=torch.uint8, device="cuda")
    g = torch.ones(1, device="cuda")
    with pytest.raises(bn.BitnetError) as err:
        bn.bitnet_ffn_noalloc(X, Pg, g, Pg, g, Pd, g, Y)
    assert err.value.code == bn.BITNET_ERR_WORKSPACE
    assert "scratch" in bn.bitnet_last_error()
    torch.cuda.synchronize()
    assert torch.all(Y == 3.0)                  # nothing was launched
