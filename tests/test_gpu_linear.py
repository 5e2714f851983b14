"""GPU parity of the BitLinear contraction and its epilogues (decode GEMV for
M <= 16, tcgen05 GEMM above) against the oracle, through the C ABI.

Each kernel gets the oracle's own codes, scales and packed weights, so the
int32 contraction must match bit for bit; fp32 outputs must be within 1e-5
relative (the dequantisation is fp64 on both sides, so they are equal except
next to an fp32 midpoint); bf16 outputs must be the nearest-even rounding of
the oracle's fp32 value.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
import ternary_weight_token_b200 as bn
from tests.gpu_util import assert_bf16_matches, assert_f32_close, dev, gpu_linear

pytestmark = pytest.mark.gpu


def _case(M, K, N, seed, prelude=oracle.PRELUDE_NONE):
    rng_w, rng_x = synthetic.streams(seed, 2)
    W = synthetic.weight(rng_w, N, K)
    X = synthetic.activations(rng_x, M, K)
    g, T, P = oracle.quantize_weights(W)
    q, s, rs = oracle.quant_act(X, prelude)
    return X, g, T, P, q, s, rs


SHAPES = [
    # decode GEMV
    (1, 16, 1), (1, 2560, 2560), (2, 80, 33), (3, 256, 512), (4, 2560, 640), (8, 256, 512),
    (15, 6912, 100), (16, 2560, 257),
    # tensor-core GEMM: several tiles and ragged tails in M (tokens) and N (weights)
    (17, 256, 128), (64, 80, 129), (127, 2560, 300), (129, 512, 128), (300, 2560, 300),
    (256, 6912, 256), (513, 1024, 1000),
]


@pytest.mark.parametrize("M,K,N", SHAPES)
def test_linear_int32_bit_exact(M, K, N):
    X, g, T, P, q, s, rs = _case(M, K, N, seed=M * 1000 + N)
    got = gpu_linear(q, s, rs, P, g, K, N, out=torch.int32)
    np.testing.assert_array_equal(got, oracle.contract(q, T))


# Shapes with more 128 x 128 tiles than the 148 persistent CTAs: every CTA
# runs two or more tiles, so each TMEM accumulator buffer is reused (the
# epilogue's zeroing, the buffer-empty barrier's phase flip, the alternating
# token-factor buffers); ragged last tiles in both directions.
MULTI_TILE = [(2048, 2560, 1280), (2048, 256, 4096), (1500, 512, 2000)]


@pytest.mark.parametrize("M,K,N", MULTI_TILE)
def test_persistent_gemm_every_epilogue_bit_exact(M, K, N):
    X, g, T, P, q, s, rs = _case(M, K, N, seed=M + 7 * N)
    acc = oracle.contract(q, T)
    np.testing.assert_array_equal(gpu_linear(q, s, rs, P, g, K, N, out=torch.int32), acc)
    y = oracle.dequant(acc, s, g)
    assert_f32_close(gpu_linear(q, s, rs, P, g, K, N, out=torch.float32), y, what="f32")
    assert_bf16_matches(gpu_linear(q, s, rs, P, g, K, N, out=torch.bfloat16), y, what="bf16")
    R = oracle.round_bf16(synthetic.activations(np.random.default_rng(M), M, N))
    gotr = gpu_linear(q, s, rs, P, g, K, N, out=torch.bfloat16, flags=bn.BITNET_EPI_RESIDUAL,
                      residual=dev(R).to(torch.bfloat16))
    assert_bf16_matches(gotr, (R + y).astype(np.float32), what="bf16 residual")


@pytest.mark.parametrize("M", [3, 5, 8])
@pytest.mark.parametrize("K,N", [(256, 512), (512, 300), (64, 77), (1024, 1024)])
def test_small_matrix_decode_every_epilogue(M, K, N):
    """3-8 tokens on weight matrices of at most 2^20 weights run the streaming
    dp4a kernel with an 8-token instantiation (ragged N, tokens short of 8):
    int32 bit-exact, fp32 / bf16 / residual / SiLU against the oracle."""
    X, g, T, P, q, s, rs = _case(M, K, N, seed=M * 7 + K + N)
    acc = oracle.contract(q, T)
    np.testing.assert_array_equal(gpu_linear(q, s, rs, P, g, K, N, out=torch.int32), acc)
    y = oracle.dequant(acc, s, g)
    assert_f32_close(gpu_linear(q, s, rs, P, g, K, N, out=torch.float32), y, what="f32")
    assert_bf16_matches(gpu_linear(q, s, rs, P, g, K, N, out=torch.bfloat16), y, what="bf16")
    R = synthetic.activations(np.random.default_rng(N + M), M, N)
    got = gpu_linear(q, s, rs, P, g, K, N, out=torch.float32, flags=bn.BITNET_EPI_RESIDUAL,
                     residual=R)
    assert_f32_close(got, (R + y).astype(np.float32), what="residual")
    got = gpu_linear(q, s, rs, P, g, K, N, out=torch.float32, flags=bn.BITNET_EPI_SILU)
    assert_f32_close(got, oracle.silu(y), what="silu")


@pytest.mark.parametrize("M,K,N", [(1, 2560, 2560), (16, 6912, 300), (300, 2560, 300),
                                   (200, 512, 2048)])
def test_linear_f32_and_bf16(M, K, N):
    X, g, T, P, q, s, rs = _case(M, K, N, seed=M + N)
    want = oracle.dequant(oracle.contract(q, T), s, g)
    got = gpu_linear(q, s, rs, P, g, K, N, out=torch.float32)
    assert_f32_close(got, want, what="f32 out")
    assert np.all(got[want == 0] == 0)
    gotb = gpu_linear(q, s, rs, P, g, K, N, out=torch.bfloat16)
    assert_bf16_matches(gotb, want, what="bf16 out")


@pytest.mark.parametrize("M", [4, 160])
def test_linear_residual_and_silu(M):
    K, N = 512, 384
    X, g, T, P, q, s, rs = _case(M, K, N, seed=77 + M)
    y = oracle.dequant(oracle.contract(q, T), s, g)
    R = synthetic.activations(np.random.default_rng(5), M, N)
    got = gpu_linear(q, s, rs, P, g, K, N, out=torch.float32, flags=bn.BITNET_EPI_RESIDUAL,
                     residual=R)
    assert_f32_close(got, (R + y).astype(np.float32), what="residual")
    Rb = oracle.round_bf16(R)
    gotb = gpu_linear(q, s, rs, P, g, K, N, out=torch.bfloat16, flags=bn.BITNET_EPI_RESIDUAL,
                      residual=dev(Rb).to(torch.bfloat16))
    assert_bf16_matches(gotb, (Rb + y).astype(np.float32), what="bf16 residual")
    got = gpu_linear(q, s, rs, P, g, K, N, out=torch.float32, flags=bn.BITNET_EPI_SILU)
    assert_f32_close(got, oracle.silu(y), what="silu")


def test_linear_extreme_codes():
    """All +127 / -128 codes against all +1 / -1 weights at K = 16384: the int32
    accumulator holds 128 * 16384 with no overflow."""
    K, N = 16384, 130
    q = np.full((20, K), 127, np.int8)
    q[1::2] = -128
    T = np.ones((N, K), np.int8)
    T[1::2] = -1
    P = oracle.pack(T)
    s = np.ones(20, np.float32)
    rs = q.astype(np.int64).sum(axis=1).astype(np.int32)
    for M in (3, 20):
        got = gpu_linear(q[:M], s[:M], rs[:M], P, np.float32(1.0), K, N, out=torch.int32)
        np.testing.assert_array_equal(got, oracle.contract(q[:M], T))


def test_linear_zero_rows_and_zero_gamma():
    K, N = 256, 200
    X, g, T, P, q, s, rs = _case(40, K, N, seed=3)
    q[5] = 0
    s[5] = 1.0
    rs[5] = 0
    got = gpu_linear(q, s, rs, P, g, K, N)
    assert np.all(got[5] == 0)
    Z = np.full_like(P, 0x55)          # every weight 0
    got = gpu_linear(q, s, rs, Z, np.float32(0.0), K, N)
    assert np.all(got == 0)


def test_linear_empty_is_noop():
    Y = torch.full((0, 8), 7.0, device="cuda")
    q = torch.empty((0, 32), dtype=torch.int8, device="cuda")
    s = torch.empty(0, device="cuda")
    rs = torch.empty(0, dtype=torch.int32, device="cuda")
    P = torch.empty((8, 16), dtype=torch.uint8, device="cuda")
    g = torch.ones(1, device="cuda")
    bn.bitnet_linear(q, s, rs, P, g, 32, Y)
    torch.cuda.synchronize()


def test_full_chain_matches_oracle():
    """pack -> quant -> linear all on the device against the oracle's chain."""
    M, K, N = 96, 2560, 640
    rng_w, rng_x = synthetic.streams(31, 2)
    W = synthetic.weight(rng_w, N, K)
    X = synthetic.activations(rng_x, M, K)
    Wd, Xd = dev(W), dev(X)
    packed, gamma, ws = bn.alloc_packed(N, K)
    bn.bitnet_pack_weights(Wd, packed, gamma, ws)
    q, s, rs = bn.alloc_quant(M, K)
    bn.bitnet_quant_act(Xd, q, s, rs)
    Y = torch.empty((M, N), device="cuda")
    bn.bitnet_linear(q, s, rs, packed, gamma, K, Y)
    torch.cuda.synchronize()
    g, T, _ = oracle.quantize_weights(W)
    assert_f32_close(Y.cpu().numpy(), oracle.bitlinear(X, T, g), what="chain")


def test_prefill_early_weight_loads_see_the_weights_packed_before():
    """BITNET_LAUNCH_PDL on a prefill call (M > 16): the GEMM loads its first
    weight tiles while the quantiser before it runs.  Each round re-packs new
    weights into the same buffer, quantises a new batch and projects it on one
    stream with no host synchronisation: every output must be the oracle's for
    that round's weights (the quantiser lets the GEMM launch only after the
    pack has completed)."""
    M, K, N = 300, 512, 640
    rng_w, rng_x = synthetic.streams(47, 2)
    P, g, ws = bn.alloc_packed(N, K)
    q, s, rs = bn.alloc_quant(M, K)
    outs = []
    for rnd in range(4):
        W = synthetic.weight(rng_w, N, K)
        X = synthetic.activations(rng_x, M, K)
        Wd, Xd = dev(W), dev(X)
        bn.bitnet_pack_weights(Wd, P, g, ws)
        bn.bitnet_quant_act(Xd, q, s, rs)
        Y = torch.empty((M, N), dtype=torch.int32, device="cuda")
        bn.bitnet_linear(q, s, rs, P, g, K, Y, epilogue=bn.BITNET_I32 | bn.BITNET_LAUNCH_PDL)
        outs.append((W, X, Y, Wd, Xd))
    torch.cuda.synchronize()
    for W, X, Y, _, _ in outs:
        _, T, _ = oracle.quantize_weights(W)
        qo, _, _ = oracle.quant_act(X)
        np.testing.assert_array_equal(Y.cpu().numpy(), oracle.contract(qo, T))


def test_decode_with_programmatic_dependent_launch():
    """Decode calls launched with BITNET_LAUNCH_PDL right behind the kernel that
    writes their activation codes still read the new codes: each step quantises
    a fresh token batch and immediately runs the projection on it."""
    M, K, N = 4, 2560, 2560
    rng_w, rng_x = synthetic.streams(41, 2)
    W = synthetic.weight(rng_w, N, K)
    g, T, P = oracle.quantize_weights(W)
    Pd, gd = dev(P), dev(np.array([g], np.float32))
    q, s, rs = bn.alloc_quant(M, K)
    outs, xs = [], []
    for step in range(6):
        X = synthetic.activations(rng_x, M, K)
        xs.append(X)
        Xd = dev(X)
        torch.cuda.synchronize()
        bn.bitnet_quant_act(Xd, q, s, rs)
        Y = torch.empty((M, N), device="cuda")
        bn.bitnet_linear(q, s, rs, Pd, gd, K, Y, epilogue=bn.BITNET_F32 | bn.BITNET_LAUNCH_PDL)
        outs.append(Y)
    torch.cuda.synchronize()
    for X, Y in zip(xs, outs):
        assert_f32_close(Y.cpu().numpy(), oracle.bitlinear(X, T, g), what="pdl step")


@pytest.mark.parametrize("M", [1, 3, 4, 16])
def test_decode_independent_projections_overlap(M):
    """BITNET_LAUNCH_PDL_INPUTS: consecutive decode calls that read one set of
    activation codes (as q/k/v or gate/up do) may run everything but their
    output stores under the preceding call.  Distinct weights, a shared
    output written by every call (the last call's values must remain) and
    distinct outputs, all bit-exact against the oracle (int32); one fp32
    output per round against the oracle's dequantisation.  One token runs the
    streaming dp4a kernel, 3-16 the cluster tensor-core decode kernel."""
    K = 2560
    rng_w, rng_x = synthetic.streams(43, 2)
    X = synthetic.activations(rng_x, M, K)
    q, s, rs = oracle.quant_act(X)
    qd, sd, rsd = dev(q), dev(s), dev(rs)
    shapes = [(2560, 0), (640, 1), (640, 2), (6912, 3), (2560, 4), (6912, 5)]
    packs = []
    for N, i in shapes:
        W = synthetic.weight(rng_w, N, K)
        g, T, P = oracle.quantize_weights(W)
        packs.append((N, T, dev(P), dev(np.array([g], np.float32))))
    shared = torch.empty((M, 6912), dtype=torch.int32, device="cuda")
    outs = []
    flags = bn.BITNET_I32 | bn.BITNET_LAUNCH_PDL_INPUTS
    f32_outs = []
    for rnd in range(3):
        for N, T, Pd, gd in packs:
            Y = torch.empty((M, N), dtype=torch.int32, device="cuda")
            bn.bitnet_linear(qd, sd, rsd, Pd, gd, K, Y, epilogue=flags)
            if N == 6912:
                bn.bitnet_linear(qd, sd, rsd, Pd, gd, K, shared, epilogue=flags)
            outs.append((Y, T))
        N, T, Pd, gd = packs[rnd]
        Yf = torch.empty((M, N), dtype=torch.float32, device="cuda")
        bn.bitnet_linear(qd, sd, rsd, Pd, gd, K, Yf,
                         epilogue=bn.BITNET_F32 | bn.BITNET_LAUNCH_PDL_INPUTS)
        f32_outs.append((Yf, T, float(gd.cpu()[0])))
    torch.cuda.synchronize()
    for Y, T in outs:
        np.testing.assert_array_equal(Y.cpu().numpy(), oracle.contract(q, T))
    for Yf, T, g in f32_outs:
        assert_f32_close(Yf.cpu().numpy(), oracle.dequant(oracle.contract(q, T), s, g),
                         what="independent f32")
    np.testing.assert_array_equal(shared.cpu().numpy(), oracle.contract(q, packs[-1][1]))
    assert bn.bitnet_check_device_error() == bn.BITNET_OK


@pytest.mark.parametrize("M", [1, 2, 3, 4, 16, 64])
@pytest.mark.parametrize("Ns", [(2560, 640, 640), (300, 77, 640, 1000)])
def test_linear_multi_matches_separate_projections(M, Ns):
    """bitnet_linear_multi: the q/k/v shapes of the 2B model (and ragged
    widths, four projections) in one call, each output bit-exact (int32) and
    equal to the bf16 rounding of the oracle, on the dp4a (M <= 2), cluster
    tensor-core (M <= 16) and prefill (M = 64) paths."""
    K = 2560
    rng_w, rng_x = synthetic.streams(sum(Ns) + M, 2)
    X = synthetic.activations(rng_x, M, K)
    q, s, rs = oracle.quant_act(X)
    packs = []
    for N in Ns:
        g, T, P = oracle.quantize_weights(synthetic.weight(rng_w, N, K))
        packs.append((N, g, T, dev(P), dev(np.array([g], np.float32))))
    for out in (torch.int32, torch.bfloat16):
        Ys = [torch.empty((M, N), dtype=out, device="cuda") for N, *_ in packs]
        flags = bn.BITNET_I32 if out == torch.int32 else bn.BITNET_BF16
        bn.bitnet_linear_multi(dev(q), dev(s), dev(rs), [pk[3] for pk in packs],
                               [pk[4] for pk in packs], K, Ys,
                               epilogue=flags | (bn.BITNET_LAUNCH_PDL if M <= 16 else 0))
        torch.cuda.synchronize()
        for Y, (N, g, T, _, _) in zip(Ys, packs):
            if out == torch.int32:
                np.testing.assert_array_equal(Y.cpu().numpy(), oracle.contract(q, T))
            else:
                want = oracle.dequant(oracle.contract(q, T), s, g)
                assert_bf16_matches(Y.float().cpu().numpy(), want, what=f"multi N={N}")
    assert bn.bitnet_check_device_error() == bn.BITNET_OK


@pytest.mark.parametrize("M", [1, 2])
@pytest.mark.parametrize("K,Ns", [(2560, (2560, 640, 640, 6912)), (6912, (300, 77, 1000, 2000))])
def test_independent_multi_projection_bulk_rows(M, K, Ns):
    """Independent 1-2 token calls on 4 MB or more of weights copy each CTA's
    weight rows into shared memory in bulk, one copy per projection the rows
    fall in: projections whose boundaries fall inside a CTA's rows (and
    ragged widths) give every output bit-exact (int32), twice in a row."""
    rng_w, rng_x = synthetic.streams(sum(Ns) + K + M, 2)
    X = synthetic.activations(rng_x, M, K)
    q, s, rs = oracle.quant_act(X)
    packs = []
    for N in Ns:
        g, T, P = oracle.quantize_weights(synthetic.weight(rng_w, N, K))
        packs.append((N, T, dev(P), dev(np.array([g], np.float32))))
    assert sum(Ns) * bn.bitnet_packed_row_bytes(K) >= 1 << 22
    for _ in range(2):
        Ys = [torch.full((M, N), -7, dtype=torch.int32, device="cuda") for N, *_ in packs]
        bn.bitnet_linear_multi(dev(q), dev(s), dev(rs), [pk[2] for pk in packs],
                               [pk[3] for pk in packs], K, Ys,
                               epilogue=bn.BITNET_I32 | bn.BITNET_LAUNCH_PDL_INPUTS)
        torch.cuda.synchronize()
        for Y, (N, T, _, _) in zip(Ys, packs):
            np.testing.assert_array_equal(Y.cpu().numpy(), oracle.contract(q, T),
                                          err_msg=f"N={N}")
    assert bn.bitnet_check_device_error() == bn.BITNET_OK


@pytest.mark.parametrize("flags", [0, bn.BITNET_LAUNCH_PDL, bn.BITNET_LAUNCH_PDL_INPUTS],
                         ids=["plain", "pdl", "pdl_inputs"])
@pytest.mark.parametrize("K,N", [(2560, 2560), (2560, 6912), (6912, 2560)])
def test_decode_shapes_all_m(K, N, flags):
    """The 2B-model decode shapes for every token count 1..16, int32
    bit-exact, in each launch mode: the mode and the token count pick the
    kernel (streaming, flat or cluster tensor-core) and the cluster split
    (3, 4, 7 or 8 CTAs per 128-row tile on these shapes)."""
    rng_w, rng_x = synthetic.streams(K + N, 2)
    W = synthetic.weight(rng_w, N, K)
    g, T, P = oracle.quantize_weights(W)
    X = synthetic.activations(rng_x, 16, K)
    q, s, rs = oracle.quant_act(X)
    for M in (1, 2, 3, 4, 5, 8, 9, 13, 16):
        got = gpu_linear(q[:M], s[:M], rs[:M], P, g, K, N, out=torch.int32, flags=flags)
        np.testing.assert_array_equal(got, oracle.contract(q[:M], T), err_msg=f"M={M}")
