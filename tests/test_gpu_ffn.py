"""GPU parity of the two FFN compositions against the oracle, through the C
ABI: the W1.58A8 block FFN (RMSNorm -> gate/up -> relu^2 * up -> ffn_sub_norm
-> down -> residual) and the H-BitLinear FFN (FWHT -> W1 -> SiLU -> FWHT ->
W2).

Both chains carry fp32 intermediates whose last bit can differ from the
oracle's only next to a rounding midpoint (fp64 sums in another order, fp64
exp in another library), so the int8 codes of the second projection fall
under the chain tolerance and the outputs under relative L2 error <= 1e-3;
the test also reports how many codes actually differ.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
import ternary_weight_token_b200 as bn
from tests.gpu_util import (assert_bf16_matches, assert_codes_chain, bf16_dev,
                            code_mismatch_stats, dev, gpu_quant)

pytestmark = pytest.mark.gpu


def _pack_dev(W):
    N, K = W.shape
    P, g, ws = bn.alloc_packed(N, K)
    bn.bitnet_pack_weights(dev(W), P, g, ws)
    return P, g


def _rel_l2(got, want):
    return float(np.linalg.norm(got.astype(np.float64) - want) / max(np.linalg.norm(want), 1e-30))


def check_chain_output(got, want, codes_dev, codes_or, what):
    """Identical second-stage codes give identical outputs (up to the bf16
    rounding of an fp32 value next to a midpoint); otherwise the chain
    tolerance applies: codes within 0.1 % / +-1 and relative L2 <= 1e-3."""
    assert_codes_chain(codes_dev, codes_or, what + " codes")
    n, _ = code_mismatch_stats(codes_dev, codes_or)
    if n == 0:
        assert_bf16_matches(got, want, what=what)
    # relative L2 against the oracle's own bf16 rounding of its fp32 output
    assert _rel_l2(got, oracle.round_bf16(want)) <= 1e-3, what


def workspace_hidden(ws_np, M, H, I):
    """m and its sub-norm codes from an FFN workspace that was filled with
    0xff bytes before the call.  The fp32 slot after the codes of x holds m
    itself (prefill GEMM, or the persistent decode launch); on the four-launch
    decode route it holds the gate output g, and the up output u sits after
    the codes' scale and sum, m = relu(g)^2 * u being formed on loading.  The
    route shows in that second slot: still 0xff unless the four-launch route
    wrote it."""
    off = 0

    def take(nbytes):
        nonlocal off
        view = ws_np[off:off + nbytes]
        off += (nbytes + 255) // 256 * 256
        return view
    take(M * H), take(M * 4), take(M * 4)
    m_dev = take(M * I * 4).view(np.float32).reshape(M, I)
    qm_dev = take(M * I).view(np.int8).reshape(M, I)
    route = "single"
    if M <= 16:
        take(M * 4), take(M * 4)
        u_raw = take(M * I * 4)
        if not np.all(u_raw == 0xFF):
            m_dev = oracle.relu2_glu(m_dev, u_raw.view(np.float32).reshape(M, I))
            route = "four launches"
    return m_dev, qm_dev, route


def run_ffn_relu2(inp, rows=None, gains=False, separate=False):
    """Device FFN over all tokens; oracle on `rows` (all when None)."""
    M, H = inp["x"].shape
    I = inp["Wg"].shape[0]
    Pg, gg = _pack_dev(inp["Wg"])
    Pu, gu = _pack_dev(inp["Wu"])
    Pd, gd = _pack_dev(inp["Wd"])
    pre = sub = None
    if gains:
        pre = np.random.default_rng(1).uniform(0.5, 1.5, H).astype(np.float32)
        sub = np.random.default_rng(2).uniform(0.5, 1.5, I).astype(np.float32)
    X = bf16_dev(inp["x_bf16"])
    Y = torch.empty((M, H), dtype=torch.bfloat16, device="cuda")
    ws = bn.alloc_ffn_workspace(M, H, I)
    ws.fill_(0xFF)
    variant = bn.BITNET_FFN_RELU2_GLU | (0 if separate else bn.BITNET_FFN_SINGLE_LAUNCH)
    bn.bitnet_ffn(X, Pg, gg, Pu, gu, Pd, gd, Y, ws, variant=variant,
                  pre_norm_gain=None if pre is None else dev(pre),
                  sub_norm_gain=None if sub is None else dev(sub), eps=1e-5)
    torch.cuda.synchronize()
    assert bn.bitnet_check_device_error() == bn.BITNET_OK
    got = Y.float().cpu().numpy()
    m_dev, qm_dev, route = workspace_hidden(ws.cpu().numpy(), M, H, I)
    if M <= 16:
        persistent_shape = H % 128 == 0 and I % 128 == 0
        assert route == ("single" if persistent_shape and not separate else "four launches")
    sel = np.arange(M) if rows is None else np.asarray(rows)
    go, To = {}, {}
    for k in ("Wg", "Wu", "Wd"):
        go[k], To[k], _ = oracle.quantize_weights(inp[k])
    out, m, qm, sm = oracle.ffn_relu2(inp["x"][sel], To["Wg"], go["Wg"], To["Wu"], go["Wu"],
                                      To["Wd"], go["Wd"], pre_gain=pre, sub_gain=sub, eps=1e-5,
                                      residual=True, keep=True)
    return got[sel], out, m_dev[sel], m, qm_dev[sel], qm


@pytest.mark.parametrize("M,H,I,gains", [(64, 256, 512, False), (300, 512, 1024, True),
                                         (9, 256, 512, False), (1, 2560, 6912, True),
                                         (1, 2560, 6912, False), (2, 256, 512, True),
                                         (2, 320, 448, False), (1, 208, 272, True),
                                         (4, 2560, 6912, False), (16, 512, 1024, True),
                                         (17, 256, 512, False), (16, 2560, 6912, False),
                                         (8, 1024, 2048, True), (3, 128, 128, False)])
@pytest.mark.parametrize("separate", [False, True])
def test_ffn_relu2_small(M, H, I, gains, separate):
    """M <= 16 runs gate and up as one decode launch and forms m in the
    sub-norm quantiser; with BITNET_FFN_SINGLE_LAUNCH and widths that are
    multiples of 128, the persistent decode launch (one cooperative grid);
    M = 17 on is the fused gate/up GEMM."""
    if separate and M > 16:
        pytest.skip("the launch option only concerns decode sizes")
    inp = synthetic.ffn_inputs(M, H, I, seed=M)
    got, want, m_dev, m, qm_dev, qm = run_ffn_relu2(inp, gains=gains, separate=separate)
    # gate/up epilogue: m = relu(g)^2 * u
    np.testing.assert_allclose(m_dev, m, rtol=1e-5, atol=0)
    assert np.all(m_dev[m == 0] == 0)
    check_chain_output(got, want, qm_dev, qm, "ffn out")


def test_ffn_relu2_is_zero_where_gate_negative_and_residual_identity():
    """relu^2 gating is exact zero at negative gates; y - x equals the FFN's
    own contribution (checked in fp32 via the oracle's no-residual path)."""
    M, H, I = 32, 256, 512
    inp = synthetic.ffn_inputs(M, H, I, seed=7)
    got, want, m_dev, m, qm_dev, qm = run_ffn_relu2(inp)
    go, To = {}, {}
    for k in ("Wg", "Wu", "Wd"):
        go[k], To[k], _ = oracle.quantize_weights(inp[k])
    G = oracle.bitlinear(inp["x"], To["Wg"], go["Wg"], oracle.PRELUDE_RMSNORM, eps=1e-5)
    assert np.all(m_dev[G <= 0] == 0)
    contrib = oracle.ffn_relu2(inp["x"], To["Wg"], go["Wg"], To["Wu"], go["Wu"], To["Wd"],
                               go["Wd"], residual=False)
    check_chain_output(got, (inp["x"] + contrib).astype(np.float32), qm_dev, qm,
                       "residual identity")


def test_hffn_small():
    M, D, F = 64, 512, 2048
    inp = synthetic.hffn_inputs(M, D, F, seed=3)
    P1, g1 = _pack_dev(inp["W1"])
    P2, g2 = _pack_dev(inp["W2"])
    X = dev(inp["X"])
    Y = torch.empty((M, D), device="cuda")
    ws = bn.alloc_ffn_workspace(M, D, F, bn.BITNET_FFN_HADAMARD_SILU)
    bn.bitnet_ffn(X, P1, g1, None, None, P2, g2, Y, ws, variant=bn.BITNET_FFN_HADAMARD_SILU)
    torch.cuda.synchronize()
    go1, T1, _ = oracle.quantize_weights(inp["W1"])
    go2, T2, _ = oracle.quantize_weights(inp["W2"])
    want, h = oracle.hffn(inp["X"], T1, go1, T2, go2, keep=True)
    got = Y.cpu().numpy()
    assert _rel_l2(got, want) <= 1e-3
    # the workspace holds the first projection's fp32 output (the second
    # quantiser applies the SiLU as it loads it) and the hidden codes
    ws_np = ws.cpu().numpy()
    a256 = lambda n: (n + 255) // 256 * 256
    off = a256(M * D) + 2 * a256(M * 4)
    y1_dev = ws_np[off:off + M * F * 4].view(np.float32).reshape(M, F)
    q1, s1, _ = oracle.quant_act(inp["X"], oracle.PRELUDE_FWHT)
    y1 = oracle.dequant(oracle.contract(q1, T1), s1, go1)
    np.testing.assert_allclose(y1_dev, y1, rtol=1e-5, atol=1e-30)
    np.testing.assert_allclose(oracle.silu(y1_dev), h, rtol=1e-5, atol=1e-30)
    off += a256(M * F * 4)
    q_dev = ws_np[off:off + M * F].view(np.int8).reshape(M, F)
    q_or, _, _ = oracle.quant_act(oracle.silu(y1_dev), oracle.PRELUDE_FWHT)
    assert_codes_chain(q_dev, q_or, "hidden codes")
    np.testing.assert_allclose(got, want, rtol=1e-3, atol=1e-3 * np.abs(want).max())


def test_hffn_decode_path():
    """M <= 16 takes the decode GEMV for both projections."""
    M, D, F = 4, 512, 2048
    inp = synthetic.hffn_inputs(M, D, F, seed=8)
    P1, g1 = _pack_dev(inp["W1"])
    P2, g2 = _pack_dev(inp["W2"])
    Y = torch.empty((M, D), device="cuda")
    ws = bn.alloc_ffn_workspace(M, D, F, bn.BITNET_FFN_HADAMARD_SILU)
    bn.bitnet_ffn(dev(inp["X"]), P1, g1, None, None, P2, g2, Y, ws,
                  variant=bn.BITNET_FFN_HADAMARD_SILU)
    torch.cuda.synchronize()
    go1, T1, _ = oracle.quantize_weights(inp["W1"])
    go2, T2, _ = oracle.quantize_weights(inp["W2"])
    want = oracle.hffn(inp["X"], T1, go1, T2, go2)
    assert _rel_l2(Y.cpu().numpy(), want) <= 1e-3


@pytest.mark.parametrize("M", [1, 2, 5])
def test_ffn_relu2_decode_fp32_io(M):
    """The decode route with fp32 input and output (the residual then adds in
    fp32) and a sub-norm gain, against the oracle block."""
    H, I = 512, 1536
    inp = synthetic.ffn_inputs(M, H, I, seed=40 + M)
    Pg, gg = _pack_dev(inp["Wg"])
    Pu, gu = _pack_dev(inp["Wu"])
    Pd, gd = _pack_dev(inp["Wd"])
    sub = np.random.default_rng(3).uniform(0.5, 1.5, I).astype(np.float32)
    go, To = {}, {}
    for k in ("Wg", "Wu", "Wd"):
        go[k], To[k], _ = oracle.quantize_weights(inp[k])
    want, m, qm, sm = oracle.ffn_relu2(inp["x"], To["Wg"], go["Wg"], To["Wu"], go["Wu"], To["Wd"],
                                       go["Wd"], sub_gain=sub, eps=1e-5, residual=True, keep=True)
    for separate in (False, True):
        Y = torch.empty((M, H), device="cuda")
        ws = bn.alloc_ffn_workspace(M, H, I)
        ws.fill_(0xFF)
        variant = bn.BITNET_FFN_RELU2_GLU | (0 if separate else bn.BITNET_FFN_SINGLE_LAUNCH)
        bn.bitnet_ffn(dev(inp["x"]), Pg, gg, Pu, gu, Pd, gd, Y, ws, variant=variant,
                      sub_norm_gain=dev(sub), eps=1e-5)
        torch.cuda.synchronize()
        assert bn.bitnet_check_device_error() == bn.BITNET_OK
        m_dev, qm_dev, route = workspace_hidden(ws.cpu().numpy(), M, H, I)
        assert route == ("four launches" if separate else "single")
        _check_fp32_io(Y, want, m_dev, m, qm_dev, qm)


def _check_fp32_io(Y, want, m_dev, m, qm_dev, qm):
    np.testing.assert_allclose(m_dev, m, rtol=1e-5, atol=0)
    assert_codes_chain(qm_dev, qm, "decode codes")
    got = Y.cpu().numpy()
    if code_mismatch_stats(qm_dev, qm)[0] == 0:
        np.testing.assert_allclose(got, want, rtol=1e-5, atol=1e-6 * np.abs(want).max())
    assert _rel_l2(got, want) <= 1e-3


@pytest.mark.parametrize("M,H,I,dtype", [(1, 2560, 6912, torch.bfloat16), (4, 512, 1024, torch.float32),
                                         (8, 2560, 6912, torch.bfloat16), (3, 256, 384, torch.float32)])
def test_block_tail_decode(M, H, I, dtype):
    """The block after attention in one launch (attn_sub_norm -> o_proj ->
    + x -> post_attention_layernorm -> FFN -> + h) against the oracle's
    block_tail: h within fp32 tolerance, the output within the chain
    tolerance, gains on every norm."""
    rng = np.random.default_rng(M + H)
    W = {k: synthetic.weight(rng, *shape) for k, shape in
         (("Wo", (H, H)), ("Wg", (I, H)), ("Wu", (I, H)), ("Wd", (H, I)))}
    a = synthetic.activations(rng, M, H)
    x = synthetic.activations(rng, M, H)
    if dtype == torch.bfloat16:
        a = oracle.round_bf16(a)
        x = oracle.round_bf16(x)
    gains = {k: rng.uniform(0.5, 1.5, n).astype(np.float32)
             for k, n in (("attn", H), ("post", H), ("sub", I))}
    packs = {k: _pack_dev(W[k]) for k in W}
    Y = torch.empty((M, H), dtype=dtype, device="cuda")
    Hout = torch.empty((M, H), dtype=dtype, device="cuda")
    ws = bn.alloc_block_tail_workspace(M, H, I)
    ws.fill_(0xFF)
    bn.bitnet_block_tail(dev(a).to(dtype), dev(x).to(dtype), *packs["Wo"], *packs["Wg"],
                         *packs["Wu"], *packs["Wd"], Y, ws, H_out=Hout,
                         attn_norm_gain=dev(gains["attn"]), post_norm_gain=dev(gains["post"]),
                         sub_norm_gain=dev(gains["sub"]), eps=1e-5)
    torch.cuda.synchronize()
    assert bn.bitnet_check_device_error() == bn.BITNET_OK
    q = {k: oracle.quantize_weights(W[k]) for k in W}
    want, h = oracle.block_tail(a, x, q["Wo"][1], q["Wo"][0], q["Wg"][1], q["Wg"][0], q["Wu"][1],
                                q["Wu"][0], q["Wd"][1], q["Wd"][0], attn_gain=gains["attn"],
                                post_gain=gains["post"], sub_gain=gains["sub"], eps=1e-5,
                                keep=True)
    got_h = Hout.float().cpu().numpy()
    got = Y.float().cpu().numpy()
    if dtype == torch.bfloat16:
        assert_bf16_matches(got_h, h, what="h")
        assert _rel_l2(got, oracle.round_bf16(want)) <= 1e-3
    else:
        np.testing.assert_allclose(got_h, h, rtol=1e-5, atol=1e-6 * np.abs(h).max())
        assert _rel_l2(got, want) <= 1e-3


def test_block_tail_rejects_prefill_sizes():
    M, H, I = 17, 256, 512
    z = torch.zeros((M, H), device="cuda")
    P = torch.zeros((I, bn.bitnet_packed_row_bytes(H)), dtype=torch.uint8, device="cuda")
    Pd = torch.zeros((H, bn.bitnet_packed_row_bytes(I)), dtype=torch.uint8, device="cuda")
    Po = torch.zeros((H, bn.bitnet_packed_row_bytes(H)), dtype=torch.uint8, device="cuda")
    g = torch.ones(1, device="cuda")
    ws = bn.alloc_block_tail_workspace(M, H, I)
    with pytest.raises(bn.BitnetError) as err:
        bn.bitnet_block_tail(z, z, Po, g, P, g, P, g, Pd, g, z.clone(), ws)
    assert err.value.code == bn.BITNET_ERR_UNSUPPORTED
