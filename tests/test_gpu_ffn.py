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


def run_ffn_relu2(inp, rows=None, gains=False):
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
    bn.bitnet_ffn(X, Pg, gg, Pu, gu, Pd, gd, Y, ws, variant=bn.BITNET_FFN_RELU2_GLU,
                  pre_norm_gain=None if pre is None else dev(pre),
                  sub_norm_gain=None if sub is None else dev(sub), eps=1e-5)
    torch.cuda.synchronize()
    got = Y.float().cpu().numpy()
    # the workspace holds the fp32 hidden activation m and its codes; at
    # decode sizes (M <= 16) the gate output g in m's place and the up output
    # u after the codes' scale and sum, m = relu(g)^2 * u formed on loading
    ws_np = ws.cpu().numpy()
    off = 0

    def take(nbytes):
        nonlocal off
        view = ws_np[off:off + nbytes]
        off += (nbytes + 255) // 256 * 256
        return view
    take(M * H), take(M * 4), take(M * 4)
    m_dev = take(M * I * 4).view(np.float32).reshape(M, I)
    qm_dev = take(M * I).view(np.int8).reshape(M, I)
    if M <= 16:
        take(M * 4), take(M * 4)
        u_dev = take(M * I * 4).view(np.float32).reshape(M, I)
        m_dev = oracle.relu2_glu(m_dev, u_dev)
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
                                         (17, 256, 512, False)])
def test_ffn_relu2_small(M, H, I, gains):
    """M <= 16 runs gate and up as one decode launch (streaming kernel for
    1-2 tokens, cluster tensor-core kernel for 3-16) and forms m in the
    sub-norm quantiser; M = 17 on is the fused gate/up GEMM."""
    inp = synthetic.ffn_inputs(M, H, I, seed=M)
    got, want, m_dev, m, qm_dev, qm = run_ffn_relu2(inp, gains=gains)
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
    # second-stage codes: quantise the device's own hidden activation too
    ws_np = ws.cpu().numpy()
    off = (M * D + 255) // 256 * 256 + 2 * ((M * 4 + 255) // 256 * 256)
    h_dev = ws_np[off:off + M * F * 4].view(np.float32).reshape(M, F)
    np.testing.assert_allclose(h_dev, h, rtol=1e-5, atol=1e-30)
    q_dev, _, _ = gpu_quant(h_dev, bn.BITNET_PRELUDE_FWHT)
    q_or, _, _ = oracle.quant_act(h, oracle.PRELUDE_FWHT)
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
    Y = torch.empty((M, H), device="cuda")
    ws = bn.alloc_ffn_workspace(M, H, I)
    bn.bitnet_ffn(dev(inp["x"]), Pg, gg, Pu, gu, Pd, gd, Y, ws, variant=bn.BITNET_FFN_RELU2_GLU,
                  sub_norm_gain=dev(sub), eps=1e-5)
    torch.cuda.synchronize()
    assert bn.bitnet_check_device_error() == bn.BITNET_OK
    go, To = {}, {}
    for k in ("Wg", "Wu", "Wd"):
        go[k], To[k], _ = oracle.quantize_weights(inp[k])
    want, m, qm, sm = oracle.ffn_relu2(inp["x"], To["Wg"], go["Wg"], To["Wu"], go["Wu"], To["Wd"],
                                       go["Wd"], sub_gain=sub, eps=1e-5, residual=True, keep=True)
    ws_np = ws.cpu().numpy()
    off = lambda n: (n + 255) // 256 * 256
    base = off(M * H) + 2 * off(M * 4)
    g_dev = ws_np[base:base + M * I * 4].view(np.float32).reshape(M, I)
    qbase = base + off(M * I * 4)
    qm_dev = ws_np[qbase:qbase + M * I].view(np.int8).reshape(M, I)
    ubase = qbase + off(M * I) + 2 * off(M * 4)
    u_dev = ws_np[ubase:ubase + M * I * 4].view(np.float32).reshape(M, I)
    np.testing.assert_allclose(oracle.relu2_glu(g_dev, u_dev), m, rtol=1e-5, atol=0)
    assert_codes_chain(qm_dev, qm, "decode codes")
    got = Y.cpu().numpy()
    if code_mismatch_stats(qm_dev, qm)[0] == 0:
        np.testing.assert_allclose(got, want, rtol=1e-5, atol=1e-6 * np.abs(want).max())
    assert _rel_l2(got, want) <= 1e-3
