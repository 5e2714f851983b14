"""Parity at the benchmark's full workload sizes, in the launch configuration
bench.py times (same entry points, same shapes, same seeds): the device runs
every token, the oracle recomputes a sample of tokens (each token's output
depends on that token only) and, where it is cheap, all of them.

Workloads (synthetic.WORKLOADS): the 256/512 tiny model linear; the
512 -> 2048 -> 512 H-BitLinear FFN at 1024 tokens; decode at the 2B model's
projection shapes for 1, 4 and 16 tokens; prefill at 4096 tokens for
(K, N) = (2560, 6912) and (6912, 2560) with the RMSNorm prelude; the 2B FFN
block at 2048 tokens.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
import ternary_weight_token_b200 as bn
from tests.gpu_util import (assert_bf16_matches, assert_codes_chain, assert_f32_close, bf16_dev,
                            code_mismatch_stats, dev)

pytestmark = pytest.mark.gpu


def _pack(W):
    P, g, ws = bn.alloc_packed(*W.shape)
    bn.bitnet_pack_weights(dev(W), P, g, ws)
    return P, g


def _rows(M, count, seed):
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(M, size=min(count, M), replace=False).tolist()) | {0, M - 1}
    return np.array(sorted(pick))


def test_tiny_model_linear_full():
    d = synthetic.WORKLOADS["tiny"].dims
    M, K, N = d["M"], d["K"], d["N"]
    inp = synthetic.linear_inputs(M, K, N, seed=0)
    P, g = _pack(inp["W"])
    q, s, rs = bn.alloc_quant(M, K)
    bn.bitnet_quant_act(dev(inp["X"]), q, s, rs)
    Y = torch.empty((M, N), device="cuda")
    bn.bitnet_linear(q, s, rs, P, g, K, Y)
    torch.cuda.synchronize()
    go, T, Po = oracle.quantize_weights(inp["W"])
    np.testing.assert_array_equal(P.cpu().numpy(), Po)
    assert_f32_close(Y.cpu().numpy(), oracle.bitlinear(inp["X"], T, go), what="tiny")


@pytest.mark.parametrize("K,N", [(2560, 6912), (6912, 2560)])
def test_prefill_full_size_sampled(K, N):
    M = synthetic.WORKLOADS["prefill"].dims["M"]
    seed = {(2560, 6912): 0, (6912, 2560): 1}[(K, N)]
    inp = synthetic.linear_inputs(M, K, N, seed=seed)       # the bench's inputs
    P, g = _pack(inp["W"])
    q, s, rs = bn.alloc_quant(M, K)
    bn.bitnet_quant_act(dev(inp["X"]), q, s, rs, prelude=bn.BITNET_PRELUDE_RMSNORM, eps=1e-5)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    bn.bitnet_linear(q, s, rs, P, g, K, Y)
    torch.cuda.synchronize()
    rows = _rows(M, 40, seed=K)
    go, T, Po = oracle.quantize_weights(inp["W"])
    assert g.item() == go
    np.testing.assert_array_equal(P.cpu().numpy(), Po)
    qo, so, rso = oracle.quant_act(inp["X"][rows], oracle.PRELUDE_RMSNORM, eps=1e-5)
    qd = q.cpu().numpy()[rows]
    assert_codes_chain(qd, qo, "prefill codes")
    # the contraction and epilogue on the device's own codes, bit for bit / RNE
    want = oracle.dequant(oracle.contract(qd, T), s.cpu().numpy()[rows], go)
    assert_bf16_matches(Y.float().cpu().numpy()[rows], want, what="prefill out")
    if code_mismatch_stats(qd, qo)[0] == 0:
        assert_bf16_matches(Y.float().cpu().numpy()[rows], oracle.dequant(oracle.contract(qo, T), so, go),
                            what="prefill chain")


@pytest.mark.parametrize("K,N", [(2560, 6912), (6912, 2560)])
def test_prefill_full_size_int32_every_row(K, N):
    """The persistent GEMM at the bench's size (4096 tokens, 1728 / 640 tiles
    on 148 CTAs, so every CTA runs several tiles and reuses each accumulator
    buffer): the int32 contraction of every token against the oracle's
    integer matmul, bit for bit, on the device's own codes; the codes
    themselves against the oracle's RMSNorm quantiser (chain tolerance); the
    bf16 outputs of every row against the oracle's dequantisation."""
    M = synthetic.WORKLOADS["prefill"].dims["M"]
    seed = {(2560, 6912): 0, (6912, 2560): 1}[(K, N)]
    inp = synthetic.linear_inputs(M, K, N, seed=seed)
    P, g = _pack(inp["W"])
    q, s, rs = bn.alloc_quant(M, K)
    bn.bitnet_quant_act(dev(inp["X"]), q, s, rs, prelude=bn.BITNET_PRELUDE_RMSNORM, eps=1e-5)
    Yi = torch.empty((M, N), dtype=torch.int32, device="cuda")
    bn.bitnet_linear(q, s, rs, P, g, K, Yi, epilogue=bn.BITNET_I32)
    Yb = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    bn.bitnet_linear(q, s, rs, P, g, K, Yb)
    torch.cuda.synchronize()
    go, T, _ = oracle.quantize_weights(inp["W"])
    qd = q.cpu().numpy()
    np.testing.assert_array_equal(rs.cpu().numpy(), qd.astype(np.int64).sum(axis=1))
    qo, so, _ = oracle.quant_act(inp["X"], oracle.PRELUDE_RMSNORM, eps=1e-5)
    assert_codes_chain(qd, qo, "prefill codes, every row")
    acc = oracle.contract(qd, T)
    np.testing.assert_array_equal(Yi.cpu().numpy(), acc)
    assert_bf16_matches(Yb.float().cpu().numpy(), oracle.dequant(acc, s.cpu().numpy(), go),
                        what="prefill bf16, every row")


@pytest.mark.parametrize("K,N", [(2560, 2560), (2560, 6912), (6912, 2560)])
def test_decode_full_rows(K, N):
    inp = synthetic.linear_inputs(16, K, N, seed=K + N)
    P, g = _pack(inp["W"])
    go, T, _ = oracle.quantize_weights(inp["W"])
    for M in (1, 4, 16):
        X = inp["X"][:M]
        q, s, rs = bn.alloc_quant(M, K)
        bn.bitnet_quant_act(dev(X), q, s, rs)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        bn.bitnet_linear(q, s, rs, P, g, K, Y, epilogue=bn.BITNET_BF16 | bn.BITNET_LAUNCH_PDL)
        torch.cuda.synchronize()
        assert_bf16_matches(Y.float().cpu().numpy(), oracle.bitlinear(X, T, go), what=f"decode M={M}")


def test_hffn_full():
    d = synthetic.WORKLOADS["hffn"].dims
    M, D, F = d["M"], d["D"], d["F"]
    inp = synthetic.hffn_inputs(M, D, F, seed=0)
    (P1, g1), (P2, g2) = _pack(inp["W1"]), _pack(inp["W2"])
    Y = torch.empty((M, D), device="cuda")
    ws = bn.alloc_ffn_workspace(M, D, F, bn.BITNET_FFN_HADAMARD_SILU)
    bn.bitnet_ffn(dev(inp["X"]), P1, g1, None, None, P2, g2, Y, ws,
                  variant=bn.BITNET_FFN_HADAMARD_SILU)
    torch.cuda.synchronize()
    go1, T1, _ = oracle.quantize_weights(inp["W1"])
    go2, T2, _ = oracle.quantize_weights(inp["W2"])
    want = oracle.hffn(inp["X"], T1, go1, T2, go2)
    got = Y.cpu().numpy()
    rel = np.linalg.norm(got.astype(np.float64) - want) / np.linalg.norm(want)
    assert rel <= 1e-3, rel


def test_ffn_block_full_size_sampled():
    d = synthetic.WORKLOADS["ffn"].dims
    M, H, I = d["M"], d["H"], d["I"]
    inp = synthetic.ffn_inputs(M, H, I, seed=0)
    packs = [_pack(inp[k]) for k in ("Wg", "Wu", "Wd")]
    Y = torch.empty((M, H), dtype=torch.bfloat16, device="cuda")
    ws = bn.alloc_ffn_workspace(M, H, I)
    bn.bitnet_ffn(bf16_dev(inp["x_bf16"]), packs[0][0], packs[0][1], packs[1][0], packs[1][1],
                  packs[2][0], packs[2][1], Y, ws, eps=1e-5)
    torch.cuda.synchronize()
    # every row: the sub-norm codes (the GLU GEMM's m through the sub-norm
    # quantiser) and the outputs
    T = {k: oracle.quantize_weights(inp[k]) for k in ("Wg", "Wu", "Wd")}
    out, m, qm, sm = oracle.ffn_relu2(inp["x"], T["Wg"][1], T["Wg"][0], T["Wu"][1],
                                      T["Wu"][0], T["Wd"][1], T["Wd"][0], eps=1e-5, keep=True)
    ws_np = ws.cpu().numpy()
    a256 = lambda n: (n + 255) // 256 * 256
    off = a256(M * H) + 2 * a256(M * 4) + a256(M * I * 4)
    qm_dev = ws_np[off:off + M * I].view(np.int8).reshape(M, I)
    assert_codes_chain(qm_dev, qm, "ffn sub-norm codes, every row")
    got = Y.float().cpu().numpy()
    if code_mismatch_stats(qm_dev, qm)[0] == 0:
        assert_bf16_matches(got, out, what="ffn out")
    want = oracle.round_bf16(out).astype(np.float64)
    assert np.linalg.norm(got - want) / np.linalg.norm(want) <= 1e-3
