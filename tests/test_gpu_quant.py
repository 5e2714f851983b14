"""GPU parity of the activation quantiser (with its preludes) and of the
weight packer against the oracle, through the C ABI.

Codes, scales and code sums are compared bit for bit.  The RMSNorm prelude
accumulates the mean square in fp64 on both sides but in a different order;
the fp32 value it rounds to can then differ only next to an fp32 midpoint, so
those cases fall under the chain tolerance (<= 0.1 % of codes, +-1 each).
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
import ternary_weight_token_b200 as bn
from tests.gpu_util import (assert_codes_chain, bf16_dev, code_mismatch_stats, dev, gpu_pack,
                            gpu_quant)

pytestmark = pytest.mark.gpu


def _acts(M, K, seed, outliers=False):
    X = synthetic.activations(np.random.default_rng(seed), M, K)
    if outliers:
        X = synthetic.outliers(np.random.default_rng(seed + 1), X)
    return X


@pytest.mark.parametrize("M,K", [(1, 16), (8, 256), (3, 80), (129, 2560), (37, 6912), (2, 16384)])
def test_quant_none_bit_exact(M, K):
    X = _acts(M, K, seed=M * 7 + K)
    X[0, :] = 0.0                       # an all-zero token
    if M > 2:
        X[2, :] = 0.0
        X[2, K // 3] = -5.5              # a one-hot token
    q, s, rs = gpu_quant(X)
    qo, so, rso = oracle.quant_act(X)
    np.testing.assert_array_equal(q, qo)
    np.testing.assert_array_equal(s, so)
    np.testing.assert_array_equal(rs, rso)


@pytest.mark.parametrize("K", [16, 64, 128, 256, 512, 1024, 2048, 4096, 8192])
def test_quant_fwht_bit_exact(K):
    """Both FWHT kernels: one warp per row in registers (128..2048 inputs) and
    the row staged in shared memory (other widths)."""
    X = _acts(33, K, seed=K, outliers=True)
    X[5] = 0.0                                  # an all-zero token
    q, s, rs = gpu_quant(X, bn.BITNET_PRELUDE_FWHT)
    qo, so, rso = oracle.quant_act(X, oracle.PRELUDE_FWHT)
    np.testing.assert_array_equal(q, qo)
    np.testing.assert_array_equal(s, so)
    np.testing.assert_array_equal(rs, rso)


@pytest.mark.parametrize("K", [128, 256, 2048])
def test_quant_fwht_bf16_bit_exact(K):
    X = _acts(21, K, seed=K + 1, outliers=True)
    bits = synthetic.to_bf16_bits(X)
    xw = oracle.bf16_bits_to_f32(bits)
    q, s, rs = gpu_quant(xw, bn.BITNET_PRELUDE_FWHT, x_dev=bf16_dev(bits))
    qo, so, rso = oracle.quant_act(xw, oracle.PRELUDE_FWHT)
    np.testing.assert_array_equal(q, qo)
    np.testing.assert_array_equal(s, so)
    np.testing.assert_array_equal(rs, rso)


@pytest.mark.parametrize("M,K,with_gain", [(64, 2560, False), (17, 6912, True), (5, 48, True)])
def test_quant_rmsnorm(M, K, with_gain):
    X = _acts(M, K, seed=K + M)
    gain = (np.random.default_rng(3).uniform(0.5, 1.5, K).astype(np.float32)
            if with_gain else None)
    q, s, rs = gpu_quant(X, bn.BITNET_PRELUDE_RMSNORM, gain=gain, eps=1e-5)
    qo, so, rso = oracle.quant_act(X, oracle.PRELUDE_RMSNORM, gain=gain, eps=1e-5)
    assert_codes_chain(q, qo, "rmsnorm codes")
    n, _ = code_mismatch_stats(q, qo)
    if n == 0:
        np.testing.assert_array_equal(s, so)
        np.testing.assert_array_equal(rs, rso)
    else:
        np.testing.assert_allclose(s, so, rtol=1e-6)


@pytest.mark.parametrize("M,K,bf16,prelude", [(2001, 2560, False, 0), (2001, 2560, True, 1),
                                               (701, 6912, False, 1), (1500, 512, False, 0),
                                               (3000, 16384, True, 0)])
def test_quant_many_rows(M, K, bf16, prelude):
    """Prefill-sized row counts on every row-kernel width (64 x 10, 128 x 14 and
    256 x 16 threads x chunks), zero and one-hot rows among them."""
    X = _acts(M, K, seed=M + K)
    X[M // 2] = 0.0
    X[M - 1] = 0.0
    X[M - 1, K // 5] = 3.25
    if bf16:
        bits = synthetic.to_bf16_bits(X)
        X = oracle.bf16_bits_to_f32(bits)
    pre = (bn.BITNET_PRELUDE_RMSNORM, oracle.PRELUDE_RMSNORM) if prelude else (
        bn.BITNET_PRELUDE_NONE, oracle.PRELUDE_NONE)
    q, s, rs = gpu_quant(X, pre[0], eps=1e-5, x_dev=bf16_dev(bits) if bf16 else None)
    qo, so, rso = oracle.quant_act(X, pre[1], eps=1e-5)
    if prelude:
        assert_codes_chain(q, qo, "rmsnorm codes")
        if code_mismatch_stats(q, qo)[0] == 0:
            np.testing.assert_array_equal(s, so)
            np.testing.assert_array_equal(rs, rso)
    else:
        np.testing.assert_array_equal(q, qo)
        np.testing.assert_array_equal(s, so)
        np.testing.assert_array_equal(rs, rso)


def test_quant_bf16_input():
    X = _acts(40, 2560, seed=5)
    bits = synthetic.to_bf16_bits(X)
    xw = oracle.bf16_bits_to_f32(bits)
    q, s, rs = gpu_quant(xw, x_dev=bf16_dev(bits))
    qo, so, rso = oracle.quant_act(xw)
    np.testing.assert_array_equal(q, qo)
    np.testing.assert_array_equal(s, so)
    np.testing.assert_array_equal(rs, rso)
    q, s, rs = gpu_quant(xw, bn.BITNET_PRELUDE_RMSNORM, x_dev=bf16_dev(bits))
    qo, so, rso = oracle.quant_act(xw, oracle.PRELUDE_RMSNORM)
    assert_codes_chain(q, qo, "bf16 rmsnorm codes")


def test_quant_scale_invariance_on_device():
    """Codes are identical under x -> 2^k x (no prelude, and RMSNorm with eps 0)."""
    X = _acts(16, 1024, seed=9)
    q0, s0, _ = gpu_quant(X)
    q1, s1, _ = gpu_quant(X * np.float32(8.0))
    np.testing.assert_array_equal(q0, q1)
    np.testing.assert_array_equal(s0, s1 * np.float32(8.0))
    r0, _, _ = gpu_quant(X, bn.BITNET_PRELUDE_RMSNORM, eps=0.0)
    r1, _, _ = gpu_quant(X * np.float32(0.25), bn.BITNET_PRELUDE_RMSNORM, eps=0.0)
    np.testing.assert_array_equal(r0, r1)


@pytest.mark.parametrize("N,K", [(1, 16), (7, 80), (512, 256), (300, 2560), (6912, 2560),
                                 (2560, 6912)])
def test_pack_bit_exact(N, K):
    W = synthetic.weight(np.random.default_rng(N + K), N, K)
    packed, gamma = gpu_pack(W)
    go = oracle.absmean(W)
    assert gamma == go, (gamma, go)
    np.testing.assert_array_equal(packed, oracle.pack(oracle.ternarize(W, go)))


def test_pack_bf16_weights_and_edge_values():
    rng = np.random.default_rng(4)
    W = synthetic.weight(rng, 64, 128)
    bits = synthetic.to_bf16_bits(W)
    Ww = oracle.bf16_bits_to_f32(bits)
    N, K = Ww.shape
    packed, gamma, ws = bn.alloc_packed(N, K)
    bn.bitnet_pack_weights(bf16_dev(bits), packed, gamma, ws)
    torch.cuda.synchronize()
    go = oracle.absmean(Ww)
    assert gamma.item() == go
    np.testing.assert_array_equal(packed.cpu().numpy(), oracle.pack(oracle.ternarize(Ww, go)))
    # ties at exactly 0.5 and 1.5 gamma, and an all-zero matrix
    T = np.array([[0.5, -1.5, 2.5, -0.5, 1.0, 0.0, -1.0, 1.0] * 2], dtype=np.float32)
    packed, gamma = gpu_pack(T)
    assert gamma == 1.0
    np.testing.assert_array_equal(packed, oracle.pack(oracle.ternarize(T, np.float32(1.0))))
    Z = np.zeros((3, 32), np.float32)
    packed, gamma = gpu_pack(Z)
    assert gamma == 0.0
    assert np.all(packed == 0x55)


@pytest.mark.parametrize("N,K", [(1, 16), (7, 80), (300, 2560), (2560, 6912)])
def test_tw2_export_and_import(N, K):
    """The device layout converts to the canonical TW2 bytes of the oracle and
    back, bit for bit (padding words of ragged rows come back as code 1)."""
    W = synthetic.weight(np.random.default_rng(N * 3 + K), N, K)
    packed, gamma = gpu_pack(W)
    t = oracle.ternarize(W, oracle.absmean(W))
    want = oracle.pack_tw2(t)
    tw2 = torch.empty((N, K // 4), dtype=torch.uint8, device="cuda")
    bn.bitnet_export_tw2(dev(packed), K, tw2)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(tw2.cpu().numpy(), want)
    back = torch.full((N, bn.bitnet_packed_row_bytes(K)), 0xEE, dtype=torch.uint8, device="cuda")
    bn.bitnet_import_tw2(dev(want), K, back)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(back.cpu().numpy(), oracle.pack(t))


def test_pack_threshold_boundary():
    """Codes of weights within a few hundred fp32 ulps of 0.5 * gamma, on both
    sides of the rounding boundary of fl(w / gamma): a ballast of +-1 entries
    fixes gamma, 512 consecutive fp32 values around the expected 0.5 * gamma
    straddle it.  Bit-exact against the oracle's IEEE division and rint."""
    n_ball, n_cand = 65536, 512
    c = 0.5 * n_ball / (n_ball + n_cand - n_cand / 2)      # gamma / 2 with the candidates in
    cand = [np.float32(c)]
    for _ in range(n_cand // 2):
        cand.append(np.nextafter(cand[-1], np.float32(1), dtype=np.float32))
        cand.insert(0, np.nextafter(cand[0], np.float32(0), dtype=np.float32))
    cand = np.array(cand[:n_cand], dtype=np.float32)
    sign = np.where(np.arange(n_cand) % 2 == 0, 1, -1).astype(np.float32)
    ball = np.where(np.arange(n_ball) % 2 == 0, 1, -1).astype(np.float32)
    W = np.concatenate([ball, cand * sign]).reshape(-1, 256)
    g = oracle.absmean(W)
    t = oracle.ternarize(W, g)
    tc = t.ravel()[n_ball:]
    assert (tc == 0).any() and (tc != 0).any()            # the boundary lies inside the run
    packed, gamma = gpu_pack(W)
    assert gamma == g
    np.testing.assert_array_equal(packed, oracle.pack(t))


def _bf16_run(center_bits, n):
    """n consecutive positive bf16 bit patterns centred on center_bits."""
    return (np.arange(n, dtype=np.int64) - n // 2 + int(center_bits)).astype(np.uint16)


@pytest.mark.parametrize("seed", range(6))
def test_pack_bf16_threshold_sweep(seed):
    """bf16 weights: a ballast of +-b (b a random bf16 in [0.5, 2)) fixes
    gamma near b, and 64 consecutive bf16 magnitudes around b / 2 with
    alternating signs straddle the rounding boundary of fl(w / gamma).  The
    packer decides t != 0 from the weight's bits; the oracle divides."""
    rng = np.random.default_rng(100 + seed)
    b_bits = np.uint16(0x3F00 + rng.integers(0, 0x100))          # [0.5, 2)
    b = oracle.bf16_bits_to_f32(np.array([b_bits]))[0]
    half_bits = synthetic.to_bf16_bits(np.array([b * np.float32(0.5)]))[0]
    cand = _bf16_run(half_bits, 64)
    cand = np.where(np.arange(64) % 2 == 0, cand, cand | np.uint16(0x8000)).astype(np.uint16)
    ball = np.where(np.arange(4096) % 2 == 0, b_bits, b_bits | np.uint16(0x8000)).astype(np.uint16)
    bits = np.concatenate([ball, cand]).reshape(-1, 64)
    Ww = oracle.bf16_bits_to_f32(bits)
    go = oracle.absmean(Ww)
    t = oracle.ternarize(Ww, go)
    tc = t.ravel()[4096:]
    assert (tc == 0).any() and (tc != 0).any()            # the boundary lies inside the run
    N, K = bits.shape
    packed, gamma, ws = bn.alloc_packed(N, K)
    bn.bitnet_pack_weights(bf16_dev(bits), packed, gamma, ws)
    torch.cuda.synchronize()
    assert gamma.item() == go
    np.testing.assert_array_equal(packed.cpu().numpy(), oracle.pack(t))


@pytest.mark.parametrize("wdtype", ["f32", "bf16"])
def test_pack_special_magnitudes(wdtype):
    """Signed zeros, subnormals, the largest finite values and ties at
    gamma / 2 and 3 gamma / 2, in both weight types: codes and gamma bit for
    bit against the oracle (subnormal-only and huge-only matrices included, so
    the threshold itself is subnormal or near the top of the range)."""
    if wdtype == "f32":
        big, sub = np.float32(3.0e38), np.float32(1.0e-40)
        mats = [
            np.array([[0.0, -0.0, sub, -sub, 2 * sub, 1e-45, -1e-45, 0.0] * 4], np.float32),
            np.array([[big, -big, big / 3, 0.0, -big / 2, big, 1.0, -1.0] * 2], np.float32),
            np.array([[0.5, -1.5, 2.5, -0.5, 1.0, 0.0, -1.0, 1.0] * 4, [1e-30, -3.0] * 16], np.float32),
        ]
        for W in mats:
            packed, gamma = gpu_pack(np.ascontiguousarray(W))
            go = oracle.absmean(W)
            assert gamma == go, (W[0, :4], gamma, go)
            np.testing.assert_array_equal(packed, oracle.pack(oracle.ternarize(W, go)))
        return
    sets = [
        np.array([0x0000, 0x8000, 0x0001, 0x8001, 0x007F, 0x807F, 0x0080, 0x0002] * 4, np.uint16),
        np.array([0x7F7F, 0xFF7F, 0x7F00, 0x0000, 0xFEFF, 0x7F7F, 0x3F80, 0xBF80] * 2, np.uint16),
        synthetic.to_bf16_bits(np.array([0.5, -1.5, 2.5, -0.5, 1.0, 0.0, -1.0, 1.0] * 4, np.float32)),
        np.array([0x0001] * 31 + [0x0003], np.uint16),
    ]
    for bits in sets:
        bits = bits.reshape(1, -1)
        Ww = oracle.bf16_bits_to_f32(bits)
        go = oracle.absmean(Ww)
        N, K = bits.shape
        packed, gamma, ws = bn.alloc_packed(N, K)
        bn.bitnet_pack_weights(bf16_dev(bits), packed, gamma, ws)
        torch.cuda.synchronize()
        assert gamma.item() == go, (bits[0, :4], gamma.item(), go)
        np.testing.assert_array_equal(packed.cpu().numpy(), oracle.pack(oracle.ternarize(Ww, go)))


def test_pack_is_deterministic():
    W = synthetic.weight(np.random.default_rng(12), 2560, 2560)
    a = gpu_pack(W)
    b = gpu_pack(W)
    assert a[1] == b[1]
    np.testing.assert_array_equal(a[0], b[0])


@pytest.mark.parametrize("fill", [0x00, 0xFF, "random"])
def test_pack_one_launch_workspace_needs_no_initialisation(fill):
    """The one-launch pack exchanges its partial sums through flags in the
    workspace tagged with a fresh epoch per launch: whatever the workspace
    holds before (zeros, ones, random bytes, a previous call's flags), the
    result is the same, call after call."""
    W = synthetic.weight(np.random.default_rng(21), 2560, 6912)
    Wd = dev(W).to(torch.bfloat16)
    Ww = Wd.float().cpu().numpy()
    go = oracle.absmean(Ww)
    want = oracle.pack(oracle.ternarize(Ww, go))
    packed, gamma, ws = bn.alloc_packed(2560, 6912)
    if fill == "random":
        ws.copy_(torch.randint(0, 256, ws.shape, dtype=torch.uint8, device="cuda"))
    else:
        ws.fill_(fill)
    for _ in range(3):
        packed.fill_(0)
        bn.bitnet_pack_weights(Wd, packed, gamma, ws)
        torch.cuda.synchronize()
        assert gamma.item() == go
        np.testing.assert_array_equal(packed.cpu().numpy(), want)
    assert bn.bitnet_check_device_error() == bn.BITNET_OK


def test_quant_rmsnorm_zero_row_with_zero_eps():
    """mean square 0 and eps 0 give r = inf; the all-zero row must still come
    out as q = 0, s = 1 (the oracle's 0 * inf products never exceed 0)."""
    X = _acts(6, 2560, seed=77)
    X[2] = 0.0
    for gain in (None, np.full(2560, 1.5, np.float32)):
        q, s, rs = gpu_quant(X, bn.BITNET_PRELUDE_RMSNORM, gain=gain, eps=0.0)
        qo, so, rso = oracle.quant_act(X, oracle.PRELUDE_RMSNORM, gain=gain, eps=0.0)
        assert not q[2].any() and s[2] == 1.0 and rs[2] == 0
        assert_codes_chain(q, qo, "rmsnorm eps 0")
