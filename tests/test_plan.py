"""Host logic of the launch plan (no GPU): bitnet_plan_linear reports the
kernel and launch shape bitnet_linear picks, computed by the same functions
the launches call.

Two kinds of checks:
- the decisions for the 2B-model shapes and the bench's workloads, which the
  library's rules were tuned to by measurement (pinned, so that a change to a
  rule shows up here before it reaches a GPU);
- invariants every plan must keep over a sweep of shapes, flags and SM
  counts: each lane's chunk budget, the token tiles the kernels instantiate,
  shared memory within the per-CTA limit, grids that cover every row, the
  cluster split's slice bound.
"""
import itertools

import pytest

import ternary_weight_token_b200 as bn

pytestmark = pytest.mark.filterwarnings("ignore")

BF16 = bn.BITNET_BF16
PDL = bn.BITNET_LAUNCH_PDL
INPUTS = bn.BITNET_LAUNCH_PDL_INPUTS
SILU = bn.BITNET_EPI_SILU

STREAM, FLAT, GEMV_TC, GEMV, GEMM_TC = (bn.BITNET_PLAN_STREAM, bn.BITNET_PLAN_FLAT,
                                        bn.BITNET_PLAN_GEMV_TC, bn.BITNET_PLAN_GEMV,
                                        bn.BITNET_PLAN_GEMM_TC)
SMEM_PER_CTA = 227 * 1024


def plan(M, N, K, flags=0, sms=148):
    return bn.bitnet_plan_linear(M, N, K, BF16 | flags, sms)


def ceil_div(a, b):
    return -(-a // b)


# (M, N, K, flags) -> (kernel, tokens, grid, a, b) on 148 SMs
PINNED = {
    # one token, independent projections: the flat kernel, about one CTA per
    # two SMs; bulk-copied rows from 4 MB of weights up
    (1, 2560, 2560, INPUTS): (FLAT, 1, 64, 5, 0),
    (1, 6912, 2560, INPUTS): (FLAT, 1, 144, 6, 1),
    (1, 2560, 6912, INPUTS): (FLAT, 1, 160, 2, 1),
    # dependent calls of 1-4 tokens on rows of at most 4096 inputs: row groups
    (1, 2560, 2560, PDL): (STREAM, 1, 160, 16, 8),
    (1, 6912, 2560, PDL): (STREAM, 1, 216, 8, 8),
    (4, 2560, 2560, PDL): (STREAM, 4, 160, 8, 4),
    # 3-16 tokens otherwise: the cluster tensor-core GEMV
    (4, 2560, 2560, INPUTS): (GEMV_TC, 16, 80, 4, 20),
    (4, 6912, 2560, INPUTS): (GEMV_TC, 16, 162, 3, 54),
    (16, 2560, 2560, 0): (GEMV_TC, 16, 80, 4, 20),
    (16, 6912, 2560, 0): (GEMV_TC, 16, 216, 4, 54),
    (16, 2560, 6912, 0): (GEMV_TC, 16, 160, 8, 20),
    (8, 2560, 2560, PDL): (GEMV_TC, 16, 160, 8, 20),
    (4, 2560, 6912, PDL): (GEMV_TC, 16, 160, 8, 20),
    # the tiny model's linear: the flat kernel's 8-token tile
    (8, 512, 256, PDL): (FLAT, 8, 64, 1, 0),
    # prefill and FFN GEMMs: 128-, 96- and 64-token tiles
    (4096, 6912, 2560, 0): (GEMM_TC, 128, 148, 1728, 0),
    (4096, 2560, 6912, 0): (GEMM_TC, 128, 148, 640, 0),
    (2048, 2560, 6912, 0): (GEMM_TC, 96, 148, 440, 0),
    (1024, 2048, 512, SILU): (GEMM_TC, 128, 128, 128, 0),
    (1024, 512, 2048, 0): (GEMM_TC, 64, 64, 64, 0),
    # decode rows longer than the cluster split takes: the plain GEMV
    (16, 2560, 16384, 0): (GEMV, 16, 160, 0, 0),
}


@pytest.mark.parametrize("key", list(PINNED), ids=[f"{m}x{n}x{k}-{f:#x}" for m, n, k, f in PINNED])
def test_plan_for_the_model_shapes(key):
    M, N, K, flags = key
    got = plan(M, N, K, flags)
    assert (got["kernel"], got["tokens"], got["grid"], got["a"], got["b"]) == PINNED[key]


def _check_invariants(M, N, K, flags, sms):
    p = plan(M, N, K, flags, sms)
    k, tok, grid, a, b = p["kernel"], p["tokens"], p["grid"], p["a"], p["b"]
    ldw = bn.bitnet_packed_row_bytes(K)
    C = ldw // 16
    where = f"M={M} N={N} K={K} flags={flags:#x} sms={sms}: {p}"
    if M > 16:
        assert k == GEMM_TC, where
        assert tok in (128, 96, 64), where
        if flags & SILU:
            assert tok == 128, where
        assert a == ceil_div(M, tok) * ceil_div(N, 128), where
        assert grid == min(a, sms), where
        return
    assert k != GEMM_TC, where
    if k == STREAM:
        assert M <= 4 and K % 64 == 0 and tok >= M and tok in (1, 2, 4), where
        L, warps = a, b
        assert L & (L - 1) == 0 and 1 <= L <= 32, where
        assert 8 * L >= C, where                       # at most 8 chunks a lane
        assert 1 <= warps <= 8, where
        rows = warps * (32 // L)
        assert grid * rows >= N > (grid - 1) * rows, where
        assert tok * K <= SMEM_PER_CTA, where
    elif k == FLAT:
        assert M <= 8 and K % 64 == 0 and tok >= M and tok in (1, 2, 8), where
        R, bulk = a, b
        assert 1 <= R <= 8 and R * C <= 256, where      # at most 8 chunks a lane
        if tok == 8:
            assert R <= 4, where                        # lane r * 8 + m holds (row, token)
        assert bulk in (0, 1), where
        if bulk:
            assert flags & INPUTS, where
        assert grid * 8 * R >= N > (grid - 1) * 8 * R, where
        assert (8 * R * ldw if bulk else 0) + tok * K <= SMEM_PER_CTA, where
    elif k == GEMV_TC:
        assert M >= 3, where                            # 1-2 tokens always stream
        S, tiles = a, b
        units = K // 64
        assert K % 64 == 0 and 1 <= S <= min(8, units), where
        assert ceil_div(units, S) <= 14, where          # a slice fits the 7-chunk stage
        assert tiles == ceil_div(N, 128) and grid == tiles * S, where
    else:
        assert k == GEMV, where
        units = K // 64
        assert K % 64 != 0 or ceil_div(units, 8) > 14, where
        assert tok >= M and grid >= 1, where


SWEEP_M = (1, 2, 3, 4, 5, 8, 9, 16, 17, 100, 1024, 4096)
SWEEP_N = (1, 77, 128, 512, 640, 2560, 6912, 13824)
SWEEP_K = (16, 80, 256, 2560, 6912, 8192, 16384)
SWEEP_FLAGS = (0, PDL, INPUTS | PDL, INPUTS, SILU)


@pytest.mark.parametrize("sms", [148, 132, 80])
def test_plan_invariants_over_a_sweep(sms):
    for M, N, K, flags in itertools.product(SWEEP_M, SWEEP_N, SWEEP_K, SWEEP_FLAGS):
        _check_invariants(M, N, K, flags, sms)


@pytest.mark.parametrize("args", [(0, 16, 64, 148), (1, 0, 64, 148), (1, 16, 10, 148),
                                  (1, 16, 32768, 148), (1, 16, 64, 0)])
def test_plan_rejects_bad_arguments(args):
    M, N, K, sms = args
    with pytest.raises(bn.BitnetError) as e:
        bn.bitnet_plan_linear(M, N, K, BF16, sms)
    assert e.value.code == bn.BITNET_ERR_INVALID_ARG
