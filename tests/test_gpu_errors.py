"""Failure handling on the device without faulting it: a bounded wait that
nobody satisfies gives up, records BITNET_ERR_TIMEOUT in the device error
word, and the context stays usable for the next real call."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
import ternary_weight_token_b200 as bn
from tests.gpu_util import gpu_quant

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    assert bn.bitnet_check_device_error() == bn.BITNET_OK
    bn.bitnet_debug_wait_timeout(1000)             # 1 ms limit on a barrier nobody arrives at
    assert bn.bitnet_check_device_error() == bn.BITNET_ERR_TIMEOUT
    assert "wait" in bn.bitnet_last_error()
    assert bn.bitnet_check_device_error() == bn.BITNET_OK      # the word was cleared
    X = synthetic.activations(np.random.default_rng(0), 8, 256)
    q, s, _ = gpu_quant(X)
    qo, so, _ = oracle.quant_act(X)
    np.testing.assert_array_equal(q, qo)


def test_invalid_call_has_no_device_side_effect():
    Y = torch.full((4, 8), 3.0, device="cuda")
    q = torch.zeros((4, 24), dtype=torch.int8, device="cuda")      # K = 24 is not a multiple of 16
    s = torch.ones(4, device="cuda")
    rs = torch.zeros(4, dtype=torch.int32, device="cuda")
    P = torch.zeros((8, 16), dtype=torch.uint8, device="cuda")
    g = torch.ones(1, device="cuda")
    with pytest.raises(bn.BitnetError) as e:
        bn.bitnet_linear(q, s, rs, P, g, 24, Y)
    assert e.value.code == bn.BITNET_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert torch.all(Y == 3.0)
    assert bn.bitnet_check_device_error() == bn.BITNET_OK
