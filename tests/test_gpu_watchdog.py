"""Failure detection on the GPU without a fault: a bounded wait that nothing completes must
expire, report through the watchdog word, and leave the context usable."""
import time

import numpy as np
import pytest
import torch

import synth
from util import assert_bf16_within_1ulp, bf16_tensor_from_bits, bits_from_bf16_tensor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bn():
    import ternary_w2a8_linear_token_b200 as m
    assert torch.cuda.is_available()
    return m


def test_bounded_wait_expires_and_is_reported(bn, oracle):
    assert bn.bitnet_check_device_errors() == 0  # clean before
    limit_ns = 20_000_000  # 20 ms
    t0 = time.perf_counter()
    bn.bitnet_selftest_wait_timeout(limit_ns)
    flags = bn.bitnet_check_device_errors()  # synchronises, reads and clears the word
    elapsed = time.perf_counter() - t0
    assert flags == bn.WATCHDOG_SELFTEST
    assert elapsed >= limit_ns * 1e-9  # the wait really waited for its limit
    assert elapsed < 5.0  # and then gave up
    assert bn.bitnet_check_device_errors() == 0  # cleared by the read

    # The context is still usable: a tensor-core forward afterwards matches the oracle.
    g = synth.rng(0, 97, 0, 0, synth.KIND_T)
    M, N, K = 64, 256, 1024
    t = synth.ternary(N, K, g, 0.4)
    s_w = synth.uniform_scale(1, g)
    x = synth.normal_x(M, K, synth.rng(0, 97, 0, 0, synth.KIND_X))
    packed = bn.bitnet_pack_ternary(torch.from_numpy(t).cuda())
    y = bn.bitnet_linear(bf16_tensor_from_bits(x), packed, torch.from_numpy(s_w).cuda(), False,
                         path=bn.PATH_TC)
    ref = oracle.bitlinear(x, oracle.pack(t), s_w, False, K)
    assert_bf16_within_1ulp(bits_from_bf16_tensor(y), ref["y"], oracle, "after self-test")
    assert bn.bitnet_check_device_errors() == 0

