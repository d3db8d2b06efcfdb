"""The no-allocation entry point, bitnet_linear_noalloc, against bitnet_linear.

Callers that cannot allocate device memory while they run (a latency-bound serving loop in
which cudaMalloc could synchronise the device, a plug-in whose host runtime owns all device
memory) use bitnet_linear_noalloc, whose tensor-core scratch is a fixed array inside the
library. It runs the same kernels as bitnet_linear on the same inputs, so the results must be
equal bit for bit, on every call in a row (each call reuses the scratch the previous one left).
This file is collected last so that a failure here never hides the other tests; it passes both
alone in a fresh process and after the rest of the suite.
"""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import ternary_w2a8_linear_token_b200 as bn
    return bn


def _case(bn, M, N, K, per_row, seed):
    g = synth.rng(0, 97, seed, M, synth.KIND_T)
    t = torch.from_numpy(synth.ternary(N, K, g, 0.4)).cuda()
    packed = bn.bitnet_pack_ternary(t)
    s_w = torch.from_numpy(synth.uniform_scale(N if per_row else 1, g)).cuda()
    x = torch.from_numpy(synth.normal_x(M, K, g).view(np.int16).copy()).cuda().view(torch.bfloat16)
    return x, packed, s_w


@pytest.mark.parametrize("M,N,K,per_row", [(300, 640, 2560, False), (2048, 256, 512, True),
                                           (17, 129, 6912, False), (4, 640, 2560, True),
                                           (8, 2560, 2560, False)])
def test_noalloc_matches_bitnet_linear_twice(bn, M, N, K, per_row):
    """Two calls in a row (different inputs, same scratch) against the allocating call:
    equal bit for bit."""
    for seed in (1, 2):
        x, packed, s_w = _case(bn, M, N, K, per_row, seed)
        ref = bn.bitnet_linear(x, packed, s_w, per_row)
        y = torch.empty_like(ref)
        got = bn.bitnet_linear_noalloc(x, packed, s_w, per_row, y=y)
        torch.cuda.synchronize()
        assert got.data_ptr() == y.data_ptr()
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), \
            f"M={M} N={N} K={K} call {seed}"
    assert bn.bitnet_check_device_errors() == 0


def test_noalloc_fp32_output(bn):
    for seed in (3, 4):
        x, packed, s_w = _case(bn, 64, 256, 1024, False, seed)
        ref = bn.bitnet_linear(x, packed, s_w, False, out_dtype=torch.float32)
        got = bn.bitnet_linear_noalloc(x, packed, s_w, False, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int32), ref.view(torch.int32)), f"call {seed}"


def test_noalloc_rejects_sizes_beyond_scratch(bn):
    M, K = 4096, 8192  # quantised activations alone are 32 MiB > 16 MiB
    assert bn.workspace_size(M, K) > bn.NOALLOC_SCRATCH_BYTES
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    packed = torch.zeros((64, K // 4), dtype=torch.uint8, device="cuda")
    s_w = torch.ones(1, dtype=torch.float32, device="cuda")
    with pytest.raises(bn.BitnetError) as e:
        bn.bitnet_linear_noalloc(x, packed, s_w, False)
    assert e.value.status == bn.ERR_WORKSPACE
    # the bound is the whole workspace of the call (split-K area included)
    M2, K2 = 1024, 15872
    assert bn.workspace_size(M2, K2) > bn.NOALLOC_SCRATCH_BYTES >= M2 * K2
    x2 = torch.zeros((M2, K2), dtype=torch.bfloat16, device="cuda")
    p2 = torch.zeros((64, K2 // 4), dtype=torch.uint8, device="cuda")
    with pytest.raises(bn.BitnetError) as e:
        bn.bitnet_linear_noalloc(x2, p2, s_w, False)
    assert e.value.status == bn.ERR_WORKSPACE
