"""GPU parity of the per-tensor activation scale (BITNET_ACT_PER_TENSOR) against the oracle.

One absmax scale for the whole (M, K) input ("BitNet 1-bit LLM推理优化" §2.2: I2_S keeps
BitNet b1.58's per-tensor int8 activations; §3.2 lists per-tensor scales). Bars as for the
per-token path: q and s_x bit-exact, bf16 y within one bf16 step of RNE(exact), fp32 y within
1e-6 relative. Covers every quantiser code path (register rows K <= 4096, four-warp rows up
to 14336, two-pass rows beyond), the GEMV (amax over its tokens in one launch) and the
tensor-core path (partial maxima kernel + quantiser + GEMM).
"""
import numpy as np
import pytest
import torch

import synth
from util import (assert_bf16_within_1ulp, assert_f32_rel, bf16_tensor_from_bits,
                  bits_from_bf16_tensor)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import ternary_w2a8_linear_token_b200 as bn
    return bn


@pytest.fixture(autouse=True)
def _watchdog_clean(request):
    yield
    if torch.cuda.is_available() and "bn" in request.fixturenames:
        bn = request.getfixturevalue("bn")
        assert bn.bitnet_check_device_errors() == 0


def _x(M, K, key):
    g = synth.rng(0, 96, M, K + key, synth.KIND_X)
    x = synth.normal_x(M, K, g)
    if M > 2:
        x[M // 2] = synth.to_bf16_bits(synth.bf16_bits_to_f32(x[M // 2]) * np.float32(8.0))
    return x


@pytest.mark.parametrize("M,K", [(1, 64), (7, 2560), (130, 4096), (33, 6912), (5, 14336),
                                 (3, 16384), (2048, 2560)])
def test_quant_act_per_tensor_bit_exact(bn, oracle, M, K):
    x = _x(M, K, 0)
    q, s_x = bn.bitnet_quant_act_ex(bf16_tensor_from_bits(x), bn.ACT_PER_TENSOR)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.quant_act_per_tensor(x)
    assert np.array_equal(s_x.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


CASES = [  # (M, N, K, per_row)
    (1, 640, 2560, False), (4, 300, 512, True), (8, 257, 1024, False), (37, 300, 2560, True),
    (300, 256, 512, False), (130, 640, 6912, True), (16, 2560, 4096, False),
]


@pytest.mark.parametrize("M,N,K,per_row", CASES)
def test_linear_per_tensor_act_matches_oracle(bn, oracle, M, N, K, per_row):
    g = synth.rng(0, 97, M * 7 + N, K, synth.KIND_T)
    t = synth.ternary(N, K, g, 0.4)
    s_w = synth.uniform_scale(N if per_row else 1, g)
    x = _x(M, K, 1)
    packed = torch.from_numpy(oracle.pack(t)).cuda()
    ref = oracle.bitlinear(x, packed.cpu().numpy(), s_w, per_row, K, act_per_tensor=True)
    xd = bf16_tensor_from_bits(x)
    paths = [bn.PATH_AUTO, bn.PATH_TC] + ([bn.PATH_GEMV] if M <= bn.GEMV_MAX_M else [])
    for path in paths:
        for dtype in (torch.bfloat16, torch.float32):
            (y,) = bn.bitnet_linear_batch_act(xd, [(packed, torch.from_numpy(s_w).cuda(),
                                                    per_row)], bn.ACT_PER_TENSOR,
                                              out_dtype=dtype, path=path)
            where = f"M={M} N={N} K={K} path={path} {dtype}"
            if dtype == torch.bfloat16:
                assert_bf16_within_1ulp(bits_from_bf16_tensor(y), ref["y"], oracle, where)
            else:
                assert_f32_rel(y.cpu().numpy(), ref["y"], where=where)


def test_per_token_mode_of_the_act_call_equals_bitnet_linear(bn, oracle):
    """ACT_PER_TOKEN through the new call is the plain call, bit for bit."""
    M, N, K = 37, 300, 2560
    t = synth.ternary(N, K, synth.rng(0, 98, 0, 0, synth.KIND_T), 0.4)
    packed = torch.from_numpy(oracle.pack(t)).cuda()
    s_w = torch.tensor([1.25], device="cuda")
    xd = bf16_tensor_from_bits(_x(M, K, 2))
    (y1,) = bn.bitnet_linear_batch_act(xd, [(packed, s_w, False)], bn.ACT_PER_TOKEN)
    y2 = bn.bitnet_linear(xd, packed, s_w, False)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("shape_idx", [0, 3])
def test_prefill_per_tensor_act_full_size_sampled(bn, oracle, shape_idx):
    """Prefill M = 2048 with the outlier-channel activations, per-tensor scale, the launch
    configuration of the benchmark's GEMM; sampled tokens x outputs checked one by one."""
    c = synth.prefill_case(shape_idx, 2048)
    packed = bn.bitnet_pack_ternary(torch.from_numpy(c["t"]).cuda())
    xd = bf16_tensor_from_bits(c["x"])
    (y,) = bn.bitnet_linear_batch_act(xd, [(packed, torch.from_numpy(c["s_w"]).cuda(), False)],
                                      bn.ACT_PER_TENSOR)
    torch.cuda.synchronize()
    rs = np.random.default_rng(shape_idx)
    m_idx = np.unique(np.concatenate([[0, 2047], rs.integers(0, 2048, 30)]))
    n_idx = np.unique(np.concatenate([[0, c["N"] - 1], rs.integers(0, c["N"], 40)]))
    ref = oracle.bitlinear_sampled_per_tensor_act(c["x"], packed.cpu().numpy(), c["s_w"], False,
                                                  c["K"], m_idx, n_idx)
    got = bits_from_bf16_tensor(y)[np.ix_(m_idx, n_idx)]
    assert_bf16_within_1ulp(got, ref["y"], oracle, f"prefill shape {shape_idx}")
