"""GPU parity of the tensor-parallel steps (bitnet_act_amax, bitnet_quant_act_amax,
bitnet_dequant, with bitnet_linear_i32 on weight slices).

One GPU cannot host ranks that wait on each other, so the ranks of a split run one after
another in this process, and the collectives are stood in for by their definitions (maximum of
the amax vectors, sum of the int32 partial accumulators, concatenation of the outputs). The
steps must then reproduce bitnet_linear on the whole row bit for bit: bf16 and fp32 outputs,
per-tensor and per-row scales, 2, 3 and 4 ranks. The steps themselves are also checked against
the oracle: amax exactly, q and s_x bit-exact.
"""
import numpy as np
import pytest
import torch

import synth
from util import bf16_tensor_from_bits

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


def _case(M, N, K, per_row, seed):
    g = synth.rng(seed, 91, M, N + K, synth.KIND_T)
    x = synth.normal_x(M, K, g)
    x[0, 7] = synth.to_bf16_bits(np.array([-60.0], dtype=np.float32))[0]  # outlier in slice 0
    if M > 2:
        x[1] = 0
    t = synth.ternary(N, K, g, 0.4)
    s_w = synth.uniform_scale(N if per_row else 1, g)
    return x, t, s_w


@pytest.mark.parametrize("M,K", [(1, 64), (5, 2560), (130, 6912), (3, 14336)])
def test_amax_and_quant_with_amax_match_the_oracle(bn, oracle, M, K):
    x, _, _ = _case(M, 8, K, False, 0)
    xd = bf16_tensor_from_bits(x)
    amax = bn.bitnet_act_amax(xd).cpu().numpy()
    xf = synth.bf16_bits_to_f32(x)
    assert np.array_equal(amax, np.abs(xf).max(axis=1).astype(np.float32))
    q, s_x = bn.bitnet_quant_act_amax(xd, torch.from_numpy(amax).cuda())
    q_ref, s_ref = oracle.quant_act(x)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s_x.cpu().numpy(), s_ref)


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("M,N,K,per_row", [(1, 2560, 2560, False), (7, 300, 6912, True),
                                           (64, 640, 4096, False), (300, 129, 1024, True)])
def test_row_split_equals_bitnet_linear(bn, M, N, K, per_row, world):
    from ternary_w2a8_linear_token_b200.tensor_parallel import split_range
    x, t, s_w = _case(M, N, K, per_row, world)
    packed = bn.bitnet_pack_ternary(torch.from_numpy(t).cuda())
    sw = torch.from_numpy(s_w).cuda()
    xd = bf16_tensor_from_bits(x)
    ranges = [split_range(K, world, r, align=64) for r in range(world)]
    slices = [(xd[:, a:b].contiguous(), packed[:, a // 4: b // 4].contiguous()) for a, b in ranges]
    amax = torch.stack([bn.bitnet_act_amax(xs) for xs, _ in slices]).amax(dim=0)  # all-reduce max
    parts = []
    for xs, ps in slices:
        q, s_x = bn.bitnet_quant_act_amax(xs, amax)
        parts.append(bn.bitnet_linear_i32(q, ps))
    acc = torch.stack(parts).sum(dim=0, dtype=torch.int32)  # all-reduce sum
    for dtype in (torch.bfloat16, torch.float32):
        y = bn.bitnet_dequant(acc, s_x, sw, per_row, out_dtype=dtype)
        ref = bn.bitnet_linear(xd, packed, sw, per_row, out_dtype=dtype)
        view = torch.int16 if dtype == torch.bfloat16 else torch.int32
        assert torch.equal(y.view(view), ref.view(view)), f"world={world} {dtype}"


@pytest.mark.parametrize("world", [2, 3])
def test_column_split_equals_bitnet_linear(bn, world):
    from ternary_w2a8_linear_token_b200.tensor_parallel import split_range
    M, N, K = 9, 1001, 2560
    x, t, s_w = _case(M, N, K, True, 5)
    packed = bn.bitnet_pack_ternary(torch.from_numpy(t).cuda())
    sw = torch.from_numpy(s_w).cuda()
    xd = bf16_tensor_from_bits(x)
    ys = []
    for r in range(world):
        a, b = split_range(N, world, r)
        ys.append(bn.bitnet_linear(xd, packed[a:b].contiguous(), sw[a:b].contiguous(), True))
    ref = bn.bitnet_linear(xd, packed, sw, True)
    assert torch.equal(torch.cat(ys, dim=1).view(torch.int16), ref.view(torch.int16))
