"""GPU parity of the base-3 weight format (five ternary weights per byte): the packing kernel
bit-exact against the oracle, and the one-token GEMV on it equal bit for bit to bitnet_linear
on the 2-bit packing of the same weights (the same quantiser, contraction and epilogue
arithmetic), and within one bf16 step of the oracle's exact result (zero where acc = 0)."""
import numpy as np
import pytest
import torch

import synth
from util import assert_bf16_within_1ulp, assert_f32_rel, bf16_tensor_from_bits, bits_from_bf16_tensor

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


@pytest.mark.parametrize("N,K", [(1, 64), (37, 512), (300, 2560), (129, 4096), (50, 6912),
                                 (33, 14336)])
def test_pack_b3_bit_exact(bn, oracle, N, K):
    t = synth.ternary(N, K, synth.rng(0, 92, N, K, synth.KIND_T), 0.4)
    got = bn.bitnet_pack_ternary_b3(torch.from_numpy(t).cuda()).cpu().numpy()
    assert np.array_equal(got, oracle.pack_b3(t))


CASES = [  # (N, K, per_row)
    (1, 64, False), (37, 512, True), (2560, 2560, False), (640, 2560, True), (1001, 4096, False),
    (2560, 6912, True), (333, 14336, False), (4096, 4096, True), (14336, 4096, True),
    (4096, 14336, True),
]


@pytest.mark.parametrize("N,K,per_row", CASES)
def test_linear_b3_matches_2bit_and_oracle(bn, oracle, N, K, per_row):
    g = synth.rng(0, 93, N, K, synth.KIND_T)
    t = synth.ternary(N, K, g, 0.4)
    s_w = synth.uniform_scale(N if per_row else 1, g)
    x = synth.normal_x(1, K, g)
    td = torch.from_numpy(t).cuda()
    p3 = bn.bitnet_pack_ternary_b3(td)
    p2 = bn.bitnet_pack_ternary(td)
    sw = torch.from_numpy(s_w).cuda()
    xd = bf16_tensor_from_bits(x)
    ref = oracle.bitlinear(x, oracle.pack(t), s_w, per_row, K)["y"]
    for dtype, view in ((torch.bfloat16, torch.int16), (torch.float32, torch.int32)):
        y3 = bn.bitnet_linear_b3(xd, p3, sw, per_row, out_dtype=dtype)
        y2 = bn.bitnet_linear(xd, p2, sw, per_row, out_dtype=dtype)
        assert torch.equal(y3.view(view), y2.view(view)), f"N={N} K={K} {dtype}"
        if dtype == torch.bfloat16:
            assert_bf16_within_1ulp(bits_from_bf16_tensor(y3), ref, oracle, f"b3 N={N} K={K}")
        else:
            assert_f32_rel(y3.cpu().numpy(), ref, where=f"b3 N={N} K={K}")


def test_linear_b3_zero_token_and_extremes(bn, oracle):
    """An all-zero token gives exact zeros; rows of all -1 / all +1 give the extreme sums."""
    N, K = 64, 2560
    t = synth.ternary(N, K, synth.rng(0, 93, 1, 1, synth.KIND_T), 0.4)
    t[0, :] = -1
    t[1, :] = 1
    p3 = bn.bitnet_pack_ternary_b3(torch.from_numpy(t).cuda())
    sw = torch.ones(1, device="cuda")
    y0 = bn.bitnet_linear_b3(torch.zeros((1, K), dtype=torch.bfloat16, device="cuda"), p3, sw, False)
    assert int((y0.view(torch.int16).cpu() & 0x7FFF).max()) == 0
    x = synth.normal_x(1, K, synth.rng(0, 93, 2, 2, synth.KIND_X))
    y = bn.bitnet_linear_b3(bf16_tensor_from_bits(x), p3, sw, False)
    ref = oracle.bitlinear(x, oracle.pack(t), np.ones(1, np.float32), False, K)["y"]
    assert_bf16_within_1ulp(bits_from_bf16_tensor(y), ref, oracle, "extremes")
