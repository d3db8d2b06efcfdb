"""GPU parity of the fused MLP gate/up + SwiGLU call against the CPU oracle.

bitnet_linear_swiglu computes, per token and output j, g and u (the gate and up BitLinear
outputs, bf16), s = bf16(silu(g)) and h = bf16(s * u) ("BitNet 深度实战" §3.2,
BitLlamaMLP). Bars:
  - bitnet_interleave_gate_up: bit-exact against the block interleave done in numpy;
  - h: inside the bound derived in ``util.assert_swiglu_within_bound`` (g and u one bf16
    step from the exactly rounded values, silu one step from its exact rounding), and equal
    to the oracle's h for at least 99 % of outputs;
  - the GEMV and tensor-core paths give the same h bit for bit (same arithmetic).
"""
import numpy as np
import pytest
import torch

import synth
from util import assert_swiglu_within_bound, bf16_tensor_from_bits, bits_from_bf16_tensor

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


def _mlp(M, I, K, per_row, seed=0, p0=0.4):
    """Seeded MLP gate/up weights (ternary, P(0) = p0) with U(0.5, 2) scales, and x ~ N(0, 1)."""
    key = 2000 + I
    tg = synth.ternary(I, K, synth.rng(seed, 4, key, 4, synth.KIND_T), p0)
    tu = synth.ternary(I, K, synth.rng(seed, 4, key, 5, synth.KIND_T), p0)
    ns = I if per_row else 1
    sg = synth.uniform_scale(ns, synth.rng(seed, 4, key, 4, synth.KIND_SW))
    su = synth.uniform_scale(ns, synth.rng(seed, 4, key, 5, synth.KIND_SW))
    x = synth.normal_x(M, K, synth.rng(seed, 4, key + M, 0, synth.KIND_X))
    return x, tg, tu, sg, su


def _device_weights(bn, oracle, tg, tu, sg, su, per_row):
    pg, pu = oracle.pack(tg), oracle.pack(tu)
    dev = lambda a: torch.from_numpy(a).cuda()
    packed_gu, s_gu = bn.bitnet_interleave_gate_up(dev(pg), dev(sg), dev(pu), dev(su), per_row)
    return pg, pu, packed_gu, s_gu


def _interleave_np(a, b, block=16):
    n = a.shape[0]
    out = np.empty((2 * n,) + a.shape[1:], dtype=a.dtype)
    for blk in range(n // block):
        out[2 * blk * block:(2 * blk + 1) * block] = a[blk * block:(blk + 1) * block]
        out[(2 * blk + 1) * block:(2 * blk + 2) * block] = b[blk * block:(blk + 1) * block]
    return out


@pytest.mark.parametrize("per_row", [False, True])
@pytest.mark.parametrize("I,K", [(16, 64), (96, 512), (6912, 2560)])
def test_interleave_gate_up_layout(bn, oracle, per_row, I, K):
    x, tg, tu, sg, su = _mlp(1, I, K, per_row)
    pg, pu, packed_gu, s_gu = _device_weights(bn, oracle, tg, tu, sg, su, per_row)
    assert np.array_equal(packed_gu.cpu().numpy(), _interleave_np(pg, pu))
    want_s = _interleave_np(sg, su) if per_row else np.array([sg[0], su[0]], dtype=np.float32)
    assert np.array_equal(s_gu.cpu().numpy(), want_s)


SWIGLU_CASES = [
    # (M, I, K, per_row, path) — GEMV for M <= 8, tensor-core tiles of 16 .. 192 tokens,
    # ragged M, several 128-row weight tiles (64 outputs each) and a partial last tile
    (1, 64, 512, False, "gemv"),
    (3, 48, 2560, True, "gemv"),
    (4, 208, 4096, False, "gemv"),
    (8, 160, 2560, True, "gemv"),
    (1, 4816, 2560, False, "gemv"),  # two gate/up pairs per warp, ragged last CTA
    (2, 4816, 1024, True, "gemv"),
    (1, 1024, 6912, True, "gemv"),  # four chunks per lane
    (8, 160, 2560, True, "tc"),
    (16, 144, 512, False, "tc"),
    (37, 208, 2560, True, "tc"),
    (130, 320, 2560, False, "tc"),
    (300, 96, 4096, True, "tc"),
]


@pytest.mark.parametrize("M,I,K,per_row,path", SWIGLU_CASES)
def test_swiglu_matches_oracle(bn, oracle, M, I, K, per_row, path):
    x, tg, tu, sg, su = _mlp(M, I, K, per_row)
    pg, pu, packed_gu, s_gu = _device_weights(bn, oracle, tg, tu, sg, su, per_row)
    p = bn.PATH_GEMV if path == "gemv" else bn.PATH_TC
    h = bn.bitnet_linear_swiglu(bf16_tensor_from_bits(x), packed_gu, s_gu, per_row, path=p)
    torch.cuda.synchronize()
    ref = oracle.swiglu_gate_up(x, pg, sg, pu, su, per_row, K)
    assert_swiglu_within_bound(bits_from_bf16_tensor(h), ref, oracle,
                               where=f"M={M} I={I} K={K} {path}")


@pytest.mark.parametrize("M", [4, 8])
def test_swiglu_paths_agree_bit_for_bit(bn, oracle, M):
    x, tg, tu, sg, su = _mlp(M, 352, 2560, False)
    _, _, packed_gu, s_gu = _device_weights(bn, oracle, tg, tu, sg, su, False)
    xd = bf16_tensor_from_bits(x)
    h1 = bn.bitnet_linear_swiglu(xd, packed_gu, s_gu, False, path=bn.PATH_GEMV)
    h2 = bn.bitnet_linear_swiglu(xd, packed_gu, s_gu, False, path=bn.PATH_TC)
    assert torch.equal(h1.view(torch.int16), h2.view(torch.int16))


def test_swiglu_2b_mlp_decode_full_size(bn, oracle):
    """2B-4T MLP gate/up (I = 6912, K = 2560) at M = 1 on the default path: every output."""
    layer = synth.stack2b_layer(0)
    g, u = layer["gate"], layer["up"]
    x = synth.stack2b_x(1, 2560)
    pg, pu, packed_gu, s_gu = _device_weights(bn, oracle, g["t"], u["t"], g["s_w"], u["s_w"],
                                              False)
    h = bn.bitnet_linear_swiglu(bf16_tensor_from_bits(x), packed_gu, s_gu, False)
    torch.cuda.synchronize()
    ref = oracle.swiglu_gate_up(x, pg, g["s_w"], pu, u["s_w"], False, 2560)
    assert_swiglu_within_bound(bits_from_bf16_tensor(h), ref, oracle, where="2B decode")


@pytest.mark.parametrize("M", [512, 2048])
def test_swiglu_2b_mlp_prefill_sampled(bn, oracle, M):
    """2B-4T MLP gate/up at prefill sizes on the tensor-core path, in the launch
    configuration the benchmark times; sampled tokens x outputs checked one by one."""
    layer = synth.stack2b_layer(0)
    g, u = layer["gate"], layer["up"]
    x = synth.stack2b_x(M, 2560)
    pg, pu, packed_gu, s_gu = _device_weights(bn, oracle, g["t"], u["t"], g["s_w"], u["s_w"],
                                              False)
    h = bn.bitnet_linear_swiglu(bf16_tensor_from_bits(x), packed_gu, s_gu, False)
    torch.cuda.synchronize()
    rs = np.random.default_rng(M)
    m_idx = np.unique(np.concatenate([[0, M - 1], rs.integers(0, M, 30)]))
    n_idx = np.unique(np.concatenate([[0, 63, 64, 6911], rs.integers(0, 6912, 60)]))
    ref = oracle.swiglu_gate_up_sampled(x, pg, g["s_w"], pu, u["s_w"], False, 2560, m_idx, n_idx)
    got = bits_from_bf16_tensor(h)[np.ix_(m_idx, n_idx)]
    assert_swiglu_within_bound(got, ref, oracle, where=f"2B prefill M={M}")


def test_swiglu_8b_mlp_per_row_sampled(bn, oracle):
    """8B-class MLP gate/up (I = 14336, K = 4096), latent weights packed with per-row
    scales, at M = 128 (tensor-core path); sampled outputs."""
    Wg = synth.stack8b_latent(0, "gate")
    Wu = synth.stack8b_latent(0, "up")
    pg, sg = oracle.pack_weights(Wg, True)
    pu, su = oracle.pack_weights(Wu, True)
    dev = lambda a: torch.from_numpy(a).cuda()
    packed_gu, s_gu = bn.bitnet_interleave_gate_up(dev(pg), dev(sg), dev(pu), dev(su), True)
    M = 128
    x = synth.stack8b_x(M, 4096)
    h = bn.bitnet_linear_swiglu(bf16_tensor_from_bits(x), packed_gu, s_gu, True)
    torch.cuda.synchronize()
    rs = np.random.default_rng(8)
    m_idx = np.unique(np.concatenate([[0, M - 1], rs.integers(0, M, 20)]))
    n_idx = np.unique(np.concatenate([[0, 14335], rs.integers(0, 14336, 60)]))
    ref = oracle.swiglu_gate_up_sampled(x, pg, sg, pu, su, True, 4096, m_idx, n_idx)
    got = bits_from_bf16_tensor(h)[np.ix_(m_idx, n_idx)]
    assert_swiglu_within_bound(got, ref, oracle, where="8B M=128")


def test_swiglu_8b_mlp_decode_stream(bn, oracle):
    """8B-class MLP gate/up at M = 1 (29 MB interleaved, the grid-stride GEMV), per-row scales,
    every output."""
    Wg = synth.stack8b_latent(0, "gate")
    Wu = synth.stack8b_latent(0, "up")
    pg, sg = oracle.pack_weights(Wg, True)
    pu, su = oracle.pack_weights(Wu, True)
    dev = lambda a: torch.from_numpy(a).cuda()
    packed_gu, s_gu = bn.bitnet_interleave_gate_up(dev(pg), dev(sg), dev(pu), dev(su), True)
    x = synth.stack8b_x(1, 4096)
    h = bn.bitnet_linear_swiglu(bf16_tensor_from_bits(x), packed_gu, s_gu, True)
    torch.cuda.synchronize()
    ref = oracle.swiglu_gate_up(x, pg, sg, pu, su, True, 4096)
    assert_swiglu_within_bound(bits_from_bf16_tensor(h), ref, oracle, where="8B decode")


def test_swiglu_one_token_grid_stride_per_tensor(bn, oracle):
    """One token, 10000 output pairs at K = 2560 (12.8 MB interleaved: the grid-stride GEMV's
    SwiGLU pairing), per-tensor gate and up scales: within the bound, and bit-equal to the
    tensor-core path (same arithmetic)."""
    I, K = 10000, 2560
    assert bn.bitnet_linear_plan(1, K, [2 * I], swiglu=True)["kernel"] == bn.KERNEL_GS
    x, tg, tu, sg, su = _mlp(1, I, K, False)
    pg, pu, packed_gu, s_gu = _device_weights(bn, oracle, tg, tu, sg, su, False)
    xd = bf16_tensor_from_bits(x)
    h = bn.bitnet_linear_swiglu(xd, packed_gu, s_gu, False)
    torch.cuda.synchronize()
    ref = oracle.swiglu_gate_up(x, pg, sg, pu, su, False, K)
    assert_swiglu_within_bound(bits_from_bf16_tensor(h), ref, oracle, where="grid-stride SwiGLU")
    h_tc = bn.bitnet_linear_swiglu(xd, packed_gu, s_gu, False, path=bn.PATH_TC)
    assert torch.equal(h.view(torch.int16), h_tc.view(torch.int16))


@pytest.mark.parametrize("per_row", [False, True])
def test_swiglu_one_token_streaming_long_rows(bn, oracle, per_row):
    """One token, rows longer than the grid-stride kernel takes (K = 8192) and 13.1 MB of
    interleaved gate/up weights: the streaming GEMV's SwiGLU pairing. Within the bound, and
    bit-equal to the tensor-core path (same arithmetic)."""
    I, K = 3200, 8192
    assert bn.bitnet_linear_plan(1, K, [2 * I], swiglu=True)["kernel"] == bn.KERNEL_STREAM
    x, tg, tu, sg, su = _mlp(1, I, K, per_row, seed=3)
    pg, pu, packed_gu, s_gu = _device_weights(bn, oracle, tg, tu, sg, su, per_row)
    xd = bf16_tensor_from_bits(x)
    h = bn.bitnet_linear_swiglu(xd, packed_gu, s_gu, per_row)
    torch.cuda.synchronize()
    ref = oracle.swiglu_gate_up(x, pg, sg, pu, su, per_row, K)
    assert_swiglu_within_bound(bits_from_bf16_tensor(h), ref, oracle, where="streaming SwiGLU")
    h_tc = bn.bitnet_linear_swiglu(xd, packed_gu, s_gu, per_row, path=bn.PATH_TC)
    assert torch.equal(h.view(torch.int16), h_tc.view(torch.int16))
