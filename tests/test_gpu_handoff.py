"""GPU parity of the SwiGLU -> down projection hand-off.

The gate/up epilogue writes, beside h, the maxima of |h| over blocks of 16 outputs
(bitnet_linear_swiglu_hmax); the down projection's quantiser takes each token's amax from
them instead of reducing the row of h (bitnet_linear_hmax, bitnet_quant_act_hmax). The
block maxima are exact, so every result must equal the plain per-token path bit for bit:
  - q and s_x of bitnet_quant_act_hmax against oracle.quant_act, with the oracle's own
    block maxima as input (register-resident, four-warp and two-pass row lengths);
  - y of bitnet_linear_hmax against the oracle's BitLinear (bf16 within one step, expected
    exact) and bit for bit against bitnet_linear on the same path;
  - hmax of bitnet_linear_swiglu_hmax: the block maxima of the h it returned, and equal to
    the oracle's block maxima wherever the block's 16 outputs equal the oracle's h; h equal
    bit for bit to bitnet_linear_swiglu's;
  - the whole MLP chain gate/up -> down through the hand-off equals the unfused chain bit
    for bit, at the 2B-4T MLP's prefill size among others.
"""
import numpy as np
import pytest
import torch

import synth
from util import (assert_bf16_within_1ulp, assert_swiglu_within_bound, bf16_tensor_from_bits,
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


def _x(M, K, seed):
    """x ~ N(0, 1) with an outlier, an all-zero token and a token whose max sits in the last
    block (the block index must not be dropped)."""
    g = synth.rng(seed, 95, M, K, synth.KIND_X)
    x = synth.normal_x(M, K, g)
    x[0, K // 3] = synth.to_bf16_bits(np.array([-75.0], dtype=np.float32))[0]
    if M > 2:
        x[1] = 0
    if M > 3:
        x[3, K - 1] = synth.to_bf16_bits(np.array([41.0], dtype=np.float32))[0]
    return x


def _dev_i16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def _block_max_np(bits):
    """The property the returned hmax must satisfy against the returned h (plain numpy)."""
    M, I = bits.shape
    return (bits & 0x7FFF).reshape(M, I // 16, 16).max(axis=2)


@pytest.mark.parametrize("M,K", [(1, 64), (7, 512), (33, 2560), (5, 6912), (3, 14336),
                                 (2, 16384), (300, 4096)])
def test_quant_act_hmax_matches_oracle(bn, oracle, M, K):
    x = _x(M, K, 1)
    xmax = oracle.block_absmax_bits(x)
    q, s_x = bn.bitnet_quant_act_hmax(bf16_tensor_from_bits(x), _dev_i16(xmax))
    q_ref, s_ref = oracle.quant_act(x)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s_x.cpu().numpy(), s_ref)


@pytest.mark.parametrize("M,N,K,per_row", [(1, 64, 512, False), (37, 300, 2560, True),
                                           (130, 640, 6912, False), (9, 129, 14336, True)])
def test_linear_hmax_matches_oracle(bn, oracle, M, N, K, per_row):
    x = _x(M, K, 2)
    g = synth.rng(2, 95, N, K, synth.KIND_T)
    t = synth.ternary(N, K, g, 0.4)
    s_w = synth.uniform_scale(N if per_row else 1, g)
    packed = torch.from_numpy(oracle.pack(t)).cuda()
    sw = torch.from_numpy(s_w).cuda()
    xd = bf16_tensor_from_bits(x)
    xm = _dev_i16(oracle.block_absmax_bits(x))
    ref = oracle.bitlinear(x, oracle.pack(t), s_w, per_row, K)
    for dtype in (torch.bfloat16, torch.float32):
        y = bn.bitnet_linear_hmax(xd, xm, packed, sw, per_row, out_dtype=dtype)
        plain = bn.bitnet_linear(xd, packed, sw, per_row, out_dtype=dtype, path=bn.PATH_TC)
        view = torch.int16 if dtype == torch.bfloat16 else torch.int32
        assert torch.equal(y.view(view), plain.view(view))
        if dtype == torch.bfloat16:
            assert_bf16_within_1ulp(bits_from_bf16_tensor(y), ref["y"], oracle,
                                    where=f"M={M} N={N} K={K}")


def _mlp_weights(bn, oracle, I, K, N, per_row, seed):
    g = synth.rng(seed, 96, I, K, synth.KIND_T)
    tg, tu, td = synth.ternary(I, K, g, 0.4), synth.ternary(I, K, g, 0.4), synth.ternary(N, I, g, 0.4)
    ns = I if per_row else 1
    sg, su = synth.uniform_scale(ns, g), synth.uniform_scale(ns, g)
    sd = synth.uniform_scale(N if per_row else 1, g)
    pg, pu, pd = oracle.pack(tg), oracle.pack(tu), oracle.pack(td)
    dev = lambda a: torch.from_numpy(a).cuda()
    packed_gu, s_gu = bn.bitnet_interleave_gate_up(dev(pg), dev(sg), dev(pu), dev(su), per_row)
    return {"pg": pg, "pu": pu, "sg": sg, "su": su, "packed_gu": packed_gu, "s_gu": s_gu,
            "pd": dev(pd), "sd": dev(sd)}


# (M, I, K, N, per_row): one token on the tensor-core path, ragged token tiles, a partial
# last weight tile (I = 1008: 2016 gate/up rows, the last 128-row tile a quarter short), and
# the 2B-4T MLP (I = 6912, K = N = 2560) at a prefill size. The down projection needs
# I % 64 == 0, so the chain runs where that holds.
MLP_CASES = [(1, 64, 512, 64, False), (5, 48, 2560, 128, True), (37, 1008, 512, 512, False),
             (37, 1024, 512, 512, True), (300, 6912, 2560, 2560, False),
             (2048, 6912, 2560, 2560, False)]


@pytest.mark.parametrize("M,I,K,N,per_row", MLP_CASES)
def test_swiglu_hmax_and_chain(bn, oracle, M, I, K, N, per_row):
    w = _mlp_weights(bn, oracle, I, K, N, per_row, seed=M)
    x = _x(M, K, 3)
    xd = bf16_tensor_from_bits(x)
    h, hmax = bn.bitnet_linear_swiglu_hmax(xd, w["packed_gu"], w["s_gu"], per_row)
    h_plain = bn.bitnet_linear_swiglu(xd, w["packed_gu"], w["s_gu"], per_row, path=bn.PATH_TC)
    assert torch.equal(h.view(torch.int16), h_plain.view(torch.int16))
    hb = bits_from_bf16_tensor(h)
    hm = hmax.cpu().numpy().view(np.uint16)
    assert np.array_equal(hm, _block_max_np(hb))  # every block, every token

    # Against the oracle: all outputs of a few tokens (all tokens when small).
    m_idx = np.arange(M) if M * I * K <= 40_000_000 else np.unique([0, 1, 3, M // 2, M - 1])
    ref = oracle.swiglu_gate_up_sampled(x, w["pg"], w["sg"], w["pu"], w["su"], per_row, K,
                                        m_idx, np.arange(I))
    assert_swiglu_within_bound(hb[m_idx], ref, oracle, where=f"M={M} I={I}")
    ref_max = oracle.block_absmax_bits(ref["h_bits"])
    same = (hb[m_idx] == ref["h_bits"]).reshape(len(m_idx), I // 16, 16).all(axis=2)
    assert same.mean() >= 0.8
    assert np.array_equal(hm[m_idx][same], ref_max[same])

    # The down projection through the hand-off equals the unfused chain bit for bit.
    if I % 64:
        return
    y = bn.bitnet_linear_hmax(h, hmax, w["pd"], w["sd"], per_row)
    y_plain = bn.bitnet_linear(h, w["pd"], w["sd"], per_row, path=bn.PATH_TC)
    assert torch.equal(y.view(torch.int16), y_plain.view(torch.int16))


def test_hand_off_repeated_calls_reuse_buffers(bn, oracle):
    """Two MLP calls in a row on one workspace: the second call's hmax and y depend on its
    own input only (nothing carried over from the first)."""
    M, I, K, N = 64, 1024, 512, 512
    w = _mlp_weights(bn, oracle, I, K, N, False, seed=9)
    ws = bn.make_workspace(M, max(K, I), torch.device("cuda"))
    outs = []
    for seed in (4, 5):
        xd = bf16_tensor_from_bits(_x(M, K, seed))
        h, hmax = bn.bitnet_linear_swiglu_hmax(xd, w["packed_gu"], w["s_gu"], False, workspace=ws)
        y = bn.bitnet_linear_hmax(h, hmax, w["pd"], w["sd"], False, workspace=ws)
        outs.append((h.clone(), y.clone()))
    for seed, (h, y) in zip((4, 5), outs):
        xd = bf16_tensor_from_bits(_x(M, K, seed))
        h_plain = bn.bitnet_linear_swiglu(xd, w["packed_gu"], w["s_gu"], False, path=bn.PATH_TC)
        y_plain = bn.bitnet_linear(h_plain, w["pd"], w["sd"], False, path=bn.PATH_TC)
        assert torch.equal(h.view(torch.int16), h_plain.view(torch.int16))
        assert torch.equal(y.view(torch.int16), y_plain.view(torch.int16))
