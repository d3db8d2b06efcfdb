"""GPU parity of the layer-stack workloads at their own token counts, on the default path.

The 2B-4T stack (q/k/v/gate/up batched over one hidden state, o, down) at M = 8, 32 and 64,
and the 8B-class stack (latent weights N(0, 0.02^2) packed per row by bitnet_pack_weights) at
M = 16, 128 and 4096 — the last in the launch configuration the benchmark times, whose
tensor-core kernel takes 192-token tiles with the plain TMA-store epilogue (asserted through
bitnet_linear_plan). Every token of each call is checked on sampled output columns (first and
last included) against the oracle's forward on that sample: bf16 within one step of the exact
value, zero where acc = 0.
"""
import numpy as np
import pytest
import torch

import synth
from util import assert_bf16_within_1ulp, bf16_tensor_from_bits, bits_from_bf16_tensor

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


BATCHED = ("q", "k", "v", "gate", "up")


def _sample(n, count, seed):
    g = np.random.default_rng(seed)
    extra = g.choice(n, min(count, n), replace=False)
    return np.unique(np.concatenate([[0, n - 1], extra]))


def _check_call(bn, oracle, x_bits, weights, ys, m_idx, seed, where):
    """weights: list of (packed_np, s_w_np, per_row, K); ys: device outputs."""
    for i, ((packed, s_w, per_row, K), y) in enumerate(zip(weights, ys)):
        N = packed.shape[0]
        n_idx = _sample(N, 40, seed + i)
        ref = oracle.bitlinear_sampled(x_bits, packed, s_w, per_row, K, m_idx, n_idx)
        got = bits_from_bf16_tensor(y)[np.ix_(m_idx, n_idx)]
        assert_bf16_within_1ulp(got, ref["y"], oracle, f"{where} projection {i}")


@pytest.mark.parametrize("M", [8, 32, 64])
def test_2b_stack_layer_at_its_token_counts(bn, oracle, M):
    layer = synth.stack2b_layer(0)
    dev = {p: (torch.from_numpy(oracle.pack(d["t"])).cuda(), torch.from_numpy(d["s_w"]).cuda())
           for p, d in layer.items()}
    x_h = synth.stack2b_x(M, 2560)
    x_f = synth.stack2b_x(M, 6912, which=1)
    xh, xf = bf16_tensor_from_bits(x_h), bf16_tensor_from_bits(x_f)
    ys = bn.bitnet_linear_batch(xh, [(dev[p][0], dev[p][1], False) for p in BATCHED])
    y_o = bn.bitnet_linear(xh, dev["o"][0], dev["o"][1], False)
    y_d = bn.bitnet_linear(xf, dev["down"][0], dev["down"][1], False)
    torch.cuda.synchronize()
    m_idx = np.arange(M)
    w = lambda p: (oracle.pack(layer[p]["t"]), layer[p]["s_w"], False, layer[p]["K"])
    _check_call(bn, oracle, x_h, [w(p) for p in BATCHED], ys, m_idx, 10, f"2B M={M} batch")
    _check_call(bn, oracle, x_h, [w("o")], [y_o], m_idx, 20, f"2B M={M} o")
    _check_call(bn, oracle, x_f, [w("down")], [y_d], m_idx, 30, f"2B M={M} down")


@pytest.fixture(scope="module")
def stack8b(bn):
    """Layer 0 of the 8B-class stack, packed per row on the GPU: device and host copies."""
    out = {}
    for p in synth.SHAPES_8B:
        W = torch.from_numpy(synth.stack8b_latent(0, p)).cuda()
        packed, s_w = bn.bitnet_pack_weights(W, True)
        del W
        out[p] = (packed, s_w, packed.cpu().numpy(), s_w.cpu().numpy())
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("M", [16, 128, 4096])
def test_8b_stack_layer_at_its_token_counts(bn, oracle, stack8b, M):
    hidden, ffn = 4096, 14336
    Ns = [stack8b[p][0].shape[0] for p in BATCHED]
    plan_b = bn.bitnet_linear_plan(M, hidden, Ns)
    plan_d = bn.bitnet_linear_plan(M, ffn, [hidden])
    if M == 4096:  # the benchmark's prefill configuration: 192-token tiles, plain epilogue
        assert plan_b["kernel"] == bn.KERNEL_TC and plan_b["tile_tokens"] == 192, plan_b
        assert plan_d["kernel"] == bn.KERNEL_TC and plan_d["tile_tokens"] == 192, plan_d
    x_h = synth.stack8b_x(M, hidden)
    x_f = synth.stack8b_x(M, ffn, which=1)
    xh, xf = bf16_tensor_from_bits(x_h), bf16_tensor_from_bits(x_f)
    ys = bn.bitnet_linear_batch(xh, [(stack8b[p][0], stack8b[p][1], True) for p in BATCHED])
    y_o = bn.bitnet_linear(xh, stack8b["o"][0], stack8b["o"][1], True)
    y_d = bn.bitnet_linear(xf, stack8b["down"][0], stack8b["down"][1], True)
    torch.cuda.synchronize()
    m_idx = np.arange(M) if M <= 128 else _sample(M, 14, 7)
    w = lambda p, K: (stack8b[p][2], stack8b[p][3], True, K)
    _check_call(bn, oracle, x_h, [w(p, hidden) for p in BATCHED], ys, m_idx, 40,
                f"8B M={M} batch")
    _check_call(bn, oracle, x_h, [w("o", hidden)], [y_o], m_idx, 50, f"8B M={M} o")
    _check_call(bn, oracle, x_f, [w("down", ffn)], [y_d], m_idx, 60, f"8B M={M} down")
