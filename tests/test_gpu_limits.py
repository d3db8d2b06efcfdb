"""GPU parity at the size limits of the kernels.

- The one-token GEMV's longest row (K = 32768) and the first K past it, which runs on the
  tensor-core path (and without a workspace is refused, not silently served).
- M * K beyond 2^31 elements on the tensor-core path (2^20 + 37 tokens x 2560): every
  activation, int8 token and output offset past the 32-bit range.
- N * K / 4 beyond 2^31 packed bytes (2^21 + 64 weight rows x 4096): weight addressing past the
  32-bit range on the tensor-core path (16 tokens) and the one-token streaming GEMV.
Inputs too large to draw on the host come from torch's seeded generator on the device
(``synth.device_*``); the sampled rows the oracle needs are copied from those draws.
Outputs are compared one by one on sampled tokens x sampled outputs (bf16 within one step of
the exact result, the usual bar).
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
    torch.cuda.empty_cache()


def _small(M, N, K, seed):
    g = synth.rng(seed, 97, M, N + K, synth.KIND_T)
    return synth.normal_x(M, K, g), synth.ternary(N, K, g, 0.4), synth.uniform_scale(1, g)


@pytest.mark.parametrize("K,kernel_name", [(32768, "KERNEL_GEMV"), (32832, "KERNEL_TC")])
def test_longest_gemv_row_and_the_next(bn, oracle, K, kernel_name):
    M, N = 1, 300
    x, t, s_w = _small(M, N, K, K)
    packed_h = oracle.pack(t)
    assert bn.bitnet_linear_plan(M, K, [N])["kernel"] == getattr(bn, kernel_name)
    xd = bf16_tensor_from_bits(x)
    packed = torch.from_numpy(packed_h).cuda()
    sw = torch.from_numpy(s_w).cuda()
    if kernel_name == "KERNEL_TC":  # without a workspace: refused before any launch
        y0 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        assert bn.lib.bitnet_linear(xd.data_ptr(), M, K, packed.data_ptr(), sw.data_ptr(), 0, N,
                                    y0.data_ptr(), 0, None, 0, None) == bn.ERR_WORKSPACE
    y = bn.bitnet_linear(xd, packed, sw, False)
    ref = oracle.bitlinear(x, packed_h, s_w, False, K)
    assert_bf16_within_1ulp(bits_from_bf16_tensor(y), ref["y"], oracle, where=f"K={K}")


def test_tokens_times_k_past_32_bits(bn, oracle):
    """2^20 + 37 tokens x K = 2560 (2.7e9 activations, 5.4 GB), one 128-row weight tile."""
    M, N, K = (1 << 20) + 37, 128, 2560
    assert M * K > 2 ** 31
    xd = synth.device_normal_bf16(M, K, seed=101, device="cuda")
    _, t, s_w = _small(1, N, K, 7)
    packed_h = oracle.pack(t)
    packed = torch.from_numpy(packed_h).cuda()
    sw = torch.from_numpy(s_w).cuda()
    ws = bn.make_workspace(M, K, torch.device("cuda"))
    y = bn.bitnet_linear(xd, packed, sw, False, workspace=ws)
    torch.cuda.synchronize()
    del ws
    cross = (2 ** 31) // K  # the token whose activations cross the 32-bit offset
    rs = np.random.default_rng(3)
    m_idx = np.unique(np.concatenate([[0, 1, cross - 1, cross, cross + 1, M - 37, M - 2, M - 1],
                                      rs.integers(0, M, 16)]))
    xs = bits_from_bf16_tensor(xd[torch.from_numpy(m_idx).cuda()])
    ref = oracle.bitlinear_sampled(xs, packed_h, s_w, False, K, np.arange(len(m_idx)),
                                   np.arange(N))
    got = bits_from_bf16_tensor(y[torch.from_numpy(m_idx).cuda()])
    assert_bf16_within_1ulp(got, ref["y"], oracle, where="M*K > 2^31")


@pytest.mark.parametrize("M", [16, 1])
def test_weight_bytes_past_32_bits(bn, oracle, M):
    """2^21 + 64 weight rows x K = 4096: 2.15 GB of packed weights."""
    N, K = (1 << 21) + 64, 4096
    assert N * K // 4 > 2 ** 31
    rs = np.random.default_rng(5)
    n_idx = np.unique(np.concatenate([[0, 1, (1 << 21) - 1, 1 << 21, (1 << 21) + 1, N - 1],
                                      rs.integers(0, N, 18)]))
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device="cuda")
    t_rows = {}
    for r0, t in synth.device_ternary_chunks(N, K, seed=202, device="cuda"):
        rows = t.shape[0]  # the chunk's packed rows, written in place
        assert bn.lib.bitnet_pack_ternary(t.data_ptr(), rows, K, packed[r0:r0 + rows].data_ptr(),
                                          torch.cuda.current_stream().cuda_stream) == bn.OK
        for n in n_idx[(n_idx >= r0) & (n_idx < r0 + t.shape[0])]:
            t_rows[int(n)] = t[int(n) - r0].cpu().numpy()
        del t
    torch.cuda.synchronize()
    x, _, s_w = _small(M, 8, K, 11)
    sw = torch.from_numpy(s_w).cuda()
    ws = bn.make_workspace(M, K, torch.device("cuda")) if M > bn.GEMV_AUTO_M else None
    y = bn.bitnet_linear(bf16_tensor_from_bits(x), packed, sw, False, workspace=ws)
    torch.cuda.synchronize()
    t_s = np.stack([t_rows[int(n)] for n in n_idx])
    ref = oracle.bitlinear_sampled(x, oracle.pack(t_s), s_w, False, K, np.arange(M),
                                   np.arange(len(n_idx)))
    got = bits_from_bf16_tensor(y[:, torch.from_numpy(n_idx).cuda()])
    assert_bf16_within_1ulp(got, ref["y"], oracle, where=f"N*K/4 > 2^31, M={M}")
