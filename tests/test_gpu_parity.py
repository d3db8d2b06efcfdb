"""GPU parity: every result of the CUDA path against the CPU oracle on the same seeded inputs.

Bars (from the method's arithmetic):
  - packed bytes, s_w, int8 q, s_x and int32 accumulators: bit-exact;
  - fp32 y: relative error <= 1e-6 against the exact fp64 value (the kernels use three
    binary32 roundings, < 1.8e-7);
  - bf16 y: at most one bf16 step from RNE(exact value), and exactly zero where acc == 0.
Shapes span several tiles and ragged tails in M, N and K; the full-size workloads are
checked on sampled outputs the oracle computes one by one.
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
    if "bn" in request.fixturenames:
        bn = request.getfixturevalue("bn")
        assert bn.bitnet_check_device_errors() == 0, "a kernel's bounded wait expired"


def _packed_dev(oracle, t):
    return torch.from_numpy(oracle.pack(t)).cuda()


# ------------------------------------------------------------------------------- packing

@pytest.mark.parametrize("per_row", [False, True])
@pytest.mark.parametrize("N,K,sigma", [(256, 512, 1.0), (37, 64, 0.02), (300, 2560, 0.02)])
def test_pack_weights_bit_exact(bn, oracle, per_row, N, K, sigma):
    W = synth.latent_w(N, K, synth.rng(0, 90, N, K, synth.KIND_W), sigma)
    W[min(3, N - 1)] = 0.0  # an all-zero row hits the eps clamp in per-row mode
    packed, s_w = bn.bitnet_pack_weights(torch.from_numpy(W).cuda(), per_row)
    p_ref, s_ref = oracle.pack_weights(W, per_row)
    assert np.array_equal(s_w.cpu().numpy(), s_ref)
    assert np.array_equal(packed.cpu().numpy(), p_ref)


def test_pack_weights_tiny_config(bn, oracle):
    cfg = synth.tiny(0)
    packed, s_w = bn.bitnet_pack_weights(torch.from_numpy(cfg["W"]).cuda(), False)
    p_ref, s_ref = oracle.pack_weights(cfg["W"], False)
    assert np.array_equal(s_w.cpu().numpy(), s_ref) and np.array_equal(packed.cpu().numpy(), p_ref)


def test_pack_weights_worked_example_row(bn, oracle):
    """The printed example row, padded to K = 64 with alternating +-5/6: the padding keeps
    the row's absmean at 5/6 (to fp32 rounding), so the six printed weights quantise as
    printed and each pad value quantises to +-1."""
    W = np.empty((1, 64), dtype=np.float32)
    W[0, 6:] = np.float32(5.0 / 6.0) * np.where(np.arange(58) % 2 == 0, 1.0, -1.0)
    W[0, :6] = [-0.3, 1.7, 0.0, -2.1, 0.8, -0.1]
    packed, s_w = bn.bitnet_pack_weights(torch.from_numpy(W).cuda(), True)
    assert abs(float(s_w.cpu()[0]) - 5.0 / 6.0) < 1e-6
    t = oracle.unpack(packed.cpu().numpy(), 64)
    assert t[0, :6].tolist() == [0, 1, 0, -1, 1, 0]
    assert t[0, 6:].tolist() == [1, -1] * 29
    assert packed.cpu().numpy()[0, 0] == 0x19  # codes (1, 2, 1, 0), as in the pack fixture
    p_ref, s_ref = oracle.pack_weights(W, True)
    assert np.array_equal(packed.cpu().numpy(), p_ref) and np.array_equal(s_w.cpu().numpy(), s_ref)


def test_pack_weights_8b_projection_full_size(bn, oracle):
    """8B-class gate projection (14336 x 4096), latent N(0, 0.02^2), per-row absmean."""
    W = synth.stack8b_latent(0, "gate")
    packed, s_w = bn.bitnet_pack_weights(torch.from_numpy(W).cuda(), True)
    p_ref, s_ref = oracle.pack_weights(W, True)
    assert np.array_equal(s_w.cpu().numpy(), s_ref)
    assert np.array_equal(packed.cpu().numpy(), p_ref)


@pytest.mark.parametrize("N,K", [(5, 64), (640, 2560), (129, 6912)])
def test_pack_ternary_bit_exact(bn, oracle, N, K):
    t = synth.ternary(N, K, synth.rng(0, 91, N, K, synth.KIND_T), 0.4)
    packed = bn.bitnet_pack_ternary(torch.from_numpy(t).cuda())
    assert np.array_equal(packed.cpu().numpy(), oracle.pack(t))


# ------------------------------------------------------------------------------- quantiser

@pytest.mark.parametrize("M,K", [(1, 64), (4, 512), (7, 2560), (33, 6912), (130, 4096),
                                 (3, 14336)])
def test_quant_act_bit_exact(bn, oracle, M, K):
    x = synth.normal_x(M, K, synth.rng(0, 92, M, K, synth.KIND_X))
    if M > 2:
        x[1] = 0  # all-zero token
    q, s_x = bn.bitnet_quant_act(bf16_tensor_from_bits(x))
    q_ref, s_ref = oracle.quant_act(x)
    assert np.array_equal(s_x.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


def test_quant_act_outliers_and_tiny_scales(bn, oracle):
    """Student-t activations with x20 outlier channels; tokens at 1e-8 scale (eps clamp)."""
    x, _ = synth.student_t_outlier_x(64, 2560, synth.rng(0, 93, 0, 0, synth.KIND_X),
                                     synth.rng(0, 93, 0, 0, synth.KIND_OUTLIER))
    tiny = synth.to_bf16_bits(synth.bf16_bits_to_f32(x[:4]) * np.float32(1e-8))
    x = np.concatenate([x, tiny])
    q, s_x = bn.bitnet_quant_act(bf16_tensor_from_bits(x))
    q_ref, s_ref = oracle.quant_act(x)
    assert np.array_equal(s_x.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


# ------------------------------------------------------------------------------- contraction

I32_CASES = [  # (M, N, K): tile multiples, ragged tails and the minimum K
    (1, 64, 64), (2, 200, 512), (3, 131, 192), (4, 640, 2560), (5, 256, 512), (8, 100, 6912),
    (9, 130, 512), (16, 128, 256), (17, 257, 512), (63, 384, 640), (64, 128, 2560),
    (65, 129, 1024), (127, 256, 512), (128, 128, 128), (129, 300, 384), (255, 128, 512),
    (256, 256, 2560), (257, 129, 512), (600, 200, 448),
    (300, 384, 2560), (1000, 640, 2560),  # 128-token tiles past M = 128
    (48, 256, 4160), (20, 200, 1088),  # split-K with 64- and 32-token tiles, K not a stage multiple
    (1, 10001, 1024), (2, 9600, 2560),  # the GEMV at four rows per warp
]


@pytest.mark.parametrize("M,N,K", I32_CASES)
def test_linear_i32_bit_exact_both_paths(bn, oracle, M, N, K):
    g = synth.rng(0, 94, M * 7 + N, K, synth.KIND_T)
    q = g.integers(-128, 128, size=(M, K)).astype(np.int8)
    q[0, :] = -128  # extreme accumulator values on one token
    t = synth.ternary(N, K, g, 0.4)
    t[0, :] = -1
    packed = _packed_dev(oracle, t)
    ref = oracle.ternary_matmul(q, t)
    qd = torch.from_numpy(q).cuda()
    paths = [bn.PATH_TC] + ([bn.PATH_GEMV] if M <= bn.GEMV_MAX_M else [])
    for path in paths:
        acc = bn.bitnet_linear_i32(qd, packed, path=path).cpu().numpy()
        assert np.array_equal(acc, ref), f"path {path}: {np.argwhere(acc != ref)[:5]}"


# ------------------------------------------------------------------------------- full forward

def _run_linear(bn, x, packed, s_w, per_row, dtype, path):
    return bn.bitnet_linear(bf16_tensor_from_bits(x), packed, torch.from_numpy(s_w).cuda(),
                            per_row, out_dtype=dtype, path=path)


def _check_y(y, ref_y, oracle, where):
    if y.dtype == torch.bfloat16:
        assert_bf16_within_1ulp(bits_from_bf16_tensor(y), ref_y, oracle, where)
    else:
        assert_f32_rel(y.cpu().numpy(), ref_y, where=where)


def test_tiny_config_forward(bn, oracle):
    """Tiny BitLinear, x (4, 512), latent W (256, 512) per-tensor, seed 0: whole output."""
    cfg = synth.tiny(0)
    packed, s_w = bn.bitnet_pack_weights(torch.from_numpy(cfg["W"]).cuda(), False)
    ref = oracle.bitlinear(cfg["x"], packed.cpu().numpy(), s_w.cpu().numpy(), False, cfg["K"])
    for path in (bn.PATH_AUTO, bn.PATH_GEMV, bn.PATH_TC):
        for dtype in (torch.bfloat16, torch.float32):
            y = bn.bitnet_linear(bf16_tensor_from_bits(cfg["x"]), packed, s_w, False,
                                 out_dtype=dtype, path=path)
            _check_y(y, ref["y"], oracle, f"tiny path={path} {dtype}")


LINEAR_CASES = [  # (M, N, K, per_row)
    (1, 640, 2560, False), (1, 2560, 6912, True), (2, 130, 512, False), (3, 96, 64, True),
    (4, 6912, 2560, False), (6, 200, 1024, True), (8, 257, 512, False), (9, 129, 512, True),
    (31, 640, 2560, False), (64, 300, 512, True), (100, 256, 1024, False),
    (129, 131, 640, True), (300, 256, 512, False), (200, 640, 1024, True),
    (40, 300, 4096, True),  # split-K, ragged tokens and rows
    (4, 200, 4096, False), (8, 100, 2048, True),  # GEMV shared memory at exactly 48 KB dynamic
    # one or two tokens past two CTAs per SM at two rows per warp: four rows per warp
    (1, 17664, 2560, False), (2, 12000, 4096, True), (1, 9473, 512, True),
]


@pytest.mark.parametrize("M,N,K,per_row", LINEAR_CASES)
def test_linear_matches_oracle(bn, oracle, M, N, K, per_row):
    g = synth.rng(0, 95, M * 13 + N, K, synth.KIND_T)
    t = synth.ternary(N, K, g, 0.4)
    s_w = synth.uniform_scale(N if per_row else 1, g)
    x = synth.normal_x(M, K, g)
    x[M // 2] = 0  # one all-zero token -> y row exactly 0
    packed = _packed_dev(oracle, t)
    ref = oracle.bitlinear(x, packed.cpu().numpy(), s_w, per_row, K)
    paths = [bn.PATH_AUTO, bn.PATH_TC] + ([bn.PATH_GEMV] if M <= bn.GEMV_MAX_M else [])
    for path in paths:
        for dtype in (torch.bfloat16, torch.float32):
            y = _run_linear(bn, x, packed, s_w, per_row, dtype, path)
            _check_y(y, ref["y"], oracle, f"M={M} N={N} K={K} path={path} {dtype}")


def test_batch_equals_separate_calls(bn, oracle):
    """q/k/v of one hidden state in one batch call == three bitnet_linear calls, bit for bit."""
    K = 2560
    shapes = [2560, 640, 640]
    for M in (1, 5, 64, 300):
        g = synth.rng(0, 96, M, 0, synth.KIND_T)
        x = bf16_tensor_from_bits(synth.normal_x(M, K, g))
        projs = []
        for i, N in enumerate(shapes):
            t = synth.ternary(N, K, g, 0.4)
            per_row = i == 1
            s_w = torch.from_numpy(synth.uniform_scale(N if per_row else 1, g)).cuda()
            projs.append((_packed_dev(oracle, t), s_w, per_row))
        ys = bn.bitnet_linear_batch(x, projs)
        for (packed, s_w, per_row), y in zip(projs, ys):
            y1 = bn.bitnet_linear(x, packed, s_w, per_row)
            assert torch.equal(y.view(torch.int16), y1.view(torch.int16)), f"M={M}"


# ------------------------------------------------------------------------------- full sizes

@pytest.mark.parametrize("shape_idx", [0, 1, 2, 3])
def test_decode_sweep_full_size(bn, oracle, shape_idx):
    """Decode GEMV sweep workload at full size, M = 1: the whole output against the oracle."""
    c = synth.decode_case(shape_idx)
    packed = bn.bitnet_pack_ternary(torch.from_numpy(c["t"]).cuda())
    y = _run_linear(bn, c["x"], packed, c["s_w"], False, torch.bfloat16, bn.PATH_AUTO)
    ref = oracle.bitlinear(c["x"], packed.cpu().numpy(), c["s_w"], False, c["K"])
    assert_bf16_within_1ulp(bits_from_bf16_tensor(y), ref["y"], oracle, f"decode {shape_idx}")


@pytest.mark.parametrize("shape_idx", [0, 1, 2, 3])
@pytest.mark.parametrize("M", [512, 2048])
def test_prefill_full_size_sampled(bn, oracle, shape_idx, M):
    """Prefill GEMM workload at full size: every token on 48 sampled output columns."""
    c = synth.prefill_case(shape_idx, M)
    packed = bn.bitnet_pack_ternary(torch.from_numpy(c["t"]).cuda())
    y = _run_linear(bn, c["x"], packed, c["s_w"], False, torch.bfloat16, bn.PATH_AUTO)
    g = np.random.default_rng(shape_idx * 10 + M)
    n_idx = np.unique(np.concatenate([[0, c["N"] - 1], g.choice(c["N"], 46, replace=False)]))
    m_idx = np.arange(M)
    ref = oracle.bitlinear_sampled(c["x"], packed.cpu().numpy(), c["s_w"], False, c["K"],
                                   m_idx, n_idx)
    got = bits_from_bf16_tensor(y)[np.ix_(m_idx, n_idx)]
    assert_bf16_within_1ulp(got, ref["y"], oracle, f"prefill {shape_idx} M={M}")


def test_8b_stack_projection_sampled(bn, oracle):
    """8B-class down projection (4096 x 14336) from latent weights, per-row scale, M = 128."""
    W = synth.stack8b_latent(0, "down")
    packed, s_w = bn.bitnet_pack_weights(torch.from_numpy(W).cuda(), True)
    x = synth.stack8b_x(128, 14336)
    y = _run_linear(bn, x, packed, s_w.cpu().numpy(), True, torch.bfloat16, bn.PATH_AUTO)
    n_idx = np.array([0, 1, 77, 2048, 4095])
    m_idx = np.array([0, 1, 64, 127])
    ref = oracle.bitlinear_sampled(x, packed.cpu().numpy(), s_w.cpu().numpy(), True, 14336,
                                   m_idx, n_idx)
    got = bits_from_bf16_tensor(y)[np.ix_(m_idx, n_idx)]
    assert_bf16_within_1ulp(got, ref["y"], oracle, "8b down")


# One token and at least 12 MiB of packed weights per call: the streaming GEMV (producer warp,
# shared-memory ring of 16-row stages; the grid-stride GEMV takes only SwiGLU calls, tested in
# test_gpu_swiglu). Ragged projections (N not a multiple of 16), every chunks-per-lane class,
# per-row scales, fp32 output, whole outputs against the oracle.
STREAM_CASES = [  # (Ns of the batch, K, per_row, kernel)
    ((2560, 640, 640, 6912, 6912, 2560, 2560), 2560, False, "stream"),  # 2B-4T projections
    ((4096, 14336 + 7), 4096, True, "stream"),    # ragged last rows
    ((4096,), 14336, True, "stream"),             # 8B down projection, K = 14336
    ((9001,), 6912, False, "stream"),             # 4 chunks per lane, ragged
    ((3000, 50011), 1024, True, "stream"),        # 1 chunk per lane
]


@pytest.mark.parametrize("Ns,K,per_row,kernel", STREAM_CASES)
def test_stream_gemv_matches_oracle(bn, oracle, Ns, K, per_row, kernel):
    assert sum(Ns) * K // 4 >= 12 << 20
    want = bn.KERNEL_GS if kernel == "gs" else bn.KERNEL_STREAM
    assert bn.bitnet_linear_plan(1, K, list(Ns))["kernel"] == want
    g = synth.rng(0, 99, len(Ns), K, synth.KIND_T)
    x = synth.normal_x(1, K, g)
    projs, refs = [], []
    for N in Ns:
        t = synth.ternary(N, K, g, 0.4)
        s_w = synth.uniform_scale(N if per_row else 1, g)
        packed = _packed_dev(oracle, t)
        projs.append((packed, torch.from_numpy(s_w).cuda(), per_row))
        refs.append(oracle.bitlinear(x, packed.cpu().numpy(), s_w, per_row, K)["y"])
    xd = bf16_tensor_from_bits(x)
    for dtype in (torch.bfloat16, torch.float32):
        ys = bn.bitnet_linear_batch(xd, projs, out_dtype=dtype)
        for y, ref, N in zip(ys, refs, Ns):
            _check_y(y, ref, oracle, f"stream N={N} K={K} {dtype}")


def test_stream_gemv_i32_contraction(bn, oracle):
    """The contraction-only call keeps the register-resident kernel (no quantiser there)."""
    N, K = 6000, 4096
    g = synth.rng(0, 99, 7, K, synth.KIND_T)
    t = synth.ternary(N, K, g, 0.4)
    q = g.integers(-127, 128, size=(1, K)).astype(np.int8)
    packed = _packed_dev(oracle, t)
    acc = bn.bitnet_linear_i32(torch.from_numpy(q).cuda(), packed, path=bn.PATH_GEMV)
    assert np.array_equal(acc.cpu().numpy(), oracle.ternary_matmul(q, t))
