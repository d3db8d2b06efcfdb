"""GPU parity of the GEMV on warp-level tensor-core MMA (up to 8 tokens; BITNET_PATH_MMA forces
it, and the automatic choice takes it for the sizes where it measured fastest) against the
CPU oracle.

The kernel gives each CTA 1, 2, 4 or 8 tiles of 16 weight rows and splits each tile's K range
over 8, 4, 2 or 1 warps, whose lanes take packed chunks t, t + 4, ... of their slice; the
tokens are the MMA's 8 columns. The cases span every tile count the planner picks, K slices
that leave some lanes without a chunk (K = 64, 1088), rows of 40 / 64 / 108 / 224 chunks
(K = 2560 / 4096 / 6912 / 14336), row counts that leave the last tile part-full, batches whose
projection boundaries fall inside a tile, 1 to 8 tokens, and the SwiGLU variant. Bars as in
test_gpu_parity: int32 accumulators bit-exact, bf16 within one step of the exact value (zero
where acc = 0), fp32 within 1e-6 relative; SwiGLU within the derived bound and bit-equal to the
tensor-core path (same arithmetic).
"""
import numpy as np
import pytest
import torch

import synth
from util import (assert_bf16_within_1ulp, assert_f32_rel, assert_swiglu_within_bound,
                  bf16_tensor_from_bits, bits_from_bf16_tensor)

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


def _dev(a):
    return torch.from_numpy(a).cuda()


def _check_y(y, ref_y, oracle, where):
    if y.dtype == torch.bfloat16:
        assert_bf16_within_1ulp(bits_from_bf16_tensor(y), ref_y, oracle, where)
    else:
        assert_f32_rel(y.cpu().numpy(), ref_y, where=where)


DECODE_CASES = [  # (Ns of the batch, K, per_row)
    ((1,), 64, False),                 # one row of one chunk
    ((37,), 512, True),                # 8 chunks per row: four rows per slot
    ((2560,), 2560, False),            # q / o projection of the 2B-4T model
    ((640,), 2560, True),              # k / v
    ((6912,), 2560, False),            # gate / up
    ((2560,), 6912, True),             # down
    ((1001,), 4096, False),            # 64 chunks per row, ragged last warp
    ((333,), 14336, True),             # 224 chunks per row
    ((2560, 640, 640), 2560, False),   # q/k/v batch: boundaries inside warps
    ((7, 100, 13, 250), 1088, True),   # 17 chunks per row, tiny projections
    ((40000,), 512, False),            # 32 rows per warp (the cap): more CTAs than SMs
]


@pytest.mark.parametrize("Ns,K,per_row", DECODE_CASES)
def test_decode_gemv_matches_oracle(bn, oracle, Ns, K, per_row):
    plan = bn.bitnet_linear_plan(1, K, list(Ns), path=bn.PATH_MMA)
    assert plan["kernel"] == bn.KERNEL_MMA_GEMV, plan
    _decode_case(bn, oracle, 1, Ns, K, per_row, bn.PATH_MMA)


@pytest.mark.parametrize("M", [2, 3, 4, 5, 8])
@pytest.mark.parametrize("Ns,K,per_row", [((2560,), 2560, False), ((300, 77), 4096, True),
                                          ((1001,), 6912, False), ((48,), 64, True)])
def test_decode_gemv_several_tokens(bn, oracle, M, Ns, K, per_row):
    plan = bn.bitnet_linear_plan(M, K, list(Ns), path=bn.PATH_MMA)
    assert plan["kernel"] == bn.KERNEL_MMA_GEMV, plan
    _decode_case(bn, oracle, M, Ns, K, per_row, bn.PATH_MMA)


def _decode_case(bn, oracle, M, Ns, K, per_row, path):
    g = synth.rng(0, 98, len(Ns) * 31 + sum(Ns) + 1000 * M, K, synth.KIND_T)
    x = synth.normal_x(M, K, g)
    if M > 2:
        x[M // 2] = 0  # an all-zero token among others
    projs, refs = [], []
    for N in Ns:
        t = synth.ternary(N, K, g, 0.4)
        s_w = synth.uniform_scale(N if per_row else 1, g)
        packed = oracle.pack(t)
        projs.append((_dev(packed), _dev(s_w), per_row))
        refs.append(oracle.bitlinear(x, packed, s_w, per_row, K)["y"])
    xd = bf16_tensor_from_bits(x)
    for dtype in (torch.bfloat16, torch.float32):
        ys = bn.bitnet_linear_batch(xd, projs, out_dtype=dtype, path=path)
        for y, ref, N in zip(ys, refs, Ns):
            _check_y(y, ref, oracle, f"decode M={M} N={N} K={K} {dtype}")
        if len(Ns) > 1:  # the batch equals separate calls bit for bit
            for (packed, s_w, pr), y in zip(projs, ys):
                y1 = bn.bitnet_linear(xd, packed, s_w, pr, out_dtype=dtype, path=path)
                assert torch.equal(y.view(torch.int16) if dtype == torch.bfloat16 else
                                   y.view(torch.int32),
                                   y1.view(torch.int16) if dtype == torch.bfloat16 else
                                   y1.view(torch.int32))


@pytest.mark.parametrize("M,N,K", [(1, 1, 64), (1, 300, 2560), (1, 77, 6912), (1, 33, 14336),
                                   (1, 5000, 1024), (4, 300, 2560), (8, 129, 4096)])
def test_decode_gemv_i32_bit_exact(bn, oracle, M, N, K):
    """The contraction alone (int8 q given), extreme values included."""
    g = synth.rng(0, 98, N + 7 * M, K, synth.KIND_X)
    q = g.integers(-128, 128, size=(M, K)).astype(np.int8)
    t = synth.ternary(N, K, g, 0.4)
    t[0, :] = -1
    if N > 1:
        q2 = np.full((M, K), -128, dtype=np.int8)
        t[1, :] = -1
    else:
        q2 = None
    packed = _dev(oracle.pack(t))
    for qq in (q, q2):
        if qq is None:
            continue
        acc = bn.bitnet_linear_i32(_dev(qq), packed, path=bn.PATH_MMA).cpu().numpy()
        ref = oracle.ternary_matmul(qq, t)
        assert np.array_equal(acc, ref), np.argwhere(acc != ref)[:5]


def test_decode_gemv_special_inputs(bn, oracle):
    """An all-zero token gives exact zeros; a token with one huge outlier quantises every
    other value to 0 or +-1 (a tie-heavy case); |x| = 1e-6 everywhere hits the eps clamp."""
    N, K = 700, 2560
    g = synth.rng(0, 98, 1, 2, synth.KIND_T)
    t = synth.ternary(N, K, g, 0.4)
    s_w = synth.uniform_scale(1, g)
    packed = oracle.pack(t)
    pd, sd = _dev(packed), _dev(s_w)
    x0 = np.zeros((1, K), dtype=np.uint16)
    y0 = bn.bitnet_linear(bf16_tensor_from_bits(x0), pd, sd, False)
    assert int(bits_from_bf16_tensor(y0).astype(np.int32).__and__(0x7FFF).max()) == 0
    xo = synth.normal_x(1, K, g)
    xo[0, 1234] = synth.to_bf16_bits(np.array([3.0e4], dtype=np.float32))[0]
    xe = synth.to_bf16_bits(np.full((1, K), 1e-6, dtype=np.float32) *
                            np.where(np.arange(K) % 3 == 0, -1, 1).astype(np.float32))
    for x in (xo, xe):
        y = bn.bitnet_linear(bf16_tensor_from_bits(x), pd, sd, False)
        ref = oracle.bitlinear(x, packed, s_w, False, K)
        assert_bf16_within_1ulp(bits_from_bf16_tensor(y), ref["y"], oracle, "special input")


def _mlp(M, I, K, per_row, seed):
    tg = synth.ternary(I, K, synth.rng(seed, 6, I, 4, synth.KIND_T), 0.4)
    tu = synth.ternary(I, K, synth.rng(seed, 6, I, 5, synth.KIND_T), 0.4)
    ns = I if per_row else 1
    sg = synth.uniform_scale(ns, synth.rng(seed, 6, I, 4, synth.KIND_SW))
    su = synth.uniform_scale(ns, synth.rng(seed, 6, I, 5, synth.KIND_SW), 1.5, 3.0)
    x = synth.normal_x(M, K, synth.rng(seed, 6, I + M, 0, synth.KIND_X))
    return x, tg, tu, sg, su


@pytest.mark.parametrize("M,I,K,per_row", [(1, 16, 64, False), (1, 48, 512, True),
                                           (1, 400, 2560, False), (1, 6912, 2560, True),
                                           (1, 1040, 6912, False), (3, 208, 4096, True),
                                           (8, 160, 2560, False)])
def test_decode_swiglu_matches_oracle(bn, oracle, M, I, K, per_row):
    plan = bn.bitnet_linear_plan(M, K, [2 * I], swiglu=True, path=bn.PATH_MMA)
    assert plan["kernel"] == bn.KERNEL_MMA_GEMV, plan
    x, tg, tu, sg, su = _mlp(M, I, K, per_row, 0)
    pg, pu = oracle.pack(tg), oracle.pack(tu)
    packed_gu, s_gu = bn.bitnet_interleave_gate_up(_dev(pg), _dev(sg), _dev(pu), _dev(su),
                                                   per_row)
    xd = bf16_tensor_from_bits(x)
    h = bn.bitnet_linear_swiglu(xd, packed_gu, s_gu, per_row, path=bn.PATH_MMA)
    torch.cuda.synchronize()
    ref = oracle.swiglu_gate_up(x, pg, sg, pu, su, per_row, K)
    assert_swiglu_within_bound(bits_from_bf16_tensor(h), ref, oracle, where=f"I={I} K={K}")
    h_tc = bn.bitnet_linear_swiglu(xd, packed_gu, s_gu, per_row, path=bn.PATH_TC)
    assert torch.equal(h.view(torch.int16), h_tc.view(torch.int16))


@pytest.mark.parametrize("path", ["auto", "mma"])
def test_decode_chain_of_calls(bn, oracle, path):
    """Back-to-back one-token calls on one stream, each reading the previous call's output
    (the dependent chain of a decode step): every output against the oracle."""
    pth = bn.PATH_AUTO if path == "auto" else bn.PATH_MMA
    K = 2560
    g = synth.rng(0, 98, 77, K, synth.KIND_T)
    ts = [synth.ternary(K, K, g, 0.4) for _ in range(4)]
    sws = [synth.uniform_scale(1, g) for _ in range(4)]
    x = synth.normal_x(1, K, g)
    cur = bf16_tensor_from_bits(x)
    outs = []
    for t, s in zip(ts, sws):
        cur = bn.bitnet_linear(cur, _dev(oracle.pack(t)), _dev(s), False, path=pth)
        outs.append(cur)
    torch.cuda.synchronize()
    xin = x
    for t, s, y in zip(ts, sws, outs):
        ref = oracle.bitlinear(xin, oracle.pack(t), s, False, K)
        got = bits_from_bf16_tensor(y)
        assert_bf16_within_1ulp(got, ref["y"], oracle, "chain")
        xin = got  # the next call reads exactly what this one wrote


def test_int_rate_probes_run_clean(bn):
    """The arithmetic rate probes behind the bench's int_rates launch, finish and leave the
    watchdog word clear."""
    out = torch.empty(16, dtype=torch.int32, device="cuda")
    for kind in (0, 1):
        assert bn.lib.bitnet_probe_int_rate(kind, 16, 256, out.data_ptr(),
                                            torch.cuda.current_stream().cuda_stream) == bn.OK
    torch.cuda.synchronize()
    assert bn.bitnet_check_device_errors() == 0
