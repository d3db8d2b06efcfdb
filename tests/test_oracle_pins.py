"""Pins of the CPU oracle against things other than itself.

Each test ties one oracle function to the pages (worked example, printed bit
order), to closed forms, to brute force on tiny inputs, or to an independent
library routine, chosen so that a dropped term, a flipped sign, a wrong index or
a transposed operand in the oracle fails at least one of them. No GPU needed.
"""
import itertools

import numpy as np
import pytest
import torch

import synth
from conftest import read_golden


# ---------------------------------------------------------------- weight quantiser

def _worked():
    g = read_golden("worked_example.txt")
    return {k: v for k, v in g.items()}


@pytest.mark.parametrize("per_row", [True, False])
def test_worked_example_scale_and_ternary(oracle, per_row):
    """The printed example of "BitNet 深度实战" §2.4: scale 0.8333, pre-clip, clamp."""
    g = _worked()
    W = np.array([[float(v) for v in g["weight"]]], dtype=np.float32)
    s = oracle.absmean_scale(W, per_row)
    assert s.shape == (1,)
    assert round(float(s[0]), 4) == float(g["scale"][0])
    # mean |W| = 5/6 exactly in real arithmetic; fp32 result within one ulp of it
    assert abs(float(s[0]) - 5.0 / 6.0) <= np.spacing(np.float32(5.0 / 6.0))
    t, r = oracle.ternarize(W, s, per_row, return_rounded=True)
    assert r[0].tolist() == [int(v) for v in g["pre_clip"]]
    assert t[0].tolist() == [int(v) for v in g["ternary"]]
    deq = (t[0].astype(np.float64) * float(s[0])).round(4)
    assert deq.tolist() == [float(v) for v in g["dequantized"]]


def test_ternarize_half_even_ties(oracle):
    """round() is half-to-even (torch.round): ties at 0.5, 1.5, 2.5 with scale exactly 1."""
    W = np.array([[0.5, -0.5, 1.5, -1.5, 1.0, 1.0, 1.0, 1.0],
                  [2.5, 0.5, 1.0, 0.0, 0.0, 0.0, 0.0, 0.0]], dtype=np.float32)
    s = oracle.absmean_scale(W, per_row=True)
    assert s.tolist() == [1.0, 0.5]  # (8/8) and (4/8)
    t, r = oracle.ternarize(W, s, True, return_rounded=True)
    # row 1: W / 0.5 = [5, 1, 2, 0, ...]
    assert r[0].tolist() == [0, 0, 2, -2, 1, 1, 1, 1]
    assert t[0].tolist() == [0, 0, 1, -1, 1, 1, 1, 1]
    assert r[1].tolist() == [5, 1, 2, 0, 0, 0, 0, 0]
    assert t[1].tolist() == [1, 1, 1, 0, 0, 0, 0, 0]
    W2 = np.array([[2.5, 0.5, 1.0, 0.0]], dtype=np.float32)  # scale 1: 2.5 -> 2 (even) -> 1
    s2 = oracle.absmean_scale(W2, True)
    assert s2.tolist() == [1.0]
    t2, r2 = oracle.ternarize(W2, s2, True, return_rounded=True)
    assert r2[0].tolist() == [2, 0, 1, 0] and t2[0].tolist() == [1, 0, 1, 0]


def test_absmean_eps_clamp(oracle):
    W = np.zeros((2, 8), dtype=np.float32)
    W[1, :] = 1e-7
    s = oracle.absmean_scale(W, True)
    assert s.tolist() == [np.float32(1e-5), np.float32(1e-5)]
    t = oracle.ternarize(W, s, True)
    assert not t.any()


def test_absmean_against_numpy_mean(oracle):
    """Per-row and per-tensor scales agree with numpy's fp64 mean to one fp32 rounding."""
    g = np.random.default_rng(7)
    W = (g.standard_normal((37, 96)) * g.uniform(0.01, 3, size=(37, 1))).astype(np.float32)
    s_row = oracle.absmean_scale(W, True)
    ref_row = np.abs(W.astype(np.float64)).mean(axis=1)
    assert np.all(np.abs(s_row - ref_row) <= np.spacing(ref_row.astype(np.float32)))
    s_t = oracle.absmean_scale(W, False)
    ref_t = np.abs(W.astype(np.float64)).mean()
    assert abs(float(s_t[0]) - ref_t) <= np.spacing(np.float32(ref_t))
    # per-row scale of row n must not depend on the other rows (index bug guard)
    s_row_sub = oracle.absmean_scale(W[5:9], True)
    assert np.array_equal(s_row_sub, s_row[5:9])


def test_ternarize_against_definition_by_interval(oracle):
    """t = +1 exactly when W/s >= 0.5 (ties to even: 0.5 -> 0), -1 when <= -0.5."""
    g = np.random.default_rng(3)
    W = g.standard_normal((16, 64)).astype(np.float32)
    s = oracle.absmean_scale(W, False)
    t = oracle.ternarize(W, s, False)
    ratio = W.astype(np.float64) / float(s[0])
    assert np.all(t[ratio > 0.5000001] == 1)
    assert np.all(t[ratio < -0.5000001] == -1)
    assert np.all(t[np.abs(ratio) < 0.4999999] == 0)
    # per-row with one row scaled by 8 gives the same ternary row (scale invariance)
    W2 = W.copy()
    W2[3] *= 8.0  # power of two: exact, so the row quantises identically
    t_row = oracle.ternarize(W, oracle.absmean_scale(W, True), True)
    t_row2 = oracle.ternarize(W2, oracle.absmean_scale(W2, True), True)
    assert np.array_equal(t_row, t_row2)


# ---------------------------------------------------------------- packing

def test_pack_worked_example_bytes(oracle):
    g = read_golden("pack_example.txt")
    t = np.array([[int(v) for v in g["ternary"]]], dtype=np.int8)
    p = oracle.pack(t)
    assert [f"0x{b:02x}" for b in p[0]] == g["bytes"]
    assert oracle.unpack(p, 8)[0].tolist() == t[0].tolist()


def test_pack_bit_positions(oracle):
    """Weight i of a group of four sits in bits 2i..2i+1 with code t+1; others are 0 -> 01."""
    for i, w in itertools.product(range(4), (-1, 0, 1)):
        t = np.zeros((1, 4), dtype=np.int8)
        t[0, i] = w
        expect = 0x55 & ~(3 << (2 * i)) | ((w + 1) << (2 * i))
        assert int(oracle.pack(t)[0, 0]) == expect
    # the second byte holds weights 4..7 (K ordering across bytes)
    t = np.zeros((2, 8), dtype=np.int8)
    t[1, 5] = -1
    p = oracle.pack(t)
    assert p.tolist() == [[0x55, 0x55], [0x55, 0x51]]


def test_pack_roundtrip_and_code_range(oracle):
    g = np.random.default_rng(11)
    t = g.integers(-1, 2, size=(23, 128)).astype(np.int8)
    p = oracle.pack(t)
    assert p.shape == (23, 32)
    codes = np.stack([(p >> (2 * i)) & 3 for i in range(4)])
    assert codes.max() <= 2  # code 3 never produced
    assert np.array_equal(oracle.unpack(p, 128), t)


def test_unpack_rejects_code3_and_pack_rejects_bad_weight(oracle):
    with pytest.raises(oracle.OracleError):
        oracle.unpack(np.array([[0xC0]], dtype=np.uint8), 4)
    with pytest.raises(oracle.OracleError):
        oracle.pack(np.array([[0, 2, 0, 0]], dtype=np.int8))


# ---------------------------------------------------------------- activation quantiser

def test_quant_act_hand_example(oracle):
    """amax = 1 -> s_x = 127; x*127 is exact in fp32 for these values, so q = rint(127 x)
    with ties to even: -63.5 -> -64, 63.5 -> 64, 31.75 -> 32, 15.875 -> 16."""
    xs = np.array([[1.0, -0.5, 0.25, 0.0, 0.75, -1.0, 0.125, 0.5]], dtype=np.float32)
    q, s = oracle.quant_act(synth.to_bf16_bits(xs))
    assert s.tolist() == [127.0]
    assert q[0].tolist() == [127, -64, 32, 0, 95, -127, 16, 64]


def test_quant_act_invariants(oracle):
    g = np.random.default_rng(5)
    x = synth.to_bf16_bits(g.standard_normal((9, 256)).astype(np.float32)
                           * g.uniform(1e-3, 50, size=(9, 1)).astype(np.float32))
    x[4] = 0  # an all-zero token
    q, s = oracle.quant_act(x)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    assert np.abs(q.astype(int)).max() <= 127
    for m in range(9):
        if m == 4:
            assert not q[m].any() and s[m] == np.float32(127.0) / np.float32(1e-5)
            continue
        amax = np.abs(xf[m]).max()
        assert np.abs(q[m].astype(int)).max() == 127
        assert s[m] == np.float32(127.0) / np.float32(amax)
        # q is the nearest integer to x*s_x: error at most half a step (+ one fp32 rounding)
        err = np.abs(q[m] - xf[m] * float(s[m]))
        assert err.max() <= 0.5 + 127 * 2.0 ** -23
        # the token's row does not leak into another token (index bug guard)
        q1, s1 = oracle.quant_act(x[m:m + 1])
        assert np.array_equal(q1[0], q[m]) and s1[0] == s[m]
    # x -> -x gives q -> -q with the same scale
    qn, sn = oracle.quant_act(x ^ np.uint16(0x8000))
    assert np.array_equal(qn, -q) and np.array_equal(sn, s)


# ---------------------------------------------------------------- contraction

@pytest.mark.parametrize("M,N,K", [(1, 1, 4), (3, 5, 8), (8, 16, 64), (5, 2, 12), (2, 7, 40)])
def test_ternary_matmul_brute_force(oracle, M, N, K):
    """add/sub/skip loop == dense int64 matmul (numpy) on tiny non-square shapes."""
    g = np.random.default_rng(M * 100 + N * 10 + K)
    q = g.integers(-128, 128, size=(M, K)).astype(np.int8)
    t = g.integers(-1, 2, size=(N, K)).astype(np.int8)
    acc = oracle.ternary_matmul(q, t)
    ref = q.astype(np.int64) @ t.astype(np.int64).T
    assert acc.shape == (M, N)
    assert np.array_equal(acc.astype(np.int64), ref)


def test_ternary_matmul_exhaustive_tiny(oracle):
    """Every ternary row of length 3 against a fixed int8 row set."""
    rows = np.array(list(itertools.product((-1, 0, 1), repeat=3)), dtype=np.int8)
    q = np.array([[127, -128, 5], [-7, 0, 99]], dtype=np.int8)
    acc = oracle.ternary_matmul(q, rows)
    for n, w in enumerate(rows):
        for m in range(2):
            assert acc[m, n] == sum(int(q[m, k]) * int(w[k]) for k in range(3))


def test_ternary_matmul_closed_forms(oracle):
    g = np.random.default_rng(9)
    q = g.integers(-127, 128, size=(4, 32)).astype(np.int8)
    rs = q.astype(np.int64).sum(axis=1)
    assert np.array_equal(oracle.ternary_matmul(q, np.ones((3, 32), np.int8)),
                          np.repeat(rs[:, None], 3, axis=1))
    assert np.array_equal(oracle.ternary_matmul(q, -np.ones((3, 32), np.int8)),
                          -np.repeat(rs[:, None], 3, axis=1))
    assert not oracle.ternary_matmul(q, np.zeros((3, 32), np.int8)).any()
    eye = np.eye(32, dtype=np.int8)[:6]  # t[n, k] = [k == n] selects activation column n
    assert np.array_equal(oracle.ternary_matmul(q, eye), q[:, :6].astype(np.int32))


def test_ternary_matmul_extreme_accumulator(oracle):
    """|acc| reaches 128*K without overflow at the largest K in the workloads."""
    K = 14336
    q = np.full((1, K), -128, dtype=np.int8)
    t = -np.ones((1, K), dtype=np.int8)
    assert oracle.ternary_matmul(q, t)[0, 0] == 128 * K


# ---------------------------------------------------------------- dequant and rounding

def test_dequant_matches_float_linear(oracle):
    """y equals the float form linear(q / s_x, t * s_w) of "BitNet 深度实战" §3.2 in fp64."""
    g = np.random.default_rng(2)
    M, N, K = 3, 6, 64
    q = g.integers(-127, 128, size=(M, K)).astype(np.int8)
    t = g.integers(-1, 2, size=(N, K)).astype(np.int8)
    s_x = g.uniform(1, 100, size=M).astype(np.float32)
    for per_row in (False, True):
        s_w = g.uniform(0.5, 2, size=N if per_row else 1).astype(np.float32)
        y = oracle.dequant(oracle.ternary_matmul(q, t), s_x, s_w, per_row)
        sw = s_w.astype(np.float64) if per_row else np.full(N, float(s_w[0]))
        ref = (q / s_x.astype(np.float64)[:, None]) @ (t * sw[:, None]).T
        np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_round_bf16_matches_torch_for_fp32_values(oracle):
    g = np.random.default_rng(4)
    f = np.concatenate([g.standard_normal(20000).astype(np.float32) * 1e3,
                        g.standard_normal(2000).astype(np.float32) * 1e-38,  # subnormal range
                        np.array([0.0, -0.0, 3.3e38, -3.3e38, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8],
                                 dtype=np.float32)])
    # ties: values exactly halfway between bf16 neighbours
    ties = ((g.integers(0, 2 ** 15, size=5000).astype(np.uint32) << 16) | 0x8000).view(np.float32)
    f = np.concatenate([f, ties[np.isfinite(ties)]])
    ours = oracle.round_bf16(f.astype(np.float64))
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_round_bf16_no_double_rounding(oracle):
    # 1 + 2^-8 + 2^-30 lies above the tie 1 + 2^-8: nearest bf16 is 1 + 2^-7. Going through
    # fp32 first would land on the tie and round to 1.0.
    v = np.array([1.0 + 2.0 ** -8 + 2.0 ** -30, -(1.0 + 2.0 ** -8 + 2.0 ** -30)])
    out = oracle.round_bf16(v)
    assert out.tolist() == [0x3F81, 0xBF81]


# ---------------------------------------------------------------- composite forward

def test_bitlinear_composite_and_sampled(oracle):
    cfg = synth.tiny(0)
    packed, s_w = oracle.pack_weights(cfg["W"], cfg["per_row"])
    K = cfg["K"]
    full = oracle.bitlinear(cfg["x"], packed, s_w, cfg["per_row"], K)
    assert full["y"].shape == (4, 256)
    # composite equals the product of its parts
    t = oracle.unpack(packed, K)
    q, s_x = oracle.quant_act(cfg["x"])
    ref = (q / s_x.astype(np.float64)[:, None]) @ (t.astype(np.float64) * float(s_w[0])).T
    np.testing.assert_allclose(full["y"], ref, rtol=1e-12, atol=1e-12)
    # sampled forward agrees with the full one on its sample
    m_idx, n_idx = np.array([3, 0]), np.array([255, 7, 128])
    smp = oracle.bitlinear_sampled(cfg["x"], packed, s_w, cfg["per_row"], K, m_idx, n_idx)
    assert np.array_equal(smp["y"], full["y"][np.ix_(m_idx, n_idx)])
    assert np.array_equal(smp["acc"], full["acc"][np.ix_(m_idx, n_idx)])
    assert np.array_equal(smp["q"], full["q"][m_idx])
    # the float product with the latent weights is close (quantisation error only)
    xf = synth.bf16_bits_to_f32(cfg["x"]).astype(np.float64)
    dense = xf @ cfg["W"].astype(np.float64).T
    assert np.corrcoef(dense.ravel(), full["y"].ravel())[0, 1] > 0.8


# ---------------------------------------------------------------- SwiGLU (MLP gate/up)
# Independent exact arithmetic for the pins below: Fractions for rational steps, Decimal
# at 50 digits for e^-z, and RNE to bf16 by integer scaling (not the oracle's frexp route).
from decimal import Decimal, getcontext
from fractions import Fraction


def _bf16_value(bits: int) -> Fraction:
    sign = -1 if bits & 0x8000 else 1
    e = (bits >> 7) & 0xFF
    m = bits & 0x7F
    if e == 0:
        return sign * Fraction(m, 1 << 133)  # subnormal: m * 2^-133
    return sign * Fraction(128 + m, 128) * Fraction(2) ** (e - 127)


def _rne_bf16(v: Fraction) -> int:
    """Exact round-half-even of a rational to bf16 bits (finite range only)."""
    if v == 0:
        return 0x0000
    sign = 0x8000 if v < 0 else 0
    a = abs(v)
    e = a.numerator.bit_length() - a.denominator.bit_length()  # 2^e <= a < 2^(e+2)
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    q_exp = max(e, -126) - 7  # quantum: 8 significant bits, or 2^-133 below the normals
    scaled = a / Fraction(2) ** q_exp
    n = scaled.numerator // scaled.denominator
    rem = scaled - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    r = n * Fraction(2) ** q_exp
    if r == 0:
        return sign
    if r >= Fraction(2) ** -126:
        e2 = r.numerator.bit_length() - r.denominator.bit_length()
        while Fraction(2) ** e2 > r:
            e2 -= 1
        while Fraction(2) ** (e2 + 1) <= r:
            e2 += 1
        mant = int(r / Fraction(2) ** (e2 - 7)) - 128
        assert e2 + 127 < 255, "overflow is outside these pins"
        return sign | ((e2 + 127) << 7) | mant
    return sign | int(r * (1 << 133))


def _silu_exact_bf16(g_bits: int) -> int:
    getcontext().prec = 50
    z = _bf16_value(g_bits)
    ez = (-Decimal(z.numerator) / Decimal(z.denominator)).exp()
    silu = z / (1 + Fraction(ez))
    return _rne_bf16(silu)


def test_rne_bf16_helper_matches_torch():
    """The pins' own rounding helper agrees with torch's fp32 -> bf16 RNE on fp32 values."""
    vals = np.array([1.0, 1.00390625, 1.005859375, 1.001953125, -3.0e-39, 2.5e-40, 0.1,
                     -123.456, 65504.0, 1e-30], dtype=np.float32)
    got = [_rne_bf16(Fraction(float(v))) for v in vals]
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    assert got == ref.tolist()


def test_swiglu_silu_exact_over_bf16_grid(oracle):
    """silu rounded to bf16 equals the exactly rounded value (50-digit exp) on a spread of
    bf16 inputs: every exponent from 2^-20 to 2^7, both signs, several mantissas."""
    bits = []
    for e in range(127 - 20, 127 + 7):
        for m in (0, 1, 37, 64, 100, 127):
            for sign in (0, 0x8000):
                bits.append(sign | (e << 7) | m)
    g = np.array(bits, dtype=np.uint16)
    u = np.full(g.shape, 0x3F80, dtype=np.uint16)  # u = 1: h = s
    s, h = oracle.swiglu(g, u)
    expect = [_silu_exact_bf16(int(b)) for b in bits]
    assert s.tolist() == expect
    assert h.tolist() == expect


def test_swiglu_closed_forms(oracle):
    """silu(0) = 0; silu(1) = 1/(1 + 1/e) = 0.7310585786 -> bf16 0.73046875; for z >= 16
    the relative deficit z e^-z is far below half a bf16 step, so silu(z) rounds to z; for
    z <= -100 |silu(z)| < 2^-134 (half the least bf16 subnormal) and rounds to -0."""
    g = np.array([0x0000, 0x3F80, 0x4180, 0x4300, 0x4780, 0xC2C8, 0xC47A], dtype=np.uint16)
    u = np.full(g.shape, 0x3F80, dtype=np.uint16)
    s, _ = oracle.swiglu(g, u)
    assert s[0] == 0x0000
    assert _bf16_value(int(s[1])) == Fraction(187, 256)  # 0.73046875
    assert s[2] == 0x4180 and s[3] == 0x4300 and s[4] == 0x4780  # 16, 128, 65536
    assert s[5] == 0x8000 and s[6] == 0x8000  # -100, -1000


def test_swiglu_product_rounding_and_operand_order(oracle):
    """h = bf16(s * u) with the exact product: u scales h; swapping g and u changes h
    (silu applies to the gate only); a tie in the product rounds to even."""
    rng = np.random.default_rng(5)
    g = synth.to_bf16_bits(rng.normal(0, 3, 400).astype(np.float32))
    u = synth.to_bf16_bits(rng.normal(0, 3, 400).astype(np.float32))
    s, h = oracle.swiglu(g, u)
    for i in range(400):
        assert int(h[i]) == _rne_bf16(_bf16_value(int(s[i])) * _bf16_value(int(u[i])))
    _, h_swapped = oracle.swiglu(u, g)
    assert np.count_nonzero(h_swapped != h) > 300
    # silu(3.125) = 2.9935 rounds to s = 3 exactly; s * u with u = 1 + 2^-7 is 3.0234375,
    # nine significant bits with a trailing 1: a tie between 3.015625 (odd last bit) and
    # 3.03125 (even), so h = 3.03125.
    _, h1 = oracle.swiglu(np.array([0x4048], dtype=np.uint16), np.array([0x3F81], dtype=np.uint16))
    assert _bf16_value(int(h1[0])) == Fraction(97, 32)


def test_swiglu_gate_up_end_to_end_exact(oracle):
    """Tiny MLP gate/up: the oracle's h equals an exact rational evaluation of the whole
    definition (quantiser, integer contraction, y = acc s_w / s_x, bf16 of g and u, silu,
    product), written here without the oracle's C code."""
    rng = np.random.default_rng(11)
    M, I, K = 3, 16, 64
    x = synth.to_bf16_bits(rng.normal(0, 1, (M, K)).astype(np.float32))
    tg = rng.integers(-1, 2, (I, K)).astype(np.int8)
    tu = rng.integers(-1, 2, (I, K)).astype(np.int8)
    sg = np.array([0.75], dtype=np.float32)
    su = np.array([1.25], dtype=np.float32)
    r = oracle.swiglu_gate_up(x, oracle.pack(tg), sg, oracle.pack(tu), su, False, K)
    xf = synth.bf16_bits_to_f32(x)
    for m in range(M):
        amax = float(np.max(np.abs(xf[m])))
        s_x = np.float32(127.0) / np.float32(max(amax, 1e-5))
        q = np.rint((xf[m] * s_x).astype(np.float32)).astype(np.int64)
        for n in range(I):
            ag = int(np.dot(q, tg[n].astype(np.int64)))
            au = int(np.dot(q, tu[n].astype(np.int64)))
            gb = _rne_bf16(Fraction(ag) * Fraction(float(sg[0])) / Fraction(float(s_x)))
            ub = _rne_bf16(Fraction(au) * Fraction(float(su[0])) / Fraction(float(s_x)))
            assert int(r["g_bits"][m, n]) == gb and int(r["u_bits"][m, n]) == ub
            sb = _silu_exact_bf16(gb)
            assert int(r["s_bits"][m, n]) == sb
            assert int(r["h_bits"][m, n]) == _rne_bf16(_bf16_value(sb) * _bf16_value(ub))


@pytest.mark.parametrize("per_row", [False, True])
def test_swiglu_gate_up_sampled_equals_full_on_its_sample(oracle, per_row):
    """The sampled MLP gate/up (used by the full-size GPU tests) against the whole-matrix
    form on a tiny MLP: every g, u, s and h of the sample must match exactly. The gate and
    up scales differ (per tensor and per row), and the sample has more outputs than tokens
    in an unsorted order, so swapped scales or a swapped token/output index fail here."""
    rng = np.random.default_rng(23)
    M, I, K = 5, 48, 128
    x = synth.to_bf16_bits(rng.normal(0, 1, (M, K)).astype(np.float32))
    tg = rng.integers(-1, 2, (I, K)).astype(np.int8)
    tu = rng.integers(-1, 2, (I, K)).astype(np.int8)
    if per_row:
        sg = rng.uniform(0.5, 2.0, I).astype(np.float32)
        su = rng.uniform(3.0, 5.0, I).astype(np.float32)
    else:
        sg = np.array([0.625], dtype=np.float32)
        su = np.array([3.5], dtype=np.float32)
    pg, pu = oracle.pack(tg), oracle.pack(tu)
    full = oracle.swiglu_gate_up(x, pg, sg, pu, su, per_row, K)
    m_idx, n_idx = np.array([4, 0, 2]), np.array([47, 3, 20, 0, 31, 9, 46])
    smp = oracle.swiglu_gate_up_sampled(x, pg, sg, pu, su, per_row, K, m_idx, n_idx)
    sel = np.ix_(m_idx, n_idx)
    for key in ("g", "u", "g_bits", "u_bits", "s_bits", "h_bits"):
        assert smp[key].shape == (3, 7), key
        assert np.array_equal(smp[key], full[key][sel]), key
    # the sample is not degenerate: gate and up differ, and h is not all zero
    assert not np.array_equal(smp["g_bits"], smp["u_bits"])
    assert np.count_nonzero(smp["h_bits"] & 0x7FFF) > 10


def test_swiglu_bound_helper_accepts_exact_and_rejects_far(oracle):
    """The GPU tests' SwiGLU bound: the oracle's own h passes; h moved 3 bf16 steps away
    from a value whose neighbourhood is flat fails."""
    from util import assert_swiglu_within_bound, bf16_from_ordered, bf16_ordered
    rng = np.random.default_rng(3)
    y_g = rng.normal(0, 4, (4, 64))
    y_u = rng.normal(0, 4, (4, 64))
    g_bits, u_bits = oracle.round_bf16(y_g), oracle.round_bf16(y_u)
    s_bits, h_bits = oracle.swiglu(g_bits, u_bits)
    ref = {"g": y_g, "u": y_u, "g_bits": g_bits, "u_bits": u_bits, "s_bits": s_bits,
           "h_bits": h_bits}
    assert_swiglu_within_bound(h_bits, ref, oracle)
    bad = h_bits.copy()
    bad[1, 5] = bf16_from_ordered(bf16_ordered(bad[1:2, 5:6]) + 40)[0, 0]
    with pytest.raises(AssertionError):
        assert_swiglu_within_bound(bad, ref, oracle)


# ---------------------------------------------------------------- per-tensor activation scale

def test_quant_per_tensor_hand_example(oracle):
    """x = [[1, -2], [4, 0.5]]: amax 4 over the whole tensor, s = 127/4 = 31.75, q = rint of
    [31.75, -63.5, 127, 15.875] = [32, -64 (tie to even), 127, 16]; both rows share s."""
    x = synth.to_bf16_bits(np.array([[1.0, -2.0], [4.0, 0.5]], dtype=np.float32))
    q, s = oracle.quant_act_per_tensor(x)
    assert s.tolist() == [31.75, 31.75]
    assert q.tolist() == [[32, -64], [127, 16]]
    q_tok, s_tok = oracle.quant_act(x)  # per token the first row has its own scale 63.5
    assert s_tok.tolist() == [63.5, 31.75] and q_tok[0].tolist() == [64, -127]


def test_quant_per_tensor_reduces_and_invariants(oracle):
    """One token: per tensor is per token. Many: |q| <= 127 with max |q| = 127 once over the
    tensor, the row holding the global amax equals its per-token quantisation, rows permute
    with q, scaling x by 2 (exact) leaves q unchanged, and an all-zero x gives q = 0."""
    rng = np.random.default_rng(21)
    x1 = synth.to_bf16_bits(rng.normal(0, 1, (1, 640)).astype(np.float32))
    assert all(np.array_equal(a, b) for a, b in zip(oracle.quant_act_per_tensor(x1),
                                                    oracle.quant_act(x1)))
    xf = rng.normal(0, 1, (7, 256)).astype(np.float32)
    xf[3] *= 5.0
    x = synth.to_bf16_bits(xf)
    q, s = oracle.quant_act_per_tensor(x)
    assert np.all(s == s[0]) and np.abs(q).max() == 127 and np.abs(q.astype(int)).max() <= 127
    r = int(np.argmax(np.abs(synth.bf16_bits_to_f32(x)).max(axis=1)))
    q_tok, _ = oracle.quant_act(x)
    assert np.array_equal(q[r], q_tok[r])
    assert np.abs(q[(r + 1) % 7]).max() < 127  # other rows use the larger common scale
    perm = rng.permutation(7)
    assert np.array_equal(oracle.quant_act_per_tensor(np.ascontiguousarray(x[perm]))[0], q[perm])
    x2 = synth.to_bf16_bits(synth.bf16_bits_to_f32(x) * np.float32(2.0))
    q2, s2 = oracle.quant_act_per_tensor(x2)
    assert np.array_equal(q2, q) and s2[0] == s[0] / 2
    qz, sz = oracle.quant_act_per_tensor(np.zeros((3, 64), dtype=np.uint16))
    assert not qz.any() and sz[0] == np.float32(127.0) / np.float32(1e-5)


def test_bitlinear_per_tensor_act_matches_float_linear(oracle):
    """The forward with a per-tensor activation scale equals linear(q / s_x, t * s_w) in fp64
    ("BitNet 深度实战" §3.2), and its sampled form equals the full one on the sample."""
    rng = np.random.default_rng(22)
    M, N, K = 5, 24, 128
    x = synth.to_bf16_bits(rng.normal(0, 1, (M, K)).astype(np.float32))
    t = rng.integers(-1, 2, (N, K)).astype(np.int8)
    s_w = rng.uniform(0.5, 2, N).astype(np.float32)
    r = oracle.bitlinear(x, oracle.pack(t), s_w, True, K, act_per_tensor=True)
    q, s = oracle.quant_act_per_tensor(x)
    ref = (q.astype(np.float64) / s.astype(np.float64)[:, None]) @ \
          (t.astype(np.float64) * s_w.astype(np.float64)[:, None]).T
    np.testing.assert_allclose(r["y"], ref, rtol=1e-12, atol=1e-12)
    m_idx, n_idx = np.array([0, 3, 4]), np.array([1, 7, 23])
    rs = oracle.bitlinear_sampled_per_tensor_act(x, oracle.pack(t), s_w, True, K, m_idx, n_idx)
    assert np.array_equal(rs["y"], r["y"][np.ix_(m_idx, n_idx)])


# ---------------------------------------------------------------- base-3 packing (5 per byte)

def test_pack_b3_hand_derived_bytes(oracle):
    """The fixture's row (K = 80) packs to the bytes derived by hand from the layout."""
    g = read_golden("pack_b3_example.txt")
    t = np.zeros((1, 80), dtype=np.int8)
    t[0, [int(v) for v in g["neg"]]] = -1
    t[0, [int(v) for v in g["pos"]]] = 1
    want = np.array([int(v) for v in g["bytes"]], dtype=np.uint8)
    assert np.array_equal(oracle.pack_b3(t)[0], want)


def test_pack_b3_digit_places(oracle):
    """Each weight of a chunk moves its byte by 3^d in its own byte only: weight k = 16d + p of
    chunk c sets digit d of byte 16c + p."""
    K = 160
    base = oracle.pack_b3(np.zeros((1, K), dtype=np.int8))[0].astype(np.int64)
    assert np.all(base == 121)
    for k in (0, 15, 16, 37, 79, 80, 101, 159):
        c, r = divmod(k, 80)
        d, p = divmod(r, 16)
        for w, delta in ((1, 1), (-1, -1)):
            t = np.zeros((1, K), dtype=np.int8)
            t[0, k] = w
            got = oracle.pack_b3(t)[0].astype(np.int64) - base
            want = np.zeros_like(got)
            want[16 * c + p] = delta * 3 ** d
            assert np.array_equal(got, want), (k, w)


@pytest.mark.parametrize("K", [64, 80, 100, 2560, 4096, 6912])
def test_pack_b3_roundtrip_and_range(oracle, K):
    g = np.random.default_rng(K)
    t = g.integers(-1, 2, size=(7, K)).astype(np.int8)
    p = oracle.pack_b3(t)
    assert p.shape == (7, 16 * ((K + 79) // 80)) and int(p.max()) <= 242
    assert np.array_equal(oracle.unpack_b3(p, K), t)
    # 1.6 bits per weight, up to the padding of the last chunk
    assert p.shape[1] * 8 <= 1.6 * K + 16 * 8


def test_unpack_b3_rejects_bad_bytes_and_padding(oracle):
    t = np.zeros((1, 64), dtype=np.int8)
    p = oracle.pack_b3(t)
    bad = p.copy()
    bad[0, 3] = 243  # no five base-3 digits
    with pytest.raises(oracle.OracleError):
        oracle.unpack_b3(bad, 64)
    pad = p.copy()
    pad[0, 0] = 121 + 81  # digit 4 of byte 0 is weight k = 64, past K = 64: must stay 0
    with pytest.raises(oracle.OracleError):
        oracle.unpack_b3(pad, 64)
    with pytest.raises(oracle.OracleError):
        oracle.pack_b3(np.full((1, 64), 2, dtype=np.int8))


# ---------------------------------------------------------------- SwiGLU -> down hand-off

def test_block_absmax_hand_example(oracle):
    """Two blocks of 16: block 0 holds -3.0 (bf16 0xC040 -> |x| = 0x4040), block 1 holds
    0.5 as its largest magnitude next to -0.25 (0x3F00); sign and position do not matter."""
    xs = np.zeros((2, 32), dtype=np.float32)
    xs[0, 3], xs[0, 15], xs[0, 20], xs[0, 31] = 1.0, -3.0, 0.5, -0.25
    xs[1, 16] = -0.0
    xs[1, 0] = 2.0 ** -130  # a subnormal bf16 still orders as its magnitude
    got = oracle.block_absmax_bits(synth.to_bf16_bits(xs))
    assert got.dtype == np.uint16 and got.shape == (2, 2)
    assert got[0].tolist() == [0x4040, 0x3F00]
    assert got[1].tolist() == [int(synth.to_bf16_bits(np.array([2.0 ** -130], np.float32))[0]), 0]


def test_block_absmax_brute_force_and_quant_scale(oracle):
    """Against a float loop over every block, and the maximum over a row's blocks gives the
    scale oracle.quant_act computes from the row (the quantiser's amax, reached two ways)."""
    g = np.random.default_rng(11)
    M, K = 5, 96
    x = synth.to_bf16_bits(g.standard_normal((M, K)).astype(np.float32)
                           * g.uniform(1e-3, 40, size=(M, 1)).astype(np.float32))
    x[2] = 0
    got = oracle.block_absmax_bits(x)
    xf = synth.bf16_bits_to_f32(x)
    for m in range(M):
        for b in range(K // 16):
            want = max(abs(float(v)) for v in xf[m, 16 * b:16 * b + 16])
            assert float(synth.bf16_bits_to_f32(got[m:m + 1, b:b + 1])[0, 0]) == want
    amax = synth.bf16_bits_to_f32(got.max(axis=1, keepdims=True))[:, 0]
    s_from_blocks = np.float32(127.0) / np.maximum(amax, np.float32(1e-5))
    _, s = oracle.quant_act(x)
    assert np.array_equal(s_from_blocks.astype(np.float32), s)
    with pytest.raises(ValueError):
        oracle.block_absmax_bits(x[:, :40])
