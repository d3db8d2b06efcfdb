"""Host checks of the integer identities the GEMV kernels rely on (no GPU, no oracle): the
arithmetic is restated in numpy from its definition and compared with the plain sum, on random
and extreme inputs, so a mistake in the reasoning behind a kernel shows up without a device.

1. Code offset: sum_k q t = sum_k q c - sum_k q with c = t + 1 (all kernels).
2. Masked codes: for a packed word w whose byte j holds four 2-bit codes, the codes at bits
   2i..2i+1 masked in place are c * 4^i; a dp4a of those unsigned bytes against signed q
   bytes gives 4^i * sum c q, and an arithmetic shift right by 2i recovers the sum exactly,
   also when it is negative (code_dot_acc / code_dot_total in the one-token GEMVs).
"""
import numpy as np


def _dp4a_u8s8(a_words, b_words):
    """sum_j u8(a_j) * s8(b_j) per 32-bit word, as int64."""
    a = a_words.astype(np.uint32).view(np.uint8).reshape(-1, 4).astype(np.int64)
    b = b_words.astype(np.uint32).view(np.int8).reshape(-1, 4).astype(np.int64)
    return (a * b).sum(axis=1)


def test_code_offset_identity():
    g = np.random.default_rng(1)
    t = g.integers(-1, 2, size=(7, 256))
    q = g.integers(-127, 128, size=(7, 256))
    assert np.array_equal((q * t).sum(1), (q * (t + 1)).sum(1) - q.sum(1))


def test_masked_code_dot_equals_shifted_dot():
    g = np.random.default_rng(2)
    n = 4096
    codes = g.integers(0, 3, size=(n, 4, 4))          # word, byte j, position i
    words = (codes * (4 ** np.arange(4))).sum(axis=2)  # byte j = sum_i c_ji 4^i
    words = (words * (256 ** np.arange(4))).sum(axis=1).astype(np.uint32)
    q = g.integers(-128, 128, size=(n, 4, 4))          # q for (byte j, position i)
    q[0] = -128                                        # extreme values
    q[1] = 127
    codes[0] = 2
    words[0] = np.uint32(0xAAAAAAAA)
    for i in range(4):
        q_words = (q[:, :, i].astype(np.int64) & 0xFF)
        q_words = (q_words * (256 ** np.arange(4))).sum(axis=1).astype(np.uint32)
        masked = words & np.uint32(0x03030303 << (2 * i))
        shifted = (words >> np.uint32(2 * i)) & np.uint32(0x03030303)
        scaled = _dp4a_u8s8(masked, q_words)
        plain = _dp4a_u8s8(shifted, q_words)
        assert np.array_equal(scaled, plain * 4 ** i)
        # accumulate over many words (a lane's share of a row) and shift back
        acc = np.cumsum(scaled).astype(np.int32)
        assert np.array_equal(acc.astype(np.int64) >> (2 * i), np.cumsum(plain))
        assert np.array_equal(plain, (codes[:, :, i] * q[:, :, i]).sum(axis=1))
