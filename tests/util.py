"""Comparison helpers shared by the GPU parity tests (no method arithmetic here)."""
import numpy as np
import torch


def bf16_ordered(bits: np.ndarray) -> np.ndarray:
    """Maps bf16 bit patterns to integers whose difference counts representable steps."""
    b = bits.astype(np.int32)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def assert_bf16_within_1ulp(got_bits: np.ndarray, y64: np.ndarray, oracle, where=""):
    """GPU bf16 output vs RNE(exact fp64 result): at most one bf16 step apart, zero exact."""
    want = oracle.round_bf16(y64)
    d = np.abs(bf16_ordered(got_bits) - bf16_ordered(want))
    bad = np.argwhere(d > 1)
    assert bad.size == 0, f"{where}: {bad.shape[0]} outputs beyond 1 bf16 ulp, first at {bad[0]}"
    zero = y64 == 0
    assert np.all(got_bits[zero] & 0x7FFF == 0), f"{where}: non-zero output where acc == 0"


def assert_f32_rel(got: np.ndarray, y64: np.ndarray, rel=1e-6, where=""):
    err = np.abs(got.astype(np.float64) - y64)
    lim = rel * np.abs(y64)
    bad = np.argwhere(err > lim)
    assert bad.size == 0, (f"{where}: {bad.shape[0]} fp32 outputs beyond rel {rel}; worst "
                           f"{(err / np.maximum(np.abs(y64), 1e-300)).max():.3e}")


def bf16_tensor_from_bits(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(bits.view(np.int16).copy()).to(device).view(torch.bfloat16)


def bits_from_bf16_tensor(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
