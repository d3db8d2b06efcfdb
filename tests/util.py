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


def bf16_from_ordered(k: np.ndarray) -> np.ndarray:
    """Inverse of bf16_ordered (negative zero maps to +0)."""
    k = k.astype(np.int32)
    return np.where(k < 0, 0x8000 | (-k), k).astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def assert_swiglu_within_bound(h_bits: np.ndarray, ref: dict, oracle, where="",
                               min_exact=0.99):
    """GPU SwiGLU output h against the oracle (``oracle.swiglu_gate_up``), with the bound
    that follows from the arithmetic: the GPU's g and u are each within one bf16 step of
    RNE(exact) (the BitLinear bar), and its binary32 silu rounded to bf16 is within one step
    of the exactly rounded silu of that g. So h = RNE(s * u) must lie in the hull of
    RNE(s' * u') over g' = g +- 1 step, u' = u +- 1 step, s' = bf16(silu(g')) +- 1 step.
    Nearly all outputs are expected to equal the oracle's h exactly (min_exact)."""
    gk, uk = bf16_ordered(ref["g_bits"]), bf16_ordered(ref["u_bits"])
    lo = np.full(h_bits.shape, np.inf)
    hi = np.full(h_bits.shape, -np.inf)
    for dg in (-1, 0, 1):
        g = bf16_from_ordered(gk + dg)
        for du in (-1, 0, 1):
            u = bf16_from_ordered(uk + du)
            s, _ = oracle.swiglu(g, u)
            sk = bf16_ordered(s)
            uf = bf16_bits_to_f64(u)
            for ds in (-1, 0, 1):
                sv = bf16_bits_to_f64(bf16_from_ordered(sk + ds))
                hv = bf16_bits_to_f64(oracle.round_bf16(sv * uf))
                lo = np.minimum(lo, hv)
                hi = np.maximum(hi, hv)
    hg = bf16_bits_to_f64(h_bits)
    bad = np.argwhere((hg < lo) | (hg > hi))
    assert bad.size == 0, (f"{where}: {bad.shape[0]} SwiGLU outputs outside the bound, first "
                           f"at {bad[0]}: got {hg[tuple(bad[0])]}, "
                           f"range [{lo[tuple(bad[0])]}, {hi[tuple(bad[0])]}]")
    exact = float(np.mean(bf16_ordered(h_bits) == bf16_ordered(ref["h_bits"])))
    assert exact >= min_exact, f"{where}: only {exact:.4f} of outputs equal the oracle's h"
