"""Seeded synthetic inputs for the W2A8 BitLinear workloads.

This module draws random numbers and nothing else: it holds none of the method's
arithmetic (no scale, no rounding to ternary, no packing, no quantisation). It is
the only code the CUDA path's tests/benchmarks and the CPU oracle share.

Every tensor comes from its own numpy PCG64 stream, keyed by
(seed, config, layer, projection, tensor kind) through ``SeedSequence`` spawn
keys, so a tensor never depends on which other tensors were drawn before it.
Activations are drawn in fp32 and rounded to bf16 (round-to-nearest-even, done
by torch's CPU cast) and returned as uint16 bit patterns.

Workload shapes follow the projection shapes of the models the pages discuss
(BitNet b1.58 2B-4T: hidden 2560, FFN 6912, 20 heads / 5 KV heads; an 8B-class
LLaMA layout: hidden 4096, FFN 14336, KV width 1024).
"""
from __future__ import annotations

import numpy as np
import torch

KIND_X, KIND_W, KIND_T, KIND_SW, KIND_OUTLIER = 1, 2, 3, 4, 5

# (N, K) of each projection of one transformer layer.
SHAPES_2B = {"q": (2560, 2560), "k": (640, 2560), "v": (640, 2560), "o": (2560, 2560),
             "gate": (6912, 2560), "up": (6912, 2560), "down": (2560, 6912)}
SHAPES_8B = {"q": (4096, 4096), "k": (1024, 4096), "v": (1024, 4096), "o": (4096, 4096),
             "gate": (14336, 4096), "up": (14336, 4096), "down": (4096, 14336)}
# The four distinct (N, K) shapes of the 2B-4T layer (decode sweep / prefill GEMM).
SWEEP_SHAPES = [(2560, 2560), (640, 2560), (6912, 2560), (2560, 6912)]
PROJ_IDS = {"q": 0, "k": 1, "v": 2, "o": 3, "gate": 4, "up": 5, "down": 6, "sweep0": 10,
            "sweep1": 11, "sweep2": 12, "sweep3": 13}


def rng(seed: int, config: int, layer: int, proj: int, kind: int) -> np.random.Generator:
    ss = np.random.SeedSequence(entropy=seed, spawn_key=(config, layer, proj, kind))
    return np.random.Generator(np.random.PCG64(ss))


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 (RNE, torch CPU cast) -> uint16 bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def normal_x(M: int, K: int, g: np.random.Generator, sigma: float = 1.0) -> np.ndarray:
    """x ~ N(0, sigma^2), bf16 bits (M, K)."""
    return to_bf16_bits(g.standard_normal((M, K), dtype=np.float32) * np.float32(sigma))


def student_t_outlier_x(M: int, K: int, g: np.random.Generator, g_out: np.random.Generator,
                        scale: float = 0.5, frac: float = 0.01, factor: float = 20.0):
    """x = scale * t_4 (t_4 = z / sqrt(chi2_4 / 4), chi2_4 from four squared normals) with
    round(frac*K) outlier channels, picked by a seeded permutation, multiplied by factor."""
    z = g.standard_normal((M, K), dtype=np.float64)
    chi = np.zeros((M, K), dtype=np.float64)
    for _ in range(4):
        n = g.standard_normal((M, K), dtype=np.float64)
        chi += n * n
    x = scale * z / np.sqrt(chi / 4.0)
    n_out = int(round(frac * K))
    cols = g_out.permutation(K)[:n_out]
    x[:, cols] *= factor
    return to_bf16_bits(x.astype(np.float32)), np.sort(cols)


def ternary(N: int, K: int, g: np.random.Generator, p0: float) -> np.ndarray:
    """Ternary weights drawn directly: P(0) = p0, P(+1) = P(-1) = (1 - p0) / 2. int8 (N, K)."""
    u = g.random((N, K), dtype=np.float32)
    pn = (1.0 - p0) / 2.0
    t = np.ones((N, K), dtype=np.int8)
    t[u < pn + p0] = 0
    t[u < pn] = -1
    return t


def latent_w(N: int, K: int, g: np.random.Generator, sigma: float) -> np.ndarray:
    """Latent fp32 weights ~ N(0, sigma^2), (N, K)."""
    return g.standard_normal((N, K), dtype=np.float32) * np.float32(sigma)


def uniform_scale(n: int, g: np.random.Generator, lo: float = 0.5, hi: float = 2.0) -> np.ndarray:
    return g.uniform(lo, hi, size=n).astype(np.float32)


# ----------------------------------------------------------------------------------------------
# The five workloads.
# ----------------------------------------------------------------------------------------------

def tiny(seed: int = 0):
    """Tiny BitLinear: x (4, 512) ~ N(0,1) bf16; latent W (256, 512) ~ N(0,1); per-tensor."""
    x = normal_x(4, 512, rng(seed, 1, 0, 0, KIND_X))
    W = latent_w(256, 512, rng(seed, 1, 0, 0, KIND_W), 1.0)
    return {"x": x, "W": W, "per_row": False, "M": 4, "N": 256, "K": 512}


def decode_case(shape_idx: int, replica: int = 0, M: int = 1, seed: int = 0):
    """Decode GEMV: ternary P(0)=0.4, s_w ~ U(0.5, 2) per tensor, x ~ N(0, 1)."""
    N, K = SWEEP_SHAPES[shape_idx]
    p = 10 + shape_idx
    t = ternary(N, K, rng(seed, 2, replica, p, KIND_T), 0.4)
    s_w = uniform_scale(1, rng(seed, 2, replica, p, KIND_SW))
    x = normal_x(M, K, rng(seed, 2, replica, p, KIND_X))
    return {"x": x, "t": t, "s_w": s_w, "per_row": False, "M": M, "N": N, "K": K}


def prefill_case(shape_idx: int, M: int, seed: int = 0):
    """Prefill GEMM: x = 0.5 t_4 with 1% x20 outlier channels; ternary P(0)=0.5; s_w ~ U(0.5, 2)."""
    N, K = SWEEP_SHAPES[shape_idx]
    p = 10 + shape_idx
    t = ternary(N, K, rng(seed, 3, 0, p, KIND_T), 0.5)
    s_w = uniform_scale(1, rng(seed, 3, 0, p, KIND_SW))
    x, cols = student_t_outlier_x(M, K, rng(seed, 3, M, p, KIND_X),
                                  rng(seed, 3, M, p, KIND_OUTLIER))
    return {"x": x, "t": t, "s_w": s_w, "per_row": False, "M": M, "N": N, "K": K,
            "outlier_cols": cols}


def stack2b_layer(layer: int, seed: int = 0):
    """One layer of the 2B-4T stack: ternary P(0)=0.4 and s_w ~ U(0.5, 2) per projection."""
    out = {}
    for name, (N, K) in SHAPES_2B.items():
        p = PROJ_IDS[name]
        out[name] = {"t": ternary(N, K, rng(seed, 4, layer, p, KIND_T), 0.4),
                     "s_w": uniform_scale(1, rng(seed, 4, layer, p, KIND_SW)),
                     "N": N, "K": K, "per_row": False}
    return out


def stack2b_x(M: int, K: int, seed: int = 0, which: int = 0):
    return normal_x(M, K, rng(seed, 4, 1000 + which, 0, KIND_X))


def stack8b_latent(layer: int, name: str, seed: int = 0):
    """Latent W ~ N(0, 0.02^2) of one 8B-class projection (quantised by the pack step, per row)."""
    N, K = SHAPES_8B[name]
    return latent_w(N, K, rng(seed, 5, layer, PROJ_IDS[name], KIND_W), 0.02)


def stack8b_x(M: int, K: int, seed: int = 0, which: int = 0):
    return normal_x(M, K, rng(seed, 5, 1000 + which, 0, KIND_X))


# ---------------------------------------------------------------- device-side draws
# For workloads too large to draw on the host in a test (billions of values): the same
# distributions drawn by torch's seeded generator on the device, in row chunks so that no
# temporary exceeds about a gigabyte. Deterministic for a given (seed, shape, chunk_rows).

def device_normal_bf16(M: int, K: int, seed: int, device, chunk_rows: int = 1 << 17):
    """x ~ N(0, 1) drawn in fp32 on the device and cast to bf16 there (RNE): (M, K) bf16."""
    g = torch.Generator(device=device).manual_seed(seed)
    out = torch.empty((M, K), dtype=torch.bfloat16, device=device)
    for r0 in range(0, M, chunk_rows):
        r1 = min(M, r0 + chunk_rows)
        out[r0:r1] = torch.randn((r1 - r0, K), generator=g, device=device).to(torch.bfloat16)
    return out


def device_ternary_chunks(N: int, K: int, seed: int, device, chunk_rows: int = 1 << 17):
    """Ternary rows drawn on the device, P(0) = 0.4, P(+1) = P(-1) = 0.3 (as ``ternary``),
    yielded as (row0, int8 tensor (rows, K)) chunks in row order."""
    g = torch.Generator(device=device).manual_seed(seed)
    for r0 in range(0, N, chunk_rows):
        r1 = min(N, r0 + chunk_rows)
        r = torch.randint(0, 10, (r1 - r0, K), generator=g, device=device, dtype=torch.int8)
        t = torch.ones_like(r)
        t[r >= 7] = -1
        t[r < 4] = 0
        del r
        yield r0, t
