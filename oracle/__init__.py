"""Plain CPU oracle for the BitNet b1.58 W2A8 BitLinear forward (test infrastructure).

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers. The product library never
imports this package, and this package imports nothing from the product.

The arithmetic lives in ``bitnet_oracle.c`` (plain C, one literal loop per step
of the method, built with ``-O1 -ffp-contract=off``); this module compiles it on
demand and marshals numpy arrays through ctypes. Each wrapper names the page and
section it follows; see the C file's header for the readings taken where the
pages are silent.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(worked example, derived packing bytes, closed forms, brute force, library
rounding); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bitnet_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O1", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-fPIC", "-shared",
           "-Wall", "-Wextra"]
_lock = threading.Lock()
_lib = None

OK, BAD_ARG, BAD_DATA = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile ``bitnet_oracle.c`` into ``liboracle.so`` (if stale or forced)."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True, capture_output=True, text=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
            lib.oracle_absmean_scale.argtypes = [P, I64, I64, I, P]
            lib.oracle_ternarize.argtypes = [P, I64, I64, I, P, P, P]
            lib.oracle_pack.argtypes = [P, I64, I64, P]
            lib.oracle_unpack.argtypes = [P, I64, I64, P]
            lib.oracle_quant_act.argtypes = [P, I64, I64, P, P]
            lib.oracle_ternary_matmul.argtypes = [P, P, I64, I64, I64, P]
            lib.oracle_dequant.argtypes = [P, P, P, I, I64, I64, P]
            lib.oracle_round_bf16.argtypes = [P, I64, P]
            lib.oracle_round_bf16.restype = None
            lib.oracle_bitlinear_sampled.argtypes = [P, I64, I64, P, P, I, I64, P, I64, P, I64,
                                                     P, P, P, P, P, P, P]
            lib.oracle_swiglu.argtypes = [P, P, I64, P, P]
            lib.oracle_pack_b3.argtypes = [P, I64, I64, P]
            lib.oracle_unpack_b3.argtypes = [P, I64, I64, P]
            lib.oracle_quant_act_per_tensor.argtypes = [P, I64, I64, P, P]
            lib.oracle_quant_act_per_tensor.restype = ctypes.c_int
            for name in ("oracle_absmean_scale", "oracle_ternarize", "oracle_pack",
                         "oracle_unpack", "oracle_quant_act", "oracle_ternary_matmul",
                         "oracle_dequant", "oracle_bitlinear_sampled", "oracle_swiglu",
                         "oracle_pack_b3", "oracle_unpack_b3"):
                getattr(lib, name).restype = ctypes.c_int
            _lib = lib
    return _lib


class OracleError(RuntimeError):
    pass


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != OK:
        raise OracleError(f"{what}: {'bad argument' if rc == BAD_ARG else 'invalid data'} ({rc})")


def absmean_scale(W: np.ndarray, per_row: bool) -> np.ndarray:
    """Absmean weight scale ("BitNet 深度实战", §2.4): fp32 [N] or [1]."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    s = np.empty(N if per_row else 1, dtype=np.float32)
    _check(_load().oracle_absmean_scale(_ptr(W), N, K, int(per_row), _ptr(s)), "absmean_scale")
    return s


def ternarize(W: np.ndarray, s_w: np.ndarray, per_row: bool, return_rounded: bool = False):
    """t = clamp(round(W / s), -1, 1) ("BitNet 深度实战", §2.4). Optionally the pre-clip values."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    s_w = np.ascontiguousarray(s_w, dtype=np.float32)
    N, K = W.shape
    t = np.empty((N, K), dtype=np.int8)
    r = np.empty((N, K), dtype=np.int32) if return_rounded else None
    _check(_load().oracle_ternarize(_ptr(W), N, K, int(per_row), _ptr(s_w), _ptr(t),
                                    _ptr(r) if r is not None else None), "ternarize")
    return (t, r) if return_rounded else t


def pack(t: np.ndarray) -> np.ndarray:
    """Codes t+1, four per byte, low bits first along K ("BitNet 深度实战", §4.3)."""
    t = np.ascontiguousarray(t, dtype=np.int8)
    N, K = t.shape
    p = np.empty((N, K // 4), dtype=np.uint8)
    _check(_load().oracle_pack(_ptr(t), N, K, _ptr(p)), "pack")
    return p


def unpack(packed: np.ndarray, K: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    N = packed.shape[0]
    t = np.empty((N, K), dtype=np.int8)
    _check(_load().oracle_unpack(_ptr(packed), N, K, _ptr(t)), "unpack")
    return t


def b3_row_bytes(K: int) -> int:
    """Bytes of one row in the base-3 format: 16 per started chunk of 80 weights."""
    return 16 * ((K + 79) // 80)


def pack_b3(t: np.ndarray) -> np.ndarray:
    """Five weights per byte in base 3 ("将 BitNet 三元查找表集成到自定义 Triton 内核中", step 1:
    4-5 ternary values per byte): byte p of 80-weight chunk c holds k = 80c + 16d + p,
    d = 0..4, as sum_d (t + 1) 3^d. Returns (N, b3_row_bytes(K)) uint8."""
    t = np.ascontiguousarray(t, dtype=np.int8)
    N, K = t.shape
    p = np.empty((N, b3_row_bytes(K)), dtype=np.uint8)
    _check(_load().oracle_pack_b3(_ptr(t), N, K, _ptr(p)), "pack_b3")
    return p


def unpack_b3(packed: np.ndarray, K: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    N = packed.shape[0]
    t = np.empty((N, K), dtype=np.int8)
    _check(_load().oracle_unpack_b3(_ptr(packed), N, K, _ptr(t)), "unpack_b3")
    return t


def pack_weights(W: np.ndarray, per_row: bool):
    """The offline weight step: absmean scale, ternarise, pack. Returns (packed, s_w)."""
    s = absmean_scale(W, per_row)
    return pack(ternarize(W, s, per_row)), s


def quant_act(x_bf16_bits: np.ndarray):
    """Per-token absmax int8 quantiser. x is uint16 bf16 bit patterns (M, K)."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    M, K = x.shape
    q = np.empty((M, K), dtype=np.int8)
    s = np.empty(M, dtype=np.float32)
    _check(_load().oracle_quant_act(_ptr(x), M, K, _ptr(q), _ptr(s)), "quant_act")
    return q, s


def quant_act_per_tensor(x_bf16_bits: np.ndarray):
    """Per-tensor absmax int8 quantiser ("BitNet 1-bit LLM推理优化", §2.2 I2_S and §3.2): one
    scale for the whole (M, K) input. Returns (q, s_x) with s_x holding that scale M times."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    M, K = x.shape
    q = np.empty((M, K), dtype=np.int8)
    s = np.empty(M, dtype=np.float32)
    _check(_load().oracle_quant_act_per_tensor(_ptr(x), M, K, _ptr(q), _ptr(s)),
           "quant_act_per_tensor")
    return q, s


def block_absmax_bits(x_bf16_bits: np.ndarray, block: int = 16) -> np.ndarray:
    """Maxima of |x| over consecutive blocks of ``block`` values along each row, as bf16 bit
    patterns (M, K / block) uint16: the hand-off from the SwiGLU producer to the down
    projection's quantiser ("BitNet-Triton", "技术架构：融合内核的三重优化" item 3: the
    activation quantiser belongs with the producer of its input). |x| of a bf16 pattern is the
    pattern with the sign bit cleared; for non-NaN values those patterns order as unsigned
    integers exactly as the magnitudes do, so the block maximum is exact, and the maximum over
    a row's blocks is the row's amax of ``quant_act``."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    M, K = x.shape
    if K % block:
        raise ValueError(f"K = {K} is not a multiple of the block {block}")
    return (x & np.uint16(0x7FFF)).reshape(M, K // block, block).max(axis=2).astype(np.uint16)


def ternary_matmul(q: np.ndarray, t: np.ndarray) -> np.ndarray:
    """int32 acc[m,n] = sum_k q[m,k] t[n,k] by add / subtract / skip ("BitNet 深度实战", §4.4)."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    t = np.ascontiguousarray(t, dtype=np.int8)
    M, K = q.shape
    N, K2 = t.shape
    assert K == K2
    acc = np.empty((M, N), dtype=np.int32)
    _check(_load().oracle_ternary_matmul(_ptr(q), _ptr(t), M, N, K, _ptr(acc)), "ternary_matmul")
    return acc


def dequant(acc: np.ndarray, s_x: np.ndarray, s_w: np.ndarray, per_row: bool) -> np.ndarray:
    """y = acc * s_w / s_x in fp64."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    s_x = np.ascontiguousarray(s_x, dtype=np.float32)
    s_w = np.ascontiguousarray(s_w, dtype=np.float32)
    M, N = acc.shape
    y = np.empty((M, N), dtype=np.float64)
    _check(_load().oracle_dequant(_ptr(acc), _ptr(s_x), _ptr(s_w), int(per_row), M, N, _ptr(y)),
           "dequant")
    return y


def round_bf16(y: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 (RNE); returns uint16 bit patterns."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    out = np.empty(y.shape, dtype=np.uint16)
    _load().oracle_round_bf16(_ptr(y), y.size, _ptr(out))
    return out


def bitlinear(x_bf16_bits: np.ndarray, packed: np.ndarray, s_w: np.ndarray, per_row: bool,
              K: int, act_per_tensor: bool = False):
    """Full forward on packed weights. Returns dict(y=fp64 (M,N), acc, q, s_x). The
    activation scale is per token, or one per tensor with act_per_tensor."""
    q, s_x = (quant_act_per_tensor if act_per_tensor else quant_act)(x_bf16_bits)
    t = unpack(packed, K)
    acc = ternary_matmul(q, t)
    y = dequant(acc, s_x, s_w, per_row)
    return {"y": y, "acc": acc, "q": q, "s_x": s_x}


def bitlinear_sampled(x_bf16_bits: np.ndarray, packed: np.ndarray, s_w: np.ndarray,
                      per_row: bool, K: int, m_idx, n_idx):
    """Forward restricted to sampled tokens m_idx and output columns n_idx (full-size parity)."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    s_w = np.ascontiguousarray(s_w, dtype=np.float32)
    M = x.shape[0]
    N = packed.shape[0]
    m_idx = np.ascontiguousarray(m_idx, dtype=np.int64)
    n_idx = np.ascontiguousarray(n_idx, dtype=np.int64)
    Ms, Ns = m_idx.size, n_idx.size
    y = np.empty((Ms, Ns), dtype=np.float64)
    acc = np.empty((Ms, Ns), dtype=np.int32)
    q = np.empty((Ms, K), dtype=np.int8)
    sx = np.empty(Ms, dtype=np.float32)
    st = np.empty(K, dtype=np.int8)
    sq = np.empty((Ms, K), dtype=np.int8)
    ssx = np.empty(Ms, dtype=np.float32)
    rc = _load().oracle_bitlinear_sampled(_ptr(x), M, K, _ptr(packed), _ptr(s_w), int(per_row),
                                          N, _ptr(m_idx), Ms, _ptr(n_idx), Ns, _ptr(y), _ptr(acc),
                                          _ptr(q), _ptr(sx), _ptr(st), _ptr(sq), _ptr(ssx))
    _check(rc, "bitlinear_sampled")
    return {"y": y, "acc": acc, "q": q, "s_x": sx}


def swiglu(g_bits: np.ndarray, u_bits: np.ndarray):
    """SwiGLU on bf16 g, u ("BitNet 深度实战", §3.2 BitLlamaMLP): s = bf16(silu(g)),
    h = bf16(s * u). Returns (s_bits, h_bits), uint16 bf16 patterns of g's shape."""
    g = np.ascontiguousarray(g_bits, dtype=np.uint16)
    u = np.ascontiguousarray(u_bits, dtype=np.uint16)
    assert g.shape == u.shape
    s = np.empty(g.shape, dtype=np.uint16)
    h = np.empty(g.shape, dtype=np.uint16)
    _check(_load().oracle_swiglu(_ptr(g), _ptr(u), g.size, _ptr(s), _ptr(h)), "swiglu")
    return s, h


def swiglu_gate_up(x_bf16_bits: np.ndarray, packed_gate: np.ndarray, s_w_gate: np.ndarray,
                   packed_up: np.ndarray, s_w_up: np.ndarray, per_row: bool, K: int):
    """The MLP's gate and up BitLinears followed by SwiGLU ("BitNet 深度实战", §3.2):
    g = bf16(gate(x)), u = bf16(up(x)), h = bf16(bf16(silu(g)) * u). Returns a dict with the
    exact fp64 g and u, their bf16 bits, and s (silu) and h bits, all (M, I)."""
    yg = bitlinear(x_bf16_bits, packed_gate, s_w_gate, per_row, K)["y"]
    yu = bitlinear(x_bf16_bits, packed_up, s_w_up, per_row, K)["y"]
    g_bits, u_bits = round_bf16(yg), round_bf16(yu)
    s_bits, h_bits = swiglu(g_bits, u_bits)
    return {"g": yg, "u": yu, "g_bits": g_bits, "u_bits": u_bits, "s_bits": s_bits,
            "h_bits": h_bits}


def swiglu_gate_up_sampled(x_bf16_bits: np.ndarray, packed_gate: np.ndarray,
                           s_w_gate: np.ndarray, packed_up: np.ndarray, s_w_up: np.ndarray,
                           per_row: bool, K: int, m_idx, n_idx):
    """swiglu_gate_up restricted to tokens m_idx and outputs n_idx (full-size parity)."""
    yg = bitlinear_sampled(x_bf16_bits, packed_gate, s_w_gate, per_row, K, m_idx, n_idx)["y"]
    yu = bitlinear_sampled(x_bf16_bits, packed_up, s_w_up, per_row, K, m_idx, n_idx)["y"]
    g_bits, u_bits = round_bf16(yg), round_bf16(yu)
    s_bits, h_bits = swiglu(g_bits, u_bits)
    return {"g": yg, "u": yu, "g_bits": g_bits, "u_bits": u_bits, "s_bits": s_bits,
            "h_bits": h_bits}


def bitlinear_sampled_per_tensor_act(x_bf16_bits: np.ndarray, packed: np.ndarray,
                                     s_w: np.ndarray, per_row: bool, K: int, m_idx, n_idx):
    """The forward with a per-tensor activation scale on sampled tokens m_idx and outputs
    n_idx: the scale needs all of x, so x is quantised whole, then the sampled rows of q meet
    the sampled weight rows (the oracle's own steps, composed)."""
    q, s_x = quant_act_per_tensor(x_bf16_bits)
    m_idx = np.asarray(m_idx, dtype=np.int64)
    n_idx = np.asarray(n_idx, dtype=np.int64)
    t = unpack(np.ascontiguousarray(packed[n_idx]), K)
    acc = ternary_matmul(q[m_idx], t)
    sw = np.ascontiguousarray(s_w[n_idx] if per_row else s_w, dtype=np.float32)
    y = dequant(acc, s_x[m_idx], sw, per_row)
    return {"y": y, "acc": acc, "q": q[m_idx], "s_x": s_x[m_idx]}
