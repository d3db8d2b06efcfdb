"""Python binding of libbitnet (the B200 W2A8 BitLinear library).

Argument marshalling only: every step of the forward runs in the CUDA kernels behind
the C ABI declared in ``include/bitnet.h``. PyTorch supplies device memory (output and
workspace tensors) and the current CUDA stream; nothing here computes on tensors.

The shared library is built in-tree by ``python ternary_w2a8_linear_token_b200/build.py``.
Importing this package without it raises ImportError: there is no fallback path.

Functions keep the C names:
    bitnet_pack_weights(W, per_row)            -> (packed, s_w)
    bitnet_pack_ternary(t)                     -> packed
    bitnet_quant_act(x)                        -> (q, s_x)
    bitnet_linear(x, packed, s_w, per_row, ...) -> y
    bitnet_linear_batch(x, projs, ...)         -> [y, ...]
    bitnet_linear_i32(q, packed, ...)          -> acc (int32)
    bitnet_interleave_gate_up(pg, sg, pu, su, per_row) -> (packed_gu, s_w_gu)
    bitnet_linear_swiglu(x, packed_gu, s_w_gu, per_row, ...) -> h (bf16)
    bitnet_check_device_errors()               -> watchdog word (0 = clean)
"""
from __future__ import annotations

import ctypes
import functools
import os
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbitnet.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python ternary_w2a8_linear_token_b200/build.py` "
        "(there is no non-CUDA fallback)")

lib = ctypes.CDLL(LIB_PATH)

# ----------------------------------------------------------------------------- constants
OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE = range(8)
SCALE_PER_TENSOR, SCALE_PER_ROW = 0, 1
OUT_BF16, OUT_F32 = 0, 1
PATH_AUTO, PATH_GEMV, PATH_TC, PATH_MMA = 0, 1, 2, 3
ACT_PER_TOKEN, ACT_PER_TENSOR = 0, 1
QUANT_WORKSPACE_BYTES = 4096
GEMV_MAX_M = 8
GEMV_AUTO_M = 4  # PATH_AUTO: GEMV up to here; 5..8 tokens take the tensor-core path given a workspace
WATCHDOG_TMA_FULL, WATCHDOG_UNPACK, WATCHDOG_EMPTY, WATCHDOG_ACCUM, WATCHDOG_DRAIN = (
    1 << 0, 1 << 1, 1 << 2, 1 << 3, 1 << 4)
WATCHDOG_SELFTEST = 1 << 6
MAX_PROJ = 8
SWIGLU_BLOCK = 16  # interleaved gate/up rows come in blocks of this many

_P, _I64, _I32, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t


class bitnet_proj(ctypes.Structure):
    _fields_ = [("packed", _P), ("s_w", _P), ("mode", _I32), ("reserved", _I32), ("N", _I64),
                ("y", _P)]


class bitnet_plan(ctypes.Structure):
    _fields_ = [("kernel", _I32), ("grid", _I32), ("tile_tokens", _I32), ("splits", _I32),
                ("tile_rows", _I32), ("reserved", _I32 * 3)]


KERNEL_GEMV, KERNEL_MMA_GEMV, KERNEL_STREAM, KERNEL_TC, KERNEL_GS = 1, 2, 3, 4, 5

_SIGS = {
    "bitnet_pack_weights": ([_P, _I64, _I64, ctypes.c_int, _P, _P, _P], ctypes.c_int),
    "bitnet_pack_ternary": ([_P, _I64, _I64, _P, _P], ctypes.c_int),
    "bitnet_quant_act": ([_P, _I64, _I64, _P, _P, _P], ctypes.c_int),
    "bitnet_linear_workspace_size": ([_I64, _I64], _SZ),
    "bitnet_quant_act_ex": ([_P, _I64, _I64, ctypes.c_int, _P, _P, _P, _SZ, _P], ctypes.c_int),
    "bitnet_linear_batch_act": ([_P, _I64, _I64, ctypes.POINTER(bitnet_proj), _I32, ctypes.c_int,
                                 ctypes.c_int, _P, _SZ, ctypes.c_int, _P], ctypes.c_int),
    "bitnet_linear": ([_P, _I64, _I64, _P, _P, ctypes.c_int, _I64, _P, ctypes.c_int, _P, _SZ, _P],
                      ctypes.c_int),
    "bitnet_linear_ex": ([_P, _I64, _I64, _P, _P, ctypes.c_int, _I64, _P, ctypes.c_int, _P, _SZ,
                          ctypes.c_int, _P], ctypes.c_int),
    "bitnet_linear_batch": ([_P, _I64, _I64, ctypes.POINTER(bitnet_proj), _I32, ctypes.c_int, _P,
                             _SZ, _P], ctypes.c_int),
    "bitnet_linear_batch_ex": ([_P, _I64, _I64, ctypes.POINTER(bitnet_proj), _I32, ctypes.c_int,
                                _P, _SZ, ctypes.c_int, _P], ctypes.c_int),
    "bitnet_linear_i32": ([_P, _I64, _I64, _P, _I64, _P, _P, _SZ, ctypes.c_int, _P], ctypes.c_int),
    "bitnet_linear_noalloc": ([_P, _I64, _I64, _P, _P, ctypes.c_int, _I64, _P, ctypes.c_int, _P],
                              ctypes.c_int),
    "bitnet_interleave_gate_up": ([_P, _P, _P, _P, ctypes.c_int, _I64, _I64, _P, _P, _P],
                                  ctypes.c_int),
    "bitnet_linear_swiglu": ([_P, _I64, _I64, _P, _P, ctypes.c_int, _I64, _P, _P, _SZ,
                             ctypes.c_int, _P], ctypes.c_int),
    "bitnet_linear_swiglu_hmax": ([_P, _I64, _I64, _P, _P, ctypes.c_int, _I64, _P, _P, _P, _SZ,
                                   _P], ctypes.c_int),
    "bitnet_linear_hmax": ([_P, _P, _I64, _I64, _P, _P, ctypes.c_int, _I64, _P, ctypes.c_int, _P,
                            _SZ, _P], ctypes.c_int),
    "bitnet_quant_act_hmax": ([_P, _P, _I64, _I64, _P, _P, _P], ctypes.c_int),
    "bitnet_b3_row_bytes": ([_I64], _I64),
    "bitnet_pack_ternary_b3": ([_P, _I64, _I64, _P, _P], ctypes.c_int),
    "bitnet_linear_b3": ([_P, _I64, _I64, _P, _P, ctypes.c_int, _I64, _P, ctypes.c_int, _P],
                         ctypes.c_int),
    "bitnet_act_amax": ([_P, _I64, _I64, _P, _P], ctypes.c_int),
    "bitnet_quant_act_amax": ([_P, _I64, _I64, _P, _P, _P, _P], ctypes.c_int),
    "bitnet_dequant": ([_P, _I64, _I64, _P, _P, ctypes.c_int, _P, ctypes.c_int, _P], ctypes.c_int),
    "bitnet_linear_plan": ([_I64, _I64, ctypes.POINTER(_I64), _I32, _I32, _SZ, ctypes.c_int,
                            ctypes.POINTER(bitnet_plan)], ctypes.c_int),
    "bitnet_check_device_errors": ([ctypes.POINTER(_I32)], ctypes.c_int),
    "bitnet_selftest_wait_timeout": ([_I64, _P], ctypes.c_int),
    "bitnet_probe_int_rate": ([_I32, _I32, _I64, _P, _P], ctypes.c_int),
    "bitnet_probe_int_ops": ([_I32, _I32, _I64], _I64),
    "bitnet_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "bitnet_version": ([], _I32),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.argtypes = _args
    _f.restype = _res


class BitnetError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib.bitnet_status_string(status).decode()} ({status})")


def _check(status: int, where: str):
    if status != OK:
        raise BitnetError(status, where)


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _dev(t: torch.Tensor, dtype: torch.dtype, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _x_ptr(x: torch.Tensor) -> int:
    if x.dtype == torch.bfloat16:
        return _dev(x, torch.bfloat16, "x")
    return _dev(x, torch.int16, "x (bf16 bits)")


def _check_proj(packed: torch.Tensor, s_w: torch.Tensor, per_row: bool, K: int,
                name: str = "packed") -> int:
    """Shape checks the C side cannot make (it sees only pointers): packed (N, K/4) and s_w
    of N (per row) or 1 (per tensor) elements. Returns N."""
    if packed.dim() != 2 or packed.shape[1] * 4 != K:
        raise ValueError(f"{name} must be (N, K/4) = (N, {K // 4}), got {tuple(packed.shape)}")
    N = packed.shape[0]
    want = N if per_row else 1
    if s_w.numel() != want:
        raise ValueError(f"s_w must have {want} element(s) ({'per row' if per_row else 'per tensor'})"
                         f", got {s_w.numel()}")
    return N


def _check_out(y: torch.Tensor, M: int, N: int, name: str = "y"):
    if tuple(y.shape) != (M, N):
        raise ValueError(f"{name} must be ({M}, {N}), got {tuple(y.shape)}")
    if y.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError(f"{name} must be bfloat16 or float32, got {y.dtype}")


def workspace_size(M: int, K: int) -> int:
    return int(lib.bitnet_linear_workspace_size(M, K))


def make_workspace(M: int, K: int, device=None) -> torch.Tensor:
    """A device buffer big enough for the tensor-core path at (M, K) (256-byte aligned)."""
    n = workspace_size(M, K)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device or "cuda")


# ----------------------------------------------------------------------------- calls
def bitnet_pack_weights(W: torch.Tensor, per_row: bool, stream=None):
    N, K = W.shape
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device=W.device)
    s_w = torch.empty(N if per_row else 1, dtype=torch.float32, device=W.device)
    _check(lib.bitnet_pack_weights(_dev(W, torch.float32, "W"), N, K, int(bool(per_row)),
                                   packed.data_ptr(), s_w.data_ptr(), _stream(stream)),
           "bitnet_pack_weights")
    return packed, s_w


def bitnet_pack_ternary(t: torch.Tensor, stream=None) -> torch.Tensor:
    N, K = t.shape
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device=t.device)
    _check(lib.bitnet_pack_ternary(_dev(t, torch.int8, "t"), N, K, packed.data_ptr(),
                                   _stream(stream)), "bitnet_pack_ternary")
    return packed


def bitnet_quant_act(x: torch.Tensor, stream=None):
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    s_x = torch.empty(M, dtype=torch.float32, device=x.device)
    _check(lib.bitnet_quant_act(_x_ptr(x), M, K, q.data_ptr(), s_x.data_ptr(), _stream(stream)),
           "bitnet_quant_act")
    return q, s_x


def bitnet_quant_act_ex(x: torch.Tensor, act: int = ACT_PER_TOKEN, stream=None):
    """bitnet_quant_act with a choice of scale granularity (ACT_PER_TOKEN / ACT_PER_TENSOR)."""
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    s_x = torch.empty(M, dtype=torch.float32, device=x.device)
    ws = torch.empty(QUANT_WORKSPACE_BYTES, dtype=torch.uint8, device=x.device)
    _check(lib.bitnet_quant_act_ex(_x_ptr(x), M, K, act, q.data_ptr(), s_x.data_ptr(),
                                   ws.data_ptr(), ws.numel(), _stream(stream)),
           "bitnet_quant_act_ex")
    return q, s_x


@functools.lru_cache(maxsize=4096)
def _takes_tc_path(M: int, K: int, path: int) -> bool:
    """Whether a call of this shape runs the tensor-core path (and so needs a workspace): the
    library's own plan query, which also covers rows too long for the GEMV."""
    if path == PATH_TC:
        return True
    if path != PATH_AUTO:
        return False
    pl = bitnet_plan()
    arr = (_I64 * 1)(64)
    st = lib.bitnet_linear_plan(M, K, arr, 1, 0, workspace_size(M, K), path, ctypes.byref(pl))
    return st == OK and pl.kernel == KERNEL_TC


def _ws_args(workspace: Optional[torch.Tensor], M: int, K: int, path: int, device):
    if workspace is None:
        if not _takes_tc_path(M, K, path):
            return None, 0, None
        workspace = make_workspace(M, K, device)
    return workspace.data_ptr(), workspace.numel() * workspace.element_size(), workspace


def bitnet_linear(x: torch.Tensor, packed: torch.Tensor, s_w: torch.Tensor, per_row: bool,
                  out_dtype: torch.dtype = torch.bfloat16, y: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, path: int = PATH_AUTO, stream=None):
    M, K = x.shape
    N = _check_proj(packed, s_w, per_row, K)
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=x.device)
    _check_out(y, M, N)
    od = OUT_BF16 if y.dtype == torch.bfloat16 else OUT_F32
    wp, wb, _keep = _ws_args(workspace, M, K, path, x.device)
    _check(lib.bitnet_linear_ex(_x_ptr(x), M, K, _dev(packed, torch.uint8, "packed"),
                                _dev(s_w, torch.float32, "s_w"), int(bool(per_row)), N,
                                _dev(y, y.dtype, "y"), od, wp, wb, path, _stream(stream)),
           "bitnet_linear")
    return y


def bitnet_linear_batch(x: torch.Tensor, projs: Sequence, out_dtype: torch.dtype = torch.bfloat16,
                        ys: Optional[Sequence[torch.Tensor]] = None,
                        workspace: Optional[torch.Tensor] = None, path: int = PATH_AUTO,
                        stream=None):
    """projs: sequence of (packed, s_w, per_row). Returns the list of outputs (M, N_i)."""
    M, K = x.shape
    n = len(projs)
    if not 1 <= n <= MAX_PROJ:
        raise ValueError(f"1..{MAX_PROJ} projections")
    Ns = [_check_proj(p[0], p[1], p[2], K) for p in projs]
    if ys is None:
        ys = [torch.empty((M, N), dtype=out_dtype, device=x.device) for N in Ns]
    if len(ys) != n:
        raise ValueError(f"{n} projections need {n} outputs, got {len(ys)}")
    for yi, N in zip(ys, Ns):
        _check_out(yi, M, N)
    if any(yi.dtype != ys[0].dtype for yi in ys):
        raise ValueError("all outputs of a batch must have one dtype")
    od = OUT_BF16 if ys[0].dtype == torch.bfloat16 else OUT_F32
    arr = (bitnet_proj * n)()
    for i, (packed, s_w, per_row) in enumerate(projs):
        arr[i].packed = _dev(packed, torch.uint8, "packed")
        arr[i].s_w = _dev(s_w, torch.float32, "s_w")
        arr[i].mode = int(bool(per_row))
        arr[i].reserved = 0
        arr[i].N = packed.shape[0]
        arr[i].y = _dev(ys[i], ys[i].dtype, "y")
    wp, wb, _keep = _ws_args(workspace, M, K, path, x.device)
    _check(lib.bitnet_linear_batch_ex(_x_ptr(x), M, K, arr, n, od, wp, wb, path, _stream(stream)),
           "bitnet_linear_batch")
    return list(ys)


def bitnet_linear_batch_act(x: torch.Tensor, projs: Sequence, act: int,
                            out_dtype: torch.dtype = torch.bfloat16,
                            ys: Optional[Sequence[torch.Tensor]] = None,
                            workspace: Optional[torch.Tensor] = None, path: int = PATH_AUTO,
                            stream=None):
    """bitnet_linear_batch with a choice of activation scale granularity (act)."""
    M, K = x.shape
    n = len(projs)
    if not 1 <= n <= MAX_PROJ:
        raise ValueError(f"1..{MAX_PROJ} projections")
    Ns = [_check_proj(p[0], p[1], p[2], K) for p in projs]
    if ys is None:
        ys = [torch.empty((M, N), dtype=out_dtype, device=x.device) for N in Ns]
    if len(ys) != n:
        raise ValueError(f"{n} projections need {n} outputs, got {len(ys)}")
    for yi, N in zip(ys, Ns):
        _check_out(yi, M, N)
    if any(yi.dtype != ys[0].dtype for yi in ys):
        raise ValueError("all outputs of a batch must have one dtype")
    od = OUT_BF16 if ys[0].dtype == torch.bfloat16 else OUT_F32
    arr = (bitnet_proj * n)()
    for i, (packed, s_w, per_row) in enumerate(projs):
        arr[i].packed = _dev(packed, torch.uint8, "packed")
        arr[i].s_w = _dev(s_w, torch.float32, "s_w")
        arr[i].mode = int(bool(per_row))
        arr[i].reserved = 0
        arr[i].N = packed.shape[0]
        arr[i].y = _dev(ys[i], ys[i].dtype, "y")
    wp, wb, _keep = _ws_args(workspace, M, K, path, x.device)
    _check(lib.bitnet_linear_batch_act(_x_ptr(x), M, K, arr, n, od, act, wp, wb, path,
                                       _stream(stream)), "bitnet_linear_batch_act")
    return list(ys)


def bitnet_linear_i32(q: torch.Tensor, packed: torch.Tensor, path: int = PATH_AUTO,
                      workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    M, K = q.shape
    if packed.dim() != 2 or packed.shape[1] * 4 != K:
        raise ValueError(f"packed must be (N, K/4) = (N, {K // 4}), got {tuple(packed.shape)}")
    N = packed.shape[0]
    acc = torch.empty((M, N), dtype=torch.int32, device=q.device)
    wp, wb, _keep = _ws_args(workspace, M, K, path, q.device)
    _check(lib.bitnet_linear_i32(_dev(q, torch.int8, "q"), M, K,
                                 _dev(packed, torch.uint8, "packed"), N, acc.data_ptr(), wp, wb,
                                 path, _stream(stream)), "bitnet_linear_i32")
    return acc


def bitnet_interleave_gate_up(packed_gate: torch.Tensor, s_w_gate: torch.Tensor,
                              packed_up: torch.Tensor, s_w_up: torch.Tensor, per_row: bool,
                              stream=None):
    """Gate and up projections (each (I, K/4) packed) -> the interleaved (2I, K/4) matrix
    and its scales (2I per row, or {s_gate, s_up}) that bitnet_linear_swiglu reads."""
    I, K4 = packed_gate.shape
    if tuple(packed_up.shape) != (I, K4):
        raise ValueError("gate and up must have the same shape")
    dev = packed_gate.device
    packed_gu = torch.empty((2 * I, K4), dtype=torch.uint8, device=dev)
    s_w_gu = torch.empty(2 * I if per_row else 2, dtype=torch.float32, device=dev)
    _check(lib.bitnet_interleave_gate_up(_dev(packed_gate, torch.uint8, "packed_gate"),
                                         _dev(s_w_gate, torch.float32, "s_w_gate"),
                                         _dev(packed_up, torch.uint8, "packed_up"),
                                         _dev(s_w_up, torch.float32, "s_w_up"),
                                         int(bool(per_row)), I, 4 * K4, packed_gu.data_ptr(),
                                         s_w_gu.data_ptr(), _stream(stream)),
           "bitnet_interleave_gate_up")
    return packed_gu, s_w_gu


def bitnet_linear_swiglu(x: torch.Tensor, packed_gu: torch.Tensor, s_w_gu: torch.Tensor,
                         per_row: bool, h: Optional[torch.Tensor] = None,
                         workspace: Optional[torch.Tensor] = None, path: int = PATH_AUTO,
                         stream=None) -> torch.Tensor:
    """h = bf16(bf16(silu(gate(x))) * up(x)), (M, I), from the interleaved gate/up matrix."""
    M, K = x.shape
    if packed_gu.dim() != 2 or packed_gu.shape[1] * 4 != K or packed_gu.shape[0] % 2:
        raise ValueError(f"packed_gu must be (2I, K/4) = (2I, {K // 4}), got "
                         f"{tuple(packed_gu.shape)}")
    I = packed_gu.shape[0] // 2
    want = 2 * I if per_row else 2
    if s_w_gu.numel() != want:
        raise ValueError(f"s_w_gu must have {want} elements, got {s_w_gu.numel()}")
    if h is None:
        h = torch.empty((M, I), dtype=torch.bfloat16, device=x.device)
    if tuple(h.shape) != (M, I):
        raise ValueError(f"h must be ({M}, {I}), got {tuple(h.shape)}")
    wp, wb, _keep = _ws_args(workspace, M, K, path, x.device)
    _check(lib.bitnet_linear_swiglu(_x_ptr(x), M, K, _dev(packed_gu, torch.uint8, "packed_gu"),
                                    _dev(s_w_gu, torch.float32, "s_w_gu"), int(bool(per_row)), I,
                                    _dev(h, torch.bfloat16, "h"), wp, wb, path, _stream(stream)),
           "bitnet_linear_swiglu")
    return h


def _check_xmax(xmax: torch.Tensor, M: int, K: int):
    if tuple(xmax.shape) != (M, K // SWIGLU_BLOCK) or not xmax.is_contiguous():
        raise ValueError(f"xmax must be contiguous ({M}, {K // SWIGLU_BLOCK}), got "
                         f"{tuple(xmax.shape)}")
    return _dev(xmax, torch.int16, "xmax")


def bitnet_linear_swiglu_hmax(x: torch.Tensor, packed_gu: torch.Tensor, s_w_gu: torch.Tensor,
                              per_row: bool, h: Optional[torch.Tensor] = None,
                              hmax: Optional[torch.Tensor] = None,
                              workspace: Optional[torch.Tensor] = None, stream=None):
    """bitnet_linear_swiglu on the tensor-core path that also returns hmax (M, I/16) int16:
    the bf16 bits of max |h| over each block of 16 outputs, for bitnet_linear_hmax."""
    M, K = x.shape
    if packed_gu.dim() != 2 or packed_gu.shape[1] * 4 != K or packed_gu.shape[0] % 2:
        raise ValueError(f"packed_gu must be (2I, K/4) = (2I, {K // 4}), got "
                         f"{tuple(packed_gu.shape)}")
    I = packed_gu.shape[0] // 2
    want = 2 * I if per_row else 2
    if s_w_gu.numel() != want:
        raise ValueError(f"s_w_gu must have {want} elements, got {s_w_gu.numel()}")
    if h is None:
        h = torch.empty((M, I), dtype=torch.bfloat16, device=x.device)
    if hmax is None:
        hmax = torch.empty((M, I // SWIGLU_BLOCK), dtype=torch.int16, device=x.device)
    if tuple(h.shape) != (M, I):
        raise ValueError(f"h must be ({M}, {I}), got {tuple(h.shape)}")
    hm = _check_xmax(hmax, M, I)
    wp, wb, _keep = _ws_args(workspace, M, K, PATH_TC, x.device)
    _check(lib.bitnet_linear_swiglu_hmax(_x_ptr(x), M, K, _dev(packed_gu, torch.uint8, "packed_gu"),
                                         _dev(s_w_gu, torch.float32, "s_w_gu"),
                                         int(bool(per_row)), I, _dev(h, torch.bfloat16, "h"),
                                         hm, wp, wb, _stream(stream)),
           "bitnet_linear_swiglu_hmax")
    return h, hmax


def bitnet_linear_hmax(x: torch.Tensor, xmax: torch.Tensor, packed: torch.Tensor,
                       s_w: torch.Tensor, per_row: bool, out_dtype: torch.dtype = torch.bfloat16,
                       y: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None, stream=None):
    """bitnet_linear on the tensor-core path with each token's amax taken from xmax, the
    (M, K/16) block maxima of |x| (as bitnet_linear_swiglu_hmax returns them for h)."""
    M, K = x.shape
    N = _check_proj(packed, s_w, per_row, K)
    xm = _check_xmax(xmax, M, K)
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=x.device)
    _check_out(y, M, N)
    od = OUT_BF16 if y.dtype == torch.bfloat16 else OUT_F32
    wp, wb, _keep = _ws_args(workspace, M, K, PATH_TC, x.device)
    _check(lib.bitnet_linear_hmax(_x_ptr(x), xm, M, K, _dev(packed, torch.uint8, "packed"),
                                  _dev(s_w, torch.float32, "s_w"), int(bool(per_row)), N,
                                  _dev(y, y.dtype, "y"), od, wp, wb, _stream(stream)),
           "bitnet_linear_hmax")
    return y


def bitnet_quant_act_hmax(x: torch.Tensor, xmax: torch.Tensor, stream=None):
    """bitnet_quant_act with each token's amax taken from xmax (M, K/16)."""
    M, K = x.shape
    xm = _check_xmax(xmax, M, K)
    q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    s_x = torch.empty(M, dtype=torch.float32, device=x.device)
    _check(lib.bitnet_quant_act_hmax(_x_ptr(x), xm, M, K, q.data_ptr(), s_x.data_ptr(),
                                     _stream(stream)), "bitnet_quant_act_hmax")
    return q, s_x


NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


def bitnet_linear_noalloc(x: torch.Tensor, packed: torch.Tensor, s_w: torch.Tensor,
                          per_row: bool, out_dtype: torch.dtype = torch.bfloat16,
                          y: Optional[torch.Tensor] = None, stream=None):
    """bitnet_linear without a workspace, for callers that cannot allocate device memory
    while they run (a serving loop where cudaMalloc could synchronise the device, a plug-in
    whose host runtime owns all device memory). The tensor-core path uses the library's
    fixed 16 MiB device scratch array; calls that can overlap on the GPU race on it. Sizes
    whose workspace exceeds the array raise BitnetError (ERR_WORKSPACE). Pass y to make the
    call itself allocate nothing (with y=None this wrapper allocates the output)."""
    M, K = x.shape
    N = _check_proj(packed, s_w, per_row, K)
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=x.device)
    _check_out(y, M, N)
    od = OUT_BF16 if y.dtype == torch.bfloat16 else OUT_F32
    _check(lib.bitnet_linear_noalloc(_x_ptr(x), M, K, _dev(packed, torch.uint8, "packed"),
                                     _dev(s_w, torch.float32, "s_w"), int(bool(per_row)), N,
                                     _dev(y, y.dtype, "y"), od, _stream(stream)),
           "bitnet_linear_noalloc")
    return y


def bitnet_pack_ternary_b3(t: torch.Tensor, stream=None) -> torch.Tensor:
    """Ternary (N, K) int8 -> the base-3 format, five weights per byte (N, 16 ceil(K / 80))."""
    N, K = t.shape
    packed = torch.empty((N, int(lib.bitnet_b3_row_bytes(K))), dtype=torch.uint8, device=t.device)
    _check(lib.bitnet_pack_ternary_b3(_dev(t, torch.int8, "t"), N, K, packed.data_ptr(),
                                      _stream(stream)), "bitnet_pack_ternary_b3")
    return packed


def bitnet_linear_b3(x: torch.Tensor, packed_b3: torch.Tensor, s_w: torch.Tensor, per_row: bool,
                     out_dtype: torch.dtype = torch.bfloat16, y: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """bitnet_linear for one token on base-3 weights (bitnet_pack_ternary_b3)."""
    M, K = x.shape
    N = packed_b3.shape[0]
    if packed_b3.dim() != 2 or packed_b3.shape[1] != int(lib.bitnet_b3_row_bytes(K)):
        raise ValueError("packed_b3 must be (N, bitnet_b3_row_bytes(K))")
    if s_w.numel() != (N if per_row else 1):
        raise ValueError("s_w must have N (per row) or 1 elements")
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=x.device)
    _check_out(y, M, N)
    od = OUT_BF16 if y.dtype == torch.bfloat16 else OUT_F32
    _check(lib.bitnet_linear_b3(_x_ptr(x), M, K, _dev(packed_b3, torch.uint8, "packed_b3"),
                                _dev(s_w, torch.float32, "s_w"), int(bool(per_row)), N,
                                _dev(y, y.dtype, "y"), od, _stream(stream)), "bitnet_linear_b3")
    return y


def bitnet_act_amax(x: torch.Tensor, stream=None) -> torch.Tensor:
    """Per-token max |x| (fp32, exact), the first tensor-parallel step of a K-split projection."""
    M, K = x.shape
    amax = torch.empty(M, dtype=torch.float32, device=x.device)
    _check(lib.bitnet_act_amax(_x_ptr(x), M, K, amax.data_ptr(), _stream(stream)),
           "bitnet_act_amax")
    return amax


def bitnet_quant_act_amax(x: torch.Tensor, amax: torch.Tensor, stream=None):
    """Per-token quantiser with the amax supplied (e.g. all-reduced over a K split): (q, s_x)."""
    M, K = x.shape
    if amax.numel() != M:
        raise ValueError(f"amax must have {M} elements, got {amax.numel()}")
    q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    s_x = torch.empty(M, dtype=torch.float32, device=x.device)
    _check(lib.bitnet_quant_act_amax(_x_ptr(x), M, K, _dev(amax, torch.float32, "amax"),
                                     q.data_ptr(), s_x.data_ptr(), _stream(stream)),
           "bitnet_quant_act_amax")
    return q, s_x


def bitnet_dequant(acc: torch.Tensor, s_x: torch.Tensor, s_w: torch.Tensor, per_row: bool,
                   out_dtype: torch.dtype = torch.bfloat16, y: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """The epilogue alone on an int32 accumulator (M, N): y = acc * (s_w * (1 / s_x))."""
    M, N = acc.shape
    if s_x.numel() != M or s_w.numel() != (N if per_row else 1):
        raise ValueError("s_x must have M elements and s_w N (per row) or 1")
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=acc.device)
    _check_out(y, M, N)
    od = OUT_BF16 if y.dtype == torch.bfloat16 else OUT_F32
    _check(lib.bitnet_dequant(_dev(acc, torch.int32, "acc"), M, N, _dev(s_x, torch.float32, "s_x"),
                              _dev(s_w, torch.float32, "s_w"), int(bool(per_row)),
                              _dev(y, y.dtype, "y"), od, _stream(stream)), "bitnet_dequant")
    return y


def bitnet_linear_plan(M: int, K: int, Ns: Sequence[int], swiglu: bool = False,
                       workspace_bytes: Optional[int] = None, path: int = PATH_AUTO) -> dict:
    """The kernels a bitnet_linear_batch (or, with swiglu, bitnet_linear_swiglu with
    Ns = [2I]) call would run: host-only, nothing is launched. workspace_bytes defaults to
    workspace_size(M, K), what make_workspace provides."""
    n = len(Ns)
    arr = (_I64 * max(n, 1))(*Ns)
    wb = workspace_size(M, K) if workspace_bytes is None else int(workspace_bytes)
    pl = bitnet_plan()
    _check(lib.bitnet_linear_plan(M, K, arr, n, int(bool(swiglu)), wb, path, ctypes.byref(pl)),
           "bitnet_linear_plan")
    return {"kernel": pl.kernel, "grid": pl.grid, "tile_tokens": pl.tile_tokens,
            "splits": pl.splits, "tile_rows": pl.tile_rows}


def bitnet_check_device_errors() -> int:
    flags = _I32(0)
    st = lib.bitnet_check_device_errors(ctypes.byref(flags))
    if st not in (OK, ERR_TIMEOUT):
        raise BitnetError(st, "bitnet_check_device_errors")
    return int(flags.value)


def bitnet_selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    """Launches the watchdog self-test: one bounded wait on a barrier nothing completes."""
    st = lib.bitnet_selftest_wait_timeout(int(limit_ns), _stream(stream))
    if st != OK:
        raise BitnetError(st, "bitnet_selftest_wait_timeout")


def bitnet_version() -> int:
    return int(lib.bitnet_version())
