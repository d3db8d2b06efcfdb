"""Host-side checks of the C ABI: the library loads, exports every declared call, and
rejects bad arguments before any launch. No GPU is needed: every call here fails its
argument checks, which run before the library touches CUDA (fake pointers below are
never dereferenced)."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitnet.h")


@pytest.fixture(scope="module")
def bn():
    import ternary_w2a8_linear_token_b200 as bn
    return bn


def declared_functions():
    src = open(HEADER, encoding="utf-8").read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bitnet_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("bitnet_pack_weights", "bitnet_quant_act", "bitnet_linear",
                     "bitnet_linear_batch"):
        assert required in names


def test_library_exports_every_declared_symbol(bn):
    missing = [n for n in declared_functions() if not hasattr(bn.lib, n)]
    assert not missing, f"not exported: {missing}"


def test_status_strings_and_version(bn):
    for code in range(8):
        assert bn.lib.bitnet_status_string(code)
    assert bn.lib.bitnet_status_string(99) == b"unknown status"
    assert bn.bitnet_version() >= 100


def test_proj_struct_layout(bn):
    assert ctypes.sizeof(bn.bitnet_proj) == 40
    assert bn.bitnet_proj.N.offset == 24 and bn.bitnet_proj.y.offset == 32


def test_workspace_size(bn):
    assert bn.workspace_size(0, 64) == 0
    ws = bn.workspace_size(300, 2560)
    assert ws >= 300 * 2560 + 2 * 300 * 4 and ws % 256 == 0


FAKE = 0x7F0000000000  # 256-byte aligned, never dereferenced (every call below fails checks)


def _linear(bn, x=FAKE, M=256, K=512, packed=FAKE, s_w=FAKE, mode=0, N=128, y=FAKE, od=0,
            ws=FAKE, wsb=1 << 30, path=0):
    return bn.lib.bitnet_linear_ex(x, M, K, packed, s_w, mode, N, y, od, ws, wsb, path, None)


def test_linear_argument_errors(bn):
    assert _linear(bn, x=None) == bn.ERR_NULL
    assert _linear(bn, packed=None) == bn.ERR_NULL
    assert _linear(bn, s_w=None) == bn.ERR_NULL
    assert _linear(bn, y=None) == bn.ERR_NULL
    assert _linear(bn, M=0) == bn.ERR_SHAPE
    assert _linear(bn, N=0) == bn.ERR_SHAPE
    assert _linear(bn, K=510) == bn.ERR_SHAPE
    assert _linear(bn, K=520) == bn.ERR_UNSUPPORTED  # K % 4 == 0 but K % 64 != 0
    assert _linear(bn, M=1 << 31) == bn.ERR_SHAPE
    assert _linear(bn, x=FAKE + 8) == bn.ERR_ALIGN
    assert _linear(bn, packed=FAKE + 4) == bn.ERR_ALIGN
    assert _linear(bn, y=FAKE + 2) == bn.ERR_ALIGN
    assert _linear(bn, mode=2) == bn.ERR_UNSUPPORTED
    assert _linear(bn, od=3) == bn.ERR_UNSUPPORTED
    assert _linear(bn, path=7) == bn.ERR_UNSUPPORTED
    # tensor-core path (M > 8): workspace checked before any launch
    assert _linear(bn, ws=None) == bn.ERR_WORKSPACE
    assert _linear(bn, wsb=1024) == bn.ERR_WORKSPACE
    assert _linear(bn, ws=FAKE + 16) == bn.ERR_ALIGN
    assert _linear(bn, M=4, path=2, ws=None) == bn.ERR_WORKSPACE


def test_batch_argument_errors(bn):
    arr = (bn.bitnet_proj * 9)()
    for i in range(9):
        arr[i].packed, arr[i].s_w, arr[i].mode, arr[i].N, arr[i].y = FAKE, FAKE, 0, 64, FAKE
    f = bn.lib.bitnet_linear_batch
    assert f(FAKE, 256, 512, arr, 0, 0, FAKE, 1 << 30, None) == bn.ERR_SHAPE
    assert f(FAKE, 256, 512, arr, 9, 0, FAKE, 1 << 30, None) == bn.ERR_SHAPE
    arr[1].reserved = 1
    assert f(FAKE, 256, 512, arr, 2, 0, FAKE, 1 << 30, None) == bn.ERR_UNSUPPORTED
    arr[1].reserved = 0
    arr[1].N = -3
    assert f(FAKE, 256, 512, arr, 2, 0, FAKE, 1 << 30, None) == bn.ERR_SHAPE
    arr[1].N = 64
    arr[1].packed = None
    assert f(FAKE, 256, 512, arr, 2, 0, FAKE, 1 << 30, None) == bn.ERR_NULL
    arr[1].packed = FAKE
    assert f(None, 256, 512, arr, 2, 0, FAKE, 1 << 30, None) == bn.ERR_NULL
    assert f(FAKE, 256, 512, None, 2, 0, FAKE, 1 << 30, None) == bn.ERR_NULL
    assert f(FAKE, 256, 512, arr, 2, 0, None, 0, None) == bn.ERR_WORKSPACE


def test_watchdog_selftest_rejects_limits_before_launch(bn):
    # Out-of-range limits are refused on the host; nothing is launched (no GPU here).
    assert bn.lib.bitnet_selftest_wait_timeout(999_999, None) == bn.ERR_UNSUPPORTED
    assert bn.lib.bitnet_selftest_wait_timeout(2_000_000_001, None) == bn.ERR_UNSUPPORTED
    assert bn.lib.bitnet_selftest_wait_timeout(-1, None) == bn.ERR_UNSUPPORTED


def test_other_calls_argument_errors(bn):
    L = bn.lib
    assert L.bitnet_pack_weights(None, 4, 64, 0, FAKE, FAKE, None) == bn.ERR_NULL
    assert L.bitnet_pack_weights(FAKE, 4, 66, 0, FAKE, FAKE, None) == bn.ERR_SHAPE
    assert L.bitnet_pack_weights(FAKE, 4, 96, 0, FAKE, FAKE, None) == bn.ERR_UNSUPPORTED
    assert L.bitnet_pack_weights(FAKE, 0, 64, 0, FAKE, FAKE, None) == bn.ERR_SHAPE
    assert L.bitnet_pack_weights(FAKE, 4, 64, 5, FAKE, FAKE, None) == bn.ERR_UNSUPPORTED
    assert L.bitnet_pack_weights(FAKE + 4, 4, 64, 0, FAKE, FAKE, None) == bn.ERR_ALIGN
    assert L.bitnet_pack_ternary(FAKE, 4, 60, FAKE, None) == bn.ERR_UNSUPPORTED
    assert L.bitnet_pack_ternary(FAKE, 4, 64, None, None) == bn.ERR_NULL
    assert L.bitnet_quant_act(FAKE, 0, 64, FAKE, FAKE, None) == bn.ERR_SHAPE
    assert L.bitnet_quant_act(FAKE, 3, 64, FAKE + 1, FAKE, None) == bn.ERR_ALIGN
    assert L.bitnet_quant_act(FAKE, 3, 64, FAKE, None, None) == bn.ERR_NULL
    assert L.bitnet_linear_i32(FAKE, 16, 64, FAKE, 16, None, FAKE, 1 << 30, 0, None) == bn.ERR_NULL
    assert L.bitnet_linear_i32(FAKE, 16, 64, FAKE, 16, FAKE, None, 0, 0, None) == bn.ERR_WORKSPACE
    assert L.bitnet_linear_i32(FAKE, 16, 64, FAKE, 16, FAKE, FAKE, 1 << 30, 9, None) == \
        bn.ERR_UNSUPPORTED
    assert L.bitnet_check_device_errors(None) == bn.ERR_NULL


def test_swiglu_calls_argument_errors(bn):
    """bitnet_interleave_gate_up and bitnet_linear_swiglu check shapes, pointers, alignment,
    mode and path before touching the device."""
    L = bn.lib

    def il(pg=FAKE, sg=FAKE, pu=FAKE, su=FAKE, mode=0, I=64, K=512, out=FAKE, sout=FAKE):
        return L.bitnet_interleave_gate_up(pg, sg, pu, su, mode, I, K, out, sout, None)

    assert il(pg=None) == bn.ERR_NULL and il(sout=None) == bn.ERR_NULL
    assert il(I=40) == bn.ERR_SHAPE          # I not a multiple of the 16-row block
    assert il(I=0) == bn.ERR_SHAPE and il(K=6) == bn.ERR_SHAPE
    assert il(K=96) == bn.ERR_UNSUPPORTED    # K % 64
    assert il(mode=2) == bn.ERR_UNSUPPORTED
    assert il(out=FAKE + 8) == bn.ERR_ALIGN and il(sg=FAKE + 2) == bn.ERR_ALIGN

    def sw(x=FAKE, M=4, K=512, pgu=FAKE, s=FAKE, mode=0, I=64, h=FAKE, ws=None, wb=0, path=0):
        return L.bitnet_linear_swiglu(x, M, K, pgu, s, mode, I, h, ws, wb, path, None)

    assert sw(h=None) == bn.ERR_NULL and sw(x=None) == bn.ERR_NULL and sw(s=None) == bn.ERR_NULL
    assert sw(I=24) == bn.ERR_SHAPE and sw(I=0) == bn.ERR_SHAPE and sw(M=0) == bn.ERR_SHAPE
    assert sw(K=96) == bn.ERR_UNSUPPORTED and sw(mode=5) == bn.ERR_UNSUPPORTED
    assert sw(path=7) == bn.ERR_UNSUPPORTED
    assert sw(h=FAKE + 2) == bn.ERR_ALIGN and sw(pgu=FAKE + 4) == bn.ERR_ALIGN
    # the tensor-core path needs the workspace
    assert sw(M=300, path=bn.PATH_TC) == bn.ERR_WORKSPACE
    assert sw(M=300, ws=FAKE, wb=16, path=bn.PATH_TC) == bn.ERR_WORKSPACE


def test_act_mode_calls_argument_errors(bn):
    L = bn.lib
    assert L.bitnet_quant_act_ex(FAKE, 4, 512, 7, FAKE, FAKE, FAKE, 4096, None) == bn.ERR_UNSUPPORTED
    assert L.bitnet_quant_act_ex(FAKE, 4, 512, 1, FAKE, FAKE, None, 0, None) == bn.ERR_WORKSPACE
    assert L.bitnet_quant_act_ex(FAKE, 4, 512, 1, FAKE, FAKE, FAKE, 100, None) == bn.ERR_WORKSPACE
    assert L.bitnet_quant_act_ex(FAKE, 4, 512, 1, FAKE, FAKE, FAKE + 2, 4096, None) == bn.ERR_ALIGN
    assert L.bitnet_quant_act_ex(None, 4, 512, 1, FAKE, FAKE, FAKE, 4096, None) == bn.ERR_NULL
    assert L.bitnet_quant_act_ex(FAKE, 4, 96, 1, FAKE, FAKE, FAKE, 4096, None) == bn.ERR_UNSUPPORTED
    pr = (bn.bitnet_proj * 1)()
    pr[0].packed, pr[0].s_w, pr[0].mode, pr[0].reserved, pr[0].N, pr[0].y = FAKE, FAKE, 0, 0, 128, FAKE
    assert L.bitnet_linear_batch_act(FAKE, 4, 512, pr, 1, 0, 9, None, 0, 0, None) == bn.ERR_UNSUPPORTED
    assert L.bitnet_linear_batch_act(FAKE, 4, 512, pr, 1, 3, 1, None, 0, 0, None) == bn.ERR_UNSUPPORTED
    assert L.bitnet_linear_batch_act(FAKE, 300, 512, pr, 1, 0, 1, None, 0, 0, None) == bn.ERR_WORKSPACE
    assert L.bitnet_linear_batch_act(None, 4, 512, pr, 1, 0, 1, None, 0, 0, None) == bn.ERR_NULL


def test_binding_rejects_wrong_shapes_before_the_call(bn):
    """The C side sees only pointers, so the binding checks every shape it can: packed
    (N, K/4), s_w of N (per row) or 1 (per tensor) elements, and outputs (M, N). These raise
    ValueError on CPU tensors, before any pointer is taken."""
    x = torch.zeros((3, 64), dtype=torch.bfloat16)
    good_p = torch.zeros((8, 16), dtype=torch.uint8)
    one = torch.ones(1, dtype=torch.float32)
    cases = [
        lambda: bn.bitnet_linear(x, torch.zeros((8, 15), dtype=torch.uint8), one, False),
        lambda: bn.bitnet_linear(x, good_p, one, True),  # per row needs 8 scales
        lambda: bn.bitnet_linear(x, good_p, torch.ones(8), False),  # per tensor needs 1
        lambda: bn.bitnet_linear(x, good_p, one, False, y=torch.zeros((3, 7), dtype=torch.bfloat16)),
        lambda: bn.bitnet_linear_noalloc(x, torch.zeros((8, 32), dtype=torch.uint8), one, False),
        lambda: bn.bitnet_linear_noalloc(x, good_p, torch.ones(7), True),
        lambda: bn.bitnet_linear_noalloc(x, good_p, one, False,
                                         y=torch.zeros((2, 8), dtype=torch.bfloat16)),
        lambda: bn.bitnet_linear_batch(x, [(good_p, one, False), (good_p, torch.ones(3), True)]),
        lambda: bn.bitnet_linear_batch(x, [(good_p, one, False)],
                                       ys=[torch.zeros((3, 9), dtype=torch.bfloat16)]),
        lambda: bn.bitnet_linear_swiglu(x, torch.zeros((32, 16), dtype=torch.uint8), one, False),
        lambda: bn.bitnet_linear_i32(torch.zeros((3, 64), dtype=torch.int8),
                                     torch.zeros((8, 17), dtype=torch.uint8)),
    ]
    for i, call in enumerate(cases):
        with pytest.raises(ValueError):
            call()


def test_plan_query_on_the_host(bn):
    """bitnet_linear_plan runs without a device (148 SMs assumed) and reports the kernel
    choices: the one-token kernels by size, the tensor-core tile width by token count, and
    the same argument errors as the call it describes."""
    assert bn.bitnet_linear_plan(1, 2560, [2560])["kernel"] == bn.KERNEL_GEMV
    assert bn.bitnet_linear_plan(1, 2560, [2560], path=bn.PATH_MMA)["kernel"] == bn.KERNEL_MMA_GEMV
    assert bn.bitnet_linear_plan(1, 2560, [2560, 640, 640, 6912, 6912])["kernel"] == \
        bn.KERNEL_GEMV  # 11.3 MB, below the streaming threshold
    assert bn.bitnet_linear_plan(1, 4096, [4096, 1024, 1024, 14336, 14336])["kernel"] == \
        bn.KERNEL_STREAM  # 35.6 MB: the streaming GEMV
    assert bn.bitnet_linear_plan(1, 4096, [28672], swiglu=True)["kernel"] == bn.KERNEL_GS
    assert bn.bitnet_linear_plan(1, 14336, [4096])["kernel"] == bn.KERNEL_STREAM  # longer rows
    assert bn.bitnet_linear_plan(3, 2560, [2560])["kernel"] == bn.KERNEL_GEMV
    # one token past the GEMV's longest row (K = 32768) takes the tensor-core path, so the
    # binding supplies a workspace for it
    assert bn.bitnet_linear_plan(1, 32768, [300])["kernel"] == bn.KERNEL_GEMV
    assert bn.bitnet_linear_plan(1, 32832, [300])["kernel"] == bn.KERNEL_TC
    assert bn._takes_tc_path(1, 32832, bn.PATH_AUTO) and not bn._takes_tc_path(1, 32768, bn.PATH_AUTO)
    # one-token GEMV rows per warp (tile_rows = 16 warps x rows), as the kernels were timed:
    # one row for 640-byte rows up to two CTAs per SM, two for 1 KB rows past one CTA per SM,
    # four past two CTAs per SM at two; SwiGLU: two gate/up pairs per warp past two CTAs per SM
    def rows(M, K, Ns, swiglu=False):
        pl = bn.bitnet_linear_plan(M, K, Ns, swiglu=swiglu)
        assert pl["kernel"] == bn.KERNEL_GEMV
        return pl["tile_rows"], pl["grid"]
    assert rows(1, 2560, [2560]) == (16, 160)
    assert rows(1, 2560, [640]) == (16, 40)
    assert rows(1, 4096, [4096]) == (32, 128)
    assert rows(1, 2560, [6912]) == (32, 216)
    assert rows(1, 6912, [2560]) == (16, 160)
    assert rows(1, 2560, [17664]) == (64, 276)
    assert rows(1, 2560, [13824], swiglu=True) == (64, 216)
    assert rows(1, 4096, [2048], swiglu=True) == (32, 64)
    assert rows(4, 2560, [2560]) == (32, 80)
    # rows longer than the warp-MMA kernel's largest slice: not available there
    with pytest.raises(bn.BitnetError) as e:
        bn.bitnet_linear_plan(1, 20480, [64], path=bn.PATH_MMA)
    assert e.value.status == bn.ERR_UNSUPPORTED
    p = bn.bitnet_linear_plan(4096, 4096, [4096, 1024, 1024, 14336, 14336])
    assert p["kernel"] == bn.KERNEL_TC and p["tile_tokens"] == 192 and p["splits"] == 1
    assert bn.bitnet_linear_plan(16, 2560, [2560])["tile_tokens"] == 16
    assert bn.bitnet_linear_plan(5, 2560, [2560], workspace_bytes=0)["kernel"] == bn.KERNEL_GEMV
    assert bn.bitnet_linear_plan(8, 2560, [6912], workspace_bytes=0)["kernel"] == bn.KERNEL_MMA_GEMV
    with pytest.raises(bn.BitnetError) as e:
        bn.bitnet_linear_plan(64, 2560, [2560], workspace_bytes=0)
    assert e.value.status == bn.ERR_WORKSPACE
    with pytest.raises(bn.BitnetError) as e:
        bn.bitnet_linear_plan(1, 102, [64])  # K % 4 != 0
    assert e.value.status == bn.ERR_SHAPE
    with pytest.raises(bn.BitnetError) as e:
        bn.bitnet_linear_plan(1, 2560, [100], swiglu=True)  # 2I must be a multiple of 32
    assert e.value.status == bn.ERR_SHAPE


def test_tensor_parallel_calls_argument_errors(bn):
    lib = bn.lib
    F = FAKE
    assert lib.bitnet_act_amax(None, 1, 64, F, None) == bn.ERR_NULL
    assert lib.bitnet_act_amax(F, 0, 64, F, None) == bn.ERR_SHAPE
    assert lib.bitnet_act_amax(F, 1, 66, F, None) == bn.ERR_SHAPE
    assert lib.bitnet_act_amax(F + 8, 1, 64, F, None) == bn.ERR_ALIGN
    assert lib.bitnet_quant_act_amax(F, 1, 64, None, F, F, None) == bn.ERR_NULL
    assert lib.bitnet_quant_act_amax(F, 1, 96, F, F, F, None) == bn.ERR_UNSUPPORTED
    assert lib.bitnet_quant_act_amax(F, 1, 64, F, F + 4, F, None) == bn.ERR_ALIGN
    assert lib.bitnet_dequant(F, 1, 8, F, None, 0, F, 0, None) == bn.ERR_NULL
    assert lib.bitnet_dequant(F, 1, 0, F, F, 0, F, 0, None) == bn.ERR_SHAPE
    assert lib.bitnet_dequant(F, 1, 8, F, F, 2, F, 0, None) == bn.ERR_UNSUPPORTED
    assert lib.bitnet_dequant(F, 1, 8, F, F, 0, F, 7, None) == bn.ERR_UNSUPPORTED
    assert lib.bitnet_dequant(F + 2, 1, 8, F, F, 0, F, 0, None) == bn.ERR_ALIGN


def test_b3_calls_argument_errors(bn):
    lib, F = bn.lib, FAKE
    assert lib.bitnet_b3_row_bytes(64) == 16 and lib.bitnet_b3_row_bytes(2560) == 512
    assert lib.bitnet_b3_row_bytes(4096) == 832 and lib.bitnet_b3_row_bytes(0) == 0
    assert lib.bitnet_pack_ternary_b3(None, 4, 64, F, None) == bn.ERR_NULL
    assert lib.bitnet_pack_ternary_b3(F, 4, 66, F, None) == bn.ERR_SHAPE
    assert lib.bitnet_pack_ternary_b3(F + 1, 4, 64, F, None) == bn.ERR_ALIGN
    args = dict(x=F, M=1, K=64, p=F, s=F, mode=0, N=8, y=F, od=0)
    def call(**kw):
        a = dict(args, **kw)
        return lib.bitnet_linear_b3(a["x"], a["M"], a["K"], a["p"], a["s"], a["mode"], a["N"],
                                    a["y"], a["od"], None)
    assert call(M=2) == bn.ERR_UNSUPPORTED      # one token only
    assert call(K=16448) == bn.ERR_UNSUPPORTED  # K <= 16384
    assert call(p=None) == bn.ERR_NULL
    assert call(mode=3) == bn.ERR_UNSUPPORTED and call(od=5) == bn.ERR_UNSUPPORTED
    assert call(y=F + 2) == bn.ERR_ALIGN


def test_hand_off_calls_argument_errors(bn):
    """bitnet_linear_swiglu_hmax, bitnet_linear_hmax and bitnet_quant_act_hmax check pointers,
    shapes and alignment before touching the device, and always need the tensor-core
    workspace (any M)."""
    lib, F = bn.lib, FAKE

    def sw(x=F, M=4, K=512, pgu=F, s=F, mode=0, I=64, h=F, hm=F, ws=None, wb=0):
        return lib.bitnet_linear_swiglu_hmax(x, M, K, pgu, s, mode, I, h, hm, ws, wb, None)

    assert sw(hm=None) == bn.ERR_NULL and sw(h=None) == bn.ERR_NULL and sw(x=None) == bn.ERR_NULL
    assert sw(I=24) == bn.ERR_SHAPE and sw(M=0) == bn.ERR_SHAPE
    assert sw(K=96) == bn.ERR_UNSUPPORTED and sw(mode=4) == bn.ERR_UNSUPPORTED
    assert sw(hm=F + 1) == bn.ERR_ALIGN and sw(h=F + 2) == bn.ERR_ALIGN
    assert sw(M=1) == bn.ERR_WORKSPACE and sw(M=300, ws=F, wb=16) == bn.ERR_WORKSPACE

    def lin(x=F, xm=F, M=4, K=512, p=F, s=F, mode=0, N=64, y=F, od=0, ws=None, wb=0):
        return lib.bitnet_linear_hmax(x, xm, M, K, p, s, mode, N, y, od, ws, wb, None)

    assert lin(xm=None) == bn.ERR_NULL and lin(p=None) == bn.ERR_NULL
    assert lin(M=0) == bn.ERR_SHAPE and lin(K=96) == bn.ERR_UNSUPPORTED
    assert lin(od=3) == bn.ERR_UNSUPPORTED and lin(mode=2) == bn.ERR_UNSUPPORTED
    assert lin(xm=F + 4) == bn.ERR_ALIGN and lin(x=F + 2) == bn.ERR_ALIGN
    assert lin(M=2) == bn.ERR_WORKSPACE

    def qa(x=F, xm=F, M=2, K=512, q=F, s=F):
        return lib.bitnet_quant_act_hmax(x, xm, M, K, q, s, None)

    assert qa(xm=None) == bn.ERR_NULL and qa(q=None) == bn.ERR_NULL
    assert qa(M=0) == bn.ERR_SHAPE and qa(K=96) == bn.ERR_UNSUPPORTED
    assert qa(xm=F + 2) == bn.ERR_ALIGN and qa(q=F + 8) == bn.ERR_ALIGN


def test_probe_calls_argument_errors_and_op_counts(bn):
    lib, F = bn.lib, FAKE
    assert lib.bitnet_probe_int_rate(2, 8, 16, F, None) == bn.ERR_UNSUPPORTED
    assert lib.bitnet_probe_int_rate(0, 0, 16, F, None) == bn.ERR_SHAPE
    assert lib.bitnet_probe_int_rate(1, 8, 0, F, None) == bn.ERR_SHAPE
    assert lib.bitnet_probe_int_rate(0, 8, 1 << 25, F, None) == bn.ERR_SHAPE
    assert lib.bitnet_probe_int_rate(0, 8, 16, None, None) == bn.ERR_NULL
    # 256 threads x 8 chains x 4 multiply-adds; 8 warps x 4 tiles x 16*8*32 multiply-adds
    assert lib.bitnet_probe_int_ops(0, 1, 1) == 256 * 8 * 8
    assert lib.bitnet_probe_int_ops(1, 3, 5) == 8 * 4 * 16 * 8 * 32 * 2 * 3 * 5
    assert lib.bitnet_probe_int_ops(7, 1, 1) == 0


def test_binding_signatures_match_the_header(bn):
    """Every call the header declares has a ctypes signature in the binding with the same
    number of parameters and a matching return type (int status, int64, size_t or string)."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER, encoding="utf-8").read(), flags=re.S)
    decls = re.findall(r"\b(bitnet_status|int64_t|size_t|int32_t|const char\s*\*)\s+"
                       r"(bitnet_[a-z0-9_]+)\s*\(([^;]*?)\)\s*;", src, flags=re.S)
    assert len(decls) == len(declared_functions())
    ret_types = {"bitnet_status": ctypes.c_int, "int64_t": ctypes.c_int64,
                 "size_t": ctypes.c_size_t, "int32_t": ctypes.c_int32}
    for ret, name, args in decls:
        a = args.strip()
        n = 0 if a in ("", "void") else len([x for x in a.split(",") if x.strip()])
        argtypes, restype = bn._SIGS[name]
        assert len(argtypes) == n, name
        want = ctypes.c_char_p if ret.startswith("const char") else ret_types[ret]
        assert restype is want, name
