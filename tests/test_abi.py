"""The C-ABI library on the CPU: it loads, exports every entry point that
include/gq.h declares, and rejects bad arguments synchronously with the
documented status before touching the GPU.  Nothing here launches a kernel:
every call below fails validation (fake device addresses are never touched).
"""
import os
import re
import subprocess

import pytest

import bit_gemv_q4_b200 as gq
from conftest import ROOT

GQ_OK, INVALID, SHAPE, ALIGN, DTYPE = 0, 1, 2, 3, 4
A = 0x10000000  # 16-byte-aligned fake device address (never dereferenced)


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "gq.h")).read()
    return sorted(set(re.findall(r"GQ_API\s+[\w\s\*]+?\b(gq_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    decl = declared_symbols()
    assert len(decl) >= 11
    assert set(decl) == set(gq.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", gq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (gq_\w+)", out))
    assert set(decl) <= exported
    # nothing but the declared entry points leaks out of the library
    assert exported == set(decl)


def test_version_and_status_strings():
    assert gq.gq_abi_version() == 1
    for s in range(10):
        assert gq.gq_status_string(s)
    assert gq.gq_status_from_dev(0) == GQ_OK
    assert gq.gq_status_from_dev(gq.GQ_DEV_RANGE) == 6
    assert gq.gq_status_from_dev(gq.GQ_DEV_NONFINITE | gq.GQ_DEV_RANGE) == 5
    assert gq.gq_status_from_dev(gq.GQ_DEV_TIMEOUT | gq.GQ_DEV_RANGE) == 7


def test_sizes():
    assert gq.gq_q4_0_bytes(32) == 18 and gq.gq_q4_0_bytes(4096 * 11008) == 4096 * 344 * 18
    assert gq.gq_ksb_bytes(256) == 138 and gq.gq_ksb_bytes(11008 * 4096) == 11008 * 16 * 138
    for bad in (-32, 31, 48):
        assert gq.gq_q4_0_bytes(bad) == 0
    for bad in (-256, 32, 288):
        assert gq.gq_ksb_bytes(bad) == 0
    assert gq.gq_q4_0_bytes(0) == 0 and gq.gq_ksb_bytes(0) == 0


@pytest.mark.parametrize("name,block", [("gq_quantize_q4_0", 32), ("gq_quantize_ksb", 256)])
def test_quantize_validation(name, block):
    f = getattr(gq.lib, name)
    assert f(A, -block, A, None, None) == INVALID
    assert f(A, block + 1, A, None, None) == SHAPE
    assert f(A, block // 2, A, None, None) == SHAPE
    assert f(None, 0, None, None, None) == GQ_OK          # empty: no launch
    assert f(None, block, A, None, None) == INVALID
    assert f(A, block, None, None, None) == INVALID
    assert f(A + 4, block, A, None, None) == ALIGN
    assert f(A, block, A + 2, None, None) == ALIGN
    assert f(A, block, A, A + 1, None) == ALIGN          # dev_status must be int-aligned


def test_quantize_rule_flag_validation():
    f = gq.lib.gq_quantize_q4_0_ex
    for flags in (2, 4, 0x80000000, 0xFFFFFFFF):
        assert f(A, 32, A, flags, None, None) == INVALID   # unknown rule bits first
    for flags in (0, gq.GQ_QUANT_REF_RULE):
        assert f(A, -32, A, flags, None, None) == INVALID
        assert f(A, 33, A, flags, None, None) == SHAPE
        assert f(None, 0, None, flags, None, None) == GQ_OK
        assert f(A + 4, 32, A, flags, None, None) == ALIGN
        assert f(A, 32, A, flags, A + 1, None) == ALIGN


@pytest.mark.parametrize("name,block", [("gq_dequantize_q4_0", 32), ("gq_dequantize_ksb", 256)])
def test_dequantize_validation(name, block):
    f = getattr(gq.lib, name)
    assert f(A, -1, A, None) == INVALID
    assert f(A, block + 32 if block == 256 else 33, A, None) == SHAPE
    assert f(None, 0, None, None) == GQ_OK
    assert f(None, block, A, None) == INVALID
    assert f(A + 8, block, A, None) == ALIGN
    assert f(A, block, A + 12, None) == ALIGN


@pytest.mark.parametrize("name,block", [("gq_gemv_q4_0", 32), ("gq_gemv_ksb", 256)])
def test_gemv_validation(name, block):
    f = getattr(gq.lib, name)
    K = 4 * block
    ok = dict(W=A, M=64, K=K, x=A, xt=1, B=1, y=A, yt=1, ws=None, wsb=0, flags=0, st=None,
              s=None)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["W"], a["M"], a["K"], a["x"], a["xt"], a["B"], a["y"], a["yt"], a["ws"],
                 a["wsb"], a["flags"], a["st"], a["s"])

    assert call(M=-1) == INVALID
    assert call(K=-block) == INVALID
    assert call(B=-1) == INVALID
    assert call(xt=7) == DTYPE
    assert call(yt=-1) == DTYPE
    assert call(flags=2) == INVALID
    assert call(K=K + 16) == SHAPE
    assert call(B=9) == SHAPE
    assert call(K=1 << 25) == SHAPE
    assert call(M=0) == GQ_OK and call(B=0) == GQ_OK     # empty: no launch
    assert call(y=None) == INVALID
    assert call(W=None) == INVALID
    assert call(x=None) == INVALID
    assert call(W=A + 2) == ALIGN
    assert call(x=A + 8) == ALIGN
    assert call(y=A + 4) == ALIGN
    assert call(st=A + 2) == ALIGN


def test_gemv_grouped_validation():
    import ctypes
    D = gq.GemvDesc
    for name in ("gq_gemv_q4_0_grouped", "gq_gemv_ksb_grouped"):
        f = getattr(gq.lib, name)
        K = 256

        def call(descs, count=None, K=K, x=A, xt=1, B=1, yt=1, flags=0, st=None):
            arr = (D * max(len(descs), 1))(*descs)
            n = len(descs) if count is None else count
            return f(ctypes.cast(arr, ctypes.c_void_p), n, K, x, xt, B, yt, flags, st, None)

        good = D(A, 16, A + 4096)
        assert call([good], count=-1) == INVALID
        assert f(None, 1, K, A, 1, 1, 1, 0, None, None) == INVALID
        assert call([D(A, -1, A)]) == INVALID
        assert call([good, D(A + 2, 16, A)]) == ALIGN           # every descriptor is checked
        assert call([good, D(A, 16, A + 8)]) == ALIGN
        assert call([good, D(None, 16, A)]) == INVALID
        assert call([good, D(A, 16, None)]) == INVALID
        assert call([good], K=K + 16) == SHAPE
        assert call([good], B=9) == SHAPE
        assert call([good], xt=7) == DTYPE and call([good], yt=7) == DTYPE
        assert call([good], flags=2) == INVALID
        assert call([good], x=None) == INVALID and call([good], x=A + 2) == ALIGN
        assert call([good], st=A + 2) == ALIGN
        assert call([], count=0) == GQ_OK                      # nothing to do: no launch
        assert call([D(None, 0, None), D(None, 0, None)]) == GQ_OK
        assert call([good], B=0) == GQ_OK


def test_gemv_tiled_grouped_validation():
    import ctypes
    D = gq.GemvDesc
    for name, K in (("gq_gemv_q4_0_tiled_grouped", 64), ("gq_gemv_ksb_tiled_grouped", 256)):
        f = getattr(gq.lib, name)

        def call(descs, count=None, K=K, x=A, xt=gq.GQ_F16, yt=gq.GQ_F16, flags=0, st=None):
            arr = (D * max(len(descs), 1))(*descs)
            n = len(descs) if count is None else count
            return f(ctypes.cast(arr, ctypes.c_void_p), n, K, x, xt, yt, flags, st, None)

        good = D(A, 16, A + 4096)
        assert call([good], count=-1) == INVALID
        assert f(None, 1, K, A, gq.GQ_F16, gq.GQ_F16, 0, None, None) == INVALID
        assert call([D(A, -1, A)]) == INVALID
        assert call([good, D(A + 2, 16, A)]) == ALIGN           # every descriptor is checked
        assert call([good, D(A, 16, A + 8)]) == ALIGN
        assert call([good, D(None, 16, A)]) == INVALID
        assert call([good, D(A, 16, None)]) == INVALID
        assert call([good], K=K + 32) == SHAPE                 # not whole tiles of units
        assert call([good], K=16384 + 256) == SHAPE
        assert call([good], xt=gq.GQ_BF16) == DTYPE and call([good], yt=7) == DTYPE
        assert call([good], flags=2) == INVALID
        assert call([good], x=None) == INVALID and call([good], x=A + 2) == ALIGN
        assert call([good], st=A + 2) == ALIGN
        assert call([], count=0) == GQ_OK                      # nothing to do: no launch
        assert call([D(None, 0, None), D(None, 0, None)]) == GQ_OK


def test_binding_refuses_host_tensors():
    import torch
    with pytest.raises(ValueError):
        gq.gq_quantize_q4_0(torch.zeros(64))


@pytest.mark.parametrize("name,block", [("gq_gemm_q4_0", 32), ("gq_gemm_ksb", 256)])
def test_gemm_validation(name, block):
    f = getattr(gq.lib, name)
    K = 4 * block
    ok = dict(W=A, M=128, K=K, X=A, xt=2, B=16, Y=A, yt=0, ws=None, wsb=0, st=None, s=None)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["W"], a["M"], a["K"], a["X"], a["xt"], a["B"], a["Y"], a["yt"], a["ws"],
                 a["wsb"], a["st"], a["s"])

    assert call(M=-1) == INVALID
    assert call(B=-2) == INVALID
    assert call(xt=1) == DTYPE          # X must be bfloat16
    assert call(yt=5) == DTYPE
    assert call(K=K + 16) == SHAPE
    assert call(B=257) == SHAPE
    assert call(M=0) == GQ_OK and call(B=0) == GQ_OK
    assert call(Y=None) == INVALID
    assert call(W=None) == INVALID
    assert call(X=None) == INVALID
    assert call(W=A + 2) == ALIGN
    assert call(X=A + 8) == ALIGN
    assert call(st=A + 1) == ALIGN
    # a valid call without (or with too small) a workspace is refused before
    # any launch
    assert call() == 9
    need = gq.gq_gemm_workspace_bytes(0, 128, K, 16)
    assert need > 0
    assert call(ws=A, wsb=need - 1) == 9
    assert call(ws=A + 16, wsb=need) == ALIGN
    # counts of the 86 tiles, then two 128 x 256 fp32 parts per SM
    big = gq.gq_gemm_workspace_bytes(0, 11008, 4096, 256)
    assert big >= 2 * 128 * 256 * 4 and big % 256 == 0


def test_gemv_workspace_sizes_and_checks():
    f = gq.lib.gq_gemv_q4_0
    Q40, KSB = gq.GQ_FMT_Q4_0, gq.GQ_FMT_KSB
    need = gq.gq_gemv_workspace_bytes(Q40, 4096, 11008, 1, gq.GQ_F16)
    # counts and partial sums of the SMs; the same for every eligible shape
    assert need > 0
    assert gq.gq_gemv_workspace_bytes(Q40, 17, 256, 1, gq.GQ_F16) == need
    # only batch-1 fp16 Q4_0 with K % 256 == 0 uses a workspace
    assert gq.gq_gemv_workspace_bytes(Q40, 4096, 11008, 2, gq.GQ_F16) == 0
    assert gq.gq_gemv_workspace_bytes(Q40, 4096, 11008, 1, gq.GQ_BF16) == 0
    assert gq.gq_gemv_workspace_bytes(Q40, 4096, 288, 1, gq.GQ_F16) == 0
    assert gq.gq_gemv_workspace_bytes(KSB, 4096, 11008, 1, gq.GQ_F16) == 0
    assert gq.gq_gemv_workspace_bytes(Q40, 0, 4096, 1, gq.GQ_F16) == 0
    args = (A, 4096, 11008, A, 1, 1, A, 1)
    # too small, then misaligned: both refused before any launch
    assert f(*args, A, need - 1, 0, None, None) == 9
    assert f(*args, A + 16, need, 0, None, None) == ALIGN


def test_stream_read_validation():
    f = gq.lib.gq_stream_read
    assert f(A, 64, None, None) == INVALID  # no sink
    assert f(None, 64, A, None) == INVALID  # bytes but no buffer
    assert f(A, 40, A, None) == SHAPE  # not whole 16-byte granules
    assert f(A + 8, 64, A, None) == ALIGN  # buffer off a 16-byte boundary
    assert f(A, 64, A + 2, None) == ALIGN  # sink off a 4-byte boundary
    assert f(None, 0, A, None) == GQ_OK  # nothing to read: no launch


def test_tiled_sizes_and_validation():
    Q, KS = gq.GQ_FMT_Q4_0, gq.GQ_FMT_KSB
    assert gq.gq_tiled_bytes(Q, 16, 64) == 16 * 36
    assert gq.gq_tiled_bytes(Q, 17, 11008) == 32 * 6192
    assert gq.gq_tiled_bytes(KS, 4096, 11008) == 4096 * 5934
    for fmt, bad_k in ((Q, 96), (Q, 32), (KS, 128), (KS, 2304 + 32)):
        assert gq.gq_tiled_bytes(fmt, 16, bad_k) == 0
    assert gq.gq_tiled_bytes(7, 16, 64) == 0 and gq.gq_tiled_bytes(Q, -1, 64) == 0
    for name, k in (("gq_repack_q4_0", 64), ("gq_repack_ksb", 256)):
        f = getattr(gq.lib, name)
        assert f(A, -1, k, A, None) == INVALID
        assert f(A, 16, k + 32, A, None) == SHAPE
        assert f(A + 8, 16, k, A, None) == ALIGN
        assert f(None, 16, k, A, None) == INVALID
        assert f(A, 0, k, A, None) == GQ_OK  # nothing to do
    for name, k in (("gq_gemv_q4_0_tiled", 64), ("gq_gemv_ksb_tiled", 256)):
        f = getattr(gq.lib, name)
        assert f(A, 16, k, A, gq.GQ_BF16, A, gq.GQ_F16, 0, None, None) == DTYPE
        assert f(A, 16, k, A, gq.GQ_F16, A, 9, 0, None, None) == DTYPE
        assert f(A, 16, k + 32, A, gq.GQ_F16, A, gq.GQ_F16, 0, None, None) == SHAPE
        assert f(A, 16, 16384 + 256, A, gq.GQ_F16, A, gq.GQ_F16, 0, None, None) == SHAPE
        assert f(A, 16, k, A, gq.GQ_F16, A, gq.GQ_F16, 2, None, None) == INVALID
        assert f(A + 2, 16, k, A, gq.GQ_F16, A, gq.GQ_F16, 0, None, None) == ALIGN
        assert f(A, 16, k, A, gq.GQ_F16, None, gq.GQ_F16, 0, None, None) == INVALID
        assert f(A, -1, k, A, gq.GQ_F16, A, gq.GQ_F16, 0, None, None) == INVALID
        assert f(A, 0, k, A, gq.GQ_F16, A, gq.GQ_F16, 0, None, None) == GQ_OK
