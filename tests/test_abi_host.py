"""Host-only checks of the C ABI: the library loads without a GPU, exports
every function include/lbq.h declares, and rejects bad arguments with the
documented status before touching the device (fake, never-dereferenced
pointers are passed on purpose; every call below fails its host checks)."""
import ctypes
import os
import re

import pytest

from quantized_gemv_group_b200 import build as lbq_build
from quantized_gemv_group_b200 import lbq, workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lbq.h")


@pytest.fixture(scope="module")
def L():
    lbq_build.build()
    return lbq.lib()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lbq_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert len(names) >= 16
    for n in names:
        assert hasattr(L, n), n


def test_version_and_status_strings(L):
    assert re.match(r"^\d+\.\d+\.\d+$", lbq.version())
    for s in range(9):
        assert lbq.status_string(s)
    assert lbq.status_string(0) == "ok"


def test_packed_bytes_closed_forms(L):
    for b in range(2, 7):
        assert lbq.lbq_packed_bytes(8192, 8192, b, lbq.LAYOUT_CANONICAL) == 8192 * 8192 * b // 8
        assert lbq.lbq_packed_bytes(8192, 28672, b, lbq.LAYOUT_KERNEL) == 8192 * 28672 * b // 8
    assert lbq.lbq_packed_bytes(17, 256, 4, lbq.LAYOUT_KERNEL) == 0      # rows not multiple of 16
    assert lbq.lbq_packed_bytes(16, 96, 3, lbq.LAYOUT_KERNEL) == 0       # k not multiple of 256
    assert lbq.lbq_packed_bytes(16, 96, 3, lbq.LAYOUT_CANONICAL) == 16 * 96 * 3 // 8
    assert lbq.lbq_packed_bytes(16, 100, 4, lbq.LAYOUT_CANONICAL) == 0   # k % 32 != 0
    assert lbq.lbq_sign_packed_bytes(3264, 8192, lbq.LAYOUT_KERNEL) == 3264 * 8192 // 8
    assert lbq.lbq_sign_packed_bytes(8192, 3264, lbq.LAYOUT_KERNEL) == 8192 * 3328 // 8
    assert lbq.lbq_sign_packed_bytes(8192, 3264, lbq.LAYOUT_CANONICAL) == 8192 * 3264 // 8


def test_schedule_matches_host_table(L):
    names = list(workloads.PROJS)
    for layer in range(80):
        for p, name in enumerate(names):
            assert lbq.lbq_schedule_bits(layer, p, 80) == workloads.schedule_bits(layer, name)
    assert lbq.lbq_schedule_bits(80, 0, 80) == 0
    assert lbq.lbq_schedule_bits(0, 7, 80) == 0


P = ctypes.c_void_p
A16 = P(0x10000)        # 16-byte aligned fake device addresses (never dereferenced)
B16 = P(0x20000)
C16 = P(0x30000)
D16 = P(0x40000)
E16 = P(0x50000)
ODD = P(0x10002)


def _gemv(L, x=A16, M=1, packed=B16, s=C16, z=D16, n=256, k=256, bits=4, group=32, layout=1, y=E16,
          ws=None, wsb=0, fn="lbq_gemv_group", dt=0):
    return getattr(L, fn)(x, dt, M, packed, s, z, n, k, bits, group, layout, y, ws, wsb, None)


def test_gemv_group_argument_errors(L):
    assert _gemv(L, bits=7) == lbq.ERR_INVALID_ARG
    assert _gemv(L, bits=1) == lbq.ERR_INVALID_ARG
    assert _gemv(L, group=16) == lbq.ERR_INVALID_ARG
    assert _gemv(L, k=96, group=64) == lbq.ERR_INVALID_ARG
    assert _gemv(L, M=17) == lbq.ERR_INVALID_ARG
    assert _gemv(L, M=-1) == lbq.ERR_INVALID_ARG
    assert _gemv(L, dt=5) == lbq.ERR_INVALID_ARG
    assert _gemv(L, layout=3) == lbq.ERR_INVALID_ARG
    assert _gemv(L, packed=None) == lbq.ERR_INVALID_ARG
    assert _gemv(L, y=None) == lbq.ERR_INVALID_ARG
    assert _gemv(L, n=24) == lbq.ERR_UNSUPPORTED
    assert _gemv(L, bits=3, k=128, group=32) == lbq.ERR_UNSUPPORTED
    assert _gemv(L, x=ODD) == lbq.ERR_MISALIGNED
    assert _gemv(L, packed=ODD) == lbq.ERR_MISALIGNED
    # empty problems are valid no-ops
    assert _gemv(L, M=0) == lbq.OK
    assert _gemv(L, n=0) == lbq.OK
    # kernel layout needs a workspace (none given)
    assert _gemv(L, ws=None, wsb=0) == lbq.ERR_WORKSPACE
    assert _gemv(L, fn="lbq_gemm_group", M=40, ws=None, wsb=0) == lbq.ERR_WORKSPACE


def test_binlr_argument_errors(L):
    def call(M=1, U=A16, Vt=B16, s1=C16, s2=D16, d_out=256, d_in=256, r=64, layout=1, y=E16, x=A16,
             fn="lbq_gemv_binlr"):
        return getattr(L, fn)(x, 0, M, U, Vt, s1, s2, d_out, d_in, r, layout, y, None, 0, None)
    assert call(r=48) == lbq.ERR_INVALID_ARG
    assert call(d_in=100) == lbq.ERR_INVALID_ARG
    assert call(M=17) == lbq.ERR_INVALID_ARG
    assert call(U=None) == lbq.ERR_INVALID_ARG
    assert call(d_out=40) == lbq.ERR_UNSUPPORTED
    assert call(U=ODD) == lbq.ERR_MISALIGNED
    assert call(M=0) == lbq.OK
    assert call() == lbq.ERR_WORKSPACE
    assert call(fn="lbq_gemm_binlr", M=40) == lbq.ERR_WORKSPACE


def test_quantize_and_pack_argument_errors(L):
    q = L.lbq_quantize_rtn
    assert q(A16, 0, 16, 64, 7, 32, B16, C16, D16, None) == lbq.ERR_INVALID_ARG
    assert q(A16, 0, 16, 64, 4, 48, B16, C16, D16, None) == lbq.ERR_INVALID_ARG
    assert q(A16, 2, 16, 64, 4, 32, B16, C16, D16, None) == lbq.ERR_INVALID_ARG
    assert q(None, 0, 16, 64, 4, 32, B16, C16, D16, None) == lbq.ERR_INVALID_ARG
    assert q(P(0x10001), 0, 16, 64, 4, 32, B16, C16, D16, None) == lbq.ERR_MISALIGNED
    assert q(A16, 0, 0, 64, 4, 32, B16, C16, D16, None) == lbq.OK
    pk = L.lbq_pack
    assert pk(A16, 16, 100, 4, 0, B16, None) == lbq.ERR_INVALID_ARG
    assert pk(A16, 20, 64, 4, 1, B16, None) == lbq.ERR_UNSUPPORTED
    assert pk(ODD, 16, 64, 4, 0, B16, None) == lbq.ERR_MISALIGNED
    assert L.lbq_pack_signs(A16, 16, 40, 0, B16, None) == lbq.ERR_INVALID_ARG
    assert L.lbq_pack_signs(A16, 20, 64, 1, B16, None) == lbq.ERR_UNSUPPORTED
    assert L.lbq_repack_signs(A16, 20, 64, B16, None) == lbq.ERR_UNSUPPORTED
    assert L.lbq_last_device_error(None, None) == lbq.ERR_INVALID_ARG
