"""CPU oracle for the low-bit weight GEMV (test infrastructure only).

Thin numpy/ctypes front end over ``lbq_oracle.c`` (plain scalar C, fp64
accumulation, strict IEEE binary32 for the quantizer steps).  Only the tests,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import this package.  It shares no code with the CUDA
library ``quantized_gemv_group_b200``; it only receives the same input arrays.

Every array argument is a numpy array.  Half-precision values travel as their
uint16 bit patterns (``np.float16(...).view(np.uint16)`` or a torch tensor's
``.view(torch.int16)``), so that no conversion happens on the way in.

Function map (pages cited by title and section):

* ``quantize_rtn`` -- "Métodos de cuantización de LLM para ejecutar un modelo
  de 70B en una sola GPU", section "RTN (Round-To-Nearest)", with the blocks of
  "TurboQuant: cuantizar modelos grandes para que quepan en local", section
  "Compresión por bloques" (shared scale and offset per block).
* ``pack`` / ``unpack`` -- the bit layouts (readings R7, R8 in lbq_oracle.c).
* ``gemv_group`` -- dequantize-then-multiply in fp64, y = x · Ŵᵀ.
* ``binlr_dense`` / ``binlr_factored`` -- "70B en 4GB de VRAM: la compresión
  neural de 2026, ¿es real?", section "1. NanoQuant — sub-1-bit PTQ", bullet
  "Formulación": Ŵ = diag(s1)·U·Vᵀ·diag(s2), y = s1 ⊙ U(Vᵀ(s2 ⊙ x)).
"""
import ctypes
import numpy as np

from .build import build_oracle

_lib = None

LAYOUT_CANONICAL = 0
LAYOUT_KERNEL = 1


def _L():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build_oracle())
        i64, i32, p = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        sig = {
            "orc_f16_decode": (ctypes.c_double, [ctypes.c_uint16]),
            "orc_bf16_decode": (ctypes.c_double, [ctypes.c_uint16]),
            "orc_f32_to_f16_ru": (ctypes.c_uint16, [ctypes.c_float]),
            "orc_f16_decode_array": (None, [p, i64, p]),
            "orc_f32_to_f16_ru_array": (None, [p, i64, p]),
            "orc_quantize_rtn": (i32, [p, i32, i64, i64, i32, i32, p, p, p]),
            "orc_pack_canonical": (i32, [p, i64, i64, i32, p]),
            "orc_unpack_canonical": (i32, [p, i64, i64, i32, p]),
            "orc_pack_kernel": (i32, [p, i64, i64, i32, p]),
            "orc_unpack_kernel": (i32, [p, i64, i64, i32, p]),
            "orc_gemv_group": (i32, [p, i32, i64, p, i32, p, p, i64, i64, i32, i32, p, i64, p]),
            "orc_gemv_dense": (i32, [p, i32, i64, p, i64, i64, p, i64, p]),
            "orc_binlr_dense": (i32, [p, i32, i64, p, p, p, p, i64, i64, i64, p]),
            "orc_binlr_factored": (i32, [p, i32, i64, p, p, p, p, i64, i64, i64, p, i64, p, p]),
            "orc_pack_signs": (i32, [p, i64, i64, p]),
            "orc_sign_cols_pad": (i64, [i64]),
            "orc_pack_signs_kernel": (i32, [p, i64, i64, p]),
            "orc_unpack_signs_kernel": (i32, [p, i64, i64, p]),
            "orc_num_threads": (i32, []),
            "orc_set_num_threads": (None, [i32]),
        }
        for name, (res, args) in sig.items():
            f = getattr(_lib, name)
            f.restype = res
            f.argtypes = args
    return _lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


# --------------------------------------------------------------------- scalars
def f16_decode(bits):
    b = _c(np.atleast_1d(bits), np.uint16)
    out = np.empty(b.shape, np.float64)
    _L().orc_f16_decode_array(_ptr(b), b.size, _ptr(out))
    return out


def bf16_decode(bits):
    b = _c(np.atleast_1d(bits), np.uint16)
    return np.array([_L().orc_bf16_decode(int(v)) for v in b.ravel()]).reshape(b.shape)


def f32_to_f16_ru(values):
    v = _c(np.atleast_1d(values), np.float32)
    out = np.empty(v.shape, np.uint16)
    _L().orc_f32_to_f16_ru_array(_ptr(v), v.size, _ptr(out))
    return out


def num_threads():
    return _L().orc_num_threads()


def set_num_threads(n):
    _L().orc_set_num_threads(int(n))


# ------------------------------------------------------------------ quantizer
def quantize_rtn(W_bits, bits, group, w_is_bf16=False):
    """Group-wise asymmetric RTN.  W_bits: uint16 [n, k] (fp16 or bf16 bits).
    Returns (codes u8 [n,k], scales u16 [n,k/g], zeros u16 [n,k/g])."""
    W = _c(W_bits, np.uint16)
    n, k = W.shape
    codes = np.empty((n, k), np.uint8)
    G = k // group if group > 0 else 0
    scales = np.empty((n, max(G, 1)), np.uint16)
    zeros = np.empty((n, max(G, 1)), np.uint16)
    rc = _L().orc_quantize_rtn(_ptr(W), int(w_is_bf16), n, k, bits, group,
                               _ptr(codes), _ptr(scales), _ptr(zeros))
    if rc == -1:
        raise FloatingPointError("non-finite weight")
    _check(rc, "quantize_rtn")
    return codes, scales[:, :G], zeros[:, :G]


# --------------------------------------------------------------------- packing
def packed_bytes(n, k, bits):
    return n * k * bits // 8


def pack(codes, bits, layout=LAYOUT_CANONICAL):
    c = _c(codes, np.uint8)
    n, k = c.shape
    out = np.empty(packed_bytes(n, k, bits), np.uint8)
    f = _L().orc_pack_canonical if layout == LAYOUT_CANONICAL else _L().orc_pack_kernel
    _check(f(_ptr(c), n, k, bits, _ptr(out)), "pack")
    return out


def unpack(packed, n, k, bits, layout=LAYOUT_CANONICAL):
    p = _c(packed, np.uint8).ravel()
    codes = np.empty((n, k), np.uint8)
    f = _L().orc_unpack_canonical if layout == LAYOUT_CANONICAL else _L().orc_unpack_kernel
    _check(f(_ptr(p), n, k, bits, _ptr(codes)), "unpack")
    return codes


def pack_signs(pm1):
    a = _c(pm1, np.int8)
    rows, cols = a.shape
    out = np.empty((rows, cols // 32), np.uint32)
    _check(_L().orc_pack_signs(_ptr(a), rows, cols, _ptr(out)), "pack_signs")
    return out


def sign_cols_pad(cols):
    return int(_L().orc_sign_cols_pad(cols))


def pack_signs_kernel(words, rows, cols):
    w = _c(words, np.uint32)
    out = np.empty(rows * sign_cols_pad(cols) // 8, np.uint8)
    _check(_L().orc_pack_signs_kernel(_ptr(w), rows, cols, _ptr(out)), "pack_signs_kernel")
    return out


def unpack_signs_kernel(packed, rows, cols):
    p = _c(packed, np.uint8).ravel()
    out = np.empty((rows, cols // 32), np.uint32)
    _check(_L().orc_unpack_signs_kernel(_ptr(p), rows, cols, _ptr(out)), "unpack_signs_kernel")
    return out


# ----------------------------------------------------------------- products
def _rows_arg(rows):
    if rows is None:
        return None, 0
    r = _c(rows, np.int64)
    return r, r.size


def gemv_group(x_bits, packed, scales, zeros, n, k, bits, group,
               layout=LAYOUT_CANONICAL, rows=None, x_is_bf16=False):
    """y[m, j] = sum_k x[m,k] * s[i,k/g] * (q[i,k] - z[i,k/g]) for i = rows[j]; fp64."""
    x = _c(np.atleast_2d(x_bits), np.uint16)
    M = x.shape[0]
    assert x.shape[1] == k
    p = _c(packed, np.uint8).ravel()
    s = _c(scales, np.uint16)
    z = _c(zeros, np.uint16)
    r, nr = _rows_arg(rows)
    y = np.empty((M, nr if r is not None else n), np.float64)
    _check(_L().orc_gemv_group(_ptr(x), int(x_is_bf16), M, _ptr(p), layout, _ptr(s), _ptr(z),
                               n, k, bits, group, _ptr(r), nr, _ptr(y)), "gemv_group")
    return y


def gemv_dense(x_bits, W_bits, rows=None, x_is_bf16=False):
    x = _c(np.atleast_2d(x_bits), np.uint16)
    W = _c(W_bits, np.uint16)
    n, k = W.shape
    M = x.shape[0]
    r, nr = _rows_arg(rows)
    y = np.empty((M, nr if r is not None else n), np.float64)
    _check(_L().orc_gemv_dense(_ptr(x), int(x_is_bf16), M, _ptr(W), n, k, _ptr(r), nr, _ptr(y)),
           "gemv_dense")
    return y


def binlr_dense(x_bits, U, Vt, s1, s2, d_out, d_in, r, x_is_bf16=False):
    x = _c(np.atleast_2d(x_bits), np.uint16)
    M = x.shape[0]
    y = np.empty((M, d_out), np.float64)
    _check(_L().orc_binlr_dense(_ptr(x), int(x_is_bf16), M, _ptr(_c(U, np.uint32)),
                                _ptr(_c(Vt, np.uint32)), _ptr(_c(s1, np.uint16)),
                                _ptr(_c(s2, np.uint16)), d_out, d_in, r, _ptr(y)), "binlr_dense")
    return y


def binlr_factored(x_bits, U, Vt, s1, s2, d_out, d_in, r, rows=None, x_is_bf16=False,
                   return_t=False):
    x = _c(np.atleast_2d(x_bits), np.uint16)
    M = x.shape[0]
    rr, nr = _rows_arg(rows)
    y = np.empty((M, nr if rr is not None else d_out), np.float64)
    t = np.empty((M, r), np.float64) if return_t else None
    _check(_L().orc_binlr_factored(_ptr(x), int(x_is_bf16), M, _ptr(_c(U, np.uint32)),
                                   _ptr(_c(Vt, np.uint32)), _ptr(_c(s1, np.uint16)),
                                   _ptr(_c(s2, np.uint16)), d_out, d_in, r, _ptr(rr), nr,
                                   _ptr(y), _ptr(t)), "binlr_factored")
    return (y, t) if return_t else y


def rel_l2(a, b):
    """||a - b||_2 / ||b||_2 in fp64 (b is the oracle's result)."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b.ravel())
    return float(np.linalg.norm((a - b).ravel()) / (den if den > 0 else 1.0))
