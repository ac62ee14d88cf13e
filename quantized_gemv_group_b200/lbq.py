"""ctypes binding of liblbq.so (the C ABI declared in include/lbq.h).

Argument marshalling only: every function forwards torch tensors' device
pointers, sizes and the current CUDA stream to the C entry point of the same
name and raises LbqError on a non-OK status.  Output tensors are allocated with
torch when not supplied.  There is no fallback: if liblbq.so is missing or a
tensor is not on a CUDA device, the call fails.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblbq.so")

# lbq_status
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_MISALIGNED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_DEVICE, \
    ERR_SCRATCH_LIMIT = range(9)
# lbq_dtype / lbq_layout / lbq_op
F16, BF16 = 0, 1
LAYOUT_CANONICAL, LAYOUT_KERNEL = 0, 1
OP_GEMV_GROUP, OP_GEMM_GROUP, OP_GEMV_BINLR, OP_GEMM_BINLR = range(4)


MAX_GEMV_PROBLEMS = 8


class GemvProblem(ctypes.Structure):
    """lbq_gemv_problem: one product of a grouped GEMV launch."""
    _fields_ = [("x", ctypes.c_void_p), ("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("zeros", ctypes.c_void_p), ("y", ctypes.c_void_p), ("n", ctypes.c_int64), ("k", ctypes.c_int64)]


class LbqError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lib = None


def lib():
    """Load liblbq.so (raises OSError if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OSError(f"liblbq.so not found at {LIB_PATH}; run quantized_gemv_group_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        i64, i32, p, sz = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
        sig = {
            "lbq_version": (ctypes.c_char_p, []),
            "lbq_status_string": (ctypes.c_char_p, [i32]),
            "lbq_packed_bytes": (sz, [i64, i64, i32, i32]),
            "lbq_quantize_rtn": (i32, [p, i32, i64, i64, i32, i32, p, p, p, p]),
            "lbq_pack": (i32, [p, i64, i64, i32, i32, p, p]),
            "lbq_unpack": (i32, [p, i64, i64, i32, i32, p, p]),
            "lbq_sign_packed_bytes": (sz, [i64, i64, i32]),
            "lbq_pack_signs": (i32, [p, i64, i64, i32, p, p]),
            "lbq_repack_signs": (i32, [p, i64, i64, p, p]),
            "lbq_workspace_bytes": (sz, [i32, i64, i64, i64, i64]),
            "lbq_gemv_group": (i32, [p, i32, i64, p, p, p, i64, i64, i32, i32, i32, p, p, sz, p]),
            "lbq_gemm_group": (i32, [p, i32, i64, p, p, p, i64, i64, i32, i32, i32, p, p, sz, p]),
            "lbq_gemv_binlr": (i32, [p, i32, i64, p, p, p, p, i64, i64, i64, i32, p, p, sz, p]),
            "lbq_gemm_binlr": (i32, [p, i32, i64, p, p, p, p, i64, i64, i64, i32, p, p, sz, p]),
            "lbq_schedule_bits": (i32, [i32, i32, i32]),
            "lbq_gemv_group_multi_workspace_bytes": (sz, [p, i32, i64]),
            "lbq_gemv_group_multi": (i32, [p, i32, i32, i64, i32, i32, p, sz, p]),
            "lbq_gemv_group_noalloc": (i32, [p, i32, i64, p, p, p, i64, i64, i32, i32, p, p]),
            "lbq_last_device_error": (i32, [p, ctypes.POINTER(ctypes.c_int)]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(status):
    return lib().lbq_status_string(int(status)).decode()


def version():
    return lib().lbq_version().decode()


def _check(status, where):
    if status != OK:
        raise LbqError(status, where)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("liblbq operates on CUDA tensors only")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.float16:
        return F16
    if t.dtype == torch.bfloat16:
        return BF16
    raise ValueError(f"unsupported dtype {t.dtype}")


# ---------------------------------------------------------------- sizes
def lbq_packed_bytes(n, k, bits, layout=LAYOUT_KERNEL):
    return int(lib().lbq_packed_bytes(n, k, bits, layout))


def lbq_sign_packed_bytes(rows, cols, layout=LAYOUT_KERNEL):
    return int(lib().lbq_sign_packed_bytes(rows, cols, layout))


def lbq_workspace_bytes(op, M, n, k, r=0):
    return int(lib().lbq_workspace_bytes(op, M, n, k, r))


def lbq_schedule_bits(layer, proj, n_layers=80):
    return int(lib().lbq_schedule_bits(layer, proj, n_layers))


# ---------------------------------------------------------------- workspace
class Workspace:
    """Zero-filled device workspace, grown on demand (calls leave it reusable)."""

    def __init__(self, device=None):
        self.device = device or torch.device("cuda", torch.cuda.current_device())
        self.buf = torch.zeros(0, dtype=torch.uint8, device=self.device)

    def get(self, nbytes):
        if self.buf.numel() < nbytes:
            self.buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        return self.buf


_default_ws = {}


def _ws_for(nbytes, device):
    key = (device.type, device.index)
    if key not in _default_ws:
        _default_ws[key] = Workspace(device)
    return _default_ws[key].get(nbytes)


# ---------------------------------------------------------------- quantize / pack
def lbq_quantize_rtn(W, bits, group, codes=None, scales=None, zeros=None, stream=None):
    n, k = W.shape
    dev = W.device
    codes = codes if codes is not None else torch.empty(n, k, dtype=torch.uint8, device=dev)
    G = k // group if group else 0
    scales = scales if scales is not None else torch.empty(n, G, dtype=torch.float16, device=dev)
    zeros = zeros if zeros is not None else torch.empty(n, G, dtype=torch.float16, device=dev)
    _check(lib().lbq_quantize_rtn(_ptr(W), _dtype_code(W), n, k, bits, group, _ptr(codes), _ptr(scales),
                                  _ptr(zeros), _stream(stream)), "lbq_quantize_rtn")
    return codes, scales, zeros


def lbq_pack(codes, bits, layout=LAYOUT_KERNEL, packed=None, stream=None):
    n, k = codes.shape
    nbytes = lbq_packed_bytes(n, k, bits, layout)
    if nbytes == 0 and n * k > 0:
        raise LbqError(ERR_UNSUPPORTED, "lbq_pack")
    packed = packed if packed is not None else torch.empty(nbytes, dtype=torch.uint8, device=codes.device)
    _check(lib().lbq_pack(_ptr(codes), n, k, bits, layout, _ptr(packed), _stream(stream)), "lbq_pack")
    return packed


def lbq_unpack(packed, n, k, bits, layout=LAYOUT_KERNEL, codes=None, stream=None):
    codes = codes if codes is not None else torch.empty(n, k, dtype=torch.uint8, device=packed.device)
    _check(lib().lbq_unpack(_ptr(packed), n, k, bits, layout, _ptr(codes), _stream(stream)), "lbq_unpack")
    return codes


def lbq_pack_signs(pm1, layout=LAYOUT_KERNEL, out=None, stream=None):
    rows, cols = pm1.shape
    nbytes = lbq_sign_packed_bytes(rows, cols, layout)
    out = out if out is not None else torch.empty(nbytes, dtype=torch.uint8, device=pm1.device)
    _check(lib().lbq_pack_signs(_ptr(pm1), rows, cols, layout, _ptr(out), _stream(stream)), "lbq_pack_signs")
    return out


def lbq_repack_signs(words, rows, cols, out=None, stream=None):
    nbytes = lbq_sign_packed_bytes(rows, cols, LAYOUT_KERNEL)
    out = out if out is not None else torch.empty(nbytes, dtype=torch.uint8, device=words.device)
    _check(lib().lbq_repack_signs(_ptr(words), rows, cols, _ptr(out), _stream(stream)), "lbq_repack_signs")
    return out


# ---------------------------------------------------------------- products
def _group_call(fn, name, op, x, packed, scales, zeros, n, k, bits, group, layout, y, ws, stream):
    M = x.shape[0] if x.dim() == 2 else 1
    y = y if y is not None else torch.empty(M, n, dtype=torch.float16, device=x.device)
    need = lbq_workspace_bytes(op, M, n, k)
    if ws is None:
        ws = _ws_for(need, x.device)
    _check(fn(_ptr(x), _dtype_code(x), M, _ptr(packed), _ptr(scales), _ptr(zeros), n, k, bits, group, layout,
              _ptr(y), _ptr(ws) if ws.numel() else None, ws.numel(), _stream(stream)), name)
    return y


def _problem_array(problems):
    arr = (GemvProblem * len(problems))()
    for i, pr in enumerate(problems):
        x, packed, scales, zeros, y, n, k = pr
        arr[i] = GemvProblem(_ptr(x), _ptr(packed), _ptr(scales), _ptr(zeros), _ptr(y), n, k)
    return arr


def lbq_gemv_group_multi_workspace_bytes(problems, M):
    arr = _problem_array(problems)
    return int(lib().lbq_gemv_group_multi_workspace_bytes(ctypes.cast(arr, ctypes.c_void_p), len(problems), M))


def lbq_gemv_group_multi(problems, bits, group, ws=None, stream=None):
    """problems: list of (x [M,k], packed, scales, zeros, y [M,n] fp16, n, k) sharing M and x dtype."""
    if not problems:
        raise ValueError("no problems")
    x0 = problems[0][0]
    M = x0.shape[0] if x0.dim() == 2 else 1
    arr = _problem_array(problems)
    need = int(lib().lbq_gemv_group_multi_workspace_bytes(ctypes.cast(arr, ctypes.c_void_p), len(problems), M))
    if ws is None:
        ws = _ws_for(need, x0.device)
    _check(lib().lbq_gemv_group_multi(ctypes.cast(arr, ctypes.c_void_p), len(problems), _dtype_code(x0), M, bits,
                                      group, _ptr(ws) if ws.numel() else None, ws.numel(), _stream(stream)),
           "lbq_gemv_group_multi")
    return [pr[4] for pr in problems]


def lbq_gemv_group_noalloc(x, packed, scales, zeros, n, k, bits, group, y=None, stream=None):
    """Group GEMV (kernel layout) without a workspace: scratch is the library's fixed array."""
    M = x.shape[0] if x.dim() == 2 else 1
    y = y if y is not None else torch.empty(M, n, dtype=torch.float16, device=x.device)
    _check(lib().lbq_gemv_group_noalloc(_ptr(x), _dtype_code(x), M, _ptr(packed), _ptr(scales), _ptr(zeros), n, k,
                                        bits, group, _ptr(y), _stream(stream)), "lbq_gemv_group_noalloc")
    return y


def lbq_gemv_group(x, packed, scales, zeros, n, k, bits, group, layout=LAYOUT_KERNEL, y=None, ws=None,
                   stream=None):
    return _group_call(lib().lbq_gemv_group, "lbq_gemv_group", OP_GEMV_GROUP, x, packed, scales, zeros, n, k,
                       bits, group, layout, y, ws, stream)


def lbq_gemm_group(x, packed, scales, zeros, n, k, bits, group, layout=LAYOUT_KERNEL, y=None, ws=None,
                   stream=None):
    return _group_call(lib().lbq_gemm_group, "lbq_gemm_group", OP_GEMM_GROUP, x, packed, scales, zeros, n, k,
                       bits, group, layout, y, ws, stream)


def _binlr_call(fn, name, op, x, U, Vt, s1, s2, d_out, d_in, r, layout, y, ws, stream):
    M = x.shape[0] if x.dim() == 2 else 1
    y = y if y is not None else torch.empty(M, d_out, dtype=torch.float16, device=x.device)
    need = lbq_workspace_bytes(op, M, d_out, d_in, r)
    if ws is None:
        ws = _ws_for(need, x.device)
    _check(fn(_ptr(x), _dtype_code(x), M, _ptr(U), _ptr(Vt), _ptr(s1), _ptr(s2), d_out, d_in, r, layout,
              _ptr(y), _ptr(ws) if ws.numel() else None, ws.numel(), _stream(stream)), name)
    return y


def lbq_gemv_binlr(x, U, Vt, s1, s2, d_out, d_in, r, layout=LAYOUT_KERNEL, y=None, ws=None, stream=None):
    return _binlr_call(lib().lbq_gemv_binlr, "lbq_gemv_binlr", OP_GEMV_BINLR, x, U, Vt, s1, s2, d_out, d_in, r,
                       layout, y, ws, stream)


def lbq_gemm_binlr(x, U, Vt, s1, s2, d_out, d_in, r, layout=LAYOUT_KERNEL, y=None, ws=None, stream=None):
    return _binlr_call(lib().lbq_gemm_binlr, "lbq_gemm_binlr", OP_GEMM_BINLR, x, U, Vt, s1, s2, d_out, d_in, r,
                       layout, y, ws, stream)


def lbq_last_device_error(stream=None):
    code = ctypes.c_int(0)
    _check(lib().lbq_last_device_error(_stream(stream), ctypes.byref(code)), "lbq_last_device_error")
    return code.value
