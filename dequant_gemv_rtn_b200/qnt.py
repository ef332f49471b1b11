"""Thin ctypes binding of libqnt (the C ABI declared in include/qnt.h).

Argument marshalling only: every computation runs in the CUDA kernels of
libqnt.so.  Functions keep the C names.  Device buffers may be passed as torch
tensors (their data_ptr is used) or as integer addresses; the stream defaults
to torch's current CUDA stream.  There is no CPU fallback: if libqnt.so is
missing or fails to load, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqnt.so")

QNT_INT4_ASYM, QNT_FP4_E2M1, QNT_FP4_AFPQ, QNT_FP4_RAZER, QNT_INT8_PERCHAN, QNT_FP16 = 1, 2, 3, 4, 5, 6
QNT_F16, QNT_BF16 = 0, 1
(QNT_OK, QNT_ERR_ARG, QNT_ERR_SHAPE, QNT_ERR_ALIGN, QNT_ERR_CUDA, QNT_ERR_TIMEOUT,
 QNT_ERR_NONFINITE, QNT_ERR_RANGE) = range(8)
FORMATS = {"int4": QNT_INT4_ASYM, "fp4": QNT_FP4_E2M1, "afpq": QNT_FP4_AFPQ, "razer": QNT_FP4_RAZER,
           "int8": QNT_INT8_PERCHAN, "fp16": QNT_FP16}


QNT_MAX_GEMV_K = 32768
QNT_SEQ_MAX_STEPS = 256
QNT_SEQ_NOALLOC_MAX_STEPS = 256


class qnt_desc(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("N", ctypes.c_int32), ("K", ctypes.c_int32), ("group", ctypes.c_int32)]


class qnt_seq_step(ctypes.Structure):
    _fields_ = [("desc", qnt_desc), ("codes", ctypes.c_void_p), ("meta", ctypes.c_void_p), ("x", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("wait", ctypes.c_int32), ("reserved", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libqnt.so not found at {LIB_PATH}; run `python -m dequant_gemv_rtn_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    D = ctypes.POINTER(qnt_desc)
    sig = {
        "qnt_version": (I, []),
        "qnt_check_desc": (I, [D]),
        "qnt_codes_bytes": (Z, [D]),
        "qnt_meta_bytes": (Z, [D]),
        "qnt_quantize": (I, [D, P, P, P, P, P]),
        "qnt_gemv": (I, [D, P, P, P, P, I, P, P]),
        "qnt_gemm": (I, [D, P, P, P, P, I, I, P, P]),
        "qnt_gemv_seq_work_bytes": (Z, [I]),
        "qnt_gemv_seq": (I, [ctypes.POINTER(qnt_seq_step), I, I, P, P, P]),
        "qnt_gemv_seq_noalloc": (I, [ctypes.POINTER(qnt_seq_step), I, I, P, P]),
        "qnt_table_create": (P, [I, I]),
        "qnt_table_set": (I, [P, ctypes.c_char_p, I, I]),
        "qnt_table_lookup": (I, [P, ctypes.c_char_p, ctypes.POINTER(I), ctypes.POINTER(I)]),
        "qnt_table_size": (I, [P]),
        "qnt_table_destroy": (None, [P]),
        "qnt_strerror": (ctypes.c_char_p, [I]),
        "qnt_last_error": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    return lib


lib = _load()


class QntError(RuntimeError):
    def __init__(self, code: int, what: str):
        extra = f" [{qnt_last_error()}]" if code == QNT_ERR_CUDA else ""
        super().__init__(f"{what}: {qnt_strerror(code)} (code {code}){extra}")
        self.code = code


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(code: int, what: str) -> int:
    if code != QNT_OK:
        raise QntError(code, what)
    return code


def desc(fmt: int, N: int, K: int, group: int | None = None) -> qnt_desc:
    if fmt in (QNT_INT8_PERCHAN, QNT_FP16):
        group = K
    return qnt_desc(int(fmt), int(N), int(K), int(group))


def qnt_version() -> int:
    return lib.qnt_version()


def qnt_strerror(code: int) -> str:
    return lib.qnt_strerror(int(code)).decode()


def qnt_last_error() -> str:
    return lib.qnt_last_error().decode()


def qnt_check_desc(d: qnt_desc) -> int:
    return lib.qnt_check_desc(ctypes.byref(d))


def qnt_codes_bytes(d: qnt_desc) -> int:
    return lib.qnt_codes_bytes(ctypes.byref(d))


def qnt_meta_bytes(d: qnt_desc) -> int:
    return lib.qnt_meta_bytes(ctypes.byref(d))


def qnt_quantize(d: qnt_desc, W, codes, meta, status=None, stream=None, check=True) -> int:
    rc = lib.qnt_quantize(ctypes.byref(d), _ptr(W), _ptr(codes), _ptr(meta), _ptr(status), _stream(stream))
    return _check(rc, "qnt_quantize") if check else rc


def qnt_gemv(d: qnt_desc, codes, meta, x, y, xdtype: int = QNT_F16, status=None, stream=None, check=True) -> int:
    rc = lib.qnt_gemv(ctypes.byref(d), _ptr(codes), _ptr(meta), _ptr(x), _ptr(y), int(xdtype), _ptr(status),
                      _stream(stream))
    return _check(rc, "qnt_gemv") if check else rc


def qnt_gemm(d: qnt_desc, codes, meta, X, Y, M: int, xdtype: int = QNT_F16, status=None, stream=None,
             check=True) -> int:
    rc = lib.qnt_gemm(ctypes.byref(d), _ptr(codes), _ptr(meta), _ptr(X), _ptr(Y), int(M), int(xdtype), _ptr(status),
                      _stream(stream))
    return _check(rc, "qnt_gemm") if check else rc


def seq_steps(items) -> ctypes.Array:
    """Build a host array of qnt_seq_step from (desc, codes, meta, x, y, wait) tuples."""
    arr = (qnt_seq_step * len(items))()
    for i, (d, codes, meta, x, y, wait) in enumerate(items):
        arr[i].desc = d
        arr[i].codes, arr[i].meta, arr[i].x, arr[i].y = _ptr(codes), _ptr(meta), _ptr(x), _ptr(y)
        arr[i].wait = int(wait)
        arr[i].reserved = 0
    return arr


def qnt_gemv_seq_work_bytes(nsteps: int) -> int:
    return lib.qnt_gemv_seq_work_bytes(int(nsteps))


def qnt_gemv_seq(steps, xdtype: int, work, status=None, stream=None, check=True) -> int:
    """steps: a ctypes array from seq_steps() (host memory)."""
    rc = lib.qnt_gemv_seq(steps, len(steps), int(xdtype), _ptr(work), _ptr(status), _stream(stream))
    return _check(rc, "qnt_gemv_seq") if check else rc


def qnt_gemv_seq_noalloc(steps, xdtype: int, status=None, stream=None, check=True) -> int:
    """qnt_gemv_seq without a caller workspace (the library's own counters)."""
    rc = lib.qnt_gemv_seq_noalloc(steps, len(steps), int(xdtype), _ptr(status), _stream(stream))
    return _check(rc, "qnt_gemv_seq_noalloc") if check else rc


class qnt_table:
    """Owner of a C qnt_table (selective precision rules)."""

    def __init__(self, default_fmt: int, default_group: int):
        self.h = lib.qnt_table_create(int(default_fmt), int(default_group))
        if not self.h:
            raise QntError(QNT_ERR_ARG, "qnt_table_create")

    def set(self, pattern: str, fmt: int, group: int) -> None:
        _check(lib.qnt_table_set(self.h, pattern.encode(), int(fmt), int(group)), "qnt_table_set")

    def lookup(self, name: str):
        f, g = ctypes.c_int(), ctypes.c_int()
        _check(lib.qnt_table_lookup(self.h, name.encode(), ctypes.byref(f), ctypes.byref(g)), "qnt_table_lookup")
        return f.value, g.value

    def __len__(self):
        return lib.qnt_table_size(self.h)

    def close(self):
        if self.h:
            lib.qnt_table_destroy(self.h)
            self.h = None

    def __del__(self):
        self.close()


def qnt_table_create(default_fmt: int, default_group: int) -> qnt_table:
    return qnt_table(default_fmt, default_group)
