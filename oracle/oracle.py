"""Python access to the CPU oracle (``qnt_oracle.c``).

TEST INFRASTRUCTURE ONLY: this module may be imported by ``tests/``, by
``__graft_entry__.smoke()`` and by the CPU-baseline / reference legs of
``bench.py``; the library under test never imports it.  It shares no code with
the CUDA library: the oracle's C file is compiled on its own (``build.py`` in
this folder) and loaded here with ctypes.

Format ids follow the library's public numbering: INT4=1 (asymmetric, fp16
scale + 4-bit zero), FP4=2 (E2M1, absmax/6 scale), AFPQ=3 (E2M1 with separate
positive/negative scales), RAZER=4 (E2M1 whose negative-zero code decodes to a
per-group special value from {+5, -5, +8, -8}), INT8=5 (symmetric per output
channel), FP16=6.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

INT4, FP4, AFPQ, RAZER, INT8, FP16 = 1, 2, 3, 4, 5, 6
FOUR_BIT = (INT4, FP4, AFPQ, RAZER)
FMT_NAMES = {INT4: "int4_asym", FP4: "fp4_e2m1", AFPQ: "fp4_afpq", RAZER: "fp4_razer",
             INT8: "int8_perchan", FP16: "fp16"}
OK, NONFINITE, RANGE = 0, 6, 7

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_p = ctypes.c_void_p
_i = ctypes.c_int
_l = ctypes.c_long


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        subprocess.check_call(["python", os.path.join(_HERE, "build.py")])
    lib = ctypes.CDLL(_LIB_PATH)
    sig = {
        "o_h2d": (ctypes.c_double, [ctypes.c_uint16]),
        "o_f2h": (ctypes.c_uint16, [ctypes.c_float]),
        "o_bf2d": (ctypes.c_double, [ctypes.c_uint16]),
        "o_f2bf": (ctypes.c_uint16, [ctypes.c_float]),
        "o_e2m1": (ctypes.c_double, [_i]),
        "o_razer_sv": (ctypes.c_double, [_i]),
        "o_quantize": (_i, [_i, _p, _i, _i, _i, _p, _p, _p, _p]),
        "o_quantize_group": (_i, [_i, _p, _i, _p, _p, _p, _p]),
        "o_dequant_one": (ctypes.c_double, [_i, _i, ctypes.c_uint16, ctypes.c_uint16, _i]),
        "o_dequant": (None, [_i, _p, _p, _p, _p, _i, _i, _i, _p]),
        "o_gemm": (None, [_i, _p, _p, _p, _p, _i, _i, _i, _p, _i, _i, _p, _p]),
        "o_codes_bytes": (_l, [_i, _l, _l]),
        "o_meta_bytes": (_l, [_i, _l, _l, _l]),
        "o_pack": (None, [_i, _i, _i, _i, _p, _p, _p, _p, _p, _p]),
        "o_unpack": (None, [_i, _i, _i, _i, _p, _p, _p, _p, _p, _p]),
        "o_f2h_array": (None, [_p, _p, _l]),
        "o_f2bf_array": (None, [_p, _p, _l]),
        "o_h2d_array": (None, [_p, _p, _l]),
        "o_threads": (_i, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- conversions
def f2h(x) -> np.ndarray:
    """binary32 -> fp16 bit patterns (round to nearest even)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint16)
    _load().o_f2h_array(_ptr(x), _ptr(out), x.size)
    return out


def f2bf(x) -> np.ndarray:
    """binary32 -> bfloat16 bit patterns (round to nearest even)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint16)
    _load().o_f2bf_array(_ptr(x), _ptr(out), x.size)
    return out


def h2d(h) -> np.ndarray:
    """fp16 bit patterns -> exact binary64 values."""
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, np.float64)
    _load().o_h2d_array(_ptr(h), _ptr(out), h.size)
    return out


def bf2d(b) -> np.ndarray:
    return np.array([_load().o_bf2d(int(v)) for v in np.asarray(b).ravel()]).reshape(np.shape(b))


def e2m1(code: int) -> float:
    return _load().o_e2m1(int(code))


def razer_sv(sel: int) -> float:
    return _load().o_razer_sv(int(sel))


def threads() -> int:
    return _load().o_threads()


# ---------------------------------------------------------------- quantize
class Quant:
    """Logical (unpacked) quantized matrix: one code per weight plus metadata."""

    def __init__(self, fmt, N, K, g, codes, s1, s2, z, status=OK):
        self.fmt, self.N, self.K, self.g = fmt, N, K, g
        self.codes, self.s1, self.s2, self.z, self.status = codes, s1, s2, z, status

    def rows(self, idx) -> "Quant":
        """The sub-matrix made of the given output rows."""
        idx = np.asarray(idx)
        G = 1 if self.fmt in (INT8, FP16) else self.K // self.g
        pick = lambda a: None if a is None else np.ascontiguousarray(a.reshape(self.N, -1)[idx].reshape(-1))
        codes = np.ascontiguousarray(self.codes.reshape(self.N, -1)[idx])
        return Quant(self.fmt, len(idx), self.K, self.g, codes, pick(self.s1), pick(self.s2), pick(self.z), self.status)


def _meta_arrays(fmt, N, K, g):
    P = N if fmt in (INT8, FP16) else N * (K // g)
    s1 = np.zeros(P, np.uint16)
    s2 = np.zeros(P, np.uint16)
    z = np.zeros(P, np.uint8)
    return s1, s2, z


def quantize(fmt: int, W, g: int) -> Quant:
    """RTN-quantize W [N, K] (binary32) in groups of g along K."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    if fmt in (INT8, FP16):
        g = K
    codes = np.zeros((N, K * (2 if fmt == FP16 else 1)), np.uint8)
    s1, s2, z = _meta_arrays(fmt, N, K, g)
    st = _load().o_quantize(fmt, _ptr(W), N, K, g, _ptr(codes), _ptr(s1), _ptr(s2), _ptr(z))
    if fmt == FP16:
        codes = codes.view(np.uint16).reshape(N, K)
    return Quant(fmt, N, K, g, codes, s1, s2, z, st)


def quantize_group(fmt: int, w):
    """Quantize one group of any size (tiny groups for brute-force checks)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    g = w.size
    codes = np.zeros(g, np.uint8)
    s1 = np.zeros(1, np.uint16)
    s2 = np.zeros(1, np.uint16)
    z = np.zeros(1, np.uint8)
    st = _load().o_quantize_group(fmt, _ptr(w), g, _ptr(codes), _ptr(s1), _ptr(s2), _ptr(z))
    return codes, int(s1[0]), int(s2[0]), int(z[0]), st


def dequant_one(fmt, code, s1, s2=0, z=0) -> float:
    return _load().o_dequant_one(fmt, int(code), int(s1), int(s2), int(z))


def dequant(q: Quant) -> np.ndarray:
    out = np.empty((q.N, q.K), np.float64)
    codes = q.codes.view(np.uint8) if q.fmt == FP16 else q.codes
    codes = np.ascontiguousarray(codes)
    _load().o_dequant(q.fmt, _ptr(codes), _ptr(q.s1), _ptr(q.s2), _ptr(q.z), q.N, q.K, q.g, _ptr(out))
    return out


def gemm(q: Quant, X_bits, xdt: int):
    """Reference Y[m, n] = sum_k dq[n, k] X[m, k] and A = sum_k |dq X| (binary64).

    X_bits: uint16 [M, K] fp16 (xdt=0) or bf16 (xdt=1) bit patterns."""
    X_bits = np.ascontiguousarray(np.atleast_2d(X_bits), dtype=np.uint16)
    M = X_bits.shape[0]
    Y = np.empty((M, q.N), np.float64)
    A = np.empty((M, q.N), np.float64)
    codes = np.ascontiguousarray(q.codes.view(np.uint8) if q.fmt == FP16 else q.codes)
    _load().o_gemm(q.fmt, _ptr(codes), _ptr(q.s1), _ptr(q.s2), _ptr(q.z), q.N, q.K, q.g,
                   _ptr(X_bits), xdt, M, _ptr(Y), _ptr(A))
    return Y, A


# ---------------------------------------------------------------- layout
def codes_bytes(fmt, N, K) -> int:
    return _load().o_codes_bytes(fmt, N, K)


def meta_bytes(fmt, N, K, g) -> int:
    return _load().o_meta_bytes(fmt, N, K, K if fmt in (INT8, FP16) else g)


def pack(q: Quant):
    """Logical -> packed (library storage layout) byte arrays (codes, meta)."""
    g = q.K if q.fmt in (INT8, FP16) else q.g
    pc = np.zeros(codes_bytes(q.fmt, q.N, q.K), np.uint8)
    pm = np.zeros(max(1, meta_bytes(q.fmt, q.N, q.K, g)), np.uint8)
    codes = np.ascontiguousarray(q.codes.view(np.uint8) if q.fmt == FP16 else q.codes)
    _load().o_pack(q.fmt, q.N, q.K, g, _ptr(codes), _ptr(q.s1), _ptr(q.s2), _ptr(q.z), _ptr(pc), _ptr(pm))
    return pc, pm


def unpack(fmt, N, K, g, pc, pm) -> Quant:
    """Packed byte arrays -> logical codes and metadata."""
    if fmt in (INT8, FP16):
        g = K
    pc = np.ascontiguousarray(pc, dtype=np.uint8)
    pm = np.ascontiguousarray(pm, dtype=np.uint8)
    codes = np.zeros((N, K * (2 if fmt == FP16 else 1)), np.uint8)
    s1, s2, z = _meta_arrays(fmt, N, K, g)
    _load().o_unpack(fmt, N, K, g, _ptr(pc), _ptr(pm), _ptr(codes), _ptr(s1), _ptr(s2), _ptr(z))
    if fmt == FP16:
        codes = codes.view(np.uint16).reshape(N, K)
    return Quant(fmt, N, K, g, codes, s1, s2, z)
