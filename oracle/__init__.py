"""CPU oracle for the mixed-bitwidth Q-GEMM (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never links, loads
or calls it, and this package never touches the CUDA library: the two share no
code.  The arithmetic lives in ``oracle.c`` (plain C, double precision); this
file compiles it with gcc and marshals numpy arrays through ctypes.

Functions (all numpy in, numpy out):

* ``word_rows(bits, K)``          sum of block widths (packed word rows)
* ``pack(codes, bits)``            uint8 [K, N] -> uint32 [sum b, N]
* ``unpack(qw, bits, K)``          inverse of ``pack``
* ``half_to_double(h)`` / ``double_to_half(v)``   exact / RNE conversions
* ``dequant_f64(qw, scales, bits, K)``   exact weights, double [K, N]
* ``dequant_f16(qw, scales, bits, K)``   RNE fp16 weights (uint16 bits)
* ``qgemm_f64(x, perm, qw, scales, bits, cols=None, threads=0)``
      y = x[:, perm] . dequant(qw), double [M, N] (or [M, len(cols)])
* ``quantize(w, bits, threads=0)``  fp16 W [K, N] -> codes, fp16 scales, the
      chosen candidate, the 96 candidate errors and the per-column errors
* ``kv_quantize(v, b)`` / ``kv_dequantize(codes, scales, D, b)``  Hadamard-
      rotated KV-cache vectors [n, D] <-> packed codes [n, D/32, b] + scales

Parity pins for every function are in ``tests/test_oracle.py``.
"""
from __future__ import annotations

import ctypes
import hashlib
import os
import subprocess

import numpy as np

_DIR = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_DIR, "oracle.c")
_LIB = os.path.join(_DIR, "liboracle.so")
_STAMP = os.path.join(_DIR, "liboracle.sha1")


def _src_hash() -> str:
    with open(_SRC, "rb") as f:
        return hashlib.sha1(f.read()).hexdigest()


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (portable -O2, no -march)."""
    h = _src_hash()
    if not force and os.path.exists(_LIB) and os.path.exists(_STAMP):
        with open(_STAMP) as f:
            if f.read().strip() == h:
                return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-o", tmp, _SRC,
                           "-lm", "-lpthread"])
    os.replace(tmp, _LIB)
    with open(_STAMP, "w") as f:
        f.write(h)
    return _LIB


def _bind(lib):
    P = ctypes.c_void_p
    lib.oracle_word_rows.restype = ctypes.c_int64
    lib.oracle_word_rows.argtypes = [P, ctypes.c_int]
    lib.oracle_pack.restype = ctypes.c_int
    lib.oracle_pack.argtypes = [P, P, ctypes.c_int, ctypes.c_int, P]
    lib.oracle_unpack.restype = ctypes.c_int
    lib.oracle_unpack.argtypes = [P, P, ctypes.c_int, ctypes.c_int, P]
    lib.oracle_dequant_f64.restype = ctypes.c_int
    lib.oracle_dequant_f64.argtypes = [P, P, P, ctypes.c_int, ctypes.c_int, P]
    lib.oracle_dequant_f16.restype = ctypes.c_int
    lib.oracle_dequant_f16.argtypes = [P, P, P, ctypes.c_int, ctypes.c_int, P]
    lib.oracle_qgemm_f64.restype = ctypes.c_int
    lib.oracle_qgemm_f64.argtypes = [P, P, P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                     P, ctypes.c_int64, P, ctypes.c_int]
    lib.oracle_quantize.restype = ctypes.c_int
    lib.oracle_quantize.argtypes = [P, P, ctypes.c_int, ctypes.c_int, P, P, P, P, ctypes.c_int]
    lib.oracle_kv_quantize.restype = ctypes.c_int
    lib.oracle_kv_quantize.argtypes = [P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, P, P]
    lib.oracle_kv_dequantize.restype = ctypes.c_int
    lib.oracle_kv_dequantize.argtypes = [P, P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, P]
    lib.oracle_half_to_double_n.restype = None
    lib.oracle_half_to_double_n.argtypes = [P, P, ctypes.c_int64]
    lib.oracle_double_to_half_n.restype = None
    lib.oracle_double_to_half_n.argtypes = [P, P, ctypes.c_int64]
    return lib


def compile_variant(src_text: str, out_path: str) -> str:
    """Compile an edited copy of oracle.c (used by the tests that plant a
    mistake in the oracle and check that the pins catch it)."""
    c_path = out_path + ".c"
    with open(c_path, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-o", out_path, c_path,
                           "-lm", "-lpthread"])
    return out_path


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


class OracleError(ValueError):
    pass


def _c(a, dtype):
    return np.ascontiguousarray(np.asarray(a), dtype=dtype)


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _check(rc: int, what: str):
    if rc < 0:
        raise OracleError(f"{what}: oracle status {rc}")
    return rc


class Oracle:
    """One loaded build of the oracle library."""

    def __init__(self, libpath: str | None = None):
        self.lib = _bind(ctypes.CDLL(libpath or build()))

    def word_rows(self, bits, K: int) -> int:
        b = _c(bits, np.uint8)
        return _check(self.lib.oracle_word_rows(_ptr(b), K), "word_rows")

    def pack(self, codes, bits) -> np.ndarray:
        c = _c(codes, np.uint8)
        b = _c(bits, np.uint8)
        K, N = c.shape
        rows = self.word_rows(b, K)
        qw = np.empty((rows, N), dtype=np.uint32)
        _check(self.lib.oracle_pack(_ptr(c), _ptr(b), K, N, _ptr(qw)), "pack")
        return qw

    def unpack(self, qw, bits, K: int) -> np.ndarray:
        w = _c(qw, np.uint32)
        b = _c(bits, np.uint8)
        N = w.shape[1]
        out = np.empty((K, N), dtype=np.uint8)
        _check(self.lib.oracle_unpack(_ptr(w), _ptr(b), K, N, _ptr(out)), "unpack")
        return out

    def half_to_double(self, h) -> np.ndarray:
        h = _c(np.asarray(h).view(np.uint16) if np.asarray(h).dtype == np.float16 else h, np.uint16)
        out = np.empty(h.shape, dtype=np.float64)
        self.lib.oracle_half_to_double_n(_ptr(h), _ptr(out), h.size)
        return out

    def double_to_half(self, v) -> np.ndarray:
        v = _c(v, np.float64)
        out = np.empty(v.shape, dtype=np.uint16)
        self.lib.oracle_double_to_half_n(_ptr(v), _ptr(out), v.size)
        return out

    @staticmethod
    def _scales_bits(scales) -> np.ndarray:
        s = np.asarray(scales)
        if s.dtype == np.float16:
            s = s.view(np.uint16)
        return _c(s, np.uint16)

    def dequant_f64(self, qw, scales, bits, K: int) -> np.ndarray:
        w = _c(qw, np.uint32)
        s = self._scales_bits(scales)
        b = _c(bits, np.uint8)
        N = w.shape[1]
        out = np.empty((K, N), dtype=np.float64)
        _check(self.lib.oracle_dequant_f64(_ptr(w), _ptr(s), _ptr(b), K, N, _ptr(out)), "dequant_f64")
        return out

    def dequant_f16(self, qw, scales, bits, K: int) -> np.ndarray:
        """fp16 dequantised weights as uint16 bit patterns [K, N]."""
        w = _c(qw, np.uint32)
        s = self._scales_bits(scales)
        b = _c(bits, np.uint8)
        N = w.shape[1]
        out = np.empty((K, N), dtype=np.uint16)
        _check(self.lib.oracle_dequant_f16(_ptr(w), _ptr(s), _ptr(b), K, N, _ptr(out)), "dequant_f16")
        return out

    def qgemm_f64(self, x, perm, qw, scales, bits, cols=None, threads: int = 0):
        """y = x[:, perm] . dequant(qw) in double.  x: [M, K] (any float dtype,
        converted exactly to double).  Returns (y, threads_used)."""
        xd = _c(np.asarray(x, dtype=np.float64), np.float64)
        M, K = xd.shape
        p = _c(perm, np.int32)
        w = _c(qw, np.uint32)
        s = self._scales_bits(scales)
        b = _c(bits, np.uint8)
        N = w.shape[1]
        if cols is None:
            cp, nc = None, N
        else:
            cc = _c(cols, np.int64)
            cp, nc = _ptr(cc), cc.size
        y = np.empty((M, nc), dtype=np.float64)
        used = _check(self.lib.oracle_qgemm_f64(_ptr(xd), _ptr(p), _ptr(w), _ptr(s), _ptr(b), M, K, N,
                                               cp, nc, _ptr(y), threads), "qgemm_f64")
        return y, used

    def quantize(self, w, bits, threads: int = 0) -> "Quantized":
        """fp16 W [K, N] (np.float16 or uint16 bit patterns) -> codes, scales."""
        wa = np.asarray(w)
        wb = _c(wa.view(np.uint16) if wa.dtype == np.float16 else wa, np.uint16)
        b = _c(bits, np.uint8)
        K, N = wb.shape
        G = (K + 127) // 128
        codes = np.empty((K, N), dtype=np.uint8)
        scales = np.empty((G, N), dtype=np.uint16)
        colerr = np.empty((96, N), dtype=np.float64)
        err = np.empty(96, dtype=np.float64)
        best = _check(self.lib.oracle_quantize(_ptr(wb), _ptr(b), K, N, _ptr(codes), _ptr(scales),
                                               _ptr(colerr), _ptr(err), threads), "quantize")
        return Quantized(codes, scales, best, err, colerr)

    def kv_quantize(self, v, b: int):
        """fp16 vectors [n, D] -> (codes uint32 [n, D/32, b], scales fp16 bits [n, D/32])."""
        va = np.asarray(v)
        vb = _c(va.view(np.uint16) if va.dtype == np.float16 else va, np.uint16)
        n, D = vb.shape
        codes = np.empty((n, D // 32, b), dtype=np.uint32)
        scales = np.empty((n, D // 32), dtype=np.uint16)
        _check(self.lib.oracle_kv_quantize(_ptr(vb), n, D, b, _ptr(codes), _ptr(scales)), "kv_quantize")
        return codes, scales

    def kv_dequantize(self, codes, scales, D: int, b: int):
        """-> fp16 bit patterns [n, D]."""
        c = _c(codes, np.uint32)
        s = self._scales_bits(scales)
        n = s.shape[0]
        out = np.empty((n, D), dtype=np.uint16)
        _check(self.lib.oracle_kv_dequantize(_ptr(c), _ptr(s), n, D, b, _ptr(out)), "kv_dequantize")
        return out


class Quantized:
    """Result of the oracle's quantiser."""

    def __init__(self, codes, scales, best, err, colerr):
        self.codes = codes        # uint8 [K, N]
        self.scales = scales      # fp16 bit patterns, uint16 [G, N]
        self.best = best          # chosen candidate index (p = (32 + best) / 96)
        self.err = err            # double [96]: E(p_i)
        self.colerr = colerr      # double [96, N]: per-column errors


def get() -> Oracle:
    """The oracle built from oracle.c as it stands."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


_default = None


def word_rows(bits, K):
    return get().word_rows(bits, K)


def pack(codes, bits):
    return get().pack(codes, bits)


def unpack(qw, bits, K):
    return get().unpack(qw, bits, K)


def half_to_double(h):
    return get().half_to_double(h)


def double_to_half(v):
    return get().double_to_half(v)


def dequant_f64(qw, scales, bits, K):
    return get().dequant_f64(qw, scales, bits, K)


def dequant_f16(qw, scales, bits, K):
    return get().dequant_f16(qw, scales, bits, K)


def quantize(w, bits, threads=0):
    return get().quantize(w, bits, threads)


def kv_quantize(v, b):
    return get().kv_quantize(v, b)


def kv_dequantize(codes, scales, D, b):
    return get().kv_dequantize(codes, scales, D, b)


def qgemm_f64(x, perm, qw, scales, bits, cols=None, threads=0):
    return get().qgemm_f64(x, perm, qw, scales, bits, cols, threads)
