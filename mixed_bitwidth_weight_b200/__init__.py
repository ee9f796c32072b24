"""Python binding of the qgemm C ABI (include/qgemm.h).

Argument marshalling only: every function checks tensor dtypes, devices and
contiguity, passes raw pointers and the current CUDA stream to the C library,
and turns a negative status into ``QGemmError``.  All arithmetic runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback, and importing this
package fails if ``libqgemm.so`` has not been built (``build()``).

Names follow the C entry points: ``qgemm_pack``, ``qgemm_dequant``, ``qgemm``,
``qgemm_workspace_bytes``, ``qgemm_packed_word_rows``, ``qgemm_offsets``,
``qgemm_validate_schedule``, ``qgemm_device_error``, ``qgemm_path_for``,
``qgemm_autotune``, ``qgemm_set_autotune``, ``qgemm_tune_lookup``,
``qgemm_tune_record``, ``qgemm_tune_clear``, ``qgemm_iqm``, ``qgemm_quantize``,
``qgemm_kv_quantize``, ``qgemm_kv_dequantize``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from ._build import LIB as _LIB_PATH
from ._build import build  # noqa: F401  (re-exported)

QGEMM_F16 = 0
QGEMM_BF16 = 1
DEV_BAD_SCHEDULE = 1
DEV_BAD_PERM = 2
DEV_TIMEOUT = 4


class QGemmError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} ({status})")
        self.status = status


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: run mixed_bitwidth_weight_b200.build() "
                          "(or __graft_entry__.build()) first")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "qgemm_version": (I, []),
        "qgemm_status_string": (ctypes.c_char_p, [I]),
        "qgemm_packed_word_rows": (I64, [P, I]),
        "qgemm_offsets": (I, [P, I, P]),
        "qgemm_validate_schedule": (I, [P, P, I, I64]),
        "qgemm_workspace_bytes": (SZ, [I, I, I]),
        "qgemm_packed_bytes": (SZ, [I64, I]),
        "qgemm_scale_bytes": (SZ, [I, I]),
        "qgemm_device_error": (I, [P, I]),
        "qgemm_path_for": (I, [I, I, I]),
        "qgemm_plan_info": (I, [I, I, I, I64, P]),
        "qgemm_pack": (I, [P, P, P, I, I, I64, P, P]),
        "qgemm_dequant": (I, [P, I64, P, P, P, I, I, P, P]),
        "qgemm": (I, [P, I, P, P, I64, P, P, P, I, I, I, P, P, SZ, P]),
        "qgemm_decode_noalloc": (I, [P, I, P, P, I64, P, P, P, I, I, I, P, P]),
        "qgemm_autotune": (I, [P, I, P, P, I64, P, P, P, I, I, I, P, P, SZ, I, I, P, P, I]),
        "qgemm_set_autotune": (I, [I]),
        "qgemm_noalloc_scratch_bytes": (SZ, [I, I, I]),
        "qgemm_noalloc_reset": (I, [P]),
        "qgemm_quantize_workspace_bytes": (SZ, [I, I]),
        "qgemm_quantize": (I, [P, P, I, I, P, P, P, P, P, SZ, P]),
        "qgemm_kv_quantize": (I, [P, I64, I, I, P, P, P]),
        "qgemm_kv_dequantize": (I, [P, P, I64, I, I, P, P]),
        "qgemm_tune_lookup": (I, [I, I, I, P, P]),
        "qgemm_tune_record": (I, [I, I, I, I, I]),
        "qgemm_tune_clear": (I, []),
        "qgemm_iqm": (ctypes.c_double, [P, I]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()
LIBRARY_PATH = _LIB_PATH


def status_string(status: int) -> str:
    return _lib.qgemm_status_string(int(status)).decode()


def _ok(status: int, where: str) -> int:
    if status < 0:
        raise QGemmError(int(status), where)
    return status


def _stream(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, dtype, name):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _shape_error(msg):
    raise ValueError(msg)


def _check_schedule_tensors(K, bits, offs):
    if K % 32 != 0:
        _shape_error(f"K = {K} is not a multiple of 32")
    if bits.numel() != K // 32:
        _shape_error(f"bits has {bits.numel()} entries, K/32 = {K // 32} expected")
    if offs.numel() != K // 32 + 1:
        _shape_error(f"offs has {offs.numel()} entries, K/32 + 1 = {K // 32 + 1} expected")


def _check_qgemm_shapes(x, perm, qw, scales, bits, offs, y):
    """Shapes of one qgemm call, checked before any pointer reaches the C ABI
    (a mismatch there would read or write past the end of a tensor)."""
    if x.dim() != 2 or y.dim() != 2:
        _shape_error("x and y must be 2-D ([M, K] and [M, N])")
    M, K = x.shape
    if y.shape[0] != M:
        _shape_error(f"y has {y.shape[0]} rows, x has {M}")
    N = y.shape[1]
    if perm.numel() != K:
        _shape_error(f"perm has {perm.numel()} entries, K = {K} expected")
    if qw.dim() != 2 or qw.shape[1] != N:
        _shape_error(f"qw must be [qw_rows, N = {N}], got {tuple(qw.shape)}")
    G = (K + 127) // 128
    if scales.numel() != G * N or (scales.dim() == 2 and tuple(scales.shape) != (G, N)):
        _shape_error(f"scales must be [ceil(K/128) = {G}, N = {N}], got {tuple(scales.shape)}")
    _check_schedule_tensors(K, bits, offs)


def _check_same_device(*tensors):
    """Every tensor on the current CUDA device (the call runs on its stream)."""
    import torch
    if not any(t.is_cuda for t in tensors):
        return  # host tensors: refused by the pointer checks that follow
    cur = torch.cuda.current_device()
    for t in tensors:
        if t.is_cuda and t.device.index != cur:
            raise ValueError(f"tensor on cuda:{t.device.index}, but the current device is cuda:{cur}")


def _host_u8(a):
    return np.ascontiguousarray(np.asarray(a), dtype=np.uint8)


# ------------------------------------------------------------- host helpers

def qgemm_version() -> int:
    return _lib.qgemm_version()


def qgemm_packed_word_rows(bits, K: int) -> int:
    b = _host_u8(bits)
    return _ok(_lib.qgemm_packed_word_rows(ctypes.c_void_p(b.ctypes.data), K), "qgemm_packed_word_rows")


def qgemm_offsets(bits, K: int) -> np.ndarray:
    b = _host_u8(bits)
    out = np.empty(K // 32 + 1, dtype=np.int32)
    _ok(_lib.qgemm_offsets(ctypes.c_void_p(b.ctypes.data), K, ctypes.c_void_p(out.ctypes.data)),
        "qgemm_offsets")
    return out


def qgemm_validate_schedule(bits, offs, K: int, qw_rows: int) -> int:
    b = _host_u8(bits)
    o = np.ascontiguousarray(np.asarray(offs), dtype=np.int32)
    return _lib.qgemm_validate_schedule(ctypes.c_void_p(b.ctypes.data), ctypes.c_void_p(o.ctypes.data),
                                        K, int(qw_rows))


def qgemm_workspace_bytes(M: int, K: int, N: int) -> int:
    return int(_lib.qgemm_workspace_bytes(M, K, N))


def qgemm_path_for(M: int, K: int, N: int) -> int:
    return int(_lib.qgemm_path_for(M, K, N))


def qgemm_plan_info(M: int, K: int, N: int, qw_rows: int) -> dict:
    out = (ctypes.c_int64 * 6)()
    _ok(_lib.qgemm_plan_info(M, K, N, int(qw_rows), out), "qgemm_plan_info")
    return dict(path=out[0], grid=out[1], ring=out[2], ctas_per_sm=out[3], smem=out[4], sms=out[5])


PATH_NAMES = {0: "integer GEMV", 1: "tensor-core GEMV", 2: "GEMM"}


def qgemm_set_autotune(mode: int) -> None:
    """1: qgemm() tunes each new shape on its first eager call; 0: never."""
    _ok(_lib.qgemm_set_autotune(int(mode)), "qgemm_set_autotune")


def qgemm_tune_lookup(M: int, K: int, N: int):
    """The recorded (path, knob) for this shape on the current device, or None."""
    path, knob = ctypes.c_int(0), ctypes.c_int(0)
    found = _ok(_lib.qgemm_tune_lookup(M, K, N, ctypes.byref(path), ctypes.byref(knob)), "qgemm_tune_lookup")
    return (path.value, knob.value) if found else None


def qgemm_tune_record(M: int, K: int, N: int, path: int, knob: int) -> None:
    _ok(_lib.qgemm_tune_record(M, K, N, int(path), int(knob)), "qgemm_tune_record")


def qgemm_tune_clear() -> None:
    _ok(_lib.qgemm_tune_clear(), "qgemm_tune_clear")


def qgemm_iqm(values) -> float:
    v = np.ascontiguousarray(np.asarray(values, dtype=np.float32))
    r = _lib.qgemm_iqm(ctypes.c_void_p(v.ctypes.data), int(v.size))
    if r < 0:
        raise ValueError("qgemm_iqm needs at least one value")
    return float(r)


def qgemm_device_error(clear: bool = True) -> int:
    code = ctypes.c_int(0)
    _ok(_lib.qgemm_device_error(ctypes.byref(code), 1 if clear else 0), "qgemm_device_error")
    return code.value


# ------------------------------------------------------------- device calls

def qgemm_pack(codes, bits, offs, qw, stream=None):
    """codes uint8 [K, N] -> qw int32/uint32 [qw_rows, N] (all CUDA tensors)."""
    import torch
    if codes.dim() != 2 or qw.dim() != 2:
        _shape_error("codes and qw must be 2-D ([K, N] and [qw_rows, N])")
    K, N = codes.shape
    rows = qw.shape[0]
    if qw.shape[1] != N:
        _shape_error(f"qw has {qw.shape[1]} columns, codes has {N}")
    _check_schedule_tensors(K, bits, offs)
    _check_same_device(codes, bits, offs, qw)
    _ok(_lib.qgemm_pack(_dev(codes, torch.uint8, "codes"), _dev(bits, torch.uint8, "bits"),
                        _dev(offs, torch.int32, "offs"), K, N, rows,
                        _dev(qw, (torch.int32, torch.uint32), "qw"), _stream(stream)), "qgemm_pack")
    return qw


def qgemm_dequant(qw, scales, bits, offs, w, stream=None):
    """qw [qw_rows, N], scales fp16 [ceil(K/128), N] -> w fp16 [K, N]."""
    import torch
    if w.dim() != 2 or qw.dim() != 2:
        _shape_error("w and qw must be 2-D ([K, N] and [qw_rows, N])")
    K, N = w.shape
    if qw.shape[1] != N:
        _shape_error(f"qw has {qw.shape[1]} columns, w has {N}")
    G = (K + 127) // 128
    if scales.numel() != G * N or (scales.dim() == 2 and tuple(scales.shape) != (G, N)):
        _shape_error(f"scales must be [ceil(K/128) = {G}, N = {N}], got {tuple(scales.shape)}")
    _check_schedule_tensors(K, bits, offs)
    _check_same_device(qw, scales, bits, offs, w)
    _ok(_lib.qgemm_dequant(_dev(qw, (torch.int32, torch.uint32), "qw"), qw.shape[0],
                           _dev(scales, torch.float16, "scales"), _dev(bits, torch.uint8, "bits"),
                           _dev(offs, torch.int32, "offs"), K, N, _dev(w, torch.float16, "w"),
                           _stream(stream)), "qgemm_dequant")
    return w


def qgemm_quantize(w, bits, codes, scales, err=None, best=None, ws=None, stream=None):
    """fp16 W [K, N] (act-order rows) -> codes uint8 [K, N] and fp16 scales
    [ceil(K/128), N]; err (float64 [96]) and best (int32 [1]) optional."""
    import torch
    if w.dim() != 2 or codes.dim() != 2 or tuple(codes.shape) != tuple(w.shape):
        _shape_error("w and codes must both be [K, N]")
    K, N = w.shape
    if K % 32 != 0:
        _shape_error(f"K = {K} is not a multiple of 32")
    if bits.numel() != K // 32:
        _shape_error(f"bits has {bits.numel()} entries, K/32 = {K // 32} expected")
    G = (K + 127) // 128
    if scales.numel() != G * N or (scales.dim() == 2 and tuple(scales.shape) != (G, N)):
        _shape_error(f"scales must be [ceil(K/128) = {G}, N = {N}], got {tuple(scales.shape)}")
    if err is not None and err.numel() != 96:
        _shape_error("err must hold 96 values")
    if best is not None and best.numel() != 1:
        _shape_error("best must hold one value")
    extra = tuple(t for t in (err, best, ws) if t is not None)
    _check_same_device(w, bits, codes, scales, *extra)
    if ws is None:
        ws = torch.empty(max(16, int(_lib.qgemm_quantize_workspace_bytes(K, N))), dtype=torch.uint8,
                         device=w.device)
    _ok(_lib.qgemm_quantize(_dev(w, torch.float16, "w"), _dev(bits, torch.uint8, "bits"), K, N,
                            _dev(codes, torch.uint8, "codes"), _dev(scales, torch.float16, "scales"),
                            ctypes.c_void_p(0) if err is None else _dev(err, torch.float64, "err"),
                            ctypes.c_void_p(0) if best is None else _dev(best, torch.int32, "best"),
                            _dev(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)), "qgemm_quantize")
    return codes, scales


def _kv_shapes(v, codes, scales, bits):
    if v.dim() < 1:
        _shape_error("v must have a last dimension D")
    D = v.shape[-1]
    if D not in (32, 64, 128, 256):
        _shape_error(f"D = {D} must be 32, 64, 128 or 256")
    nvec = v.numel() // D
    if codes.numel() != nvec * (D // 32) * bits:
        _shape_error(f"codes must hold {nvec} x {D // 32} x {bits} words, got {codes.numel()}")
    if scales.numel() != nvec * (D // 32):
        _shape_error(f"scales must hold {nvec} x {D // 32} values, got {scales.numel()}")
    return nvec, D


def qgemm_kv_quantize(v, bits, codes, scales, stream=None):
    """fp16 vectors v [..., D] -> codes int32/uint32 [..., D/32, bits] and fp16
    scales [..., D/32] (Hadamard rotation, then b-bit groups of 32)."""
    import torch
    nvec, D = _kv_shapes(v, codes, scales, bits)
    _check_same_device(v, codes, scales)
    _ok(_lib.qgemm_kv_quantize(_dev(v, torch.float16, "v"), nvec, D, int(bits),
                               _dev(codes, (torch.int32, torch.uint32), "codes"),
                               _dev(scales, torch.float16, "scales"), _stream(stream)), "qgemm_kv_quantize")
    return codes, scales


def qgemm_kv_dequantize(codes, scales, bits, v, stream=None):
    """codes [..., D/32, bits] and fp16 scales -> fp16 vectors v [..., D]."""
    import torch
    nvec, D = _kv_shapes(v, codes, scales, bits)
    _check_same_device(v, codes, scales)
    _ok(_lib.qgemm_kv_dequantize(_dev(codes, (torch.int32, torch.uint32), "codes"),
                                 _dev(scales, torch.float16, "scales"), nvec, D, int(bits),
                                 _dev(v, torch.float16, "v"), _stream(stream)), "qgemm_kv_dequantize")
    return v


def qgemm(x, perm, qw, scales, bits, offs, y, ws=None, stream=None):
    """y [M, N] fp16 = x[:, perm] . dequant(qw); x fp16 or bf16 [M, K]."""
    import torch
    _check_qgemm_shapes(x, perm, qw, scales, bits, offs, y)
    _check_same_device(x, perm, qw, scales, bits, offs, y, *(() if ws is None else (ws,)))
    M, K = x.shape
    N = y.shape[1]
    if x.dtype == torch.float16:
        xdt = QGEMM_F16
    elif x.dtype == torch.bfloat16:
        xdt = QGEMM_BF16
    else:
        raise TypeError("x must be float16 or bfloat16")
    if ws is None:
        wsp, wsb = ctypes.c_void_p(0), 0
    else:
        wsp, wsb = _dev(ws, torch.uint8, "ws"), ws.numel()
    _ok(_lib.qgemm(_dev(x, None, "x"), xdt, _dev(perm, torch.int32, "perm"),
                   _dev(qw, (torch.int32, torch.uint32), "qw"), qw.shape[0],
                   _dev(scales, torch.float16, "scales"), _dev(bits, torch.uint8, "bits"),
                   _dev(offs, torch.int32, "offs"), M, K, N, _dev(y, torch.float16, "y"),
                   wsp, wsb, _stream(stream)), "qgemm")
    return y


def qgemm_autotune(x, perm, qw, scales, bits, offs, y, ws, warmup=20, iters=200, stream=None):
    """Time every kernel variant of this shape on these operands and record
    the fastest (see include/qgemm.h).  Returns one dict per candidate
    (path, knob, us: IQM per call or None when skipped) and the chosen one."""
    import torch
    _check_qgemm_shapes(x, perm, qw, scales, bits, offs, y)
    _check_same_device(x, perm, qw, scales, bits, offs, y, ws)
    M, K = x.shape
    N = y.shape[1]
    if x.dtype == torch.float16:
        xdt = QGEMM_F16
    elif x.dtype == torch.bfloat16:
        xdt = QGEMM_BF16
    else:
        raise TypeError("x must be float16 or bfloat16")
    rows = (ctypes.c_int64 * (3 * 16))()
    n = _ok(_lib.qgemm_autotune(_dev(x, None, "x"), xdt, _dev(perm, torch.int32, "perm"),
                                _dev(qw, (torch.int32, torch.uint32), "qw"), qw.shape[0],
                                _dev(scales, torch.float16, "scales"), _dev(bits, torch.uint8, "bits"),
                                _dev(offs, torch.int32, "offs"), M, K, N, _dev(y, torch.float16, "y"),
                                _dev(ws, torch.uint8, "ws"), ws.numel(), int(warmup), int(iters),
                                _stream(stream), rows, 16), "qgemm_autotune")
    cands = [dict(path=int(rows[3 * i]), knob=int(rows[3 * i + 1]),
                  us=(rows[3 * i + 2] / 1e3 if rows[3 * i + 2] >= 0 else None)) for i in range(n)]
    chosen = qgemm_tune_lookup(M, K, N)
    return dict(candidates=cands, path=chosen[0], knob=chosen[1])


NOALLOC_SCRATCH_BYTES = 8 << 20


def qgemm_noalloc_scratch_bytes(M: int, K: int, N: int) -> int:
    return int(_lib.qgemm_noalloc_scratch_bytes(M, K, N))


def qgemm_noalloc_reset(stream=None) -> None:
    """Zero the built-in buffer's tickets (after a QGEMM_DEV_TIMEOUT)."""
    _ok(_lib.qgemm_noalloc_reset(_stream(stream)), "qgemm_noalloc_reset")


def qgemm_decode_noalloc(x, perm, qw, scales, bits, offs, y, stream=None):
    """As qgemm() for M <= 4, with no workspace: the scratch is a buffer built
    into the library, so nothing is allocated (for callers that cannot
    allocate device memory).  Calls that overlap on the GPU race on that
    buffer; the first call on a device should come before any stream capture."""
    import torch
    _check_qgemm_shapes(x, perm, qw, scales, bits, offs, y)
    _check_same_device(x, perm, qw, scales, bits, offs, y)
    M, K = x.shape
    N = y.shape[1]
    if x.dtype == torch.float16:
        xdt = QGEMM_F16
    elif x.dtype == torch.bfloat16:
        xdt = QGEMM_BF16
    else:
        raise TypeError("x must be float16 or bfloat16")
    _ok(_lib.qgemm_decode_noalloc(_dev(x, None, "x"), xdt, _dev(perm, torch.int32, "perm"),
                                  _dev(qw, (torch.int32, torch.uint32), "qw"), qw.shape[0],
                                  _dev(scales, torch.float16, "scales"), _dev(bits, torch.uint8, "bits"),
                                  _dev(offs, torch.int32, "offs"), M, K, N, _dev(y, torch.float16, "y"),
                                  _stream(stream)), "qgemm_decode_noalloc")
    return y


def workspace(M: int, K: int, N: int, device="cuda"):
    """A zero-filled workspace tensor of the size qgemm needs for this shape."""
    import torch
    return torch.zeros(max(16, qgemm_workspace_bytes(M, K, N)), dtype=torch.uint8, device=device)
