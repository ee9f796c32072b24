"""The C ABI without a GPU: the library loads, exports every entry point its
header declares, and its host-side helpers and argument checks behave."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import mixed_bitwidth_weight_b200 as q
import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qgemm.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\**\s+\**\s*(qgemm[a-z_0-9]*)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = header_functions()
    for required in ("qgemm", "qgemm_pack", "qgemm_dequant", "qgemm_workspace_bytes",
                     "qgemm_packed_word_rows", "qgemm_offsets", "qgemm_device_error"):
        assert required in names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", q.LIBRARY_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(\S+)$", out, flags=re.M))
    missing = [n for n in header_functions() if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    lib = ctypes.CDLL(q.LIBRARY_PATH)
    for n in header_functions():
        assert getattr(lib, n) is not None


def test_library_has_no_oracle_dependency():
    out = subprocess.run(["nm", "-D", q.LIBRARY_PATH], capture_output=True, text=True).stdout
    assert "oracle" not in out
    ldd = subprocess.run(["ldd", q.LIBRARY_PATH], capture_output=True, text=True).stdout
    assert "liboracle" not in ldd and "libtorch" not in ldd


def test_version_and_status_strings():
    assert q.qgemm_version() >= 100
    for st in range(-8, 1):
        assert q.status_string(st) and q.status_string(st) != "unknown status"
    assert q.status_string(-99) == "unknown status"


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_word_rows_and_offsets_match_schedule(name):
    w = W.WORKLOADS[name]
    shapes = [(K, N) for _, K, N in w.matrices] if w.matrices else [(w.K, w.N)]
    for K, N in shapes:
        bits = W.schedule_for(w, K)
        assert q.qgemm_packed_word_rows(bits, K) == int(bits.astype(np.int64).sum())
        offs = q.qgemm_offsets(bits, K)
        assert np.array_equal(offs, W.offsets(bits))
        assert q.qgemm_validate_schedule(bits, offs, K, int(offs[-1])) == 0


def test_schedule_validation_errors():
    bits = np.array([4, 2, 8, 3], np.uint8)
    offs = q.qgemm_offsets(bits, 128)
    assert q.qgemm_validate_schedule(bits, offs, 128, 16) == -3       # qw_rows mismatch
    bad = offs.copy()
    bad[2] += 1
    assert q.qgemm_validate_schedule(bits, bad, 128, 17) == -3
    with pytest.raises(q.QGemmError):
        q.qgemm_packed_word_rows(np.array([7], np.uint8), 32)
    with pytest.raises(q.QGemmError):
        q.qgemm_packed_word_rows(np.array([4], np.uint8), 33)


def test_workspace_and_sizes():
    assert q.qgemm_workspace_bytes(1, 8192, 28672) > 0
    assert q.qgemm_workspace_bytes(0, 8192, 28672) == 0
    assert q.qgemm_workspace_bytes(1, 33, 64) == 0
    lib = q._lib
    assert lib.qgemm_packed_bytes(621, 28672) == 4 * 621 * 28672
    assert lib.qgemm_scale_bytes(8192, 28672) == 2 * 64 * 28672
    assert lib.qgemm_scale_bytes(160, 8) == 2 * 2 * 8
    assert q.qgemm_path_for(1, 8192, 8192) == 0      # integer GEMV
    assert q.qgemm_path_for(4, 8192, 8192) == 0
    assert q.qgemm_path_for(5, 8192, 8192) == 1      # tensor-core GEMV
    assert q.qgemm_path_for(11, 8192, 8192) == 1
    assert q.qgemm_path_for(12, 8192, 8192) == 2     # few tiles: the split-k GEMM
    assert q.qgemm_path_for(16, 8192, 28672) == 1    # 112 tiles, no split: the GEMV
    assert q.qgemm_path_for(17, 8192, 8192) == 2
    assert q.qgemm_path_for(2048, 8192, 8192) == 2   # GEMM


def _fake(addr):
    return ctypes.c_void_p(addr)


def test_host_argument_errors_return_status_without_launching():
    lib = q._lib
    A = 0x7f0000000000  # never dereferenced: every case fails before any CUDA call
    good = dict(x=_fake(A), dt=0, perm=_fake(A), qw=_fake(A), rows=16, s=_fake(A), b=_fake(A),
                o=_fake(A), M=1, K=128, N=64, y=_fake(A), ws=_fake(A), wsb=1 << 20, st=_fake(0))

    def call(**kw):
        a = dict(good, **kw)
        return lib.qgemm(a["x"], a["dt"], a["perm"], a["qw"], a["rows"], a["s"], a["b"], a["o"],
                         a["M"], a["K"], a["N"], a["y"], a["ws"], a["wsb"], a["st"])

    assert call(x=_fake(0)) == -1
    assert call(y=_fake(0)) == -1
    assert call(dt=7) == -6
    assert call(K=100) == -2
    assert call(N=60) == -2
    assert call(M=0) == -2
    assert call(rows=7) == -2          # fewer than 2 rows per block
    assert call(rows=33) == -2         # more than 8 rows per block
    assert call(x=_fake(A + 8)) == -4
    assert call(qw=_fake(A + 4)) == -4
    assert lib.qgemm_pack(_fake(0), _fake(A), _fake(A), 128, 64, 16, _fake(A), _fake(0)) == -1
    assert lib.qgemm_pack(_fake(A), _fake(A), _fake(A), 128, 64, 16, _fake(A + 2), _fake(0)) == -4
    assert lib.qgemm_dequant(_fake(A), 16, _fake(A), _fake(A), _fake(A), 100, 64, _fake(A), _fake(0)) == -2


def test_gemm_plan_and_workspace():
    """M > 16: one 256 x 256 output tile per CTA, the permuted activations in
    the workspace, shared memory within the 227 KB a CTA may use up to K = 65536."""
    plan = q.qgemm_plan_info(2048, 8192, 28672, 992)
    assert plan["path"] == 2
    # 896 tiles: six whole waves of 148, the last 8 tiles split 4 ways (the cap)
    assert plan["ring"] == 4 and plan["grid"] == 888 + 8 * 4
    assert plan["smem"] <= 227 * 1024
    assert q.qgemm_workspace_bytes(2048, 8192, 28672) >= 2048 * 8192 * 2 + 8 * 4 * 256 * 256 * 4
    big = q.qgemm_plan_info(17, 65536, 8, 2 * 2048)
    assert big["smem"] <= 227 * 1024
    # one output tile: k is split (at most 4 ways), 8+ k steps each
    ks = big["ring"]
    assert ks == 4 and big["grid"] == ks
    assert q.qgemm_workspace_bytes(17, 65536, 8) >= 17 * 65536 * 2 + ks * 256 * 256 * 4


def _cpu_args(M=2, K=256, N=64):
    import torch
    nb = K // 32
    rows = 2 * nb
    return dict(
        x=torch.zeros(M, K, dtype=torch.float16), perm=torch.arange(K, dtype=torch.int32),
        qw=torch.zeros(rows, N, dtype=torch.int32),
        scales=torch.zeros((K + 127) // 128, N, dtype=torch.float16),
        bits=torch.full((nb,), 2, dtype=torch.uint8),
        offs=torch.arange(0, 2 * nb + 1, 2, dtype=torch.int32),
        y=torch.zeros(M, N, dtype=torch.float16))


@pytest.mark.parametrize("fn", ["qgemm", "qgemm_decode_noalloc"])
@pytest.mark.parametrize("bad", ["y_rows", "perm", "qw_cols", "scales", "bits", "offs", "x_1d"])
def test_binding_rejects_mismatched_shapes(fn, bad):
    """The binding checks every shape before a pointer reaches the C ABI, so a
    mismatch is a ValueError on the host, never an out-of-bounds access."""
    import torch
    a = _cpu_args()
    if bad == "y_rows":
        a["y"] = torch.zeros(4, 64, dtype=torch.float16)
    elif bad == "perm":
        a["perm"] = torch.arange(255, dtype=torch.int32)
    elif bad == "qw_cols":
        a["qw"] = torch.zeros(16, 72, dtype=torch.int32)
    elif bad == "scales":
        a["scales"] = torch.zeros(3, 64, dtype=torch.float16)
    elif bad == "bits":
        a["bits"] = torch.full((7,), 2, dtype=torch.uint8)
    elif bad == "offs":
        a["offs"] = torch.zeros(8, dtype=torch.int32)
    elif bad == "x_1d":
        a["x"] = torch.zeros(256, dtype=torch.float16)
    with pytest.raises(ValueError):
        getattr(q, fn)(**a)


def test_binding_shapes_ok_then_needs_cuda_tensors():
    """Consistent shapes pass the shape checks; host tensors are then refused."""
    with pytest.raises(TypeError):
        q.qgemm(**_cpu_args())


def test_pack_and_dequant_reject_mismatched_shapes():
    import torch
    a = _cpu_args()
    with pytest.raises(ValueError):
        q.qgemm_pack(torch.zeros(256, 64, dtype=torch.uint8), a["bits"], a["offs"],
                     torch.zeros(16, 56, dtype=torch.int32))
    with pytest.raises(ValueError):
        q.qgemm_dequant(a["qw"], torch.zeros(3, 64, dtype=torch.float16), a["bits"], a["offs"],
                        torch.zeros(256, 64, dtype=torch.float16))


def test_noalloc_scratch_size_agrees_and_serves_every_decode_shape():
    """The binding's copy of QGEMM_NOALLOC_SCRATCH_BYTES is the header's, and
    the largest decode shape the ABI accepts (M = 4, K = 65536, N = 2^24)
    needs no more scratch than the built-in buffer holds."""
    text = open(HEADER).read()
    m = re.search(r"#define QGEMM_NOALLOC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", text)
    assert m, "header constant not found"
    assert int(m.group(1)) << int(m.group(2)) == q.NOALLOC_SCRATCH_BYTES
    for M in (1, 2, 3, 4):
        assert 0 < q.qgemm_noalloc_scratch_bytes(M, 65536, 1 << 24) <= q.NOALLOC_SCRATCH_BYTES


def test_kv_cache_entry_points_check_arguments_on_the_host():
    lib = q._lib
    P = ctypes.c_void_p
    dummy = P(16)
    assert lib.qgemm_kv_quantize(None, 1, 128, 4, dummy, dummy, None) == -1       # null
    assert lib.qgemm_kv_quantize(dummy, 1, 96, 4, dummy, dummy, None) == -2       # D not a power of two
    assert lib.qgemm_kv_quantize(dummy, -1, 128, 4, dummy, dummy, None) == -2     # negative count
    assert lib.qgemm_kv_quantize(dummy, 1, 128, 7, dummy, dummy, None) == -3      # width
    assert lib.qgemm_kv_quantize(P(17), 1, 128, 4, dummy, dummy, None) == -4      # alignment
    assert lib.qgemm_kv_quantize(P(4100), 1, 128, 4, dummy, dummy, None) == -4    # fp16 vectors: 8 bytes
    assert lib.qgemm_kv_dequantize(dummy, dummy, 1, 128, 4, P(4100), None) == -4
    assert lib.qgemm_kv_dequantize(dummy, dummy, 1, 512, 4, dummy, None) == -2
    assert lib.qgemm_kv_dequantize(dummy, dummy, 1, 128, 1, dummy, None) == -3
    assert lib.qgemm_kv_quantize(dummy, 0, 128, 4, dummy, dummy, None) == 0       # nothing to do


def test_quantize_entry_point_checks_arguments_on_the_host():
    lib = q._lib
    P = ctypes.c_void_p
    d = P(256)
    ws = q._lib.qgemm_quantize_workspace_bytes(256, 64)
    assert ws > 0
    assert lib.qgemm_quantize(None, d, 256, 64, d, d, None, None, d, ws, None) == -1
    assert lib.qgemm_quantize(d, d, 250, 64, d, d, None, None, d, ws, None) == -2   # K % 32
    assert lib.qgemm_quantize(d, d, 256, 64, P(264), d, None, None, d, ws, None) == -4
    assert lib.qgemm_quantize(d, d, 256, 64, d, d, None, None, d, ws - 1, None) == -5
