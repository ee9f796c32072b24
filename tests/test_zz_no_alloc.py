"""The allocation-free decode entry point, qgemm_decode_noalloc.

Some callers cannot allocate device memory: a runtime that plans every byte
up front and owns the only allocator, a plugin that may not allocate behind
its host's back, a decode loop that cannot pay for cudaFree's device-wide
synchronisation.  For them the library has one entry point whose scratch is a
buffer built into the library.  These tests call it through the C ABI and
compare it with the CPU oracle, within the tolerance of the other GEMV tests,
and with qgemm() (which takes a caller workspace and runs the same kernel
and schedule) bit for bit, on two calls in a row (the second call finds the
buffer as the first left it) and across shapes that share the buffer.  A
warmed call must leave the caching allocator's statistics and the device's
free memory as it found them.

The file name makes pytest collect it last, so a run that stops at the first
failure has run every other test before this one.
"""
import numpy as np
import pytest
import torch

from tests import problems as P

pytestmark = pytest.mark.gpu

CASES = [
    (1, 8192, 4104, torch.float16),
    (2, 1024, 1048, torch.float16),
    (3, 160, 264, torch.bfloat16),
    (4, 4096, 776, torch.bfloat16),
]


@pytest.fixture(scope="module")
def q():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import mixed_bitwidth_weight_b200 as lib
    lib.qgemm_device_error(clear=True)
    yield lib
    torch.cuda.synchronize()
    assert lib.qgemm_device_error(clear=True) == 0


def _qgemm(q, g, M, K, N):
    """The same product through qgemm() with its own zeroed workspace."""
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y, q.workspace(M, K, N))
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("M,K,N,x_dtype", CASES, ids=lambda v: str(v))
def test_noalloc_matches_oracle_and_qgemm_on_two_calls_in_a_row(q, M, K, N, x_dtype):
    pr = P.make(K, N, M=M, kind="shuffled", seed=101 + M, x_dtype=x_dtype)
    g = P.to_gpu(pr)
    ref = P.ref_y(pr)
    y_qgemm = _qgemm(q, g, M, K, N)
    P.check_close(y_qgemm, ref)
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        q.qgemm_decode_noalloc(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y)
        torch.cuda.synchronize()
        P.check_close(y, ref)
        assert torch.equal(y, y_qgemm)


def test_noalloc_warmed_call_allocates_nothing(q):
    M, K, N = 1, 4096, 2056
    pr = P.make(K, N, M=M, kind="shuffled", seed=55)
    g = P.to_gpu(pr)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    args = (g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y)
    q.qgemm_decode_noalloc(*args)  # first call: module load, scratch address lookup
    torch.cuda.synchronize()
    stats0 = torch.cuda.memory_stats()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        q.qgemm_decode_noalloc(*args)
    torch.cuda.synchronize()
    stats1 = torch.cuda.memory_stats()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    for key in ("allocation.all.allocated", "segment.all.allocated", "allocated_bytes.all.allocated",
                "reserved_bytes.all.allocated"):
        assert stats1.get(key, 0) == stats0.get(key, 0), key
    P.check_close(y, P.ref_y(pr))


def test_noalloc_buffer_carries_no_state_between_shapes(q):
    """Calls of different shapes back to back on one stream: each leaves the
    shared buffer in a state the next must not depend on."""
    probs = []
    for i, (M, K, N, x_dtype) in enumerate(CASES):
        pr = P.make(K, N, M=M, kind="sorted", seed=7 + i, x_dtype=x_dtype)
        g = P.to_gpu(pr)
        probs.append((M, K, N, g, P.ref_y(pr)))
    ys = []
    for M, K, N, g, _ in probs + probs[::-1]:
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        q.qgemm_decode_noalloc(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y)
        ys.append(y)
    torch.cuda.synchronize()
    for (M, K, N, g, ref), y in zip(probs + probs[::-1], ys):
        P.check_close(y, ref)


def test_noalloc_refuses_what_it_cannot_serve(q):
    K, N = 256, 264
    pr = P.make(K, N, M=5, kind="shuffled", seed=3)
    g = P.to_gpu(pr)
    y = torch.empty((5, N), dtype=torch.float16, device="cuda")
    with pytest.raises(q.QGemmError, match="unsupported shape"):
        q.qgemm_decode_noalloc(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y)
    # the largest decode shape the library accepts still fits the built-in buffer
    assert 0 < q.qgemm_noalloc_scratch_bytes(4, 65536, 1 << 24) <= q.NOALLOC_SCRATCH_BYTES


def test_noalloc_reset_then_calls_stay_correct(q):
    """qgemm_noalloc_reset (the recovery after a call that gave up on a wait)
    zeroes the tickets; calls before and after it agree with the oracle."""
    M, K, N = 2, 2048, 1032
    pr = P.make(K, N, M=M, kind="shuffled", seed=404)
    g = P.to_gpu(pr)
    ref = P.ref_y(pr)
    args = (g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"])
    y0 = torch.empty((M, N), dtype=torch.float16, device="cuda")
    q.qgemm_decode_noalloc(*args, y0)
    q.qgemm_noalloc_reset()
    y1 = torch.empty((M, N), dtype=torch.float16, device="cuda")
    q.qgemm_decode_noalloc(*args, y1)
    torch.cuda.synchronize()
    P.check_close(y0, ref)
    assert torch.equal(y0, y1)
