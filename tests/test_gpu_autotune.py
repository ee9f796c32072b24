"""The autotuner on the GPU: it times every candidate variant of a shape,
records the fastest, dispatch then follows it, and the tuned call stays at
parity with the CPU oracle (as does every candidate)."""
import pytest
import torch

from tests import problems as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import mixed_bitwidth_weight_b200 as lib
    lib.qgemm_device_error(clear=True)
    lib.qgemm_tune_clear()
    yield lib
    torch.cuda.synchronize()
    lib.qgemm_tune_clear()
    lib.qgemm_set_autotune(0)
    assert lib.qgemm_device_error(clear=True) == 0


@pytest.mark.parametrize("M,K,N", [(1, 2048, 2056), (3, 1024, 1032), (9, 2048, 776), (40, 1536, 1288)])
def test_autotune_times_every_candidate_and_stays_at_parity(q, M, K, N):
    pr = P.make(K, N, M=M, kind="shuffled", seed=300 + M)
    g = P.to_gpu(pr)
    ref = P.ref_y(pr)
    y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    ws = q.workspace(M, K, N)
    res = q.qgemm_autotune(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y, ws,
                           warmup=3, iters=20)
    torch.cuda.synchronize()
    P.check_close(y, ref)                      # the last timed call's product
    timed = [c for c in res["candidates"] if c["us"] is not None]
    assert len(timed) == len(res["candidates"]) >= 2
    best = min(timed, key=lambda c: c["us"])
    assert (res["path"], res["knob"]) == (best["path"], best["knob"])
    assert q.qgemm_tune_lookup(M, K, N) == (best["path"], best["knob"])
    assert q.qgemm_path_for(M, K, N) == best["path"]
    # every candidate is a correct product
    for c in res["candidates"]:
        q.qgemm_tune_record(M, K, N, c["path"], c["knob"])
        y2 = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y2, ws)
        torch.cuda.synchronize()
        P.check_close(y2, ref)


def test_first_eager_call_tunes_and_capture_keeps_builtin(q):
    M, K, N = 2, 1024, 1048
    pr = P.make(K, N, M=M, kind="sorted", seed=77)
    g = P.to_gpu(pr)
    ref = P.ref_y(pr)
    ws = q.workspace(M, K, N)
    q.qgemm_tune_clear()
    q.qgemm_set_autotune(1)
    try:
        # inside a capture: no tuning, the built-in choice is captured
        y = torch.empty((M, N), dtype=torch.float16, device="cuda")
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y, ws)
        assert q.qgemm_tune_lookup(M, K, N) is None
        graph.replay()
        torch.cuda.synchronize()
        P.check_close(y, ref)
        # the first eager call tunes, then computes
        y3 = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y3, ws)
        torch.cuda.synchronize()
        assert q.qgemm_tune_lookup(M, K, N) is not None
        P.check_close(y3, ref)
    finally:
        q.qgemm_set_autotune(0)
