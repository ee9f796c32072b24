"""Prefill GEMM (M > 16) against the oracle, through the C ABI: tcgen05 MMAs on
tiles dequantised into shared memory.  Within 1e-2 * rms(y_ref) elementwise;
unit activations bit-exact for fp16 input."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import problems as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import mixed_bitwidth_weight_b200 as q
    q.qgemm_device_error(clear=True)
    return q


@pytest.fixture
def q(cuda_lib):
    yield cuda_lib
    torch.cuda.synchronize()
    assert cuda_lib.qgemm_device_error(clear=True) == 0


def run(q, pr):
    g = P.to_gpu(pr)
    M, K, N = pr["M"], pr["K"], pr["N"]
    assert q.qgemm_path_for(M, K, N) == 2
    y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y, q.workspace(M, K, N))
    torch.cuda.synchronize()
    return y


# ragged M (not a multiple of 256), ragged N (not a multiple of 256), K with an
# odd number of 32-row blocks (a half k step), several tiles each way
SHAPES = [(17, 64, 256), (64, 96, 264), (256, 1024, 520), (300, 2048, 776), (513, 640, 1032)]


@pytest.mark.parametrize("M,K,N", SHAPES)
@pytest.mark.parametrize("x_dtype", [torch.float16, torch.bfloat16], ids=["f16", "bf16"])
def test_gemm_parity(q, M, K, N, x_dtype):
    pr = P.make(K, N, M=M, kind="shuffled", seed=M + K + N, x_dtype=x_dtype)
    P.check_close(run(q, pr), P.ref_y(pr))


@pytest.mark.parametrize("M,K,N", [(64, 8192, 512), (200, 4096, 256), (33, 2048, 1032)])
def test_gemm_split_k(q, M, K, N):
    """Few output tiles: k is split across CTAs; the last one adds the partial
    sums in split order (the same bits on every call, tickets back to zero)."""
    plan = q.qgemm_plan_info(M, K, N, int(P.make(K, 8, kind="shuffled", seed=1)["offs"][-1]))
    assert plan["ring"] > 1                       # k splits
    pr = P.make(K, N, M=M, kind="shuffled", seed=M + N, x_dtype=torch.bfloat16)
    a = run(q, pr)
    P.check_close(a, P.ref_y(pr))
    assert torch.equal(a, run(q, pr))


@pytest.mark.parametrize("kind", ["u2", "u3", "u4", "u5", "u6", "u8", "sorted"])
def test_gemm_parity_every_width(q, kind):
    pr = P.make(512, 520, M=96, kind=kind, seed=5)
    P.check_close(run(q, pr), P.ref_y(pr))


def test_gemm_one_hot_bit_exact_f16(q):
    """fp16 x = unit rows: y is a row of the fp16 dequantised matrix exactly
    (the B tile holds fp16(w), one product by 1.0, fp32 sum of one term)."""
    K, N, M = 512, 520, 64
    pr = P.make(K, N, M=M, kind="shuffled", seed=9)
    rng = np.random.default_rng(1)
    js = rng.integers(0, K, size=M)
    x = torch.zeros(M, K, dtype=torch.float16)
    x[np.arange(M), js] = 1.0
    pr["x"] = x
    y = run(q, pr)
    w16 = oracle.dequant_f16(pr["qw"], pr["scales"].numpy(), pr["bits"], K)
    inv = np.argsort(pr["perm"])
    assert np.array_equal(y.cpu().numpy().view(np.uint16), w16[inv[js]])


def test_gemm_subnormal_scales(q):
    pr = P.make(256, 264, M=40, kind="u8", seed=2, subnormal_scales=True)
    P.check_close(run(q, pr), P.ref_y(pr))


def test_gemm_whole_tiles_deterministic(q):
    """At least one whole wave of tiles: no k split, a fixed summation order,
    the same bits on every call."""
    M, K, N = 256, 512, 148 * 256
    plan = q.qgemm_plan_info(M, K, N, int(P.make(K, 8, kind="shuffled", seed=4)["offs"][-1]))
    assert plan["ring"] == 1
    pr = P.make(K, N, M=M, kind="shuffled", seed=4, x_dtype=torch.bfloat16)
    a, b = run(q, pr), run(q, pr)
    assert torch.equal(a, b)
    P.check_close(a, P.ref_y(pr))


def test_gemm_rejects_bad_device_schedule(q):
    K, N, M = 256, 256, 64
    pr = P.make(K, N, M=M, kind="shuffled", seed=3)
    g = P.to_gpu(pr)
    bad = g["bits"].clone()
    bad[1] = 7
    y = torch.zeros((M, N), dtype=torch.float16, device="cuda")
    q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], bad, g["offs"], y, q.workspace(M, K, N))
    torch.cuda.synchronize()
    assert q.qgemm_device_error(clear=True) & q.DEV_BAD_SCHEDULE
    assert bool((y == 0).all())


def test_gemm_reports_bad_perm(q):
    K, N, M = 256, 256, 32
    pr = P.make(K, N, M=M, kind="shuffled", seed=3)
    g = P.to_gpu(pr)
    perm = g["perm"].clone()
    perm[5] = K + 3
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    q.qgemm(g["x"], perm, g["qw"], g["scales"], g["bits"], g["offs"], y, q.workspace(M, K, N))
    torch.cuda.synchronize()
    assert q.qgemm_device_error(clear=True) & q.DEV_BAD_PERM


def test_gemm_prefill_layer_sampled_columns(q):
    """The 2048 x 8192 x 28672 prefill layer at 4.0 bpw (bf16 x) in the launch
    configuration the benchmark times; 96 sampled columns against the oracle."""
    w = W.WORKLOADS["prefill_2048x8192x28672_4p0"]
    M = 2048
    pr = W.make_problem(w, M, device="cuda")
    bits = torch.as_tensor(pr["bits"], device="cuda")
    offs = torch.as_tensor(pr["offs"], device="cuda")
    y = torch.empty((M, w.N), dtype=torch.float16, device="cuda")
    q.qgemm(pr["x"], pr["perm"], pr["words"], pr["scales"], bits, offs, y, q.workspace(M, w.K, w.N))
    torch.cuda.synchronize()
    cols = np.sort(np.random.default_rng(0).choice(w.N, size=96, replace=False))
    yr, _ = oracle.qgemm_f64(pr["x"].cpu().to(torch.float64).numpy(), pr["perm"].cpu().numpy(),
                             pr["words"].cpu().numpy().view(np.uint32), pr["scales"].cpu().numpy(),
                             pr["bits"], cols=cols)
    yg = y[:, torch.as_tensor(cols, device="cuda")]
    # rms over the sampled outputs stands in for the whole output's rms
    P.check_close(yg, yr)


@pytest.mark.parametrize("M", [1, 5, 16, 48, 64])
@pytest.mark.parametrize("knob", [1, 4])
def test_gemm_few_rows_forced(q, M, knob):
    """The GEMM at few rows of x (the MMA operands swapped, N = M rounded up
    to 16), chosen through a recorded tuning entry: whole tiles (knob 1) and
    k split four ways (knob 4); fp16 and bf16 input; one-hot rows exact."""
    K, N = 1024, 776
    try:
        q.qgemm_tune_record(M, K, N, 2, knob)
        for x_dtype in (torch.float16, torch.bfloat16):
            pr = P.make(K, N, M=M, kind="shuffled", seed=M + knob, x_dtype=x_dtype)
            g = P.to_gpu(pr)
            y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
            q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y, q.workspace(M, K, N))
            torch.cuda.synchronize()
            P.check_close(y, P.ref_y(pr))
        rng = np.random.default_rng(M)
        js = rng.integers(0, K, size=M)
        x = torch.zeros(M, K, dtype=torch.float16)
        x[np.arange(M), js] = 1.0
        pr["x"] = x
        g = P.to_gpu(pr)
        q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y, q.workspace(M, K, N))
        w16 = oracle.dequant_f16(pr["qw"], pr["scales"].numpy(), pr["bits"], K)
        inv = np.argsort(pr["perm"])
        assert np.array_equal(y.cpu().numpy().view(np.uint16), w16[inv[js]])
    finally:
        q.qgemm_tune_clear()
