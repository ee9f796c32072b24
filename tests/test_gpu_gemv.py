"""CUDA path against the oracle: pack and dequant bit-exact, the decode GEMV
within 1e-2 * rms(y_ref), plus edge cases and device-side error handling.
All calls go through the C ABI (mixed_bitwidth_weight_b200)."""
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


SHAPES = [(32, 8), (96, 24), (320, 264), (1024, 520), (4096, 776)]
KINDS = ["u2", "u3", "u4", "u5", "u6", "u8", "sorted", "shuffled"]


@pytest.mark.parametrize("K,N", SHAPES)
@pytest.mark.parametrize("kind", KINDS)
def test_pack_bit_exact(q, K, N, kind):
    if kind == "sorted" and K < 320:
        pytest.skip("sorted schedule needs >= 10 blocks")
    pr = P.make(K, N, kind=kind, seed=K + N)
    g = P.to_gpu(pr)
    qw = torch.full((int(pr["offs"][-1]), N), -1, dtype=torch.int32, device="cuda")
    q.qgemm_pack(g["codes"], g["bits"], g["offs"], qw)
    assert np.array_equal(qw.cpu().numpy().view(np.uint32), pr["qw"])


def test_pack_ignores_bits_above_the_width(q):
    """Codes wider than their block's width: only the low b bits are packed."""
    import oracle
    K, N = 1024, 1032
    pr = P.make(K, N, kind="shuffled", seed=5)
    rng = np.random.default_rng(6)
    wide = rng.integers(0, 256, size=pr["codes"].shape, dtype=np.uint8)
    widths = np.repeat(pr["bits"].astype(np.int64), 32)[:, None]
    low = (wide & ((1 << widths) - 1)).astype(np.uint8)
    g = P.to_gpu(pr)
    qw = torch.full((int(pr["offs"][-1]), N), -1, dtype=torch.int32, device="cuda")
    q.qgemm_pack(torch.as_tensor(wide).cuda(), g["bits"], g["offs"], qw)
    assert np.array_equal(qw.cpu().numpy().view(np.uint32), oracle.pack(low, pr["bits"]))


@pytest.mark.parametrize("K,N", SHAPES)
@pytest.mark.parametrize("kind", KINDS)
def test_dequant_bit_exact(q, K, N, kind):
    if kind == "sorted" and K < 320:
        pytest.skip("sorted schedule needs >= 10 blocks")
    pr = P.make(K, N, kind=kind, seed=3 * K + N, subnormal_scales=(kind == "shuffled"))
    g = P.to_gpu(pr)
    w = torch.empty(K, N, dtype=torch.float16, device="cuda")
    q.qgemm_dequant(g["qw"], g["scales"], g["bits"], g["offs"], w)
    ref = oracle.dequant_f16(pr["qw"], pr["scales"].numpy(), pr["bits"], K)
    assert np.array_equal(w.cpu().numpy().view(np.uint16), ref)


GEMV_SHAPES = [(32, 8), (160, 264), (1024, 1048), (2048, 4104), (4096, 776), (8192, 256)]


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 9, 12, 16])
@pytest.mark.parametrize("K,N", GEMV_SHAPES)
def test_gemv_parity(q, K, N, M):
    pr = P.make(K, N, M=M, kind="shuffled", seed=7 * M + K)
    g = P.to_gpu(pr)
    y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y, q.workspace(M, K, N))
    P.check_close(y, P.ref_y(pr))


@pytest.mark.parametrize("M", [1, 4, 13])
@pytest.mark.parametrize("K,N", [(160, 264), (4096, 1032)])
def test_gemv_parity_bf16(q, K, N, M):
    pr = P.make(K, N, M=M, kind="shuffled", seed=11 * M + N, x_dtype=torch.bfloat16)
    g = P.to_gpu(pr)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y, q.workspace(M, K, N))
    P.check_close(y, P.ref_y(pr))


def test_gemv_bf16_large_and_tiny_activations(q):
    K, N, M = 1024, 512, 3
    pr = P.make(K, N, M=M, kind="shuffled", seed=5, x_dtype=torch.bfloat16)
    pr["x"] = (pr["x"].float() * torch.tensor([[1e30], [1e-30], [1.0]])).to(torch.bfloat16)
    g = P.to_gpu(pr)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y, q.workspace(M, K, N))
    yr = P.ref_y(pr)
    # row 0 overflows fp16 output by design; rows 1 (tiny) and 2 must match
    assert torch.isinf(y[0]).any()
    P.check_close(y[2:3], yr[2:3])
    assert (y[1] == 0).all() or np.abs(y[1].float().cpu().numpy()).max() < 1e-3


@pytest.mark.parametrize("M", [1, 4, 8])
@pytest.mark.parametrize("kind", ["u2", "u3", "u4", "u5", "u6", "u8", "shuffled"])
def test_gemv_one_hot_bit_exact(q, kind, M):
    """x = unit rows: y is a row of the fp16 dequantised matrix, exactly (both
    GEMV families compute (q - z) * s exactly before the one rounding)."""
    K, N = 512, 520
    pr = P.make(K, N, M=M, kind=kind, seed=17)
    rng = np.random.default_rng(M)
    js = rng.choice(K, size=M, replace=False)
    x = torch.zeros(M, K, dtype=torch.float16)
    x[np.arange(M), js] = 1.0
    pr["x"] = x
    g = P.to_gpu(pr)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y, q.workspace(M, K, N))
    w16 = oracle.dequant_f16(pr["qw"], pr["scales"].numpy(), pr["bits"], K)
    inv = np.argsort(pr["perm"])
    assert np.array_equal(y.cpu().numpy().view(np.uint16), w16[inv[js]])


@pytest.mark.parametrize("M", [1, 2, 4])
@pytest.mark.parametrize("x_dtype", [torch.float16, torch.bfloat16])
def test_gemv_int_group_ranges_and_outliers(q, M, x_dtype):
    """The integer GEMV scales activations per (128-row group, token): groups
    whose magnitudes differ by 10^+-2 (fp16) or 10^+-3 (bf16), a group of
    zeros and one 20x outlier per group must all stay within the output
    tolerance."""
    K, N = 2048, 776
    pr = P.make(K, N, M=M, kind="shuffled", seed=31 + M, x_dtype=x_dtype)
    x = pr["x"].double()
    rng = np.random.default_rng(M)
    ng = K // 128
    span = 2 if x_dtype == torch.float16 else 3
    gscale = torch.tensor(10.0 ** rng.uniform(-span, span, size=(M, ng)))
    gscale[:, 3] = 0.0
    inv = np.argsort(pr["perm"])                       # x column -> act-order row
    grp = torch.as_tensor(inv // 128)
    x = x * gscale[:, grp]
    for m in range(M):
        for gi in range(ng):
            cols = np.nonzero(inv // 128 == gi)[0]
            x[m, cols[rng.integers(len(cols))]] *= 20.0
    pr["x"] = x.to(x_dtype)
    assert bool(torch.isfinite(pr["x"].float()).all())
    g = P.to_gpu(pr)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y, q.workspace(M, K, N))
    yr = P.ref_y(pr)
    assert np.abs(yr).max() < 60000.0                  # the fp16 output does not overflow
    P.check_close(y, yr)


def test_gemv_zero_activations_give_zero(q):
    K, N, M = 1024, 264, 2
    pr = P.make(K, N, M=M, kind="shuffled", seed=3)
    pr["x"] = torch.zeros(M, K, dtype=torch.float16)
    g = P.to_gpu(pr)
    y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y, q.workspace(M, K, N))
    assert bool((y == 0).all())


def test_gemv_deterministic_and_workspace_reset(q):
    K, N, M = 4096, 3000 // 8 * 8, 4
    pr = P.make(K, N, M=M, kind="shuffled", seed=21)
    g = P.to_gpu(pr)
    ws = q.workspace(M, K, N)
    ys = []
    for _ in range(3):
        y = torch.empty((M, N), dtype=torch.float16, device="cuda")
        q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y, ws)
        ys.append(y)
    torch.cuda.synchronize()
    assert all(torch.equal(ys[0], t) for t in ys[1:])
    tickets = ws[: (N + 255) // 256 * 4].view(torch.int32)
    assert int(tickets.abs().sum()) == 0


def test_gemv_identity_perm_uniform4(q):
    """Config-1 style: uniform 4-bit, identity perm."""
    K, N = 4096, 4096
    pr = P.make(K, N, M=1, kind="u4", identity=True, seed=0)
    g = P.to_gpu(pr)
    y = torch.empty((1, N), dtype=torch.float16, device="cuda")
    q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y, q.workspace(1, K, N))
    P.check_close(y, P.ref_y(pr))


def test_gemv_rejects_bad_device_schedule(q):
    K, N = 256, 256
    pr = P.make(K, N, M=1, kind="shuffled", seed=1)
    g = P.to_gpu(pr)
    bad = g["offs"].clone()
    bad[3] += 1                                  # inconsistent prefix sums
    y = torch.full((1, N), 7.0, dtype=torch.float16, device="cuda")
    q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], bad, y, q.workspace(1, K, N))
    torch.cuda.synchronize()
    assert q.qgemm_device_error(clear=True) & q.DEV_BAD_SCHEDULE
    assert (y == 7.0).all()
    badbits = g["bits"].clone()
    badbits[0] = 7
    q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], badbits, g["offs"], y, q.workspace(1, K, N))
    torch.cuda.synchronize()
    assert q.qgemm_device_error(clear=True) & q.DEV_BAD_SCHEDULE


def test_gemv_reports_bad_perm(q):
    K, N = 256, 256
    pr = P.make(K, N, M=1, kind="shuffled", seed=2)
    g = P.to_gpu(pr)
    perm = g["perm"].clone()
    perm[5] = K + 100
    y = torch.empty((1, N), dtype=torch.float16, device="cuda")
    q.qgemm(g["x"], perm, g["qw"], g["scales"], g["bits"], g["offs"], y, q.workspace(1, K, N))
    torch.cuda.synchronize()
    assert q.qgemm_device_error(clear=True) & q.DEV_BAD_PERM


def test_pack_rejects_bad_device_schedule(q):
    K, N = 128, 64
    pr = P.make(K, N, kind="u4", seed=3)
    g = P.to_gpu(pr)
    bad = g["offs"].clone()
    bad[-1] += 4
    qw = torch.zeros((int(pr["offs"][-1]), N), dtype=torch.int32, device="cuda")
    q.qgemm_pack(g["codes"], g["bits"], bad, qw)
    torch.cuda.synchronize()
    assert q.qgemm_device_error(clear=True) & q.DEV_BAD_SCHEDULE


def test_host_errors_on_device(q):
    pr = P.make(128, 64, kind="u4", seed=3)
    g = P.to_gpu(pr)
    y = torch.empty((1, 64), dtype=torch.float16, device="cuda")
    with pytest.raises(q.QGemmError):      # workspace too small
        q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y,
                torch.zeros(16, dtype=torch.uint8, device="cuda"))
    with pytest.raises(q.QGemmError):      # missing workspace
        q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y, None)


def test_generator_cpu_gpu_identical(q):
    a = W.words(40, 1024, seed=9, layer=3, matrix=2, device="cpu")
    b = W.words(40, 1024, seed=9, layer=3, matrix=2, device="cuda").cpu()
    assert torch.equal(a, b)
