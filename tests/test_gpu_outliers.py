"""Outlier activations over zero weights, against the oracle.

One activation per chosen 128-row group is made huge (1e4 or 6e4, near the
fp16 maximum) and every code of its weight row is set to the zero point, so
that row's weights are exactly 0 and the outlier contributes nothing to y.
The product the pages define (fp32 accumulation of x times the dequantised
weights) is then unaffected by the outlier, so every decode path must keep the
rest of the group's contribution within the usual 1e-2 * rms(y_ref): an
activation encoding whose error scales with the group's largest magnitude
fails here."""
import numpy as np
import pytest
import torch

import oracle
from tests import problems as P

pytestmark = pytest.mark.gpu


@pytest.fixture
def q():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import mixed_bitwidth_weight_b200 as lib
    lib.qgemm_device_error(clear=True)
    yield lib
    torch.cuda.synchronize()
    assert lib.qgemm_device_error(clear=True) == 0


def outlier_problem(K, N, M, mag, seed, n_groups=8, kind="shuffled"):
    pr = P.make(K, N, M=M, kind=kind, seed=seed)
    codes = pr["codes"].copy()
    bits = pr["bits"]
    rng = np.random.default_rng(seed)
    groups = rng.choice(K // 128, size=min(n_groups, K // 128), replace=False)
    x = pr["x"].clone()
    rows = []
    for g in groups:
        k = int(g) * 128 + int(rng.integers(128))       # act-order row of the outlier
        b = int(bits[k // 32])
        codes[k, :] = 1 << (b - 1)                       # zero point: w[k, :] == 0 exactly
        x[:, int(pr["perm"][k])] = mag * (1 if rng.integers(2) else -1)
        rows.append(k)
    pr["codes"] = codes
    pr["qw"] = oracle.pack(codes, bits)
    pr["x"] = x
    return pr, rows


@pytest.mark.parametrize("M", [1, 2, 4, 8, 13])
@pytest.mark.parametrize("mag", [1e4, 6e4])
def test_outlier_over_zero_row(q, M, mag):
    K, N = 8192, 1032
    pr, rows = outlier_problem(K, N, M, mag, seed=int(mag) % 97 + M)
    w16 = oracle.dequant_f16(pr["qw"], pr["scales"].numpy(), pr["bits"], K)
    assert not np.any(w16[rows].view(np.uint16) & 0x7FFF), "outlier rows must dequantise to zero"
    g = P.to_gpu(pr)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y, q.workspace(M, K, N))
    P.check_close(y, P.ref_y(pr))


@pytest.mark.parametrize("M", [1, 4])
def test_outlier_over_live_row(q, M):
    """The same outliers over ordinary weights: y is then dominated by them and
    must match to the same relative tolerance."""
    K, N = 4096, 520
    pr = P.make(K, N, M=M, kind="shuffled", seed=77 + M)
    x = pr["x"].clone()
    rng = np.random.default_rng(M)
    for g in rng.choice(K // 128, size=6, replace=False):
        x[:, int(pr["perm"][int(g) * 128 + int(rng.integers(128))])] = 3e4
    pr["x"] = x
    g = P.to_gpu(pr)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y, q.workspace(M, K, N))
    P.check_close(y, P.ref_y(pr))


def bf16_outlier_problem(K, N, M, mag, seed):
    """bf16 activations with one outlier of magnitude mag per chosen group,
    each over a zero-point weight row (as outlier_problem), so that the rest
    of each row spans a range of mag to 1."""
    pr, rows = outlier_problem(K, N, M, 1.0, seed)
    x = P.make(K, N, M=M, kind="shuffled", seed=seed, x_dtype=torch.bfloat16)["x"].clone()
    for k in rows:
        x[:, int(pr["perm"][k])] = mag
    pr["x"] = x
    return pr, rows


# The integer GEMV (M <= 4) encodes a group as int16 on the grid of its
# largest magnitude plus a second int16 part on a grid 2^15 times finer, so a
# value 2^24 below the group's maximum keeps about 5 bits (measured: 3.6e-2 *
# rms at M = 1); the fp16 paths scale whole rows, exactly for every value
# within 2^24 of the row maximum.
BF16_RANGES = [(M, 2.0 ** 20) for M in (1, 4, 8, 13, 32, 96)] + [(M, 2.0 ** 24) for M in (8, 13, 32, 96)]


@pytest.mark.parametrize("M,mag", BF16_RANGES)
def test_bf16_outlier_over_zero_row(q, M, mag):
    """bf16 input is brought to fp16 (or to integers) with a power-of-two
    scale set by the largest magnitude of its row or group: with the rest of
    the row 2^20 below that maximum every decode path (the integer GEMV, the
    tensor-core GEMV and the GEMM) keeps y within the usual tolerance, and the
    two fp16 paths still at 2^24."""
    K, N = 4096, 520
    pr, rows = bf16_outlier_problem(K, N, M, mag, seed=M + int(np.log2(mag)))
    w16 = oracle.dequant_f16(pr["qw"], pr["scales"].numpy(), pr["bits"], K)
    assert not np.any(w16[rows].view(np.uint16) & 0x7FFF), "outlier rows must dequantise to zero"
    g = P.to_gpu(pr)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    q.qgemm(g["x"], g["perm"], g["qw"], g["scales"], g["bits"], g["offs"], y, q.workspace(M, K, N))
    P.check_close(y, P.ref_y(pr))
