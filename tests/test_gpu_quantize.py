"""The GPU quantiser (qgemm_quantize) against the CPU oracle's: codes and
scales bit for bit, the 96 candidate errors and the chosen candidate exactly,
on seeded weights with the shapes, value spread and outlier rows of LLM
layers, across width schedules and ragged shapes; then the quantised layer
through pack and qgemm against the oracle's product."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import problems as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import mixed_bitwidth_weight_b200 as lib
    lib.qgemm_device_error(clear=True)
    yield lib
    torch.cuda.synchronize()
    assert lib.qgemm_device_error(clear=True) == 0


def weights(K, N, seed, outliers=True):
    rng = np.random.default_rng(seed)
    col = np.exp(rng.normal(0.0, 0.5, size=(1, N)))             # per-column spread
    w = rng.standard_normal((K, N)) * 0.02 * col
    if outliers:
        rows = rng.choice(K, size=max(1, K // 256), replace=False)
        w[rows] *= 25.0                                          # outlier input channels
    return w.astype(np.float16)


def run_gpu(q, w, bits):
    K, N = w.shape
    wd = torch.as_tensor(w.view(np.uint16).astype(np.int16)).view(torch.float16).cuda()
    bd = torch.as_tensor(bits).cuda()
    codes = torch.empty((K, N), dtype=torch.uint8, device="cuda")
    scales = torch.empty(((K + 127) // 128, N), dtype=torch.float16, device="cuda")
    err = torch.empty(96, dtype=torch.float64, device="cuda")
    best = torch.empty(1, dtype=torch.int32, device="cuda")
    q.qgemm_quantize(wd, bd, codes, scales, err=err, best=best)
    torch.cuda.synchronize()
    return (codes.cpu().numpy(), scales.cpu().view(torch.int16).numpy().view(np.uint16),
            err.cpu().numpy(), int(best.item()))


CASES = [
    (32, 8, "shuffled", 1),
    (256, 64, "shuffled", 2),
    (384, 136, "sorted", 3),           # a ragged last group (384 = 3 groups), N not a multiple of 64
    (1056, 520, "shuffled", 4),        # K % 128 = 32: a one-block last group
    (2048, 776, "sorted", 5),
]


@pytest.mark.parametrize("K,N,kind,seed", CASES, ids=lambda v: str(v))
def test_quantize_bit_exact_against_oracle(q, K, N, kind, seed):
    bits = P.schedule(kind, K // 32, seed=seed)
    w = weights(K, N, seed)
    ref = oracle.quantize(w, bits)
    codes, scales, err, best = run_gpu(q, w, bits)
    assert best == ref.best
    assert np.array_equal(err, ref.err)
    assert np.array_equal(scales, ref.scales)
    assert np.array_equal(codes, ref.codes)


@pytest.mark.parametrize("b", [2, 3, 4, 5, 6, 8])
def test_quantize_uniform_widths_and_special_columns(q, b):
    K, N = 512, 72
    bits = np.full(K // 32, b, dtype=np.uint8)
    w = weights(K, N, 10 + b)
    w[:, 5] = 0                                  # an all-zero column
    w[:, 6] = np.float16(3.0)                    # a constant column
    w[7, 7] = np.float16(-65504.0)               # the largest fp16 magnitude
    ref = oracle.quantize(w, bits)
    codes, scales, err, best = run_gpu(q, w, bits)
    assert best == ref.best and np.array_equal(err, ref.err)
    assert np.array_equal(scales, ref.scales) and np.array_equal(codes, ref.codes)


def test_quantize_then_pack_then_qgemm_matches_oracle(q):
    """The whole offline-to-online path: fp16 W -> GPU quantise -> GPU pack ->
    GPU qgemm, against the oracle's product of its own quantised layer."""
    K, N, M = 4096, 1032, 2
    wl = W.WORKLOADS["decode_8192x28672_2p55"]
    bits = W.bit_schedule(K // 32, wl.allowed, W.target_word_rows(K // 32, 2.55), 0, 0, 0)
    offs = W.offsets(bits)
    w = weights(K, N, 99)
    ref = oracle.quantize(w, bits)
    codes, scales, err, best = run_gpu(q, w, bits)
    assert np.array_equal(codes, ref.codes) and np.array_equal(scales, ref.scales)
    qw = torch.zeros((int(offs[-1]), N), dtype=torch.int32, device="cuda")
    q.qgemm_pack(torch.as_tensor(codes).cuda(), torch.as_tensor(bits).cuda(),
                 torch.as_tensor(offs).cuda(), qw)
    rng = np.random.default_rng(5)
    x = rng.standard_normal((M, K)).astype(np.float16)
    perm = rng.permutation(K).astype(np.int32)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    q.qgemm(torch.as_tensor(x).cuda(), torch.as_tensor(perm).cuda(), qw,
            torch.as_tensor(scales.view(np.float16)).cuda(), torch.as_tensor(bits).cuda(),
            torch.as_tensor(offs).cuda(), y, q.workspace(M, K, N))
    torch.cuda.synchronize()
    y_ref, _ = oracle.qgemm_f64(x.astype(np.float64), perm, oracle.pack(ref.codes, bits),
                                ref.scales, bits)
    P.check_close(y, y_ref)
