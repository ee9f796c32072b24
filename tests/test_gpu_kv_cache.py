"""Hadamard-rotated KV-cache quantisation on the GPU against the CPU oracle:
codes and scales bit for bit, dequantised vectors bit for bit, for every
head size and width, on seeded K/V-like vectors (per-head spread, a few
outlier channels), and the round trip within the oracle-pinned bound."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import mixed_bitwidth_weight_b200 as lib
    lib.qgemm_device_error(clear=True)
    yield lib
    torch.cuda.synchronize()
    assert lib.qgemm_device_error(clear=True) == 0


def kv_vectors(tokens, heads, D, seed):
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((tokens, heads, D)) * np.exp(0.5 * rng.standard_normal((1, heads, 1)))
    v[:, :, rng.choice(D, size=2, replace=False)] *= 20.0      # outlier channels
    return v.astype(np.float16)


def to_gpu_f16(a):
    return torch.as_tensor(np.ascontiguousarray(a).view(np.int16)).view(torch.float16).cuda()


@pytest.mark.parametrize("D", [32, 64, 128, 256])
@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
def test_kv_quantize_and_dequantize_match_oracle(q, D, bits):
    v = kv_vectors(37, 8, D, seed=D + bits)                     # 296 vectors: a ragged last CTA
    n = v.shape[0] * v.shape[1]
    codes = torch.empty((37, 8, D // 32, bits), dtype=torch.int32, device="cuda")
    scales = torch.empty((37, 8, D // 32), dtype=torch.float16, device="cuda")
    q.qgemm_kv_quantize(to_gpu_f16(v), bits, codes, scales)
    back = torch.empty((37, 8, D), dtype=torch.float16, device="cuda")
    q.qgemm_kv_dequantize(codes, scales, bits, back)
    torch.cuda.synchronize()
    rc, rs = oracle.kv_quantize(v.reshape(n, D), bits)
    assert np.array_equal(codes.cpu().numpy().view(np.uint32).reshape(n, D // 32, bits), rc)
    assert np.array_equal(scales.cpu().view(torch.int16).numpy().view(np.uint16).reshape(n, D // 32), rs)
    rb = oracle.kv_dequantize(rc, rs, D, bits)
    assert np.array_equal(back.cpu().view(torch.int16).numpy().view(np.uint16).reshape(n, D), rb)


def test_kv_large_cache_sampled(q):
    """A 4-bit cache of 8192 tokens x 8 heads x 128 (Llama-3-70B K or V of
    one layer): bit-exact on sampled vectors, and the round-trip error of
    every vector within its group scales' bound."""
    T, H, D, b = 8192, 8, 128, 4
    v = kv_vectors(T, H, D, seed=7)
    codes = torch.empty((T, H, D // 32, b), dtype=torch.int32, device="cuda")
    scales = torch.empty((T, H, D // 32), dtype=torch.float16, device="cuda")
    vd = to_gpu_f16(v)
    q.qgemm_kv_quantize(vd, b, codes, scales)
    back = torch.empty_like(vd)
    q.qgemm_kv_dequantize(codes, scales, b, back)
    torch.cuda.synchronize()
    n = T * H
    idx = np.random.default_rng(1).choice(n, size=512, replace=False)
    rc, rs = oracle.kv_quantize(v.reshape(n, D)[idx], b)
    assert np.array_equal(codes.cpu().numpy().view(np.uint32).reshape(n, D // 32, b)[idx], rc)
    s = scales.float().double().reshape(n, D // 32)
    bound = 32 * s.sum(dim=1) / 2 / D * (1 + 1e-3)
    err = (back.double() - vd.double()).abs().reshape(n, D)
    assert bool((err <= bound[:, None] + back.double().abs().reshape(n, D) * 2.0 ** -11 + 1e-7).all())
