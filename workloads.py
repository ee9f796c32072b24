"""Seeded synthetic inputs for the mixed-bitwidth Q-GEMM workloads.

This module only draws inputs: bit schedules, permutations, codes, packed words,
scales and activations.  It contains none of the method's arithmetic (no packing,
unpacking, dequantisation or multiplication), so the CPU oracle and the CUDA
path can both be fed from it without sharing any computation.

Every draw comes from one counter-based generator, SplitMix64 (Steele, Lea and
Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014):

    state_i = key + (i + 1) * 0x9E3779B97F4A7C15   (mod 2^64)
    out_i   = mix64(state_i)

``mix64`` is the published SplitMix64 finaliser (xor-shift 30, multiply
0xBF58476D1CE4E5B9, xor-shift 27, multiply 0x94D049BB133111EB, xor-shift 31).
Values are computed with torch int64 tensors whose wrap-around arithmetic equals
uint64 arithmetic, so the same code gives bit-identical integers on the CPU and
on a CUDA device.  Floating-point draws (normals, log-normals) are computed in
float64 and rounded float64 -> float32 -> float16/bfloat16 (both steps RNE).

Streams: 1 bit schedule, 2 permutation, 3 packed words, 4 scales, 5 activations,
6 unpacked codes.  A stream key is mix64((seed << 32) ^ (layer << 16) ^
(matrix << 8) ^ stream).

The workloads are synthetic stand-ins: the pages describe 70B-class Llama
decoding at about 2.5 bits per weight on one consumer GPU (nightvoyager.top
exllamav2 report, "核心价值提炼"; promptquorum "EXL2量化是什么"), and no real
weights or datasets are used.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
MIX1 = 0xBF58476D1CE4E5B9
MIX2 = 0x94D049BB133111EB

STREAM_SCHEDULE = 1
STREAM_PERM = 2
STREAM_WORDS = 3
STREAM_SCALES = 4
STREAM_X = 5
STREAM_CODES = 6

BLOCK_ROWS = 32      # rows of W that share one bitwidth
GROUP_ROWS = 128     # rows of W that share one fp16 scale per column
ALLOWED_BITS = (2, 3, 4, 5, 6, 8)


def _s64(v: int) -> int:
    """Python int -> the int64 with the same low 64 bits."""
    v &= MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def _mix64_int(z: int) -> int:
    z &= MASK64
    z = ((z ^ (z >> 30)) * MIX1) & MASK64
    z = ((z ^ (z >> 27)) * MIX2) & MASK64
    return z ^ (z >> 31)


def _srl(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix64(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _srl(z, 30)) * _s64(MIX1)
    z = (z ^ _srl(z, 27)) * _s64(MIX2)
    return z ^ _srl(z, 31)


def stream_key(seed: int, stream: int, layer: int = 0, matrix: int = 0) -> int:
    return _mix64_int((seed << 32) ^ (layer << 16) ^ (matrix << 8) ^ stream)


def raw(key: int, idx: torch.Tensor) -> torch.Tensor:
    """SplitMix64 outputs (int64 bit patterns) for counter values ``idx``."""
    idx = idx.to(torch.int64)
    return _mix64(idx * _s64(GAMMA) + _s64(key + GAMMA))


def _u53(v: torch.Tensor) -> torch.Tensor:
    """Top 53 bits as an exact float64 in [0, 1)."""
    return _srl(v, 11).to(torch.float64) * (2.0 ** -53)


def normals(key: int, idx: torch.Tensor) -> torch.Tensor:
    """Standard normals by Box-Muller (cosine branch), float64."""
    idx = idx.to(torch.int64)
    u1 = _u53(raw(key, 2 * idx))
    u2 = _u53(raw(key, 2 * idx + 1))
    return torch.sqrt(-2.0 * torch.log(1.0 - u1)) * torch.cos(2.0 * math.pi * u2)


def _to_half(v64: torch.Tensor, dtype=torch.float16) -> torch.Tensor:
    return v64.to(torch.float32).to(dtype)


# --------------------------------------------------------------------------
# schedules, permutations, codes, words, scales, activations
# --------------------------------------------------------------------------

def target_word_rows(nb: int, target_bpw: float) -> int:
    """Sum of block widths for a target average bpw that counts the scale.

    One fp16 scale per 128 rows adds 16/128 = 0.125 bpw, so the mean block
    width is target - 0.125; the sum is rounded half to even (Python round).
    """
    return int(round((target_bpw - 0.125) * nb))


def bit_schedule(nb: int, allowed, target_sum: int, seed: int = 0, layer: int = 0,
                 matrix: int = 0, hi_frac: float = 0.1, sort: bool = True) -> np.ndarray:
    """Seeded per-block bitwidths with sum ``target_sum``.

    The first ceil(hi_frac * nb) blocks start at the smallest allowed width that
    is >= 5, the rest at the smallest allowed width.  Random blocks are then
    bumped to the next allowed width while the sum stays <= target_sum.  With
    ``sort`` the widths are sorted non-increasing, so the act-order-first rows
    get the most bits.
    """
    A = sorted(allowed)
    n_hi = int(math.ceil(hi_frac * nb))
    hi0 = min(a for a in A if a >= 5) if any(a >= 5 for a in A) else A[-1]
    b = [hi0] * n_hi + [A[0]] * (nb - n_hi)
    total = sum(b)
    if total > target_sum:
        raise ValueError(f"schedule infeasible: start sum {total} > target {target_sum}")
    key = stream_key(seed, STREAM_SCHEDULE, layer, matrix)
    tries, chunk = 0, None
    while total < target_sum and tries < 1_000_000:
        if tries % 4096 == 0:
            chunk = _srl(raw(key, torch.arange(tries, tries + 4096)), 11).tolist()
        j = chunk[tries % 4096] % nb
        tries += 1
        i = A.index(b[j])
        if i + 1 < len(A):
            nxt = A[i + 1]
            if total - b[j] + nxt <= target_sum:
                total += nxt - b[j]
                b[j] = nxt
    if sort:
        b.sort(reverse=True)
    return np.asarray(b, dtype=np.uint8)


def random_schedule(nb: int, allowed=ALLOWED_BITS, seed: int = 0, layer: int = 0,
                    matrix: int = 0) -> np.ndarray:
    """Unsorted widths drawn uniformly from ``allowed`` (test schedules that a
    kernel must not assume to be monotone)."""
    key = stream_key(seed, STREAM_SCHEDULE, layer, matrix ^ 0x80)
    r = _srl(raw(key, torch.arange(nb)), 11).numpy()
    A = np.asarray(sorted(allowed), dtype=np.uint8)
    return A[r % len(A)]


def uniform_schedule(nb: int, bits: int) -> np.ndarray:
    return np.full(nb, bits, dtype=np.uint8)


def permutation(K: int, seed: int = 0, layer: int = 0, matrix: int = 0,
                identity: bool = False) -> np.ndarray:
    """Seeded Fisher-Yates shuffle: for i = K-1..1, j = r_i mod (i+1), swap."""
    p = np.arange(K, dtype=np.int32)
    if identity:
        return p
    key = stream_key(seed, STREAM_PERM, layer, matrix)
    r = _srl(raw(key, torch.arange(K)), 11).numpy()
    for i in range(K - 1, 0, -1):
        j = int(r[i] % (i + 1))
        p[i], p[j] = p[j], p[i]
    return p


def offsets(bits: np.ndarray) -> np.ndarray:
    """Prefix sums of the block widths: the caller-side table the API takes."""
    o = np.zeros(len(bits) + 1, dtype=np.int32)
    o[1:] = np.cumsum(bits.astype(np.int64))
    return o


def codes(bits: np.ndarray, N: int, seed: int = 0, layer: int = 0, matrix: int = 0,
          device="cpu") -> torch.Tensor:
    """Unpacked codes uint8 [K, N], uniform in [0, 2^b - 1] for the row's block."""
    K = len(bits) * BLOCK_ROWS
    key = stream_key(seed, STREAM_CODES, layer, matrix)
    v = raw(key, torch.arange(K * N, device=device, dtype=torch.int64))
    b_row = torch.as_tensor(np.repeat(bits.astype(np.int64), BLOCK_ROWS), device=device)
    mask = (torch.ones_like(b_row) << b_row) - 1
    return (v.view(K, N) & mask[:, None]).to(torch.uint8)


def words(word_rows: int, N: int, seed: int = 0, layer: int = 0, matrix: int = 0,
          device="cpu", cols=None, row_chunk: int = 64) -> torch.Tensor:
    """Packed words as int32 bit patterns [word_rows, N] (or [word_rows, len(cols)]).

    Uniform random 32-bit words are exactly uniform codes for every width, so
    large workloads draw the packed stream directly.
    """
    key = stream_key(seed, STREAM_WORDS, layer, matrix)
    if cols is not None:
        c = torch.as_tensor(cols, dtype=torch.int64, device=device)
        idx = torch.arange(word_rows, device=device, dtype=torch.int64)[:, None] * N + c[None, :]
        return (raw(key, idx) & 0xFFFFFFFF).to(torch.int32)
    out = torch.empty(word_rows, N, dtype=torch.int32, device=device)
    for r0 in range(0, word_rows, row_chunk):
        r1 = min(word_rows, r0 + row_chunk)
        idx = torch.arange(r0 * N, r1 * N, device=device, dtype=torch.int64)
        out[r0:r1] = (raw(key, idx) & 0xFFFFFFFF).to(torch.int32).view(r1 - r0, N)
    return out


def group_bits(bits: np.ndarray) -> np.ndarray:
    """Widest block in each 128-row group (the scale law's b)."""
    per = GROUP_ROWS // BLOCK_ROWS
    G = (len(bits) + per - 1) // per
    return np.array([bits[g * per:(g + 1) * per].max() for g in range(G)], dtype=np.int64)


def scales(bits: np.ndarray, N: int, seed: int = 0, layer: int = 0, matrix: int = 0,
           device="cpu", cols=None, base: float = 0.02, sigma: float = 0.25) -> torch.Tensor:
    """fp16 scales [G, N]: (base / 2^(b_g - 1)) * lognormal(0, sigma)."""
    bg = torch.as_tensor(group_bits(bits), device=device, dtype=torch.float64)
    G = bg.numel()
    key = stream_key(seed, STREAM_SCALES, layer, matrix)
    c = torch.arange(N, device=device, dtype=torch.int64) if cols is None else \
        torch.as_tensor(cols, dtype=torch.int64, device=device)
    idx = torch.arange(G, device=device, dtype=torch.int64)[:, None] * N + c[None, :]
    ln = torch.exp(sigma * normals(key, idx))
    return _to_half((base / torch.exp2(bg - 1.0))[:, None] * ln)


def activations(M: int, K: int, seed: int = 0, layer: int = 0, matrix: int = 0,
                dtype=torch.float16, device="cpu") -> torch.Tensor:
    """x ~ N(0, 1), shape [M, K], rounded to fp16 or bf16."""
    key = stream_key(seed, STREAM_X, layer, matrix)
    idx = torch.arange(M * K, device=device, dtype=torch.int64)
    return _to_half(normals(key, idx), dtype).view(M, K)


# --------------------------------------------------------------------------
# the five workloads
# --------------------------------------------------------------------------

LLAMA70B_MATRICES = (          # (name, K, N): y[M, N] = x[M, K] . W[K, N]
    ("q", 8192, 8192), ("k", 8192, 1024), ("v", 8192, 1024), ("o", 8192, 8192),
    ("gate", 8192, 28672), ("up", 8192, 28672), ("down", 28672, 8192),
)


@dataclass(frozen=True)
class Workload:
    name: str
    K: int
    N: int
    Ms: tuple
    allowed: tuple = ALLOWED_BITS
    target_bpw: float | None = None
    uniform_bits: int | None = None
    identity_perm: bool = False
    x_dtype: torch.dtype = torch.float16
    layers: int = 1
    matrices: tuple = field(default=())
    description: str = ""


WORKLOADS = {
    "single_4096x4096_u4": Workload(
        "single_4096x4096_u4", 4096, 4096, (1,), uniform_bits=4, identity_perm=True,
        description="one linear layer, uniform 4-bit, identity perm, M=1"),
    "decode_8192x28672_2p55": Workload(
        "decode_8192x28672_2p55", 8192, 28672, (1, 2, 4, 8), target_bpw=2.55,
        description="70B MLP up_proj shape, 2.55 bpw mixed {2,3,4,5,6,8}, M in {1,2,4,8}"),
    "llama70b_stack_2p5": Workload(
        "llama70b_stack_2p5", 0, 0, (1,), target_bpw=2.5, layers=80,
        matrices=LLAMA70B_MATRICES,
        description="80 layers x 7 Llama-3-70B linears, 2.5 bpw, M=1 per token"),
    "prefill_2048x8192x28672_4p0": Workload(
        "prefill_2048x8192x28672_4p0", 8192, 28672, (2048,), allowed=(3, 4, 5, 6),
        target_bpw=4.0, x_dtype=torch.bfloat16,
        description="prefill M=2048, 4.0 bpw mixed {3,4,5,6}, bf16 x"),
    "sweep_8192x8192_3p75": Workload(
        "sweep_8192x8192_3p75", 8192, 8192, (1, 2, 4, 8, 16, 32, 64, 128, 256, 512),
        target_bpw=3.75, description="M sweep at 3.75 bpw for the GEMV/GEMM crossover"),
}


def schedule_for(w: Workload, K: int, layer: int = 0, matrix: int = 0, seed: int = 0):
    nb = K // BLOCK_ROWS
    if w.uniform_bits is not None:
        return uniform_schedule(nb, w.uniform_bits)
    return bit_schedule(nb, w.allowed, target_word_rows(nb, w.target_bpw), seed, layer, matrix)


def make_problem(w: Workload, M: int, layer: int = 0, matrix: int = 0, seed: int = 0,
                 device="cpu", K: int | None = None, N: int | None = None, cols=None):
    """All inputs of one Q-GEMM call: bits, offs (host numpy), perm, words,
    scales, x (torch tensors on ``device``)."""
    if w.matrices:
        _, K0, N0 = w.matrices[matrix]
    else:
        K0, N0 = w.K, w.N
    K = K0 if K is None else K
    N = N0 if N is None else N
    bits = schedule_for(w, K, layer, matrix, seed)
    offs = offsets(bits)
    perm = permutation(K, seed, layer, matrix, identity=w.identity_perm)
    return dict(
        K=K, N=N, M=M, bits=bits, offs=offs,
        perm=torch.as_tensor(perm, device=device),
        words=words(int(offs[-1]), N, seed, layer, matrix, device=device, cols=cols),
        scales=scales(bits, N, seed, layer, matrix, device=device, cols=cols),
        x=activations(M, K, seed, layer, matrix, dtype=w.x_dtype, device=device),
    )
