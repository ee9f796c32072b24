"""Seeded test problems and comparison helpers shared by the GPU tests.

Inputs come from ``workloads`` (no arithmetic of the method); expected values
come only from the CPU oracle.  Nothing here calls the CUDA library.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads as W

TOL = 1e-2  # |y - y_ref| <= TOL * rms(y_ref), elementwise over the call's output


def schedule(kind: str, nb: int, seed: int = 0) -> np.ndarray:
    if kind.startswith("u"):                      # uniform width, e.g. "u4"
        return W.uniform_schedule(nb, int(kind[1:]))
    if kind == "sorted":                          # act-order: widest first, >=5 in the first 10%
        hi = int(np.ceil(0.1 * nb))
        lo = W.target_word_rows(nb, 3.0)
        lo = max(lo, 5 * hi + 2 * (nb - hi))
        return W.bit_schedule(nb, W.ALLOWED_BITS, lo, seed=seed)
    if kind == "shuffled":                        # any order, every width
        return W.random_schedule(nb, seed=seed)
    if kind == "prefill":                         # widths {3,4,5,6}
        return W.random_schedule(nb, (3, 4, 5, 6), seed=seed)
    raise ValueError(kind)


def make(K, N, M=1, kind="shuffled", seed=0, x_dtype=torch.float16, identity=False,
         subnormal_scales=False, words=False):
    """A problem with codes packed by the oracle (or random words with words=True)."""
    nb = K // 32
    bits = schedule(kind, nb, seed)
    offs = W.offsets(bits)
    if words:
        codes = None
        qw = W.words(int(offs[-1]), N, seed).numpy().view(np.uint32)
    else:
        codes = W.codes(bits, N, seed).numpy()
        qw = oracle.pack(codes, bits)
    s = W.scales(bits, N, seed)
    if subnormal_scales:
        s = s.clone()
        sv = s.view(torch.int16)
        sv[:, ::5] = (sv[:, ::5] & 0x03FF) | 1        # subnormal fp16 patterns
    x = W.activations(M, K, seed, dtype=x_dtype)
    perm = W.permutation(K, seed, identity=identity)
    return dict(K=K, N=N, M=M, bits=bits, offs=offs, codes=codes, qw=qw, scales=s, x=x,
                perm=perm)


def to_gpu(pr):
    d = "cuda"
    return dict(
        bits=torch.as_tensor(pr["bits"], device=d),
        offs=torch.as_tensor(pr["offs"], device=d),
        qw=torch.as_tensor(pr["qw"].view(np.int32), device=d),
        scales=pr["scales"].to(d),
        x=pr["x"].to(d),
        perm=torch.as_tensor(pr["perm"], device=d),
        codes=None if pr["codes"] is None else torch.as_tensor(pr["codes"], device=d),
    )


def x_f64(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.float64).numpy()


def ref_y(pr, cols=None):
    y, _ = oracle.qgemm_f64(x_f64(pr["x"]), pr["perm"], pr["qw"], pr["scales"].numpy(),
                            pr["bits"], cols=cols)
    return y


def check_close(y_gpu: torch.Tensor, y_ref: np.ndarray, tol: float = TOL, rms=None):
    y = y_gpu.detach().to(torch.float64).cpu().numpy()
    assert y.shape == y_ref.shape
    assert np.isfinite(y).all(), "non-finite output"
    rms = float(np.sqrt(np.mean(y_ref ** 2))) if rms is None else rms
    err = np.abs(y - y_ref)
    worst = float(err.max() / rms) if err.size else 0.0
    assert worst <= tol, f"max |y - y_ref| / rms(y_ref) = {worst:.3e} > {tol}"
    return worst
