"""Work split of the integer tensor-core decode GEMV, checked on the CPU.

tests/i8_plan_model.py restates the planner and the kernel's device-side
bookkeeping; here it must agree with the library's own plan (qgemm_plan_info,
qgemm_workspace_bytes) and, for every benchmark layer and a spread of shapes
and schedules, compute every (tile, group part) unit exactly once, keep every
index inside its buffer and give every tile a ticket count equal to its real
contributors."""
import numpy as np
import pytest

import mixed_bitwidth_weight_b200 as q
import workloads as W
from tests import i8_plan_model as model


def _cases():
    out = []
    for name, w in W.WORKLOADS.items():
        shapes = [(K, N) for _, K, N in w.matrices] if w.matrices else [(w.K, w.N)]
        for K, N in shapes:
            out.append((f"{name}:{K}x{N}", K, N, W.schedule_for(w, K)))
    rng = np.random.default_rng(5)
    for K in (32, 96, 160, 1024, 8192, 28672, 65536):
        for N in (8, 120, 136, 4104):
            out.append((f"rand:{K}x{N}", K, N, rng.choice([2, 3, 4, 5, 6, 8], size=K // 32).astype(np.uint8)))
            out.append((f"u8:{K}x{N}", K, N, np.full(K // 32, 8, np.uint8)))
            out.append((f"u2:{K}x{N}", K, N, np.full(K // 32, 2, np.uint8)))
    return out


CASES = _cases()


@pytest.mark.parametrize("name,K,N,bits", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("M", [1, 4])
def test_split_covers_every_unit_once(name, K, N, bits, M):
    pl = model.check(M, K, N, bits)
    W_ = int(np.asarray(bits, dtype=np.int64).sum())
    info = q.qgemm_plan_info(M, K, N, W_)
    assert info["path"] == 0
    assert (info["grid"], info["ring"], info["smem"]) == (pl["grid"], pl["ring"], pl["smem"])
    assert q.qgemm_workspace_bytes(M, K, N) == model.ws_bound(M, K, N)
    assert pl["smem"] <= 227 * 1024
