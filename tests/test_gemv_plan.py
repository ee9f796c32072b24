"""Host-side checks of the decode GEMV launch plan, without a GPU.

Both decode kernels (csrc/gemv_int.cuh for M <= 4, csrc/gemv.cuh for M <= 16)
split the (256-column tile, 128-row group) units into contiguous, equal-cost
ranges, one per CTA.  This file replays that
split in Python for the workload shapes and checks what keeps the kernel in
bounds: every unit is owned by exactly one CTA, the CTA that owns a unit is the
one the reducer expects (cta_of), a unit fits the shared-memory ring, and partial-sum slots stay
inside the workspace.
"""
import bisect

import numpy as np
import pytest

import mixed_bitwidth_weight_b200 as q
import workloads as W
from tests import problems as P

TILE = 256


def replay(offs, tiles, G, bpu=4):
    """The kernel's split: units are (tile, bpu blocks), numbered t*ng + g; a
    unit costs its word rows plus one.  bpu = 4 (one 128-row group) for the
    tensor-core GEMV, 8 (two groups) for the integer GEMV."""
    nb = len(offs) - 1
    ng = (nb + bpu - 1) // bpu
    Wt = int(offs[-1]) + ng
    C = tiles * Wt
    goffs = [int(offs[min(bpu * g, nb)]) + g for g in range(ng + 1)]

    def unit_start(i):
        if i >= G:
            return tiles * ng
        pos = (i * C + G - 1) // G
        t = pos // Wt
        rem = pos - t * Wt
        return t * ng + bisect.bisect_left(goffs, rem)

    def cta_of(u):
        t, g = divmod(u, ng)
        return ((t * Wt + goffs[g]) * G) // C

    return [unit_start(i) for i in range(G + 1)], cta_of, ng


def shapes():
    out = []
    for name, w in W.WORKLOADS.items():
        mats = [(K, N) for _, K, N in w.matrices] if w.matrices else [(w.K, w.N)]
        for K, N in mats:
            bits = W.schedule_for(w, K)
            out.append((name, K, N, bits))
    for K, N in [(32, 8), (160, 264), (1024, 1048), (2048, 4104), (8192, 256), (65536, 8)]:
        out.append(("small", K, N, P.schedule("shuffled", K // 32, seed=K)))
        out.append(("small_u2", K, N, W.uniform_schedule(K // 32, 2)))
        out.append(("small_u8", K, N, W.uniform_schedule(K // 32, 8)))
    return out


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 9, 16])
@pytest.mark.parametrize("case", shapes(), ids=lambda c: f"{c[0]}-{c[1]}x{c[2]}")
def test_gemv_plan_keeps_kernel_in_bounds(case, M):
    name, K, N, bits = case
    offs = W.offsets(bits)
    nb = K // 32
    rows = int(offs[-1])
    tiles = (N + TILE - 1) // TILE
    plan = q.qgemm_plan_info(M, K, N, rows)
    if plan["path"] == 2:
        pytest.skip("this shape's M runs the split-k GEMM")
    integer = plan["path"] == 0
    G = plan["grid"]
    cps = plan["ctas_per_sm"]
    if integer:
        mp = 1 if M == 1 else 2 if M == 2 else 4 if M <= 4 else 8 if M <= 8 else 16
        assert cps == (2 if mp <= 2 else 1)
    else:
        mp = 8 if M <= 8 else 16
        assert cps == 1                          # each CTA holds all of TMEM
    assert 1 <= G <= cps * plan["sms"]
    # resident CTAs fit the SM's 228 KB (1 KB reserved per CTA)
    assert cps * (plan["smem"] + 1024) <= 228 * 1024
    assert plan["ring"] >= 80
    bpu = 8 if integer else 4
    starts, cta_of, ng = replay(offs, tiles, G, bpu)
    assert starts[0] == 0 and starts[-1] == tiles * ng
    assert all(a <= b for a, b in zip(starts, starts[1:]))
    ws = q.qgemm_workspace_bytes(M, K, N)
    slot_bytes = mp * TILE * 4
    rec = (140 * mp + 4 + 15) // 16 * 16 if integer else 64 * mp   # integer: two int16 parts, three int32 arrays, a flag
    act_bytes = nb * rec + (0 if integer else ((nb + 3) // 4) * mp * 4 + 64)
    assert ws >= ((tiles * 4 + 255) // 256 * 256) + G * 2 * slot_bytes + act_bytes
    rng = np.random.default_rng(K + N + M)
    for i in range(G):
        u0, u1 = starts[i], starts[i + 1]
        n = u1 - u0
        assert n > 0, f"CTA {i} owns no unit (the reduction needs every range non-empty)"
        for u in {u0, u1 - 1, *rng.integers(u0, u1, size=min(4, n)).tolist()}:
            assert cta_of(u) == i
    # the reducer of a tile adds exactly the CTAs that own one of its units
    for t in range(tiles):
        owners = {cta_of(u) for u in range(t * ng, (t + 1) * ng)}
        first, last = cta_of(t * ng), cta_of(t * ng + ng - 1)
        expect = {c for c in range(first, last + 1) if starts[c] < starts[c + 1]}
        assert owners == expect, t
    # a unit (scale row, a group's word rows, activation records) fits the ring
    row_bytes = 1024 if integer else 1056
    need = max(1 + int(offs[min(bpu * g + bpu, nb)] - offs[bpu * g]) + -(-min(bpu, nb - bpu * g) * rec // row_bytes)
               for g in range(ng))
    assert need <= plan["ring"]


def ring_progress(rows_seq, R, slots=16):
    """Replay the producer's admission rule with the consumers releasing units
    in order only when asked: every unit must be admitted at the latest once all
    earlier units are released (no wait that can never end)."""
    def alloc(pos, total, need):
        if pos + need > R:
            total += R - pos
            pos = 0
        return pos, pos + need, total + need

    pos = pos_rel = 0
    total = total_rel = 0
    k_rel = 0
    for k, need in enumerate(rows_seq):
        assert need <= R
        _, ppos, ptotal = alloc(pos, total, need)
        while k - k_rel >= slots or (ptotal - total_rel > R and k_rel < k):
            _, pos_rel, total_rel = alloc(pos_rel, total_rel, rows_seq[k_rel])
            k_rel += 1
        _, pos, total = alloc(pos, total, need)


@pytest.mark.parametrize("M", [1, 2, 4])
@pytest.mark.parametrize("case", shapes(), ids=lambda c: f"{c[0]}-{c[1]}x{c[2]}")
def test_integer_gemv_ring_always_admits(case, M):
    name, K, N, bits = case
    offs = W.offsets(bits)
    nb = K // 32
    plan = q.qgemm_plan_info(M, K, N, int(offs[-1]))
    assert plan["path"] == 0
    mp = 1 if M == 1 else 2 if M == 2 else 4 if M <= 4 else 8 if M <= 8 else 16
    rec = (140 * mp + 4 + 15) // 16 * 16   # two int16 parts, three int32 arrays, a flag
    nu = (nb + 7) // 8
    rows = [1 + int(offs[min(8 * g + 8, nb)] - offs[8 * g]) + -(-min(8, nb - 8 * g) * rec // 1024)
            for g in range(nu)]
    seq = rows * 3                      # a CTA range can run over several tiles
    for start in range(0, nu, max(1, nu // 8)):
        ring_progress(seq[start:start + 2 * nu], plan["ring"])
