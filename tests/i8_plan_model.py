"""CPU model of the integer tensor-core decode GEMV's work split.

It restates, in Python, the planner (slices S, CTAs per slice, partial slots,
activation-tile capacity, ring rows) and the device-side bookkeeping (slice
boundaries, group parts, each CTA's unit range, the tiles it touches, the
contributors and ticket count of every tile) of gemv_i8_kernel, so that tests
can check on the CPU that every unit is computed exactly once, that every index
stays inside its buffer and that every tile's ticket count matches the CTAs
that really contribute.  It is test infrastructure: the library does not use it.
"""
from __future__ import annotations

import numpy as np

COLS = 256          # output columns per tile
HALF = 128
UNIT_COST = 24
MAX_SLICES = 160
MAX_PARTS = 40
MAX_BLOCKS = 128
SLICE_SEARCH = 6
ROW_BYTES = 1024
MAX_UNITS = (40 + 1) // 2
SMEM_BUDGET = 227 * 1024
SLOTS = 32
SETS = 4


def slice_blocks(nb, W, S):
    if S == 1:
        return nb
    return min(nb, ((W + S - 1) // S + 8) // 2 + 1)


def mp_of(M):
    return 1 if M <= 1 else 2 if M <= 2 else 4


def smem_layout(nb, S, bcap, ring, mp, maxt):
    o = 0
    o += ((nb + 1) * 4 + 15) & ~15
    o += (2 * SLOTS + (2 + 3 + 1) * SETS + 2) * 8
    o += 64
    o += SLOTS * 4
    o += (maxt * 4 + 15) & ~15
    o += ((3 * S + 1) * 4 + 15) & ~15
    o += ((MAX_PARTS + 1 + MAX_UNITS + 1 + MAX_PARTS) * 4 + 15) & ~15
    o += MAX_PARTS * 4 * 4 + MAX_PARTS * 4 * 8 + MAX_PARTS * 4 * 4
    o += 2 * SETS * mp * HALF * 4
    o = (o + 127) & ~127
    o += bcap * 32 * 16
    o = (o + 1023) & ~1023
    b_end = o
    o += ring * ROW_BYTES
    return o, b_end


def plan(M, K, N, W, sms=148):
    nb = K // 32
    T = -(-N // COLS)
    smin = 1
    while smin <= MAX_SLICES and slice_blocks(nb, W, smin) > MAX_BLOCKS:
        smin += 1
    assert smin <= MAX_SLICES
    smax = min(smin + SLICE_SEARCH, MAX_SLICES, nb, max(1, W // 8))
    best, bS, bC = 1e30, 0, 0
    for S in range(smin, max(smin, smax) + 1):
        if slice_blocks(nb, W, S) > MAX_BLOCKS:
            continue
        cap = sms // S
        if cap < 1:
            break
        rows = W // S - 8
        work = T * rows // (64 + UNIT_COST) if rows > 0 else 1
        cps = max(1, min(cap, work))
        eff = S * cps / sms
        score = (1.0 / eff) * (1.0 + 0.004 * S)
        if score < best:
            best, bS, bC = score, S, cps
    assert bS > 0
    mp = mp_of(M)
    bcap = slice_blocks(nb, W, bS)
    maxt = T // bC + 3
    total0, _ = smem_layout(nb, bS, bcap, 0, mp, maxt)
    ring = min((SMEM_BUDGET - total0) // ROW_BYTES, 1024)
    assert ring >= 2 * 65
    smem, _ = smem_layout(nb, bS, bcap, ring, mp, maxt)
    return dict(S=bS, cps=bC, grid=bS * bC, maxt=maxt, bcap=bcap, ring=ring, mp=mp,
                smem=smem, T=T, nb=nb)


def ws_bound(M, K, N, sms=148):
    nb = K // 32
    T = -(-N // COLS)
    smin = 1
    while smin < MAX_SLICES and slice_blocks(nb, 8 * nb, smin) > MAX_BLOCKS:
        smin += 1
    smax = min(smin + SLICE_SEARCH, MAX_SLICES, nb)
    slots = smax * T + 3 * sms
    return ((T * 4 + 255) // 256) * 256 + slots * mp_of(M) * COLS * 4


def device_split(pl, offs):
    """Everything the kernel derives from the schedule: per slice the block
    range, tile cost and last-part start; per CTA its unit range."""
    S, cps, T = pl["S"], pl["cps"], pl["T"]
    nb = len(offs) - 1
    W = int(offs[nb])
    jb = []
    for s in range(S + 1):
        if s == 0:
            jb.append(0)
        elif s == S:
            jb.append(nb)
        else:
            lo, hi = 0, nb
            while lo < hi:
                mid = (lo + hi) // 2
                if int(offs[mid]) * S >= s * W:
                    hi = mid
                else:
                    lo = mid + 1
            jb.append(lo)
    slices = []
    for s in range(S):
        j0, j1 = jb[s], jb[s + 1]
        g0, g1 = j0 >> 2, (j1 - 1) >> 2
        P = g1 - g0 + 1
        Q = (P + 1) // 2
        ct = int(offs[j1] - offs[j0]) + UNIT_COST * Q
        pj0 = [j0 if i == 0 else (j1 if i == P else 4 * (g0 + i)) for i in range(P + 1)]
        jl = pj0[2 * (Q - 1)]
        lastc = ct - (int(offs[j1] - offs[jl]) + UNIT_COST)
        uc = [int(offs[pj0[min(2 * q, P)]] - offs[j0]) + UNIT_COST * q for q in range(Q + 1)]
        slices.append(dict(j0=j0, j1=j1, P=P, Q=Q, ct=ct, lastc=lastc, pj0=pj0, uc=uc))
    return jb, slices


def unit_start(cc, cps, Ct, T, Q, uc):
    Ctot = T * Ct
    target = (cc * Ctot + cps - 1) // cps
    t, rem = divmod(target, Ct)
    if rem == 0:
        return t * Q
    for q in range(1, Q):
        if uc[q] >= rem:
            return t * Q + q
    return (t + 1) * Q


def first_tile(cc, cps, Ct, lastc, T):
    Ctot = T * Ct
    target = (cc * Ctot + cps - 1) // cps
    t, rem = divmod(target, Ct)
    return t + (1 if rem > lastc else 0)


def check(M, K, N, bits, sms=148):
    """Raise AssertionError if any coverage or bounds property fails."""
    offs = np.zeros(len(bits) + 1, dtype=np.int64)
    offs[1:] = np.cumsum(np.asarray(bits, dtype=np.int64))
    W = int(offs[-1])
    pl = plan(M, K, N, W, sms)
    S, cps, T, maxt = pl["S"], pl["cps"], pl["T"], pl["maxt"]
    jb, slices = device_split(pl, offs)
    assert all(jb[s] < jb[s + 1] for s in range(S)), "empty slice"
    ws_units = pl["grid"] * maxt
    assert ((T * 4 + 255) // 256) * 256 + ws_units * pl["mp"] * COLS * 4 <= ws_bound(M, K, N, sms)
    contrib = {}
    for s, sd in enumerate(slices):
        P, Q, ct = sd["P"], sd["Q"], sd["ct"]
        assert P <= MAX_PARTS
        assert sd["j1"] - sd["j0"] <= pl["bcap"], "activation tiles exceed capacity"
        covered = np.zeros(T * Q, dtype=np.int64)
        for cc in range(cps):
            u0 = unit_start(cc, cps, ct, T, Q, sd["uc"])
            u1 = unit_start(cc + 1, cps, ct, T, Q, sd["uc"])
            assert u1 > u0, "a CTA without units breaks the ticket count"
            covered[u0:u1] += 1
            t0, t1 = u0 // Q, (u1 - 1) // Q
            assert t1 - t0 + 1 <= maxt, "partial slot index out of range"
            assert first_tile(cc, cps, ct, sd["lastc"], T) == t0
            for u in range(u0, u1):
                t, q = divmod(u, Q)
                # CTA of a unit from its cost start
                assert (t * ct + sd["uc"][q]) * cps // (T * ct) == cc
                rows = int(offs[sd["pj0"][min(2 * q + 2, P)]] - offs[sd["pj0"][2 * q]])
                assert 1 + rows <= pl["ring"] and rows <= 64
            for t in range(t0, t1 + 1):
                contrib.setdefault(t, set()).add(s * cps + cc)
        assert (covered == 1).all(), "unit computed zero or several times"
    for t in range(T):
        first = t * cps // T
        expected = 0
        for s, sd in enumerate(slices):
            last = (t * sd["ct"] + sd["lastc"]) * cps // (T * sd["ct"])
            expected += last - first + 1
        assert expected == len(contrib[t]), (t, expected, len(contrib[t]))
    return pl
