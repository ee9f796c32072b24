"""Pins that tie the CPU oracle to facts outside itself.

Each ``pin_*`` takes a loaded ``oracle.Oracle`` and raises AssertionError when
the oracle disagrees with the fact it checks.  The facts are:

* hand-derived packed words for K=32, N=1 (tests/golden/pack_k32_n1.txt);
* the closed-form packed size 4*N*sum(b) bytes and average bpw
  mean(b) + 16/128;
* bit-exact pack/unpack round trips;
* IEEE binary16 conversions against numpy's (exhaustive for fp16 -> double,
  random and constructed ties for double -> fp16);
* dequantisation special cases (s = 1, s = 2^e, subnormal s, zero codes);
* a hand-written brute-force loop for y at K = 32, N = 1;
* reduction to a dense numpy matmul for uniform widths and identity perm;
* invariants: one-hot x, row permutation inside blocks, linearity,
  per-row independence of x, column subsets;
* the quantiser: weights built on its own grid come back exactly (codes,
  scales, the p = 1 candidate, zero error); its error equals the squared
  distance to the pinned dequantisation of its output; ties round to even;
  an all-zero column gives zero-point codes and zero scales; codes stay
  within each block's width and scales on the 16-level grid of the chosen p;
* the KV-cache quantiser: dequantisation equals scipy's Sylvester Hadamard
  matrix applied to the codes' values and divided by D; vectors built on the
  grid come back as their codes and scales exactly; random vectors come back
  within the rounding bound of their group scales.

``tests/test_oracle.py`` runs them on the oracle and on copies of the oracle
with planted mistakes, which must each fail at least one pin.
"""
from __future__ import annotations

import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
BITS = (2, 3, 4, 5, 6, 8)


def _rng(seed):
    return np.random.default_rng(seed)


def _golden_pack():
    rows = []
    with open(os.path.join(HERE, "golden", "pack_k32_n1.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            rows.append((int(parts[0]), parts[1], [int(w, 16) for w in parts[2:]]))
    return rows


def _golden_codes(b, rule):
    r = np.arange(32)
    if rule == "r":
        q = r
    elif rule.startswith("r%"):
        q = r % int(rule[2:])
    elif rule == "max":
        q = np.full(32, (1 << b) - 1)
    elif rule == "last_top":
        q = np.zeros(32, dtype=np.int64)
        q[31] = 1 << (b - 1)
    else:
        raise ValueError(rule)
    return q.astype(np.uint8).reshape(32, 1)


def _expand_scales(s_f64, K):
    """[G, N] -> [K, N]: row k uses group k // 128."""
    return np.repeat(s_f64, 128, axis=0)[:K]


def _rand_problem(rng, bits, N, M=2, subnormal_scales=False):
    bits = np.asarray(bits, dtype=np.uint8)
    K = 32 * len(bits)
    codes = np.empty((K, N), dtype=np.uint8)
    for j, b in enumerate(bits):
        codes[32 * j:32 * j + 32] = rng.integers(0, 1 << int(b), size=(32, N))
    G = (K + 127) // 128
    s = rng.uniform(1e-3, 4e-2, size=(G, N)).astype(np.float16)
    if subnormal_scales:
        s[:, ::3] = (rng.integers(1, 1024, size=s[:, ::3].shape)).astype(np.uint16).view(np.float16)
    x = rng.standard_normal((M, K)).astype(np.float16)
    perm = rng.permutation(K).astype(np.int32)
    return bits, codes, s, x, perm


def _w_from_codes(codes, bits, s):
    """Dense double W from the unpacked codes (no packed words involved)."""
    K = codes.shape[0]
    z = np.repeat(np.left_shift(1, bits.astype(np.int64) - 1), 32)[:, None]
    return (codes.astype(np.int64) - z).astype(np.float64) * _expand_scales(s.astype(np.float64), K)


# --------------------------------------------------------------------------

def pin_golden_pack(o):
    for b, rule, expect in _golden_pack():
        qw = o.pack(_golden_codes(b, rule), np.array([b], dtype=np.uint8))
        got = [int(v) for v in qw.ravel()]
        assert got == expect, f"b={b} {rule}: {[hex(v) for v in got]} != {[hex(v) for v in expect]}"
        back = o.unpack(np.array(expect, dtype=np.uint32).reshape(-1, 1), np.array([b], np.uint8), 32)
        assert np.array_equal(back, _golden_codes(b, rule)), f"unpack golden b={b} {rule}"


def pin_closed_form_size(o):
    import workloads as W
    for name, w in W.WORKLOADS.items():
        shapes = [(K, N) for _, K, N in w.matrices] if w.matrices else [(w.K, w.N)]
        for K, N in shapes:
            bits = W.schedule_for(w, K)
            rows = o.word_rows(bits, K)
            assert rows == int(bits.astype(np.int64).sum())
            packed_bytes = 4 * N * rows
            assert packed_bytes == sum(32 * int(b) * N // 8 for b in bits)
            bpw = (packed_bytes * 8 + 2 * ((K + 127) // 128) * N * 8) / (K * N)
            assert abs(bpw - (bits.mean() + 16 / 128)) < 1e-12
            if w.target_bpw is not None:
                assert abs(bpw - w.target_bpw) < 0.5 / (K // 32) + 1e-12, (name, bpw)
    rng = _rng(1)
    bits = rng.choice(BITS, size=7).astype(np.uint8)
    codes = _rand_problem(rng, bits, 8)[1]
    assert o.pack(codes, bits).shape == (int(bits.astype(int).sum()), 8)


def pin_roundtrip(o):
    rng = _rng(2)
    schedules = [np.full(5, b, np.uint8) for b in BITS]
    schedules.append(rng.choice(BITS, size=9).astype(np.uint8))           # shuffled mix
    schedules.append(np.sort(rng.choice(BITS, size=9))[::-1].astype(np.uint8))
    for bits in schedules:
        _, codes, _, _, _ = _rand_problem(rng, bits, 24)
        qw = o.pack(codes, bits)
        assert np.array_equal(o.unpack(qw, bits, codes.shape[0]), codes), f"roundtrip {bits}"
        words = rng.integers(0, 1 << 32, size=qw.shape, dtype=np.uint64).astype(np.uint32)
        assert np.array_equal(o.pack(o.unpack(words, bits, codes.shape[0]), bits), words)


def pin_pack_rejects_wide_code(o):
    import oracle
    for b in BITS:
        if b == 8:
            continue
        c = np.zeros((32, 4), dtype=np.uint8)
        c[5, 2] = 1 << b
        try:
            o.pack(c, np.array([b], np.uint8))
        except oracle.OracleError:
            continue
        raise AssertionError(f"code {1 << b} accepted at b={b}")


def pin_half_to_double(o):
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = h.view(np.float16).astype(np.float64)
    got = o.half_to_double(h)
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all(), f"{int((~same).sum())} fp16 patterns convert differently"


def pin_double_to_half(o):
    rng = _rng(3)
    mags = np.exp2(rng.uniform(-30, 17, size=200_000))
    v = mags * rng.choice([-1.0, 1.0], size=mags.size)
    # midpoints between neighbouring fp16 values (ties) and points just off them
    h = rng.integers(0, 0x7bff, size=20_000).astype(np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).astype(np.uint16).view(np.float16).astype(np.float64)
    mid = (lo + hi) / 2
    v = np.concatenate([v, mid, -mid, np.nextafter(mid, 0), np.nextafter(mid, np.inf),
                        [0.0, -0.0, 65504.0, 65520.0, 65519.99, 1e6, 2.0 ** -25, 2.0 ** -26,
                         3 * 2.0 ** -26, 2.0 ** -24 * 1.5, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11]])
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).view(np.uint16)
    got = o.double_to_half(v)
    bad = got != ref
    assert not bad.any(), f"{int(bad.sum())} doubles round differently, e.g. {v[bad][:3]}"


def pin_dequant_special(o):
    rng = _rng(4)
    for b in BITS:
        bits = np.full(4, b, np.uint8)
        codes = rng.integers(0, 1 << b, size=(128, 6)).astype(np.uint8)
        qw = o.pack(codes, bits)
        z = 1 << (b - 1)
        for sbits in (0x3C00, 0x4000, 0x3400, 0x0001, 0x0200, 0xBC00):   # 1, 2, 1/4, 2^-24, 2^-15, -1
            s = np.full((1, 6), sbits, np.uint16)
            sv = float(np.array([sbits], np.uint16).view(np.float16)[0])
            w = o.dequant_f64(qw, s, bits, 128)
            assert np.array_equal(w, (codes.astype(np.float64) - z) * sv), (b, hex(sbits))
            w16 = o.dequant_f16(qw, s, bits, 128)
            assert np.array_equal(w16, w.astype(np.float16).view(np.uint16)), (b, hex(sbits))
        mid = o.pack(np.full((128, 3), z, np.uint8), bits)
        assert not o.dequant_f64(mid, np.full((1, 3), 0x3C00, np.uint16), bits, 128).any()


def pin_dequant_vs_codes(o):
    rng = _rng(5)
    for bits in (rng.choice(BITS, size=10), np.full(5, 8), rng.choice(BITS, size=3)):
        bits = bits.astype(np.uint8)
        _, codes, s, _, _ = _rand_problem(rng, bits, 16, subnormal_scales=True)
        qw = o.pack(codes, bits)
        K = codes.shape[0]
        w = o.dequant_f64(qw, s, bits, K)
        assert np.array_equal(w, _w_from_codes(codes, bits, s))
        assert np.array_equal(o.dequant_f16(qw, s, bits, K), w.astype(np.float16).view(np.uint16))


def pin_brute_force_k32(o):
    rng = _rng(6)
    for b in BITS:
        for trial in range(3):
            q = rng.integers(0, 1 << b, size=32)
            s16 = np.float16(rng.uniform(1e-4, 3e-2)) if trial else np.float16(2.0 ** -20)
            x = rng.standard_normal(32).astype(np.float16)
            perm = rng.permutation(32)
            y = 0.0
            for k in range(32):                      # the definition, written out
                y += float(x[perm[k]]) * ((int(q[k]) - 2 ** (b - 1)) * float(s16))
            qw = o.pack(q.astype(np.uint8).reshape(32, 1), np.array([b], np.uint8))
            got, _ = o.qgemm_f64(x.reshape(1, 32), perm.astype(np.int32), qw,
                                 np.array([[s16]]), np.array([b], np.uint8))
            scale = sum(abs(float(x[perm[k]]) * (int(q[k]) - 2 ** (b - 1)) * float(s16)) for k in range(32))
            assert abs(got[0, 0] - y) <= 1e-14 * scale + 1e-300, (b, got[0, 0], y)


def pin_dense_reduction(o):
    rng = _rng(7)
    for b in BITS:
        bits = np.full(10, b, np.uint8)                      # K = 320: 3 groups, ragged
        _, codes, s, x, _ = _rand_problem(rng, bits, 40, M=3)
        K = codes.shape[0]
        perm = np.arange(K, dtype=np.int32)
        qw = o.pack(codes, bits)
        y, _ = o.qgemm_f64(x, perm, qw, s, bits)
        ref = x.astype(np.float64) @ _w_from_codes(codes, bits, s)
        tol = 1e-12 * (np.abs(x.astype(np.float64)) @ np.abs(_w_from_codes(codes, bits, s)))
        assert (np.abs(y - ref) <= tol).all(), f"dense reduction b={b}"


def pin_one_hot(o):
    rng = _rng(8)
    bits = rng.choice(BITS, size=8).astype(np.uint8)
    _, codes, s, _, perm = _rand_problem(rng, bits, 12)
    K = codes.shape[0]
    qw = o.pack(codes, bits)
    w = _w_from_codes(codes, bits, s)
    inv = np.argsort(perm)
    for j in rng.choice(K, size=12, replace=False):
        x = np.zeros((1, K))
        x[0, j] = 1.0
        y, _ = o.qgemm_f64(x, perm, qw, s, bits)
        assert np.array_equal(y[0], w[inv[j]]), f"one-hot j={j}"


def pin_perm_consistency(o):
    rng = _rng(9)
    bits = rng.choice(BITS, size=12).astype(np.uint8)
    _, codes, s, x, perm = _rand_problem(rng, bits, 20, M=2)
    K = codes.shape[0]
    y0, _ = o.qgemm_f64(x, perm, o.pack(codes, bits), s, bits)
    # shuffle rows inside every block (same width, same group) together with perm
    sigma = np.concatenate([32 * j + rng.permutation(32) for j in range(len(bits))])
    y1, _ = o.qgemm_f64(x, perm[sigma], o.pack(codes[sigma], bits), s, bits)
    mag = np.abs(x.astype(np.float64)[:, perm]) @ np.abs(_w_from_codes(codes, bits, s))
    assert (np.abs(y1 - y0) <= 1e-12 * mag).all()


def pin_linearity_and_rows(o):
    rng = _rng(10)
    bits = rng.choice(BITS, size=6).astype(np.uint8)
    _, codes, s, x, perm = _rand_problem(rng, bits, 16, M=3)
    qw = o.pack(codes, bits)
    x = x.astype(np.float64)
    y, _ = o.qgemm_f64(x, perm, qw, s, bits)
    for m in range(3):
        ym, _ = o.qgemm_f64(x[m:m + 1], perm, qw, s, bits)
        assert np.array_equal(ym[0], y[m]), "rows of x must be independent"
    yl, _ = o.qgemm_f64(2.0 * x[0:1] + x[1:2], perm, qw, s, bits)
    mag = np.abs(x[:, perm]) @ np.abs(_w_from_codes(codes, bits, s))
    assert (np.abs(yl[0] - (2 * y[0] + y[1])) <= 1e-12 * (2 * mag[0] + mag[1])).all()


def pin_column_subset(o):
    rng = _rng(11)
    bits = rng.choice(BITS, size=5).astype(np.uint8)
    _, codes, s, x, perm = _rand_problem(rng, bits, 33, M=2)
    qw = o.pack(codes, bits)
    y, _ = o.qgemm_f64(x, perm, qw, s, bits)
    cols = rng.choice(33, size=9, replace=False)
    yc, _ = o.qgemm_f64(x, perm, qw, s, bits, cols=cols)
    assert np.array_equal(yc, y[:, cols])


# ------------------------------------------------------------- quantiser

def _grid_problem(rng, bits, N):
    """W exactly representable by the quantiser at p = 1: per column a power
    of two S and per group qs in {4, 8, 12, 16} (one group at 16), scales
    s = S qs^2 / 256, codes with at least one 0 per group (so the group's
    largest |W| / 2^(b-1) is s)."""
    bits = np.asarray(bits, dtype=np.uint8)
    K = 32 * len(bits)
    G = (K + 127) // 128
    codes = np.empty((K, N), dtype=np.uint8)
    for j, b in enumerate(bits):
        codes[32 * j:32 * j + 32] = rng.integers(0, 1 << int(b), size=(32, N))
    for g in range(G):
        codes[128 * g + rng.integers(0, min(128, K - 128 * g)), :] = 0
    qs = rng.choice([4, 8, 12, 16], size=(G, N))
    qs[rng.integers(0, G, size=N), np.arange(N)] = 16
    S = np.ldexp(1.0, rng.integers(-12, -4, size=N))
    s = (S[None, :] * qs.astype(np.float64) ** 2 / 256.0).astype(np.float16)
    assert np.array_equal(s.astype(np.float64), S[None, :] * qs.astype(np.float64) ** 2 / 256.0)
    w = _w_from_codes(codes, bits, s).astype(np.float16)
    assert np.array_equal(w.astype(np.float64), _w_from_codes(codes, bits, s))
    return bits, codes, s, w


def pin_quantize_grid_roundtrip(o):
    rng = _rng(21)
    bits = rng.choice(BITS, size=12).astype(np.uint8)
    bits, codes, s, w = _grid_problem(rng, bits, 40)
    r = o.quantize(w, bits)
    assert r.best == 64                                     # p = 96/96 = 1
    assert r.err[64] == 0.0 and (r.err[:64] > 0).all() and (r.err[65:] > 0).all()
    assert np.array_equal(r.codes, codes)
    assert np.array_equal(r.scales, s.view(np.uint16))


def pin_quantize_error_is_distance_to_dequant(o):
    rng = _rng(22)
    bits = rng.choice(BITS, size=9).astype(np.uint8)
    K, N = 32 * len(bits), 17
    w = (rng.standard_normal((K, N)) * 0.03).astype(np.float16)
    w[5, 3] = np.float16(0.9)                               # an outlier
    r = o.quantize(w, bits)
    wd = o.dequant_f64(o.pack(r.codes, bits), r.scales, bits, K)
    d = w.astype(np.float64) - wd
    col = np.array([np.cumsum(d[:, n] ** 2)[-1] for n in range(N)])
    assert np.array_equal(col, r.colerr[r.best])            # same terms, same k order
    assert r.err[r.best] == np.cumsum(col)[-1]
    assert r.err[r.best] == r.err.min() and int(np.argmin(r.err)) == r.best
    assert np.array_equal(r.err, np.array([np.cumsum(r.colerr[i])[-1] for i in range(96)]))


def pin_quantize_ranges_and_scale_grid(o):
    rng = _rng(23)
    bits = rng.choice(BITS, size=16).astype(np.uint8)
    K, N = 32 * len(bits), 24
    w = (rng.standard_normal((K, N)) * np.exp(rng.standard_normal((1, N)))).astype(np.float16)
    r = o.quantize(w, bits)
    widths = np.repeat(bits.astype(np.int64), 32)[:, None]
    assert (r.codes.astype(np.int64) < (1 << widths)).all()
    p = np.float32(32 + r.best) / np.float32(96)
    for n in range(N):
        wf = np.abs(w[:, n].astype(np.float64)) / np.left_shift(1, widths[:, 0] - 1)
        base = np.array([wf[128 * g:128 * g + 128].max() for g in range(r.scales.shape[0])])
        grid = {o.double_to_half(np.array([float(np.float32(p) * np.float32(np.float32(base.max()) *
                                                                         np.float32(q * q / 256.0)))]))[0]
                for q in range(1, 17)}
        assert set(r.scales[:, n].tolist()) <= grid


def pin_quantize_ties_to_even_and_zero_column(o):
    bits = np.array([8, 8, 8, 8], dtype=np.uint8)
    K, N = 128, 3
    q0 = np.tile(np.arange(128, dtype=np.int64)[:, None], (1, N))   # codes 0..127, z = 128
    w = ((q0 - 128).astype(np.float64)).astype(np.float16)          # s = 1 at p = 1
    w[10, 1] = np.float16(-117.5)                                   # between -118 and -117
    w[11, 1] = np.float16(-116.5)                                   # between -117 and -116
    w[:, 2] = 0
    r = o.quantize(w, bits)
    assert r.best == 64
    assert r.scales[0, 0] == np.float16(1.0).view(np.uint16)
    assert r.codes[10, 1] == 128 - 118 and r.codes[11, 1] == 128 - 116   # even neighbours
    assert (r.codes[:, 2] == 128).all() and r.scales[0, 2] == 0 and r.colerr[:, 2].max() == 0.0


def pin_quantize_ties_between_candidates_take_the_first(o):
    """An all-zero layer has zero error under every candidate: the lowest
    index wins, and the output is zero-point codes with zero scales."""
    bits = np.array([2, 5, 3, 8, 6], dtype=np.uint8)
    w = np.zeros((160, 9), dtype=np.float16)
    r = o.quantize(w, bits)
    assert r.best == 0 and (r.err == 0).all()
    assert (r.codes == np.repeat(np.left_shift(1, bits - 1), 32)[:, None]).all()
    assert (r.scales == 0).all()


# ------------------------------------------------------------- KV cache

def _kv_pack(q, b):
    """Codes [n, G, 32] -> words [n, G, b], code r at stream bits [r b, r b + b)."""
    n, G, _ = q.shape
    w = np.zeros((n, G, b), dtype=np.uint32)
    for r in range(32):
        for k in range(b):
            p = r * b + k
            w[:, :, p // 32] |= (((q[:, :, r] >> k) & 1).astype(np.uint32) << np.uint32(p % 32))
    return w


def pin_kv_dequant_is_scaled_hadamard(o):
    import scipy.linalg
    rng = _rng(31)
    for D in (32, 64, 128, 256):
        for b in (2, 4, 8):
            n, z = 6, 1 << (b - 1)
            q = rng.integers(0, 1 << b, size=(n, D // 32, 32))
            s = np.ldexp(1.0, rng.integers(-3, 2, size=(n, D // 32)))          # exact fp16
            u = ((q - z) * s[:, :, None]).reshape(n, D)
            want = (u @ scipy.linalg.hadamard(D).T.astype(np.float64)) / D      # exact in double
            got = o.kv_dequantize(_kv_pack(q, b), s.astype(np.float16), D, b).view(np.float16)
            assert np.array_equal(got.astype(np.float64), want.astype(np.float16).astype(np.float64)), (D, b)


def pin_kv_grid_roundtrip(o):
    import scipy.linalg
    rng = _rng(32)
    for D in (32, 128, 256):
        for b in (2, 3, 4, 5, 6, 8):
            n, z = 5, 1 << (b - 1)
            m = min(z - 1, 3)                             # small codes keep H u exact in fp16
            q = z + rng.integers(-m, m + 1, size=(n, D // 32, 32))
            q[:, :, 7] = 2 * z - 1                        # |q - z| reaches z - 1 in every group
            s = np.repeat(np.ldexp(1.0, rng.integers(-6, 0, size=(n, 1))), D // 32, axis=1)  # one per vector
            u = ((q - z) * s[:, :, None]).reshape(n, D)
            v = (u @ scipy.linalg.hadamard(D).T.astype(np.float64)) / D
            assert np.array_equal(v.astype(np.float16).astype(np.float64), v)  # exactly representable
            codes, scales = o.kv_quantize(v.astype(np.float16), b)
            assert np.array_equal(scales, s.astype(np.float16).view(np.uint16)), (D, b)
            assert np.array_equal(codes, _kv_pack(q, b)), (D, b)


def pin_kv_ties_round_to_even(o):
    import scipy.linalg
    D, b, z = 32, 4, 8
    s = 0.125
    u = np.zeros(D)
    u[7] = (z - 1) * s                  # fixes the scale at s
    u[3], u[5], u[9] = 0.5 * s, 2.5 * s, -1.5 * s
    v = (scipy.linalg.hadamard(D).astype(np.float64) @ u) / D
    assert np.array_equal(v.astype(np.float16).astype(np.float64), v)
    codes, scales = o.kv_quantize(v.astype(np.float16)[None, :], b)
    q = np.full((1, 1, 32), z)
    q[0, 0, 7], q[0, 0, 3], q[0, 0, 5], q[0, 0, 9] = 2 * z - 1, z, z + 2, z - 2   # ties to even
    assert scales[0, 0] == np.float16(s).view(np.uint16)
    assert np.array_equal(codes, _kv_pack(q, b))


def pin_kv_error_within_bound(o):
    rng = _rng(33)
    D, n = 128, 64
    v = (rng.standard_normal((n, D)) * np.exp(rng.standard_normal((n, 1)))).astype(np.float16)
    v[3, 17] = np.float16(200.0)                          # an outlier channel
    for b in (2, 4, 8):
        codes, scales = o.kv_quantize(v, b)
        back = o.kv_dequantize(codes, scales, D, b).view(np.float16).astype(np.float64)
        s = o.half_to_double(scales)                      # [n, D/32]
        bound = 32 * s.sum(axis=1) / 2 / D * (1 + 1e-3)   # |H (u - u')| / D <= sum |u - u'| / D
        err = np.abs(back - v.astype(np.float64))
        assert (err <= bound[:, None] + np.abs(back) * 2.0 ** -11 + 1e-7).all(), b


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]


def run_all(o):
    """Run every pin; return the names of those that fail."""
    failed = []
    for p in PINS:
        try:
            p(o)
        except Exception as e:  # noqa: BLE001 - any failure counts
            failed.append(f"{p.__name__}: {type(e).__name__}: {str(e)[:120]}")
    return failed


if __name__ == "__main__":          # used by the planted-mistake test
    import sys
    sys.path.insert(0, os.path.dirname(HERE))
    import oracle
    bad = run_all(oracle.Oracle(sys.argv[1]))
    print("\n".join(bad))
    sys.exit(1 if bad else 0)
