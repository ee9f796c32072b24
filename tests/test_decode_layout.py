"""The integer-MMA decoder's byte placement, checked on the CPU.

decode_block_i8<b> (csrc/decode_i8.cuh) turns a block's b packed words into the
32 A-operand bytes of one column; the activation side relies on its table
code -> (byte slot, bit offset P).  Here the oracle packs random codes, the
kernel's own decoder (compiled for the host) places them, and every byte must
equal code << P at the slot the table names, for every width, with each code
in exactly one slot.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
WIDTHS = (2, 3, 4, 5, 6, 8)


@pytest.fixture(scope="module")
def driver(tmp_path_factory):
    exe = str(tmp_path_factory.mktemp("dec") / "decode_layout")
    subprocess.run(["g++", "-O1", "-std=c++17", "-o", exe, os.path.join(HERE, "decode_layout_main.cpp")],
                   check=True)
    return exe


def run(exe, lines):
    out = subprocess.run([exe], input="\n".join(lines) + "\n", capture_output=True, text=True,
                         check=True).stdout.strip().splitlines()
    table = np.array(out[0].split(), dtype=np.int64).reshape(6, 32)
    rows = [np.array(l.split(), dtype=np.int64) for l in out[1:]]
    return table, rows


def test_slot_table_is_a_bijection_with_valid_offsets(driver):
    table, _ = run(driver, [])
    for wi, b in enumerate(WIDTHS):
        slots = table[wi] & 0xFF
        shifts = table[wi] >> 8
        assert sorted(slots.tolist()) == list(range(32)), b
        assert (shifts + b <= 8).all() and (shifts <= 6).all(), b


@pytest.mark.parametrize("b", WIDTHS)
def test_decoder_places_oracle_packed_codes(driver, b):
    rng = np.random.default_rng(b)
    N = 257
    codes = rng.integers(0, 1 << b, size=(32, N), dtype=np.uint8)
    codes[:, 0] = (1 << b) - 1                      # all ones
    codes[:, 1] = 0
    codes[:, 2] = np.arange(32) % (1 << b)
    words = oracle.pack(codes, np.array([b], dtype=np.uint8))   # [b, N] uint32
    lines = [f"{b} " + " ".join(str(int(words[i, n])) for i in range(b)) for n in range(N)]
    table, rows = run(driver, lines)
    wi = WIDTHS.index(b)
    slot = table[wi] & 0xFF
    shift = table[wi] >> 8
    for n in range(N):
        got = rows[n]
        want = np.zeros(32, dtype=np.int64)
        want[slot] = codes[:, n].astype(np.int64) << shift
        assert np.array_equal(got, want), (b, n)
