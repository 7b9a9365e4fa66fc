"""Pins of the oracle's code packing and pool layout against hand-written vectors."""
import os

import numpy as np
import pytest

from oracle import stq_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "packing_vectors.txt")


def _golden():
    out = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        b, codes, by = [s.strip() for s in line.split(";")]
        out.append((int(b), [int(x) for x in codes.split()], bytes.fromhex(by)))
    return out


@pytest.mark.parametrize("bits,codes,expect", _golden())
def test_pack_matches_hand_vectors(bits, codes, expect):
    got = O.pack_row(np.array(codes), bits)
    assert bytes(got.tobytes()) == expect
    back = O.unpack_row(np.frombuffer(expect, dtype=np.uint8), bits, len(codes))
    assert list(back) == codes


@pytest.mark.parametrize("bits", [2, 4, 6, 8])
def test_pack_round_trip_random(bits):
    rng = np.random.default_rng(bits)
    u = rng.integers(0, 1 << bits, size=(5, 3, 128))
    buf = O.pack_row(u, bits)
    assert buf.shape == (5, 3, 128 * bits // 8)
    assert np.array_equal(O.unpack_row(buf, bits, 128), u)


def test_six_bit_packs_four_codes_in_three_bytes():
    assert O.pack_row(np.zeros(128, dtype=np.int64), 6).size == 96


def test_layout_offsets_small():
    rb = np.array([[8, 8, 16, 4], [16, 16, 16, 16], [6, 2, 6, 2]])
    L = O.Layout(rb)  # d = 4 here, so rows are d*b/8 bytes
    assert list(L.row_code_offset[0]) == [0, 4, 8, 8]
    assert L.row_code_offset[2, 0] == 10 and L.row_code_offset[2, 1] == 13
    assert L.slot_code_bytes == 10 + 3 + 1 + 3 + 1
    assert L.n_pivot_rows == 5
    assert list(L.pivot_index[1]) == [1, 2, 3, 4] and L.pivot_index[0, 2] == 0


def test_pool_write_read_round_trip():
    rng = np.random.default_rng(0)
    rb = np.array([[6] * 8, [16] * 8, [2, 4, 6, 8, 16, 8, 4, 2]])
    L = O.Layout(rb)
    P = O.Pool(L, 4)
    B = 2
    u = np.zeros((B, 3, 8, 8), dtype=np.int64)
    for h in range(3):
        for i in range(8):
            b = rb[h, i]
            if b != 16:
                u[:, h, i] = rng.integers(1, 1 << b, size=(B, 8))
    r = rng.random((B, 3, 8)).astype(np.float32)
    c = rng.random((B, 3, 8)).astype(np.float32)
    piv = rng.standard_normal((B, 3, 8, 8)).astype(np.float16)
    P.write_heads([3, 1], u, r, c, piv)
    u2, r2, c2, piv2 = P.read_heads([3, 1])
    assert np.array_equal(u2, u)
    assert np.array_equal(r2, r) and np.array_equal(c2, c)
    mask = (rb == 16)[None, :, :, None] & np.ones((B, 3, 8, 8), bool)
    assert np.array_equal(piv2[mask], piv[mask])
