"""CPU checks of the test-side helpers that read GPU output (no GPU needed): the numpy
decoder of the packed layout against the hand-derived layout vectors, and the exact-grid
construction's claims."""
import os

import numpy as np
import pytest

from parity import codes_at_zero_np, np_unpack

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pack_layout.txt")


def _golden():
    rows = []
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        nb, codes, hexs = [x.strip() for x in line.split("|")]
        rows.append((int(nb), [int(c) for c in codes.split()],
                     bytes(int(h, 16) for h in hexs.split())))
    return rows


@pytest.mark.parametrize("nbits,codes,packed", _golden())
def test_np_unpack_reads_the_hand_derived_layout(nbits, codes, packed):
    got = np_unpack(np.frombuffer(packed, np.uint8), len(codes), nbits)
    assert got.tolist() == codes


def test_codes_at_zero_np_closed_forms():
    w = np.array([0.0, 0.25, 0.5, 1.0], np.float32)  # s = 3/1 = 3 at 2 bits
    assert codes_at_zero_np(w, 2, 0.0).tolist() == [0, 1, 2, 3]  # rint(0.75) = 1, rint(1.5) = 2
    assert codes_at_zero_np(w, 2, -1.0).tolist() == [0, 0, 0, 2]  # rint(0.5) = 0 (half to even)
    assert codes_at_zero_np(np.full(4, 2.0, np.float32), 4, 3.0).tolist() == [5, 5, 5, 5]
