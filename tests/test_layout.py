"""The test-side converter of the pair-interleaved V code layout."""
import numpy as np
import pytest

from tests.layout import pairv_to_rows, rows_to_pairv


@pytest.mark.parametrize("bits,rb", [(4, 64), (3, 48), (2, 32)])
def test_round_trip(bits, rb):
    rng = np.random.default_rng(5)
    rows = rng.integers(0, 256, size=(2, 3, 256, rb), dtype=np.uint8)
    pv = rows_to_pairv(rows, bits)
    assert not np.array_equal(pv, rows)
    assert np.array_equal(pairv_to_rows(pv, bits), rows)


def test_worked_example():
    # four INT4 rows of 64 bytes: row r byte b = 64 r + b (mod 256)
    rows = ((np.arange(4)[:, None] * 64 + np.arange(64)[None, :]) % 256).astype(np.uint8)
    pv = rows_to_pairv(rows, 4).reshape(-1)
    # pair 0 (rows 0, 1): word u = bytes (2u, 2u + 1) of row 0 then of row 1
    assert list(pv[0:8]) == [0, 1, 64, 65, 2, 3, 66, 67]
    # pair 1 (rows 2, 3), odd: chunk 0 of the pair block stored at chunk 2
    p1 = pv[128:256]
    assert list(p1[32:36]) == [128, 129, 192, 193]
    assert list(p1[0:4]) == [(128 + 16) % 256, (129 + 16) % 256, (192 + 16) % 256, (193 + 16) % 256]
    # INT3 / INT2: no chunk permutation
    pv2 = rows_to_pairv(rows[:, :32], 2).reshape(-1)
    assert list(pv2[64:68]) == [128, 129, 192, 193]
