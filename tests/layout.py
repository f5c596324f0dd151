"""Byte layout of the library's packed V codes at head dim 128, test side.

The library stores V code rows of head dim 128 pair-interleaved: the rows of
tokens 2k and 2k + 1 form a pair block of 2 * row_bytes bytes whose 32-bit
word u (little endian) holds the 2-byte unit u (bytes 2u, 2u + 1) of row 2k
in its low half and of row 2k + 1 in its high half; for INT4 the 16-byte
chunk c of pair block k sits at chunk c ^ (2 (k & 1)).  The oracle keeps
token-major rows.  These helpers convert between the two so that tests can
compare codes byte for byte; they share nothing with the library.
"""
import numpy as np


def pairv_applies(d: int) -> bool:
    return d == 128


def _chunk_index(bits: int, npairs: int, nchunks: int) -> np.ndarray:
    """[npairs, nchunks]: stored chunk position of logical chunk c of pair k."""
    c = np.arange(nchunks)[None, :]
    k = np.arange(npairs)[:, None]
    return c ^ (2 * (k & 1)) if bits == 4 else np.broadcast_to(c, (npairs, nchunks))


def _permute_chunks(x: np.ndarray, bits: int, rb: int) -> np.ndarray:
    """Pair blocks [..., P, 2 rb] with chunk c moved from/to c ^ xor (an involution)."""
    if bits != 4:
        return x
    *lead, P, nb = x.shape
    nch = nb // 16
    ch = x.reshape(*lead, P, nch, 16)
    idx = _chunk_index(bits, P, nch).reshape((1,) * len(lead) + (P, nch, 1))
    return np.take_along_axis(ch, np.broadcast_to(idx, ch.shape), axis=-2).reshape(*lead, P, nb)


def pairv_to_rows(codes: np.ndarray, bits: int) -> np.ndarray:
    """[..., n, rb] pair-interleaved V codes (n even) -> token-major rows."""
    codes = np.asarray(codes, dtype=np.uint8)
    *lead, n, rb = codes.shape
    assert n % 2 == 0 and rb % 4 == 0
    x = _permute_chunks(codes.reshape(*lead, n // 2, 2 * rb), bits, rb)
    w = x.reshape(*lead, n // 2, rb // 2, 2, 2)  # [pair, unit, row, byte]
    return np.ascontiguousarray(np.swapaxes(w, -3, -2)).reshape(*lead, n, rb)


def rows_to_pairv(rows: np.ndarray, bits: int) -> np.ndarray:
    """Token-major rows [..., n, rb] -> pair-interleaved V codes."""
    rows = np.asarray(rows, dtype=np.uint8)
    *lead, n, rb = rows.shape
    assert n % 2 == 0 and rb % 4 == 0
    w = rows.reshape(*lead, n // 2, 2, rb // 2, 2)  # [pair, row, unit, byte]
    x = np.ascontiguousarray(np.swapaxes(w, -3, -2)).reshape(*lead, n // 2, 2 * rb)
    return _permute_chunks(x, bits, rb).reshape(*lead, n, rb)
