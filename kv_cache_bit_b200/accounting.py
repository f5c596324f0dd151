"""Algorithmic byte counts of the library calls (what a call must move
through HBM at minimum), used for GB/s and roofline fractions.

Per quantized token and tensor: row_bytes codes + 2 * ntok bytes of fp16
per-token parameters + 2 * d / 128 bytes of per-block channel scales (and as
much again for NSN channel means, or under DQ the block record's bytes /
128); residual tokens cost 2 * d bytes.
"""
from __future__ import annotations

T = 128


def row_bytes(d: int, bits: int) -> int:
    return d * bits // 8


NSN, DQ = 4, 16


def ntok(flags: int) -> int:
    return (1 if flags & DQ else 2) if flags & NSN else 1


def dq_record_bytes(d: int) -> int:
    """Block record of the double-quantized NSN parameters: 4-bit codes of the
    d means and of the 128 s1, three fp16 values, padding to 16 bytes."""
    return (d // 2 + T // 2 + 6 + 15) // 16 * 16


def token_bytes(d: int, bits: int, flags: int) -> float:
    """Bytes of one quantized token of one tensor, block parameters amortized."""
    side = 0
    if flags & NSN:
        side = dq_record_bytes(d) if flags & DQ else 2 * d
    per_block = (2 * d if flags & 2 else 0) + side
    return row_bytes(d, bits) + 2 * ntok(flags) + per_block / T


def decode_bytes(d: int, bits: int, flags: int, B: int, Hkv: int, Hq: int, length: int) -> float:
    """One decode call: packed K and V plus side parameters of the quantized
    tokens, the fp16 residual tokens, the fp16 queries and the fp32 output."""
    nq = (length // T) * T
    r = length - nq
    per_bh = 2 * nq * token_bytes(d, bits, flags) + 2 * r * 2 * d
    return B * Hkv * per_bh + B * Hq * d * (2 + 4)


def quantize_bytes(d: int, bits: int, flags: int, B: int, Hkv: int, ntokens: int) -> float:
    """One bulk quantize of ntokens per (b, h) of K and V: fp16 read + packed write."""
    return 2 * B * Hkv * ntokens * (2 * d + token_bytes(d, bits, flags))


def append_bytes(d: int, bits: int, flags: int, B: int, Hkv: int, flush: bool) -> float:
    """One append: the fp16 token of K and V read and written; a flush also
    reads the 127 held tokens and writes one quantized block."""
    b = 2 * B * Hkv * (2 * d) * 2
    if flush:
        b += 2 * B * Hkv * (127 * 2 * d + T * token_bytes(d, bits, flags))
    return b
