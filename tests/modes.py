"""Test helper: map a workload mode name onto the oracle's configuration."""
import numpy as np

import oracle
from kv_cache_bit_b200 import synth


def oracle_cfg(mode: str, d: int, bits: int) -> oracle.Cfg:
    names, seeded = synth.MODES[mode]
    flags = 0
    for n in names:
        flags |= getattr(oracle, n)
    signs = oracle.make_signs(synth.SIGN_SEED, d) if seeded else None
    return oracle.Cfg(d=d, bits=bits, flags=flags, signs=signs)


def f16bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float16).view(np.uint16)
