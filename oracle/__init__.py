"""Python face of the plain-C CPU oracle (oracle/kvq_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may use it; the CUDA library never does.
Everything here is argument marshalling (numpy arrays -> C pointers) plus a
thread pool over independent (batch, kv-head) slices; all arithmetic of the
method lives in the C file.

Array conventions (numpy):
  fp16 data is carried as ``uint16`` bit patterns (``arr.view(np.uint16)``).
  x        [B, H, S, d]        fp16 bits, tokens to quantize
  codes    [B, H, S_max, rb]   uint8 packed offset-binary codes
  tok      [B, H, S_max, nt]   fp16 bits per-token parameters
  chan     [B, H, S_max/128, d] fp16 bits per-channel scales (pchan)
  off      [B, H, S_max/128, d] fp16 bits per-channel means (NSN)
"""
from __future__ import annotations

import ctypes
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass
from typing import Optional

import numpy as np

from . import build as _build

NORM_SEP, PER_CHANNEL, NSN, HADAMARD, DQ = 1, 2, 4, 8, 16
T = 128

_lib = None
_P = ctypes.c_void_p


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.ko_f32_to_f16.restype = ctypes.c_uint16
        L.ko_f32_to_f16.argtypes = [ctypes.c_float]
        L.ko_f16_to_f32.restype = ctypes.c_float
        L.ko_f16_to_f32.argtypes = [ctypes.c_uint16]
        L.ko_f32_to_f16_array.argtypes = [_P, ctypes.c_long, _P]
        L.ko_f16_to_f32_array.argtypes = [_P, ctypes.c_long, _P]
        L.ko_splitmix64_next.restype = ctypes.c_uint64
        L.ko_splitmix64_next.argtypes = [ctypes.POINTER(ctypes.c_uint64)]
        L.ko_make_signs.argtypes = [ctypes.c_uint64, ctypes.c_int, _P]
        L.ko_fwht.argtypes = [_P, ctypes.c_int]
        L.ko_pairwise_sum.restype = ctypes.c_float
        L.ko_pairwise_sum.argtypes = [_P, ctypes.c_long, ctypes.c_long]
        L.ko_qmax.argtypes = [ctypes.c_int]
        L.ko_row_bytes.argtypes = [ctypes.c_int, ctypes.c_int]
        L.ko_ntok.argtypes = [ctypes.c_uint]
        L.ko_pack_row.argtypes = [_P, ctypes.c_int, ctypes.c_int, _P]
        L.ko_unpack_row.argtypes = [_P, ctypes.c_int, ctypes.c_int, _P]
        L.ko_quantize_block.argtypes = [_P, _P, _P, _P, _P, _P]
        L.ko_dequantize_block.argtypes = [_P, _P, _P, _P, _P, _P]
        L.ko_quantize_slice.argtypes = [_P, _P, ctypes.c_long, ctypes.c_long, _P, _P, _P, _P]
        L.ko_quantize_slice_y.argtypes = [_P, _P, ctypes.c_long, ctypes.c_long, _P, _P, _P, _P, _P]
        L.ko_dequantize_slice.argtypes = [_P, _P, _P, _P, _P, ctypes.c_long, ctypes.c_long, _P]
        L.ko_attention_f64.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_long, _P, _P, _P,
                                       ctypes.c_double, _P]
        L.ko_dq_record_bytes.argtypes = [ctypes.c_int]
        L.ko_off_words.argtypes = [ctypes.c_uint, ctypes.c_int]
        L.ko_dq_decode.argtypes = [_P, ctypes.c_int, _P, _P]
        L.ko_select_signs.restype = ctypes.c_int
        L.ko_select_signs.argtypes = [_P, _P, ctypes.c_long, _P, ctypes.c_int, _P]
        _lib = L
    return _lib


class _KoCfg(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int), ("bits", ctypes.c_int), ("flags", ctypes.c_uint),
                ("signs", ctypes.c_void_p)]


@dataclass
class Cfg:
    """Quantizer configuration: head dim, bit width, flag set, optional signs."""
    d: int
    bits: int
    flags: int
    signs: Optional[np.ndarray] = None   # int8 [d] of +-1, None = plain Hadamard

    def c(self):
        if self.signs is not None:
            self._signs_keep = np.ascontiguousarray(self.signs, dtype=np.int8)
            sp = self._signs_keep.ctypes.data
        else:
            sp = None
        s = _KoCfg(self.d, self.bits, self.flags, sp)
        return s


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _pool(threads: int):
    return ThreadPoolExecutor(max_workers=max(1, threads))


# ---------------------------------------------------------------- scalars

def f32_to_f16_bits(x) -> np.ndarray:
    a = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.uint16)
    lib().ko_f32_to_f16_array(_ptr(a), a.size, _ptr(out))
    return out


def f16_bits_to_f32(h) -> np.ndarray:
    a = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(a.shape, dtype=np.float32)
    lib().ko_f16_to_f32_array(_ptr(a), a.size, _ptr(out))
    return out


def qmax(bits: int) -> int:
    return lib().ko_qmax(bits)


def row_bytes(d: int, bits: int) -> int:
    return lib().ko_row_bytes(d, bits)


def ntok(flags: int) -> int:
    return lib().ko_ntok(flags)


def off_words(flags: int, d: int) -> int:
    """fp16 words per block of the NSN offsets array: d means, or under DQ
    the block's side-parameter record (its bytes / 2)."""
    return lib().ko_off_words(flags, d)


def dq_record_bytes(d: int) -> int:
    return lib().ko_dq_record_bytes(d)


def dq_decode(rec: np.ndarray, d: int):
    """(o_hat float32 [d], s1_hat float32 [128]) of one DQ record."""
    rec = np.ascontiguousarray(rec).view(np.uint8)
    o = np.empty(d, np.float32)
    s1 = np.empty(T, np.float32)
    lib().ko_dq_decode(_ptr(rec), d, _ptr(o), _ptr(s1))
    return o, s1


def splitmix64(seed: int, n: int) -> list:
    st = ctypes.c_uint64(seed)
    return [lib().ko_splitmix64_next(ctypes.byref(st)) for _ in range(n)]


def make_signs(seed: int, d: int) -> np.ndarray:
    out = np.empty(d, dtype=np.int8)
    lib().ko_make_signs(ctypes.c_uint64(seed), d, _ptr(out))
    return out


def fwht(v) -> np.ndarray:
    """Unnormalized Walsh-Hadamard butterflies over the last axis (fp32)."""
    a = np.array(v, dtype=np.float32, copy=True, order="C")
    d = a.shape[-1]
    flat = a.reshape(-1, d)
    for i in range(flat.shape[0]):
        lib().ko_fwht(ctypes.c_void_p(flat[i:].ctypes.data), d)
    return a


def pairwise_sum(v) -> np.float32:
    a = np.ascontiguousarray(v, dtype=np.float32)
    return np.float32(lib().ko_pairwise_sum(_ptr(a), a.size, 1))


def pack_rows(q: np.ndarray, bits: int) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.int8)
    n, d = q.shape
    out = np.empty((n, row_bytes(d, bits)), dtype=np.uint8)
    for i in range(n):
        lib().ko_pack_row(ctypes.c_void_p(q[i].ctypes.data), d, bits,
                          ctypes.c_void_p(out[i].ctypes.data))
    return out


def unpack_rows(codes: np.ndarray, d: int, bits: int):
    """Returns (q int8 [n, d], number of illegal zero codes)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    n = codes.shape[0]
    q = np.empty((n, d), dtype=np.int8)
    bad = 0
    for i in range(n):
        bad += lib().ko_unpack_row(ctypes.c_void_p(codes[i].ctypes.data), d, bits,
                                   ctypes.c_void_p(q[i].ctypes.data))
    return q, bad


# ---------------------------------------------------------------- cache level

def empty_cache(cfg: Cfg, B: int, H: int, S_max: int) -> dict:
    assert S_max % T == 0
    nt = ntok(cfg.flags)
    nb = S_max // T
    return {
        "codes": np.zeros((B, H, S_max, row_bytes(cfg.d, cfg.bits)), np.uint8),
        "tok": np.zeros((B, H, S_max, nt), np.uint16) if nt else None,
        "chan": np.zeros((B, H, nb, cfg.d), np.uint16) if cfg.flags & PER_CHANNEL else None,
        "off": np.zeros((B, H, nb, off_words(cfg.flags, cfg.d)), np.uint16) if cfg.flags & NSN else None,
    }


def quantize_into(cfg: Cfg, x16: np.ndarray, cache: dict, t0: int = 0, threads: int = 1):
    """Quantize x16 [B, H, n, d] (fp16 bits, n % 128 == 0) into cache blocks
    starting at token t0 (t0 % 128 == 0)."""
    x16 = np.ascontiguousarray(x16, dtype=np.uint16)
    B, H, n, d = x16.shape
    assert d == cfg.d and n % T == 0 and t0 % T == 0
    c = cfg.c()
    L = lib()

    def one(bh):
        b, h = bh
        L.ko_quantize_slice(ctypes.byref(c), _ptr(x16[b, h]), t0, n,
                            _ptr(cache["codes"][b, h]),
                            None if cache["tok"] is None else _ptr(cache["tok"][b, h]),
                            None if cache["chan"] is None else _ptr(cache["chan"][b, h]),
                            None if cache["off"] is None else _ptr(cache["off"][b, h]))

    with _pool(threads) as ex:
        list(ex.map(one, [(b, h) for b in range(B) for h in range(H)]))
    return cache


def quantize_products(cfg: Cfg, x16: np.ndarray, cache: dict, t0: int = 0, threads: int = 1) -> np.ndarray:
    """Quantize like quantize_into and return the exact pre-rounding
    product u * (1/sigma16) of every code, float64 [B, H, n, d]: each code is
    clamp(round-half-even(y)).  Used to tell a rounding half-point from a
    real disagreement."""
    x16 = np.ascontiguousarray(x16, dtype=np.uint16)
    B, H, n, d = x16.shape
    assert d == cfg.d and n % T == 0 and t0 % T == 0
    y = np.empty((B, H, n, d), np.float64)
    c = cfg.c()
    L = lib()

    def one(bh):
        b, h = bh
        L.ko_quantize_slice_y(ctypes.byref(c), _ptr(x16[b, h]), t0, n,
                              _ptr(cache["codes"][b, h]),
                              None if cache["tok"] is None else _ptr(cache["tok"][b, h]),
                              None if cache["chan"] is None else _ptr(cache["chan"][b, h]),
                              None if cache["off"] is None else _ptr(cache["off"][b, h]),
                              _ptr(y[b, h]))

    with _pool(threads) as ex:
        list(ex.map(one, [(b, h) for b in range(B) for h in range(H)]))
    return y


def half_point_distance(y: np.ndarray) -> np.ndarray:
    """Distance of |y| from the nearest rounding half-point k + 1/2."""
    a = np.abs(np.asarray(y, np.float64))
    return np.abs(a - np.floor(a) - 0.5)


def quantize(cfg: Cfg, x16: np.ndarray, S_max: Optional[int] = None, threads: int = 1) -> dict:
    B, H, n, _ = x16.shape
    cache = empty_cache(cfg, B, H, S_max or n)
    return quantize_into(cfg, x16, cache, 0, threads)


def dequantize(cfg: Cfg, cache: dict, t0: int, n: int, threads: int = 1):
    """fp32 [B, H, n, d] rebuilt from blocks [t0, t0+n); also returns the
    count of illegal zero codes met."""
    B, H = cache["codes"].shape[:2]
    out = np.empty((B, H, n, cfg.d), np.float32)
    c = cfg.c()
    L = lib()
    bad = [0] * (B * H)

    def one(i):
        b, h = divmod(i, H)
        bad[i] = L.ko_dequantize_slice(
            ctypes.byref(c), _ptr(cache["codes"][b, h]),
            None if cache["tok"] is None else _ptr(cache["tok"][b, h]),
            None if cache["chan"] is None else _ptr(cache["chan"][b, h]),
            None if cache["off"] is None else _ptr(cache["off"][b, h]),
            t0, n, _ptr(out[b, h]))

    with _pool(threads) as ex:
        list(ex.map(one, range(B * H)))
    return out, sum(bad)


def attention(q16: np.ndarray, k: np.ndarray, v: np.ndarray, scale: Optional[float] = None,
              threads: int = 1) -> np.ndarray:
    """fp64 softmax attention.  q16 [B, Hq, d] fp16 bits; k, v [B, Hkv, L, d]
    fp32.  Query head j reads kv head j // (Hq // Hkv)."""
    q16 = np.ascontiguousarray(q16, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.float32)
    v = np.ascontiguousarray(v, dtype=np.float32)
    B, Hq, d = q16.shape
    Hkv, Ln = k.shape[1], k.shape[2]
    g = Hq // Hkv
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(d)
    out = np.empty((B, Hq, d), np.float64)
    L = lib()

    def one(i):
        b, h = divmod(i, Hkv)
        L.ko_attention_f64(g, d, Ln, _ptr(q16[b, h * g:(h + 1) * g]), _ptr(k[b, h]), _ptr(v[b, h]),
                           float(scale), _ptr(out[b, h * g:(h + 1) * g]))

    with _pool(threads) as ex:
        list(ex.map(one, range(B * Hkv)))
    return out


def cache_tokens(cfg: Cfg, cache: dict, resid16: np.ndarray, length: int, threads: int = 1):
    """fp32 [B, H, length, d]: dequantized full blocks followed by the
    residual tokens taken as their fp16 values."""
    nq = (length // T) * T
    parts = []
    if nq:
        deq, bad = dequantize(cfg, cache, 0, nq, threads)
        assert bad == 0, "illegal zero code in cache"
        parts.append(deq)
    r = length - nq
    if r:
        parts.append(f16_bits_to_f32(resid16[:, :, :r, :]))
    if not parts:
        B, H = cache["codes"].shape[:2]
        return np.zeros((B, H, 0, cfg.d), np.float32)
    return np.concatenate(parts, axis=2)


def cache_attention(cfg: Cfg, q16, cache_k, cache_v, resid_k16, resid_v16, length: int,
                    scale: Optional[float] = None, threads: int = 1) -> np.ndarray:
    k = cache_tokens(cfg, cache_k, resid_k16, length, threads)
    v = cache_tokens(cfg, cache_v, resid_v16, length, threads)
    return attention(q16, k, v, scale, threads)


def select_signs(cfg: Cfg, x16: np.ndarray, signs: np.ndarray):
    """Sign-pattern selection for the randomized Hadamard rotation: x16 the
    sample as whole blocks (fp16 bits [n_blocks, 128, d]), signs [n_cand, d]
    of +-1.  Returns (index of the smallest reconstruction error, errors
    float64 [n_cand]); cfg.signs is ignored."""
    x16 = np.ascontiguousarray(x16, dtype=np.uint16)
    signs = np.ascontiguousarray(signs, dtype=np.int8)
    nb, t, d = x16.shape
    assert t == T and d == cfg.d and signs.shape[1] == d
    err = np.empty(signs.shape[0], np.float64)
    c = Cfg(cfg.d, cfg.bits, cfg.flags, None).c()
    best = lib().ko_select_signs(ctypes.byref(c), _ptr(x16), nb, _ptr(signs), signs.shape[0], _ptr(err))
    return int(best), err


def default_threads() -> int:
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
