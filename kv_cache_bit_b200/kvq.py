"""Thin ctypes binding of libkvq (include/kvq.h): the same call names, with
argument marshalling only.  Every step of the quantizer and of decode
attention runs in the library's CUDA kernels; PyTorch is used here only to
hold device memory and to name the current CUDA stream.

Loading fails loudly (ImportError) when libkvq.so has not been built: there
is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "_lib", "libkvq.so")

KVQ_OK, KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED, KVQ_ERR_CAPACITY, KVQ_ERR_WORKSPACE, KVQ_ERR_CUDA = range(6)
KVQ_NORM_SEP, KVQ_PER_CHANNEL, KVQ_NSN, KVQ_HADAMARD, KVQ_DQ = 1, 2, 4, 8, 16
NORM_SEP, PER_CHANNEL, NSN, HADAMARD, DQ = KVQ_NORM_SEP, KVQ_PER_CHANNEL, KVQ_NSN, KVQ_HADAMARD, KVQ_DQ
BLOCK_TOKENS = 128

EXPORTS = ["kvq_row_bytes", "kvq_tok_params", "kvq_off_words", "kvq_make_signs", "kvq_quantize_block", "kvq_append_token",
           "kvq_decode_workspace_bytes", "kvq_decode_attention", "kvq_decode_attention_noalloc", "kvq_dequantize",
           "kvq_select_signs_workspace_bytes", "kvq_select_signs", "kvq_read_device_errors",
           "kvq_status_string"]


class kvq_config(ctypes.Structure):
    _fields_ = [("head_dim", ctypes.c_int32), ("bits", ctypes.c_int32), ("flags", ctypes.c_uint32),
                ("reserved", ctypes.c_int32), ("signs", ctypes.c_void_p)]


class kvq_cache(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("capacity", ctypes.c_int32), ("len", ctypes.c_int64),
                ("codes", ctypes.c_void_p * 2), ("tok", ctypes.c_void_p * 2), ("chan", ctypes.c_void_p * 2),
                ("off", ctypes.c_void_p * 2), ("resid", ctypes.c_void_p * 2)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libkvq.so not built ({LIB_PATH}); run kv_cache_bit_b200/build.py")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    L.kvq_row_bytes.restype = ctypes.c_int32
    L.kvq_row_bytes.argtypes = [ctypes.c_int32, ctypes.c_int32]
    L.kvq_tok_params.restype = ctypes.c_int32
    L.kvq_tok_params.argtypes = [ctypes.c_uint32]
    L.kvq_off_words.restype = ctypes.c_int32
    L.kvq_off_words.argtypes = [ctypes.c_uint32, ctypes.c_int32]
    L.kvq_make_signs.restype = ctypes.c_int
    L.kvq_make_signs.argtypes = [ctypes.c_uint64, ctypes.c_int32, P]
    L.kvq_quantize_block.restype = ctypes.c_int
    L.kvq_quantize_block.argtypes = [ctypes.POINTER(kvq_config), ctypes.POINTER(kvq_cache), P, P,
                                     ctypes.c_int64, ctypes.c_int64, P]
    L.kvq_append_token.restype = ctypes.c_int
    L.kvq_append_token.argtypes = [ctypes.POINTER(kvq_config), ctypes.POINTER(kvq_cache), P, P, P]
    L.kvq_decode_workspace_bytes.restype = ctypes.c_size_t
    L.kvq_decode_workspace_bytes.argtypes = [ctypes.POINTER(kvq_config), ctypes.POINTER(kvq_cache), ctypes.c_int32]
    L.kvq_decode_attention.restype = ctypes.c_int
    L.kvq_decode_attention.argtypes = [ctypes.POINTER(kvq_config), ctypes.POINTER(kvq_cache), P, ctypes.c_int32,
                                       ctypes.c_float, P, P, ctypes.c_size_t, P]
    L.kvq_decode_attention_noalloc.restype = ctypes.c_int
    L.kvq_decode_attention_noalloc.argtypes = [ctypes.POINTER(kvq_config), ctypes.POINTER(kvq_cache), P,
                                               ctypes.c_int32, ctypes.c_float, P, P]
    L.kvq_dequantize.restype = ctypes.c_int
    L.kvq_dequantize.argtypes = [ctypes.POINTER(kvq_config), ctypes.POINTER(kvq_cache), ctypes.c_int32,
                                 ctypes.c_int64, ctypes.c_int64, P, P]
    L.kvq_select_signs_workspace_bytes.restype = ctypes.c_size_t
    L.kvq_select_signs_workspace_bytes.argtypes = [ctypes.c_int32, ctypes.c_int64]
    L.kvq_select_signs.restype = ctypes.c_int
    L.kvq_select_signs.argtypes = [ctypes.POINTER(kvq_config), P, ctypes.c_int64, P, ctypes.c_int32, P, P, P,
                                   ctypes.c_size_t, P]
    L.kvq_read_device_errors.restype = ctypes.c_int
    L.kvq_read_device_errors.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int32]
    L.kvq_status_string.restype = ctypes.c_char_p
    L.kvq_status_string.argtypes = [ctypes.c_int]
    return L


lib = _load()


class KvqError(RuntimeError):
    def __init__(self, status: int, call: str):
        super().__init__(f"{call}: {lib.kvq_status_string(status).decode()} (status {status})")
        self.status = status


def _check(status: int, call: str):
    if status != KVQ_OK:
        raise KvqError(status, call)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


# ------------------------------------------------------------------ calls

def kvq_row_bytes(head_dim: int, bits: int) -> int:
    return lib.kvq_row_bytes(head_dim, bits)


def kvq_tok_params(flags: int) -> int:
    return lib.kvq_tok_params(flags)


def kvq_off_words(flags: int, head_dim: int) -> int:
    return lib.kvq_off_words(flags, head_dim)


def kvq_make_signs(seed: int, head_dim: int):
    """Host +-1 signs (numpy int8) from SplitMix64."""
    import numpy as np
    out = np.empty(head_dim, np.int8)
    _check(lib.kvq_make_signs(ctypes.c_uint64(seed), head_dim, out.ctypes.data), "kvq_make_signs")
    return out


def kvq_quantize_block(cfg: "Config", cache: "KVCache", k, v, t0: int, ntok: int, stream=None):
    _check(lib.kvq_quantize_block(ctypes.byref(cfg.c), ctypes.byref(cache.c), _ptr(k), _ptr(v), t0, ntok,
                                  _stream(stream)), "kvq_quantize_block")


def kvq_append_token(cfg: "Config", cache: "KVCache", k_new, v_new, stream=None):
    _check(lib.kvq_append_token(ctypes.byref(cfg.c), ctypes.byref(cache.c), _ptr(k_new), _ptr(v_new),
                                _stream(stream)), "kvq_append_token")


def kvq_decode_workspace_bytes(cfg: "Config", cache: "KVCache", q_heads: int) -> int:
    return lib.kvq_decode_workspace_bytes(ctypes.byref(cfg.c), ctypes.byref(cache.c), q_heads)


def kvq_decode_attention(cfg: "Config", cache: "KVCache", q, q_heads: int, scale: float, out, ws, ws_bytes: int,
                         stream=None):
    _check(lib.kvq_decode_attention(ctypes.byref(cfg.c), ctypes.byref(cache.c), _ptr(q), q_heads, scale,
                                    _ptr(out), _ptr(ws), ws_bytes, _stream(stream)), "kvq_decode_attention")


def kvq_decode_attention_noalloc(cfg: "Config", cache: "KVCache", q, q_heads: int, scale: float, out,
                                 stream=None):
    """Decode attention with the library's own fixed device scratch (no
    workspace argument, no allocation); see include/kvq.h."""
    _check(lib.kvq_decode_attention_noalloc(ctypes.byref(cfg.c), ctypes.byref(cache.c), _ptr(q), q_heads, scale,
                                            _ptr(out), _stream(stream)), "kvq_decode_attention_noalloc")


NOALLOC_SCRATCH_BYTES = 32 << 20


def kvq_dequantize(cfg: "Config", cache: "KVCache", tensor: int, t0: int, ntok: int, out, stream=None):
    _check(lib.kvq_dequantize(ctypes.byref(cfg.c), ctypes.byref(cache.c), tensor, t0, ntok, _ptr(out),
                              _stream(stream)), "kvq_dequantize")


SELECT_MAX_CANDIDATES = 256


def kvq_select_signs_workspace_bytes(n_cand: int, n_blocks: int) -> int:
    return lib.kvq_select_signs_workspace_bytes(n_cand, n_blocks)


def kvq_select_signs(cfg: "Config", x, n_blocks: int, signs, n_cand: int, err, best, ws, ws_bytes: int,
                     stream=None):
    """Sign-pattern selection (see include/kvq.h): x fp16 [n_blocks, 128,
    head_dim], signs int8 [n_cand, head_dim], err float64 [n_cand] and best
    int32 [1] outputs, all device tensors."""
    _check(lib.kvq_select_signs(ctypes.byref(cfg.c), _ptr(x), n_blocks, _ptr(signs), n_cand, _ptr(err), _ptr(best),
                                _ptr(ws), ws_bytes, _stream(stream)), "kvq_select_signs")


def kvq_read_device_errors(clear: bool = True) -> int:
    v = ctypes.c_uint32(0)
    _check(lib.kvq_read_device_errors(ctypes.byref(v), 1 if clear else 0), "kvq_read_device_errors")
    return v.value


# ------------------------------------------------------------------ plumbing

class Config:
    """kvq_config plus the device copy of the rotation signs it points to."""

    def __init__(self, head_dim: int, bits: int, flags: int, signs=None, device="cuda"):
        import torch
        self.head_dim, self.bits, self.flags = head_dim, bits, flags
        self.signs_dev = None
        if signs is not None:
            self.signs_dev = torch.as_tensor(signs, dtype=torch.int8).to(device).contiguous()
        self.c = kvq_config(head_dim, bits, flags, 0, _ptr(self.signs_dev))


@dataclass
class KVCache:
    """Caller-side allocation of a kvq_cache (torch tensors on the GPU)."""
    c: kvq_cache
    codes: list
    tok: list
    chan: list
    off: list
    resid: list

    @classmethod
    def allocate(cls, cfg: Config, batch: int, kv_heads: int, capacity: int, device="cuda") -> "KVCache":
        import torch
        assert capacity % BLOCK_TOKENS == 0
        rb = kvq_row_bytes(cfg.head_dim, cfg.bits)
        nt = kvq_tok_params(cfg.flags)
        if rb <= 0 or nt <= 0:
            raise KvqError(KVQ_ERR_UNSUPPORTED, "KVCache.allocate")
        nb = capacity // BLOCK_TOKENS
        d = cfg.head_dim
        mk = lambda shape, dt: torch.zeros(shape, dtype=dt, device=device)
        codes = [mk((batch, kv_heads, capacity, rb), torch.uint8) for _ in range(2)]
        tok = [mk((batch, kv_heads, capacity, nt), torch.int16) for _ in range(2)]
        pchan = bool(cfg.flags & PER_CHANNEL)
        chan = [mk((batch, kv_heads, nb, d), torch.int16) if pchan else None for _ in range(2)]
        ow = kvq_off_words(cfg.flags, d)
        off = [mk((batch, kv_heads, nb, ow), torch.int16) if cfg.flags & NSN else None for _ in range(2)]
        resid = [mk((batch, kv_heads, BLOCK_TOKENS, d), torch.int16) for _ in range(2)]
        c = kvq_cache(batch, kv_heads, d, capacity, 0,
                      (ctypes.c_void_p * 2)(*[_ptr(x) for x in codes]),
                      (ctypes.c_void_p * 2)(*[_ptr(x) for x in tok]),
                      (ctypes.c_void_p * 2)(*[_ptr(x) for x in chan]),
                      (ctypes.c_void_p * 2)(*[_ptr(x) for x in off]),
                      (ctypes.c_void_p * 2)(*[_ptr(x) for x in resid]))
        return cls(c, codes, tok, chan, off, resid)

    def rows(self, b0: int, b1: int) -> "KVCache":
        """A view of batch rows [b0, b1) sharing this cache's memory (its own
        kvq_cache struct, len copied)."""
        sl = lambda ts: [t[b0:b1] if t is not None else None for t in ts]
        codes, tok, chan, off, resid = sl(self.codes), sl(self.tok), sl(self.chan), sl(self.off), sl(self.resid)
        c = kvq_cache(b1 - b0, self.c.kv_heads, self.c.head_dim, self.c.capacity, self.c.len,
                      (ctypes.c_void_p * 2)(*[_ptr(x) for x in codes]),
                      (ctypes.c_void_p * 2)(*[_ptr(x) for x in tok]),
                      (ctypes.c_void_p * 2)(*[_ptr(x) for x in chan]),
                      (ctypes.c_void_p * 2)(*[_ptr(x) for x in off]),
                      (ctypes.c_void_p * 2)(*[_ptr(x) for x in resid]))
        return KVCache(c, codes, tok, chan, off, resid)

    @property
    def len(self) -> int:
        return self.c.len

    def snapshot(self) -> dict:
        """A host copy of the cache (checkpoint): every buffer and the
        token count.  The cache is plain caller-owned memory, so this is the
        whole state."""
        cp = lambda ts: [t.cpu() if t is not None else None for t in ts]
        return {"len": self.c.len, "codes": cp(self.codes), "tok": cp(self.tok), "chan": cp(self.chan),
                "off": cp(self.off), "resid": cp(self.resid)}

    def restore(self, snap: dict) -> None:
        """Load a snapshot taken from a cache of the same configuration and
        shape (resume)."""
        for name in ("codes", "tok", "chan", "off", "resid"):
            for dst, src in zip(getattr(self, name), snap[name]):
                if (dst is None) != (src is None) or (dst is not None and dst.shape != src.shape):
                    raise KvqError(KVQ_ERR_INVALID_ARG, "KVCache.restore: snapshot of another cache shape")
                if dst is not None:
                    dst.copy_(src)
        self.c.len = snap["len"]

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for group in (self.codes, self.tok, self.chan, self.off, self.resid)
                   for t in group if t is not None)
