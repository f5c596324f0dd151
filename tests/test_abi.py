"""The C-ABI library loads, exports every symbol include/kvq.h declares, and
rejects bad arguments on the host before anything reaches a GPU (CPU only).

Calls made here with placeholder device addresses always carry an argument
that the host-side checks reject, so nothing is ever launched with them.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvq.h")


@pytest.fixture(scope="module")
def kvq():
    from kv_cache_bit_b200 import build
    build.build()
    from kv_cache_bit_b200 import kvq as mod
    return mod


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("kvq_quantize_block", "kvq_append_token", "kvq_decode_attention", "kvq_dequantize",
              "kvq_decode_workspace_bytes", "kvq_make_signs", "kvq_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(kvq):
    lib = ctypes.CDLL(kvq.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), n
    assert sorted(kvq.EXPORTS) == declared_functions()


def test_make_signs_matches_splitmix_known_answers(kvq):
    gold = [int(l, 16) for l in open(os.path.join(ROOT, "tests", "golden", "splitmix64_seed0.txt"))
            if l.strip() and not l.startswith("#")]
    s = kvq.kvq_make_signs(0, len(gold))
    assert [int(v < 0) for v in s] == [(g >> 63) & 1 for g in gold]
    for seed in (0, 1, 0x5EED, 2 ** 63 + 5):
        assert np.array_equal(kvq.kvq_make_signs(seed, 128), oracle.make_signs(seed, 128))
    assert kvq.lib.kvq_make_signs(0, 16, None) == kvq.KVQ_ERR_INVALID_ARG


def test_sizes(kvq):
    assert kvq.kvq_row_bytes(128, 4) == 64 and kvq.kvq_row_bytes(128, 3) == 48
    assert kvq.kvq_row_bytes(128, 2) == 32 and kvq.kvq_row_bytes(64, 4) == 32
    assert kvq.kvq_row_bytes(96, 4) == 0 and kvq.kvq_row_bytes(128, 5) == 0
    for d in (64, 128):
        for b in (2, 3, 4):
            assert kvq.kvq_row_bytes(d, b) == oracle.row_bytes(d, b)
    assert kvq.kvq_tok_params(kvq.NORM_SEP | kvq.PER_CHANNEL) == 1
    assert kvq.kvq_tok_params(0) == 1
    assert kvq.kvq_tok_params(kvq.NSN | kvq.PER_CHANNEL | kvq.HADAMARD) == 2
    assert kvq.kvq_tok_params(kvq.NORM_SEP) == -1          # nsep-only: oracle only
    assert kvq.kvq_tok_params(kvq.HADAMARD) == -1          # rotated naive: oracle only


def _fake_cache(kvq, B=2, H=2, d=128, cap=256, length=0, naive=False, nsn=False):
    a = 1 << 20  # placeholder, 16-byte aligned, never dereferenced
    P2 = ctypes.c_void_p * 2
    return kvq.kvq_cache(B, H, d, cap, length, P2(a, a), P2(a, a),
                         P2(None, None) if naive else P2(a, a),
                         P2(a, a) if nsn else P2(None, None), P2(a, a))


def _cfg(kvq, d=128, bits=4, flags=3, reserved=0):
    return kvq.kvq_config(d, bits, flags, reserved, None)


def test_host_side_rejections(kvq):
    L = kvq.lib
    cfg, cache = _cfg(kvq), _fake_cache(kvq)
    A = 1 << 20
    by = ctypes.byref
    INV, UNS, CAP, WS = kvq.KVQ_ERR_INVALID_ARG, kvq.KVQ_ERR_UNSUPPORTED, kvq.KVQ_ERR_CAPACITY, kvq.KVQ_ERR_WORKSPACE
    # quantize: offsets and sizes
    assert L.kvq_quantize_block(by(cfg), by(cache), A, A, 1, 128, None) == INV
    assert L.kvq_quantize_block(by(cfg), by(cache), A, A, 0, 100, None) == INV
    assert L.kvq_quantize_block(by(cfg), by(cache), A, A, 0, 0, None) == INV
    assert L.kvq_quantize_block(by(cfg), by(cache), A, A, 128, 256, None) == CAP
    assert L.kvq_quantize_block(by(cfg), by(cache), None, A, 0, 128, None) == INV
    assert L.kvq_quantize_block(by(cfg), by(cache), A + 4, A, 0, 128, None) == INV
    assert L.kvq_quantize_block(None, by(cache), A, A, 0, 128, None) == INV
    # unsupported configurations
    for bad in (_cfg(kvq, d=96), _cfg(kvq, bits=5), _cfg(kvq, flags=1), _cfg(kvq, flags=8)):
        assert L.kvq_quantize_block(by(bad), by(cache), A, A, 0, 128, None) == UNS
    assert L.kvq_quantize_block(by(_cfg(kvq, reserved=1)), by(cache), A, A, 0, 128, None) == INV
    # cache shape checks
    for c in (_fake_cache(kvq, cap=200), _fake_cache(kvq, d=64), _fake_cache(kvq, B=0),
              _fake_cache(kvq, length=300)):
        assert L.kvq_quantize_block(by(cfg), by(c), A, A, 0, 128, None) == INV
    nochan = _fake_cache(kvq, naive=True)
    assert L.kvq_quantize_block(by(cfg), by(nochan), A, A, 0, 128, None) == INV
    nsn_cfg = _cfg(kvq, flags=kvq.NSN | kvq.PER_CHANNEL)
    assert L.kvq_quantize_block(by(nsn_cfg), by(cache), A, A, 0, 128, None) == INV   # off[] missing
    # residual tokens still held cannot be overwritten by a bulk quantize
    held = _fake_cache(kvq, length=130)
    assert L.kvq_quantize_block(by(cfg), by(held), A, A, 128, 128, None) == INV
    # append past capacity
    full = _fake_cache(kvq, length=256)
    assert L.kvq_append_token(by(cfg), by(full), A, A, None) == CAP
    assert L.kvq_append_token(by(cfg), by(cache), None, A, None) == INV
    # decode: heads and workspace
    need = L.kvq_decode_workspace_bytes(by(cfg), by(cache), 8)
    assert need > 0
    assert L.kvq_decode_workspace_bytes(by(cfg), by(cache), 3) == 0      # not a multiple of kv heads
    assert L.kvq_decode_workspace_bytes(by(cfg), by(cache), 2 * 9) == 0  # more than 8 q heads per kv head
    assert L.kvq_decode_attention(by(cfg), by(cache), A, 8, 0.0, A, A, need - 1, None) == WS
    assert L.kvq_decode_attention(by(cfg), by(cache), A, 8, 0.0, A, None, need, None) == WS
    assert L.kvq_decode_attention(by(cfg), by(cache), A, 3, 0.0, A, A, need, None) == INV
    assert L.kvq_decode_attention(by(cfg), by(cache), A, 18, 0.0, A, A, 1 << 30, None) == UNS
    # device pointers must be 16-byte aligned: query, output, workspace
    assert L.kvq_decode_attention(by(cfg), by(cache), A + 8, 8, 0.0, A, A, need, None) == INV
    assert L.kvq_decode_attention(by(cfg), by(cache), A, 8, 0.0, A + 4, A, need, None) == INV
    assert L.kvq_decode_attention(by(cfg), by(cache), A, 8, 0.0, A, A + 4, need, None) == WS
    # dequantize ranges
    c300 = _fake_cache(kvq, length=200)
    assert L.kvq_dequantize(by(cfg), by(c300), 2, 0, 128, A, None) == INV
    assert L.kvq_dequantize(by(cfg), by(c300), 0, 0, 256, A, None) == INV
    assert L.kvq_dequantize(by(cfg), by(c300), 0, 64, 128, A, None) == INV
    # failed checks leave len untouched
    assert held.len == 130 and full.len == 256
    assert kvq.lib.kvq_status_string(kvq.KVQ_ERR_CAPACITY) == b"cache capacity exceeded"


def test_select_signs_host_checks(kvq):
    a = 1 << 20  # placeholder, 16-byte aligned, never dereferenced: every call below fails a host check
    L = kvq.lib
    assert L.kvq_select_signs_workspace_bytes(8, 10) == 8 * 10 * 8
    assert L.kvq_select_signs_workspace_bytes(0, 10) == 0
    assert L.kvq_select_signs_workspace_bytes(kvq.SELECT_MAX_CANDIDATES + 1, 10) == 0
    had = _cfg(kvq, flags=kvq.NORM_SEP | kvq.PER_CHANNEL | kvq.HADAMARD)
    nsn = _cfg(kvq, flags=kvq.NSN | kvq.PER_CHANNEL | kvq.HADAMARD)
    plain = _cfg(kvq, flags=kvq.NORM_SEP | kvq.PER_CHANNEL)
    args = lambda cfg, x=a, nb=4, s=a, nc=2, ws=a, wsb=64: L.kvq_select_signs(
        ctypes.byref(cfg), x, nb, s, nc, a, a, ws, wsb, None)
    assert args(plain) == kvq.KVQ_ERR_UNSUPPORTED
    assert args(_cfg(kvq, flags=0)) == kvq.KVQ_ERR_UNSUPPORTED
    assert args(had, x=None) == kvq.KVQ_ERR_INVALID_ARG
    assert args(had, x=a + 4) == kvq.KVQ_ERR_INVALID_ARG
    assert args(nsn, s=None) == kvq.KVQ_ERR_INVALID_ARG
    assert args(had, nc=0) == kvq.KVQ_ERR_INVALID_ARG
    assert args(had, nb=0) == kvq.KVQ_ERR_INVALID_ARG
    assert args(had, ws=None) == kvq.KVQ_ERR_WORKSPACE
    assert args(had, wsb=63) == kvq.KVQ_ERR_WORKSPACE


def test_dq_flag_sizes(kvq):
    nsn_dq = kvq.NSN | kvq.PER_CHANNEL | kvq.DQ
    assert kvq.kvq_tok_params(nsn_dq) == 1 and kvq.kvq_tok_params(nsn_dq | kvq.HADAMARD) == 1
    assert kvq.kvq_tok_params(kvq.NORM_SEP | kvq.PER_CHANNEL | kvq.DQ) == -1    # DQ only with NSN
    for d in (64, 128):
        assert kvq.kvq_off_words(nsn_dq, d) == oracle.off_words(oracle.NSN | oracle.PER_CHANNEL | oracle.DQ, d)
        assert kvq.kvq_off_words(nsn_dq, d) * 2 == oracle.dq_record_bytes(d)
        assert kvq.kvq_off_words(kvq.NSN | kvq.PER_CHANNEL, d) == d
        assert kvq.kvq_off_words(kvq.NORM_SEP | kvq.PER_CHANNEL, d) == 0
    assert kvq.kvq_off_words(nsn_dq, 96) == -1
    assert oracle.ntok(oracle.NSN | oracle.PER_CHANNEL | oracle.DQ) == 1


def test_cache_snapshot_and_restore_on_host_tensors(kvq):
    """Checkpoint / resume of the binding's cache object: a snapshot holds
    every buffer and the token count; restore refuses another shape."""
    import torch
    cfg = kvq.Config(128, 4, kvq.NSN | kvq.PER_CHANNEL | kvq.HADAMARD, None, device="cpu")
    c = kvq.KVCache.allocate(cfg, 2, 2, 256, device="cpu")
    g = torch.Generator().manual_seed(0)
    for grp in (c.codes, c.tok, c.chan, c.off, c.resid):
        for t in grp:
            t.copy_(torch.randint(-100, 100, t.shape, generator=g).to(t.dtype))
    c.c.len = 200
    snap = c.snapshot()
    d = kvq.KVCache.allocate(cfg, 2, 2, 256, device="cpu")
    d.restore(snap)
    assert d.len == 200
    for name in ("codes", "tok", "chan", "off", "resid"):
        for a, b in zip(getattr(c, name), getattr(d, name)):
            assert torch.equal(a, b), name
    small = kvq.KVCache.allocate(cfg, 2, 2, 128, device="cpu")
    with pytest.raises(kvq.KvqError):
        small.restore(snap)
