"""Helpers shared by the GPU parity tests: run the same seeded inputs through
the CUDA library (via the ctypes binding) and through the CPU oracle, and
compare the results."""
from __future__ import annotations

import numpy as np

import oracle
from kv_cache_bit_b200 import synth
from tests.modes import f16bits, oracle_cfg
from tests.layout import pairv_applies, pairv_to_rows

T = 128


def gpu_cfg(mode: str, d: int, bits: int):
    from kv_cache_bit_b200 import kvq
    names, seeded = synth.MODES[mode]
    flags = 0
    for n in names:
        flags |= getattr(kvq, n)
    signs = kvq.kvq_make_signs(synth.SIGN_SEED, d) if seeded else None
    return kvq.Config(d, bits, flags, signs)


def to_dev(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host16(t) -> np.ndarray:
    """int16 device tensor holding fp16 bits -> uint16 numpy."""
    return t.cpu().numpy().view(np.uint16)


def gpu_prefill(mode, d, bits, K, V, cap=None, ntok=None):
    """Quantize K, V (float16 [B, H, S, d]) into a fresh GPU cache."""
    import torch
    from kv_cache_bit_b200 import kvq
    B, H, S, _ = K.shape
    ntok = S if ntok is None else ntok
    cfg = gpu_cfg(mode, d, bits)
    cache = kvq.KVCache.allocate(cfg, B, H, cap or S)
    if ntok:
        kd = to_dev(f16bits(K[:, :, :ntok]).view(np.int16))
        vd = to_dev(f16bits(V[:, :, :ntok]).view(np.int16))
        kvq.kvq_quantize_block(cfg, cache, kd, vd, 0, ntok)
    torch.cuda.synchronize()
    return cfg, cache


def oracle_prefill(mode, d, bits, K, V, cap=None, ntok=None, threads=8):
    """The oracle's caches of K and V.  Each cache dict also carries "y":
    the exact pre-rounding product of every code of the quantized tokens
    (float64 [B, H, ntok, d]), which tells a rounding half-point apart."""
    B, H, S, _ = K.shape
    ntok = S if ntok is None else ntok
    cfg = oracle_cfg(mode, d, bits)
    ck = oracle.empty_cache(cfg, B, H, cap or S)
    cv = oracle.empty_cache(cfg, B, H, cap or S)
    ck["y"] = cv["y"] = None
    if ntok:
        ck["y"] = oracle.quantize_products(cfg, f16bits(K[:, :, :ntok]), ck, 0, threads)
        cv["y"] = oracle.quantize_products(cfg, f16bits(V[:, :, :ntok]), cv, 0, threads)
    return cfg, ck, cv


def fp16_ulp_diff(a_bits: np.ndarray, b_bits: np.ndarray) -> int:
    """Largest distance in fp16 ulps between two arrays of fp16 bit patterns."""
    def key(x):
        x = x.astype(np.int32)
        return np.where(x & 0x8000, -(x & 0x7FFF), x)
    if a_bits.size == 0:
        return 0
    return int(np.max(np.abs(key(a_bits) - key(b_bits))))


# A code may differ from the oracle's only where the exact product it rounds
# lies within this distance of a rounding half-point.
HALF_POINT_TOL = 1e-6

# Half-point cases met by the GPU parity tests of this session, reported in
# the pytest terminal summary (tests/conftest.py).
HALF_POINT_LOG = []
# (test, max |GPU - oracle|) of every decode-attention comparison, for the
# run summary: the margin left under the tolerance
ATTN_ERR_LOG = []


def check_attention(name, got, ref, atol):
    """Max-abs difference of GPU attention outputs from the oracle's,
    recorded for the run summary and checked against atol."""
    import numpy as np
    err = float(np.max(np.abs(np.asarray(got, np.float64) - np.asarray(ref, np.float64)))) if np.size(got) else 0.0
    ATTN_ERR_LOG.append((name, err))
    assert err <= atol, (name, err)
    return err


def compare_cache(gcache, ck, cv, d, bits, nq, bh_slice=slice(None), t0=0):
    """Codes bit-exact except at rounding half-points, side parameters within
    1 fp16 ulp.  ck / cv are oracle caches whose "y" holds the exact products
    of the oracle's codes for tokens [t0, nq).  A code that differs from the
    oracle's must be a neighbour whose product lies within HALF_POINT_TOL of
    a half-point; such codes are counted ("half_points") and logged.
    Returns a dict of counts and largest parameter differences in ulps."""
    rb = oracle.row_bytes(d, bits)
    res = {"code_mismatch": 0, "half_points": 0, "tok_ulp": 0, "chan_ulp": 0, "off_ulp": 0, "codes": 0}
    nb = nq // T
    for i, oc in enumerate((ck, cv)):
        g_codes = gcache.codes[i][bh_slice][:, :, t0:nq].cpu().numpy()
        if i == 1 and pairv_applies(d):
            g_codes = pairv_to_rows(g_codes, bits)  # the library's V layout -> token-major rows
        o_codes = oc["codes"][:, :, t0:nq]
        if not np.array_equal(g_codes, o_codes):
            gq, _ = oracle.unpack_rows(g_codes.reshape(-1, rb), d, bits)
            oq, _ = oracle.unpack_rows(o_codes.reshape(-1, rb), d, bits)
            diff = gq.astype(int) - oq.astype(int)
            assert np.abs(diff).max() <= 1, "codes differ by more than one step"
            y = oc.get("y")
            assert y is not None, "codes differ and the oracle's products were not kept"
            y = y[:, :, t0:nq].reshape(diff.shape)
            bad = (diff != 0) & (oracle.half_point_distance(y) > HALF_POINT_TOL)
            assert not bad.any(), f"{int(bad.sum())} code(s) differ away from a rounding half-point"
            n = int(np.count_nonzero(diff))
            res["code_mismatch"] += n
            res["half_points"] += n
        res["codes"] += o_codes.size * 8 // bits
        res["tok_ulp"] = max(res["tok_ulp"], fp16_ulp_diff(host16(gcache.tok[i][bh_slice][:, :, t0:nq]),
                                                           oc["tok"][:, :, t0:nq]))
        b0 = t0 // T
        if oc["chan"] is not None:
            res["chan_ulp"] = max(res["chan_ulp"], fp16_ulp_diff(host16(gcache.chan[i][bh_slice][:, :, b0:nb]),
                                                                 oc["chan"][:, :, b0:nb]))
        if oc["off"] is not None:
            g_off = host16(gcache.off[i][bh_slice][:, :, b0:nb])
            if oc["off"].shape[-1] == d:
                res["off_ulp"] = max(res["off_ulp"], fp16_ulp_diff(g_off, oc["off"][:, :, b0:nb]))
            else:
                # DQ block records (4-bit codes of o and s1, fp16 parameters):
                # byte for byte
                assert np.array_equal(g_off, oc["off"][:, :, b0:nb]), "DQ block records differ"
    HALF_POINT_LOG.append((res["half_points"], res["codes"]))
    return res


def assert_cache_parity(res):
    """fp16 side parameters within 1 ulp; every code difference was already
    proven a half-point case by compare_cache."""
    assert res["tok_ulp"] <= 1 and res["chan_ulp"] <= 1 and res["off_ulp"] <= 1, res
    assert res["code_mismatch"] == res["half_points"], res


def gpu_decode(cfg, cache, q16: np.ndarray, scale: float = 0.0):
    import torch
    from kv_cache_bit_b200 import kvq
    B, Hq, d = q16.shape
    qd = to_dev(f16bits(q16).view(np.int16))
    out = torch.empty((B, Hq, d), dtype=torch.float32, device="cuda")
    nbytes = kvq.kvq_decode_workspace_bytes(cfg, cache, Hq)
    ws = torch.zeros(max(nbytes, 16), dtype=torch.uint8, device="cuda")
    kvq.kvq_decode_attention(cfg, cache, qd, Hq, scale, out, ws, nbytes)
    torch.cuda.synchronize()
    return out.cpu().numpy()
