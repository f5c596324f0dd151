"""Parity at the full sizes of the five workload configurations, in the launch
configuration the benchmark times (one quantize call over the whole prefill,
the persistent decode grid over the whole batch, appends streamed one token
at a time).

The oracle cannot redo a whole configuration in test time, so it checks
sampled (batch row, kv head) slices: quantization of a slice depends on that
slice alone, and decode of a slice's query heads depends on that slice's
cache alone.  Every output is also checked for properties that hold at any
size: finite decode outputs and no zero code field (offset-binary codes are
never zero).
"""
import numpy as np
import pytest

import oracle
from kv_cache_bit_b200 import synth
from tests.gpu_helpers import assert_cache_parity, check_attention, compare_cache, gpu_decode, gpu_prefill, host16, to_dev
from tests.layout import pairv_applies, pairv_to_rows
from tests.modes import f16bits, oracle_cfg

pytestmark = pytest.mark.gpu

ATOL = 2e-3
T = 128

# (workload, mode, bits, appended tokens); the throughput workload streams
# all of its 256 tokens, as in the benchmark step
CASES = [
    ("tiny", "nsep+pchan", 4, 0),
    ("qwen2-7b-gqa", "nsep+pchan", 4, 37),
    ("pythia-6.9b-mha", "nsep+pchan", 4, 0),
    ("pythia-6.9b-mha", "nsep+pchan", 3, 0),
    ("pythia-6.9b-mha", "naive", 4, 0),
    ("llama-long-ctx", "rht+nsep+pchan", 4, 5),
    ("throughput", "nsn+hadamard", 4, 256),
    ("throughput", "nsn+hadamard", 2, 256),
    ("throughput", "nsn+hadamard+dq", 4, 256),
]


def _sample_pairs(B, H, rng):
    pairs = {(0, 0), (B - 1, H - 1)}
    while len(pairs) < min(4, B * H):
        pairs.add((int(rng.integers(B)), int(rng.integers(H))))
    return sorted(pairs)


def _no_zero_fields(codes_u8, bits):
    """True when no code field of the packed rows is zero."""
    import torch
    c = codes_u8.to(torch.int32)
    if bits == 4:
        return bool(((c & 0xF) != 0).all()) and bool(((c >> 4) != 0).all())
    if bits == 2:
        return all(bool((((c >> (2 * i)) & 3) != 0).all()) for i in range(4))
    # INT3: low 2-bit plane then the bit-2 plane; a field is zero only when
    # both of its parts are, so rebuild the 3-bit codes of the first plane's
    # bytes from both planes
    d8 = c.shape[-1] // 3  # d/8 bytes of the high plane, d/4 of the low plane
    lo = c[..., : 2 * d8]
    hi = c[..., 2 * d8:]
    ok = True
    for i in range(4):
        low = (lo >> (2 * i)) & 3                       # channel 4j + i
        j = torch.arange(2 * d8, device=c.device)
        ch = 4 * j + i
        bit = (hi[..., ch // 8] >> (ch % 8)) & 1
        ok = ok and bool(((low | (bit << 2)) != 0).all())
    return ok


_last = {}


def _inputs(w, n_app):
    """K, V and the streamed tokens of a workload (the last one is kept: two
    cases share the throughput workload)."""
    key = (w.name, n_app)
    if key not in _last:
        _last.clear()
        K, V = synth.kv(w)
        ks, vs = synth.stream_tokens(w, n_app) if n_app else (None, None)
        _last[key] = (K, V, ks, vs)
    return _last[key]


@pytest.mark.parametrize("name,mode,bits,n_app", CASES)
def test_full_size_sampled_parity(name, mode, bits, n_app):
    import torch
    from kv_cache_bit_b200 import kvq
    w = synth.WORKLOADS[name]
    d, B, H, G = w.d, w.B, w.Hkv, w.Hq // w.Hkv
    S = w.S
    K, V, ks, vs = _inputs(w, n_app)
    length = S + n_app
    cap = ((length + T - 1) // T) * T
    cfg, cache = gpu_prefill(mode, d, bits, K, V, cap=cap, ntok=S)
    for i in range(n_app):
        kvq.kvq_append_token(cfg, cache, to_dev(f16bits(ks[i]).view(np.int16)),
                             to_dev(f16bits(vs[i]).view(np.int16)))
    assert cache.len == length
    q = synth.queries(w)
    out = gpu_decode(cfg, cache, q)
    assert np.all(np.isfinite(out))
    nq = (length // T) * T
    for i in range(2):
        c = cache.codes[i][:, :, :nq]
        if i == 1 and bits == 3 and pairv_applies(d):
            # the INT3 check reads the two planes of token-major rows
            c = torch.from_numpy(pairv_to_rows(c.cpu().numpy(), bits)).to(c.device)
        assert _no_zero_fields(c, bits)

    ocfg = oracle_cfg(mode, d, bits)
    rng = np.random.default_rng(11)
    for (b, h) in _sample_pairs(B, H, rng):
        # the slice's full token sequence: prefill then streamed tokens
        kk = K[b, h]
        vv = V[b, h]
        if n_app:
            kk = np.concatenate([kk, ks[:, b, h]], axis=0)
            vv = np.concatenate([vv, vs[:, b, h]], axis=0)
        kk, vv = kk[None, None], vv[None, None]
        ck = oracle.empty_cache(ocfg, 1, 1, cap)
        cv = oracle.empty_cache(ocfg, 1, 1, cap)
        ck["y"] = cv["y"] = None
        if nq:
            ck["y"] = oracle.quantize_products(ocfg, f16bits(kk[:, :, :nq]), ck, 0, 1)
            cv["y"] = oracle.quantize_products(ocfg, f16bits(vv[:, :, :nq]), cv, 0, 1)
        res = compare_cache(cache, ck, cv, d, bits, nq, bh_slice=(slice(b, b + 1), slice(h, h + 1)))
        assert_cache_parity(res)
        r = length - nq
        if r:
            assert np.array_equal(host16(cache.resid[0])[b, h, :r], f16bits(kk[0, 0, nq:length]))
        ref = oracle.cache_attention(ocfg, f16bits(q[b:b + 1, h * G:(h + 1) * G]), ck, cv,
                                     f16bits(kk[:, :, nq:length]), f16bits(vv[:, :, nq:length]), length,
                                     threads=1)
        check_attention(f"full size {name} {mode} int{bits} ({b}, {h})", out[b, h * G:(h + 1) * G], ref[0], ATOL)
    del cache
    torch.cuda.empty_cache()
