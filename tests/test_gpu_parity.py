"""GPU parity: the CUDA library (called through the C ABI) against the CPU
oracle on the same seeded inputs.

Bars: packed codes bit-exact (neighbouring codes allowed only at rounding
half-points, counted); fp16 side parameters within 1 ulp; dequantized fp32
values bit-exact (same operation order on both sides); decode attention
within max-abs 2e-3 of the oracle's fp64 attention over the oracle's
dequantized cache.
"""
import numpy as np
import pytest

import oracle
from kv_cache_bit_b200 import synth
from tests.gpu_helpers import (assert_cache_parity, check_attention, compare_cache, gpu_decode, gpu_prefill, host16,
                               oracle_prefill, to_dev)
from tests.modes import f16bits

pytestmark = pytest.mark.gpu

ATOL = 2e-3
MODES = ["nsep+pchan", "naive", "rht+nsep+pchan", "nsn+hadamard", "nsn", "nsn+hadamard+dq", "nsn+dq"]


def small_workload(mode, d, B=2, H=2, Hq=None, S=384, seed=3):
    nsn = mode.startswith("nsn")
    return synth.Workload("small", B=B, Hq=Hq or H, Hkv=H, d=d, S=S, sigma_n=0.6,
                          mean_sd=3.0 if nsn else None,
                          spike_p=0.01 if mode.startswith("rht") else 0.0, spike_amp=10.0,
                          k_outliers=None if nsn else synth.Outliers("mul", 4, factors=(50.0,) * 4), seed=seed)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("bits", [4, 3, 2])
@pytest.mark.parametrize("d", [128, 64])
def test_quantize_and_dequantize_match_oracle(d, bits, mode):
    import torch
    from kv_cache_bit_b200 import kvq
    w = small_workload(mode, d)
    K, V = synth.kv(w)
    cap = 512
    cfg, cache = gpu_prefill(mode, d, bits, K, V, cap=cap)
    ocfg, ck, cv = oracle_prefill(mode, d, bits, K, V, cap=cap)
    res = compare_cache(cache, ck, cv, d, bits, w.S)
    assert_cache_parity(res)
    assert cache.len == w.S
    # the blocks past the quantized range are untouched
    assert int(cache.codes[0][:, :, w.S:].abs().sum()) == 0
    for tensor, oc in ((0, ck), (1, cv)):
        out = torch.empty((w.B, w.Hkv, w.S, d), dtype=torch.float32, device="cuda")
        kvq.kvq_dequantize(cfg, cache, tensor, 0, w.S, out)
        torch.cuda.synchronize()
        ref, bad = oracle.dequantize(ocfg, oc, 0, w.S)
        assert bad == 0
        if res["code_mismatch"] == 0 and res["tok_ulp"] == 0 and res["chan_ulp"] == 0 and res["off_ulp"] == 0:
            assert np.array_equal(out.cpu().numpy(), ref)
        else:
            assert np.allclose(out.cpu().numpy(), ref, rtol=1e-2, atol=1e-3)
        # a sub-range starting past block 0
        out2 = torch.empty((w.B, w.Hkv, 128, d), dtype=torch.float32, device="cuda")
        kvq.kvq_dequantize(cfg, cache, tensor, 128, 128, out2)
        torch.cuda.synchronize()
        assert np.array_equal(out2.cpu().numpy(), out.cpu().numpy()[:, :, 128:256])


def test_repeat_runs_are_deterministic():
    K, V = synth.kv(small_workload("nsn+hadamard", 128, S=512))
    _, c1 = gpu_prefill("nsn+hadamard", 128, 4, K, V)
    _, c2 = gpu_prefill("nsn+hadamard", 128, 4, K, V)
    for i in range(2):
        assert bool((c1.codes[i] == c2.codes[i]).all()) and bool((c1.tok[i] == c2.tok[i]).all())
        assert bool((c1.chan[i] == c2.chan[i]).all()) and bool((c1.off[i] == c2.off[i]).all())


def _oracle_attention(ocfg, ck, cv, K, V, q, length, scale=None):
    resid_k = f16bits(K[:, :, (length // 128) * 128: length])
    resid_v = f16bits(V[:, :, (length // 128) * 128: length])
    return oracle.cache_attention(ocfg, f16bits(q), ck, cv, resid_k, resid_v, length, scale, threads=8)


DECODE_CASES = [
    # (mode, d, bits, B, Hkv, Hq, S prefilled, appended tokens)
    ("nsep+pchan", 64, 4, 1, 8, 8, 256, 0),       # tiny workload geometry
    ("nsep+pchan", 128, 4, 2, 4, 28, 512, 37),    # Qwen2-7B-shaped GQA (g = 7), ragged residual
    ("nsep+pchan", 128, 4, 2, 4, 4, 384, 0),      # Pythia-shaped MHA
    ("nsep+pchan", 128, 3, 2, 4, 4, 384, 5),
    ("naive", 128, 4, 2, 4, 4, 384, 0),
    ("rht+nsep+pchan", 128, 4, 1, 2, 8, 1024, 100),   # long-context geometry (g = 4)
    ("nsn+hadamard", 128, 4, 2, 2, 8, 512, 140),      # throughput geometry, with a flush
    ("nsn+hadamard", 128, 2, 2, 2, 8, 512, 3),
    ("nsn", 128, 4, 1, 2, 4, 256, 0),
    ("nsep+pchan", 128, 2, 1, 2, 16, 256, 0),     # g = 8
    ("nsep+pchan", 64, 3, 1, 2, 2, 128, 1),
    # rotation with one and two query heads per kv head (idle fragment columns)
    ("rht+nsep+pchan", 128, 4, 2, 2, 2, 256, 7),
    ("nsn+hadamard", 128, 2, 1, 2, 4, 256, 0),
    # rotation with two n-tiles of query heads (G = 6 and 8)
    ("rht+nsep+pchan", 128, 4, 1, 2, 12, 384, 9),
    ("nsn+hadamard", 128, 4, 1, 1, 8, 256, 3),
    # one long pair spread over every CTA of the persistent grid: more than
    # 128 candidate partials per pair in the combine
    ("nsn+hadamard", 128, 4, 1, 1, 4, 200 * 128, 17),
    # double-quantized NSN side parameters (both decode paths, flushes)
    ("nsn+hadamard+dq", 128, 4, 2, 2, 8, 512, 140),
    ("nsn+hadamard+dq", 128, 2, 1, 2, 16, 384, 5),
    ("nsn+dq", 128, 3, 2, 2, 4, 256, 0),
    ("nsn+dq", 64, 4, 1, 4, 8, 384, 130),
    ("nsn+hadamard+dq", 64, 2, 1, 2, 2, 256, 1),
]


@pytest.mark.parametrize("mode,d,bits,B,Hkv,Hq,S,n_app", DECODE_CASES)
def test_decode_matches_oracle(mode, d, bits, B, Hkv, Hq, S, n_app):
    from kv_cache_bit_b200 import kvq
    w = small_workload(mode, d, B=B, H=Hkv, Hq=Hq, S=S + n_app)
    K, V = synth.kv(w)
    q = synth.queries(w)
    cap = ((S + n_app + 127) // 128 + 1) * 128
    cfg, cache = gpu_prefill(mode, d, bits, K, V, cap=cap, ntok=S)
    for t in range(S, S + n_app):
        kvq.kvq_append_token(cfg, cache, to_dev(f16bits(K[:, :, t]).view(np.int16)),
                             to_dev(f16bits(V[:, :, t]).view(np.int16)))
    length = S + n_app
    assert cache.len == length
    nq = (length // 128) * 128
    ocfg, ck, cv = oracle_prefill(mode, d, bits, K, V, cap=cap, ntok=nq)
    assert_cache_parity(compare_cache(cache, ck, cv, d, bits, nq))
    # residual slots hold the fp16 tokens past the last full block
    r = length - nq
    if r:
        assert np.array_equal(host16(cache.resid[0])[:, :, :r], f16bits(K[:, :, nq:length]))
        assert np.array_equal(host16(cache.resid[1])[:, :, :r], f16bits(V[:, :, nq:length]))
    out = gpu_decode(cfg, cache, q)
    ref = _oracle_attention(ocfg, ck, cv, K, V, q, length)
    check_attention(f"decode {mode} d{d} int{bits} B{B} S{S}+{n_app}", out, ref, ATOL)


def test_decode_custom_scale_and_empty_cache():
    mode, d, bits = "nsep+pchan", 128, 4
    w = small_workload(mode, d, B=1, H=2, Hq=4, S=256)
    K, V = synth.kv(w)
    q = synth.queries(w)
    cfg, cache = gpu_prefill(mode, d, bits, K, V, cap=256, ntok=0)
    assert np.all(gpu_decode(cfg, cache, q) == 0)
    cfg, cache = gpu_prefill(mode, d, bits, K, V, cap=256)
    ocfg, ck, cv = oracle_prefill(mode, d, bits, K, V)
    out = gpu_decode(cfg, cache, q, scale=0.02)
    ref = _oracle_attention(ocfg, ck, cv, K, V, q, 256, scale=0.02)
    check_attention("decode custom scale", out, ref, ATOL)


def test_residual_only_cache():
    from kv_cache_bit_b200 import kvq
    mode, d, bits = "nsn+hadamard", 128, 4
    w = small_workload(mode, d, B=2, H=2, Hq=8, S=77)
    K, V = synth.kv(w)
    q = synth.queries(w)
    cfg, cache = gpu_prefill(mode, d, bits, K, V, cap=128, ntok=0)
    for t in range(77):
        kvq.kvq_append_token(cfg, cache, to_dev(f16bits(K[:, :, t]).view(np.int16)),
                             to_dev(f16bits(V[:, :, t]).view(np.int16)))
    out = gpu_decode(cfg, cache, q)
    ref = oracle.attention(f16bits(q), K.astype(np.float32), V.astype(np.float32))
    check_attention("decode residual only", out, ref, ATOL)


def test_streaming_flush_equals_bulk_quantize():
    """Appending 256 tokens one by one (two flushes) stores the same blocks
    that one bulk quantize of those tokens stores."""
    from kv_cache_bit_b200 import kvq
    mode, d, bits = "nsn+hadamard", 128, 4
    w = small_workload(mode, d, B=2, H=2, S=384)
    K, V = synth.kv(w)
    cfg, cache = gpu_prefill(mode, d, bits, K, V, cap=512, ntok=128)
    for t in range(128, 384):
        kvq.kvq_append_token(cfg, cache, to_dev(f16bits(K[:, :, t]).view(np.int16)),
                             to_dev(f16bits(V[:, :, t]).view(np.int16)))
    _, bulk = gpu_prefill(mode, d, bits, K, V, cap=512)
    for i in range(2):
        assert bool((cache.codes[i][:, :, :384] == bulk.codes[i][:, :, :384]).all())
        assert bool((cache.tok[i][:, :, :384] == bulk.tok[i][:, :, :384]).all())
        assert bool((cache.chan[i][:, :, :3] == bulk.chan[i][:, :, :3]).all())
        assert bool((cache.off[i][:, :, :3] == bulk.off[i][:, :, :3]).all())


def test_batch_row_views_quantize_and_decode_like_the_whole_cache():
    """kvq_quantize_block on batch-row views (KVCache.rows) stores the same
    bytes as one call over the whole batch, and decode over the whole cache
    then gives the same outputs; the views share the cache's memory."""
    import torch
    from kv_cache_bit_b200 import kvq
    mode, d, bits = "nsn+hadamard", 128, 4
    w = small_workload(mode, d, B=4, H=2, Hq=8, S=384)
    K, V = synth.kv(w)
    q = synth.queries(w)
    cfg, whole = gpu_prefill(mode, d, bits, K, V, cap=512)
    _, parts = gpu_prefill(mode, d, bits, K, V, cap=512, ntok=0)
    kd = to_dev(f16bits(K).view(np.int16))
    vd = to_dev(f16bits(V).view(np.int16))
    for b0 in (0, 1, 3):
        b1 = {0: 1, 1: 3, 3: 4}[b0]
        view = parts.rows(b0, b1)
        kvq.kvq_quantize_block(cfg, view, kd[b0:b1], vd[b0:b1], 0, w.S)
    torch.cuda.synchronize()
    for i in range(2):
        assert bool((parts.codes[i] == whole.codes[i]).all())
        assert bool((parts.tok[i] == whole.tok[i]).all())
        assert bool((parts.chan[i] == whole.chan[i]).all())
        assert bool((parts.off[i] == whole.off[i]).all())
    parts.c.len = w.S
    assert np.array_equal(gpu_decode(cfg, parts, q), gpu_decode(cfg, whole, q))
