"""The allocation-free decode entry point.

kvq_decode_attention_noalloc serves callers that are handed only their
input and output buffers and cannot allocate device memory (an operator
plugin inside an engine that plans all device memory up front, or a
latency-critical path where cudaMalloc would synchronize the device).  It
keeps its split-K partials in the library's own fixed-size device scratch
array instead of a caller workspace.  These checks call it through the C ABI
and compare it with kvq_decode_attention on the same cache and with the
oracle's fp64 attention, twice in a row on a cache that changes in between
(the scratch keeps the previous call's contents), on both decode paths.  This file is collected
last so that a run stopping at its first failure has run everything else.
"""
import ctypes

import numpy as np
import pytest

import oracle
from kv_cache_bit_b200 import synth
from tests.gpu_helpers import check_attention, gpu_decode, gpu_prefill, oracle_prefill, to_dev
from tests.modes import f16bits

ATOL = 2e-3


# (head dim, mode): the tensor-core decode path (head dim 128) and the
# split-K CUDA-core path (head dim 64), each with its own partial layout in
# the shared scratch
CASES = [(128, "nsn+hadamard"), (64, "nsep+pchan")]


@pytest.mark.gpu
@pytest.mark.parametrize("d,mode", CASES)
def test_noalloc_decode_matches_workspace_decode_and_oracle_twice(d, mode):
    import torch
    from kv_cache_bit_b200 import kvq
    w = synth.WORKLOADS["throughput"].scaled(B=2, Hkv=2, Hq=8, d=d, S=640, stream=0)
    K, V = synth.kv(w)
    cfg, cache = gpu_prefill(mode, w.d, 4, K, V, cap=768, ntok=512)
    for t in range(512, 640):                       # one flush, then a residual-free cache
        kvq.kvq_append_token(cfg, cache, to_dev(f16bits(K[:, :, t]).view(np.int16)),
                             to_dev(f16bits(V[:, :, t]).view(np.int16)))
    assert kvq.kvq_decode_workspace_bytes(cfg, cache, w.Hq) <= kvq.NOALLOC_SCRATCH_BYTES
    qs = synth.queries(w, steps=2)
    extra = f16bits(K[:, :, 0:1]), f16bits(V[:, :, 0:1])   # the token appended between the calls
    ocfg, ck, cv = oracle_prefill(mode, w.d, 4, K, V, cap=768, ntok=640, threads=4)
    for step in range(2):
        q = qs[step]
        length = 640 + step
        ref = gpu_decode(cfg, cache, q)
        out = torch.full((w.B, w.Hq, w.d), float("nan"), dtype=torch.float32, device="cuda")
        kvq.kvq_decode_attention_noalloc(cfg, cache, to_dev(f16bits(q).view(np.int16)), w.Hq, 0.0, out)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.all(np.isfinite(got))
        assert np.max(np.abs(got - ref)) <= ATOL
        # and the oracle's fp64 attention over its own cache (residual: the appended tokens)
        rk = extra[0][:, :, :step] if step else np.zeros((w.B, w.Hkv, 0, w.d), np.uint16)
        rv = extra[1][:, :, :step] if step else np.zeros((w.B, w.Hkv, 0, w.d), np.uint16)
        oref = oracle.cache_attention(ocfg, f16bits(q), ck, cv, rk, rv, length, threads=4)
        check_attention(f"no-alloc decode {mode} d{d} call {step}", got, oref, ATOL)
        # a token more between the calls changes the cache the second call sees
        kvq.kvq_append_token(cfg, cache, to_dev(f16bits(K[:, :, 0]).view(np.int16)),
                             to_dev(f16bits(V[:, :, 0]).view(np.int16)))


def test_noalloc_rejects_workspace_beyond_its_scratch():
    """A cache whose decode would need more than the fixed scratch is refused
    on the host before anything is enqueued (placeholder addresses are never
    dereferenced because the size check fails first)."""
    from kv_cache_bit_b200 import kvq
    a = 1 << 20
    P2 = ctypes.c_void_p * 2
    big = kvq.kvq_cache(64, 32, 128, 128, 0, P2(a, a), P2(a, a), P2(a, a), P2(a, a), P2(a, a))
    cfg = kvq.kvq_config(128, 4, kvq.NSN | kvq.PER_CHANNEL | kvq.HADAMARD, 0, None)
    need = kvq.lib.kvq_decode_workspace_bytes(ctypes.byref(cfg), ctypes.byref(big), 256)
    assert need > kvq.NOALLOC_SCRATCH_BYTES
    st = kvq.lib.kvq_decode_attention_noalloc(ctypes.byref(cfg), ctypes.byref(big), a, 256, 0.0, a, None)
    assert st == kvq.KVQ_ERR_WORKSPACE
