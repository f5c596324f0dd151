"""The kernels' give-up path, on the GPU, without a fault or a hang.

The test build of the library (libkvq_waittest.so: the product sources
compiled with KVQ_WAIT_TEST) lets a test scale the poll limit of the
kernels' main-loop waits; at 0 every such wait gives up at once.  The
quantize kernel then records a TMA-wait timeout and the decode kernel a
barrier timeout in the device error word, each drains its copies in flight
with its normal bounded waits and returns.  With the scale back at 1 the
same calls give the oracle's results and set no error bit.
"""
import ctypes
import os

import numpy as np
import pytest

import oracle
from kv_cache_bit_b200 import synth
from tests.gpu_helpers import assert_cache_parity, compare_cache, gpu_decode, oracle_prefill, to_dev
from tests.modes import f16bits

pytestmark = pytest.mark.gpu

ERR_TMA, ERR_BARRIER = 1, 2


@pytest.fixture()
def waitlib(monkeypatch):
    from kv_cache_bit_b200 import build, kvq
    assert os.path.exists(build.TEST_LIB), "the test build libkvq_waittest.so is missing (run the build)"
    product = kvq.LIB_PATH
    kvq.LIB_PATH = build.TEST_LIB
    try:
        L = kvq._load()
    finally:
        kvq.LIB_PATH = product
    L.kvq_test_set_wait_scale.restype = ctypes.c_int
    L.kvq_test_set_wait_scale.argtypes = [ctypes.c_uint32]
    monkeypatch.setattr(kvq, "lib", L)
    kvq.kvq_read_device_errors(clear=True)
    yield L
    L.kvq_test_set_wait_scale(1)


@pytest.mark.parametrize("mode", ["nsn+hadamard", "nsep+pchan"])
def test_quantize_and_decode_give_up_and_recover(waitlib, mode):
    import torch
    from kv_cache_bit_b200 import kvq
    from tests.gpu_helpers import gpu_cfg
    d, bits, S = 128, 4, 384
    w = synth.Workload("waits", B=2, Hq=8, Hkv=2, d=d, S=S, sigma_n=0.6,
                       mean_sd=3.0 if mode.startswith("nsn") else None, seed=5)
    K, V = synth.kv(w)
    q = synth.queries(w)
    cfg = gpu_cfg(mode, d, bits)
    kd = to_dev(f16bits(K).view(np.int16))
    vd = to_dev(f16bits(V).view(np.int16))

    # every main-loop wait gives up: the quantizer reports the TMA wait
    assert waitlib.kvq_test_set_wait_scale(0) == kvq.KVQ_OK
    cache = kvq.KVCache.allocate(cfg, w.B, w.Hkv, S)
    kvq.kvq_quantize_block(cfg, cache, kd, vd, 0, S)
    torch.cuda.synchronize()
    assert kvq.kvq_read_device_errors(clear=True) & ERR_TMA

    # normal limits: the oracle's cache, no error
    assert waitlib.kvq_test_set_wait_scale(1) == kvq.KVQ_OK
    cache = kvq.KVCache.allocate(cfg, w.B, w.Hkv, S)
    kvq.kvq_quantize_block(cfg, cache, kd, vd, 0, S)
    torch.cuda.synchronize()
    assert kvq.kvq_read_device_errors(clear=True) == 0
    ocfg, ck, cv = oracle_prefill(mode, d, bits, K, V, cap=S, threads=4)
    assert_cache_parity(compare_cache(cache, ck, cv, d, bits, S))

    # decode gives up on its ring barriers, then recovers
    assert waitlib.kvq_test_set_wait_scale(0) == kvq.KVQ_OK
    gpu_decode(cfg, cache, q)
    assert kvq.kvq_read_device_errors(clear=True) & ERR_BARRIER
    assert waitlib.kvq_test_set_wait_scale(1) == kvq.KVQ_OK
    out = gpu_decode(cfg, cache, q)
    assert kvq.kvq_read_device_errors(clear=True) == 0
    ref = oracle.cache_attention(ocfg, f16bits(q), ck, cv, np.zeros((w.B, w.Hkv, 0, d), np.uint16),
                                 np.zeros((w.B, w.Hkv, 0, d), np.uint16), S, threads=4)
    assert float(np.max(np.abs(out - ref))) <= 2e-3
