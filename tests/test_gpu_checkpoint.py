"""Checkpoint / resume of a cache (GPU): the cache is plain caller-owned
memory, so a host snapshot of its buffers and token count is its whole
state.  A fresh cache restored from the snapshot decodes exactly like the
original, and both go on identically when the same tokens are appended."""
import numpy as np
import pytest

from kv_cache_bit_b200 import synth
from tests.gpu_helpers import gpu_decode, gpu_prefill, to_dev
from tests.modes import f16bits

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode,d,bits", [("nsn+hadamard", 128, 4), ("nsep+pchan", 64, 3), ("nsn+hadamard+dq", 128, 2)])
def test_snapshot_restore_decodes_identically(mode, d, bits):
    import torch
    from kv_cache_bit_b200 import kvq
    w = synth.WORKLOADS["throughput"].scaled(B=2, Hkv=2, Hq=8, d=d, S=300, stream=0)
    K, V = synth.kv(w)
    q = synth.queries(w, steps=2)
    cfg, cache = gpu_prefill(mode, d, bits, K, V, cap=512, ntok=256)
    tok = lambda X, t: to_dev(f16bits(X[:, :, t]).view(np.int16))
    for t in range(256, 270):                       # 14 residual tokens
        kvq.kvq_append_token(cfg, cache, tok(K, t), tok(V, t))
    snap = cache.snapshot()
    assert snap["len"] == 270
    out1 = gpu_decode(cfg, cache, q[0])
    fresh = kvq.KVCache.allocate(cfg, w.B, w.Hkv, 512)
    fresh.restore(snap)
    assert fresh.len == 270
    assert np.array_equal(gpu_decode(cfg, fresh, q[0]), out1)
    # both caches take the same tokens (a flush at 384 included) and stay equal
    for t in range(270, 300):
        for c in (cache, fresh):
            kvq.kvq_append_token(cfg, c, tok(K, t), tok(V, t))
    torch.cuda.synchronize()
    assert np.array_equal(gpu_decode(cfg, fresh, q[1]), gpu_decode(cfg, cache, q[1]))
    for name in ("codes", "tok", "chan", "off", "resid"):
        for a, b in zip(getattr(cache, name), getattr(fresh, name)):
            assert (a is None) == (b is None)
            if a is not None:
                assert torch.equal(a, b), name
    # a snapshot of another shape is refused
    other = kvq.KVCache.allocate(cfg, w.B, w.Hkv, 256)
    with pytest.raises(kvq.KvqError):
        other.restore(snap)
