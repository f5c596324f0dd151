"""GPU parity on the method's degenerate cases (tests/edges.py): an all-zero
token, an all-zero channel (scale 0, codes 0), channels whose scale is an
fp16 subnormal coarse enough to force the clamp of the codes, tiny tokens
for the naive per-token scale, and an all-zero residual token.  Blocks 0
and 1 come from kvq_quantize_block, block 2 from the flush of
kvq_append_token; every mode, bit width and head dim, against the oracle.
Bars as in the other parity tests: codes bit-exact except at rounding
half-points, fp16 side parameters within 1 ulp, dequantized values
bit-exact, decode within 2e-3."""
import numpy as np
import pytest

import oracle
from tests.edges import T, edge_kv
from tests.gpu_helpers import (assert_cache_parity, check_attention, compare_cache, gpu_decode, gpu_prefill, host16,
                               oracle_prefill, to_dev)
from tests.modes import f16bits

pytestmark = pytest.mark.gpu

ATOL = 2e-3
MODES = ["nsep+pchan", "naive", "rht+nsep+pchan", "nsn+hadamard", "nsn", "nsn+hadamard+dq"]


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("bits", [4, 3, 2])
@pytest.mark.parametrize("d", [128, 64])
def test_degenerate_inputs_match_oracle(d, bits, mode):
    import torch
    from kv_cache_bit_b200 import kvq
    B, H, G = 1, 2, 2
    K, V = edge_kv(mode, d, B=B, H=H)
    S = K.shape[2]                      # 3 blocks + 9 residual tokens
    cap = 4 * T
    cfg, cache = gpu_prefill(mode, d, bits, K, V, cap=cap, ntok=2 * T)
    kd = to_dev(f16bits(K).view(np.int16))
    vd = to_dev(f16bits(V).view(np.int16))
    for t in range(2 * T, S):           # block 2 by the append flush, then residual tokens
        kvq.kvq_append_token(cfg, cache, kd[:, :, t].contiguous(), vd[:, :, t].contiguous())
    torch.cuda.synchronize()
    assert cache.len == S
    nq = 3 * T
    ocfg, ck, cv = oracle_prefill(mode, d, bits, K, V, cap=cap, ntok=nq)
    res = compare_cache(cache, ck, cv, d, bits, nq)
    assert_cache_parity(res)
    exact = res["code_mismatch"] == 0 and res["tok_ulp"] == 0 and res["chan_ulp"] == 0 and res["off_ulp"] == 0
    r = S - nq
    assert np.array_equal(host16(cache.resid[0])[:, :, :r], f16bits(K[:, :, nq:S]))
    assert np.array_equal(host16(cache.resid[1])[:, :, :r], f16bits(V[:, :, nq:S]))
    for tensor, oc in ((0, ck), (1, cv)):
        out = torch.empty((B, H, nq, d), dtype=torch.float32, device="cuda")
        kvq.kvq_dequantize(cfg, cache, tensor, 0, nq, out)
        torch.cuda.synchronize()
        ref, bad = oracle.dequantize(ocfg, oc, 0, nq)
        assert bad == 0
        got = out.cpu().numpy()
        assert np.all(np.isfinite(got))
        if exact:
            assert np.array_equal(got, ref)
        else:   # a half-point code or a 1-ulp parameter moves its values by one step
            assert np.allclose(got, ref, rtol=1e-2, atol=1e-3)
    q = np.random.default_rng(1).standard_normal((B, H * G, d)).astype(np.float16)
    out = gpu_decode(cfg, cache, q)
    ref = oracle.cache_attention(ocfg, f16bits(q), ck, cv, f16bits(K[:, :, nq:S]), f16bits(V[:, :, nq:S]), S,
                                 threads=2)
    assert np.all(np.isfinite(out))
    check_attention(f"edges {mode} d{d} int{bits}", out, ref, ATOL)
