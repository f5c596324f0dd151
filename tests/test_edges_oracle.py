"""The degenerate-case inputs of tests/edges.py do what the GPU edge test
relies on, checked on the oracle (CPU): zero scales for the zero channel
(zero code, stored scale 0), fp16-subnormal scales for the tiny channels or
tokens, products u / sigma16 past qmax + 1/2 that the clamp brings back to
+-qmax, and a zero stored norm with all-zero codes for the zero token."""
import numpy as np
import pytest

import oracle
from tests.edges import EDGE_BLOCKS, T, TINY_CHANNELS, TINY_TOKENS, ZERO_CHANNEL, ZERO_TOKEN, edge_kv
from tests.modes import f16bits, oracle_cfg


def _quantize(mode, d, bits, X):
    cfg = oracle_cfg(mode, d, bits)
    c = oracle.empty_cache(cfg, X.shape[0], X.shape[1], 3 * T)
    y = oracle.quantize_products(cfg, f16bits(X[:, :, :3 * T]), c)
    q, bad = oracle.unpack_rows(c["codes"].reshape(-1, oracle.row_bytes(d, bits)), d, bits)
    assert bad == 0
    return c, y, q.reshape(y.shape)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("mode", ["nsep+pchan", "nsn", "naive"])
@pytest.mark.parametrize("bits", [4, 3])
def test_edge_inputs_force_the_clamp(mode, d, bits):
    K, V = edge_kv(mode, d)
    qm = oracle.qmax(bits)
    clamped = subnormal = 0
    for X in (K, V):
        c, y, q = _quantize(mode, d, bits, X)
        over = np.abs(y) > qm + 0.5
        clamped += int(over.sum())
        # every clamped product codes to the end of the range, with its sign
        assert np.all(q[over] == np.sign(y[over]) * qm)
        if mode == "naive":
            s = c["tok"][..., 0].view(np.float16).astype(np.float64)
            for blk in EDGE_BLOCKS:
                for tok in TINY_TOKENS:
                    v = s[:, :, blk * T + tok]
                    assert np.all(v < 2.0 ** -14)                   # subnormal (or flushed) token scale
                    subnormal += int(np.sum(v > 0))
                assert np.all(s[:, :, blk * T + ZERO_TOKEN] == 0)
        else:
            sig = c["chan"].view(np.float16).astype(np.float64)
            for blk in EDGE_BLOCKS:
                assert np.all(sig[:, :, blk, ZERO_CHANNEL] == 0)
                for ch in TINY_CHANNELS:
                    v = sig[:, :, blk, ch]
                    assert np.all(v < 2.0 ** -14)                   # subnormal (or flushed) channel scale
                    subnormal += int(np.sum(v > 0))
                assert np.all(q[:, :, blk * T:(blk + 1) * T, ZERO_CHANNEL] == 0)
        for blk in EDGE_BLOCKS:
            if mode != "nsn":
                # (under NSN a zero token becomes -o after the shift, so only its s1 is 0)
                assert np.all(q[:, :, blk * T + ZERO_TOKEN] == 0)
            if mode != "naive":
                assert np.all(c["tok"][:, :, blk * T + ZERO_TOKEN, 0] == 0)   # stored norm / s1 is 0
    assert clamped > 0 and subnormal > 0


@pytest.mark.parametrize("mode", ["rht+nsep+pchan", "nsn+hadamard"])
def test_edge_inputs_with_the_rotation(mode):
    """Under the rotation the zero token keeps a zero norm / s1 (and codes to
    zeros under nsep); the zero and tiny channels are mixed by the rotation."""
    K, _ = edge_kv(mode, 128)
    c, y, q = _quantize(mode, 128, 4, K)
    for blk in EDGE_BLOCKS:
        assert np.all(c["tok"][:, :, blk * T + ZERO_TOKEN, 0] == 0)
        if mode.startswith("rht"):
            assert np.all(q[:, :, blk * T + ZERO_TOKEN] == 0)
