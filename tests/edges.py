"""Inputs with the method's degenerate cases, shared by the CPU check of the
construction and the GPU parity test: in blocks 0 and 2 of every (batch,
kv head) slice, one all-zero token, one all-zero channel, one channel of
tiny values (its per-channel scale max|u| / qmax falls into the fp16
subnormal range, where the stored scale is so coarse that some products
u / sigma16 round past qmax and must be clamped) and, for the per-token
scale of the naive mode only, tokens of tiny values; plus one all-zero token
among the residual tokens.  The values are drawn with the seed given."""
import numpy as np

from kv_cache_bit_b200 import synth

T = 128
ZERO_TOKEN, ZERO_CHANNEL = 5, 3
# channel -> magnitude of its tiny values: a subnormal scale that stays
# exact enough (2e-4), and two coarse enough to force clamping at INT4 / INT3
TINY_CHANNELS = {7: 2.5e-6, 11: 1e-6, 13: 2e-4}
# tiny tokens -> their largest |value| in fp16 subnormal quanta (2^-24):
# per-token scales of 10/7 and 4/3 quanta round down to one quantum, which
# forces clamping at INT4 and at INT3
TINY_TOKENS = {9: 10, 10: 4}
EDGE_BLOCKS = (0, 2)


def edge_kv(mode: str, d: int, B: int = 1, H: int = 2, S: int = 3 * T + 9, seed: int = 7):
    nsn = mode.startswith("nsn")
    w = synth.Workload("edges", B=B, Hq=H, Hkv=H, d=d, S=S, sigma_n=0.5,
                       mean_sd=3.0 if nsn else None, spike_p=0.0, spike_amp=10.0,
                       k_outliers=None, seed=seed)
    K, V = synth.kv(w)
    rng = np.random.default_rng(seed + 100)
    out = []
    for X in (K, V):
        X = X.astype(np.float32)
        for blk in EDGE_BLOCKS:
            b0 = blk * T
            rows = slice(b0, b0 + T)
            X[:, :, rows, ZERO_CHANNEL] = 0.0
            for ch, mag in TINY_CHANNELS.items():
                sgn = rng.choice([-1.0, 1.0], size=X[:, :, rows, ch].shape)
                X[:, :, rows, ch] = sgn * rng.uniform(0.5, 1.0, size=sgn.shape) * mag
            for tok, quanta in (TINY_TOKENS.items() if mode == "naive" else ()):
                # (in the normalized modes a tiny token's direction is not tiny)
                tt = X[:, :, b0 + tok, :]
                X[:, :, b0 + tok, :] = tt / np.abs(tt).max(axis=-1, keepdims=True) * (quanta * 2.0 ** -24)
            X[:, :, b0 + ZERO_TOKEN, :] = 0.0
        # a zero token among the residual tokens past the last full block
        X[:, :, 3 * T + 2, :] = 0.0
        out.append(X.astype(np.float16))
    return out[0], out[1]
