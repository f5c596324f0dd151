"""Pins of the oracle's sign-pattern selection (CPU): its errors are the
reconstruction errors that the oracle's own quantize and dequantize give,
summed exactly (math.fsum) they agree to rounding; the chosen index is the
smallest error and the lowest index among equal ones; sign vectors that
differ from the rotation's effect only by a global sign give equal errors.
The selection follows the "Activation-guided compensation and orthogonal
residuals" abstract: sample several random sign patterns, keep the best."""
import math

import numpy as np
import pytest

import oracle
from kv_cache_bit_b200 import synth
from tests.modes import f16bits, oracle_cfg

T = oracle.T


def _sample(mode, d=128, nb=3, seed=1):
    nsn = mode.startswith("nsn")
    w = synth.Workload("sel", B=1, Hq=nb, Hkv=nb, d=d, S=T, sigma_n=0.6, mean_sd=3.0 if nsn else None,
                       k_outliers=None if nsn else synth.Outliers("mul", 8, factors=(50.0,) * 8), seed=seed)
    K, _ = synth.kv(w)
    return f16bits(K).reshape(nb, T, d)


@pytest.mark.parametrize("mode,bits", [("rht+nsep+pchan", 4), ("nsn+hadamard", 4), ("rht+nsep+pchan", 2)])
def test_errors_are_the_reconstruction_errors(mode, bits):
    d = 128
    x = _sample(mode)
    cfg = oracle_cfg(mode, d, bits)
    signs = np.stack([oracle.make_signs(s, d) for s in range(5)])
    best, err = oracle.select_signs(cfg, x, signs)
    for k in range(len(signs)):
        c = oracle.Cfg(d, bits, cfg.flags, signs[k])
        cache = oracle.quantize(c, x[:, None])                    # [nb, 1, T, ...]
        xh, bad = oracle.dequantize(c, cache, 0, T)
        assert bad == 0
        diff = xh.astype(np.float64) - x.view(np.float16).astype(np.float64)[:, None]
        exact = math.fsum((diff * diff).ravel().tolist())
        assert abs(err[k] - exact) <= 1e-12 * exact
    assert err[best] == err.min() and best == int(np.argmin(err))


def test_ties_take_the_lowest_index_and_global_sign_is_neutral():
    """Flipping every sign flips the sign of the rotated row: the norms,
    scales and |codes| are the same and so is the error."""
    d = 128
    x = _sample("rht+nsep+pchan", nb=2, seed=4)
    cfg = oracle_cfg("rht+nsep+pchan", d, 4)
    s0 = oracle.make_signs(7, d)
    s1 = oracle.make_signs(8, d)
    best, err = oracle.select_signs(cfg, x, np.stack([s1, s0, -s0]))
    assert err[1] == err[2]
    if err[1] < err[0]:
        assert best == 1
    _, err2 = oracle.select_signs(cfg, x, np.stack([s0, s0]))
    b2, _ = oracle.select_signs(cfg, x, np.stack([s0, s0]))
    assert err2[0] == err2[1] and b2 == 0


def test_selection_prefers_signs_that_spread_persistent_outliers():
    """Eight persistent outlier channels of equal value: under the plain
    Hadamard rotation (all signs +1) their sum lands on few rotated channels
    (constructive interference), random signs spread it; the selection
    therefore does better than the all-ones pattern."""
    d = 128
    rng = np.random.default_rng(2)
    z = rng.standard_normal((2, T, d)).astype(np.float32)
    z[:, :, :8] = 40.0                       # channels 0..7: one persistent outlier value
    x = f16bits(z)
    cfg = oracle_cfg("rht+nsep+pchan", d, 4)
    cands = np.stack([np.ones(d, np.int8)] + [oracle.make_signs(s, d) for s in range(1, 8)])
    best, err = oracle.select_signs(cfg, x, cands)
    assert best != 0 and err[best] < err[0]
