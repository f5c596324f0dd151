"""GPU sign-pattern selection (kvq_select_signs) against the oracle's: the
per-candidate reconstruction errors agree (bit for bit unless a code sits at
a rounding half-point) and the chosen index is the oracle's (or, where the
two best errors agree to 1e-9, one of them)."""
import numpy as np
import pytest

import oracle
from kv_cache_bit_b200 import synth
from tests.gpu_helpers import gpu_cfg, to_dev
from tests.modes import f16bits, oracle_cfg

pytestmark = pytest.mark.gpu

T = 128


def _sample(mode, d, nb, seed):
    nsn = mode.startswith("nsn")
    w = synth.Workload("sel", B=1, Hq=nb, Hkv=nb, d=d, S=T, sigma_n=0.6, mean_sd=3.0 if nsn else None,
                       k_outliers=None if nsn else synth.Outliers("mul", 8, factors=(50.0,) * 8), seed=seed)
    K, _ = synth.kv(w)
    return f16bits(K).reshape(nb, T, d)


@pytest.mark.parametrize("mode,d,bits,nb,ncand", [("rht+nsep+pchan", 128, 4, 6, 8), ("nsn+hadamard", 128, 4, 5, 6),
                                                  ("rht+nsep+pchan", 64, 3, 3, 4), ("nsn+hadamard", 128, 2, 2, 3),
                                                  ("rht+nsep+pchan", 128, 4, 1, 1)])
def test_select_signs_matches_oracle(mode, d, bits, nb, ncand):
    import torch
    from kv_cache_bit_b200 import kvq
    x = _sample(mode, d, nb, seed=nb)
    signs = np.stack([oracle.make_signs(s, d) for s in range(ncand)])
    best_o, err_o = oracle.select_signs(oracle_cfg(mode, d, bits), x, signs)
    cfg = gpu_cfg(mode, d, bits)
    ws_bytes = kvq.kvq_select_signs_workspace_bytes(ncand, nb)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    err = torch.full((ncand,), float("nan"), dtype=torch.float64, device="cuda")
    best = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    kvq.kvq_select_signs(cfg, to_dev(x.view(np.int16)), nb, to_dev(signs), ncand, err, best, ws, ws_bytes)
    torch.cuda.synchronize()
    e = err.cpu().numpy()
    assert np.all(np.abs(e - err_o) <= 1e-9 * err_o), (e, err_o)
    b = int(best.cpu()[0])
    if b != best_o:
        assert abs(err_o[b] - err_o[best_o]) <= 1e-9 * err_o[best_o]
    assert e[b] == e.min()


def test_select_signs_rejects_bad_arguments():
    import torch
    from kv_cache_bit_b200 import kvq
    d = 128
    x = torch.zeros((1, T, d), dtype=torch.int16, device="cuda")
    signs = torch.ones((2, d), dtype=torch.int8, device="cuda")
    err = torch.zeros(2, dtype=torch.float64, device="cuda")
    best = torch.zeros(4, dtype=torch.int32, device="cuda")
    ws = torch.zeros(64, dtype=torch.uint8, device="cuda")
    no_had = kvq.Config(d, 4, kvq.NORM_SEP | kvq.PER_CHANNEL)
    with pytest.raises(kvq.KvqError) as ei:
        kvq.kvq_select_signs(no_had, x, 1, signs, 2, err, best, ws, 64)
    assert ei.value.status == kvq.KVQ_ERR_UNSUPPORTED
    cfg = kvq.Config(d, 4, kvq.NORM_SEP | kvq.PER_CHANNEL | kvq.HADAMARD)
    with pytest.raises(kvq.KvqError) as ei:
        kvq.kvq_select_signs(cfg, x, 1, signs, 2, err, best, ws, 8)
    assert ei.value.status == kvq.KVQ_ERR_WORKSPACE
    with pytest.raises(kvq.KvqError) as ei:
        kvq.kvq_select_signs(cfg, x, 1, signs, 0, err, best, ws, 64)
    assert ei.value.status == kvq.KVQ_ERR_INVALID_ARG
