"""The GPU parity checker itself, run on the CPU against a stand-in of the
library's cache built from the oracle's own bytes: identical caches pass, a
code one step away from the oracle's passes only where the oracle's exact
product sits at a rounding half-point (and is counted), and anything else is
rejected."""
from types import SimpleNamespace

import numpy as np
import pytest
import torch

import oracle
from kv_cache_bit_b200 import synth
from tests.gpu_helpers import HALF_POINT_LOG, assert_cache_parity, compare_cache, oracle_prefill
from tests.layout import rows_to_pairv


@pytest.fixture(autouse=True)
def _keep_the_gpu_log_clean():
    """These checks compare the oracle with itself: keep them out of the
    session's half-point report of GPU parity."""
    n = len(HALF_POINT_LOG)
    yield
    del HALF_POINT_LOG[n:]


def _fake_gpu_cache(ck, cv, d, bits):
    """The oracle's caches in the library's layout (V rows pair-interleaved
    at head dim 128), as CPU tensors."""
    t16 = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a).view(np.int16))
    vcodes = rows_to_pairv(cv["codes"], bits) if d == 128 else cv["codes"]
    return SimpleNamespace(codes=[torch.from_numpy(ck["codes"].copy()), torch.from_numpy(vcodes.copy())],
                           tok=[t16(ck["tok"]), t16(cv["tok"])], chan=[t16(ck["chan"]), t16(cv["chan"])],
                           off=[t16(ck["off"]), t16(cv["off"])])


def _flip_code(codes, y, bits, pick):
    """Move one INT4 code of K (token-major rows) one step toward zero at the
    flat element index `pick` of y; returns the modified code array."""
    assert bits == 4
    d = y.shape[-1]
    flat = codes.reshape(-1, codes.shape[-1]).copy()
    row, c = divmod(pick, d)
    q, _ = oracle.unpack_rows(flat[row:row + 1], d, bits)
    q[0, c] += -1 if q[0, c] > 0 else 1
    flat[row] = oracle.pack_rows(q, bits)[0]
    return flat.reshape(codes.shape)


@pytest.fixture(scope="module")
def caches():
    d, bits = 128, 4
    w = synth.WORKLOADS["qwen2-7b-gqa"].scaled(B=1, Hkv=2, Hq=2, S=256)
    K, V = synth.kv(w)
    _, ck, cv = oracle_prefill("nsep+pchan", d, bits, K, V, threads=2)
    return d, bits, ck, cv


def test_identical_caches_pass(caches):
    d, bits, ck, cv = caches
    res = compare_cache(_fake_gpu_cache(ck, cv, d, bits), ck, cv, d, bits, 256)
    assert_cache_parity(res)
    assert res["code_mismatch"] == 0 and res["codes"] == 2 * 2 * 256 * d


def test_code_off_a_half_point_is_rejected(caches):
    d, bits, ck, cv = caches
    y = ck["y"].reshape(-1)
    pick = int(np.argmax(oracle.half_point_distance(y) > 0.25))   # far from any half-point
    g = _fake_gpu_cache(ck, cv, d, bits)
    g.codes[0] = torch.from_numpy(_flip_code(ck["codes"], ck["y"], bits, pick))
    with pytest.raises(AssertionError, match="away from a rounding half-point"):
        compare_cache(g, ck, cv, d, bits, 256)


def test_code_at_a_half_point_is_accepted_and_counted(caches):
    d, bits, ck, cv = caches
    pick = 12345
    g = _fake_gpu_cache(ck, cv, d, bits)
    g.codes[0] = torch.from_numpy(_flip_code(ck["codes"], ck["y"], bits, pick))
    # the oracle's product planted at an exact half-point next to its code
    ck2 = dict(ck)
    y = ck["y"].copy()
    yf = y.reshape(-1)
    yf[pick] = np.floor(yf[pick]) + 0.5
    ck2["y"] = y
    res = compare_cache(g, ck2, cv, d, bits, 256)
    assert res["code_mismatch"] == 1 and res["half_points"] == 1
    assert_cache_parity(res)


def test_parameter_two_ulps_off_is_rejected(caches):
    d, bits, ck, cv = caches
    g = _fake_gpu_cache(ck, cv, d, bits)
    chan = ck["chan"].copy()
    chan.reshape(-1)[7] += 2
    g.chan[0] = torch.from_numpy(chan.view(np.int16))
    with pytest.raises(AssertionError):
        assert_cache_parity(compare_cache(g, ck, cv, d, bits, 256))
