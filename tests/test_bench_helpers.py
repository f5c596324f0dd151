"""Host-side plumbing of bench.py (CPU only): the DRAM-traffic figure is
reported only while the kernel sources match the ones it was captured for,
and the sampled oracle comparison counts code differences and tells
half-point cases from real ones."""
import hashlib
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture()
def bench(monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py"])
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import bench as b
    return b


def _sources_sha(b):
    h = hashlib.sha256()
    for f in b.KERNEL_SOURCES:
        with open(os.path.join(ROOT, "kv_cache_bit_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def test_traffic_reported_for_matching_sources(bench, tmp_path, monkeypatch):
    p = tmp_path / "traffic.md"
    p.write_text(f"x\ntraffic_bytes_per_call: 1234\nsource_sha256: {_sources_sha(bench)}\n")
    monkeypatch.setattr(bench, "TRAFFIC_PROFILE", str(p))
    assert bench.decode_traffic() == 1234.0


def test_traffic_withheld_after_a_source_change(bench, tmp_path, monkeypatch):
    p = tmp_path / "traffic.md"
    p.write_text("traffic_bytes_per_call: 1234\nsource_sha256: " + "0" * 64 + "\n")
    monkeypatch.setattr(bench, "TRAFFIC_PROFILE", str(p))
    assert bench.decode_traffic() is None


def test_traffic_withheld_without_a_profile(bench, tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "TRAFFIC_PROFILE", str(tmp_path / "missing.md"))
    assert bench.decode_traffic() is None


def _fake_gpu_cache(state, w, bits, cap):
    """The oracle's caches laid out as the library stores them (batch rows of
    one kv head each, V rows pair-interleaved at head dim 128), CPU tensors."""
    from types import SimpleNamespace
    import numpy as np
    import torch
    from tests.layout import rows_to_pairv
    cfg, ck, cv, _, _ = state

    def pad(a, n):
        out = np.zeros(a.shape[:2] + (n,) + a.shape[3:], a.dtype)
        out[:, :, :a.shape[2]] = a
        return out

    vcodes = rows_to_pairv(cv["codes"], bits) if w.d == 128 else cv["codes"]
    codes = [torch.from_numpy(pad(ck["codes"], cap)), torch.from_numpy(pad(vcodes, cap))]
    t16 = lambda a, n: None if a is None else torch.from_numpy(pad(a, n).view(np.int16))
    return SimpleNamespace(codes=codes, tok=[t16(ck["tok"], cap), t16(cv["tok"], cap)],
                           chan=[t16(ck["chan"], cap // 128), t16(cv["chan"], cap // 128)],
                           off=[t16(ck["off"], cap // 128), t16(cv["off"], cap // 128)])


def test_sampled_parity_of_the_bench(bench):
    """The bench's sampled oracle comparison: identical caches give no
    mismatch; a code moved away from a half-point is reported as such."""
    import numpy as np
    import torch
    import oracle
    from kv_cache_bit_b200 import synth
    w = synth.WORKLOADS["throughput"].scaled(B=1, Hkv=2, Hq=8, S=256)
    K, V = synth.kv(w)
    pairs, bits = 2, 4
    data = (K.reshape(-1, 1, w.S, w.d)[:pairs], V.reshape(-1, 1, w.S, w.d)[:pairs])
    *_, state = bench.run_oracle_sample(w, "nsn+hadamard", bits, pairs, 2, 0.0, data)
    cache = _fake_gpu_cache(state, w, bits, 384)
    res = bench.sampled_parity(w, bits, state, cache, pairs)
    assert res["codes_compared"] == 2 * pairs * w.S * w.d
    assert res["code_mismatches"] == 0 and res["max_param_ulp"] == 0
    # one K code one step toward zero, far from a half-point
    y = state[3].reshape(-1)
    pick = int(np.argmax(oracle.half_point_distance(y) > 0.25))
    row, c = divmod(pick, w.d)
    flat = cache.codes[0].numpy().reshape(-1, 384, 64)
    q, _ = oracle.unpack_rows(flat[row // w.S, row % w.S][None], w.d, bits)
    q[0, c] += -1 if q[0, c] > 0 else 1
    flat[row // w.S, row % w.S] = oracle.pack_rows(q, bits)[0]
    res = bench.sampled_parity(w, bits, state, cache, pairs)
    assert res["code_mismatches"] == 1 and res["non_half_point_mismatches"] == 1 and res["half_point_cases"] == 0
