"""Pins of the oracle's double quantization (DQ) of the NSN side parameters
(CPU).  NSNQuant explainer, "3. Vector Quantization and Codebook -> Double
Quantization (DQ)": the NSN mean o and scale s1 are themselves quantized to
4 bits.  Reading: per 128-token block, o with symmetric codes and one fp16
scale (max|o| / 7), s1 with unsigned codes over [lo, lo + 15 step]
(lo = min s1, step = (max s1 - lo) / 15, both fp16); the encoder subtracts
the reconstructed mean, as the decoder adds it back."""
import math

import numpy as np
import pytest

import oracle
from kv_cache_bit_b200 import synth
from tests.modes import f16bits

T = oracle.T
DQ = oracle.DQ


def f16(v):
    return np.float32(v).astype(np.float16).astype(np.float64)


def _data(seed=3):
    w = synth.WORKLOADS["throughput"].scaled(B=1, Hkv=2, Hq=2, S=256, seed=seed)
    K, _ = synth.kv(w)
    return K


def test_record_layout_worked_example():
    """A hand-built record: o codes, s1 codes and the three fp16 values."""
    d = 64
    rb = oracle.dq_record_bytes(d)
    assert rb == (32 + 64 + 6 + 15) // 16 * 16 == 112
    rec = np.zeros(rb, np.uint8)
    qo = np.array([(c % 15) - 7 for c in range(d)])
    for c in range(d):
        rec[c // 2] |= (qo[c] + 8) << (4 * (c % 2))
    qs = np.array([t % 16 for t in range(T)])
    for t in range(T):
        rec[d // 2 + t // 2] |= qs[t] << (4 * (t % 2))
    rec[d // 2 + T // 2: d // 2 + T // 2 + 6] = np.array([0.25, 0.5, 0.125], np.float16).view(np.uint8)
    o, s1 = oracle.dq_decode(rec, d)
    assert np.array_equal(o, (qo * 0.25).astype(np.float32))
    assert np.array_equal(s1, (0.5 + qs * 0.125).astype(np.float32))


@pytest.mark.parametrize("had", [False, True])
def test_dq_closed_form(had):
    d = 128
    K = _data()
    x = K.astype(np.float64)
    flags = oracle.NSN | oracle.PER_CHANNEL | DQ | (oracle.HADAMARD if had else 0)
    c = oracle.quantize(oracle.Cfg(d, 4, flags), f16bits(K))
    assert c["tok"].shape[-1] == 1 and c["off"].shape[-1] == oracle.dq_record_bytes(d) // 2
    sd = math.sqrt(d)
    n1 = np.linalg.norm(x, axis=-1)
    s1 = n1 / sd                                          # [1, 2, 256]
    a = x * (sd / n1[..., None])
    B, H, S, _ = x.shape
    ab = a.reshape(B, H, S // T, T, d)
    o = ab.mean(axis=3)                                   # [1, 2, 2, d]
    for b in range(B):
        for h in range(H):
            for k in range(S // T):
                rec = c["off"][b, h, k].view(np.uint8)
                oh, s1h = oracle.dq_decode(rec, d)
                so = rec[d // 2 + T // 2: d // 2 + T // 2 + 6].view(np.float16).astype(np.float64)
                # o: sigma_o = fp16(max|o| / 7); codes = rne(o / sigma_o) away from half-points
                assert abs(so[0] - f16(np.abs(o[b, h, k]).max() / 7)) <= 1e-3 * so[0]
                qo = o[b, h, k] / so[0]
                near = np.abs(np.abs(qo - np.trunc(qo)) - 0.5) < 1e-4
                assert np.all((np.rint(qo) == np.rint(oh / so[0])) | near)
                assert np.all(np.abs(oh - o[b, h, k]) <= 0.5 * so[0] * (1 + 1e-4) + 1e-6)
                # s1: lo = fp16(min), step = fp16((max - lo) / 15), |s1_hat - s1| <= step / 2
                sb = s1[b, h, k * T:(k + 1) * T]
                assert so[1] == f16(sb.min()) or abs(so[1] - f16(sb.min())) <= 1e-3 * so[1]
                assert abs(so[2] - f16((sb.max() - so[1]) / 15)) <= 1e-3 * so[2]
                assert np.all(np.abs(s1h - sb) <= 0.5 * so[2] * (1 + 1e-3) + 1e-4 * sb)
                # the encoder subtracted the reconstructed mean: s2 = ||a - o_hat|| / sqrt(d)
                s2 = c["tok"][b, h, k * T:(k + 1) * T, 0].view(np.float16).astype(np.float64)
                n2 = np.linalg.norm(ab[b, h, k] - oh[None, :].astype(np.float64), axis=-1)
                assert np.all(np.abs(s2 - n2 / sd) <= 1e-3 * n2 / sd + 1e-6)


def test_dq_reconstruction_bound_and_no_dq_unchanged():
    d = 128
    K = _data(5)
    x = K.astype(np.float64)
    base = oracle.Cfg(d, 4, oracle.NSN | oracle.PER_CHANNEL | oracle.HADAMARD)
    dq = oracle.Cfg(d, 4, base.flags | DQ)
    cb, cd = oracle.quantize(base, f16bits(K)), oracle.quantize(dq, f16bits(K))
    # the codes' scales and the s2 of the non-DQ path are unaffected by the
    # flag only through o_hat; with o exactly representable both would agree,
    # here the DQ error is bounded by the side parameters' quantization steps
    xb, _ = oracle.dequantize(base, cb, 0, 256)
    xd, bad = oracle.dequantize(dq, cd, 0, 256)
    assert bad == 0
    rel_b = np.linalg.norm(xb - x) / np.linalg.norm(x)
    rel_d = np.linalg.norm(xd - x) / np.linalg.norm(x)
    assert rel_b < rel_d < 0.2
    # per token: x_hat = s1_hat (...) so the error is at most the s1 step plus the base error
    for k in range(2):
        rec = cd["off"][0, 0, k].view(np.uint8)
        _, s1h = oracle.dq_decode(rec, d)
        st = rec[d // 2 + T // 2 + 4: d // 2 + T // 2 + 6].view(np.float16).astype(np.float64)[0]
        tokn = np.linalg.norm(x[0, 0, k * T:(k + 1) * T], axis=-1)
        err = np.linalg.norm(xd[0, 0, k * T:(k + 1) * T] - x[0, 0, k * T:(k + 1) * T], axis=-1)
        # ||x_hat - x|| <= |s1_hat - s1| sqrt(d) (1 + rel) + s1 * (base error per token)
        assert np.all(err <= (0.5 * st * math.sqrt(d)) * 1.3 + 0.25 * tokn)
