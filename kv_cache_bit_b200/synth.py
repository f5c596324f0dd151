"""Seeded synthetic K/V/Q generators shaped like the pages' workloads.

This module holds no arithmetic of the quantization method: it only draws
random numbers.  Both the CUDA path and the CPU oracle are fed from here.

Recipe (numpy ``default_rng``; float32 draws, fp16 round-to-nearest-even last):
  base     z ~ N(0, 1)
  offsets  z += mu[h, c], mu ~ N(0, mean_sd)          (throughput workload)
  spikes   z += amp * t3 on Bernoulli(p) entries       (long-context workload)
  norms    z *= r[h, t], r ~ lognormal(0, sigma_n)     (token-norm spread)
  outliers K only, channels drawn without replacement once per workload and
           shared by all heads: either z[..., c] *= factor, or
           z[..., c] = clip(N(0, sd), -clip, clip)
  queries  q ~ N(0, 1)
Sub-streams: rng([seed, kind, b]) with kind K=1, V=2, Q=3, channel choice=4,
means=7; one stream per batch row, so large workloads are drawn in slices.

The outlier statistics follow the "nsep+pchan" post (Qwen2-7B layer 0 has 8
channels with absmax 167; outlier channels 8-100x the mean; per-token norm
spread 2-5x); the shapes follow the models it names (Qwen2-7B 28/4 heads,
Pythia-6.9B 32 heads, head dim 128).  No public dataset is used.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional, Sequence

import numpy as np


@dataclass(frozen=True)
class Outliers:
    kind: str                 # "mul" or "replace"
    count: int
    factors: Sequence[float] = ()
    sd: float = 0.0
    clip: float = 0.0


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    S: int
    sigma_n: Optional[float] = None
    mean_sd: Optional[float] = None
    spike_p: float = 0.0
    spike_amp: float = 0.0
    k_outliers: Optional[Outliers] = None
    v_outliers: Optional[Outliers] = None
    stream: int = 0                       # tokens appended one per decode step
    modes: Sequence[tuple] = field(default_factory=tuple)   # (mode name, bits)
    seed: int = 0

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", B=1, Hq=8, Hkv=8, d=64, S=256, sigma_n=0.5,
                     k_outliers=Outliers("mul", 4, factors=(50.0,) * 4),
                     modes=(("nsep+pchan", 4),)),
    "qwen2-7b-gqa": Workload("qwen2-7b-gqa", B=8, Hq=28, Hkv=4, d=128, S=4096, sigma_n=0.6,
                             k_outliers=Outliers("replace", 8, sd=60.0, clip=167.0),
                             modes=(("nsep+pchan", 4),)),
    "pythia-6.9b-mha": Workload("pythia-6.9b-mha", B=16, Hq=32, Hkv=32, d=128, S=2048,
                                sigma_n=0.7,
                                k_outliers=Outliers("mul", 6, factors=(20., 36., 52., 68., 84., 100.)),
                                modes=(("nsep+pchan", 4), ("nsep+pchan", 3), ("naive", 4))),
    "llama-long-ctx": Workload("llama-long-ctx", B=4, Hq=32, Hkv=8, d=128, S=32768,
                               spike_p=0.01, spike_amp=10.0,
                               k_outliers=Outliers("mul", 8, factors=(50.0,) * 8),
                               modes=(("rht+nsep+pchan", 4),)),
    "throughput": Workload("throughput", B=64, Hq=32, Hkv=8, d=128, S=8192, sigma_n=0.6,
                           mean_sd=3.0, stream=256,
                           modes=(("nsn+hadamard", 4), ("nsn+hadamard", 2))),
}


def _rng(seed: int, kind: int, b: int = 0) -> np.random.Generator:
    return np.random.default_rng([seed, kind, b])


def outlier_channels(w: Workload) -> np.ndarray:
    if w.k_outliers is None:
        return np.zeros(0, np.int64)
    return np.sort(_rng(w.seed, 4).choice(w.d, size=w.k_outliers.count, replace=False))


def channel_means(w: Workload) -> Optional[np.ndarray]:
    if not w.mean_sd:
        return None
    return _rng(w.seed, 7).normal(0.0, w.mean_sd, size=(w.Hkv, w.d)).astype(np.float32)


def _draw(w: Workload, kind: int, b: int, S: int, outl: Optional[Outliers],
          chans: np.ndarray, mu: Optional[np.ndarray], t_offset: int = 0) -> np.ndarray:
    """One batch row [Hkv, S, d] as float16."""
    r = _rng(w.seed, kind, b)
    if t_offset:
        # tokens past the prefill come from their own stream so that the
        # prefill draw does not depend on how many tokens are streamed later
        r = _rng(w.seed, kind + 100, b)
    z = r.standard_normal((w.Hkv, S, w.d), dtype=np.float32)
    if mu is not None:
        z += mu[:, None, :]
    if w.spike_p > 0:
        mask = r.random((w.Hkv, S, w.d), dtype=np.float32) < w.spike_p
        z += (w.spike_amp * r.standard_t(3, size=z.shape)).astype(np.float32) * mask
    if w.sigma_n:
        z *= r.lognormal(0.0, w.sigma_n, size=(w.Hkv, S, 1)).astype(np.float32)
    if outl is not None and len(chans):
        if outl.kind == "mul":
            z[..., chans] *= np.asarray(outl.factors, np.float32)
        else:
            rep = r.normal(0.0, outl.sd, size=(w.Hkv, S, len(chans))).astype(np.float32)
            z[..., chans] = np.clip(rep, -outl.clip, outl.clip)
    return z.astype(np.float16)


def kv(w: Workload, S: Optional[int] = None, t_offset: int = 0):
    """(K, V) as float16 [B, Hkv, S, d]."""
    S = w.S if S is None else S
    chans = outlier_channels(w)
    mu = channel_means(w)
    K = np.empty((w.B, w.Hkv, S, w.d), np.float16)
    V = np.empty_like(K)
    for b in range(w.B):
        K[b] = _draw(w, 1, b, S, w.k_outliers, chans, mu, t_offset)
        V[b] = _draw(w, 2, b, S, w.v_outliers, chans, mu, t_offset)
    return K, V


def stream_tokens(w: Workload, n: Optional[int] = None):
    """(K, V) float16 [n, B, Hkv, d]: the tokens appended after the prefill,
    one per decode step."""
    n = w.stream if n is None else n
    K, V = kv(w, S=n, t_offset=1)
    return np.ascontiguousarray(K.transpose(2, 0, 1, 3)), np.ascontiguousarray(V.transpose(2, 0, 1, 3))


def queries(w: Workload, steps: int = 1) -> np.ndarray:
    """float16 [steps, B, Hq, d] (steps == 1 squeezes to [B, Hq, d])."""
    q = _rng(w.seed, 3).standard_normal((steps, w.B, w.Hq, w.d), dtype=np.float32).astype(np.float16)
    return q[0] if steps == 1 else q


# mode name -> (flag names, seeded random signs?).  Each side maps the flag
# names onto its own constants.
MODES = {
    "nsep+pchan": (("NORM_SEP", "PER_CHANNEL"), False),
    "naive": ((), False),
    "rht+nsep+pchan": (("NORM_SEP", "PER_CHANNEL", "HADAMARD"), True),
    "nsn+hadamard": (("NSN", "PER_CHANNEL", "HADAMARD"), False),
    "nsn": (("NSN", "PER_CHANNEL"), False),
    "nsn+hadamard+dq": (("NSN", "PER_CHANNEL", "HADAMARD", "DQ"), False),
    "nsn+dq": (("NSN", "PER_CHANNEL", "DQ"), False),
    "nsep-only": (("NORM_SEP",), False),
    "pchan-only": (("PER_CHANNEL",), False),
}

SIGN_SEED = 0x5EED  # seed of the randomized-Hadamard signs for seeded modes
