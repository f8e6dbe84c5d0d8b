"""Seeded synthetic workloads: router top-K ids, gate weights and bf16 rows.

This module only draws inputs; it holds none of the dispatch/combine
arithmetic.  Both the device path and the CPU oracle are fed from it.

Recipe (stand-ins for the serving traces the source pages measure on, which
are not available here):

* A token's router logits are ``z[e] = noise + bias[e]``, where ``bias[e]``
  is the log of an expert-popularity law.  ``ids`` are the top-K of ``z``,
  in descending order of ``z`` (ties have probability zero with float64
  noise).  ``w`` is the softmax over the K selected logits, computed in
  float64 and stored as float32, so it sums to 1 within fp32 rounding.
* The noise is N(0,1) for ``tiny``, whose description fixes it.  For the
  others, whose descriptions give the experts' popularity, it is standard
  Gumbel: the top-K of log-popularity plus Gumbel noise draws K distinct
  experts in proportion to their popularity (sampling without
  replacement), so "popularity" is read as the selection probability.
* ``hidden`` and independent expert outputs ``y`` are N(0,1) rounded to bf16.
* Every draw uses numpy PCG64 seeded by ``SeedSequence([seed, config, step,
  stream])``, so each tensor is reproducible on its own.

The five named workloads:

* ``tiny``   P=4  E=16  K=2 S=64    H=128  R=1, Zipf s=1.0, identity ranking.
* ``mid``    P=8  E=64  K=6 S=4096  H=2048 R=2, Zipf s=1.2, ranking permuted
  per seed, C=0.1.
* ``hot``    P=8  E=384 K=8 S=8192  H=7168 R=2; popularity ranks 5..384
  follow Zipf s=0.8 and the 4 hottest experts share one level, log p_5 +
  delta with delta >= 0, found by bisection on a seeded calibration draw so
  they take 13% (+-0.5%) of all assignments (the hot-expert share ISER-MoE
  reports under "Key Observations"); the shape is the MoonEP benchmark
  default S=8192, E=384, H=7168, K=8, EP=8.
* ``hier``   P=32 (4 nodes x 8 GPUs) E=256 K=8 S=2048 H=7168 R=2, Zipf
  s=1.1, C=0.1, two-level locality cost.
* ``drift``  P=8 E=384 K=8 S=16384 H=7168 R=2, 64 steps; log-popularity
  starts at log Zipf(1.0) and takes a Gaussian random walk, sigma=0.15 per
  step per expert.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from functools import lru_cache

import numpy as np

STREAM_IDS, STREAM_HIDDEN, STREAM_Y, STREAM_PERM, STREAM_CAL, STREAM_WALK = range(6)


@dataclass(frozen=True)
class Workload:
    name: str
    index: int           # workload number used in the seed sequence
    P: int
    E: int
    K: int
    S: int
    H: int
    R: int
    C: float = 0.0
    gpus_per_node: int = 1
    zipf_s: float = 1.0
    permute: bool = False
    hot_share: float | None = None   # target share of the 4 hottest experts
    hot_zipf_s: float = 0.8
    steps: int = 1
    walk_sigma: float = 0.0
    noise: str = "gumbel"            # "normal" or "gumbel" logit noise

    @property
    def N(self) -> int:
        return self.P * self.S * self.K

    @property
    def tokens(self) -> int:
        return self.P * self.S

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, P=4, E=16, K=2, S=64, H=128, R=1, zipf_s=1.0,
                     noise="normal"),
    "mid": Workload("mid", 2, P=8, E=64, K=6, S=4096, H=2048, R=2, C=0.1, zipf_s=1.2,
                    permute=True),
    "hot": Workload("hot", 3, P=8, E=384, K=8, S=8192, H=7168, R=2, hot_share=0.13,
                    hot_zipf_s=0.8),
    "hier": Workload("hier", 4, P=32, E=256, K=8, S=2048, H=7168, R=2, C=0.1,
                     gpus_per_node=8, zipf_s=1.1),
    "drift": Workload("drift", 5, P=8, E=384, K=8, S=16384, H=7168, R=2, zipf_s=1.0,
                      steps=64, walk_sigma=0.15),
}


def rng(wl: Workload, seed: int, step: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(
        [seed, wl.index, step, stream])))


def zipf_log_bias(E: int, s: float) -> np.ndarray:
    """log p_r with p_r proportional to 1/r^s, rank r = 1..E (rank 1 hottest)."""
    r = np.arange(1, E + 1, dtype=np.float64)
    p = r ** (-s)
    return np.log(p / p.sum())


def _top_k(z: np.ndarray, K: int) -> tuple[np.ndarray, np.ndarray]:
    """Top-K indices of each row of z (descending z) and their softmax."""
    part = np.argpartition(-z, K - 1, axis=1)[:, :K]
    zs = np.take_along_axis(z, part, axis=1)
    order = np.lexsort((part, -zs), axis=1)  # descending z, ties to lower id
    ids = np.take_along_axis(part, order, axis=1)
    zk = np.take_along_axis(zs, order, axis=1)
    ex = np.exp(zk - zk[:, :1])
    w = ex / ex.sum(axis=1, keepdims=True)
    return ids.astype(np.int32), w.astype(np.float32)


def _noise(g: np.random.Generator, kind: str, shape) -> np.ndarray:
    return g.gumbel(size=shape) if kind == "gumbel" else g.standard_normal(shape)


def _hot_share(noise: np.ndarray, bias: np.ndarray, K: int, hot: np.ndarray) -> float:
    ids, _ = _top_k(noise + bias[None, :], K)
    return float(np.isin(ids, hot).mean())


def _hot_bias(E: int, s: float, delta: float) -> np.ndarray:
    b = zipf_log_bias(E, s)
    b[:4] = b[4] + delta
    return b


@lru_cache(maxsize=None)
def _hot_delta(wl_index: int, E: int, K: int, s: float, share: float, kind: str,
               seed: int) -> float:
    """Level delta (above the 5th expert's) of the 4 hottest experts that
    gives them ``share`` of the top-K assignments on a seeded calibration draw
    of 8192 tokens (bisection; the share grows with delta)."""
    cal = np.random.Generator(np.random.PCG64(np.random.SeedSequence(
        [seed, wl_index, 0, STREAM_CAL])))
    noise = _noise(cal, kind, (8192, E))
    hot = np.arange(4)
    lo, hi = 0.0, 12.0
    for _ in range(50):
        mid = 0.5 * (lo + hi)
        if _hot_share(noise, _hot_bias(E, s, mid), K, hot) < share:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def expert_bias(wl: Workload, seed: int, step: int = 0) -> np.ndarray:
    """Per-expert logit bias of a workload at a step (expert ids, not ranks)."""
    E = wl.E
    if wl.hot_share is not None:
        b = _hot_bias(E, wl.hot_zipf_s, _hot_delta(wl.index, E, wl.K, wl.hot_zipf_s,
                                                   wl.hot_share, wl.noise, seed))
    else:
        b = zipf_log_bias(E, wl.zipf_s)
    if wl.walk_sigma > 0 and step > 0:
        walk = rng(wl, seed, 0, STREAM_WALK).standard_normal((step, E))
        b = b + wl.walk_sigma * walk.sum(axis=0)
    if wl.permute:
        perm = rng(wl, seed, 0, STREAM_PERM).permutation(E)
        out = np.empty_like(b)
        out[perm] = b       # expert perm[r] gets popularity rank r
        b = out
    return b


def routing(wl: Workload, seed: int = 0, step: int = 0) -> tuple[np.ndarray, np.ndarray]:
    """(ids int32 [P,S,K], w float32 [P,S,K]) for one invocation."""
    g = rng(wl, seed, step, STREAM_IDS)
    bias = expert_bias(wl, seed, step)
    ids = np.empty((wl.P, wl.S, wl.K), np.int32)
    w = np.empty((wl.P, wl.S, wl.K), np.float32)
    for i in range(wl.P):
        z = _noise(g, wl.noise, (wl.S, wl.E)) + bias[None, :]
        if wl.S:
            ids[i], w[i] = _top_k(z, wl.K)
    return ids, w


def _normal_bf16_bits(g: np.random.Generator, shape) -> np.ndarray:
    """N(0,1) samples rounded to bf16 (nearest, ties to even), as uint16 bits.
    Rounding uses torch's CPU conversion; this is input preparation only."""
    import torch
    x = torch.from_numpy(g.standard_normal(shape, dtype=np.float32))
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def hidden_bits(wl: Workload, seed: int = 0, step: int = 0) -> np.ndarray:
    """hidden [P,S,H] as bf16 bit patterns (uint16)."""
    return _normal_bf16_bits(rng(wl, seed, step, STREAM_HIDDEN), (wl.P, wl.S, wl.H))


def y_bits(wl: Workload, rows: int, seed: int = 0, step: int = 0) -> np.ndarray:
    """Independent expert outputs [rows,H] as bf16 bit patterns (uint16)."""
    return _normal_bf16_bits(rng(wl, seed, step, STREAM_Y), (rows, wl.H))


def hidden_device(wl: Workload, seed: int, step: int, device, stream: int = STREAM_HIDDEN):
    """A [P,S,H] bf16 tensor of N(0,1) rows drawn on the device by torch's
    seeded generator: for the large workloads, where host generation is slow.
    Its rows can be copied back for sampled checks."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(int(np.random.SeedSequence([seed, wl.index, step, stream]).generate_state(1)[0]))
    return torch.randn((wl.P, wl.S, wl.H), generator=gen, device=device,
                       dtype=torch.float32).to(torch.bfloat16)
