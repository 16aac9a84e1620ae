"""fp64 CPU oracle of in-kernel token sampling (test infrastructure only).

TEST INFRASTRUCTURE, like ``oracle.decoder``: only the tests, ``smoke()`` and
``bench.py``'s CPU legs may import it; the GPU engine shares no code with it.

What it computes. The monokernel of the pages performs the token choice
("sampling") inside the persistent program
("メモリの壁を打破する：標準的なGPUで3,000 tokens/sの推論を実現する", section
"1. The Monokernel Runtime"). The workloads decode greedily, which is the
temperature-0 case; this module defines the stochastic case the engine also
offers. The pages fix none of it, so the definition taken is the common one:

1. temperature T: z_i = logit_i / T (T = 0 means greedy argmax, lowest index
   on ties);
2. top-k (k >= 1): keep the k largest z, ties broken by the lower index;
3. probabilities over the kept set: p_i = exp(z_i - max z) / sum;
4. top-p (0 < p <= 1): in the order of decreasing p (ties: lower index
   first), keep the shortest prefix whose cumulative probability reaches p;
5. renormalise over what is kept and invert the CDF in that same order with
   one uniform u in [0, 1): the first token whose cumulative probability
   exceeds u.

The uniform of decode step s comes from Philox4x32-10 (Salmon, Moraes, Dror
and Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC 2011) with key
(seed low 32 bits, seed high 32 bits) and counter (s, 0, 0, 0): the top 24
bits of the first output word, times 2^-24.
"""
from __future__ import annotations

import math

import numpy as np

MASK32 = 0xFFFFFFFF
# The Philox4x32 round multipliers and the Weyl key increments, as published.
PHILOX_M0, PHILOX_M1 = 0xD2511F53, 0xCD9E8D57
PHILOX_W0, PHILOX_W1 = 0x9E3779B9, 0xBB67AE85


def _mulhilo(a: int, b: int) -> tuple[int, int]:
    p = a * b
    return (p >> 32) & MASK32, p & MASK32


def philox4x32(counter, key, rounds: int = 10) -> tuple[int, int, int, int]:
    """Philox4x32-R on a 4-word counter and a 2-word key (Python ints)."""
    c0, c1, c2, c3 = (int(v) & MASK32 for v in counter)
    k0, k1 = (int(v) & MASK32 for v in key)
    for r in range(rounds):
        if r:
            k0 = (k0 + PHILOX_W0) & MASK32
            k1 = (k1 + PHILOX_W1) & MASK32
        hi0, lo0 = _mulhilo(PHILOX_M0, c0)
        hi1, lo1 = _mulhilo(PHILOX_M1, c2)
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return c0, c1, c2, c3


def step_uniform(seed: int, step: int) -> float:
    """The uniform in [0, 1) of decode step ``step`` (a multiple of 2^-24)."""
    w = philox4x32((step, 0, 0, 0), (seed & MASK32, (seed >> 32) & MASK32))[0]
    return (w >> 8) * 2.0 ** -24


def sample_token(logits, temperature: float, top_k: int, top_p: float, u: float) -> int:
    """The token the definition above picks for uniform ``u``."""
    z = np.asarray(logits, dtype=np.float64)
    if temperature <= 0.0:
        return int(np.flatnonzero(z == z.max())[0])
    z = z / float(temperature)
    order = sorted(range(len(z)), key=lambda i: (-z[i], i))
    if top_k >= 1:
        order = order[:top_k]
    m = z[order[0]]
    w = [math.exp(z[i] - m) for i in order]
    tot = sum(w)
    if top_p < 1.0:
        cum, keep = 0.0, 0
        for x in w:
            cum += x / tot
            keep += 1
            if cum >= top_p:
                break
        order, w = order[:keep], w[:keep]
        tot = sum(w)
    target = u * tot
    cum = 0.0
    for i, x in zip(order, w):
        cum += x
        if cum > target:
            return int(i)
    return int(order[-1])


def sample_margin(logits, temperature: float, top_k: int, top_p: float, u: float) -> float:
    """How far ``u`` lies from the nearest CDF bucket edge, and how far the
    top-p cumulative sum lies from ``top_p`` at the cut, whichever is closer
    (in probability units). A second implementation in other arithmetic may
    pick another token only when this is within its rounding error."""
    z = np.asarray(logits, dtype=np.float64) / float(temperature)
    order = sorted(range(len(z)), key=lambda i: (-z[i], i))
    if top_k >= 1:
        order = order[:top_k]
    m = z[order[0]]
    p = np.array([math.exp(z[i] - m) for i in order])
    p /= p.sum()
    best = 1.0
    if top_p < 1.0:
        c = np.cumsum(p)
        keep = int(np.searchsorted(c, top_p) + 1)
        keep = min(keep, len(p))
        best = min(best, abs(c[keep - 1] - top_p))
        if keep >= 2:
            best = min(best, abs(c[keep - 2] - top_p))
        p = p[:keep] / p[:keep].sum()
    edges = np.cumsum(p)
    return float(min(best, np.min(np.abs(edges - u))))
