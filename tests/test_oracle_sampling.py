"""Pins for the sampling oracle (oracle.sampling): the Philox generator against
its published known-answer vectors, the sampling definition against hand
values, a fine-grid measure check and invariances."""
import math

import numpy as np
import pytest

from oracle import sampling as SM


# Known-answer vectors of Philox4x32-10 published with the generator's
# reference implementation (counter, key -> output).
KAT = [
    ((0, 0, 0, 0), (0, 0), (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
    ((0xFFFFFFFF,) * 4, (0xFFFFFFFF,) * 2, (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
    ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
     (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
]


@pytest.mark.parametrize("ctr,key,want", KAT)
def test_philox_known_answers(ctr, key, want):
    assert SM.philox4x32(ctr, key) == want


def test_step_uniform_range_and_determinism():
    us = [SM.step_uniform(7, s) for s in range(2000)]
    assert all(0.0 <= u < 1.0 for u in us)
    assert all(u * 2 ** 24 == int(u * 2 ** 24) for u in us)      # multiples of 2^-24
    assert us == [SM.step_uniform(7, s) for s in range(2000)]
    assert len(set(us)) > 1990
    assert abs(np.mean(us) - 0.5) < 0.02
    assert SM.step_uniform(8, 0) != SM.step_uniform(7, 0)


def test_greedy_special_cases():
    lg = np.array([0.1, 2.0, -1.0, 2.0, 0.5])
    assert SM.sample_token(lg, 0.0, 0, 1.0, 0.99) == 1           # T = 0: argmax, lowest index
    for u in (0.0, 0.3, 0.999):
        assert SM.sample_token(lg, 1.3, 1, 1.0, u) == 1          # top-1 = argmax
        assert SM.sample_token(lg, 1.3, 1, 0.2, u) == 1


def test_hand_values_inverse_cdf_and_top_p():
    # probabilities 1/2, 1/4, 1/8, 1/8 at T = 1 (logits are their logs, shifted)
    lg = np.log([0.5, 0.25, 0.125, 0.125]) + 3.0
    cases = [(0.10, 0), (0.49, 0), (0.51, 1), (0.74, 1), (0.76, 2), (0.87, 2), (0.88, 3), (0.999, 3)]
    for u, want in cases:
        assert SM.sample_token(lg, 1.0, 4, 1.0, u) == want, u
    # top-p 0.7 keeps {0, 1} (cumulative 0.5, then 0.75): renormalised 2/3, 1/3
    for u, want in [(0.6, 0), (0.66, 0), (0.67, 1), (0.95, 1)]:
        assert SM.sample_token(lg, 1.0, 4, 0.7, u) == want, u
    # top-k 2 gives the same set; top-k 3 with top-p 0.99 keeps three:
    # renormalised 4/7, 2/7, 1/7
    assert SM.sample_token(lg, 1.0, 2, 1.0, 0.67) == 1
    for u, want in [(0.57, 0), (0.58, 1), (0.85, 1), (0.86, 2)]:
        assert SM.sample_token(lg, 1.0, 3, 0.99, u) == want, u
    # ties keep the lower index first: tokens 2 and 3 tie, 2 comes first
    assert SM.sample_token(lg, 1.0, 3, 1.0, 0.99) == 2


def test_measure_of_each_token_on_a_fine_grid():
    # Over u on a fine grid, each token is picked for a share of the grid equal
    # to its renormalised probability (computed here by a plain listing of the
    # kept set: sort, cut at k, softmax, cut at p).
    rng = np.random.default_rng(5)
    lg = rng.normal(size=40) * 2.0
    T, k, p = 0.7, 12, 0.9
    idx = sorted(range(40), key=lambda i: (-lg[i], i))[:k]
    e = np.array([math.exp((lg[i] - lg[idx[0]]) / T) for i in idx])
    pr = e / e.sum()
    n = 1
    while pr[:n].sum() < p:
        n += 1
    kept = pr[:n] / pr[:n].sum()
    N = 20000
    counts = {}
    for j in range(N):
        t = SM.sample_token(lg, T, k, p, (j + 0.5) / N)
        counts[t] = counts.get(t, 0) + 1
    assert set(counts) == set(idx[:n])
    for i, q in zip(idx[:n], kept):
        assert abs(counts[i] / N - q) <= 1.0 / N + 1e-12


def test_temperature_is_a_logit_scale():
    rng = np.random.default_rng(6)
    lg = rng.normal(size=30)
    for u in np.linspace(0.01, 0.99, 25):
        assert SM.sample_token(lg, 0.8, 10, 0.95, u) == SM.sample_token(2 * lg, 1.6, 10, 0.95, u)


def test_margin_is_distance_to_the_nearest_edge():
    lg = np.log([0.5, 0.25, 0.125, 0.125])
    assert abs(SM.sample_margin(lg, 1.0, 4, 1.0, 0.49) - 0.01) < 1e-12
    assert abs(SM.sample_margin(lg, 1.0, 4, 1.0, 0.8) - 0.05) < 1e-12
