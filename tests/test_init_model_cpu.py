"""The K-means init kernel's parallel form of the seeded Fisher-Yates draw, restated in
Python, equals the oracle's sequential shuffle (init reading of ClusterKV explainer section
3.2: the first C entries of a Fisher-Yates shuffle of 0..m-1 driven by SplitMix64).

The sequential shuffle runs, for i = 0..C-1: j = i + bounded(x_i, m - i); chosen[i] = a[j];
a[j] = a[i] (position i is never read again). The kernel computes every draw target j_i at
once (SplitMix64 is counter-based) and then resolves each chosen[i] without the loop:
* position p >= i changed before step i only as the target of an earlier step; so
  a[p] before step i is the value that position s held just before step s, where s is the
  last step < i whose target is p (prev), or p itself if there is none;
* the value position s held just before step s follows the same rule with the last step
  < s whose target is s (link): a chain of earlier steps that ends at a step whose own
  position was never a target, and whose index is the value.
This model is checked against ``oracle.init_indices`` over many (m, C), including m == C (a
full permutation, where targets collide often) and tiny m. It is a check of the algorithm;
the GPU test of the init stage checks the kernel.
"""
import numpy as np

import oracle

MASK = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15


def _splitmix64_at(key: int, i: int) -> int:
    """Output i of SplitMix64 seeded with key (counter form: state before draw i)."""
    z = (key + (i + 1) * GAMMA) & MASK
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK
    return z ^ (z >> 31)


def parallel_init(m: int, C: int, key: int) -> list:
    target = [i + ((_splitmix64_at(key, i) >> 32) * (m - i) >> 32) for i in range(C)]
    prev, link = [-1] * C, [-1] * C
    for t in range(C):  # one thread per step in the kernel, scanning backwards
        for s in range(t - 1, -1, -1):
            if prev[t] < 0 and target[s] == target[t]:
                prev[t] = s
            if link[t] < 0 and target[s] == t:
                link[t] = s
            if prev[t] >= 0 and link[t] >= 0:
                break
    chosen = []
    for i in range(C):
        x = prev[i]
        if x < 0:
            chosen.append(target[i])
        else:
            while link[x] >= 0:
                x = link[x]
            chosen.append(x)
    return chosen


def test_counter_form_of_splitmix64_matches_the_oracle():
    key = 0x1234_5678_9ABC_DEF0
    assert [_splitmix64_at(key, i) for i in range(6)] == oracle.splitmix64(key, 6)


def test_parallel_init_equals_the_sequential_shuffle():
    rng = np.random.default_rng(1)
    cases = [(1, 1), (2, 2), (3, 1), (5, 5), (32, 32), (40, 32), (64, 63), (320, 4), (300, 300),
             (2032, 32), (1000, 999), (5000, 400)]
    cases += [(int(m), int(rng.integers(1, m + 1))) for m in rng.integers(1, 700, 40)]
    for k, (m, C) in enumerate(cases):
        key = oracle.stream_key(int(rng.integers(0, 2**63)), k, k % 3)
        want = oracle.init_indices(m, C, key).tolist()
        got = parallel_init(m, C, key)
        assert got == want, (m, C)
        assert len(set(got)) == C and all(0 <= g < m for g in got)
