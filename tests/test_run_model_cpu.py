"""The decode kernel's run decomposition, restated in Python and checked exhaustively.

The decode copies a chunk [c0, c1) of selection positions into the shared-memory ring run by
run: the thread at a run's first position copies the run's rows with one bulk copy. The
positions are the sinks, the pending tokens (a ring of `pring` rows read from `pstart`), the
whole clusters in walk order (prefixes `pre`, store offsets `off`), then partial rows. This
model restates how each position decides whether a run starts there and where it ends, and
checks on random layouts (empty clusters, pending runs that wrap, chunk boundaries anywhere)
that the runs tile the chunk, that each run reads consecutive store rows, and that the bytes
a chunk announces equal one K and one V row per position.
"""
import numpy as np
import pytest


def position_source(idx, n_sink, pstart, pring, base_w, base_p, pre, off, prow, p_lo):
    """('sp', row) for a sink or pending token, ('kp', row) for a clustered row."""
    if idx < n_sink:
        return "sp", idx
    if idx < base_w:
        return "sp", n_sink + (pstart + idx - n_sink) % pring
    if idx < base_p:
        x = idx - base_w
        k = max(i for i in range(len(pre) - 1) if pre[i] <= x)  # last prefix <= x
        return "kp", off[k] + (x - pre[k])
    return "kp", prow[idx - base_p - p_lo]


def run_at(idx, c0, c1, n_sink, pstart, pring, base_w, base_p, pre):
    """(starts, run_end) as the kernel computes them for position idx of chunk [c0, c1)."""
    if idx < n_sink:
        return idx == c0 or idx == 0, min(c1, n_sink)
    if idx < base_w:
        i = idx - n_sink
        q = (pstart + i) % pring
        return idx == c0 or i == 0 or q == 0, min(c1, base_w, idx + (pring - q))
    if idx < base_p:
        x = idx - base_w
        k = max(i for i in range(len(pre) - 1) if pre[i] <= x)
        return idx == c0 or x == pre[k], min(c1, base_w + pre[k + 1])
    return True, idx + 1


@pytest.mark.parametrize("seed", range(60))
def test_runs_tile_each_chunk_and_read_consecutive_rows(seed):
    rng = np.random.default_rng(seed)
    n_sink = int(rng.integers(0, 20))
    pring = int(rng.integers(1, 40))
    pending = int(rng.integers(0, pring + 1))
    pstart = int(rng.integers(0, pring))
    sizes = rng.integers(0, 30, size=int(rng.integers(1, 12)))
    sizes[rng.random(len(sizes)) < 0.2] = 0  # empty clusters inside the walk
    pre = np.concatenate([[0], np.cumsum(sizes)]).astype(int)
    off = rng.permutation(len(sizes)) * 1000  # walk order is not store order
    n_part = int(rng.integers(0, 12))
    prow = rng.integers(0, 5000, size=n_part)
    base_w = n_sink + pending
    base_p = base_w + int(pre[-1])
    T = base_p + n_part
    lo = int(rng.integers(0, max(T, 1)))
    chunk = int(rng.integers(1, 40))
    for c0 in range(lo, T, chunk):
        c1 = min(c0 + chunk, T)
        covered = []
        announced = 0
        for idx in range(c0, c1):
            starts, end = run_at(idx, c0, c1, n_sink, pstart, pring, base_w, base_p, pre)
            assert idx < end <= c1
            if not starts:
                continue
            announced += (end - idx) * 512  # K and V rows of 256 bytes
            kind0, row0 = position_source(idx, n_sink, pstart, pring, base_w, base_p, pre, off, prow, 0)
            for j, pos in enumerate(range(idx, end)):
                kind, row = position_source(pos, n_sink, pstart, pring, base_w, base_p, pre, off, prow, 0)
                assert (kind, row) == (kind0, row0 + j), (idx, pos)  # one bulk copy reads it
                covered.append(pos)
        assert sorted(covered) == list(range(c0, c1))  # every position once
        assert announced == (c1 - c0) * 512
