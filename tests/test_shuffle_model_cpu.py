"""The transposed warp reduction used by the decode's centroid scoring, the drift check and
the split's 2-means, simulated lane by lane.

Each of 32 lanes holds partial sums of V values; each exchange step (xor with a lane
distance `half`-multiple) keeps half of the values a lane holds and adds the partner's copy of
the same values, so after log2(V) steps a lane holds one value summed over the lanes that
took part, and the remaining xor steps finish the sum over all 32 lanes. These tests restate
the three kernels' index choices and check which value every lane ends with against direct
sums of the partials.
"""
import numpy as np


def shfl_xor(vals, d):
    """vals[lane] read from lane ^ d, for every lane."""
    return vals[np.arange(32) ^ d]


def reduce_8_over_32(p):
    """Decode scoring: p [32 lanes, 8 values]; lane bits 4, 3, 2 pick the kept half."""
    lane = np.arange(32)
    hA, hB, hC = (lane & 16) != 0, (lane & 8) != 0, (lane & 4) != 0
    q = np.empty((32, 4))
    for i in range(4):
        keep = np.where(hA, p[:, 4 + i], p[:, i])
        give = np.where(hA, p[:, i], p[:, 4 + i])
        q[:, i] = keep + shfl_xor(give, 16)
    r0 = np.where(hB, q[:, 2], q[:, 0]) + shfl_xor(np.where(hB, q[:, 0], q[:, 2]), 8)
    r1 = np.where(hB, q[:, 3], q[:, 1]) + shfl_xor(np.where(hB, q[:, 1], q[:, 3]), 8)
    v = np.where(hC, r1, r0) + shfl_xor(np.where(hC, r0, r1), 4)
    v = v + shfl_xor(v, 2)
    return v + shfl_xor(v, 1)


def reduce_32_over_32(p):
    """Drift check: p [32 lanes, 32 values]; halves 16, 8, 4, 2, 1 in turn."""
    lane = np.arange(32)
    v = p.copy()
    half = 16
    while half >= 1:
        up = (lane & half) != 0
        nv = v.copy()
        for t in range(half):
            keep = np.where(up, v[:, half + t], v[:, t])
            give = np.where(up, v[:, t], v[:, half + t])
            nv[:, t] = keep + shfl_xor(give, half)
        v = nv
        half //= 2
    return v[:, 0]


def reduce_8_split(p):
    """Split 2-means: 8 values, exchanges at lane distances 16, 8, 4, then 2 and 1."""
    lane = np.arange(32)
    v = p.copy()
    half = 4
    while half >= 1:
        up = (lane & (4 * half)) != 0
        nv = v.copy()
        for t in range(half):
            keep = np.where(up, v[:, half + t], v[:, t])
            give = np.where(up, v[:, t], v[:, half + t])
            nv[:, t] = keep + shfl_xor(give, 4 * half)
        v = nv
        half //= 2
    out = v[:, 0] + shfl_xor(v[:, 0], 2)
    return out + shfl_xor(out, 1)


def test_scoring_lane_l_holds_centroid_l_over_4():
    rng = np.random.default_rng(0)
    for _ in range(20):
        p = rng.integers(-1000, 1000, size=(32, 8)).astype(np.float64)  # exact sums
        got = reduce_8_over_32(p)
        want = p.sum(axis=0)
        for lane in range(32):
            assert got[lane] == want[lane >> 2]


def test_drift_lane_l_holds_value_l():
    rng = np.random.default_rng(1)
    for _ in range(20):
        p = rng.integers(-1000, 1000, size=(32, 32)).astype(np.float64)
        got = reduce_32_over_32(p)
        assert np.array_equal(got, p.sum(axis=0))
        # the kernel then pairs value 2 r (k.mu) at even lanes with 2 r + 1 (k.k) one lane up
        kk = shfl_xor(got, 1)
        for r in range(16):
            assert got[2 * r] == p[:, 2 * r].sum() and kk[2 * r] == p[:, 2 * r + 1].sum()


def test_split_lane_8r_and_8r_plus_4_hold_row_r():
    rng = np.random.default_rng(2)
    for _ in range(20):
        p = rng.integers(-1000, 1000, size=(32, 8)).astype(np.float64)
        got = reduce_8_split(p)
        want = p.sum(axis=0)
        for lane in range(32):
            assert got[lane] == want[lane >> 2]
        other = shfl_xor(got, 4)
        for r in range(4):  # lane 8 r: value 2 r (first half), its partner lane 8 r + 4: 2 r + 1
            assert got[8 * r] == want[2 * r] and other[8 * r] == want[2 * r + 1]
