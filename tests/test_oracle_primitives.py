"""Pins of the oracle's primitives: the seeded init generator and the bf16 rounding.

Each test checks the oracle against something outside it: a published test vector, a
library routine (torch's float32->bf16 conversion), a closed form, or a statistical
property of the definition.
"""
import collections
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_splitmix_golden():
    out = {}
    with open(os.path.join(GOLDEN, "splitmix64.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            seed, vals = line.split(":")
            out[int(seed)] = [int(v) for v in vals.split()]
    return out


def test_splitmix64_published_vectors():
    for seed, expected in _read_splitmix_golden().items():
        assert oracle.splitmix64(seed, len(expected)) == expected


def test_bounded_closed_forms():
    # multiply-shift: floor((x >> 32) * r / 2^32)
    assert oracle.bounded(1 << 63, 10) == 5
    assert oracle.bounded(0, 1000) == 0
    assert oracle.bounded(2**64 - 1, 1) == 0
    for r in (1, 2, 7, 320, 32752, 2**31):
        assert oracle.bounded(2**64 - 1, r) == r - 1
    rng = np.random.default_rng(0)
    for x in rng.integers(0, 2**63, size=200, dtype=np.int64):
        x = int(x) * 2 + 1
        for r in (3, 400, 131056):
            assert oracle.bounded(x, r) == ((x >> 32) * r) >> 32


def test_stream_key_distinct_per_unit_and_window():
    keys = {oracle.stream_key(7, u, w) for u in range(64) for w in range(8)}
    assert len(keys) == 64 * 8
    assert oracle.stream_key(7, 0, 0) == 7


def test_init_indices_are_distinct_and_in_range():
    for m, c in [(1, 1), (5, 5), (100, 7), (32752, 400), (131056, 1600)]:
        idx = oracle.init_indices(m, c, oracle.stream_key(3, 1, 0))
        assert idx.shape == (c,)
        assert idx.min() >= 0 and idx.max() < m
        assert len(set(idx.tolist())) == c


def test_init_indices_full_shuffle_is_uniform():
    # Fisher-Yates with an (almost) unbiased bounded draw: every permutation of 4 items
    # is equally likely. 24 cells and 24000 draws give a chi-square with 23 dof.
    counts = collections.Counter(tuple(oracle.init_indices(4, 4, s).tolist()) for s in range(24000))
    assert set(counts) == set(itertools.permutations(range(4)))
    chi2 = sum((v - 1000) ** 2 / 1000 for v in counts.values())
    assert chi2 < 60.0  # p < 1e-4 for 23 dof


def test_init_first_draw_matches_splitmix_definition():
    # The first chosen index is bounded(first SplitMix64 output, m).
    for seed in (0, 1, 99):
        for m in (10, 320, 32752):
            first = oracle.splitmix64(seed, 1)[0]
            assert oracle.init_indices(m, 1, seed)[0] == oracle.bounded(first, m)


def _torch_bf16(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def test_bf16_rounding_matches_torch_on_float32_values():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, 1e-40, -1e-40, 1e-45, 65504.0]),
    ]).astype(np.float32)
    # exact halfway cases between neighbouring bf16 values (ties go to even)
    base = (rng.integers(0, 2**15, 5000).astype(np.uint32) << 16)
    halfway = (base | 0x8000).view(np.float32)
    x = np.concatenate([x, halfway[np.isfinite(halfway)]])
    got = oracle.bf16_from_f64(x.astype(np.float64))
    np.testing.assert_array_equal(got, _torch_bf16(x))


def test_bf16_roundtrip_and_known_patterns():
    assert oracle.bf16_from_f64([1.0])[0] == 0x3F80
    assert oracle.bf16_from_f64([1.0 + 2**-8])[0] == 0x3F80        # tie -> even (down)
    assert oracle.bf16_from_f64([1.0 + 3 * 2**-8])[0] == 0x3F82    # tie -> even (up)
    assert oracle.bf16_from_f64([-2.5])[0] == 0xC020
    b = np.arange(0, 2**16, 7, dtype=np.uint16)
    b = b[((b >> 7) & 0xFF) != 0xFF]  # drop inf/nan patterns
    np.testing.assert_array_equal(oracle.bf16_from_f64(oracle.bf16_to_f64(b)), b)


def test_normalize_unit_norm_and_zero():
    rng = np.random.default_rng(2)
    mu = rng.standard_normal((50, 128)) * 5.0
    mu[7] = 0.0
    mh = oracle.bf16_to_f64(oracle.normalize(mu))
    norms = np.linalg.norm(mh, axis=1)
    assert np.all(mh[7] == 0.0)
    nz = np.delete(np.arange(50), 7)
    # each component is within half a bf16 ulp (2^-9 relative) of the exact unit vector
    exact = mu[nz] / np.linalg.norm(mu[nz], axis=1, keepdims=True)
    assert np.all(np.abs(mh[nz] - exact) <= np.abs(exact) * 2.0**-8 + 1e-30)
    assert np.all(np.abs(norms[nz] - 1.0) < 1e-2)
    # direction, not magnitude: scaling a centroid by 37 leaves mu_hat unchanged
    np.testing.assert_array_equal(oracle.normalize(mu * 37.0)[nz], oracle.normalize(mu)[nz])


def test_bf16_to_f64_is_exact_widening():
    b = np.array([0x3F80, 0xC020, 0x0001, 0x7F7F], np.uint16)
    v = oracle.bf16_to_f64(b)
    assert v[0] == 1.0 and v[1] == -2.5
    assert v[2] == 2.0**-133
    assert v[3] == (2 - 2.0**-7) * 2.0**127
    assert math.isclose(v[3], 3.3895313892515355e38)
