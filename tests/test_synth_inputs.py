"""The synthetic input recipe: unit-norm centers, keys 8 * (c_j + 0.3 * N(0, I)) with j
uniform, values and queries N(0, 1), all rounded to bf16; seeded and deterministic. The
torch generator (used for units no check reads) follows the same distribution."""
import numpy as np
import torch

import synth_inputs as si

D = 128


def test_centers_are_unit_vectors_and_deterministic():
    c = si.centers(3, 7, 50)
    np.testing.assert_allclose(np.linalg.norm(c, axis=1), 1.0, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(c, si.centers(3, 7, 50))
    assert not np.array_equal(c, si.centers(3, 8, 50))


def test_keys_follow_the_mixture():
    n, n_centers = 40_000, 20
    K, V, lab = si.keys_values_labeled(1, 2, n, n_centers)
    k = si.bf16_bits_to_f32(K).astype(np.float64) / 8.0
    resid = k - si.centers(1, 2, n_centers)[lab]
    assert abs(resid.mean()) < 2e-3
    assert abs(resid.std() - 0.3) < 3e-3                    # sigma, plus bf16 rounding
    counts = np.bincount(lab, minlength=n_centers)
    assert counts.min() > 0.9 * n / n_centers and counts.max() < 1.1 * n / n_centers
    v = si.bf16_bits_to_f32(V).astype(np.float64)
    assert abs(v.mean()) < 5e-3 and abs(v.std() - 1.0) < 5e-3
    K2, V2 = si.keys_values(1, 2, n, n_centers)
    np.testing.assert_array_equal(K, K2)
    np.testing.assert_array_equal(V, V2)


def test_queries_and_appended_tokens():
    q = si.bf16_bits_to_f32(si.queries(4, 3, 1, 64, 32)).astype(np.float64)
    assert q.shape == (64, 32, D) and abs(q.std() - 1.0) < 1e-2
    ka, va = si.appended_tokens(4, 5, 20_000, 10)
    k = si.bf16_bits_to_f32(ka).astype(np.float64) / 8.0
    # per-dimension variance of the mixture: the centers' share (1/128) plus sigma^2
    assert abs(k.var() - (1 / D + 0.09)) < 3e-3
    assert abs(si.bf16_bits_to_f32(va).std() - 1.0) < 1e-2


def test_torch_generator_matches_the_recipe():
    k, v = si.keys_values_torch(2, 0, 40_000, 20, "cpu")
    assert k.dtype == torch.bfloat16 and k.shape == (40_000, D)
    kf = k.float().double() / 8.0
    assert abs(float(kf.var()) - (1 / D + 0.09)) < 3e-3
    assert abs(float(v.float().std()) - 1.0) < 1e-2
    k2, _ = si.keys_values_torch(2, 0, 40_000, 20, "cpu")
    assert torch.equal(k, k2)
