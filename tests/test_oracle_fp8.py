"""Pins of the oracle's fp8 copy for far clusters (ClusterKV explainer, section 7: a
lower-precision KV cache for the clusters far from the current query).

Readings (the page gives no format): e4m3 codes with one fp32 scale per row
(scale = max|x| / 448), rounding to nearest with ties to even; the selected clusters at walk
rank >= n_near are attended from that copy. Pins: torch's own float8_e4m3fn conversion on
every representable value, every halfway point and random values; its decoding of all 256
codes; the quantisation error bound; exact round trips of representable rows; and which
rows the attention reads from the copy.
"""
import numpy as np
import torch

import oracle
import synth_inputs as si

D = 128


def _torch_codes(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.float8_e4m3fn) \
        .view(torch.uint8).numpy()


def _grid() -> np.ndarray:
    """Every finite e4m3 value, as float32, ascending."""
    v = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn) \
        .to(torch.float32).numpy()
    v = v[np.isfinite(v)]
    return np.unique(v)


def test_encoding_matches_torch_on_grid_halfway_points_and_random_values():
    g = _grid()
    assert g.min() == -448 and g.max() == 448
    pos = g[g >= 0]
    half = (pos[:-1].astype(np.float64) + pos[1:]) / 2  # exact in float32
    rng = np.random.default_rng(0)
    mag = np.exp2(rng.uniform(-12, np.log2(448), 200_000))
    vals = np.concatenate([g, half, -half, mag * rng.choice([-1, 1], mag.size), [0.0, -0.0]])
    vals = vals.astype(np.float32)
    vals = vals[np.abs(vals) <= 448]
    np.testing.assert_array_equal(oracle.e4m3_from_f32(vals), _torch_codes(vals))


def test_decoding_of_every_code_matches_torch():
    want = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn) \
        .to(torch.float64).numpy()
    got = oracle.e4m3_to_f64(np.arange(256))
    np.testing.assert_array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    np.testing.assert_array_equal(got[ok], want[ok])


def test_out_of_range_saturates_to_448():
    codes = oracle.e4m3_from_f32(np.array([470.0, 1e6, -3e38, 464.0], np.float32))
    np.testing.assert_array_equal(codes, [0x7E, 0x7E, 0xFE, 0x7E])


def test_row_quantisation_error_bound():
    K, _ = si.keys_values(1, 0, 600, 8)
    codes, scales = oracle.quantize_rows_e4m3(K)
    x = oracle.bf16_to_f64(K)
    xh = oracle.e4m3_to_f64(codes) * scales[:, None].astype(np.float64)
    # half a step of a 3-bit significand (2^-4 relative), or half the subnormal step
    bound = np.maximum(np.abs(x) * 2.0 ** -4, scales[:, None] * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(np.abs(xh - x) <= bound)
    # the largest magnitude of every row maps to +-448
    amax = np.argmax(np.abs(x), axis=1)
    assert np.all(np.abs(oracle.e4m3_to_f64(codes[np.arange(600), amax])) == 448)
    np.testing.assert_array_equal(scales, (np.abs(x).max(axis=1).astype(np.float32) / np.float32(448)))


def test_zero_row_and_exactly_representable_rows():
    g = _grid()
    rng = np.random.default_rng(3)
    rows = []
    for k in (-3, 0, 2):
        r = rng.choice(g, D).astype(np.float64)
        r[5] = 448.0
        rows.append(r * 2.0 ** k)
    rows.append(np.zeros(D))
    bits = si.to_bf16_bits(np.array(rows, np.float32))
    assert np.array_equal(oracle.bf16_to_f64(bits), np.array(rows))  # bf16 holds them exactly
    codes, scales = oracle.quantize_rows_e4m3(bits)
    np.testing.assert_array_equal(scales, [2.0 ** -3, 1.0, 4.0, 0.0])
    xh = oracle.e4m3_to_f64(codes) * scales[:, None].astype(np.float64)
    np.testing.assert_array_equal(xh, np.array(rows))
    assert not codes[3].any()


def _store(seed=2, n=1500, C=12):
    K, V = si.keys_values(seed, 0, n, 10)
    st, _ = oracle.prefill_unit(K, V, C, oracle.stream_key(seed, 0, 0), iters=5)
    return st


def test_mixed_attention_reads_only_far_clusters_from_the_copy():
    st = _store()
    q = si.queries(2, 0, 0, 1, 4)[0]
    sel = oracle.select(st, q, 700)
    k8, ks = oracle.quantize_rows_e4m3(st.kp)
    v8, vs = oracle.quantize_rows_e4m3(st.vp)
    base = oracle.attend(st, q, sel)
    # n_near past every cluster: nothing is read from the copy
    np.testing.assert_array_equal(oracle.attend_mixed(st, q, sel, st.C, k8, ks, v8, vs), base)
    rank = oracle.walk_rank(st, sel)
    n_near = 2
    mixed = oracle.attend_mixed(st, q, sel, n_near, k8, ks, v8, vs)
    assert np.abs(mixed - base).max() > 0
    # destroying the copy of the near clusters' rows changes nothing
    near_rows = np.concatenate([np.arange(st.offsets[c], st.offsets[c + 1])
                                for c in range(st.C) if rank[c] < n_near])
    k8b, v8b = k8.copy(), v8.copy()
    k8b[near_rows] = 0x7E
    v8b[near_rows] = 0x7E
    np.testing.assert_array_equal(oracle.attend_mixed(st, q, sel, n_near, k8b, ks, v8b, vs), mixed)
    # the first far cluster (rank == n_near) is selected, and both its K and its V copy are read
    far = [c for c in range(st.C) if rank[c] == n_near][0]
    lo, hi = st.offsets[far], st.offsets[far + 1]
    assert np.isin(st.ids[lo:hi], sel.ids).any()
    k8c, v8c = k8.copy(), v8.copy()
    k8c[lo:hi] = 0
    v8c[lo:hi] = 0
    assert np.abs(oracle.attend_mixed(st, q, sel, n_near, k8c, ks, v8, vs) - mixed).max() > 1e-6
    assert np.abs(oracle.attend_mixed(st, q, sel, n_near, k8, ks, v8c, vs) - mixed).max() > 1e-6


def test_mixed_attention_is_exact_on_representable_rows():
    st = _store(5)
    g = _grid()
    rng = np.random.default_rng(5)
    rows = rng.choice(g[np.abs(g) <= 14], (st.m, D)).astype(np.float64)
    rows[:, 0] = 14.0  # every row's largest magnitude: 14 / 32 / 448 = 2^-10 exactly
    bits = si.to_bf16_bits((rows / 32).astype(np.float32))
    st2 = oracle.Store(st.sp_k, st.sp_v, bits, bits.copy(), st.ids, st.offsets, st.mu)
    q = si.queries(5, 0, 0, 1, 4)[0]
    sel = oracle.select(st2, q, 900)
    k8, ks = oracle.quantize_rows_e4m3(st2.kp)
    np.testing.assert_array_equal(oracle.attend_mixed(st2, q, sel, 0, k8, ks, k8, ks),
                                  oracle.attend(st2, q, sel))
