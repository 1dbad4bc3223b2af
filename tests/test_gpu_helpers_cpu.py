"""The GPU parity tests' acceptance rules reject planted errors (runs on CPU).

The comparisons in gpu_helpers excuse a disagreement only at a near-tie. Here the device
result is replaced by the oracle's own answer with one planted mistake, and every rule
must reject it, while the exact answer and genuine ties pass.
"""
import numpy as np
import pytest

import oracle
import synth_inputs as si
from gpu_helpers import check_assign, check_decode_unit, check_mu_hat


def _case(budget=400):
    K, V = si.keys_values(12, 3, 1600, 12)
    st, _ = oracle.prefill_unit(K, V, 16, oracle.stream_key(12, 3, 0), iters=4)
    q = si.queries(12, 0, 0, 1, 4)[0]
    sel = oracle.select(st, q, budget)
    out = oracle.attend(st, q, sel)
    ids = np.full(budget, -1, np.int32)
    ids[: len(sel.ids)] = sel.ids
    return st, q, sel, out, ids


def test_exact_answer_passes():
    st, q, sel, out, ids = _case()
    assert check_decode_unit(st, q, 400, out, ids, len(sel.ids)) < 1e-12


def test_wrong_count_duplicates_and_padding_are_rejected():
    st, q, sel, out, ids = _case()
    with pytest.raises(AssertionError):
        check_decode_unit(st, q, 400, out, ids, len(sel.ids) - 1)
    dup = ids.copy()
    dup[5] = dup[6]
    with pytest.raises(AssertionError):
        check_decode_unit(st, q, 400, out, dup, len(sel.ids))
    # a budget above n: the entries past the count must stay -1
    st2, q2, sel2, out2, ids2 = _case(2000)
    assert len(sel2.ids) == st2.n_total < 2000
    check_decode_unit(st2, q2, 2000, out2, ids2, len(sel2.ids))
    bad_pad = ids2.copy()
    bad_pad[-1] = 0
    with pytest.raises(AssertionError):
        check_decode_unit(st2, q2, 2000, out2, bad_pad, len(sel2.ids))


def test_swapped_token_without_a_near_tie_is_rejected():
    st, q, sel, out, ids = _case()
    outside = np.setdiff1d(st.ids, sel.ids)
    bad = ids.copy()
    bad[len(sel.ids) - 1] = outside[0]
    with pytest.raises(AssertionError, match="near-tie"):
        check_decode_unit(st, q, 400, out, bad, len(sel.ids))


def test_output_error_above_tolerance_is_rejected():
    st, q, sel, out, ids = _case()
    check_decode_unit(st, q, 400, out + 1.5e-3, ids, len(sel.ids))
    with pytest.raises(AssertionError, match="max-abs"):
        check_decode_unit(st, q, 400, out + 3e-3, ids, len(sel.ids))


def test_assignment_rules():
    K, _ = si.keys_values(13, 0, 400, 6)
    mh = oracle.normalize(oracle.bf16_to_f64(K[:6]))
    a = oracle.assign(K, mh)
    assert check_assign(K, mh, a) == 0
    # a clear mistake: every key sent to its worst cluster
    s = oracle.bf16_to_f64(K) @ oracle.bf16_to_f64(mh).T
    with pytest.raises(AssertionError):
        check_assign(K, mh, np.argmin(s, axis=1).astype(np.int32))
    # an exact tie (a duplicated centroid) may go either way
    mh2 = np.concatenate([mh, mh[:1]])
    a2 = oracle.assign(K, mh2)
    alt = np.where(a2 == 0, 6, a2).astype(np.int32)
    assert check_assign(K, mh2, alt) == int((a2 == 0).sum())


def test_mu_hat_rule_rejects_two_step_errors():
    mu = oracle.bf16_to_f64(si.keys_values(14, 0, 20, 4)[0])
    mh = oracle.normalize(mu)
    check_mu_hat(mu.astype(np.float32), mh)
    bad = mh.copy()
    bad[3, 7] = bad[3, 7] + 2  # two bf16 steps in the last bits
    with pytest.raises(AssertionError):
        check_mu_hat(mu.astype(np.float32), bad)
