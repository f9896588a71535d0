"""Pins of the oracle's target distribution for the variant that forms p from the main
attention (oracle.main_softmax_l1norm_arrays), checked against what holds independently of it:
a library softmax for one head, hand-worked cases, invariances of a softmax over the slots,
and a planted mistake (softmax over the heads instead of the slots) that the pins catch."""

import json
import os

import numpy as np
import pytest
import scipy.special

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "main_p_hand.json")


def one_batch(q_m, k_m, idx, scale, **kw):
    T1, K = np.asarray(idx).shape
    return oracle.main_softmax_l1norm_arrays(q_m, k_m, np.asarray(idx), np.array([0, T1]),
                                             np.array([0, len(k_m)]), scale, **kw)


def random_case(rng, T1=6, Nm=5, Dm=8, T2=30, K=12, invalid=0.25):
    q_m = rng.standard_normal((T1, Nm, Dm))
    k_m = rng.standard_normal((T2, Dm))
    idx = rng.integers(0, T2, size=(T1, K))
    idx[rng.random((T1, K)) < invalid] = -1
    return q_m, k_m, idx


def test_hand_worked_cases():
    for case in json.load(open(GOLDEN))["cases"]:
        q_m = np.array(case["q_m"])[None]
        k_m = np.array(case["k_m"])
        idx = np.array(case["idx"])[None]
        p = one_batch(q_m, k_m, idx, case["scale"])[0]
        assert np.allclose(p, case["p"], rtol=0, atol=1e-9), case["name"]


def test_single_head_is_the_library_softmax():
    rng = np.random.default_rng(1)
    q_m, k_m, idx = random_case(rng, Nm=1)
    p = one_batch(q_m, k_m, idx, 0.7)
    for t in range(idx.shape[0]):
        ok = idx[t] >= 0
        ref = scipy.special.softmax(0.7 * (k_m[idx[t][ok]] @ q_m[t, 0]))
        assert np.allclose(p[t][ok], ref, rtol=1e-12, atol=0)
        assert np.all(p[t][~ok] == 0)


def test_identical_heads_equal_one_head():
    rng = np.random.default_rng(2)
    q_m, k_m, idx = random_case(rng, Nm=1)
    many = np.repeat(q_m, 7, axis=1)
    assert np.allclose(one_batch(many, k_m, idx, 0.3), one_batch(q_m, k_m, idx, 0.3),
                       rtol=1e-12, atol=1e-15)


def test_invariants():
    rng = np.random.default_rng(3)
    q_m, k_m, idx = random_case(rng)
    p = one_batch(q_m, k_m, idx, 0.5)
    ok = idx >= 0
    assert np.all(p >= 0) and np.all(p[~ok] == 0)
    assert np.allclose(p.sum(axis=1)[ok.any(axis=1)], 1.0, atol=1e-12)
    # a shift of every key by one vector moves each head's scores by a constant
    c = rng.standard_normal(k_m.shape[1])
    assert np.allclose(one_batch(q_m, k_m + c, idx, 0.5), p, rtol=1e-9, atol=1e-12)
    # scale 0: uniform over the valid slots
    p0 = one_batch(q_m, k_m, idx, 0.0)
    cnt = ok.sum(axis=1, keepdims=True)
    assert np.allclose(p0, np.where(ok, 1.0 / np.maximum(cnt, 1), 0.0), atol=1e-15)
    # permuting the heads changes nothing; permuting the slots permutes p
    assert np.allclose(one_batch(q_m[:, ::-1], k_m, idx, 0.5), p, rtol=1e-12, atol=1e-15)
    perm = rng.permutation(idx.shape[1])
    assert np.allclose(one_batch(q_m, k_m, idx[:, perm], 0.5), p[:, perm], rtol=1e-12, atol=1e-15)


def test_used_lengths_and_padding_rows():
    rng = np.random.default_rng(4)
    q_m, k_m, idx = random_case(rng, T1=8, T2=40)
    qs, ks = np.array([0, 5, 8]), np.array([0, 25, 40])
    idx[5:] = np.minimum(idx[5:], 14)                         # batch 1 has 15 keys
    idx[:5] = np.minimum(idx[:5], 24)
    p = oracle.main_softmax_l1norm_arrays(q_m, k_m, idx, qs, ks, 0.4, q_used=[3, 3],
                                          k_used=[10, 15])
    assert np.all(p[3:5] == 0)                                # padding rows of batch 0
    masked = idx.copy()
    masked[:5][masked[:5] >= 10] = -1                         # keys past seq_used_k: invalid
    ref = oracle.main_softmax_l1norm_arrays(q_m, k_m, masked, qs, ks, 0.4)
    assert np.allclose(p[:3], ref[:3], rtol=0, atol=0) and np.allclose(p[5:], ref[5:], 0, 0)


def test_planted_mistakes_are_caught(monkeypatch):
    """Two plausible mistakes planted in the oracle: a softmax over the heads instead of the
    slots (p comes out uniform: the hand-worked cases and the one-head library softmax catch
    it), and invalid slots taking part in the softmax (the invariants catch it)."""
    real = oracle.main_softmax_l1norm_arrays

    def over_heads(q_m, k_m, idx, q_start, k_start, scale, q_used=None, k_used=None):
        p = np.zeros(np.asarray(idx).shape)
        for t in range(idx.shape[0]):
            ok = np.nonzero(idx[t] >= 0)[0]
            if ok.size:
                S = scale * (np.asarray(q_m)[t] @ np.asarray(k_m)[idx[t][ok]].T)
                A = np.exp(S - S.max(axis=0, keepdims=True))
                A /= A.sum(axis=0, keepdims=True)
                h = A.sum(axis=0)
                p[t, ok] = h / h.sum()
        return p

    def with_invalid(q_m, k_m, idx, q_start, k_start, scale, q_used=None, k_used=None):
        idx = np.asarray(idx)
        return real(q_m, k_m, np.where(idx >= 0, idx, 0), q_start, k_start, scale)

    monkeypatch.setattr(oracle, "main_softmax_l1norm_arrays", over_heads)
    with pytest.raises(AssertionError):
        test_hand_worked_cases()
    with pytest.raises(AssertionError):
        test_single_head_is_the_library_softmax()
    monkeypatch.setattr(oracle, "main_softmax_l1norm_arrays", with_invalid)
    with pytest.raises(AssertionError):
        test_invariants()
    monkeypatch.setattr(oracle, "main_softmax_l1norm_arrays", real)
