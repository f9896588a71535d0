"""Pins of the dense-variant oracle (oracle.dense_grad_arrays), independent of itself.

The dense operator (DenseLightningIndexerKLLossGrad, named by the article on its metadata
generator, lmnt.cn) is read as the sparse operator's formulas (aclnnSparseLightningIndexer-
KLLossGrad, 计算公式) over every key of the batch that maskMode leaves visible. Pinned by:
- the mask geometry against counts worked by hand from the article's description (golden);
- torch fp64 autograd of the KL loss L = sum_t KL(p_t || softmax(I_t)) over the visible keys;
- central finite differences of the same loss with respect to w;
- the sparse C oracle (a different implementation) fed the visible keys as index lists,
  with and without used lengths.
"""

import json
import os

import numpy as np
import pytest
import torch

import oracle
import slikl_inputs as si

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_mask_geometry_hand_worked():
    with open(os.path.join(GOLDEN, "dense_mask_counts.json")) as f:
        fx = json.load(f)
    for c in fx["cases"]:
        got = [oracle.dense_visible(c["mask_mode"], s, c["qlen"], c["klen"]) for s in range(c["qlen"])]
        assert got == c["counts"], c


def flat(wl):
    T1, T2, N1, D = wl.T1, wl.T2, wl.N1, wl.D
    q = wl.q.double().numpy().reshape(T1, N1, D)
    k = wl.k.double().numpy().reshape(T2, D)
    w = wl.w.double().numpy().reshape(T1, N1)
    p = wl.p.double().numpy().reshape(T1, wl.Ld)
    # exact fp64 normalisation over each row's visible keys: the KL gradient with respect to
    # the logits is y - p only when p sums to one
    tot = p.sum(axis=1, keepdims=True)
    p = p / np.where(tot > 0, tot, 1.0)
    qs, ks = oracle.row_starts(wl.layout, wl.layout, wl.B, wl.S1, wl.S2,
                               None if wl.cu_seqlens_q is None else wl.cu_seqlens_q.numpy(),
                               None if wl.cu_seqlens_k is None else wl.cu_seqlens_k.numpy())
    return q, k, w, p, qs, ks


def torch_loss(q, k, w, p, qs, ks, mask_mode):
    """KL loss of the dense reading written with torch ops (masked softmax over visible keys)."""
    total = torch.zeros((), dtype=torch.float64)
    for b in range(len(qs) - 1):
        q0, q1, k0, k1 = int(qs[b]), int(qs[b + 1]), int(ks[b]), int(ks[b + 1])
        for s in range(q1 - q0):
            L = oracle.dense_visible(mask_mode, s, q1 - q0, k1 - k0)
            if L == 0:
                continue
            t = q0 + s
            S = torch.einsum("hd,jd->hj", q[t], k[k0:k0 + L])
            I = torch.einsum("h,hj->j", w[t], torch.relu(S))
            logy = torch.log_softmax(I, dim=0)
            pv = p[t, :L]
            pos = pv > 0
            total = total + torch.sum(pv[pos] * (torch.log(pv[pos]) - logy[pos]))
    return total


CASES = [
    dict(seed=1, layout="BSND", B=2, S1=6, S2=9, N1=3, D=64, mask_mode=3),
    dict(seed=2, layout="BSND", B=1, S1=5, S2=5, N1=2, D=64, mask_mode=0),
    dict(seed=3, layout="TND", B=3, S1=7, S2=8, N1=4, D=64, mask_mode=3,
         lens_q=[7, 2, 5], lens_k=[8, 6, 3]),
    dict(seed=4, layout="TND", B=2, S1=4, S2=6, N1=2, D=128, mask_mode=0, lens_q=[4, 3],
         lens_k=[6, 1]),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"s{c['seed']}")
def test_dense_oracle_matches_torch_autograd(case):
    wl = si.dense_small(qk_scale=1.0, w_var=0.5, **case)
    q, k, w, p, qs, ks = flat(wl)
    ref = oracle.dense_grad_arrays(q, k, w, p, qs, ks, wl.mask_mode)
    tq, tk, tw = (torch.tensor(a, requires_grad=True) for a in (q, k, w))
    L = torch_loss(tq, tk, tw, torch.tensor(p), qs, ks, wl.mask_mode)
    L.backward()
    assert np.allclose(ref["dq"], tq.grad.numpy(), rtol=1e-9, atol=1e-11)
    assert np.allclose(ref["dk"], tk.grad.numpy(), rtol=1e-9, atol=1e-11)
    assert np.allclose(ref["dw"], tw.grad.numpy(), rtol=1e-9, atol=1e-11)
    assert abs(ref["loss"].sum() - L.item()) <= 1e-10 * max(1.0, abs(L.item()))


def test_dense_oracle_finite_differences_w():
    wl = si.dense_small(seed=5, layout="BSND", B=1, S1=4, S2=6, N1=3, D=64, mask_mode=3,
                        qk_scale=1.0, w_var=0.5)
    q, k, w, p, qs, ks = flat(wl)
    ref = oracle.dense_grad_arrays(q, k, w, p, qs, ks, 3)
    eps = 1e-6
    for t in range(wl.T1):
        for h in range(wl.N1):
            wp, wm = w.copy(), w.copy()
            wp[t, h] += eps
            wm[t, h] -= eps
            lp = oracle.dense_grad_arrays(q, k, wp, p, qs, ks, 3)["loss"].sum()
            lm = oracle.dense_grad_arrays(q, k, wm, p, qs, ks, 3)["loss"].sum()
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - ref["dw"][t, h]) <= 1e-6 * max(1.0, abs(fd))


def as_sparse(wl, q_used=None, k_used=None):
    """The visible keys of each row as index lists (slot j = key j, -1 past the visible ones)."""
    q, k, w, p, qs, ks = flat(wl)
    idx = np.full((wl.T1, wl.Ld), -1, dtype=np.int32)
    for b in range(wl.B):
        qlen = int(qs[b + 1] - qs[b]) if q_used is None else q_used[b]
        klen = int(ks[b + 1] - ks[b]) if k_used is None else k_used[b]
        for s in range(int(qs[b + 1] - qs[b])):
            if s < qlen:
                L = oracle.dense_visible(wl.mask_mode, s, qlen, klen)
                idx[int(qs[b]) + s, :L] = np.arange(L)
    return q, k, w, p, idx, qs, ks


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"s{c['seed']}")
def test_dense_oracle_matches_sparse_oracle(case):
    wl = si.dense_small(**case)
    q, k, w, p, idx, qs, ks = as_sparse(wl)
    ref = oracle.dense_grad_arrays(q, k, w, p, qs, ks, wl.mask_mode)
    sp = oracle.grad_arrays(q, k, w, p, idx, qs, ks)
    for n in ("y", "dw", "dq", "dk", "loss"):
        assert np.allclose(ref[n], sp[n], rtol=1e-11, atol=1e-13), n


def test_dense_oracle_used_lengths_match_sparse_oracle():
    qu, ku = [3, 5], [4, 2]
    wl = si.dense_small(seed=6, layout="BSND", B=2, S1=6, S2=7, N1=3, D=64, mask_mode=3,
                        used_q=qu, used_k=ku)
    q, k, w, p, idx, qs, ks = as_sparse(wl, qu, ku)
    ref = oracle.dense_grad_arrays(q, k, w, p, qs, ks, 3, q_used=qu, k_used=ku)
    sp = oracle.grad_arrays(q, k, w, p, idx, qs, ks)
    for n in ("y", "dw", "dq", "dk"):
        assert np.allclose(ref[n], sp[n], rtol=1e-11, atol=1e-13), n
