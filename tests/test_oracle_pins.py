"""Pins for the fp64 oracle: checks against things other than the oracle itself.

* central finite differences of the KL loss L = sum_t KL(p_t || Softmax(I_t))
  (aclnnSparseLightningIndexerKLLossGrad, section 计算公式) w.r.t. q, k and w;
* a dense brute force that writes the top-k gather as one-hot matrices;
* torch fp64 autograd of the same loss through gather / relu / log_softmax;
* hand-derived closed forms (tests/golden/*.json);
* the textbook special case N1=1, w=1, S>0, identity indices, where the operator
  reduces to the softmax cross-entropy gradient;
* invariants: sum y = 1 over valid slots, y = 0 off them, untouched dk rows exactly 0,
  unreferenced key rows and p at invalid slots have no influence, and the identities
  w_h dW_h = <q_h, dq_h> and sum_t,h w dW = sum_r <k_r, dk_r>;
* used lengths (seqUsedQ / seqUsedK): equal to the excluded slots rewritten to -1,
  padding rows never read, finite differences of the loss over the slots in use.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import slikl_inputs as si

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def sigma(x):
    return 1.0 / (1.0 + math.exp(-x))


def tiny_problem(seed, B=2, lens_q=(3, 2), lens_k=(4, 3), N1=3, D=4, K=4, invalid=True,
                 margin=2e-2):
    """Random fp64 problem (not rounded) with |S| > margin on every valid slot and
    p normalised over the valid slots."""
    rng = np.random.default_rng(seed)
    qs = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int64)
    ks = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int64)
    T1, T2 = int(qs[-1]), int(ks[-1])
    while True:
        q = rng.standard_normal((T1, N1, D))
        k = rng.standard_normal((T2, D))
        w = rng.standard_normal((T1, N1))
        idx = np.full((T1, K), -1, dtype=np.int32)
        for b in range(B):
            for t in range(qs[b], qs[b + 1]):
                nk = int(lens_k[b])
                sel = rng.permutation(nk)[: min(K, nk)]
                idx[t, : sel.size] = sel
                if invalid and rng.random() < 0.5 and sel.size > 1:
                    idx[t, rng.integers(0, sel.size)] = -1
        ok = True
        for t in range(T1):
            b = int(np.searchsorted(qs, t, side="right") - 1)
            for j in range(K):
                if idx[t, j] >= 0:
                    s = q[t] @ k[ks[b] + idx[t, j]]
                    if np.min(np.abs(s)) < margin:
                        ok = False
        if ok:
            break
    e = np.exp(rng.standard_normal((T1, K))) * (idx >= 0)
    p = e / np.maximum(e.sum(1, keepdims=True), 1e-300)
    return dict(q=q, k=k, w=w, p=p, idx=idx, q_start=qs, k_start=ks)


def run(pr, **kw):
    return oracle.grad_arrays(pr["q"], pr["k"], pr["w"], pr["p"], pr["idx"], pr["q_start"],
                              pr["k_start"], **kw)


def total_loss(pr):
    return run(pr)["loss"].sum()


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_finite_differences_of_kl_loss(seed):
    pr = tiny_problem(seed)
    g = run(pr)
    h = 1e-6
    for name, grad in (("q", g["dq"]), ("k", g["dk"]), ("w", g["dw"])):
        x = pr[name]
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            old = x[i]
            x[i] = old + h
            lp = total_loss(pr)
            x[i] = old - h
            lm = total_loss(pr)
            x[i] = old
            fd[i] = (lp - lm) / (2 * h)
        scale = np.abs(grad).max()
        assert scale > 1e-3
        err = np.abs(fd - grad).max() / scale
        assert err < 1e-6, (name, err)


def one_hot_brute_force(pr):
    """Dense formulation: K_t = G_t k_b with one-hot G_t, everything as fp64 matmuls."""
    q, k, w, p, idx = pr["q"], pr["k"], pr["w"], pr["p"], pr["idx"]
    qs, ks = pr["q_start"], pr["k_start"]
    T1, N1, D = q.shape
    K = idx.shape[1]
    out = dict(y=np.zeros((T1, K)), dw=np.zeros((T1, N1)), dq=np.zeros((T1, N1, D)),
               dk=np.zeros_like(k))
    for b in range(len(qs) - 1):
        kb = k[ks[b]:ks[b + 1]]
        for t in range(qs[b], qs[b + 1]):
            valid = idx[t] >= 0
            G = np.zeros((K, kb.shape[0]))
            G[np.nonzero(valid)[0], idx[t][valid]] = 1.0
            Kt = G @ kb                                   # [K, D]
            S = q[t] @ Kt.T                               # [N1, K]
            R = np.maximum(S, 0.0)
            I = w[t] @ R                                  # [K]
            if not valid.any():
                continue
            e = np.where(valid, np.exp(I - I[valid].max()), 0.0)
            y = e / e.sum()
            dI = np.where(valid, y - p[t], 0.0)
            dS = (w[t][:, None] * (S > 0)) * dI[None, :]
            out["y"][t] = y
            out["dw"][t] = R @ dI
            out["dq"][t] = dS @ Kt
            out["dk"][ks[b]:ks[b + 1]] += G.T @ (dS.T @ q[t])
    return out


@pytest.mark.parametrize("seed", [3, 4])
def test_one_hot_brute_force(seed):
    pr = tiny_problem(seed, B=3, lens_q=(4, 1, 5), lens_k=(7, 2, 9), N1=4, D=6, K=5)
    g = run(pr)
    bf = one_hot_brute_force(pr)
    for name in ("y", "dw", "dq", "dk"):
        np.testing.assert_allclose(g[name], bf[name], rtol=1e-11, atol=1e-13, err_msg=name)


def torch_autograd(pr):
    q = torch.tensor(pr["q"], requires_grad=True)
    k = torch.tensor(pr["k"], requires_grad=True)
    w = torch.tensor(pr["w"], requires_grad=True)
    p = torch.tensor(pr["p"])
    idx = torch.tensor(pr["idx"]).long()
    qs, ks = pr["q_start"], pr["k_start"]
    T1 = q.shape[0]
    batch = torch.tensor(np.searchsorted(qs, np.arange(T1), side="right") - 1)
    valid = idx >= 0
    rows = torch.where(valid, idx + torch.tensor(ks)[batch][:, None], torch.zeros_like(idx))
    Kt = k[rows]                                          # [T1, K, D]
    S = torch.einsum("thd,tjd->thj", q, Kt)
    I = torch.einsum("th,thj->tj", w, torch.relu(S))
    I = I.masked_fill(~valid, float("-inf"))
    logy = torch.log_softmax(I, dim=-1)
    has = valid.any(-1)
    terms = torch.where(valid & (p > 0), p * (torch.log(torch.where(p > 0, p, 1.0)) - logy),
                        torch.zeros_like(p))
    L = terms[has].sum()
    dq, dk, dw = torch.autograd.grad(L, (q, k, w))
    y = torch.where(has[:, None], logy.exp(), torch.zeros_like(p))
    return dict(y=y.detach().numpy(), dq=dq.numpy(), dk=dk.numpy(), dw=dw.numpy())


@pytest.mark.parametrize("seed", [5, 6])
def test_torch_fp64_autograd(seed):
    pr = tiny_problem(seed, B=2, lens_q=(6, 5), lens_k=(11, 8), N1=5, D=7, K=6)
    g = run(pr)
    ta = torch_autograd(pr)
    for name in ("y", "dw", "dq", "dk"):
        np.testing.assert_allclose(g[name], ta[name], rtol=1e-10, atol=1e-12, err_msg=name)


def test_duplicate_indices_are_independent_slots():
    """Repeated keys in one row: each slot is its own softmax entry and both scatter-add
    (autograd through the gather sums them the same way)."""
    pr = tiny_problem(7, B=1, lens_q=(4,), lens_k=(5,), N1=3, D=4, K=5, invalid=False)
    pr["idx"][:, 1] = pr["idx"][:, 0]
    e = np.exp(np.random.default_rng(0).standard_normal(pr["p"].shape))
    pr["p"] = e / e.sum(1, keepdims=True)
    g = run(pr)
    ta = torch_autograd(pr)
    for name in ("y", "dw", "dq", "dk"):
        np.testing.assert_allclose(g[name], ta[name], rtol=1e-10, atol=1e-12, err_msg=name)


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        fx = json.load(f)
    inp = fx["inputs"]
    q = np.array(inp["q"], dtype=np.float64)
    k = np.array(inp["k"], dtype=np.float64)
    pr = dict(q=q, k=k, w=np.array(inp["w"], dtype=np.float64),
              p=np.array(inp["p"], dtype=np.float64), idx=np.array(inp["idx"], dtype=np.int32),
              q_start=np.array([0, q.shape[0]]), k_start=np.array([0, k.shape[0]]))
    return run(pr)


def test_golden_two_slot_closed_form():
    g = _golden("two_slot_closed_form.json")
    a = sigma(1.0) - 0.5
    np.testing.assert_allclose(g["y"], [[sigma(1.0), sigma(-1.0), 0.0]], rtol=1e-14)
    assert g["y"][0, 2] == 0.0
    np.testing.assert_allclose(g["dw"], [[a]], rtol=1e-13)
    np.testing.assert_allclose(g["dq"], [[[a]]], rtol=1e-13)
    np.testing.assert_allclose(g["dk"], [[a], [-a]], rtol=1e-13)


def test_golden_relu_kink_closed_form():
    g = _golden("relu_kink_closed_form.json")
    b = sigma(-4.0) - 0.25
    np.testing.assert_allclose(g["y"], [[sigma(-4.0), sigma(4.0)]], rtol=1e-14)
    np.testing.assert_allclose(g["dw"], [[-2 * b, 0.0]], rtol=1e-13, atol=1e-16)
    np.testing.assert_allclose(g["dq"], [[[-4 * b], [0.0]]], rtol=1e-13, atol=1e-16)
    np.testing.assert_allclose(g["dk"], [[2 * b], [-2 * b]], rtol=1e-13)


def test_textbook_softmax_cross_entropy():
    """N1=1, w=1, q,k > 0 (so S > 0 everywhere), identity indices over all keys:
    I = q K^T and the gradients are the softmax cross-entropy ones,
    dq = (y - p) K and dk_r = (y_r - p_r) q."""
    rng = np.random.default_rng(11)
    T, S2, D = 5, 9, 6
    q = rng.random((T, 1, D)) * 0.5 + 0.01
    k = rng.random((S2, D)) * 0.5 + 0.01
    p = rng.random((T, S2))
    p /= p.sum(1, keepdims=True)
    idx = np.tile(np.arange(S2, dtype=np.int32), (T, 1))
    pr = dict(q=q, k=k, w=np.ones((T, 1)), p=p, idx=idx, q_start=np.array([0, T]),
              k_start=np.array([0, S2]))
    g = run(pr)
    logits = q[:, 0, :] @ k.T
    y = np.exp(logits - logits.max(1, keepdims=True))
    y /= y.sum(1, keepdims=True)
    np.testing.assert_allclose(g["y"], y, rtol=1e-13)
    np.testing.assert_allclose(g["dq"][:, 0, :], (y - p) @ k, rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(g["dk"], (y - p).T @ q[:, 0, :], rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(g["dw"][:, 0], ((y - p) * logits).sum(1), rtol=1e-10, atol=1e-14)


@pytest.fixture(scope="module")
def cfg0():
    wl = si.config(0)
    return wl, oracle.grad(wl)


def test_invariants_softmax(cfg0):
    wl, g = cfg0
    idx = wl.idx.numpy().reshape(wl.T1, wl.K)
    valid = idx >= 0
    np.testing.assert_allclose(g["y"].sum(1), np.where(valid.any(1), 1.0, 0.0), rtol=1e-12)
    assert np.all(g["y"][~valid] == 0.0)
    assert np.all(g["y"][valid] > 0.0)


def test_invariants_untouched_rows_and_invalid_p(cfg0):
    wl, g = cfg0
    idx = wl.idx.numpy().reshape(wl.T1, wl.K)
    referenced = np.zeros(wl.T2, dtype=bool)
    referenced[idx[idx >= 0]] = True            # one batch: local index = row
    assert (~referenced).any()
    assert np.all(g["dk"][~referenced] == 0.0)
    # perturb unreferenced key rows and p at invalid slots: nothing may change
    q = wl.q.double().numpy().reshape(wl.T1, wl.N1, wl.D)
    k = wl.k.double().numpy().reshape(wl.T2, wl.D).copy()
    k[~referenced] += 7.0
    p = wl.p.double().numpy().reshape(wl.T1, wl.K).copy()
    p[idx < 0] = 0.3
    qs, ks = np.array([0, wl.T1]), np.array([0, wl.T2])
    g2 = oracle.grad_arrays(q, k, wl.w.double().numpy().reshape(wl.T1, wl.N1), p, idx, qs, ks)
    for name in ("y", "dw", "dq", "dk"):
        assert np.array_equal(g[name], g2[name]), name


def test_invariants_bilinear_identities(cfg0):
    """sum_d q_hd dq_hd = sum_j dS_hj S_hj = w_h dW_h per token and head; summed over all
    tokens this also equals sum_r <k_r, dk_r>."""
    wl, g = cfg0
    q = wl.q.double().numpy().reshape(wl.T1, wl.N1, wl.D)
    k = wl.k.double().numpy().reshape(wl.T2, wl.D)
    w = wl.w.double().numpy().reshape(wl.T1, wl.N1)
    lhs = (q * g["dq"]).sum(-1)
    rhs = w * g["dw"]
    np.testing.assert_allclose(lhs, rhs, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose((k * g["dk"]).sum(), rhs.sum(), rtol=1e-9)


def test_token_subset_matches_full(cfg0):
    wl, g = cfg0
    toks = np.array([0, 5, 63, 64, 200, 255])
    gs = oracle.grad(wl, tokens=toks)
    for name in ("y", "dw", "dq"):
        np.testing.assert_array_equal(gs[name][toks], g[name][toks])


def test_thread_count_does_not_change_results(cfg0):
    wl, g = cfg0
    g1 = oracle.grad(wl, nthreads=1)
    for name in ("y", "dw", "dq", "dk"):
        assert np.array_equal(g1[name], g[name]), name


def test_out_of_range_index_rejected():
    pr = tiny_problem(8)
    pr["idx"][0, 0] = 99
    with pytest.raises(ValueError):
        run(pr)


def test_all_invalid_row():
    pr = tiny_problem(9)
    pr["idx"][1, :] = -1
    pr["p"][1, :] = 0.0
    g = run(pr)
    assert np.all(g["y"][1] == 0) and np.all(g["dw"][1] == 0) and np.all(g["dq"][1] == 0)
    assert g["loss"][1] == 0.0


# ---------------------------------------------------------------------------
# work split (metadata generator)
# ---------------------------------------------------------------------------

def test_split_golden_sample_shapes():
    with open(os.path.join(GOLDEN, "metadata_sample_shapes.json")) as f:
        fx = json.load(f)
    for case in fx["cases"]:
        cuq = np.array(case["cu_seqlens_q"])
        cuk = np.array(case["cu_seqlens_k"])
        total = int(cuq[-1])
        maxk = int(np.diff(cuk).max())
        hdr, ranges = oracle.split_equal(total, case["cores"], maxk)
        assert list(hdr) == case["header"]
        _check_tiling(ranges, total)


def _check_tiling(ranges, total):
    assert ranges[0, 0] == 0 and ranges[-1, 1] == total
    assert np.all(ranges[1:, 0] == ranges[:-1, 1])
    assert np.all(ranges[:, 1] >= ranges[:, 0])


@pytest.mark.parametrize("total,cores", [(0, 7), (1, 148), (147, 148), (148, 148), (149, 148),
                                         (4096, 148), (35147, 148), (511, 24), (100000, 3)])
def test_split_equal_properties(total, cores):
    hdr, ranges = oracle.split_equal(total, cores, 1)
    _check_tiling(ranges, total)
    sizes = ranges[:, 1] - ranges[:, 0]
    former = -(-total // cores) if total else 0
    assert hdr[1] == former and hdr[2] == max(former - 1, 0)
    used = min(cores, total)
    assert hdr[4] == used and np.count_nonzero(sizes) == used
    assert set(sizes[:used].tolist()) <= {former, max(former - 1, 0)}
    assert np.count_nonzero(sizes == hdr[2]) - (cores - used if hdr[2] == 0 else 0) == hdr[3]


def test_split_weighted_brute_force():
    rng = np.random.default_rng(3)
    for trial in range(20):
        T1 = int(rng.integers(1, 60))
        K = int(rng.integers(1, 400))
        cores = int(rng.integers(1, 20))
        idx = np.where(rng.random((T1, K)) < rng.random(), rng.integers(0, 9, (T1, K)), -1)
        idx = idx.astype(np.int32)
        ranges = oracle.split_weighted(idx, cores)
        _check_tiling(ranges, T1)
        cost = np.array([1 + sum(int((idx[t, j:j + 128] >= 0).any()) for j in range(0, K, 128))
                         for t in range(T1)])
        P = np.concatenate([[0], np.cumsum(cost)])
        for c in range(cores):
            # the start of worker c is the first row whose prefix reaches c/cores of the total
            target = c * P[-1]
            t = ranges[c, 0]
            assert P[t] * cores >= target
            assert t == 0 or P[t - 1] * cores < target


def golden_split_rows(fx):
    """Index rows of the hand-worked split fixture: the listed slots valid, the rest -1."""
    idx = np.full((len(fx["rows_valid_slots"]), fx["topk"]), -1, dtype=np.int32)
    for t, slots in enumerate(fx["rows_valid_slots"]):
        for j in slots:
            idx[t, j] = j % 7
    return idx


def test_split_weighted_hand_worked():
    """The cost-weighted split against ranges worked out by hand (tests/golden)."""
    with open(os.path.join(GOLDEN, "split_weighted_hand.json")) as f:
        fx = json.load(f)
    idx = golden_split_rows(fx)
    for case in fx["cases"]:
        ranges = oracle.split_weighted(idx, case["cores"])
        assert ranges.tolist() == case["ranges"], case["cores"]


# ---------------------------------------------------------------------------
# used lengths (seqUsedQOptional / seqUsedKOptional: the page fixes only their type; the
# reading is "rows of each batch in use": query rows past q_used[b] are padding, slots
# naming a key past k_used[b] are invalid)
# ---------------------------------------------------------------------------

def used_valid(pr, q_used, k_used):
    """Valid-slot mask under used lengths, written from the reading alone."""
    idx, qs = pr["idx"], pr["q_start"]
    valid = np.zeros(idx.shape, dtype=bool)
    for b in range(qs.size - 1):
        for t in range(qs[b], qs[b + 1]):
            if t - qs[b] < q_used[b]:
                valid[t] = (idx[t] >= 0) & (idx[t] < k_used[b])
    return valid


def test_seq_used_equals_masked_indices():
    """Used lengths act exactly as rewriting the slots they exclude to -1."""
    pr = tiny_problem(10, lens_q=(3, 2), lens_k=(4, 3))
    qu, ku = [2, 1], [3, 1]
    valid = used_valid(pr, qu, ku)
    assert valid.any() and (~valid & (pr["idx"] >= 0)).any()
    g = run(pr, q_used=qu, k_used=ku)
    pm = dict(pr, idx=np.where(valid, pr["idx"], -1).astype(np.int32))
    gm = run(pm)
    for name in ("y", "dw", "dq", "dk", "loss"):
        assert np.array_equal(g[name], gm[name]), name
    # padding rows (local position >= q_used) are all zero
    for t in (2, 4):
        assert np.all(g["y"][t] == 0) and np.all(g["dw"][t] == 0) and np.all(g["dq"][t] == 0)
    # key rows past k_used are never named, so their dk rows are exactly zero
    assert np.all(g["dk"][[3, 5, 6]] == 0)


def test_seq_used_padding_rows_not_read():
    pr = tiny_problem(12, lens_q=(3, 2), lens_k=(4, 3))
    qu, ku = [1, 2], [4, 3]
    g = run(pr, q_used=qu, k_used=ku)
    bad = dict(pr, idx=pr["idx"].copy())
    bad["idx"][1] = 99            # padding rows of batch 0: out of range, never read
    bad["idx"][2] = -5
    g2 = run(bad, q_used=qu, k_used=ku)
    for name in ("y", "dw", "dq", "dk", "loss"):
        assert np.array_equal(g[name], g2[name]), name
    with pytest.raises(ValueError):
        run(bad)                   # without used lengths those rows break the contract


def test_seq_used_finite_differences():
    """The gradients under used lengths are those of the KL loss over the slots in use (p
    normalised over them)."""
    pr = tiny_problem(11, lens_q=(3, 2), lens_k=(4, 3))
    qu, ku = [3, 1], [2, 3]
    valid = used_valid(pr, qu, ku)
    e = np.where(valid, pr["p"] + 0.1, 0.0)
    pr["p"] = e / np.maximum(e.sum(1, keepdims=True), 1e-300)
    g = run(pr, q_used=qu, k_used=ku)
    h = 1e-6

    def loss():
        return run(pr, q_used=qu, k_used=ku)["loss"].sum()

    for name, grad in (("q", g["dq"]), ("k", g["dk"]), ("w", g["dw"])):
        x = pr[name]
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            old = x[i]
            x[i] = old + h
            lp = loss()
            x[i] = old - h
            lm = loss()
            x[i] = old
            fd[i] = (lp - lm) / (2 * h)
        scale = np.abs(grad).max()
        assert scale > 1e-3
        assert np.abs(fd - grad).max() / scale < 1e-6, name


def test_seq_used_out_of_range_rejected():
    pr = tiny_problem(13, lens_q=(3, 2), lens_k=(4, 3))
    for qu, ku in (([4, 1], None), ([-1, 1], None), (None, [5, 3]), (None, [1, -2])):
        with pytest.raises(ValueError):
            run(pr, q_used=qu, k_used=ku)
