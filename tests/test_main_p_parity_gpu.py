"""GPU parity of the variant that forms p from the main attention (slikl_grad_recompute_p,
through the C ABI) against the oracle on the same seeded inputs: p itself (rel-L2 <= 1e-5,
exactly 0 at invalid slots and on rows without a valid slot), then the backward's outputs at
the sparse operator's tolerances, and the per-row loss (absolute bound derived below)."""

import numpy as np
import pytest
import torch

import oracle
import slikl_inputs as si
import sparse_lightning_indexer_b200 as sli

pytestmark = pytest.mark.gpu

TOL = {"p": (1e-5, None), "y": (1e-5, None), "dw": (1e-4, None), "dq": (5e-3, 2e-2),
       "dk": (5e-3, 2e-2)}


def rel_l2(got, ref):
    n = np.linalg.norm(ref)
    d = np.linalg.norm(got - ref)
    return d / n if n > 0 else (0.0 if d == 0 else np.inf)


def check_close(name, got, ref):
    rtol, mtol = TOL[name]
    assert np.all(np.isfinite(got)), name
    e = rel_l2(got, ref)
    assert e <= rtol, f"{name}: rel-L2 {e:.3e} > {rtol}"
    if mtol is not None:
        assert np.abs(got - ref).max() <= mtol * np.abs(ref).max() + 1e-30, name


def run(wl, main, **kw):
    res = sli.grad_recompute_p_workload(wl, main, **kw)
    torch.cuda.synchronize()
    flags = sli.slikl_read_device_status(res["workspace"].data_ptr())
    T1, T2 = wl.T1, wl.T2
    got = {n: res[n].double().cpu().numpy() for n in res if n != "workspace"}
    got["p"] = got["p"].reshape(T1, wl.K)
    got["y"] = got.pop("softmax_out").reshape(T1, wl.K)
    got["dw"] = got["dw"].reshape(T1, wl.N1)
    got["dq"] = got["dq"].reshape(T1, wl.N1, wl.D)
    got["dk"] = got["dk"].reshape(T2, wl.D)
    got["flags"] = flags
    return got


def check_all(got, ref, loss=False):
    assert got["flags"] == 0
    check_close("p", got["p"], ref["p"])
    assert np.all(got["p"][ref["p"] == 0] == 0.0), "p must be exactly 0 off the valid slots"
    for n in ("y", "dw", "dq", "dk"):
        check_close(n, got[n], ref[n])
    if loss:
        # L_t = sum_j p log(p / y) moves by sum_j p_j (dp_j / p_j - dy_j / y_j) under relative
        # errors of p and y: with both within 1e-5 that is at most 2e-5 absolute, whatever the
        # size of L_t (a smooth p from many heads gives a small loss, so a bound relative to
        # L_t alone does not follow from the arithmetic)
        err = np.abs(got["loss"] - ref["loss"])
        assert np.all(err <= 1e-5 * np.abs(ref["loss"]) + 2e-5), err.max()
        assert np.all(got["loss"][ref["loss"] == 0] == 0.0)


CASES = [
    dict(case=dict(seed=51, layout="BSND", B=2, S1=40, S2=300, N1=16, D=128, K=200), Nm=16, Dm=128),
    dict(case=dict(seed=52, layout="TND", B=3, S1=50, S2=400, N1=32, D=128, K=300,
                   dtype=torch.float16, pattern="causal"), Nm=128, Dm=64),
    dict(case=dict(seed=53, layout="BSND", B=2, S1=30, S2=100, N1=16, D=64, K=160,
                   pattern="dup", invalid_frac=0.2), Nm=1, Dm=64),
    dict(case=dict(seed=54, layout="BSND", B=1, S1=24, S2=3000, N1=64, D=128, K=2048,
                   qk_scale=0.1, w_var=1 / 64), Nm=96, Dm=128),
    dict(case=dict(seed=55, layout="TND", B=3, lens_q=[0, 5, 3], lens_k=[4, 0, 6], N1=16, D=128,
                   K=8), Nm=8, Dm=128),
    dict(case=dict(seed=56, layout="BSND", B=1, S1=9, S2=50, N1=16, D=128, K=64, pattern="none"),
         Nm=16, Dm=128),
]
MODES = [(False, "auto"), (False, "scatter"), (True, "auto")]


@pytest.mark.parametrize("c", CASES, ids=lambda c: f"s{c['case']['seed']}")
@pytest.mark.parametrize("mode", MODES, ids=["auto", "scatter", "det"])
def test_recompute_p_parity(c, mode):
    det, path = mode
    wl = si.small(**c["case"])
    main = si.main_attention(wl, c["Nm"], c["Dm"], seed=c["case"]["seed"] + 1000)
    ref = oracle.grad_recompute_p(wl, main)
    check_all(run(wl, main, deterministic=det, dk_path=path, loss=True), ref, loss=True)


def test_recompute_p_used_lengths():
    wl = si.small(seed=57, layout="BSND", B=3, S1=40, S2=300, N1=16, D=128, K=200)
    main = si.main_attention(wl, 32, 128, seed=99, scale=0.05)
    qu, ku = [40, 17, 0], [300, 150, 7]
    ref = oracle.grad_recompute_p(wl, main, seq_used_q=qu, seq_used_k=ku)
    check_all(run(wl, main, seq_used_q=qu, seq_used_k=ku, loss=True), ref, loss=True)


def test_recompute_p_full_size():
    """The causal S=4096, topk=2048, N1=64 workload with a 128-head main attention (Dm=128):
    p and every output of every row against the oracle."""
    wl = si.config(1)
    main = si.main_attention(wl, 128, 128, seed=123, qk_scale=0.5)
    ref = oracle.grad_recompute_p(wl, main)
    check_all(run(wl, main, loss=True), ref, loss=True)
