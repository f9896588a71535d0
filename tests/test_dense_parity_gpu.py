"""GPU parity of the dense variant (slikl_dense_grad, through the C ABI) against the dense fp64
oracle on the same seeded inputs. Tolerances as the sparse operator's: softmax_out rel-L2 <=
1e-5; dw <= 1e-4; dq, dk rel-L2 <= 5e-3 and max-abs <= 2e-2 * max|ref|; softmax_out exactly 0
past each row's visible keys; dk exactly +0 on keys no row sees."""

import numpy as np
import pytest
import torch

import oracle
import slikl_inputs as si
import sparse_lightning_indexer_b200 as sli

pytestmark = pytest.mark.gpu

TOL = {"y": (1e-5, None), "dw": (1e-4, None), "dq": (5e-3, 2e-2), "dk": (5e-3, 2e-2)}


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
        m = np.abs(ref).max()
        assert np.abs(got - ref).max() <= mtol * m + 1e-30, name


def run_dense(wl, **kw):
    res = sli.dense_grad_workload(wl, **kw)
    torch.cuda.synchronize()
    flags = sli.slikl_read_device_status(res["workspace"].data_ptr())
    T1, T2 = wl.T1, wl.T2
    got = dict(y=res["softmax_out"].double().cpu().numpy().reshape(T1, wl.Ld),
               dw=res["dw"].double().cpu().numpy().reshape(T1, wl.N1),
               dq=res["dq"].double().cpu().numpy().reshape(T1, wl.N1, wl.D),
               dk=res["dk"].double().cpu().numpy().reshape(T2, wl.D),
               dk_raw=res["dk"].cpu().reshape(T2, wl.D), flags=flags)
    if "loss" in res:
        got["loss"] = res["loss"].double().cpu().numpy()
    return got


def seen_keys(wl, used_q=None, used_k=None):
    """Keys that some query row sees, from the mask geometry alone."""
    seen = np.zeros(wl.T2, dtype=bool)
    for b in range(wl.B):
        if wl.layout == "TND":
            q0, q1 = int(wl.cu_seqlens_q[b]), int(wl.cu_seqlens_q[b + 1])
            k0, k1 = int(wl.cu_seqlens_k[b]), int(wl.cu_seqlens_k[b + 1])
        else:
            q0, q1, k0, k1 = b * wl.S1, (b + 1) * wl.S1, b * wl.S2, (b + 1) * wl.S2
        qlen = q1 - q0 if used_q is None else used_q[b]
        klen = k1 - k0 if used_k is None else used_k[b]
        far = max((oracle.dense_visible(wl.mask_mode, s, qlen, klen) for s in range(qlen)),
                  default=0)
        seen[k0:k0 + min(far, wl.Ld)] = True
    return seen


def check_all(wl, got, ref, used_q=None, used_k=None):
    for n in ("y", "dw", "dq", "dk"):
        check_close(n, got[n], ref[n])
    assert np.all(got["y"][ref["y"] == 0] == 0.0), "softmax_out must be exactly 0 off the visible keys"
    unseen = torch.from_numpy(~seen_keys(wl, used_q, used_k))
    assert torch.all(got["dk_raw"][unseen].view(torch.int16) == 0), "unseen keys need dk = +0"


CASES = [
    dict(seed=1, layout="BSND", B=2, S1=70, S2=300, N1=16, D=128, mask_mode=3),
    dict(seed=2, layout="BSND", B=1, S1=200, S2=200, N1=64, D=128, mask_mode=3, qk_scale=0.1,
         w_var=1 / 64),
    dict(seed=3, layout="BSND", B=2, S1=33, S2=130, N1=8, D=64, mask_mode=0),
    dict(seed=4, layout="TND", B=3, S1=90, S2=400, N1=32, D=128, mask_mode=3,
         dtype=torch.float16, lens_q=[90, 17, 64], lens_k=[400, 9, 30]),
    dict(seed=5, layout="TND", B=2, S1=40, S2=150, N1=24, D=128, mask_mode=0,
         lens_q=[40, 11], lens_k=[150, 77], Ld=160),
    dict(seed=6, layout="BSND", B=1, S1=20, S2=257, N1=128, D=128, mask_mode=3),
]
MODES = [(False, "auto"), (False, "scatter"), (False, "keymajor"), (True, "auto")]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"s{c['seed']}")
@pytest.mark.parametrize("mode", MODES, ids=["auto", "scatter", "keymajor", "det"])
def test_dense_parity(case, mode):
    det, path = mode
    wl = si.dense_small(**case)
    ref = oracle.dense_grad(wl)
    got = run_dense(wl, deterministic=det, dk_path=path)
    assert got["flags"] == 0
    check_all(wl, got, ref)


def test_dense_used_lengths_and_loss():
    qu, ku = [50, 9], [120, 300]
    wl = si.dense_small(seed=7, layout="BSND", B=2, S1=60, S2=300, N1=16, D=128, mask_mode=3,
                        used_q=qu, used_k=ku)
    ref = oracle.dense_grad(wl, seq_used_q=qu, seq_used_k=ku)
    got = run_dense(wl, seq_used_q=qu, seq_used_k=ku, loss=True)
    assert got["flags"] == 0
    check_all(wl, got, ref, qu, ku)
    assert rel_l2(got["loss"], ref["loss"]) <= 1e-5


def test_dense_row_len_below_keys_is_flagged():
    """TND keys with a batch longer than the row length: flagged, the keys past it left out."""
    wl = si.dense_small(seed=8, layout="TND", B=2, S1=30, S2=200, N1=16, D=128, mask_mode=0,
                        lens_q=[30, 10], lens_k=[200, 50], Ld=128)
    got = run_dense(wl)
    assert got["flags"] & sli.SLIKL_DEV_ROW_LEN_BELOW_KEYS
    assert np.all(np.isfinite(got["y"]))


_FULL = {}


def dense_full_ref():
    if not _FULL:
        wl = si.dense_full()
        _FULL["wl"], _FULL["ref"] = wl, oracle.dense_grad(wl)
    return _FULL["wl"], _FULL["ref"]


@pytest.mark.parametrize("mode", [(False, "auto"), (False, "scatter"), (True, "auto")],
                         ids=["auto", "scatter", "det"])
def test_dense_full_size_parity(mode):
    """The dense workload the bench times (causal, 4096 queries x 4096 keys, N1 = 64), every
    output of every row against the oracle."""
    det, path = mode
    wl, ref = dense_full_ref()
    got = run_dense(wl, deterministic=det, dk_path=path)
    assert got["flags"] == 0
    check_all(wl, got, ref)
