"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the same seeded
inputs.

Tolerances (floating point): softmax_out rel-L2 <= 1e-5; dw rel-L2 <= 1e-4; dq and dk
rel-L2 <= 5e-3 and max-abs <= 2e-2 * max|ref|. Bit-exact: softmax_out = 0 at invalid
slots, dk = 0 on key rows no valid slot names, the work split, and deterministic-mode
repeats.

Full-size workloads (configs 1-4): every token's softmax_out, dw and dq and the full dk are
compared with one full oracle run of the same workload, on the auto and scatter dK paths and
(configs 1 and 4) the deterministic reduction.
"""

import json
import os

import numpy as np
import pytest
import torch

import oracle
import slikl_inputs as si
import sparse_lightning_indexer_b200 as sli

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TOL = {"y": (1e-5, None), "dw": (1e-4, None), "dq": (5e-3, 2e-2), "dk": (5e-3, 2e-2)}


def rel_l2(got, ref):
    n = np.linalg.norm(ref)
    d = np.linalg.norm(got - ref)
    return d / n if n > 0 else (0.0 if d == 0 else np.inf)


def assert_close(name, got, ref):
    rtol, mtol = TOL[name]
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), name
    e = rel_l2(got, ref)
    assert e <= rtol, f"{name}: rel-L2 {e:.3e} > {rtol}"
    if mtol is not None:
        m = np.abs(ref).max()
        a = np.abs(got - ref).max()
        assert a <= mtol * m, f"{name}: max-abs {a:.3e} > {mtol} * {m:.3e}"


def run_gpu(wl, deterministic=False, dk_path="auto", **kw):
    res = sli.grad_workload(wl, deterministic=deterministic, dk_path=dk_path, **kw)
    torch.cuda.synchronize()
    flags = sli.slikl_read_device_status(res["workspace"].data_ptr())
    T1, T2, N1, D, K = wl.T1, wl.T2, wl.N1, wl.D, wl.K
    return dict(y=res["softmax_out"].double().cpu().numpy().reshape(T1, K),
                dw=res["dw"].double().cpu().numpy().reshape(T1, N1),
                dq=res["dq"].double().cpu().numpy().reshape(T1, N1, D),
                dk=res["dk"].double().cpu().numpy().reshape(T2, D),
                dk_raw=res["dk"].cpu(), flags=flags,
                loss=res["loss"].double().cpu().numpy() if "loss" in res else None)


def referenced_rows(wl):
    """Key rows named by some valid slot (index in [0, len_k(b)))."""
    idx = wl.idx.numpy().reshape(wl.T1, wl.K)
    qs, ks = oracle.row_starts(wl.layout, wl.layout, wl.B, wl.S1, wl.S2,
                               None if wl.cu_seqlens_q is None else wl.cu_seqlens_q.numpy(),
                               None if wl.cu_seqlens_k is None else wl.cu_seqlens_k.numpy())
    batch = np.searchsorted(qs, np.arange(wl.T1), side="right") - 1
    rows = idx + ks[batch][:, None]
    ref = np.zeros(wl.T2, dtype=bool)
    ref[rows[idx >= 0]] = True
    return ref


def check_exact(wl, got):
    idx = wl.idx.numpy().reshape(wl.T1, wl.K)
    assert np.all(got["y"][idx < 0] == 0.0), "softmax_out must be exactly 0 at invalid slots"
    untouched = ~referenced_rows(wl)
    raw = got["dk_raw"].reshape(wl.T2, wl.D)
    assert torch.all(raw[torch.from_numpy(untouched)].view(torch.int16) == 0), \
        "dk must be exactly +0 on rows no valid slot names"


def check_against(wl, got, ref, tokens=None):
    sel = slice(None) if tokens is None else tokens
    for name in ("y", "dw", "dq"):
        assert_close(name, got[name][sel], ref[name][sel])
    assert_close("dk", got["dk"], ref["dk"])


SMALL = [
    dict(seed=1, layout="BSND", B=2, S1=40, S2=300, N1=16, D=128, K=200),
    dict(seed=2, layout="TND", B=3, S1=50, S2=400, N1=32, D=128, K=300, dtype=torch.float16,
         pattern="causal"),
    dict(seed=3, layout="BSND", B=1, S1=33, S2=7, N1=1, D=64, K=1),
    dict(seed=4, layout="BSND", B=1, S1=64, S2=64, N1=8, D=64, K=64, pattern="causal",
         qk_scale=1.0, w_var=1 / 8),
    dict(seed=5, layout="BSND", B=1, S1=24, S2=3000, N1=64, D=128, K=2048, qk_scale=0.1,
         w_var=1 / 64),
    dict(seed=6, layout="TND", B=2, S1=20, S2=600, N1=128, D=128, K=257),
    dict(seed=7, layout="BSND", B=2, S1=17, S2=500, N1=24, D=128, K=130, dtype=torch.float16),
    dict(seed=8, layout="BSND", B=2, S1=30, S2=100, N1=16, D=128, K=160, pattern="dup"),
    dict(seed=9, layout="BSND", B=2, S1=30, S2=700, N1=16, D=64, K=512, invalid_frac=0.3),
    dict(seed=10, layout="BSND", B=1, S1=9, S2=50, N1=16, D=128, K=64, pattern="none"),
    dict(seed=11, layout="TND", B=3, lens_q=[0, 5, 3], lens_k=[4, 0, 6], N1=16, D=128, K=8,
         pattern="uniform"),
    dict(seed=12, layout="TND", B=4, S1=70, S2=900, N1=48, D=64, K=700, dtype=torch.float16,
         pattern="causal", invalid_frac=0.1),
    # 64 < N1 <= 128: the 128-head tensor-core instances (heads past N1 padded with zeros)
    dict(seed=13, layout="BSND", B=1, S1=24, S2=2100, N1=128, D=128, K=2048, qk_scale=0.1,
         w_var=1 / 128),
    dict(seed=14, layout="TND", B=2, S1=30, S2=500, N1=96, D=64, K=300, dtype=torch.float16,
         pattern="causal"),
    dict(seed=15, layout="BSND", B=2, S1=25, S2=200, N1=65, D=128, K=130, pattern="dup",
         invalid_frac=0.2),
]


MODES = [(False, "scatter"), (False, "keymajor"), (True, "scatter"), (True, "keymajor")]
MODE_IDS = ["scatter", "keymajor", "det", "det_keymajor"]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"s{c['seed']}")
@pytest.mark.parametrize("mode", MODES, ids=MODE_IDS)
def test_small_parity(case, mode):
    det, path = mode
    wl = si.small(**case)
    ref = oracle.grad(wl)
    got = run_gpu(wl, deterministic=det, dk_path=path)
    assert got["flags"] == 0
    check_exact(wl, got)
    check_against(wl, got, ref)


def test_config0_full_parity():
    wl = si.config(0)
    ref = oracle.grad(wl)
    for det, path in MODES + [(False, "auto")]:
        got = run_gpu(wl, deterministic=det, dk_path=path)
        assert got["flags"] == 0
        check_exact(wl, got)
        check_against(wl, got, ref)


def test_keymajor_key_range_bound_too_small_flagged():
    """TND keys with a promised key-range bound below a batch's real key count: the batch is
    left out of the key-major records and the call flags it instead of faulting."""
    wl = si.small(seed=23, layout="TND", B=3, S1=30, S2=700, N1=16, D=128, K=64,
                  pattern="causal")
    real = sli.key_range_bound_of(wl)
    dev = torch.device("cuda")
    t = {n: getattr(wl, n).to(dev) for n in ("q", "k", "w", "p", "idx")}
    res = sli.grad(t["q"], t["k"], t["w"], t["p"], t["idx"], "TND", "TND",
                   wl.cu_seqlens_q.to(dev), wl.cu_seqlens_k.to(dev), dk_path="keymajor",
                   key_range_bound=max(1, real - 100))
    torch.cuda.synchronize()
    flags = sli.slikl_read_device_status(res["workspace"].data_ptr())
    assert flags & sli.SLIKL_DEV_KEY_RANGE_ABOVE_S2


_CFG_CACHE = {}


def cfg(cid):
    if cid not in _CFG_CACHE:
        _CFG_CACHE[cid] = si.config(cid)
    return _CFG_CACHE[cid]


# dK modes compared in full at each full-size workload: the auto path (key-major where the
# key range allows it), the scatter path, and deterministic mode on configs 1 and 4 on both
# paths (key-major with fixed-point records, and the sorted per-slot reduction)
FULL_MODES = {
    1: [(False, "auto"), (False, "scatter"), (True, "auto"), (True, "scatter")],
    2: [(False, "auto"), (False, "scatter")],
    3: [(False, "auto")],
    4: [(False, "auto"), (False, "scatter"), (True, "auto"), (True, "scatter")],
}


@pytest.mark.parametrize("cid", [1, 2, 3, 4])
def test_full_size_parity(cid):
    """Every output of the full-size workload against one full oracle run: softmax_out, dw and
    dq of every token and the full dk (unmasked: every hot key with all its adds), element by
    element, on each dK mode; plus the bit-exact zeros."""
    wl = cfg(cid)
    ref = oracle.grad(wl)
    for det, path in FULL_MODES[cid]:
        got = run_gpu(wl, deterministic=det, dk_path=path)
        assert got["flags"] == 0, (det, path)
        check_exact(wl, got)
        check_against(wl, got, ref)
        del got
    _CFG_CACHE.pop(cid, None)


def test_full_size_parity_128_heads():
    """The 128-head workload (causal S=4096, topk=2048, N1=128) in full on each dK mode."""
    wl = si.wide_heads()
    ref = oracle.grad(wl)
    for det, path in [(False, "auto"), (False, "scatter"), (True, "auto")]:
        got = run_gpu(wl, deterministic=det, dk_path=path)
        assert got["flags"] == 0, (det, path)
        check_exact(wl, got)
        check_against(wl, got, ref)
        del got


@pytest.mark.parametrize("cid", [1, 3])
def test_full_size_identities(cid):
    """Properties that hold at any size, checked on the full GPU outputs:
    sum_d q_hd dq_hd = w_h dW_h per token and head, and
    sum_r <k_r, dk_r> = sum_t,h w_th dW_th."""
    wl = si.config(cid)
    got = run_gpu(wl)
    q = wl.q.double().numpy().reshape(wl.T1, wl.N1, wl.D)
    k = wl.k.double().numpy().reshape(wl.T2, wl.D)
    w = wl.w.double().numpy().reshape(wl.T1, wl.N1)
    lhs = (q * got["dq"]).sum(-1)
    rhs = w * got["dw"]
    assert rel_l2(lhs, rhs) < 1e-2
    total = (k * got["dk"]).sum()
    assert abs(total - rhs.sum()) <= 1e-2 * np.abs(rhs).sum()


def bits(t):
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)


def repeat_case(name):
    if name == "dup":
        # every key named about eight times per row: the key-major records sum many dI
        return si.small(seed=41, layout="BSND", B=2, S1=64, S2=64, N1=32, D=128, K=512,
                        pattern="dup")
    return si.config(name)


@pytest.mark.parametrize("cid,path", [(1, "auto"), (4, "auto"), (4, "scatter"), ("dup", "auto"),
                                      ("dup", "scatter")],
                         ids=["cfg1-keymajor", "cfg4-keymajor", "cfg4-sorted", "dup-keymajor",
                              "dup-sorted"])
def test_deterministic_bitwise_repeat(cid, path):
    """Deterministic mode: ten calls on the same inputs give bit-identical outputs."""
    wl = repeat_case(cid)
    dev = torch.device("cuda")
    t = {n: getattr(wl, n).to(dev) for n in ("q", "k", "w", "p", "idx")}
    cuq = wl.cu_seqlens_q.to(dev) if wl.cu_seqlens_q is not None else None
    cuk = wl.cu_seqlens_k.to(dev) if wl.cu_seqlens_k is not None else None
    first = None
    ws = None
    for rep in range(10):
        res = sli.grad(t["q"], t["k"], t["w"], t["p"], t["idx"], wl.layout, wl.layout, cuq, cuk,
                       deterministic=True, workspace=ws, dk_path=path)
        ws = res["workspace"]
        cur = [bits(res[n]).clone() for n in ("dq", "dk", "dw", "softmax_out")]
        if first is None:
            first = cur
        else:
            for a, b in zip(first, cur):
                assert torch.equal(a, b)


def test_out_of_range_index_flagged_and_ignored():
    wl = si.small(seed=21, layout="TND", B=2, S1=10, S2=50, N1=16, D=128, K=40)
    idx = wl.idx.clone().reshape(wl.T1, wl.K)
    klen0 = int(wl.cu_seqlens_k[1] - wl.cu_seqlens_k[0])
    idx[0, 3] = klen0            # one past the batch's key range
    idx[1, 5] = -7               # below -1
    bad = si.Workload(**{f: getattr(wl, f) for f in wl.__dataclass_fields__})
    bad.idx = idx.reshape(wl.idx.shape).contiguous()
    got = run_gpu(bad)
    assert got["flags"] & sli.SLIKL_DEV_INDEX_OUT_OF_RANGE
    fixed = idx.clone()
    fixed[0, 3] = -1
    fixed[1, 5] = -1
    good = si.Workload(**{f: getattr(wl, f) for f in wl.__dataclass_fields__})
    good.idx = fixed.reshape(wl.idx.shape).contiguous()
    ref = oracle.grad(good)
    check_against(good, got, ref)


def test_bad_cu_seqlens_flagged():
    wl = si.small(seed=22, layout="TND", B=2, S1=10, S2=50, N1=16, D=128, K=40)
    bad = si.Workload(**{f: getattr(wl, f) for f in wl.__dataclass_fields__})
    cuk = wl.cu_seqlens_k.clone()
    cuk[1] = cuk[2] + 5            # not monotone and beyond T2
    bad.cu_seqlens_k = cuk
    got = run_gpu(bad)
    assert got["flags"] & sli.SLIKL_DEV_BAD_CU_SEQLENS_K
    assert np.all(got["y"] == 0) and np.all(got["dk"] == 0)


def metadata_gpu(wl, workers, mode):
    dev = torch.device("cuda")
    idx = wl.idx.to(dev)
    pr = sli.make_problem(wl.q, wl.k, wl.idx, wl.layout, wl.layout, False,
                          B=wl.B if wl.layout == "TND" else None)
    tn = sli.slikl_tensors()
    tn.sparse_indices = idx.data_ptr()
    cuq = cuk = None
    if wl.layout == "TND":
        cuq, cuk = wl.cu_seqlens_q.to(dev), wl.cu_seqlens_k.to(dev)
        tn.cu_seqlens_q, tn.cu_seqlens_k = cuq.data_ptr(), cuk.data_ptr()
    n = sli.slikl_grad_metadata_size(workers)
    meta = torch.full((n,), -5, dtype=torch.int32, device=dev)
    wsb = sli.slikl_grad_metadata_workspace_size(pr)
    ws = torch.empty(max(wsb, 256), dtype=torch.uint8, device=dev)
    sli.slikl_grad_metadata(pr, tn, workers, mode, meta.data_ptr(), ws.data_ptr(), ws.numel(),
                            torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return meta.cpu().numpy().astype(np.int64)


@pytest.mark.parametrize("cid", [0, 2, 4])
@pytest.mark.parametrize("workers", [148, 37])
def test_metadata_bit_exact(cid, workers):
    wl = cfg(cid)
    idx = wl.idx.numpy().reshape(wl.T1, wl.K)
    cuk = None if wl.cu_seqlens_k is None else wl.cu_seqlens_k.numpy()
    maxk = wl.S2 if cuk is None else int(np.diff(cuk).max())
    hdr, ranges_eq = oracle.split_equal(wl.T1, workers, maxk)
    m0 = metadata_gpu(wl, workers, 0)
    assert list(m0[:6]) == list(hdr) and m0[6] == 0 and m0[7] == workers
    assert np.array_equal(m0[8:].reshape(workers, 2), ranges_eq)
    m1 = metadata_gpu(wl, workers, 1)
    assert list(m1[:6]) == list(hdr) and m1[6] == 1
    assert np.array_equal(m1[8:].reshape(workers, 2), oracle.split_weighted(idx, workers))


def test_metadata_golden_sample_shapes():
    with open(os.path.join(GOLDEN, "metadata_sample_shapes.json")) as f:
        fx = json.load(f)
    for case in fx["cases"]:
        cuq = case["cu_seqlens_q"]
        cuk = case["cu_seqlens_k"]
        lq, lk = np.diff(cuq), np.diff(cuk)
        wl = si.small(seed=0, layout="TND", B=len(lq), lens_q=list(lq), lens_k=list(lk), N1=8,
                      D=128, K=4)
        m = metadata_gpu(wl, case["cores"], 0)
        assert list(m[:6]) == case["header"]


def test_metadata_weighted_hand_worked():
    """The device's cost-weighted split (mode 1) on the hand-worked fixture of tests/golden."""
    with open(os.path.join(GOLDEN, "split_weighted_hand.json")) as f:
        fx = json.load(f)
    rows = fx["rows_valid_slots"]
    wl = si.small(seed=0, layout="BSND", B=1, S1=len(rows), S2=300, N1=8, D=128,
                  K=fx["topk"], pattern="none")
    idx = torch.full((len(rows), fx["topk"]), -1, dtype=torch.int32)
    for t, slots in enumerate(rows):
        for j in slots:
            idx[t, j] = j % 7
    wl.idx = idx.reshape(wl.idx.shape).contiguous()
    for case in fx["cases"]:
        m = metadata_gpu(wl, case["cores"], 1)
        assert m[8:].reshape(case["cores"], 2).tolist() == case["ranges"], case["cores"]


@pytest.mark.parametrize("case", [SMALL[0], SMALL[1], SMALL[7], SMALL[8], SMALL[9], SMALL[10]],
                         ids=lambda c: f"s{c['seed']}")
@pytest.mark.parametrize("path", ["scatter", "keymajor"])
def test_kl_loss_output(case, path):
    """The optional per-row KL loss output against the oracle's L_t (rel-L2 <= 1e-5, rows
    without a valid slot exactly 0), on the dK paths that can run the case."""
    wl = si.small(**case)
    ref = oracle.grad(wl)
    res = sli.grad_workload(wl, dk_path=path, loss=True)
    torch.cuda.synchronize()
    got = res["loss"].double().cpu().numpy()
    assert got.shape == ref["loss"].shape
    assert np.all(np.isfinite(got))
    e = rel_l2(got, ref["loss"])
    assert e <= 1e-5, f"loss rel-L2 {e:.3e}"
    idx = wl.idx.numpy().reshape(wl.T1, wl.K)
    empty = ~(idx >= 0).any(axis=1)
    assert np.all(got[empty] == 0.0)


def test_kl_loss_output_config0():
    wl = si.config(0)
    ref = oracle.grad(wl)
    res = sli.grad_workload(wl, loss=True)
    torch.cuda.synchronize()
    assert rel_l2(res["loss"].double().cpu().numpy(), ref["loss"]) <= 1e-5


# ---------------------------------------------------------------------------
# used lengths (seq_used_q / seq_used_k): query rows past seq_used_q[b] are padding, slots
# naming a key past seq_used_k[b] are invalid
# ---------------------------------------------------------------------------

def batch_starts(wl):
    return oracle.row_starts(wl.layout, wl.layout, wl.B, wl.S1, wl.S2,
                             None if wl.cu_seqlens_q is None else wl.cu_seqlens_q.numpy(),
                             None if wl.cu_seqlens_k is None else wl.cu_seqlens_k.numpy())


def used_masked(wl, qu, ku):
    """Same workload with every slot the used lengths exclude set to -1."""
    qs, _ = batch_starts(wl)
    idx = wl.idx.clone().reshape(wl.T1, wl.K)
    for b in range(wl.B):
        for t in range(int(qs[b]), int(qs[b + 1])):
            if t - qs[b] >= qu[b]:
                idx[t] = -1
            else:
                idx[t][idx[t] >= ku[b]] = -1
    out = si.Workload(**{f: getattr(wl, f) for f in wl.__dataclass_fields__})
    out.idx = idx.reshape(wl.idx.shape).contiguous()
    return out


def with_garbage_in_padding(wl, qu):
    """Padding rows get indices that break the contract: they must not be read."""
    qs, _ = batch_starts(wl)
    idx = wl.idx.clone().reshape(wl.T1, wl.K)
    for b in range(wl.B):
        for t in range(int(qs[b] + qu[b]), int(qs[b + 1])):
            idx[t, 0::2] = 1 << 30
            idx[t, 1::2] = -9
    out = si.Workload(**{f: getattr(wl, f) for f in wl.__dataclass_fields__})
    out.idx = idx.reshape(wl.idx.shape).contiguous()
    return out


def lengths(wl):
    qs, ks = batch_starts(wl)
    return [int(qs[b + 1] - qs[b]) for b in range(wl.B)], [int(ks[b + 1] - ks[b]) for b in range(wl.B)]


SEQ_USED = [
    dict(case=dict(seed=31, layout="BSND", B=3, S1=40, S2=300, N1=16, D=128, K=200),
         used=lambda lq, lk: ([lq[0], 17, 0], [lk[0], 150, 7])),
    dict(case=dict(seed=32, layout="TND", B=3, S1=50, S2=400, N1=32, D=128, K=300,
                   dtype=torch.float16, pattern="causal"),
         used=lambda lq, lk: ([lq[0] // 2, lq[1], 1], [lk[0] // 3 + 1, lk[1], lk[2]])),
    dict(case=dict(seed=33, layout="BSND", B=2, S1=24, S2=3000, N1=64, D=128, K=2048,
                   qk_scale=0.1, w_var=1 / 64),
         used=lambda lq, lk: ([20, 24], [1000, 2999])),
    dict(case=dict(seed=34, layout="TND", B=2, S1=20, S2=600, N1=128, D=128, K=257),
         used=lambda lq, lk: ([lq[0], lq[1] // 2], [lk[0] // 2, lk[1]])),
]


@pytest.mark.parametrize("sc", SEQ_USED, ids=lambda c: f"s{c['case']['seed']}")
@pytest.mark.parametrize("mode", MODES, ids=MODE_IDS)
def test_seq_used_parity(sc, mode):
    det, path = mode
    case = sc["case"]
    wl = si.small(**case)
    lq, lk = lengths(wl)
    qu, ku = sc["used"](lq, lk)
    wm = used_masked(wl, qu, ku)
    idx = wl.idx.reshape(wl.T1, wl.K)
    assert (wm.idx.reshape(wl.T1, wl.K) != idx).any()     # the lengths exclude something
    ref = oracle.grad(wl, seq_used_q=qu, seq_used_k=ku)
    got = run_gpu(with_garbage_in_padding(wl, qu), deterministic=det, dk_path=path,
                  seq_used_q=qu, seq_used_k=ku, loss=True)
    assert got["flags"] == 0
    check_against(wm, got, ref)
    check_exact(wm, got)
    assert rel_l2(got["loss"], ref["loss"]) <= 1e-5
    assert np.all(got["loss"][ref["loss"] == 0] == 0)      # padding rows: exactly 0


def test_seq_used_out_of_range_is_flagged_and_clamped():
    wl = si.small(seed=35, layout="BSND", B=2, S1=30, S2=200, N1=16, D=128, K=150)
    got = run_gpu(wl, seq_used_q=[wl.S1 + 5, -3], seq_used_k=[wl.S2 + 1, 60])
    assert got["flags"] & sli.SLIKL_DEV_BAD_SEQ_USED
    assert not got["flags"] & sli.SLIKL_DEV_INDEX_OUT_OF_RANGE
    qu, ku = [wl.S1, 0], [wl.S2, 60]
    ref = oracle.grad(wl, seq_used_q=qu, seq_used_k=ku)
    wm = used_masked(wl, qu, ku)
    check_against(wm, got, ref)
    check_exact(wm, got)


def test_seq_used_keeps_the_index_contract_check():
    """An index at or past the batch's whole key range is still flagged in a row in use;
    one inside the range but past seq_used_k is not."""
    wl = si.small(seed=36, layout="BSND", B=1, S1=12, S2=100, N1=16, D=128, K=40)
    idx = wl.idx.clone().reshape(wl.T1, wl.K)
    idx[0, 0] = 99                       # inside the key range, past the used keys: invalid
    fine = si.Workload(**{f: getattr(wl, f) for f in wl.__dataclass_fields__})
    fine.idx = idx.reshape(wl.idx.shape).contiguous()
    assert run_gpu(fine, seq_used_k=[50])["flags"] == 0
    idx[3, 1] = 100                      # past the batch's key range
    bad = si.Workload(**{f: getattr(wl, f) for f in wl.__dataclass_fields__})
    bad.idx = idx.reshape(wl.idx.shape).contiguous()
    assert run_gpu(bad, seq_used_k=[50])["flags"] & sli.SLIKL_DEV_INDEX_OUT_OF_RANGE


# ---------------------------------------------------------------------------
# empty problems (TND): no query rows, or no key rows
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("mode", MODES, ids=MODE_IDS)
def test_no_query_rows(mode):
    """Every query batch empty (T1 = 0; the query-side tensors have no elements and go in as
    NULL): nothing is computed and dk is exactly +0."""
    det, path = mode
    wl = si.small(seed=41, layout="TND", B=2, lens_q=[0, 0], lens_k=[5, 7], N1=16, D=128, K=8)
    assert wl.T1 == 0 and wl.T2 == 12
    got = run_gpu(wl, deterministic=det, dk_path=path)
    assert got["flags"] == 0
    assert got["y"].shape == (0, wl.K) and got["dq"].shape == (0, wl.N1, wl.D)
    assert torch.all(got["dk_raw"].view(torch.int16) == 0)


@pytest.mark.parametrize("det", [False, True], ids=["scatter", "det"])
def test_no_key_rows(det):
    """Every key batch empty (T2 = 0; k and dk go in as NULL): no slot can be valid, so
    softmax_out, dq and dw are exactly 0."""
    wl = si.small(seed=42, layout="TND", B=2, lens_q=[3, 2], lens_k=[0, 0], N1=16, D=128, K=8,
                  pattern="none")
    assert wl.T1 == 5 and wl.T2 == 0
    got = run_gpu(wl, deterministic=det)
    assert got["flags"] == 0
    for name in ("y", "dw", "dq"):
        assert np.all(got[name] == 0.0), name
    ref = oracle.grad(wl)
    for name in ("y", "dw", "dq"):
        assert np.array_equal(got[name], ref[name]), name
