"""slikl_grad_noalloc: the entry point for callers that cannot allocate device memory when
they call. It must give the same results as slikl_grad (which takes a caller-owned
workspace) on the same inputs, call after call, while reusing the library's one fixed
device scratch array. This file is collected last so that a run that stops at the first
failure has already run every other test."""

import ctypes

import numpy as np
import pytest
import torch

import slikl_inputs as si
import sparse_lightning_indexer_b200 as sli

pytestmark = pytest.mark.gpu

TOL = {"softmax_out": (1e-5, None), "dw": (1e-4, None), "dq": (5e-3, 2e-2), "dk": (5e-3, 2e-2)}


def rel_l2(a, b):
    n = np.linalg.norm(b)
    return np.linalg.norm(a - b) / n if n > 0 else float(np.linalg.norm(a))


def check_close(name, got, ref):
    got = got.double().cpu().numpy()
    ref = ref.double().cpu().numpy()
    rtol, mtol = TOL[name]
    assert rel_l2(got, ref) <= rtol, name
    if mtol is not None:
        assert np.abs(got - ref).max() <= mtol * max(np.abs(ref).max(), 1e-30), name


def device_tensors(wl):
    dev = torch.device("cuda")
    return {n: getattr(wl, n).to(dev) for n in ("q", "k", "w", "p", "idx")}


def outputs_like(t):
    return dict(dq=torch.empty_like(t["q"]), dk=torch.empty_like(t["k"]),
                dw=torch.empty_like(t["w"]), softmax_out=torch.empty_like(t["p"]))


def struct(t, o):
    tn = sli.slikl_tensors()
    tn.q, tn.k, tn.w = t["q"].data_ptr(), t["k"].data_ptr(), t["w"].data_ptr()
    tn.attn_softmax_l1norm, tn.sparse_indices = t["p"].data_ptr(), t["idx"].data_ptr()
    tn.dq, tn.dk, tn.dw, tn.softmax_out = (o["dq"].data_ptr(), o["dk"].data_ptr(),
                                           o["dw"].data_ptr(), o["softmax_out"].data_ptr())
    return tn


@pytest.mark.parametrize("cfg", ["small", "config0"])
def test_noalloc_matches_slikl_grad_on_two_calls_in_a_row(cfg):
    if cfg == "small":
        wl = si.small(seed=31, layout="BSND", B=2, S1=40, S2=700, N1=64, D=128, K=384,
                      qk_scale=0.1, w_var=1 / 64, invalid_frac=0.2)
    else:
        wl = si.config(0)
    t = device_tensors(wl)
    pr = sli.make_problem(t["q"], t["k"], t["idx"], "BSND", "BSND", False)
    # reference: the workspace entry point
    ref = outputs_like(t)
    ws = torch.empty(sli.slikl_grad_workspace_size(pr), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    sli.slikl_grad(pr, struct(t, ref), ws.data_ptr(), ws.numel(), stream)
    torch.cuda.synchronize()
    for call in range(2):
        got = outputs_like(t)
        for o in got.values():
            o.fill_(7)                      # stale values must be overwritten
        sli.slikl_grad_noalloc(pr, struct(t, got), stream)
        torch.cuda.synchronize()
        for name in ("softmax_out", "dw", "dq", "dk"):
            check_close(name, got[name], ref[name])
        assert torch.equal(got["softmax_out"], ref["softmax_out"])


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = sli.load_library()
    pr = sli.slikl_problem()
    pr.dtype, pr.layout_q, pr.layout_k, pr.deterministic = sli.SLIKL_BF16, sli.SLIKL_BSND, sli.SLIKL_BSND, 0
    pr.B, pr.S1, pr.S2, pr.N1, pr.D, pr.topk = 1, 1024, 131072, 64, 128, 2048
    tn = sli.slikl_tensors()
    # T2 * D * 4 bytes of fp32 accumulator alone exceed the fixed scratch
    assert lib.slikl_grad_noalloc(ctypes.byref(pr), ctypes.byref(tn), None) == sli.SLIKL_ERR_WORKSPACE_TOO_SMALL
    pr.S2, pr.deterministic = 1024, 1
    assert lib.slikl_grad_noalloc(ctypes.byref(pr), ctypes.byref(tn), None) == sli.SLIKL_ERR_PARAM_INVALID
