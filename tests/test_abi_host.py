"""Host-side checks of the C ABI: the library loads, exports every entry point that
include/slikl.h declares, and phase 1 validates parameters per the operator's constraints
(aclnnSparseLightningIndexerKLLossGrad, "公共约束" / "规格约束"; return codes after the aclnn
convention). No compute call runs here."""

import ctypes
import os
import re

import pytest
import torch

import sparse_lightning_indexer_b200 as sli
from sparse_lightning_indexer_b200 import build as slibuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    slibuild.build()
    return sli.load_library()


def declared_symbols():
    with open(os.path.join(ROOT, "include", "slikl.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"SLIKL_API\s+[\w\s\*]+?\b(slikl_\w+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert len(names) >= 7
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(sli.EXPORTED) == names


def base_problem(**kw):
    pr = sli.slikl_problem()
    pr.dtype, pr.layout_q, pr.layout_k, pr.deterministic = sli.SLIKL_BF16, sli.SLIKL_BSND, sli.SLIKL_BSND, 0
    pr.B, pr.S1, pr.S2, pr.T1, pr.T2, pr.N1, pr.D, pr.topk = 1, 4096, 4096, 0, 0, 64, 128, 2048
    for k, v in kw.items():
        setattr(pr, k, v)
    return pr


def ws_rc(lib, pr):
    n = ctypes.c_size_t(0)
    return lib.slikl_grad_workspace_size(ctypes.byref(pr), ctypes.byref(n)), n.value


def test_workspace_size_valid(lib):
    rc, n = ws_rc(lib, base_problem())
    assert rc == sli.SLIKL_OK
    # fp32 dk accumulator alone is T2*D*4 bytes
    assert n >= 4096 * 128 * 4
    # deterministic mode on the scatter path: one fp32 dK row per slot
    rc, n_det = ws_ex(lib, base_problem(deterministic=1), "scatter")
    assert rc == sli.SLIKL_OK
    assert n_det >= 4096 * 2048 * 128 * 4
    # ... on the key-major path (auto here): records, the fp32 rows and the per-CTA scratch
    rc, n_km = ws_rc(lib, base_problem(deterministic=1))
    assert rc == sli.SLIKL_OK
    assert 4096 * 4096 * 16 + 4096 * 128 * 4 + 256 * 2 * 256 * 128 * 4 <= n_km < n_det


@pytest.mark.parametrize("field,value", [
    ("dtype", 2), ("layout_q", 2), ("layout_k", -1), ("deterministic", 2), ("B", 0),
    ("N1", 0), ("N1", 129), ("D", 96), ("D", 256), ("topk", 0), ("topk", 8193), ("S1", 0),
    ("S2", 0),
])
def test_workspace_size_rejects(lib, field, value):
    rc, _ = ws_rc(lib, base_problem(**{field: value}))
    assert rc == sli.SLIKL_ERR_PARAM_INVALID


def test_tnd_sizes(lib):
    pr = base_problem(layout_q=sli.SLIKL_TND, layout_k=sli.SLIKL_TND, B=8, S1=0, S2=0,
                      T1=35000, T2=35000, N1=32)
    assert ws_rc(lib, pr)[0] == sli.SLIKL_OK
    assert ws_rc(lib, base_problem(layout_q=sli.SLIKL_TND, T1=-1))[0] == sli.SLIKL_ERR_PARAM_INVALID
    # T1*topk must stay below 2^31
    big = base_problem(layout_q=sli.SLIKL_TND, T1=2 ** 20, topk=4096)
    assert ws_rc(lib, big)[0] == sli.SLIKL_ERR_PARAM_INVALID


def test_null_pointers(lib):
    n = ctypes.c_size_t(0)
    assert lib.slikl_grad_workspace_size(None, ctypes.byref(n)) == sli.SLIKL_ERR_PARAM_NULLPTR
    pr = base_problem()
    assert lib.slikl_grad_workspace_size(ctypes.byref(pr), None) == sli.SLIKL_ERR_INNER_NULLPTR
    tn = sli.slikl_tensors()
    # every tensor NULL -> 161001 before any CUDA call
    assert lib.slikl_grad(ctypes.byref(pr), ctypes.byref(tn), None, 0, None) == sli.SLIKL_ERR_PARAM_NULLPTR
    assert lib.slikl_grad(ctypes.byref(pr), None, None, 0, None) == sli.SLIKL_ERR_PARAM_NULLPTR
    assert lib.slikl_grad(None, ctypes.byref(tn), None, 0, None) == sli.SLIKL_ERR_PARAM_NULLPTR
    flags = ctypes.c_uint32(0)
    assert lib.slikl_read_device_status(None, None, ctypes.byref(flags)) == sli.SLIKL_ERR_PARAM_NULLPTR
    assert lib.slikl_read_device_status(ctypes.c_void_p(256), None, None) == sli.SLIKL_ERR_INNER_NULLPTR


def fake_tensors(tnd_q=False, tnd_k=False):
    """Non-NULL pointers that are never dereferenced by host validation."""
    tn = sli.slikl_tensors()
    for i, (name, _) in enumerate(sli.slikl_tensors._fields_):
        setattr(tn, name, 0x1000 * (i + 1))
    if not tnd_q:
        tn.cu_seqlens_q = None
    if not tnd_k:
        tn.cu_seqlens_k = None
    return tn


def test_tnd_requires_cu_seqlens(lib):
    pr = base_problem(layout_q=sli.SLIKL_TND, T1=100)
    tn = fake_tensors(tnd_q=False)
    assert lib.slikl_grad(ctypes.byref(pr), ctypes.byref(tn), ctypes.c_void_p(1 << 20), 1 << 40,
                          None) == sli.SLIKL_ERR_PARAM_NULLPTR


def test_workspace_checks(lib):
    pr = base_problem()
    tn = fake_tensors()
    _, need = ws_rc(lib, pr)
    # misaligned workspace -> invalid; too small -> 161003 (both before any CUDA call)
    assert lib.slikl_grad(ctypes.byref(pr), ctypes.byref(tn), ctypes.c_void_p((1 << 20) + 8), need,
                          None) == sli.SLIKL_ERR_PARAM_INVALID
    assert lib.slikl_grad(ctypes.byref(pr), ctypes.byref(tn), ctypes.c_void_p(1 << 20), need - 1,
                          None) == sli.SLIKL_ERR_WORKSPACE_TOO_SMALL


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_no_device_is_an_error_not_a_fallback(lib):
    pr = base_problem()
    tn = fake_tensors()
    _, need = ws_rc(lib, pr)
    assert lib.slikl_grad(ctypes.byref(pr), ctypes.byref(tn), ctypes.c_void_p(1 << 20), need,
                          None) == sli.SLIKL_ERR_CUDA


def test_metadata_size_and_strings(lib):
    assert lib.slikl_grad_metadata_size(148) == 8 + 2 * 148
    assert lib.slikl_grad_metadata_size(0) == -1
    assert lib.slikl_grad_metadata_size(4097) == -1
    for code in (0, 161001, 161002, 161003, 561103, 561001, 12345):
        assert len(lib.slikl_status_string(code)) > 0
    pr = base_problem()
    n = ctypes.c_size_t(0)
    assert lib.slikl_grad_metadata_workspace_size(ctypes.byref(pr), ctypes.byref(n)) == 0
    assert 0 < n.value < 4096 * 128 * 4 + 4096 * 64


def dk_path(lib, pr, path=None):
    v = ctypes.c_int32(-1)
    opt = sli.make_options(path) if path is not None else None
    rc = lib.slikl_grad_dk_path(ctypes.byref(pr), ctypes.byref(opt) if opt is not None else None,
                                ctypes.byref(v))
    return rc, v.value


def ws_ex(lib, pr, path):
    n = ctypes.c_size_t(0)
    opt = sli.make_options(path)
    rc = lib.slikl_grad_workspace_size_ex(ctypes.byref(pr), ctypes.byref(opt), ctypes.byref(n))
    return rc, n.value


def test_dk_path_choice(lib):
    # key range (4096) within 16x topk: key-major on auto
    assert dk_path(lib, base_problem()) == (sli.SLIKL_OK, sli.SLIKL_DK_KEYMAJOR)
    assert dk_path(lib, base_problem(), "scatter") == (sli.SLIKL_OK, sli.SLIKL_DK_SCATTER)
    # up to 128 heads on key-major (32-byte records), deterministic mode too
    assert dk_path(lib, base_problem(N1=128)) == (sli.SLIKL_OK, sli.SLIKL_DK_KEYMAJOR)
    assert dk_path(lib, base_problem(deterministic=1)) == (sli.SLIKL_OK, sli.SLIKL_DK_KEYMAJOR)
    # long key ranges: scatter on auto, key-major refused
    for kw in (dict(S2=131072), dict(S2=20000, topk=4096), dict(S2=131072, deterministic=1)):
        assert dk_path(lib, base_problem(**kw)) == (sli.SLIKL_OK, sli.SLIKL_DK_SCATTER), kw
        assert dk_path(lib, base_problem(**kw), "keymajor")[0] == sli.SLIKL_ERR_PARAM_INVALID, kw
    # key range above 16x topk: scatter on auto, key-major still possible on request
    sparse = base_problem(S2=8192, topk=256)
    assert dk_path(lib, sparse) == (sli.SLIKL_OK, sli.SLIKL_DK_SCATTER)
    assert dk_path(lib, sparse, "keymajor") == (sli.SLIKL_OK, sli.SLIKL_DK_KEYMAJOR)
    # TND keys: key-major only with a key-range bound in S2
    tnd = dict(layout_q=sli.SLIKL_TND, layout_k=sli.SLIKL_TND, B=8, T1=35000, T2=35000, N1=32)
    assert dk_path(lib, base_problem(S2=0, **tnd)) == (sli.SLIKL_OK, sli.SLIKL_DK_SCATTER)
    assert dk_path(lib, base_problem(S2=8192, **tnd)) == (sli.SLIKL_OK, sli.SLIKL_DK_KEYMAJOR)
    # unknown path value, NULL output
    assert dk_path(lib, base_problem(), 7)[0] == sli.SLIKL_ERR_PARAM_INVALID
    assert lib.slikl_grad_dk_path(ctypes.byref(base_problem()), None, None) == sli.SLIKL_ERR_INNER_NULLPTR


def test_keymajor_workspace_holds_the_records(lib):
    pr = base_problem()                        # T1 = 4096, S2 = 4096, N1 = 64: 16-byte records
    rc_s, n_s = ws_ex(lib, pr, "scatter")
    rc_k, n_k = ws_ex(lib, pr, "keymajor")
    assert rc_s == rc_k == sli.SLIKL_OK
    assert n_k - n_s >= 4096 * 4096 * 16
    # plus the w-scaled copy of q (T1 x N1 x D elements of the input type): the key-major
    # workspace grows with N1 beyond the records' own growth
    rc_k16, n_k16 = ws_ex(lib, base_problem(N1=16), "keymajor")
    rc_k48, n_k48 = ws_ex(lib, base_problem(N1=48), "keymajor")
    assert rc_k16 == rc_k48 == sli.SLIKL_OK
    assert n_k48 - n_k16 >= 4096 * 32 * 128 * 2 + 4096 * 4096 * (16 - 8)
    assert n_k - n_s >= 4096 * 4096 * 16 + 4096 * 64 * 128 * 2
    pr32 = base_problem(N1=32, S2=1000)        # 8-byte records, rows rounded up to 1024 keys
    rc, n32 = ws_ex(lib, pr32, "keymajor")
    assert rc == sli.SLIKL_OK and n32 - ws_ex(lib, pr32, "scatter")[1] >= 4096 * 1024 * 8
    # deterministic mode: 16-byte records (64-bit fixed-point dI) and no sort buffers
    prd = base_problem(N1=32, S2=1000, deterministic=1)
    rc_d, n_d = ws_ex(lib, prd, "keymajor")
    rc_ds, n_ds = ws_ex(lib, prd, "scatter")
    assert rc_d == rc_ds == sli.SLIKL_OK and n_d >= 4096 * 1024 * 16 and n_d < n_ds
    pr128 = base_problem(N1=128)               # 32-byte records
    rc, n128 = ws_ex(lib, pr128, "keymajor")
    assert rc == sli.SLIKL_OK and n128 - ws_ex(lib, pr128, "scatter")[1] >= 4096 * 4096 * 32
    # the plain size call is the auto path
    assert ws_rc(lib, pr)[1] == n_k


def grad_ex_rc(lib, pr, tn, ws, nbytes, opt):
    return lib.slikl_grad_ex(ctypes.byref(pr), ctypes.byref(tn), ctypes.c_void_p(ws), nbytes, None,
                             ctypes.byref(opt) if opt is not None else None)


def test_grad_ex_host_validation(lib):
    """slikl_grad_ex checks everything the host can see before any CUDA call."""
    pr = base_problem()
    tn = fake_tensors()
    _, need_auto = ws_ex(lib, pr, "auto")
    _, need_scatter = ws_ex(lib, pr, "scatter")
    assert need_auto > need_scatter                   # auto is key-major here: records
    # the workspace must be sized for the path the options select
    assert grad_ex_rc(lib, pr, tn, 1 << 20, need_scatter, sli.make_options("auto")) == \
        sli.SLIKL_ERR_WORKSPACE_TOO_SMALL
    assert grad_ex_rc(lib, pr, tn, 1 << 20, need_auto - 1, None) == sli.SLIKL_ERR_WORKSPACE_TOO_SMALL
    # unknown path, key-major on a problem it cannot run
    assert grad_ex_rc(lib, pr, tn, 1 << 20, need_auto, sli.make_options(5)) == \
        sli.SLIKL_ERR_PARAM_INVALID
    assert grad_ex_rc(lib, base_problem(S2=131072), tn, 1 << 20, 1 << 40,
                      sli.make_options("keymajor")) == sli.SLIKL_ERR_PARAM_INVALID
    # loss output and used-length inputs must be 4-byte aligned
    assert grad_ex_rc(lib, pr, tn, 1 << 20, need_auto, sli.make_options(loss=0x1002)) == \
        sli.SLIKL_ERR_PARAM_INVALID
    assert grad_ex_rc(lib, pr, tn, 1 << 20, need_auto, sli.make_options(seq_used_q=0x1001)) == \
        sli.SLIKL_ERR_PARAM_INVALID
    assert grad_ex_rc(lib, pr, tn, 1 << 20, need_auto, sli.make_options(seq_used_k=0x1003)) == \
        sli.SLIKL_ERR_PARAM_INVALID
    # NULL tensors / workspace
    assert lib.slikl_grad_ex(ctypes.byref(pr), None, None, 0, None, None) == sli.SLIKL_ERR_PARAM_NULLPTR
    assert grad_ex_rc(lib, pr, tn, 0, need_auto, None) == sli.SLIKL_ERR_PARAM_NULLPTR


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_grad_ex_no_device_is_an_error(lib):
    pr = base_problem()
    tn = fake_tensors()
    for path in ("auto", "scatter", "keymajor"):
        _, need = ws_ex(lib, pr, path)
        assert grad_ex_rc(lib, pr, tn, 1 << 20, need, sli.make_options(path)) == sli.SLIKL_ERR_CUDA


def header_struct_fields(struct_name):
    """Field names of a typedef'd struct in include/slikl.h, in declaration order."""
    text = open(os.path.join(ROOT, "include", "slikl.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    body = re.search(r"typedef struct \{([^}]*)\}\s*" + struct_name + ";", text).group(1)
    return [re.search(r"(\w+)\s*(\[[^\]]*\])?\s*$", d.strip()).group(1)
            for d in body.split(";") if d.strip()]


def test_options_struct_layout():
    """The ctypes mirror of slikl_options matches the header's field order and pointer sizes."""
    names = [n for n, _ in sli.slikl_options._fields_]
    assert names == header_struct_fields("slikl_options")
    assert names == ["dk_path", "fused_begin", "fused_end", "dk_begin", "dk_end", "loss",
                     "seq_used_q", "seq_used_k"]
    assert ctypes.sizeof(sli.slikl_options) == 8 + 7 * ctypes.sizeof(ctypes.c_void_p)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks host validation up to the first CUDA call")
def test_empty_tensors_may_be_null(lib):
    """With TND and no query rows (T1 = 0) the query-side tensors may be NULL, with no key rows
    (T2 = 0) k and dk may be; validation then passes and the call reaches the device (which is
    absent here: SLIKL_ERR_CUDA). Non-empty tensors stay required."""
    q_side = ("q", "w", "attn_softmax_l1norm", "sparse_indices", "dq", "dw", "softmax_out")
    pr = base_problem(layout_q=sli.SLIKL_TND, layout_k=sli.SLIKL_TND, B=2, T1=0, T2=50, S2=30)
    need = ws_ex(lib, pr, "auto")[1]
    tn = fake_tensors(tnd_q=True, tnd_k=True)
    for name in q_side:
        setattr(tn, name, None)
    assert grad_ex_rc(lib, pr, tn, 1 << 20, need, None) == sli.SLIKL_ERR_CUDA
    tn.k = None                                          # T2 > 0: k is required
    assert grad_ex_rc(lib, pr, tn, 1 << 20, need, None) == sli.SLIKL_ERR_PARAM_NULLPTR

    pr = base_problem(layout_q=sli.SLIKL_TND, layout_k=sli.SLIKL_TND, B=2, T1=40, T2=0, S2=0)
    need = ws_ex(lib, pr, "auto")[1]
    tn = fake_tensors(tnd_q=True, tnd_k=True)
    tn.k = tn.dk = None
    assert grad_ex_rc(lib, pr, tn, 1 << 20, need, None) == sli.SLIKL_ERR_CUDA
    for name in q_side:                                  # T1 > 0: each query-side tensor required
        tn2 = fake_tensors(tnd_q=True, tnd_k=True)
        tn2.k = tn2.dk = None
        setattr(tn2, name, None)
        assert grad_ex_rc(lib, pr, tn2, 1 << 20, need, None) == sli.SLIKL_ERR_PARAM_NULLPTR, name


def test_binding_rejects_bad_used_lengths():
    """grad() checks the used-length tensors before any CUDA call: int32, on the device,
    contiguous, B entries."""
    q = torch.zeros(6, 16, 128, dtype=torch.bfloat16)
    k = torch.zeros(10, 1, 128, dtype=torch.bfloat16)
    w = torch.zeros(6, 16)
    p = torch.zeros(6, 1, 8)
    idx = torch.full((6, 1, 8), -1, dtype=torch.int32)
    cuq = torch.tensor([0, 2, 6], dtype=torch.int32)
    cuk = torch.tensor([0, 4, 10], dtype=torch.int32)
    bad = [torch.tensor([1, 2], dtype=torch.int64),          # wrong dtype
           torch.tensor([1, 2, 3], dtype=torch.int32),       # wrong length
           torch.tensor([1, 2], dtype=torch.int32)]          # host tensor
    for u in bad:
        for name in ("seq_used_q", "seq_used_k"):
            with pytest.raises(ValueError, match=name):
                sli.grad(q, k, w, p, idx, "TND", "TND", cuq, cuk, **{name: u})


# ---------------------------------------------------------------------------
# dense variant: host-side validation and workspace size (no CUDA call)
# ---------------------------------------------------------------------------

def dense_problem(**kw):
    pr = sli.slikl_dense_problem()
    pr.dtype, pr.layout_q, pr.layout_k = sli.SLIKL_BF16, sli.SLIKL_BSND, sli.SLIKL_BSND
    pr.deterministic = 0
    pr.B, pr.S1, pr.S2, pr.T1, pr.T2, pr.N1, pr.D = 2, 64, 96, 0, 0, 16, 128
    pr.row_len, pr.mask_mode, pr.reserved = 0, 3, 0
    for f, v in kw.items():
        setattr(pr, f, v)
    return pr


def dense_code(pr, opt=None):
    n = ctypes.c_size_t(0)
    return sli.load_library().slikl_dense_grad_workspace_size(
        ctypes.byref(pr), ctypes.byref(opt) if opt is not None else None, ctypes.byref(n)), n.value


def test_dense_validation_codes(lib):
    assert dense_code(dense_problem())[0] == sli.SLIKL_OK
    assert dense_code(dense_problem(mask_mode=0))[0] == sli.SLIKL_OK
    for bad in (dict(mask_mode=1), dict(mask_mode=2), dict(reserved=1), dict(row_len=8193),
                dict(row_len=50), dict(layout_k=sli.SLIKL_TND, row_len=0), dict(N1=129),
                dict(D=96)):
        assert dense_code(dense_problem(**bad))[0] == sli.SLIKL_ERR_PARAM_INVALID, bad
    assert sli.load_library().slikl_dense_grad_workspace_size(None, None, ctypes.byref(ctypes.c_size_t())) \
        == sli.SLIKL_ERR_PARAM_NULLPTR
    assert sli.load_library().slikl_dense_grad_workspace_size(ctypes.byref(dense_problem()), None, None) \
        == sli.SLIKL_ERR_INNER_NULLPTR


def test_dense_workspace_holds_the_index_rows(lib):
    """The dense workspace is the sparse problem's (topk = the row length) plus the index rows
    [T1 x Ld] int32 and a flag word."""
    pr = dense_problem(row_len=128)
    code, dense_bytes = dense_code(pr)
    assert code == sli.SLIKL_OK
    sp = sli.slikl_problem()
    for f in ("dtype", "layout_q", "layout_k", "deterministic", "B", "S1", "S2", "T1", "T2",
              "N1", "D"):
        setattr(sp, f, getattr(pr, f))
    sp.topk = 128
    sparse = sli.slikl_grad_workspace_size(sp)
    T1 = pr.B * pr.S1
    assert dense_bytes >= sparse + T1 * 128 * 4 + 4
    assert dense_bytes <= (sparse + 255) // 256 * 256 + (T1 * 128 * 4 + 255) // 256 * 256 + 256


def test_dense_launch_rejects_bad_arguments_without_a_gpu(lib):
    """Argument errors are found on the host, before any CUDA call."""
    pr = dense_problem()
    tn = sli.slikl_dense_tensors()
    rc = sli.load_library().slikl_dense_grad(ctypes.byref(pr), None, None, 0, None, None)
    assert rc == sli.SLIKL_ERR_PARAM_NULLPTR
    rc = sli.load_library().slikl_dense_grad(ctypes.byref(pr), ctypes.byref(tn), None, 0, None, None)
    assert rc == sli.SLIKL_ERR_PARAM_NULLPTR
    rc = sli.load_library().slikl_dense_grad(ctypes.byref(pr), ctypes.byref(tn), 256, 16, None, None)
    assert rc == sli.SLIKL_ERR_WORKSPACE_TOO_SMALL
    need = dense_code(pr)[1]
    rc = sli.load_library().slikl_dense_grad(ctypes.byref(pr), ctypes.byref(tn), 256, need, None, None)
    assert rc == sli.SLIKL_ERR_PARAM_NULLPTR          # tensors not given


def test_dense_dk_path_query(lib):
    """The dense call's dK path is the sparse operator's choice for top-k = the row length
    (key-major: the key range never exceeds the row length); an unknown request is refused."""
    assert sli.slikl_dense_grad_dk_path(dense_problem()) == sli.SLIKL_DK_KEYMAJOR
    assert sli.slikl_dense_grad_dk_path(dense_problem(N1=128)) == sli.SLIKL_DK_KEYMAJOR
    assert sli.slikl_dense_grad_dk_path(dense_problem(deterministic=1)) == sli.SLIKL_DK_KEYMAJOR
    assert sli.slikl_dense_grad_dk_path(dense_problem(), sli.make_options("scatter")) \
        == sli.SLIKL_DK_SCATTER
    with pytest.raises(sli.SliklError):
        sli.slikl_dense_grad_dk_path(dense_problem(), sli.make_options(7))
    with pytest.raises(sli.SliklError):
        sli.slikl_dense_grad_dk_path(dense_problem(mask_mode=1))
    assert sli.load_library().slikl_dense_grad_dk_path(ctypes.byref(dense_problem()), None, None) \
        == sli.SLIKL_ERR_INNER_NULLPTR


# ---------------------------------------------------------------------------
# variant that forms p from the main attention: host-side checks (no CUDA call)
# ---------------------------------------------------------------------------

def main_attn(**kw):
    m = sli.slikl_main_attention()
    m.Nm, m.Dm, m.scale, m.reserved = 16, 128, 0.125, 0
    for f, v in kw.items():
        setattr(m, f, v)
    return m


def test_recompute_p_workspace_and_validation(lib):
    pr = base_problem()
    opt = sli.make_options("auto")
    assert sli.slikl_grad_recompute_p_workspace_size(pr, main_attn(), opt) == \
        sli.slikl_grad_workspace_size_ex(pr, opt)
    n = ctypes.c_size_t(0)
    for bad in (dict(Nm=0), dict(Nm=129), dict(Dm=96), dict(reserved=1),
                dict(scale=float("nan")), dict(scale=float("inf"))):
        rc = lib.slikl_grad_recompute_p_workspace_size(
            ctypes.byref(pr), ctypes.byref(main_attn(**bad)), None, ctypes.byref(n))
        assert rc == sli.SLIKL_ERR_PARAM_INVALID, bad
    assert lib.slikl_grad_recompute_p_workspace_size(ctypes.byref(pr), None, None,
                                                     ctypes.byref(n)) == sli.SLIKL_ERR_PARAM_NULLPTR


def test_recompute_p_launch_rejects_bad_arguments_without_a_gpu(lib):
    pr = base_problem()
    m = main_attn()
    tn = fake_tensors()
    need = sli.slikl_grad_recompute_p_workspace_size(pr, m)

    def rc(q_main, k_main, p_out, tensors=tn, ws=1 << 20, nbytes=need):
        return lib.slikl_grad_recompute_p(ctypes.byref(pr), ctypes.byref(m),
                                          ctypes.byref(tensors) if tensors is not None else None,
                                          q_main, k_main, p_out, ws, nbytes, None, None)

    assert rc(0x1000, 0x2000, 0x3000, tensors=None) == sli.SLIKL_ERR_PARAM_NULLPTR
    assert rc(None, 0x2000, 0x3000) == sli.SLIKL_ERR_PARAM_NULLPTR
    assert rc(0x1000, None, 0x3000) == sli.SLIKL_ERR_PARAM_NULLPTR
    assert rc(0x1000, 0x2000, None) == sli.SLIKL_ERR_PARAM_NULLPTR
    assert rc(0x1008, 0x2000, 0x3000) == sli.SLIKL_ERR_PARAM_INVALID      # q_main not 16-aligned
    assert rc(0x1000, 0x2000, 0x3002) == sli.SLIKL_ERR_PARAM_INVALID      # p_out not 4-aligned
    assert rc(0x1000, 0x2000, 0x3000, nbytes=need - 1) == sli.SLIKL_ERR_WORKSPACE_TOO_SMALL
