"""The C ABI from a plain C99 caller (tests/c_caller.c), on the host.

The header must compile as strict C (-std=c99 -pedantic -Werror), the struct layouts the C
compiler produces must be the ones the Python binding mirrors with ctypes, and phase-1 calls
made from C must give the same answers as the same calls made through the binding.
"""

import ctypes
import os
import shutil
import subprocess

import pytest

import sparse_lightning_indexer_b200 as sli

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "sparse_lightning_indexer_b200")

pytestmark = pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")

# dtype, layout, B, S1, S2, T1, T2, N1, D, topk, deterministic, dk_path
PROBLEMS = [
    (sli.SLIKL_BF16, sli.SLIKL_BSND, 1, 4096, 4096, 0, 0, 64, 128, 2048, 0, sli.SLIKL_DK_AUTO),
    (sli.SLIKL_BF16, sli.SLIKL_BSND, 1, 4096, 4096, 0, 0, 64, 128, 2048, 0, sli.SLIKL_DK_SCATTER),
    (sli.SLIKL_FP16, sli.SLIKL_TND, 8, 0, 8192, 34816, 34816, 32, 128, 2048, 0, sli.SLIKL_DK_AUTO),
    (sli.SLIKL_BF16, sli.SLIKL_BSND, 4, 8192, 8192, 0, 0, 16, 128, 512, 1, sli.SLIKL_DK_AUTO),
    (sli.SLIKL_BF16, sli.SLIKL_BSND, 1, 256, 256, 0, 0, 8, 64, 64, 0, sli.SLIKL_DK_KEYMAJOR),
    (sli.SLIKL_BF16, sli.SLIKL_BSND, 1, 64, 64, 0, 0, 200, 128, 64, 0, sli.SLIKL_DK_AUTO),  # N1 too large
    # key-major asked for on a key range above its limit
    (sli.SLIKL_BF16, sli.SLIKL_BSND, 1, 64, 131072, 0, 0, 128, 128, 64, 1, sli.SLIKL_DK_KEYMAJOR),
]


@pytest.fixture(scope="module")
def c_output(tmp_path_factory):
    lib = sli.load_library()
    libdir = os.path.dirname(lib._name)
    exe = str(tmp_path_factory.mktemp("c_caller") / "c_caller")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_caller.c"),
                    "-o", exe, "-L", libdir, "-lslikl", "-Wl,-rpath," + libdir],
                   check=True, capture_output=True, text=True)
    args = [",".join(str(int(v)) for v in p) for p in PROBLEMS]
    out = subprocess.run([exe, *args], check=True, capture_output=True, text=True).stdout
    return out.splitlines()


def test_struct_layouts_match_the_binding(c_output):
    mirrors = {"slikl_problem": sli.slikl_problem, "slikl_tensors": sli.slikl_tensors,
               "slikl_options": sli.slikl_options,
               "slikl_dense_problem": sli.slikl_dense_problem,
               "slikl_dense_tensors": sli.slikl_dense_tensors,
               "slikl_main_attention": sli.slikl_main_attention}
    seen = set()
    for line in c_output:
        parts = line.split()
        if parts[0] == "size":
            assert ctypes.sizeof(mirrors[parts[1]]) == int(parts[2]), parts[1]
        elif parts[0] == "field":
            cls = mirrors[parts[1]]
            assert getattr(cls, parts[2]).offset == int(parts[3]), (parts[1], parts[2])
            seen.add((parts[1], parts[2]))
    for name, cls in mirrors.items():
        assert {(name, f) for f, _ in cls._fields_} == {s for s in seen if s[0] == name}


def make_problem(p):
    pr = sli.slikl_problem()
    pr.dtype, pr.layout_q, pr.layout_k = p[0], p[1], p[1]
    pr.B, pr.S1, pr.S2, pr.T1, pr.T2 = p[2], p[3], p[4], p[5], p[6]
    pr.N1, pr.D, pr.topk, pr.deterministic = p[7], p[8], p[9], p[10]
    return pr


def test_phase_one_from_c_matches_the_binding(c_output):
    lib = sli.load_library()
    rows = [line.split()[1:] for line in c_output if line.startswith("problem ")]
    assert len(rows) == len(PROBLEMS)
    for p, row in zip(PROBLEMS, rows):
        rc_plain, rc_ex, rc_path, plain, ex, path = (int(x) for x in row)
        pr = make_problem(p)
        opt = sli.slikl_options()
        opt.dk_path = p[11]
        n = ctypes.c_size_t(0)
        assert lib.slikl_grad_workspace_size(ctypes.byref(pr), ctypes.byref(n)) == rc_plain
        if rc_plain == sli.SLIKL_OK:
            assert n.value == plain
        n2 = ctypes.c_size_t(0)
        assert lib.slikl_grad_workspace_size_ex(ctypes.byref(pr), ctypes.byref(opt),
                                                ctypes.byref(n2)) == rc_ex
        if rc_ex == sli.SLIKL_OK:
            assert n2.value == ex
        got = ctypes.c_int32(-1)
        assert lib.slikl_grad_dk_path(ctypes.byref(pr), ctypes.byref(opt), ctypes.byref(got)) == rc_path
        if rc_path == sli.SLIKL_OK:
            assert got.value == path
    # the cases cover success, the plain call equal to the auto path, and both rejections
    assert rows[0][0] == "0" and rows[0][3] == rows[0][4]
    assert rows[5][0] == str(sli.SLIKL_ERR_PARAM_INVALID)
    assert rows[6][1] == str(sli.SLIKL_ERR_PARAM_INVALID)


def test_status_string_from_c(c_output):
    line = [ln for ln in c_output if ln.startswith("status ")][0]
    code, text = line.split(" ", 2)[1:]
    assert int(code) == sli.SLIKL_ERR_PARAM_INVALID
    assert text == sli.status_string(sli.SLIKL_ERR_PARAM_INVALID)
