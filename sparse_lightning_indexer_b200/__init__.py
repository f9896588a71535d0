"""Python binding of the sm_100a sparse Lightning Indexer KL-loss backward library.

Argument marshalling only: every step of the operator runs in the CUDA kernels of
``libslikl.so`` behind the C ABI declared in ``include/slikl.h``. The functions here keep
the C names (``slikl_grad_workspace_size``, ``slikl_grad``, ...) and take ctypes structs;
``grad()`` is a convenience wrapper that allocates outputs and the workspace with torch and
calls through the same ABI. There is no CPU fallback: if the library is missing or no
sm_100 device is present the calls raise.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libslikl.so")

SLIKL_OK = 0
SLIKL_ERR_PARAM_NULLPTR = 161001
SLIKL_ERR_PARAM_INVALID = 161002
SLIKL_ERR_WORKSPACE_TOO_SMALL = 161003
SLIKL_ERR_INNER_NULLPTR = 561103
SLIKL_ERR_CUDA = 561001

SLIKL_FP16 = 0
SLIKL_BF16 = 1
SLIKL_BSND = 0
SLIKL_TND = 1

SLIKL_DEV_INDEX_OUT_OF_RANGE = 0x1
SLIKL_DEV_BAD_CU_SEQLENS_Q = 0x2
SLIKL_DEV_BAD_CU_SEQLENS_K = 0x4
SLIKL_DEV_WAIT_TIMEOUT = 0x8
SLIKL_DEV_KEY_RANGE_ABOVE_S2 = 0x10
SLIKL_DEV_BAD_SEQ_USED = 0x20
SLIKL_DEV_ROW_LEN_BELOW_KEYS = 0x40

SLIKL_DK_AUTO = 0
SLIKL_DK_SCATTER = 1
SLIKL_DK_KEYMAJOR = 2
_DK_PATHS = {"auto": SLIKL_DK_AUTO, "scatter": SLIKL_DK_SCATTER, "keymajor": SLIKL_DK_KEYMAJOR}

EXPORTED = ("slikl_grad_workspace_size", "slikl_grad", "slikl_grad_with_events",
            "slikl_grad_workspace_size_ex", "slikl_grad_ex", "slikl_grad_dk_path",
            "slikl_read_device_status",
            "slikl_grad_metadata_size", "slikl_grad_metadata_workspace_size",
            "slikl_grad_metadata", "slikl_status_string", "slikl_grad_noalloc",
            "slikl_dense_grad_workspace_size", "slikl_dense_grad", "slikl_dense_grad_dk_path",
            "slikl_grad_recompute_p_workspace_size", "slikl_grad_recompute_p")

SLIKL_NOALLOC_SCRATCH_BYTES = 32 << 20


class slikl_problem(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int32), ("layout_q", ctypes.c_int32),
                ("layout_k", ctypes.c_int32), ("deterministic", ctypes.c_int32),
                ("B", ctypes.c_int64), ("S1", ctypes.c_int64), ("S2", ctypes.c_int64),
                ("T1", ctypes.c_int64), ("T2", ctypes.c_int64), ("N1", ctypes.c_int64),
                ("D", ctypes.c_int64), ("topk", ctypes.c_int64)]


class slikl_tensors(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in
                ("q", "k", "w", "attn_softmax_l1norm", "sparse_indices", "cu_seqlens_q",
                 "cu_seqlens_k", "dq", "dk", "dw", "softmax_out")]


class slikl_dense_problem(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int32), ("layout_q", ctypes.c_int32),
                ("layout_k", ctypes.c_int32), ("deterministic", ctypes.c_int32),
                ("B", ctypes.c_int64), ("S1", ctypes.c_int64), ("S2", ctypes.c_int64),
                ("T1", ctypes.c_int64), ("T2", ctypes.c_int64), ("N1", ctypes.c_int64),
                ("D", ctypes.c_int64), ("row_len", ctypes.c_int64), ("mask_mode", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class slikl_dense_tensors(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in
                ("q", "k", "w", "attn_softmax_l1norm", "cu_seqlens_q", "cu_seqlens_k", "dq",
                 "dk", "dw", "softmax_out")]


class slikl_main_attention(ctypes.Structure):
    _fields_ = [("Nm", ctypes.c_int32), ("Dm", ctypes.c_int32), ("scale", ctypes.c_float),
                ("reserved", ctypes.c_int32)]


class slikl_options(ctypes.Structure):
    _fields_ = [("dk_path", ctypes.c_int32), ("fused_begin", ctypes.c_void_p),
                ("fused_end", ctypes.c_void_p), ("dk_begin", ctypes.c_void_p),
                ("dk_end", ctypes.c_void_p), ("loss", ctypes.c_void_p),
                ("seq_used_q", ctypes.c_void_p), ("seq_used_k", ctypes.c_void_p)]


def make_options(dk_path="auto", fused_begin: int = 0, fused_end: int = 0, dk_begin: int = 0,
                 dk_end: int = 0, loss: int = 0, seq_used_q: int = 0,
                 seq_used_k: int = 0) -> slikl_options:
    """Options of slikl_grad_ex; the event arguments are cudaEvent_t handles (ints) or 0;
    `loss` is the device address of an fp32 [T1] output for the per-row KL loss, or 0;
    `seq_used_q` / `seq_used_k` are device addresses of int32 [B] used lengths, or 0."""
    o = slikl_options()
    o.dk_path = _DK_PATHS[dk_path] if isinstance(dk_path, str) else int(dk_path)
    o.fused_begin = fused_begin or None
    o.fused_end = fused_end or None
    o.dk_begin = dk_begin or None
    o.dk_end = dk_end or None
    o.loss = loss or None
    o.seq_used_q = seq_used_q or None
    o.seq_used_k = seq_used_k or None
    return o


class SliklError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} ({code})")


_lib = None


def load_library() -> ctypes.CDLL:
    """Load libslikl.so (built by sparse_lightning_indexer_b200.build). Raises if missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run python -m sparse_lightning_indexer_b200.build")
        lib = ctypes.CDLL(LIB_PATH)
        P, VP = ctypes.POINTER, ctypes.c_void_p
        lib.slikl_grad_workspace_size.argtypes = [P(slikl_problem), P(ctypes.c_size_t)]
        lib.slikl_grad.argtypes = [P(slikl_problem), P(slikl_tensors), VP, ctypes.c_size_t, VP]
        lib.slikl_grad_with_events.argtypes = [P(slikl_problem), P(slikl_tensors), VP,
                                               ctypes.c_size_t, VP, VP, VP]
        lib.slikl_grad_workspace_size_ex.argtypes = [P(slikl_problem), P(slikl_options),
                                                     P(ctypes.c_size_t)]
        lib.slikl_grad_ex.argtypes = [P(slikl_problem), P(slikl_tensors), VP, ctypes.c_size_t,
                                      VP, P(slikl_options)]
        lib.slikl_grad_dk_path.argtypes = [P(slikl_problem), P(slikl_options), P(ctypes.c_int32)]
        lib.slikl_grad_dk_path.restype = ctypes.c_int32
        lib.slikl_read_device_status.argtypes = [VP, VP, P(ctypes.c_uint32)]
        lib.slikl_grad_metadata_size.argtypes = [ctypes.c_int32]
        lib.slikl_grad_metadata_size.restype = ctypes.c_int64
        lib.slikl_grad_metadata_workspace_size.argtypes = [P(slikl_problem), P(ctypes.c_size_t)]
        lib.slikl_grad_metadata.argtypes = [P(slikl_problem), P(slikl_tensors), ctypes.c_int32,
                                            ctypes.c_int32, VP, VP, ctypes.c_size_t, VP]
        lib.slikl_grad_noalloc.argtypes = [P(slikl_problem), P(slikl_tensors), VP]
        lib.slikl_grad_noalloc.restype = ctypes.c_int32
        lib.slikl_dense_grad_workspace_size.argtypes = [P(slikl_dense_problem), P(slikl_options),
                                                        P(ctypes.c_size_t)]
        lib.slikl_dense_grad_workspace_size.restype = ctypes.c_int32
        lib.slikl_dense_grad.argtypes = [P(slikl_dense_problem), P(slikl_dense_tensors), VP,
                                         ctypes.c_size_t, VP, P(slikl_options)]
        lib.slikl_dense_grad.restype = ctypes.c_int32
        lib.slikl_dense_grad_dk_path.argtypes = [P(slikl_dense_problem), P(slikl_options),
                                                 P(ctypes.c_int32)]
        lib.slikl_dense_grad_dk_path.restype = ctypes.c_int32
        lib.slikl_grad_recompute_p_workspace_size.argtypes = [
            P(slikl_problem), P(slikl_main_attention), P(slikl_options), P(ctypes.c_size_t)]
        lib.slikl_grad_recompute_p_workspace_size.restype = ctypes.c_int32
        lib.slikl_grad_recompute_p.argtypes = [P(slikl_problem), P(slikl_main_attention),
                                               P(slikl_tensors), VP, VP, VP, VP, ctypes.c_size_t,
                                               VP, P(slikl_options)]
        lib.slikl_grad_recompute_p.restype = ctypes.c_int32
        lib.slikl_status_string.argtypes = [ctypes.c_int32]
        lib.slikl_status_string.restype = ctypes.c_char_p
        for name in ("slikl_grad_workspace_size", "slikl_grad", "slikl_grad_with_events",
                     "slikl_grad_workspace_size_ex", "slikl_grad_ex", "slikl_read_device_status",
                     "slikl_grad_metadata_workspace_size", "slikl_grad_metadata"):
            getattr(lib, name).restype = ctypes.c_int32
        _lib = lib
    return _lib


def status_string(code: int) -> str:
    return load_library().slikl_status_string(int(code)).decode()


# --- C names, marshalling only -------------------------------------------------------

def slikl_grad_workspace_size(problem: slikl_problem) -> int:
    n = ctypes.c_size_t(0)
    rc = load_library().slikl_grad_workspace_size(ctypes.byref(problem), ctypes.byref(n))
    if rc != SLIKL_OK:
        raise SliklError(rc, "slikl_grad_workspace_size")
    return int(n.value)


def slikl_grad(problem: slikl_problem, tensors: slikl_tensors, workspace: int,
               workspace_bytes: int, stream: int = 0) -> None:
    rc = load_library().slikl_grad(ctypes.byref(problem), ctypes.byref(tensors), workspace,
                                   workspace_bytes, stream)
    if rc != SLIKL_OK:
        raise SliklError(rc, "slikl_grad")


def slikl_grad_with_events(problem: slikl_problem, tensors: slikl_tensors, workspace: int,
                           workspace_bytes: int, stream: int = 0, fused_begin: int = 0,
                           fused_end: int = 0) -> None:
    rc = load_library().slikl_grad_with_events(ctypes.byref(problem), ctypes.byref(tensors),
                                               workspace, workspace_bytes, stream,
                                               fused_begin or None, fused_end or None)
    if rc != SLIKL_OK:
        raise SliklError(rc, "slikl_grad_with_events")


def slikl_grad_workspace_size_ex(problem: slikl_problem, options: Optional[slikl_options]) -> int:
    n = ctypes.c_size_t(0)
    rc = load_library().slikl_grad_workspace_size_ex(
        ctypes.byref(problem), ctypes.byref(options) if options is not None else None,
        ctypes.byref(n))
    if rc != SLIKL_OK:
        raise SliklError(rc, "slikl_grad_workspace_size_ex")
    return int(n.value)


def slikl_grad_ex(problem: slikl_problem, tensors: slikl_tensors, workspace: int,
                  workspace_bytes: int, stream: int = 0,
                  options: Optional[slikl_options] = None) -> None:
    rc = load_library().slikl_grad_ex(ctypes.byref(problem), ctypes.byref(tensors), workspace,
                                      workspace_bytes, stream,
                                      ctypes.byref(options) if options is not None else None)
    if rc != SLIKL_OK:
        raise SliklError(rc, "slikl_grad_ex")


def slikl_grad_dk_path(problem: slikl_problem, options: Optional[slikl_options] = None) -> int:
    """SLIKL_DK_SCATTER or SLIKL_DK_KEYMAJOR: the dK path slikl_grad_ex would take."""
    v = ctypes.c_int32(0)
    rc = load_library().slikl_grad_dk_path(
        ctypes.byref(problem), ctypes.byref(options) if options is not None else None,
        ctypes.byref(v))
    if rc != SLIKL_OK:
        raise SliklError(rc, "slikl_grad_dk_path")
    return int(v.value)


def slikl_read_device_status(workspace: int, stream: int = 0) -> int:
    flags = ctypes.c_uint32(0)
    rc = load_library().slikl_read_device_status(workspace, stream, ctypes.byref(flags))
    if rc != SLIKL_OK:
        raise SliklError(rc, "slikl_read_device_status")
    return int(flags.value)


def slikl_grad_noalloc(problem: slikl_problem, tensors: slikl_tensors, stream: int = 0) -> None:
    """slikl_grad with the library's fixed device scratch array instead of a caller workspace
    (for callers that cannot allocate device memory when they call)."""
    rc = load_library().slikl_grad_noalloc(ctypes.byref(problem), ctypes.byref(tensors), stream)
    if rc != SLIKL_OK:
        raise SliklError(rc, "slikl_grad_noalloc")


def slikl_dense_grad_workspace_size(problem: slikl_dense_problem,
                                    options: Optional[slikl_options] = None) -> int:
    n = ctypes.c_size_t(0)
    rc = load_library().slikl_dense_grad_workspace_size(
        ctypes.byref(problem), ctypes.byref(options) if options is not None else None,
        ctypes.byref(n))
    if rc != SLIKL_OK:
        raise SliklError(rc, "slikl_dense_grad_workspace_size")
    return int(n.value)


def slikl_dense_grad_dk_path(problem: slikl_dense_problem,
                             options: Optional[slikl_options] = None) -> int:
    """SLIKL_DK_SCATTER or SLIKL_DK_KEYMAJOR: the dK path slikl_dense_grad would take."""
    v = ctypes.c_int32(0)
    rc = load_library().slikl_dense_grad_dk_path(
        ctypes.byref(problem), ctypes.byref(options) if options is not None else None,
        ctypes.byref(v))
    if rc != SLIKL_OK:
        raise SliklError(rc, "slikl_dense_grad_dk_path")
    return int(v.value)


def slikl_dense_grad(problem: slikl_dense_problem, tensors: slikl_dense_tensors, workspace: int,
                     workspace_bytes: int, stream: int = 0,
                     options: Optional[slikl_options] = None) -> None:
    rc = load_library().slikl_dense_grad(ctypes.byref(problem), ctypes.byref(tensors), workspace,
                                         workspace_bytes, stream,
                                         ctypes.byref(options) if options is not None else None)
    if rc != SLIKL_OK:
        raise SliklError(rc, "slikl_dense_grad")


def slikl_grad_metadata_size(num_workers: int) -> int:
    return int(load_library().slikl_grad_metadata_size(num_workers))


def slikl_grad_metadata_workspace_size(problem: slikl_problem) -> int:
    n = ctypes.c_size_t(0)
    rc = load_library().slikl_grad_metadata_workspace_size(ctypes.byref(problem), ctypes.byref(n))
    if rc != SLIKL_OK:
        raise SliklError(rc, "slikl_grad_metadata_workspace_size")
    return int(n.value)


def slikl_grad_metadata(problem: slikl_problem, tensors: slikl_tensors, num_workers: int,
                        mode: int, metadata: int, workspace: int, workspace_bytes: int,
                        stream: int = 0) -> None:
    rc = load_library().slikl_grad_metadata(ctypes.byref(problem), ctypes.byref(tensors),
                                            num_workers, mode, metadata, workspace,
                                            workspace_bytes, stream)
    if rc != SLIKL_OK:
        raise SliklError(rc, "slikl_grad_metadata")


# --- torch convenience ------------------------------------------------------------------

_DT = {torch.bfloat16: SLIKL_BF16, torch.float16: SLIKL_FP16}


def make_problem(q: torch.Tensor, k: torch.Tensor, sparse_indices: torch.Tensor,
                 layout_q: str = "BSND", layout_k: str = "BSND", deterministic: bool = False,
                 B: Optional[int] = None, key_range_bound: int = 0) -> slikl_problem:
    """Problem struct from tensor shapes (BSND q [B,S1,N1,D]; TND q [T1,N1,D]).

    For TND keys, `key_range_bound` (> 0) promises that no batch has more key rows; it goes
    to problem.S2 and lets the key-major dK path run."""
    pr = slikl_problem()
    if q.dtype not in _DT or k.dtype != q.dtype:
        raise ValueError("q and k must share dtype float16 or bfloat16")
    pr.dtype = _DT[q.dtype]
    pr.layout_q = SLIKL_BSND if layout_q == "BSND" else SLIKL_TND
    pr.layout_k = SLIKL_BSND if layout_k == "BSND" else SLIKL_TND
    pr.deterministic = 1 if deterministic else 0
    if layout_q == "BSND":
        pr.B, pr.S1, pr.N1, pr.D = q.shape
        pr.T1 = pr.B * pr.S1
    else:
        pr.T1, pr.N1, pr.D = q.shape
        if B is None:
            raise ValueError("TND needs B (len(cu_seqlens) - 1)")
        pr.B = B
    if layout_k == "BSND":
        pr.S2 = k.shape[1]
        pr.T2 = k.shape[0] * k.shape[1]
    else:
        pr.T2 = k.shape[0]
        pr.S2 = int(key_range_bound)
    pr.topk = sparse_indices.shape[-1]
    return pr


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("tensors must be contiguous CUDA tensors")
    return t.data_ptr()


def grad(q, k, w, attn_softmax_l1norm, sparse_indices, layout_q="BSND", layout_k="BSND",
         cu_seqlens_q=None, cu_seqlens_k=None, deterministic=False, stream=None, out=None,
         workspace=None, dk_path="auto", key_range_bound=0, loss=False, seq_used_q=None,
         seq_used_k=None):
    """Run slikl_grad_ex on CUDA tensors. Returns dict(dq, dk, dw, softmax_out, workspace).

    `out` may supply preallocated dq/dk/dw/softmax_out, `workspace` a uint8 CUDA buffer;
    `dk_path` is "auto", "scatter" or "keymajor"; `key_range_bound` as in make_problem;
    `loss=True` also returns the per-row KL loss (fp32 [T1]) as res["loss"];
    `seq_used_q` / `seq_used_k` are optional int32 [B] CUDA tensors of the query / key rows of
    each batch in use (rows past them are padding).
    """
    B = None
    if layout_q == "TND":
        B = cu_seqlens_q.numel() - 1
    elif layout_k == "TND":
        B = cu_seqlens_k.numel() - 1
    pr = make_problem(q, k, sparse_indices, layout_q, layout_k, deterministic, B,
                      key_range_bound)
    loss_t = torch.empty(pr.T1, dtype=torch.float32, device=q.device) if loss else None
    for name, u in (("seq_used_q", seq_used_q), ("seq_used_k", seq_used_k)):
        if u is not None and (u.dtype != torch.int32 or not u.is_cuda or not u.is_contiguous()
                              or u.numel() != pr.B):
            raise ValueError(f"{name} must be a contiguous int32 CUDA tensor of B entries")
    opt = make_options(dk_path, loss=loss_t.data_ptr() if loss_t is not None else 0,
                       seq_used_q=_ptr(seq_used_q) or 0, seq_used_k=_ptr(seq_used_k) or 0)
    nbytes = slikl_grad_workspace_size_ex(pr, opt)
    if workspace is None or workspace.numel() < nbytes:
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device)
    if out is None:
        out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k),
                   dw=torch.empty_like(w), softmax_out=torch.empty_like(attn_softmax_l1norm))
    tn = slikl_tensors()
    tn.q, tn.k, tn.w = _ptr(q), _ptr(k), _ptr(w)
    tn.attn_softmax_l1norm = _ptr(attn_softmax_l1norm)
    tn.sparse_indices = _ptr(sparse_indices)
    tn.cu_seqlens_q = _ptr(cu_seqlens_q) if layout_q == "TND" else None
    tn.cu_seqlens_k = _ptr(cu_seqlens_k) if layout_k == "TND" else None
    tn.dq, tn.dk, tn.dw = _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dw"])
    tn.softmax_out = _ptr(out["softmax_out"])
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    slikl_grad_ex(pr, tn, workspace.data_ptr(), workspace.numel(), s.cuda_stream, opt)
    res = dict(out)
    res["workspace"] = workspace
    if loss_t is not None:
        res["loss"] = loss_t
    return res


def slikl_grad_recompute_p_workspace_size(problem: slikl_problem, main: slikl_main_attention,
                                          options: Optional[slikl_options] = None) -> int:
    n = ctypes.c_size_t(0)
    rc = load_library().slikl_grad_recompute_p_workspace_size(
        ctypes.byref(problem), ctypes.byref(main),
        ctypes.byref(options) if options is not None else None, ctypes.byref(n))
    if rc != SLIKL_OK:
        raise SliklError(rc, "slikl_grad_recompute_p_workspace_size")
    return int(n.value)


def slikl_grad_recompute_p(problem: slikl_problem, main: slikl_main_attention,
                           tensors: slikl_tensors, q_main: int, k_main: int, p_out: int,
                           workspace: int, workspace_bytes: int, stream: int = 0,
                           options: Optional[slikl_options] = None) -> None:
    rc = load_library().slikl_grad_recompute_p(
        ctypes.byref(problem), ctypes.byref(main), ctypes.byref(tensors), q_main, k_main, p_out,
        workspace, workspace_bytes, stream, ctypes.byref(options) if options is not None else None)
    if rc != SLIKL_OK:
        raise SliklError(rc, "slikl_grad_recompute_p")


def make_main_attention(q_main: torch.Tensor, scale: float) -> slikl_main_attention:
    """Main-attention shape from q_main [.., Nm, Dm] and the softmax scale."""
    m = slikl_main_attention()
    m.Nm, m.Dm = int(q_main.shape[-2]), int(q_main.shape[-1])
    m.scale = float(scale)
    m.reserved = 0
    return m


def grad_recompute_p(q, k, w, sparse_indices, q_main, k_main, scale, layout_q="BSND",
                     layout_k="BSND", cu_seqlens_q=None, cu_seqlens_k=None, deterministic=False,
                     stream=None, workspace=None, dk_path="auto", key_range_bound=0, loss=False,
                     seq_used_q=None, seq_used_k=None):
    """Run slikl_grad_recompute_p on CUDA tensors: p from the main attention (q_main
    [.., Nm, Dm], k_main [.., 1, Dm], softmax scale), then the backward with it.
    Returns dict(dq, dk, dw, softmax_out, p, workspace[, loss])."""
    B = None
    if layout_q == "TND":
        B = cu_seqlens_q.numel() - 1
    elif layout_k == "TND":
        B = cu_seqlens_k.numel() - 1
    pr = make_problem(q, k, sparse_indices, layout_q, layout_k, deterministic, B,
                      key_range_bound)
    main = make_main_attention(q_main, scale)
    loss_t = torch.empty(pr.T1, dtype=torch.float32, device=q.device) if loss else None
    opt = make_options(dk_path, loss=loss_t.data_ptr() if loss_t is not None else 0,
                       seq_used_q=_ptr(seq_used_q) or 0, seq_used_k=_ptr(seq_used_k) or 0)
    nbytes = slikl_grad_recompute_p_workspace_size(pr, main, opt)
    if workspace is None or workspace.numel() < nbytes:
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device)
    p = torch.empty(sparse_indices.shape, dtype=torch.float32, device=q.device)
    out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dw=torch.empty_like(w),
               softmax_out=torch.empty(sparse_indices.shape, dtype=torch.float32, device=q.device))
    tn = slikl_tensors()
    tn.q, tn.k, tn.w = _ptr(q), _ptr(k), _ptr(w)
    tn.attn_softmax_l1norm = None
    tn.sparse_indices = _ptr(sparse_indices)
    tn.cu_seqlens_q = _ptr(cu_seqlens_q) if layout_q == "TND" else None
    tn.cu_seqlens_k = _ptr(cu_seqlens_k) if layout_k == "TND" else None
    tn.dq, tn.dk, tn.dw = _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dw"])
    tn.softmax_out = _ptr(out["softmax_out"])
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    slikl_grad_recompute_p(pr, main, tn, _ptr(q_main), _ptr(k_main), p.data_ptr(),
                           workspace.data_ptr(), workspace.numel(), s.cuda_stream, opt)
    res = dict(out)
    res["p"] = p
    res["workspace"] = workspace
    if loss_t is not None:
        res["loss"] = loss_t
    return res


def grad_recompute_p_workload(wl, main, device="cuda", deterministic=False, stream=None,
                              dk_path="auto", loss=False, seq_used_q=None, seq_used_k=None):
    """Move a slikl_inputs.Workload and its MainAttention to the device and run
    grad_recompute_p (seq_used_q / seq_used_k: host lists of B used lengths, or None)."""
    dev = torch.device(device)
    t = {n: getattr(wl, n).to(dev) for n in ("q", "k", "w", "idx")}
    cuq = wl.cu_seqlens_q.to(dev) if wl.cu_seqlens_q is not None else None
    cuk = wl.cu_seqlens_k.to(dev) if wl.cu_seqlens_k is not None else None
    uq = None if seq_used_q is None else torch.tensor(list(seq_used_q), dtype=torch.int32, device=dev)
    uk = None if seq_used_k is None else torch.tensor(list(seq_used_k), dtype=torch.int32, device=dev)
    return grad_recompute_p(t["q"], t["k"], t["w"], t["idx"], main.q.to(dev), main.k.to(dev),
                            main.scale, wl.layout, wl.layout, cuq, cuk, deterministic, stream,
                            dk_path=dk_path, key_range_bound=key_range_bound_of(wl), loss=loss,
                            seq_used_q=uq, seq_used_k=uk)


def key_range_bound_of(wl) -> int:
    """Longest key range of a workload's batches (host data), for TND problems."""
    if wl.cu_seqlens_k is None:
        return 0
    c = wl.cu_seqlens_k.tolist()
    return max((c[i + 1] - c[i] for i in range(len(c) - 1)), default=0)


def grad_workload(wl, device="cuda", deterministic=False, stream=None, dk_path="auto",
                  loss=False, seq_used_q=None, seq_used_k=None):
    """Move a slikl_inputs.Workload to the device and run grad() (seq_used_q / seq_used_k:
    optional host int sequences of B used lengths)."""
    dev = torch.device(device)
    t = {n: getattr(wl, n).to(dev) for n in ("q", "k", "w", "p", "idx")}
    cuq = wl.cu_seqlens_q.to(dev) if wl.cu_seqlens_q is not None else None
    cuk = wl.cu_seqlens_k.to(dev) if wl.cu_seqlens_k is not None else None
    uq = None if seq_used_q is None else torch.tensor(list(seq_used_q), dtype=torch.int32, device=dev)
    uk = None if seq_used_k is None else torch.tensor(list(seq_used_k), dtype=torch.int32, device=dev)
    return grad(t["q"], t["k"], t["w"], t["p"], t["idx"], wl.layout, wl.layout, cuq, cuk,
                deterministic=deterministic, stream=stream, dk_path=dk_path,
                key_range_bound=key_range_bound_of(wl), loss=loss, seq_used_q=uq,
                seq_used_k=uk)


def make_dense_problem(q: torch.Tensor, k: torch.Tensor, p: torch.Tensor, layout_q: str = "BSND",
                       layout_k: str = "BSND", mask_mode: int = 3, deterministic: bool = False,
                       B: Optional[int] = None, key_range_bound: int = 0) -> slikl_dense_problem:
    """Dense problem struct from tensor shapes; the row length is p's last dimension."""
    sp = make_problem(q, k, p, layout_q, layout_k, deterministic, B, key_range_bound)
    pr = slikl_dense_problem()
    for f in ("dtype", "layout_q", "layout_k", "deterministic", "B", "S1", "S2", "T1", "T2",
              "N1", "D"):
        setattr(pr, f, getattr(sp, f))
    pr.row_len = p.shape[-1]
    pr.mask_mode = mask_mode
    pr.reserved = 0
    return pr


def dense_grad(q, k, w, attn_softmax_l1norm, layout_q="BSND", layout_k="BSND", cu_seqlens_q=None,
               cu_seqlens_k=None, mask_mode=3, deterministic=False, stream=None, out=None,
               workspace=None, dk_path="auto", loss=False, seq_used_q=None, seq_used_k=None):
    """Run slikl_dense_grad on CUDA tensors (p and the returned softmax_out are [.., 1, Ld]).
    Returns dict(dq, dk, dw, softmax_out, workspace[, loss])."""
    B = None
    if layout_q == "TND":
        B = cu_seqlens_q.numel() - 1
    elif layout_k == "TND":
        B = cu_seqlens_k.numel() - 1
    pr = make_dense_problem(q, k, attn_softmax_l1norm, layout_q, layout_k, mask_mode,
                            deterministic, B)
    loss_t = torch.empty(pr.T1, dtype=torch.float32, device=q.device) if loss else None
    opt = make_options(dk_path, loss=loss_t.data_ptr() if loss_t is not None else 0,
                       seq_used_q=_ptr(seq_used_q) or 0, seq_used_k=_ptr(seq_used_k) or 0)
    nbytes = slikl_dense_grad_workspace_size(pr, opt)
    if workspace is None or workspace.numel() < nbytes:
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device)
    if out is None:
        out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dw=torch.empty_like(w),
                   softmax_out=torch.empty_like(attn_softmax_l1norm))
    tn = slikl_dense_tensors()
    tn.q, tn.k, tn.w = _ptr(q), _ptr(k), _ptr(w)
    tn.attn_softmax_l1norm = _ptr(attn_softmax_l1norm)
    tn.cu_seqlens_q = _ptr(cu_seqlens_q) if layout_q == "TND" else None
    tn.cu_seqlens_k = _ptr(cu_seqlens_k) if layout_k == "TND" else None
    tn.dq, tn.dk, tn.dw = _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dw"])
    tn.softmax_out = _ptr(out["softmax_out"])
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    slikl_dense_grad(pr, tn, workspace.data_ptr(), workspace.numel(), s.cuda_stream, opt)
    res = dict(out)
    res["workspace"] = workspace
    if loss_t is not None:
        res["loss"] = loss_t
    return res


def dense_grad_workload(wl, device="cuda", deterministic=False, stream=None, dk_path="auto",
                        loss=False, seq_used_q=None, seq_used_k=None):
    """Move a slikl_inputs.DenseWorkload to the device and run dense_grad()."""
    dev = torch.device(device)
    t = {n: getattr(wl, n).to(dev) for n in ("q", "k", "w", "p")}
    cuq = wl.cu_seqlens_q.to(dev) if wl.cu_seqlens_q is not None else None
    cuk = wl.cu_seqlens_k.to(dev) if wl.cu_seqlens_k is not None else None
    uq = None if seq_used_q is None else torch.tensor(list(seq_used_q), dtype=torch.int32, device=dev)
    uk = None if seq_used_k is None else torch.tensor(list(seq_used_k), dtype=torch.int32, device=dev)
    return dense_grad(t["q"], t["k"], t["w"], t["p"], wl.layout, wl.layout, cuq, cuk,
                      mask_mode=wl.mask_mode, deterministic=deterministic, stream=stream,
                      dk_path=dk_path, loss=loss, seq_used_q=uq, seq_used_k=uk)
