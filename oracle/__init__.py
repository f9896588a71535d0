"""fp64 CPU oracle for the sparse Lightning Indexer KL-loss backward.

TEST INFRASTRUCTURE ONLY: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The CUDA product path
(``sparse_lightning_indexer_b200``) never imports it, and this package never
imports the product.

The arithmetic lives in ``slikl_oracle.c`` (plain fp64 loops, OpenMP over query
tokens). This module only builds that library, maps the BSND/TND layouts of
aclnnSparseLightningIndexerKLLossGrad ("公共约束": layoutQ/layoutK are BSND or TND,
TND needs cuSeqLens) onto flat query/key rows, and converts arrays.

Layout reading (the parameter tables of the page did not survive extraction):
the key tensor has a single head, so

* BSND: query row of (b, s) = b*S1 + s; key rows of batch b start at b*S2.
* TND:  query rows of batch b start at cu_seqlens_q[b]; key rows at cu_seqlens_k[b].

Every function here is pinned by tests/test_oracle_pins.py (finite differences of
the KL loss, a dense one-hot brute force, torch fp64 autograd, closed forms and
invariants).
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "slikl_oracle.c")
_LIB = os.path.join(_HERE, "_liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into oracle/_liboracle.so (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", "-o", tmp,
                               _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Problem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("T1", ctypes.c_int64), ("T2", ctypes.c_int64),
                ("N1", ctypes.c_int64), ("D", ctypes.c_int64), ("K", ctypes.c_int64),
                ("q_start", ctypes.POINTER(ctypes.c_int64)),
                ("k_start", ctypes.POINTER(ctypes.c_int64)),
                ("q_used", ctypes.POINTER(ctypes.c_int64)),
                ("k_used", ctypes.POINTER(ctypes.c_int64))]


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.POINTER
        lib.oracle_grad.restype = ctypes.c_int
        lib.oracle_grad.argtypes = [P(_Problem), P(ctypes.c_double), P(ctypes.c_double),
                                    P(ctypes.c_double), P(ctypes.c_double), P(ctypes.c_int32),
                                    P(ctypes.c_int64), ctypes.c_int64, ctypes.c_int,
                                    P(ctypes.c_double), P(ctypes.c_double), P(ctypes.c_double),
                                    P(ctypes.c_double), P(ctypes.c_double)]
        lib.oracle_split_equal.restype = None
        lib.oracle_split_equal.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                           P(ctypes.c_int64), P(ctypes.c_int64)]
        lib.oracle_split_weighted.restype = None
        lib.oracle_split_weighted.argtypes = [P(ctypes.c_int32), ctypes.c_int64, ctypes.c_int64,
                                              ctypes.c_int64, P(ctypes.c_int64)]
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray], ctype):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def row_starts(layout_q: str, layout_k: str, B: int, S1: int, S2: int,
               cu_seqlens_q: Optional[Sequence[int]], cu_seqlens_k: Optional[Sequence[int]]):
    """First query row and first key row of each batch ([B+1] each, int64)."""
    if layout_q == "BSND":
        qs = np.arange(B + 1, dtype=np.int64) * S1
    else:
        qs = np.asarray(cu_seqlens_q, dtype=np.int64)
    if layout_k == "BSND":
        ks = np.arange(B + 1, dtype=np.int64) * S2
    else:
        ks = np.asarray(cu_seqlens_k, dtype=np.int64)
    if qs.shape != (B + 1,) or ks.shape != (B + 1,):
        raise ValueError("cu_seqlens must have B+1 entries")
    return qs, ks


def grad_arrays(q: np.ndarray, k: np.ndarray, w: np.ndarray, p: np.ndarray, idx: np.ndarray,
                q_start: np.ndarray, k_start: np.ndarray, tokens: Optional[np.ndarray] = None,
                nthreads: int = 0, q_used: Optional[Sequence[int]] = None,
                k_used: Optional[Sequence[int]] = None) -> dict:
    """Oracle on flat fp64 arrays.

    q [T1,N1,D], k [T2,D], w [T1,N1], p [T1,K], idx [T1,K] int32, q_start/k_start [B+1];
    q_used / k_used: optional [B] rows of each batch in use (seqUsedQ / seqUsedK reading:
    query rows past q_used[b] are padding, keys past k_used[b] are invalid slots).
    Returns fp64 y [T1,K], dw [T1,N1], dq [T1,N1,D], dk [T2,D], loss [T1].
    """
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    w = np.ascontiguousarray(w, dtype=np.float64)
    p = np.ascontiguousarray(p, dtype=np.float64)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T1, N1, D = q.shape
    T2 = k.shape[0]
    K = idx.shape[1]
    assert k.shape == (T2, D) and w.shape == (T1, N1) and p.shape == (T1, K)
    assert idx.shape == (T1, K)
    qs = np.ascontiguousarray(q_start, dtype=np.int64)
    ks = np.ascontiguousarray(k_start, dtype=np.int64)
    B = qs.size - 1
    qu = None if q_used is None else np.ascontiguousarray(q_used, dtype=np.int64)
    ku = None if k_used is None else np.ascontiguousarray(k_used, dtype=np.int64)
    if (qu is not None and qu.shape != (B,)) or (ku is not None and ku.shape != (B,)):
        raise ValueError("q_used / k_used must have B entries")
    prob = _Problem(B, T1, T2, N1, D, K, _ptr(qs, ctypes.c_int64), _ptr(ks, ctypes.c_int64),
                    _ptr(qu, ctypes.c_int64), _ptr(ku, ctypes.c_int64))
    y = np.zeros((T1, K))
    dw = np.zeros((T1, N1))
    dq = np.zeros((T1, N1, D))
    dk = np.zeros((T2, D))
    loss = np.zeros(T1)
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    rc = _load().oracle_grad(ctypes.byref(prob), _ptr(q, ctypes.c_double),
                             _ptr(k, ctypes.c_double), _ptr(w, ctypes.c_double),
                             _ptr(p, ctypes.c_double), _ptr(idx, ctypes.c_int32),
                             _ptr(tok, ctypes.c_int64), 0 if tok is None else tok.size,
                             int(nthreads), _ptr(y, ctypes.c_double), _ptr(dw, ctypes.c_double),
                             _ptr(dq, ctypes.c_double), _ptr(dk, ctypes.c_double),
                             _ptr(loss, ctypes.c_double))
    if rc != 0:
        raise ValueError({1: "bad shape or used length", 2: "index outside its batch's key range",
                          3: "out of memory"}.get(rc, f"oracle error {rc}"))
    return {"y": y, "dw": dw, "dq": dq, "dk": dk, "loss": loss}


def grad(wl, tokens: Optional[np.ndarray] = None, nthreads: int = 0,
         seq_used_q: Optional[Sequence[int]] = None,
         seq_used_k: Optional[Sequence[int]] = None) -> dict:
    """Oracle on a slikl_inputs.Workload (inputs converted exactly from their dtypes);
    seq_used_q / seq_used_k as q_used / k_used of grad_arrays."""
    T1, T2, N1, D, K = wl.T1, wl.T2, wl.N1, wl.D, wl.K
    q = wl.q.double().numpy().reshape(T1, N1, D)
    k = wl.k.double().numpy().reshape(T2, D)
    w = wl.w.double().numpy().reshape(T1, N1)
    p = wl.p.double().numpy().reshape(T1, K)
    idx = wl.idx.numpy().reshape(T1, K)
    cuq = None if wl.cu_seqlens_q is None else wl.cu_seqlens_q.numpy()
    cuk = None if wl.cu_seqlens_k is None else wl.cu_seqlens_k.numpy()
    qs, ks = row_starts(wl.layout, wl.layout, wl.B, wl.S1, wl.S2, cuq, cuk)
    return grad_arrays(q, k, w, p, idx, qs, ks, tokens=tokens, nthreads=nthreads,
                       q_used=seq_used_q, k_used=seq_used_k)


def split_equal(total: int, cores: int, max_seq_k: int):
    """Row split of the pages' metadata generator. Returns (header[6], ranges[cores,2])."""
    out = np.zeros(6, dtype=np.int64)
    ranges = np.zeros(2 * cores, dtype=np.int64)
    _load().oracle_split_equal(total, cores, max_seq_k, _ptr(out, ctypes.c_int64),
                               _ptr(ranges, ctypes.c_int64))
    return out, ranges.reshape(cores, 2)


def split_weighted(idx: np.ndarray, cores: int) -> np.ndarray:
    """Cost-weighted contiguous split of query rows. Returns ranges[cores,2]."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T1, K = idx.shape
    ranges = np.zeros(2 * cores, dtype=np.int64)
    _load().oracle_split_weighted(_ptr(idx, ctypes.c_int32), T1, K, cores,
                                  _ptr(ranges, ctypes.c_int64))
    return ranges.reshape(cores, 2)
