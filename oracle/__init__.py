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

Every function here is pinned: the sparse operator by tests/test_oracle_pins.py (finite
differences of the KL loss, a dense one-hot brute force, torch fp64 autograd, closed forms
and invariants), the dense variant by tests/test_dense_oracle_pins.py, and the target
distribution formed from the main attention by tests/test_main_p_oracle_pins.py (a library
softmax, hand-worked cases, invariances, planted mistakes).
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


# ---------------------------------------------------------------------------------------------
# Dense variant (DenseLightningIndexerKLLossGrad)
#
# The article on DenseLightningIndexerKLLossGradMetadata (lmnt.cn) names the dense operator and
# its interface (sections 功能定位, 第一段接口参数说明, 特殊约束): one key head, headDim 128, layouts
# BSND / TND, maskMode 0 (no mask) or 3 (rightDownCausal: the lower triangle aligned to the
# bottom-right corner), cmpRatio 1 for uncompressed keys. It prints no formula of its own. The
# reading taken here: the formulas of aclnnSparseLightningIndexerKLLossGrad (计算公式) with the
# top-k slots of a query replaced by every key of its batch that the mask leaves visible, slot j
# being key j of the batch; attn_softmax_l1norm and softmax_out are [T1, Ld] rows with Ld at
# least the longest key range.
# ---------------------------------------------------------------------------------------------

def dense_visible(mask_mode: int, s: int, qlen: int, klen: int) -> int:
    """Keys of a batch visible to its query at local position s: all klen of them with no
    mask; with the right-down causal mask, keys 0 .. s + (klen - qlen), i.e. the diagonal runs
    through the last query and the last key (none when that bound is negative)."""
    if mask_mode == 0:
        return klen
    if mask_mode == 3:
        return min(klen, max(0, s + klen - qlen + 1))
    raise ValueError("mask_mode must be 0 or 3")


def dense_grad_arrays(q: np.ndarray, k: np.ndarray, w: np.ndarray, p: np.ndarray,
                      q_start: np.ndarray, k_start: np.ndarray, mask_mode: int,
                      q_used: Optional[Sequence[int]] = None,
                      k_used: Optional[Sequence[int]] = None) -> dict:
    """Dense oracle on flat fp64 arrays: q [T1,N1,D], k [T2,D], w [T1,N1], p [T1,Ld];
    q_start / k_start [B+1]; optional used lengths [B] (rows past them are padding, keys past
    them are not visible). Plain fp64 per query row: S = q_t K^T over the visible keys, then the
    sparse operator's formulas. Returns y [T1,Ld], dw, dq, dk [T2,D], loss [T1]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    p = np.asarray(p, dtype=np.float64)
    T1, N1, D = q.shape
    T2 = k.shape[0]
    Ld = p.shape[1]
    B = len(q_start) - 1
    y = np.zeros((T1, Ld))
    dw = np.zeros((T1, N1))
    dq = np.zeros((T1, N1, D))
    dk = np.zeros((T2, D))
    loss = np.zeros(T1)
    for b in range(B):
        q0, q1 = int(q_start[b]), int(q_start[b + 1])
        k0, k1 = int(k_start[b]), int(k_start[b + 1])
        qlen = q1 - q0 if q_used is None else int(q_used[b])
        klen = k1 - k0 if k_used is None else int(k_used[b])
        for s in range(qlen):
            t = q0 + s
            L = dense_visible(mask_mode, s, qlen, klen)
            if L == 0:
                continue
            if L > Ld:
                raise ValueError("row length below the visible key count")
            Kv = k[k0:k0 + L]                               # [L, D]
            S = q[t] @ Kv.T                                 # [N1, L]
            R = np.maximum(S, 0.0)
            I = w[t] @ R                                    # [L]
            e = np.exp(I - I.max())
            yv = e / e.sum()
            pv = p[t, :L]
            dI = yv - pv                                    # dI = Softmax(I) - p
            y[t, :L] = yv
            dw[t] = R @ dI                                  # dW = dI . ReLU(S)^T
            dS = dI[None, :] * w[t][:, None] * (S > 0.0)    # chain rule on I = W . ReLU(S)
            dq[t] = dS @ Kv                                 # dq = dS . K
            dk[k0:k0 + L] += dS.T @ q[t]                    # dK = dS^T . q
            pos = pv > 0.0
            loss[t] = float(np.sum(pv[pos] * np.log(pv[pos] / yv[pos])))
    return {"y": y, "dw": dw, "dq": dq, "dk": dk, "loss": loss}


def dense_grad(wl, seq_used_q: Optional[Sequence[int]] = None,
               seq_used_k: Optional[Sequence[int]] = None) -> dict:
    """Dense oracle on a slikl_inputs.DenseWorkload."""
    T1, T2, N1, D = wl.T1, wl.T2, wl.N1, wl.D
    q = wl.q.double().numpy().reshape(T1, N1, D)
    k = wl.k.double().numpy().reshape(T2, D)
    w = wl.w.double().numpy().reshape(T1, N1)
    p = wl.p.double().numpy().reshape(T1, wl.Ld)
    cuq = None if wl.cu_seqlens_q is None else wl.cu_seqlens_q.numpy()
    cuk = None if wl.cu_seqlens_k is None else wl.cu_seqlens_k.numpy()
    qs, ks = row_starts(wl.layout, wl.layout, wl.B, wl.S1, wl.S2, cuq, cuk)
    return dense_grad_arrays(q, k, w, p, qs, ks, wl.mask_mode, seq_used_q, seq_used_k)


# ---------------------------------------------------------------------------------------------
# The old fused variant's target distribution (SparseLightningIndexerGradKLLoss)
#
# aclnnSparseLightningIndexerKLLossGrad (功能说明 and 计算公式) says that the older operator
# computed p inside its kernel from the main attention's scores, summed over the heads and
# L1-normalised, and that attn_softmax_l1norm now carries that result. The pages give none of
# that operator's inputs. The reading taken here: a main-attention query q_m [T1, Nm, Dm], one
# main-attention key head k_m [T2, Dm] on the same key rows as k, and a softmax scale; each
# head's attention is the softmax of scale * q_m[t, h] . k_m[j] over the row's valid top-k
# slots (the keys a sparse main attention attends to); p is the sum over heads, divided by its
# sum over the slots (the L1 norm). Invalid slots and rows without a valid slot get 0.
# ---------------------------------------------------------------------------------------------

def main_softmax_l1norm_arrays(q_m: np.ndarray, k_m: np.ndarray, idx: np.ndarray,
                               q_start: np.ndarray, k_start: np.ndarray, scale: float,
                               q_used: Optional[Sequence[int]] = None,
                               k_used: Optional[Sequence[int]] = None) -> np.ndarray:
    """p [T1, K] (fp64) from q_m [T1, Nm, Dm], k_m [T2, Dm], idx [T1, K]; valid slots and
    padding rows as in grad_arrays (q_used / k_used the optional used lengths)."""
    q_m = np.asarray(q_m, dtype=np.float64)
    k_m = np.asarray(k_m, dtype=np.float64)
    idx = np.asarray(idx)
    T1, K = idx.shape
    p = np.zeros((T1, K))
    B = len(q_start) - 1
    for b in range(B):
        q0, q1 = int(q_start[b]), int(q_start[b + 1])
        k0, k1 = int(k_start[b]), int(k_start[b + 1])
        qlen = q1 - q0 if q_used is None else int(q_used[b])
        klen = k1 - k0 if k_used is None else int(k_used[b])
        for t in range(q0, q0 + qlen):
            v = idx[t].astype(np.int64)
            slots = np.nonzero((v >= 0) & (v < klen))[0]
            if slots.size == 0:
                continue
            S = scale * (q_m[t] @ k_m[k0 + v[slots]].T)          # [Nm, valid slots]
            A = np.exp(S - S.max(axis=1, keepdims=True))
            A /= A.sum(axis=1, keepdims=True)                   # softmax over the slots, per head
            hsum = A.sum(axis=0)                                # sum over the heads
            p[t, slots] = hsum / np.abs(hsum).sum()             # L1 normalisation
    return p


def main_softmax_l1norm(wl, main, seq_used_q: Optional[Sequence[int]] = None,
                        seq_used_k: Optional[Sequence[int]] = None) -> np.ndarray:
    """main_softmax_l1norm_arrays on a slikl_inputs.Workload and its MainAttention inputs."""
    T1, T2, K = wl.T1, wl.T2, wl.K
    q_m = main.q.double().numpy().reshape(T1, main.Nm, main.Dm)
    k_m = main.k.double().numpy().reshape(T2, main.Dm)
    idx = wl.idx.numpy().reshape(T1, K)
    cuq = None if wl.cu_seqlens_q is None else wl.cu_seqlens_q.numpy()
    cuk = None if wl.cu_seqlens_k is None else wl.cu_seqlens_k.numpy()
    qs, ks = row_starts(wl.layout, wl.layout, wl.B, wl.S1, wl.S2, cuq, cuk)
    return main_softmax_l1norm_arrays(q_m, k_m, idx, qs, ks, main.scale, seq_used_q, seq_used_k)


def grad_recompute_p(wl, main, seq_used_q: Optional[Sequence[int]] = None,
                     seq_used_k: Optional[Sequence[int]] = None) -> dict:
    """The old variant end to end: p from the main attention, then the backward of the KL loss
    with that p (grad's outputs, loss included, plus p itself)."""
    p = main_softmax_l1norm(wl, main, seq_used_q, seq_used_k)
    T1, T2, N1, D, K = wl.T1, wl.T2, wl.N1, wl.D, wl.K
    cuq = None if wl.cu_seqlens_q is None else wl.cu_seqlens_q.numpy()
    cuk = None if wl.cu_seqlens_k is None else wl.cu_seqlens_k.numpy()
    qs, ks = row_starts(wl.layout, wl.layout, wl.B, wl.S1, wl.S2, cuq, cuk)
    out = grad_arrays(wl.q.double().numpy().reshape(T1, N1, D),
                      wl.k.double().numpy().reshape(T2, D),
                      wl.w.double().numpy().reshape(T1, N1), p,
                      wl.idx.numpy().reshape(T1, K), qs, ks, q_used=seq_used_q, k_used=seq_used_k)
    out["p"] = p
    return out
