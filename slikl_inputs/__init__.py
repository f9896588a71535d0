"""Seeded synthetic inputs for the sparse Lightning Indexer KL-loss backward.

This module only draws random numbers and rounds them to the input dtypes; it
holds none of the operator's arithmetic. Both the fp64 oracle (``oracle/``) and
the CUDA library (``sparse_lightning_indexer_b200``) consume the arrays it
returns, so the two sides always see bit-identical inputs.

Tensor shapes follow the operator's statement (aclnnSparseLightningIndexerKLLossGrad,
"公共约束" and "计算公式"), with the key head count fixed to one:

* BSND: q [B,S1,N1,D], k [B,S2,1,D], w [B,S1,N1], sparse_indices and
  attn_softmax_l1norm [B,S1,1,K].
* TND:  q [T1,N1,D],  k [T2,1,D],  w [T1,N1],  sparse_indices and
  attn_softmax_l1norm [T1,1,K], with cu_seqlens_q/k [B+1] (first entry 0).

Valid indices are local to their batch's key range; -1 marks an invalid slot.

Random generator: numpy ``default_rng`` (PCG64) seeded with 20261202 + config id.
Normal draws use numpy's standard normal; "N(0, v)" is read as variance v.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

SEED_BASE = 20261202


@dataclasses.dataclass
class Workload:
    """One synthetic problem. Every array is a CPU torch tensor."""

    name: str
    layout: str                 # "BSND" or "TND" (used for both q and k)
    dtype: torch.dtype          # torch.bfloat16 or torch.float16 for q, k
    B: int
    S1: int                     # BSND: query length; TND: max query length
    S2: int                     # BSND: key length; TND: max key length
    T1: int                     # total query rows
    T2: int                     # total key rows
    N1: int
    D: int
    K: int
    q: torch.Tensor
    k: torch.Tensor
    w: torch.Tensor
    p: torch.Tensor             # attn_softmax_l1norm
    idx: torch.Tensor           # sparse_indices, int32
    cu_seqlens_q: Optional[torch.Tensor] = None
    cu_seqlens_k: Optional[torch.Tensor] = None
    q_pos0: int = 0             # absolute position of the first query (long-context recipe)

    def valid_slots(self) -> int:
        return int((self.idx >= 0).sum())


# ----------------------------------------------------------------------------
# Index samplers (return int64 arrays of local key indices, length <= K)
# ----------------------------------------------------------------------------

def _distinct_uniform(rng: np.random.Generator, n: int, K: int) -> np.ndarray:
    """K distinct keys drawn uniformly from [0, n) (all n of them if n <= K), ascending."""
    if n <= K:
        return np.arange(n, dtype=np.int64)
    if n <= 4 * K:
        return np.sort(rng.permutation(n)[:K])
    # sequential rejection of repeats: keep the first K distinct draws
    draws = rng.integers(0, n, size=K + K // 4 + 16)
    while True:
        vals, first = np.unique(draws, return_index=True)
        if vals.size >= K:
            keep = np.sort(first)[:K]
            return np.sort(draws[keep])
        draws = np.concatenate([draws, rng.integers(0, n, size=K)])


def _zipf_cdf(alpha: float, nmax: int) -> np.ndarray:
    z = np.arange(1, nmax + 1, dtype=np.float64)
    return np.cumsum(z ** (-alpha))


def _zipf_recent_low(rng: np.random.Generator, t: int, K: int, cdf: np.ndarray) -> np.ndarray:
    """Keys in [0, t] with a Zipf preference for recent (t-(Z-1)) and low (Z-1) keys.

    Each draw takes Z ~ Zipf(alpha) truncated to [1, t+1] and, with probability
    1/2 each, key t-(Z-1) or Z-1; repeats are rejected (the first K distinct
    draws are kept, in draw order). If t+1 <= K all t+1 keys are taken in a
    random order.
    """
    n = t + 1
    if n <= K:
        return rng.permutation(n).astype(np.int64)
    top = cdf[n - 1]
    keys = np.empty(0, dtype=np.int64)
    batch = 4 * K
    while True:
        u = rng.random(batch) * top
        z = np.searchsorted(cdf, u, side="right") + 1          # in [1, n]
        z = np.minimum(z, n)
        recent = rng.random(batch) < 0.5
        draw = np.where(recent, t - (z - 1), z - 1).astype(np.int64)
        keys = np.concatenate([keys, draw])
        vals, first = np.unique(keys, return_index=True)
        if vals.size >= K:
            keep = np.sort(first)[:K]
            return keys[keep]
        batch *= 2


def _round(x: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    """Round fp64 draws to the input dtype (round-to-nearest-even)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(dtype)


def _target_distribution(rng: np.random.Generator, idx: np.ndarray) -> np.ndarray:
    """p = exp(N(0,1)) normalised to sum 1 over the valid slots of each row; 0 elsewhere."""
    e = np.exp(rng.standard_normal(idx.shape))
    e = np.where(idx >= 0, e, 0.0)
    s = e.sum(axis=-1, keepdims=True)
    s = np.where(s > 0, s, 1.0)
    return (e / s).astype(np.float32)


# ----------------------------------------------------------------------------
# The five workload recipes
# ----------------------------------------------------------------------------

def _finish(name, layout, dtype, B, S1, S2, q_lens, k_lens, N1, D, K, qk_scale, w_var,
            idx_rows, rng, q_pos0=0) -> Workload:
    T1 = int(sum(q_lens))
    T2 = int(sum(k_lens))
    idx = np.full((T1, K), -1, dtype=np.int32)
    for t, row in enumerate(idx_rows):
        idx[t, : row.size] = row
    q = rng.standard_normal((T1, N1, D)) * qk_scale
    k = rng.standard_normal((T2, D)) * qk_scale
    w = rng.standard_normal((T1, N1)) * np.sqrt(w_var)
    p = _target_distribution(rng, idx)
    qt = _round(q, dtype)
    kt = _round(k, dtype)
    wt = torch.from_numpy(w.astype(np.float32))
    pt = torch.from_numpy(p)
    it = torch.from_numpy(idx)
    if layout == "BSND":
        qt = qt.reshape(B, S1, N1, D)
        kt = kt.reshape(B, S2, 1, D)
        wt = wt.reshape(B, S1, N1)
        pt = pt.reshape(B, S1, 1, K)
        it = it.reshape(B, S1, 1, K)
        cuq = cuk = None
    else:
        qt = qt.reshape(T1, N1, D)
        kt = kt.reshape(T2, 1, D)
        pt = pt.reshape(T1, 1, K)
        it = it.reshape(T1, 1, K)
        cuq = torch.tensor(np.concatenate([[0], np.cumsum(q_lens)]), dtype=torch.int32)
        cuk = torch.tensor(np.concatenate([[0], np.cumsum(k_lens)]), dtype=torch.int32)
    return Workload(name=name, layout=layout, dtype=dtype, B=B, S1=S1, S2=S2, T1=T1, T2=T2,
                    N1=N1, D=D, K=K, q=qt.contiguous(), k=kt.contiguous(), w=wt.contiguous(),
                    p=pt.contiguous(), idx=it.contiguous(), cu_seqlens_q=cuq,
                    cu_seqlens_k=cuk, q_pos0=q_pos0)


def causal_bsnd(name, B, S, N1, D, K, dtype, qk_scale, w_var, seed) -> Workload:
    """Query t of each batch takes min(K, t+1) distinct uniform keys from [0, t]."""
    rng = np.random.default_rng(seed)
    rows = []
    for _b in range(B):
        for t in range(S):
            rows.append(_distinct_uniform(rng, t + 1, K))
    return _finish(name, "BSND", dtype, B, S, S, [S] * B, [S] * B, N1, D, K, qk_scale,
                   w_var, rows, rng)


def varlen_tnd(name, B, len_lo, len_hi, N1, D, K, dtype, qk_scale, w_var, seed) -> Workload:
    """B sequences with lengths uniform in [len_lo, len_hi]; per-sequence causal indices."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(len_lo, len_hi + 1, size=B).astype(np.int64)
    rows = []
    for b in range(B):
        for t in range(int(lens[b])):
            rows.append(_distinct_uniform(rng, t + 1, K))
    return _finish(name, "TND", dtype, B, int(lens.max()), int(lens.max()), list(lens),
                   list(lens), N1, D, K, qk_scale, w_var, rows, rng)


def long_context_bsnd(name, S1, S2, pos0, N1, D, K, dtype, qk_scale, w_var, seed) -> Workload:
    """S1 queries at absolute positions pos0..pos0+S1-1 over S2 keys; K distinct uniform keys
    from [0, pos_t] per query."""
    rng = np.random.default_rng(seed)
    rows = [_distinct_uniform(rng, pos0 + s + 1, K) for s in range(S1)]
    return _finish(name, "BSND", dtype, 1, S1, S2, [S1], [S2], N1, D, K, qk_scale, w_var,
                   rows, rng, q_pos0=pos0)


def zipf_bsnd(name, B, S, N1, D, K, dtype, qk_scale, w_var, alpha, invalid_frac, seed) -> Workload:
    """Causal Zipf(alpha) preference for recent and low-index keys; each slot is then set
    to -1 independently with probability invalid_frac (interspersed, not sorted)."""
    rng = np.random.default_rng(seed)
    cdf = _zipf_cdf(alpha, S)
    rows = []
    for _b in range(B):
        for t in range(S):
            keys = _zipf_recent_low(rng, t, K, cdf)
            row = np.full(K, -1, dtype=np.int64)
            row[: keys.size] = keys
            drop = rng.random(K) < invalid_frac
            row[drop] = -1
            rows.append(row)
    return _finish(name, "BSND", dtype, B, S, S, [S] * B, [S] * B, N1, D, K, qk_scale,
                   w_var, rows, rng)


CONFIG_NAMES = {
    0: "tiny-causal-bsnd B1 S256 N1=8 D64 K64 bf16",
    1: "causal-bsnd B1 S4096 N1=64 D128 K2048 bf16",
    2: "varlen-tnd B8 len[512,8192] N1=32 D128 K2048 fp16",
    3: "long-context-bsnd S1=8192@122880 S2=131072 N1=64 D128 K2048 bf16",
    4: "zipf-skew-bsnd B4 S8192 N1=16 D128 K512 bf16 (30% invalid)",
}


def config(cid: int) -> Workload:
    """The five workload recipes (sizes, dtypes and index structure per config)."""
    seed = SEED_BASE + cid
    name = CONFIG_NAMES[cid]
    if cid == 0:
        return causal_bsnd(name, 1, 256, 8, 64, 64, torch.bfloat16, 1.0, 1.0 / 8, seed)
    if cid == 1:
        return causal_bsnd(name, 1, 4096, 64, 128, 2048, torch.bfloat16, 0.1, 1.0 / 64, seed)
    if cid == 2:
        return varlen_tnd(name, 8, 512, 8192, 32, 128, 2048, torch.float16, 0.1, 1.0 / 64, seed)
    if cid == 3:
        return long_context_bsnd(name, 8192, 131072, 122880, 64, 128, 2048, torch.bfloat16,
                                 0.1, 1.0 / 64, seed)
    if cid == 4:
        return zipf_bsnd(name, 4, 8192, 16, 128, 512, torch.bfloat16, 0.1, 1.0 / 64, 1.1, 0.3,
                         seed)
    raise ValueError(f"unknown config {cid}")


def small(seed: int, layout: str = "BSND", B: int = 2, S1: int = 40, S2: int = 300,
          N1: int = 16, D: int = 128, K: int = 200, dtype: torch.dtype = torch.bfloat16,
          qk_scale: float = 0.3, w_var: float = 1.0 / 16, pattern: str = "uniform",
          invalid_frac: float = 0.0, lens_q=None, lens_k=None) -> Workload:
    """A small problem for parity tests that spans several 128-slot tiles with a ragged tail.

    pattern: "uniform" (K distinct keys uniform over the batch's whole key range),
    "causal" (key range [0, s] for query s), "dup" (keys drawn with repeats allowed),
    or "none" (every slot -1).
    """
    rng = np.random.default_rng(seed)
    if layout == "TND":
        if lens_q is None:
            lens_q = list(rng.integers(1, S1 + 1, size=B))
        if lens_k is None:
            lens_k = list(rng.integers(1, S2 + 1, size=B))
    else:
        lens_q = [S1] * B
        lens_k = [S2] * B
    rows = []
    for b in range(B):
        nk = int(lens_k[b])
        for s in range(int(lens_q[b])):
            if pattern == "uniform":
                r = rng.permutation(nk)[: min(K, nk)]
            elif pattern == "causal":
                r = _distinct_uniform(rng, min(s + 1, nk), K)
            elif pattern == "dup":
                r = rng.integers(0, nk, size=K)
            elif pattern == "none":
                r = np.empty(0, dtype=np.int64)
            else:
                raise ValueError(pattern)
            r = np.asarray(r, dtype=np.int64)
            if invalid_frac > 0 and r.size:
                row = np.full(K, -1, dtype=np.int64)
                row[: r.size] = r
                row[rng.random(K) < invalid_frac] = -1
                r = row
            rows.append(r)
    return _finish(f"small-{layout}-{pattern}", layout, dtype, B, max(lens_q), max(lens_k),
                   [int(x) for x in lens_q], [int(x) for x in lens_k], N1, D, K, qk_scale,
                   w_var, rows, rng)


# ----------------------------------------------------------------------------
# Dense variant inputs (every visible key of the batch is a slot)
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class DenseWorkload:
    """One synthetic dense problem. attn_softmax_l1norm p is [.., 1, Ld]: slot j of a row is
    key j of its batch; Ld >= the longest key range."""

    name: str
    layout: str
    dtype: torch.dtype
    mask_mode: int              # 0 = no mask, 3 = right-down causal
    B: int
    S1: int
    S2: int
    T1: int
    T2: int
    N1: int
    D: int
    Ld: int
    q: torch.Tensor
    k: torch.Tensor
    w: torch.Tensor
    p: torch.Tensor
    cu_seqlens_q: Optional[torch.Tensor] = None
    cu_seqlens_k: Optional[torch.Tensor] = None


def _visible_count(mask_mode: int, s: int, qlen: int, klen: int) -> int:
    # the input's structure (which slots carry target mass): every key with no mask; with the
    # right-down causal mask the keys up to the diagonal through the last query and key
    if mask_mode == 0:
        return klen
    return min(klen, max(0, s + klen - qlen + 1))


def dense_small(seed: int, layout: str = "BSND", B: int = 2, S1: int = 40, S2: int = 300,
                N1: int = 16, D: int = 128, mask_mode: int = 3,
                dtype: torch.dtype = torch.bfloat16, qk_scale: float = 0.3,
                w_var: float = 1.0 / 16, lens_q=None, lens_k=None, Ld: Optional[int] = None,
                used_q=None, used_k=None, name: Optional[str] = None) -> DenseWorkload:
    """A dense problem; p = exp(N(0,1)) normalised over each row's visible keys (the used
    lengths, when given, decide the visible set), 0 elsewhere."""
    rng = np.random.default_rng(seed)
    if layout == "TND":
        if lens_q is None:
            lens_q = list(rng.integers(1, S1 + 1, size=B))
        if lens_k is None:
            lens_k = list(rng.integers(1, S2 + 1, size=B))
    else:
        lens_q = [S1] * B
        lens_k = [S2] * B
    lens_q = [int(x) for x in lens_q]
    lens_k = [int(x) for x in lens_k]
    T1, T2 = sum(lens_q), sum(lens_k)
    if Ld is None:
        Ld = max(lens_k) if lens_k else 1
    q = rng.standard_normal((T1, N1, D)) * qk_scale
    k = rng.standard_normal((T2, D)) * qk_scale
    w = rng.standard_normal((T1, N1)) * np.sqrt(w_var)
    e = np.exp(rng.standard_normal((T1, Ld)))
    mask = np.zeros((T1, Ld), dtype=bool)
    t = 0
    for b in range(B):
        qlen = lens_q[b] if used_q is None else int(used_q[b])
        klen = lens_k[b] if used_k is None else int(used_k[b])
        for s in range(lens_q[b]):
            if s < qlen:
                mask[t, : _visible_count(mask_mode, s, qlen, klen)] = True
            t += 1
    e = np.where(mask, e, 0.0)
    tot = e.sum(axis=-1, keepdims=True)
    p = (e / np.where(tot > 0, tot, 1.0)).astype(np.float32)
    qt, kt = _round(q, dtype), _round(k, dtype)
    wt, pt = torch.from_numpy(w.astype(np.float32)), torch.from_numpy(p)
    if layout == "BSND":
        qt = qt.reshape(B, S1, N1, D)
        kt = kt.reshape(B, S2, 1, D)
        wt = wt.reshape(B, S1, N1)
        pt = pt.reshape(B, S1, 1, Ld)
        cuq = cuk = None
    else:
        qt = qt.reshape(T1, N1, D)
        kt = kt.reshape(T2, 1, D)
        pt = pt.reshape(T1, 1, Ld)
        cuq = torch.tensor(np.concatenate([[0], np.cumsum(lens_q)]), dtype=torch.int32)
        cuk = torch.tensor(np.concatenate([[0], np.cumsum(lens_k)]), dtype=torch.int32)
    return DenseWorkload(name=name or f"dense-{layout}-mask{mask_mode}", layout=layout, dtype=dtype,
                         mask_mode=mask_mode, B=B, S1=max(lens_q) if lens_q else 0,
                         S2=max(lens_k) if lens_k else 0, T1=T1, T2=T2, N1=N1, D=D, Ld=Ld,
                         q=qt.contiguous(), k=kt.contiguous(), w=wt.contiguous(),
                         p=pt.contiguous(), cu_seqlens_q=cuq, cu_seqlens_k=cuk)


WIDE_HEADS_NAME = "causal-bsnd B1 S4096 N1=128 D128 K2048 bf16"


def wide_heads(seed: int = SEED_BASE + 110) -> Workload:
    """The 128-head workload: the causal S=4096, topk=2048 recipe with N1 = 128 query heads
    (w of variance 1/128)."""
    return causal_bsnd(WIDE_HEADS_NAME, 1, 4096, 128, 128, 2048, torch.bfloat16, 0.1,
                       1.0 / 128, seed)


DENSE_FULL_NAME = "dense-causal-bsnd B1 S4096 N1=64 D128 mask3 bf16"


def dense_full(seed: int = SEED_BASE + 100) -> DenseWorkload:
    """The full-size dense problem: one batch of 4096 queries over 4096 keys under the
    right-down causal mask (query s sees keys 0..s), N1 = 64, D = 128, bf16, row length 4096;
    values drawn like the causal sparse workload's (q, k scaled by 0.1, w of variance 1/64)."""
    return dense_small(seed, "BSND", 1, 4096, 4096, 64, 128, 3, torch.bfloat16, 0.1, 1.0 / 64,
                       name=DENSE_FULL_NAME)


def dense_visible_slots(wl: DenseWorkload) -> int:
    """Number of (query row, key) pairs that the mask leaves visible (the slots in use)."""
    if wl.layout == "TND":
        lq = np.diff(wl.cu_seqlens_q.numpy())
        lk = np.diff(wl.cu_seqlens_k.numpy())
    else:
        lq, lk = [wl.S1] * wl.B, [wl.S2] * wl.B
    return int(sum(min(_visible_count(wl.mask_mode, s, int(a), int(b)), wl.Ld)
                   for a, b in zip(lq, lk) for s in range(int(a))))


# ----------------------------------------------------------------------------
# main-attention inputs of the variant that forms p itself
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class MainAttention:
    """Main-attention query q [.., Nm, Dm] (same rows as the indexer's q) and one key head
    k [.., 1, Dm] (same rows as the indexer's k), with the softmax scale."""

    q: torch.Tensor
    k: torch.Tensor
    Nm: int
    Dm: int
    scale: float


def main_attention(wl: Workload, Nm: int, Dm: int = 128, seed: int = 7,
                   dtype: Optional[torch.dtype] = None, qk_scale: float = 1.0,
                   scale: Optional[float] = None) -> MainAttention:
    """Seeded N(0,1) * qk_scale draws in the workload's layout and dtype; softmax scale
    1/sqrt(Dm) unless given."""
    rng = np.random.default_rng(seed)
    dt = wl.dtype if dtype is None else dtype
    q = _round(rng.standard_normal((wl.T1, Nm, Dm)) * qk_scale, dt)
    k = _round(rng.standard_normal((wl.T2, Dm)) * qk_scale, dt)
    if wl.layout == "BSND":
        q = q.reshape(wl.B, wl.S1, Nm, Dm)
        k = k.reshape(wl.B, wl.S2, 1, Dm)
    else:
        q = q.reshape(wl.T1, Nm, Dm)
        k = k.reshape(wl.T2, 1, Dm)
    return MainAttention(q=q.contiguous(), k=k.contiguous(), Nm=Nm, Dm=Dm,
                         scale=float(1.0 / np.sqrt(Dm)) if scale is None else float(scale))
