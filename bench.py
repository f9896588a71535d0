"""Benchmark of the sparse Lightning Indexer KL-loss backward on B200.

One step = one slikl_grad call (work split, fused per-token kernel, dK cast) on the
headline workload: causal BSND, B=1, S1=S2=4096, N1=64, D=128, topk=2048, bf16 q/k,
inputs already resident in HBM. L2 is flushed (256 MiB write) before every timed step,
outside the step's events.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--deterministic]
  python bench.py --impl reference ...    # the fp64 CPU oracle on the host cores

With N > 1 (torchrun, one process per GPU) every rank runs an independent replica of the
workload (the operator has no cross-GPU exchange): weak scaling, value = all ranks' tokens
divided by the slowest rank's device time.

Prints ONE JSON line on rank 0.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import slikl_inputs as si  # noqa: E402

METRIC = "query-tokens/s & TFLOP/s, % of B200 roofline (N1=64, D=128, topk=2048)"
UNIT = "query-tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def workload_stats(wl):
    """Nominal / valid FLOPs and compulsory bytes of one call (roofline definition:
    unique gathered key rows, q, w, p, indices, outputs and the fp32 dK workspace)."""
    T1, T2, N1, D, K = wl.T1, wl.T2, wl.N1, wl.D, wl.K
    idx = wl.idx.numpy().reshape(T1, K)
    valid = int((idx >= 0).sum())
    flop_nom = 6.0 * N1 * K * D * T1
    flop_valid = 6.0 * N1 * D * valid
    # unique key rows referenced
    if wl.layout == "BSND":
        batch = np.arange(T1) // wl.S1
        rows = idx + (batch * wl.S2)[:, None]
    else:
        cuq = wl.cu_seqlens_q.numpy()
        cuk = wl.cu_seqlens_k.numpy()
        batch = np.searchsorted(cuq, np.arange(T1), side="right") - 1
        rows = idx + cuk[batch][:, None]
    uniq = np.unique(rows[idx >= 0]).size
    el = 2  # bf16 / fp16
    bytes_comp = (uniq * D * el                        # gathered key rows
                  + T1 * N1 * D * el                   # q
                  + T1 * N1 * 4 + T1 * K * 4 + T1 * K * 4   # w, p, indices
                  + T1 * K * 4 + T1 * N1 * 4 + T1 * N1 * D * el  # softmax_out, dw, dq
                  + T2 * D * el                        # dk
                  + T2 * D * 4)                        # fp32 dK workspace
    return dict(valid=valid, flop_nom=flop_nom, flop_valid=flop_valid, bytes=bytes_comp,
                uniq_rows=int(uniq))


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            self.path = f"/tmp/slikl_clocks_{os.getpid()}.csv"
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = max(mx, float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def raw_event():
    """A timing cudaEvent_t created through the CUDA runtime (recorded by the C library)."""
    from cuda.bindings import runtime as cudart
    err, ev = cudart.cudaEventCreate()
    if err != cudart.cudaError_t.cudaSuccess:
        raise RuntimeError(f"cudaEventCreate: {err}")
    return ev


def raw_elapsed_ms(a, b):
    from cuda.bindings import runtime as cudart
    err, ms = cudart.cudaEventElapsedTime(a, b)
    if err != cudart.cudaError_t.cudaSuccess:
        raise RuntimeError(f"cudaEventElapsedTime: {err}")
    return ms


# DRAM bytes (read + write) of one fused-kernel launch on the headline workload, read from an
# ncu capture of that launch (dram__bytes_read.sum + dram__bytes_write.sum). The figure holds
# only while the kernel's sources are the ones captured (hash of the four files below);
# otherwise the traffic is reported as unknown (null).
FUSED_TRAFFIC = {"sources_sha256_16": "2e1620996d7e261b", "workload_config": 1,
                 "dk_path": "keymajor", "bytes": 121.880064e6 + 193.059072e6}


def fused_sources_hash():
    import hashlib
    h = hashlib.sha256()
    for f in ("slikl_fused_sm100.cu", "slikl_fused_pair_sm100.cu", "slikl_sm100.cuh",
              "slikl_common.cuh"):
        with open(os.path.join(ROOT, "sparse_lightning_indexer_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def combine_over_ranks(local, world, device):
    """Max over ranks of each per-rank time (seconds); local list of floats. With one rank the
    values are returned as they are. Every rank must call this (it is a collective)."""
    if world <= 1:
        return list(local)
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(local), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def fused_algorithmic_flop(wl, dk_path, valid_slots=None):
    """Algorithmic FLOPs of one fused-kernel launch: the S and dq products (2 N1 D each per
    slot), plus the dK product (2 N1 D) when the fused kernel forms dK itself (scatter path).
    With valid_slots the count is over the slots that hold an index (the work the kernel
    does: tiles without a valid slot are skipped); without it, over all T1 * topk slots
    (nominal). The second S product of the softmax's second pass is recomputation, not
    counted."""
    per_slot = 4.0 if dk_path == "keymajor" else 6.0
    slots = wl.K * wl.T1 if valid_slots is None else valid_slots
    return per_slot * wl.N1 * wl.D * slots


def oracle_rate(wl, ntok, seed=0, min_seconds=0.0):
    """fp64 oracle on seeded samples of ntok query tokens each (without replacement within a
    sample), repeated with new seeds until min_seconds of oracle time have passed; returns
    (tokens/s, cores, seconds, tokens)."""
    import oracle  # CPU baseline leg only
    oracle.build()
    done, secs, k = 0, 0.0, 0
    while True:
        rng = np.random.default_rng(seed + 7919 * k)
        toks = np.sort(rng.choice(wl.T1, size=min(ntok, wl.T1), replace=False))
        t0 = time.perf_counter()
        oracle.grad(wl, tokens=toks)
        secs += time.perf_counter() - t0
        done += len(toks)
        k += 1
        if secs >= min_seconds:
            break
    return done / secs, os.cpu_count(), secs, done


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = si.config(args.config)
    ntok = args.ref_tokens
    for _ in range(args.warmup):
        oracle_rate(wl, max(ntok // 4, 1), seed=1)
    total_tok, total_s = 0, 0.0
    for s in range(args.steps):
        _, cores, dt, n = oracle_rate(wl, ntok, seed=100 + s)
        total_tok += n
        total_s += dt
    value = total_tok / total_s
    sample = f"{ntok} seeded query tokens of the workload per step (full per-token outputs and their dk contributions)"
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_s / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": wl.name, "T1": wl.T1},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


NOMINAL_BF16_TFLOPS = 2250.0   # B200 dense bf16 at the boost clock (context beside the measured peak)


class Runner:
    """One workload resident on the device, called through slikl_grad_ex on `stream`."""

    def __init__(self, sli, wl, dev, stream, deterministic, dk_path):
        import torch
        self.sli, self.wl, self.dev, self.stream = sli, wl, dev, stream
        self.q, self.k, self.w, self.p, self.idx = (getattr(wl, n).to(dev)
                                                   for n in ("q", "k", "w", "p", "idx"))
        self.cuq = wl.cu_seqlens_q.to(dev) if wl.cu_seqlens_q is not None else None
        self.cuk = wl.cu_seqlens_k.to(dev) if wl.cu_seqlens_k is not None else None
        B = wl.B if wl.layout == "TND" else None
        self.pr = sli.make_problem(self.q, self.k, self.idx, wl.layout, wl.layout,
                                   deterministic, B, sli.key_range_bound_of(wl))
        self.dk_path_arg = dk_path
        self.opt = sli.make_options(dk_path)
        self.dk_path = ("keymajor" if sli.slikl_grad_dk_path(self.pr, self.opt)
                        == sli.SLIKL_DK_KEYMAJOR else "scatter")
        self.nbytes = sli.slikl_grad_workspace_size_ex(self.pr, self.opt)
        self.ws = torch.empty(self.nbytes, dtype=torch.uint8, device=dev)
        self.out = dict(dq=torch.empty_like(self.q), dk=torch.empty_like(self.k),
                        dw=torch.empty_like(self.w), softmax_out=torch.empty_like(self.p))
        self.tn = self.tensors(self.q, self.k, self.w, self.p, self.idx)

    def tensors(self, qq, kk, ww, pp, ii):
        tn = self.sli.slikl_tensors()
        tn.q, tn.k, tn.w, tn.attn_softmax_l1norm, tn.sparse_indices = (
            qq.data_ptr(), kk.data_ptr(), ww.data_ptr(), pp.data_ptr(), ii.data_ptr())
        tn.cu_seqlens_q = self.cuq.data_ptr() if self.cuq is not None else None
        tn.cu_seqlens_k = self.cuk.data_ptr() if self.cuk is not None else None
        o = self.out
        tn.dq, tn.dk, tn.dw, tn.softmax_out = (o["dq"].data_ptr(), o["dk"].data_ptr(),
                                               o["dw"].data_ptr(), o["softmax_out"].data_ptr())
        return tn

    def step(self, evs=None, tn=None):
        opt = self.opt if evs is None else self.sli.make_options(self.dk_path_arg,
                                                                 *(int(e) for e in evs))
        self.sli.slikl_grad_ex(self.pr, tn or self.tn, self.ws.data_ptr(), self.nbytes,
                               self.stream.cuda_stream, opt)

    def timed(self, steps, warmup, flush, barrier=None):
        """W untimed calls, then `steps` calls each after an L2 flush (outside the events);
        returns per-step lists (ms) of the whole call, the fused kernel and the dK stage."""
        import torch
        for _ in range(warmup):
            flush.fill_(1)
            self.step()
        torch.cuda.synchronize(self.dev)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        kev = [tuple(raw_event() for _ in range(4)) for _ in range(steps)]
        if barrier:
            barrier()
        for i in range(steps):
            flush.fill_(1)
            ev[i][0].record(self.stream)
            self.step(kev[i])
            ev[i][1].record(self.stream)
        torch.cuda.synchronize(self.dev)
        if barrier:
            barrier()
        return ([a.elapsed_time(b) for a, b in ev], [raw_elapsed_ms(e[0], e[1]) for e in kev],
                [raw_elapsed_ms(e[2], e[3]) for e in kev])

    def status(self):
        return self.sli.slikl_read_device_status(self.ws.data_ptr(), self.stream.cuda_stream)


class DenseRunner(Runner):
    """The dense variant's workload resident on the device, called through slikl_dense_grad
    on `stream` (timing, flush and status as Runner)."""

    def __init__(self, sli, wl, dev, stream, deterministic, dk_path):
        import torch
        self.sli, self.wl, self.dev, self.stream = sli, wl, dev, stream
        self.q, self.k, self.w, self.p = (getattr(wl, n).to(dev) for n in ("q", "k", "w", "p"))
        self.cuq = wl.cu_seqlens_q.to(dev) if wl.cu_seqlens_q is not None else None
        self.cuk = wl.cu_seqlens_k.to(dev) if wl.cu_seqlens_k is not None else None
        B = wl.B if wl.layout == "TND" else None
        self.pr = sli.make_dense_problem(self.q, self.k, self.p, wl.layout, wl.layout,
                                         wl.mask_mode, deterministic, B)
        self.dk_path_arg = dk_path
        self.opt = sli.make_options(dk_path)
        self.dk_path = ("keymajor" if sli.slikl_dense_grad_dk_path(self.pr, self.opt)
                        == sli.SLIKL_DK_KEYMAJOR else "scatter")
        self.nbytes = sli.slikl_dense_grad_workspace_size(self.pr, self.opt)
        self.ws = torch.empty(self.nbytes, dtype=torch.uint8, device=dev)
        self.out = dict(dq=torch.empty_like(self.q), dk=torch.empty_like(self.k),
                        dw=torch.empty_like(self.w), softmax_out=torch.empty_like(self.p))
        tn = sli.slikl_dense_tensors()
        tn.q, tn.k, tn.w, tn.attn_softmax_l1norm = (self.q.data_ptr(), self.k.data_ptr(),
                                                    self.w.data_ptr(), self.p.data_ptr())
        tn.cu_seqlens_q = self.cuq.data_ptr() if self.cuq is not None else None
        tn.cu_seqlens_k = self.cuk.data_ptr() if self.cuk is not None else None
        o = self.out
        tn.dq, tn.dk, tn.dw, tn.softmax_out = (o["dq"].data_ptr(), o["dk"].data_ptr(),
                                               o["dw"].data_ptr(), o["softmax_out"].data_ptr())
        self.tn = tn

    def step(self, evs=None, tn=None):
        opt = self.opt if evs is None else self.sli.make_options(self.dk_path_arg,
                                                                 *(int(e) for e in evs))
        self.sli.slikl_dense_grad(self.pr, tn or self.tn, self.ws.data_ptr(), self.nbytes,
                                  self.stream.cuda_stream, opt)


class RecomputePRunner(Runner):
    """A workload with main-attention inputs, called through slikl_grad_recompute_p (p formed
    from the main attention, then the backward); timing, flush and status as Runner."""

    def __init__(self, sli, wl, main, dev, stream, deterministic, dk_path):
        super().__init__(sli, wl, dev, stream, deterministic, dk_path)
        self.qm, self.km = main.q.to(dev), main.k.to(dev)
        self.main = sli.make_main_attention(self.qm, main.scale)
        self.p_out = torch_empty_like_f32(self.idx)
        self.nbytes = sli.slikl_grad_recompute_p_workspace_size(self.pr, self.main, self.opt)

    def step(self, evs=None, tn=None):
        opt = self.opt if evs is None else self.sli.make_options(self.dk_path_arg,
                                                                 *(int(e) for e in evs))
        self.sli.slikl_grad_recompute_p(self.pr, self.main, tn or self.tn, self.qm.data_ptr(),
                                        self.km.data_ptr(), self.p_out.data_ptr(),
                                        self.ws.data_ptr(), self.nbytes,
                                        self.stream.cuda_stream, opt)


def torch_empty_like_f32(t):
    import torch
    return torch.empty(t.shape, dtype=torch.float32, device=t.device)


def dense_stats(wl):
    """workload_stats for a dense problem: the slots are the Ld positions of every query row,
    the valid ones those the mask leaves visible; the compulsory bytes are every key row once,
    q, w, p, softmax_out, dw, dq, dk and the fp32 dK workspace (no index rows: a dense caller
    passes none)."""
    T1, T2, N1, D, Ld = wl.T1, wl.T2, wl.N1, wl.D, wl.Ld
    valid = si.dense_visible_slots(wl)
    el = 2
    bytes_comp = (T2 * D * el + T1 * N1 * D * el + T1 * N1 * 4 + T1 * Ld * 4
                  + T1 * Ld * 4 + T1 * N1 * 4 + T1 * N1 * D * el + T2 * D * el + T2 * D * 4)
    return dict(valid=valid, flop_nom=6.0 * N1 * Ld * D * T1, flop_valid=6.0 * N1 * D * valid,
                bytes=bytes_comp, uniq_rows=T2)


def step_roofline_ms(stats, peaks, peak_tf):
    return 1e3 * max(stats["flop_nom"] / (peak_tf * 1e12), stats["bytes"] / (peaks["hbm_gbs"] * 1e9))


def per_config_lines(sli, dev, stream, flush, peaks, steps, warmup):
    """The other full-size workloads, timed the same way as the headline (device time, L2
    flushed before every step): configs 2, 3 and 4 on the auto dK path, the deterministic
    reduction on configs 4 and 1, the 128-head causal workload, the dense variant's causal
    workload in both modes, and the causal workload with p formed from a 128-head main
    attention (the p kernel's time falls in the memset-and-split stage)."""
    import torch
    out = []
    for cid, det in ((2, False), (3, False), (4, False), (4, True), (1, True), ("n1_128", False),
                     ("dense", False), ("dense", True), ("recompute_p", False)):
        if cid == "recompute_p":
            wl = si.config(1)
            stats = workload_stats(wl)
            r = RecomputePRunner(sli, wl, si.main_attention(wl, 128, 128, seed=123, qk_scale=0.5),
                                 dev, stream, det, "auto")
        elif cid == "n1_128":
            wl = si.wide_heads()
            stats = workload_stats(wl)
            r = Runner(sli, wl, dev, stream, det, "auto")
        elif cid == "dense":
            wl = si.dense_full()
            stats = dense_stats(wl)
            r = DenseRunner(sli, wl, dev, stream, det, "auto")
        else:
            wl = si.config(cid)
            stats = workload_stats(wl)
            r = Runner(sli, wl, dev, stream, det, "auto")
        with torch.cuda.stream(stream):
            step_ms, kern_ms, dk_ms = r.timed(steps, warmup, flush)
        st = statistics.mean(step_ms)
        roof_meas = step_roofline_ms(stats, peaks, peaks["bf16_tflops"])
        roof_nom = step_roofline_ms(stats, peaks, NOMINAL_BF16_TFLOPS)
        kf = statistics.mean(kern_ms)
        kflop = fused_algorithmic_flop(wl, r.dk_path, stats["valid"])
        out.append({
            "config": cid, "workload": wl.name, "deterministic": det, "dk_path": r.dk_path,
            "T1": wl.T1, "steps": steps, "warmup": warmup,
            "ms_per_step": st, "query_tokens_per_s": wl.T1 / (st / 1e3),
            "tflops_nominal": stats["flop_nom"] / st / 1e9,
            "tflops_valid": stats["flop_valid"] / st / 1e9,
            "step_roofline_ms": roof_meas, "step_roofline_frac": roof_meas / st,
            "step_roofline_frac_nominal_peak": roof_nom / st,
            "stages_ms": {"fused": kf, "dk": statistics.mean(dk_ms),
                          "memset_and_work_split": st - kf - statistics.mean(dk_ms)},
            "fused_valid_slot_tflops": kflop / kf / 1e9,
            "fused_valid_slot_frac": kflop / kf / 1e9 / peaks["bf16_tflops"],
            "device_status": r.status(),
        })
        del r
        torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=1)
    ap.add_argument("--deterministic", action="store_true")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--ref-tokens", type=int, default=512)
    ap.add_argument("--cpu-baseline-tokens", type=int, default=12000)
    ap.add_argument("--dk-path", default="auto", choices=["auto", "scatter", "keymajor"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per-config block (the other workloads and deterministic mode)")
    ap.add_argument("--per-config-steps", type=int, default=10)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist
    import sparse_lightning_indexer_b200 as sli

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=__import__("datetime").timedelta(seconds=300))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    barrier = dist.barrier if world > 1 else None

    wl = si.config(args.config)
    stats = workload_stats(wl)
    stream = torch.cuda.Stream(device=dev)
    r = Runner(sli, wl, dev, stream, args.deterministic, args.dk_path)
    dk_path = r.dk_path
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    clocks = ClockSampler(vis.split(",")[local] if vis else str(local))
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush.fill_(1)
            r.step()
        torch.cuda.synchronize(dev)
        clocks.start()
        time.sleep(0.3)
        step_ms, kern_ms, dk_ms = r.timed(args.steps, 0, flush, barrier)
        flags = r.status()

        # end to end through the public API with pinned host buffers
        hq, hk, hw, hp, hi = (t.cpu().pin_memory() for t in (r.q, r.k, r.w, r.p, r.idx))
        hout = {n: torch.empty(t.shape, dtype=t.dtype).pin_memory() for n, t in r.out.items()}
        q2, k2, w2, p2, i2 = (torch.empty_like(t) for t in (r.q, r.k, r.w, r.p, r.idx))
        tn2 = r.tensors(q2, k2, w2, p2, i2)
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hw, hp, hi))
        d2h = sum(t.numel() * t.element_size() for t in hout.values())
        e2e_ms = []
        for i in range(args.warmup + args.steps):
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for dst, src in ((q2, hq), (k2, hk), (w2, hw), (p2, hp), (i2, hi)):
                dst.copy_(src, non_blocking=True)
            r.step(tn=tn2)
            for n, t in r.out.items():
                hout[n].copy_(t, non_blocking=True)
            b.record(stream)
            b.synchronize()
            if i >= args.warmup:
                e2e_ms.append(a.elapsed_time(b))
        del hq, hk, hw, hp, hi, hout, q2, k2, w2, p2, i2
    peaks, peak_src = load_peaks()
    per_config = None
    if world == 1 and not args.no_per_config and args.config == 1 and not args.deterministic:
        del r
        torch.cuda.empty_cache()
        per_config = per_config_lines(sli, dev, stream, flush, peaks, args.per_config_steps,
                                      args.warmup)
    clk = clocks.stop()

    t_total, t_e2e, t_kern, t_dk = combine_over_ranks(
        [sum(step_ms) / 1e3, sum(e2e_ms) / 1e3, sum(kern_ms) / 1e3, sum(dk_ms) / 1e3], world, dev)
    tokens = wl.T1 * args.steps * world
    value = tokens / t_total
    k_avg = t_kern / args.steps
    dk_avg = t_dk / args.steps
    flop = stats["flop_nom"]
    kflop = fused_algorithmic_flop(wl, dk_path, stats["valid"])
    kflop_nom = fused_algorithmic_flop(wl, dk_path)
    achieved_tf = kflop / k_avg / 1e12
    peak_tf = peaks["bf16_tflops"]
    traffic = None
    if (FUSED_TRAFFIC["workload_config"] == args.config and FUSED_TRAFFIC["dk_path"] == dk_path
            and not args.deterministic and fused_sources_hash() == FUSED_TRAFFIC["sources_sha256_16"]):
        traffic = FUSED_TRAFFIC["bytes"]
    step_avg = t_total / args.steps
    t_roof = step_roofline_ms(stats, peaks, peak_tf) / 1e3
    t_roof_nom = step_roofline_ms(stats, peaks, NOMINAL_BF16_TFLOPS) / 1e3
    # our kernels per call: 3 work-split + fused + cast; the key-major path adds 2 metadata
    # kernels, the w-scaled copy of q and its dK kernel (and in deterministic mode the combine
    # of cut runs); the sorted
    # reduction replaces the cast by sort init, 3 per radix pass, row pointers and the
    # segmented reduce
    launches_per_step = 5 + (4 if dk_path == "keymajor" else 0)
    if args.deterministic and dk_path == "keymajor":
        launches_per_step += 1
    elif args.deterministic:
        passes = (int(wl.T2).bit_length() + 7) // 8
        launches_per_step = 3 + 1 + 1 + 3 * passes + 2
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, cores, dt, ntok = oracle_rate(wl, args.cpu_baseline_tokens, min_seconds=12.0)
        cpu = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{ntok} seeded query tokens of the workload in samples of at most "
                         f"{min(args.cpu_baseline_tokens, wl.T1)} ({dt:.1f} s of fp64 oracle)"}
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * step_avg,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if wl.dtype.__repr__().endswith("bfloat16") else "fp16",
            "data": "synthetic (seeded, shaped like the operator's workloads)",
            "config": {"workload": wl.name, "T1": wl.T1, "T2": wl.T2, "N1": wl.N1, "D": wl.D,
                       "topk": wl.K, "deterministic": bool(args.deterministic),
                       "dk_path": dk_path,
                       "l2": "flushed before every timed step (256 MiB write, outside the events)",
                       "parallelism": f"replicas x{world}"},
            "tflops_nominal": flop / step_avg / 1e12,
            "tflops_valid": stats["flop_valid"] / step_avg / 1e12,
            "roofline_step": {"t_roof_ms": 1e3 * t_roof, "frac": t_roof / step_avg,
                              "t_roof_ms_nominal_peak": 1e3 * t_roof_nom,
                              "frac_nominal_peak": t_roof_nom / step_avg,
                              "flop_nominal": flop, "compulsory_bytes": stats["bytes"],
                              "peaks": f"bf16 {peak_tf} TFLOP/s ({peak_src}); "
                                       f"nominal {NOMINAL_BF16_TFLOPS} TFLOP/s; "
                                       f"hbm {peaks['hbm_gbs']} GB/s ({peak_src})"},
            "roofline": {"bound": "tensor", "achieved": achieved_tf, "peak": peak_tf,
                         "unit": "TFLOP/s", "frac": achieved_tf / peak_tf, "traffic": traffic,
                         "kernel": ("fused_pair_sm100 (fused per-token kernel, items of two slot "
                                    "tiles)" if dk_path == "keymajor" and wl.N1 <= 64 else
                                    "fused_sm100 (fused per-token kernel)"),
                         "algorithmic_flop_per_launch": kflop,
                         "flop_basis": "valid slots (tiles without a valid slot are skipped)",
                         "achieved_nominal_slots": kflop_nom / k_avg / 1e12,
                         "frac_nominal_slots": kflop_nom / k_avg / 1e12 / peak_tf,
                         "frac_of_nominal_peak": achieved_tf / NOMINAL_BF16_TFLOPS,
                         "peak_source": f"bf16_tflops, burst ({peak_src})"},
            "stages_ms": {"fused": 1e3 * k_avg, "dk": 1e3 * dk_avg,
                          "memset_and_work_split": 1e3 * (step_avg - k_avg - dk_avg)},
            "e2e": {"value": tokens / t_e2e, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * args.steps,
            "device_status": flags,
            "clocks": clk,
            "per_config": per_config,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
