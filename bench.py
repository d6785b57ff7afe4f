"""Throughput of the MSA forward hot path on B200: 128K prefill query-tokens/s
(plus 128K decode tokens/s), with the roofline fraction of the dominant kernel
and of the whole path, an end-to-end number through the public API with host
buffers, and the fp64 CPU oracle timed on the host cores as a baseline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl msa|reference]

Under torchrun each rank runs its own independent problem (weak scaling, no
collective on the data path); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import multiprocessing as mp
import os
import shutil
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_gqa_04_b200.workload import (VARLEN_MIX, WORKLOADS, Workload,  # noqa: E402
                                                make_inputs, make_varlen_inputs, sample_rows)

METRIC = "128K prefill query-tokens/s & decode tok/s on 1 B200; % tensor/HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
SMS = 148
FP32_LANES_PER_SM = 128


# ---------------------------------------------------------------------------
# algorithmic counts
# ---------------------------------------------------------------------------

def positions(w: Workload) -> np.ndarray:
    return (w.q_pos0 + np.arange(w.q_len, dtype=np.int64))


def counts(w: Workload) -> dict:
    """Algorithmic work of one forward, from the definitions of the method."""
    t = positions(w)
    c_t = t // w.block_size
    ksel = np.minimum(w.top_k, c_t + 1)
    B = w.batch
    vis_keys = float(B * np.sum(t + 1))
    sel_blocks = float(B * np.sum(ksel))           # per group
    index_flops = 2.0 * w.index_dim * w.num_kv_heads * vis_keys
    main_flops = 4.0 * w.head_dim * w.num_q_heads * w.block_size * sel_blocks  # S and P V
    esz = 4 if w.dtype == "f32" else 2
    # NVFP4: half a byte per element plus one scale byte per 16 elements
    kidx_row = {"fp8": w.index_dim, "nvfp4": w.index_dim // 2 + w.index_dim // 16}.get(
        w.index_dtype, w.index_dim * esz)
    kidx_bytes = float(B * w.kv_len * kidx_row)
    bmax_read = float(B * w.num_kv_heads * np.sum(c_t) * 4)
    partial_bytes = float(w.num_q_heads * sel_blocks * (w.head_dim * esz + 4))
    out_bytes = float(w.rows * w.num_q_heads * w.head_dim * esz)
    return {"index_flops": index_flops, "main_flops": main_flops, "kidx_bytes": kidx_bytes,
            "index_fp8": w.index_dtype == "fp8", "qk_fp8": w.qk_dtype == "fp8",
            "bmax_read_bytes": bmax_read, "partial_bytes": partial_bytes,
            "out_bytes": out_bytes, "sel_blocks_per_group": sel_blocks,
            "q2k_bytes": float(w.num_kv_heads * w.rows * w.top_k * 4)}


def selected_kv_bytes(w: Workload, q2k: torch.Tensor) -> float:
    """K and V bytes of the distinct (sequence, group, block) triples selected."""
    Hkv, T, k = q2k.shape
    b = (torch.arange(T, device=q2k.device) // w.q_len).view(1, T, 1)
    g = torch.arange(Hkv, device=q2k.device).view(Hkv, 1, 1)
    key = (b.to(torch.int64) * Hkv + g) * w.nblk + q2k.to(torch.int64)
    key = key[q2k >= 0]
    n = int(torch.unique(key).numel())
    esz = 4 if w.dtype == "f32" else 2
    return float(n) * w.block_size * w.head_dim * ((1 if w.qk_dtype == "fp8" else esz) + esz)


def load_peaks() -> tuple:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        if shutil.which("nvidia-smi"):
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self) -> dict:
        if not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) >= 9 and p[1].isdigit():
                    rows.append(p)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [int(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": int(rows[0][2]),
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())
                if any(r[3].replace(".", "").isdigit() for r in rows) else None}


# ---------------------------------------------------------------------------
# oracle on the host cores (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------

class RowStore:
    """Query-side tensors of a few rows behind the [B, Sq, ...] indexing the
    oracle uses (only the sampled rows are ever read)."""

    def __init__(self, full_shape, rows_np: dict):
        self.shape = full_shape
        self._rows = rows_np

    def __getitem__(self, idx):
        b, i = idx[0], idx[1]
        x = self._rows[(int(b), int(i))]
        return x[idx[2:]] if len(idx) > 2 else x


_W = {}
_THREAD_VARS = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")


def _oracle_worker_init(files: dict, meta: dict):
    _W["k"] = np.load(files["k"], mmap_mode="r")
    _W["v"] = np.load(files["v"], mmap_mode="r")
    _W["k_idx"] = np.load(files["k_idx"], mmap_mode="r")
    _W["meta"] = meta


def _oracle_rows(task):
    from oracle import msa_oracle as O
    rows, qrows, qirows = task
    m = _W["meta"]
    q = RowStore(tuple(m["q_shape"]), qrows)
    qi = RowStore(tuple(m["qi_shape"]), qirows)
    O.forward(q, _W["k"], _W["v"], qi, _W["k_idx"], m["q_pos0"], m["block_size"], m["top_k"],
              rows=rows)
    return len(rows)


def oracle_rows(w: Workload) -> int:
    """Rows of the oracle sample: 4096 for the prefill workloads (a few seconds
    of wall time on 16 host cores at 128K), every row when there are fewer."""
    return min(w.rows, 4096)


def time_oracle(w: Workload, x: dict, n_rows: int, seed: int = 0) -> dict:
    """Times the oracle forward on ``n_rows`` evenly spread rows with a spawn
    pool over all host cores and extrapolates to the whole workload."""
    cores = len(os.sched_getaffinity(0))
    rows = sample_rows(w, n_rows, seed)
    tmp = tempfile.mkdtemp(prefix="msa_oracle_")
    files = {}
    try:
        for name in ("k", "v", "k_idx"):
            files[name] = os.path.join(tmp, name + ".npy")
            np.save(files[name], x[name].float().cpu().numpy())
        qrows, qirows = {}, {}
        qc, qic = x["q"], x["q_idx"]
        for r in rows:
            b, i = divmod(r, w.q_len)
            qrows[(b, i)] = qc[b, i].float().cpu().numpy()
            qirows[(b, i)] = qic[b, i].float().cpu().numpy()
        meta = {"q_shape": list(x["q"].shape), "qi_shape": list(x["q_idx"].shape),
                "q_pos0": w.q_pos0, "block_size": w.block_size, "top_k": w.top_k}
        nproc = max(1, min(cores, len(rows)))
        chunks = [rows[i::nproc] for i in range(nproc)]
        tasks = [(c, {(divmod(r, w.q_len)): qrows[divmod(r, w.q_len)] for r in c},
                  {(divmod(r, w.q_len)): qirows[divmod(r, w.q_len)] for r in c}) for c in chunks]
        ctx = mp.get_context("spawn")
        # one BLAS thread per worker process: the pool already uses every core
        saved = {k: os.environ.get(k) for k in _THREAD_VARS}
        os.environ.update({k: "1" for k in _THREAD_VARS})
        try:
            pool = ctx.Pool(nproc, initializer=_oracle_worker_init, initargs=(files, meta))
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
        with pool:
            pool.map(_oracle_rows, [(c[:1], t1, t2) for c, t1, t2 in tasks])  # warm imports
            t0 = time.perf_counter()
            done = sum(pool.map(_oracle_rows, tasks))
            wall = time.perf_counter() - t0
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
    # rows are spread evenly over positions, so their mean cost is the workload's
    full = wall * w.rows / done
    return {"value": w.rows / full, "unit": "query-tokens/s", "cores": nproc,
            "kind": "oracle", "sample_wall_s": wall,
            "sample": f"{done} of {w.rows} query rows of {w.name} spread evenly over positions "
                      f"(fp64 NumPy oracle, spawn pool of {nproc} processes); whole-workload "
                      f"time extrapolated as wall * rows / sampled rows"}


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------

def _events(n):
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for e in ev:
        e.record()  # materialise the underlying CUDA event
    return ev


def run_steps(msa, w, x, ws, out, steps, warmup, stage_timing=True, extra=None):
    """Warm-up, then exactly ``steps`` timed forwards.  Returns (ms/step, stage ms)."""
    kw = dict(q_pos0=w.q_pos0, block_size=w.block_size, top_k=w.top_k, workspace=ws, out=out)
    kw.update(extra or {})
    for _ in range(warmup):
        msa.forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], **kw)
    per = [(_events(1)[0], _events(5)) for _ in range(steps)] if stage_timing else []
    start, end = _events(2)
    torch.cuda.synchronize()
    start.record()
    for s in range(steps):
        if stage_timing:
            per[s][0].record()
            msa.set_stage_events(per[s][1])
        msa.forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], **kw)
    end.record()
    msa.set_stage_events(None)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / steps
    stage = {}
    if stage_timing:
        for i, name in enumerate(msa.STAGES):
            tot = 0.0
            for s0, evs in per:
                prev = s0 if i == 0 else evs[i - 1]
                tot += prev.elapsed_time(evs[i])
            stage[name] = tot / steps
    return ms, stage


def run_e2e(msa, w, xh, out_h, steps, warmup):
    """Same metric through the public API with pinned host buffers: every step
    copies its inputs host->device and its output device->host (the library
    overlaps a step's output copy with the next step's input copy and kernels;
    the timed region ends when the last output copy has landed)."""
    kw = dict(q_pos0=w.q_pos0, block_size=w.block_size, top_k=w.top_k, out=out_h)
    for _ in range(warmup):
        msa.forward(xh["q"], xh["k"], xh["v"], xh["q_idx"], xh["k_idx"], **kw)
    torch.cuda.synchronize()
    start, end = _events(2)
    start.record()
    for _ in range(steps):
        msa.forward(xh["q"], xh["k"], xh["v"], xh["q_idx"], xh["k_idx"], **kw)
    # the last output copy runs on the library's copy stream: include it
    torch.cuda.current_stream().wait_stream(msa.host_output_stream())
    end.record()
    torch.cuda.synchronize()
    h2d = sum(xh[n].numel() * xh[n].element_size() for n in ("q", "k", "v", "q_idx", "k_idx"))
    d2h = out_h.numel() * out_h.element_size()
    return start.elapsed_time(end) / steps, h2d, d2h


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of a
# kernel, with the git blob id of the kernel source the capture ran: once that
# source changes the entry no longer applies and the bench reports traffic as
# null.  The counters come from a capture of one launch on the 12288-row prefill
# (724,992 selected entries) scaled to the 128K prefill's 8,327,168 entries:
# the partial-state writes grow exactly with the entries, the Q-gather reads
# grow faster (fewer L2 hits at full size), so the scaled figure is a lower
# bound on the reads.
NCU_TRAFFIC = {
    # stage: (workload, source file, git blob id, bytes per launch)
    "attn": ("prefill_128k", "block_sparse_gqa_04_b200/csrc/attn_tc.cu",
             "14b66a335fad31600ee1ed6bbb190907efbfc464",
             round((415465472 + 2956862976) * 8327168 / 724992)),
}


def _blob_id(path: str) -> str:
    import hashlib
    data = open(path, "rb").read()
    return hashlib.sha1(b"blob %d\0" % len(data) + data).hexdigest()


def measured_traffic(stage: str, workload: str):
    ent = NCU_TRAFFIC.get(stage)
    if not ent or ent[0] != workload:
        return None
    src = os.path.join(ROOT, ent[1])
    if not os.path.exists(src) or _blob_id(src) != ent[2]:
        return None
    return ent[3]


FP8_RATIO = 2.0  # nominal dense fp8 : bf16 tensor throughput (4.5 : 2.25 PFLOP/s)


def tensor_seconds(cnt, bf16_tflops):
    """Time of the step's contractions at the tensor peak of each one's dtype:
    the index GEMM, S = Q K^T (half of the main FLOPs) and P V (bf16)."""
    r_idx = FP8_RATIO if cnt["index_fp8"] else 1.0
    r_qk = FP8_RATIO if cnt["qk_fp8"] else 1.0
    half = cnt["main_flops"] / 2
    return {"index": cnt["index_flops"] / (bf16_tflops * r_idx * 1e12),
            "attn": half / (bf16_tflops * r_qk * 1e12) + half / (bf16_tflops * 1e12)}


def kernel_roofline(w, cnt, stage_ms, path, peaks, kv_sel_bytes):
    """Roofline entry of the slowest stage of the step.  A contraction's peak is
    its dtype's: the measured bf16 peak, times the nominal fp8 ratio for fp8
    operands (the attention mixes an fp8 S with a bf16 P V when q/k are fp8).
    The step lasts well under a second, so `frac` divides by the burst peak;
    `frac_sustained` gives the same against the seconds-long sustained peak."""
    name = max(stage_ms, key=stage_ms.get)
    ms = stage_ms[name]
    t_peak = tensor_seconds(cnt, peaks["bf16_tflops"])
    t_sus = tensor_seconds(cnt, peaks.get("bf16_tflops_sustained") or peaks["bf16_tflops"])
    alu_peak = SMS * FP32_LANES_PER_SM * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
    peak_sus = None
    if name == "index":
        tc = "index:tc" in path
        bound, unit, work = ("tensor" if tc else "alu"), "TFLOP/s", cnt["index_flops"]
        peak = work / t_peak["index"] / 1e12 if tc else alu_peak
        peak_sus = work / t_sus["index"] / 1e12 if tc else None
        achieved = work / (ms * 1e-3) / 1e12
    elif name == "attn":
        tc = "attn:tc" in path
        bound, unit, work = ("tensor" if tc else "alu"), "TFLOP/s", cnt["main_flops"]
        peak = work / t_peak["attn"] / 1e12 if tc else alu_peak
        peak_sus = work / t_sus["attn"] / 1e12 if tc else None
        achieved = work / (ms * 1e-3) / 1e12
    else:
        bound, unit = "hbm", "GB/s"
        work = {"topk": cnt["bmax_read_bytes"] + cnt["q2k_bytes"],
                "lists": 3 * cnt["q2k_bytes"],
                "combine": cnt["partial_bytes"] + cnt["out_bytes"] + cnt["q2k_bytes"]}[name]
        peak = peaks["hbm_gbs"]
        achieved = work / (ms * 1e-3) / 1e9
    res = {"kernel": name, "bound": bound, "achieved": round(achieved, 2), "peak": round(peak, 2),
           "unit": unit, "frac": round(achieved / peak, 4),
           "traffic": measured_traffic(name, w.name),
           "ms": round(ms, 4), "algorithmic_per_launch": work,
           "peak_kind": ("measured burst bf16" + (" (x 2 for fp8 operands)" if
                                                   (cnt["index_fp8"] or cnt["qk_fp8"]) else ""))
                        if bound == "tensor" else
                        ("derived: 148 SMs x 128 FP32 lanes x 2 x max SM clock" if bound == "alu"
                         else "measured copy bandwidth")}
    if peak_sus:
        res["frac_sustained"] = round(achieved / peak_sus, 4)
        res["peak_sustained"] = round(peak_sus, 2)
    return res


def path_roofline(cnt, kv_sel_bytes, ms, peaks):
    F = cnt["index_flops"] + cnt["main_flops"]
    Bytes = cnt["kidx_bytes"] + kv_sel_bytes
    t_tensor = sum(tensor_seconds(cnt, peaks["bf16_tflops"]).values())
    t_hbm = Bytes / (peaks["hbm_gbs"] * 1e9)
    t_roof = max(t_tensor, t_hbm)
    return {"flops": F, "bytes": Bytes, "bound": "tensor" if t_tensor >= t_hbm else "hbm",
            "t_roofline_ms": round(t_roof * 1e3, 4), "t_measured_ms": round(ms, 4),
            "frac": round(t_roof * 1e3 / ms, 4),
            "note": "roofline = max(index+main FLOPs at the burst tensor peak of their "
                    "dtype (bf16 measured, fp8 = 2 x bf16), (k_idx + distinct selected K/V "
                    "bytes) / HBM peak)"}


def measure_varlen(msa, dev, steps, warmup, peaks, lens=VARLEN_MIX):
    """The packed variable-length batch ``lens`` (msa_forward_varlen) on inputs
    resident in HBM: ``steps`` timed calls after ``warmup``, CUDA events on the
    launching stream.  Algorithmic work and the path roofline are the sums over
    the sequences, each counted as its own one-sequence workload."""
    lens_q, lens_k = lens
    Hq, Hkv, D, di, k = 64, 4, 128, 128, 16
    x = make_varlen_inputs(lens_q, lens_k, Hq, Hkv, D, di, "bf16", seed=0, device=dev)
    p, cq, ck = msa.varlen_problem(x["cu_q"], x["cu_k"], Hq, Hkv, D, di, top_k=k)
    ws = torch.empty(msa.varlen_workspace_size(p, cq, ck) + 256, dtype=torch.uint8, device=dev)
    out = torch.empty(x["q"].shape, dtype=x["v"].dtype, device=dev)
    args = (x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], x["cu_q"], x["cu_k"])
    _, q2k = msa.forward_varlen(*args, top_k=k, workspace=ws, out=out, return_q2k=True)
    cnt = None
    kv_sel = 0.0
    for b, (nq, nk) in enumerate(zip(lens_q, lens_k)):
        if nq == 0:
            continue
        wb = Workload(f"varlen_seq{b}", 1, nq, nk, nk - nq, Hq, Hkv, D, di, 128, k, "bf16", 0)
        c = counts(wb)
        cnt = c if cnt is None else {n: (cnt[n] + c[n] if isinstance(c[n], float) else c[n])
                                     for n in c}
        q0 = x["cu_q"][b]
        kv_sel += selected_kv_bytes(wb, q2k[:, q0:q0 + nq])
    del q2k
    for _ in range(warmup):
        msa.forward_varlen(*args, top_k=k, workspace=ws, out=out)
    start, end = _events(2)
    idx = dev.index if dev.index is not None else 0
    with ClockSampler(idx) as clk:
        torch.cuda.synchronize()
        start.record()
        for _ in range(steps):
            msa.forward_varlen(*args, top_k=k, workspace=ws, out=out)
        end.record()
        torch.cuda.synchronize()
    ms = start.elapsed_time(end) / steps
    return {"rows": sum(lens_q), "ms": ms, "cnt": cnt, "kv_sel": kv_sel,
            "launches": msa.varlen_launch_count(p, cq, ck) * steps, "clocks": clk.summary(),
            "sequences": len(lens_q)}


def page_inputs(x, w, dev, seed=0):
    """Moves k, v and k_idx into a shuffled pool of 128-token pages (64 spare
    pages, zero tails) and returns the forward's paging kwargs.  Untimed."""
    B, nblk = w.batch, w.nblk
    npages = B * nblk + 64
    g = torch.Generator(device=dev).manual_seed(seed + 1)
    perm = torch.randperm(npages, generator=g, device=dev)[: B * nblk]
    for name in ("k", "v", "k_idx"):
        t = x[name].view(torch.uint8)  # bytes: index_copy_ takes every dtype that way
        tail = tuple(t.shape[2:])
        pad = nblk * 128 - w.kv_len
        if pad:
            t = torch.cat([t, torch.zeros((B, pad) + tail, dtype=t.dtype, device=dev)], dim=1)
        pool = torch.zeros((npages, 128) + tail, dtype=torch.uint8, device=dev)
        pool.index_copy_(0, perm, t.reshape((B * nblk, 128) + tail))
        x[name] = pool.view(x[name].dtype)
        del t
    table = perm.view(B, nblk).to(torch.int32).contiguous()
    return {"block_table": table, "kv_len": w.kv_len}, npages


def measure_workload(msa, w, dev, steps, warmup, peaks, with_e2e, paged=False):
    x = make_inputs(w, seed=0, device=dev)
    x.pop("needles")
    extra = {}
    if "q_idx_scale" in x:  # NVFP4 index tensors: codes + scales
        extra["index_scales"] = (x["q_idx_scale"], x["k_idx_scale"])
    p = msa.problem_of(w, index_scales=extra.get("index_scales"))
    if paged:
        pextra, npages = page_inputs(x, w, dev)
        extra.update(pextra)
        p = msa.make_problem(w.batch, w.q_len, w.kv_len, w.num_q_heads, w.num_kv_heads,
                             w.head_dim, w.index_dim, w.block_size, w.top_k, w.torch_dtype,
                             w.q_pos0, index_dtype=w.torch_index_dtype,
                             qk_dtype=w.torch_qk_dtype, num_pages=npages,
                             block_table=extra["block_table"])
        torch.cuda.empty_cache()
    path = msa.kernel_path(p)
    ws = msa.new_workspace(p, msa.OP_FORWARD, dev)
    out = torch.empty(x["q"].shape, dtype=x["v"].dtype, device=dev)  # out has v's dtype
    _, q2k = msa.forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], q_pos0=w.q_pos0,
                         block_size=w.block_size, top_k=w.top_k, workspace=ws, return_q2k=True,
                         **extra)
    kv_sel = selected_kv_bytes(w, q2k)
    del q2k
    cnt = counts(w)
    idx = dev.index if dev.index is not None else 0
    with ClockSampler(idx) as clk:
        ms, stage = run_steps(msa, w, x, ws, out, steps, warmup, extra=extra)
    res = {"w": w, "ms": ms, "stage": stage, "path": path, "cnt": cnt, "kv_sel": kv_sel,
           "clocks": clk.summary(), "launches": msa.launch_count(p) * steps, "x": x}
    if with_e2e and not paged and w.index_dtype != "nvfp4":
        xh = {n: x[n].cpu().pin_memory() for n in ("q", "k", "v", "q_idx", "k_idx")}
        del ws
        torch.cuda.empty_cache()
        out_h = torch.empty(x["q"].shape, dtype=x["v"].dtype).pin_memory()
        e_ms, h2d, d2h = run_e2e(msa, w, xh, out_h, max(1, steps // 2), 1)
        res["e2e"] = (e_ms, h2d, d2h)
    return res


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(v: float, world: int) -> float:
    """Largest per-rank value (step time) over all ranks; the same on every rank."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_value(rows_per_rank: int, ms_local: float, world: int) -> tuple:
    """Whole-job throughput of independent per-rank problems: every rank's rows
    divided by the slowest rank's step time.  Returns (value, max ms)."""
    ms = max_over_ranks(ms_local, world)
    return world * rows_per_rank / (ms * 1e-3), ms


def workload_config(w: Workload, world: int) -> dict:
    return {"workload": w.name, "index_dtype": w.index_dtype or w.dtype,
            "qk_dtype": w.qk_dtype or w.dtype,
            "batch": w.batch, "q_len": w.q_len, "kv_len": w.kv_len,
            "q_pos0": w.q_pos0, "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads,
            "head_dim": w.head_dim, "index_dim": w.index_dim, "block_size": w.block_size,
            "top_k": w.top_k, "parallelism": f"replicas x{world} (independent problems)"}


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def index_kl_flops(w: Workload, q2k: torch.Tensor) -> float:
    """Algorithmic FLOPs of one msa_index_kl: per (row, group) and selected
    visible token, the teacher's logits (G heads x D MACs), the index score and
    its dq_idx term (2 x di MACs), and its dk_idx term (di MACs)."""
    Hkv, T, K = q2k.shape
    pos = (w.q_pos0 + torch.arange(T, device=q2k.device) % w.q_len).view(1, T, 1)
    c = q2k.to(torch.int64)
    vis = torch.clamp(pos - c * w.block_size + 1, 0, w.block_size) * (c >= 0)
    tokens = float(vis.sum().item())
    G = w.num_q_heads // w.num_kv_heads
    return 2.0 * tokens * (G * w.head_dim + 3 * w.index_dim)


def bench_index_kl(a, w, world, rank, local, peaks):
    """Times msa_index_kl on the workload's inputs and its own selection (made
    once, untimed): exactly a.steps calls after a.warmup, CUDA events on the
    launching stream, max over ranks."""
    from block_sparse_gqa_04_b200 import msa
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    x = make_inputs(w, seed=rank, device=dev)
    x.pop("needles")
    q2k = msa.select(x["q_idx"], x["k_idx"], q_pos0=w.q_pos0, block_size=w.block_size,
                     top_k=w.top_k)
    p = msa.problem_of(w)
    ws = msa.new_workspace(p, msa.OP_INDEX_KL, dev)
    kw = dict(q_pos0=w.q_pos0, block_size=w.block_size, workspace=ws)
    for _ in range(a.warmup):
        msa.index_kl(x["q"], x["k"], x["q_idx"], x["k_idx"], q2k, **kw)
    start, end = _events(2)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        start.record()
        for _ in range(a.steps):
            msa.index_kl(x["q"], x["k"], x["q_idx"], x["k_idx"], q2k, **kw)
        end.record()
        torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(start.elapsed_time(end) / a.steps, world)
    flops = index_kl_flops(w, q2k)
    alu_peak = SMS * FP32_LANES_PER_SM * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
    achieved = flops / (ms * 1e-3) / 1e12
    if rank == 0:
        line = {"metric": "index KL-alignment loss + q_idx/k_idx gradients (training side), "
                          "query-tokens/s", "value": world * w.rows / (ms * 1e-3),
                "unit": "query-tokens/s", "n_gpus": world, "steps": a.steps,
                "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None,
                "dtype": "f32" if w.dtype == "f32" else "f32 (bf16/e4m3 inputs)",
                "data": "synthetic (seeded N(0,1/d) inputs with planted needle blocks)",
                "config": dict(workload_config(w, world),
                               kernel_path=msa.kernel_path(p, msa.OP_INDEX_KL)),
                "clocks": clk.summary(),
                "gpu_launches": a.steps * msa.launch_count(p, msa.OP_INDEX_KL),
                "roofline": {"kernel": "index_kl", "bound": "alu", "achieved": round(achieved, 2),
                             "peak": round(alu_peak, 2), "unit": "TFLOP/s",
                             "frac": round(achieved / alu_peak, 4), "traffic": None,
                             "algorithmic_per_launch": flops,
                             "peak_kind": "derived: 148 SMs x 128 FP32 lanes x 2 x max SM clock"}}
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="msa", choices=["msa", "reference"])
    ap.add_argument("--workload", default="prefill_128k", choices=list(WORKLOADS))
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the prefill_32k and chunk_1m lines beside the headline")
    ap.add_argument("--cpu-rows", type=int, default=0, help="oracle sample rows (0 = auto)")
    ap.add_argument("--seq", type=int, default=0,
                    help="prefill length override (a smaller case of the same structure, "
                         "e.g. for profiling); needles scale with the length")
    ap.add_argument("--index-dtype", default="", choices=["", "fp8", "nvfp4"],
                    help="fp8: q_idx and k_idx in fp8 e4m3 (bf16 workloads)")
    ap.add_argument("--qk-dtype", default="", choices=["", "fp8"],
                    help="fp8: the main branch's q and k in fp8 e4m3, v bf16 (bf16 workloads)")
    ap.add_argument("--paged", action="store_true",
                    help="k, v and k_idx in a shuffled pool of 128-token pages (paged KV "
                         "cache, block table) instead of contiguous sequences")
    ap.add_argument("--index-kl", action="store_true",
                    help="time the KL-alignment loss and its index-branch gradients "
                         "(training side, msa_index_kl) instead of the forward")
    ap.add_argument("--batch", type=int, default=0,
                    help="batch override (a smaller case of the same structure, e.g. for "
                         "profiling); needles per sequence are kept")
    a = ap.parse_args()
    if a.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if a.index_dtype == "nvfp4" and (a.paged or a.index_kl or a.impl == "reference"):
        raise SystemExit("--index-dtype nvfp4 is measured on contiguous forward steps only")
    world, rank, local = dist_setup()
    w = WORKLOADS[a.workload]
    if a.seq:
        if w.q_pos0 != 0 or w.batch != 1:
            raise SystemExit("--seq applies to the prefill workloads")
        w = w.with_(name=f"{w.name}@{a.seq}", q_len=a.seq, kv_len=a.seq,
                    needles=max(1, w.needles * a.seq // w.q_len))
    suffix = (f"+idx_{a.index_dtype}" if a.index_dtype else "") + \
        (f"+qk_{a.qk_dtype}" if a.qk_dtype else "") + ("+paged" if a.paged else "")
    w = w.with_(name=w.name + suffix, index_dtype=a.index_dtype, qk_dtype=a.qk_dtype)
    if a.batch:
        w = w.with_(name=f"{w.name}@b{a.batch}", batch=a.batch)
    peaks, peak_src = load_peaks()

    if a.index_kl and a.impl != "reference":
        return bench_index_kl(a, w, world, rank, local, peaks)

    if a.impl == "reference":
        # the reference arm is the fp64 oracle on the host cores, rank 0 only
        if rank != 0:
            barrier(world)
            return
        dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
        x = make_inputs(w, seed=0, device=dev)
        n_rows = a.cpu_rows or oracle_rows(w)
        # every step times the same evenly spread rows as the cpu_baseline leg
        vals = [time_oracle(w, x, n_rows) for _ in range(a.warmup + a.steps)]
        timed = vals[a.warmup:]
        v = statistics.mean(t["value"] for t in timed)
        ms = w.rows / v * 1e3
        cb = dict(timed[-1])
        cb["value"] = v
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "query-tokens/s",
                "n_gpus": world, "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64", "data": "synthetic",
                "config": workload_config(w, world),
                "cpu_baseline": cb,
                "e2e": {"value": v, "unit": "query-tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0},
                "gpu_launches": 0}
        print(json.dumps(line), flush=True)
        barrier(world)
        return

    from block_sparse_gqa_04_b200 import msa
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    msa.load()
    barrier(world)
    main_res = measure_workload(msa, w, dev, a.steps, a.warmup, peaks, not a.no_e2e,
                                paged=a.paged)
    value, ms = weak_value(w.rows, main_res["ms"], world)
    cnt = main_res["cnt"]
    line = {
        "metric": METRIC, "value": value, "unit": "query-tokens/s", "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": ("f32" if w.dtype == "f32" else
                  "e2m1+bf16" if w.index_dtype == "nvfp4" else
                  "e4m3+bf16" if (w.index_dtype == "fp8" or w.qk_dtype == "fp8") else "bf16"),
        "data": "synthetic (seeded N(0,1/d) inputs with planted needle blocks)",
        "config": dict(workload_config(w, world), kernel_path=main_res["path"],
                       l2="inputs larger than L2 (q alone is %.2f GB per step)" %
                          (main_res["x"]["q"].numel() * main_res["x"]["q"].element_size() / 1e9)),
        "clocks": main_res["clocks"],
        "gpu_launches": main_res["launches"],
        "stage_ms": {k: round(v, 4) for k, v in main_res["stage"].items()},
        "roofline": kernel_roofline(w, cnt, main_res["stage"], main_res["path"], peaks,
                                    main_res["kv_sel"]),
        "path_roofline": path_roofline(cnt, main_res["kv_sel"], ms, peaks),
        "peaks": {"source": peak_src, "hbm_gbs": peaks["hbm_gbs"],
                  "bf16_tflops": peaks["bf16_tflops"],
                  "bf16_tflops_sustained": peaks.get("bf16_tflops_sustained")},
    }
    if "e2e" in main_res:
        e_ms, h2d, d2h = main_res["e2e"]
        e_val, e_ms = weak_value(w.rows, e_ms, world)
        line["e2e"] = {"value": e_val, "unit": "query-tokens/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "ms_per_step": e_ms}
    x_main = main_res.pop("x")
    if not a.no_decode:
        wd = WORKLOADS["decode_128k"]
        wd = wd.with_(name=wd.name + suffix, index_dtype=a.index_dtype, qk_dtype=a.qk_dtype)
        del x_main
        torch.cuda.empty_cache()
        dres = measure_workload(msa, wd, dev, a.steps, a.warmup, peaks, False, paged=a.paged)
        dval, dms = weak_value(wd.rows, dres["ms"], world)
        dcnt = dres["cnt"]
        dbytes = dcnt["kidx_bytes"] + dres["kv_sel"]
        line["decode"] = {
            "workload": wd.name, "value": dval, "unit": "tokens/s",
            "ms_per_step": dms, "kernel_path": dres["path"],
            "stage_ms": {k: round(v, 4) for k, v in dres["stage"].items()},
            "hbm_roofline": {"bytes": dbytes, "t_roofline_ms": dbytes / (peaks["hbm_gbs"] * 1e9) * 1e3,
                             "achieved_gbs": dbytes / (dms * 1e-3) / 1e9,
                             "frac": dbytes / (peaks["hbm_gbs"] * 1e9) / (dms * 1e-3)},
            "clocks": dres["clocks"]}
        dres.pop("x")
        x_main = None
    extra_names = [] if (a.no_extra or a.seq or a.batch or a.index_kl) else \
        [n for n in ("prefill_32k", "chunk_1m") if n != a.workload]
    for name in extra_names:
        # the other large workloads, each timed the same way (steps, warm-up,
        # CUDA events, max over ranks) and reported beside the headline
        we = WORKLOADS[name]
        we = we.with_(name=we.name + suffix, index_dtype=a.index_dtype, qk_dtype=a.qk_dtype)
        torch.cuda.empty_cache()
        eres = measure_workload(msa, we, dev, a.steps, a.warmup, peaks, False, paged=a.paged)
        eval_, ems = weak_value(we.rows, eres["ms"], world)
        line[name] = {
            "workload": we.name, "value": eval_, "unit": "query-tokens/s",
            "ms_per_step": ems, "kernel_path": eres["path"],
            "stage_ms": {k: round(v, 4) for k, v in eres["stage"].items()},
            "roofline": kernel_roofline(we, eres["cnt"], eres["stage"], eres["path"], peaks,
                                        eres["kv_sel"]),
            "path_roofline": path_roofline(eres["cnt"], eres["kv_sel"], ems, peaks),
            "gpu_launches": eres["launches"], "clocks": eres["clocks"]}
        eres.pop("x")
    if extra_names and not (a.index_dtype or a.qk_dtype or a.paged):
        # a packed batch of sequences of different lengths (msa_forward_varlen)
        torch.cuda.empty_cache()
        vres = measure_varlen(msa, dev, a.steps, a.warmup, peaks)
        vval, vms = weak_value(vres["rows"], vres["ms"], world)
        line["varlen_mix"] = {
            "workload": "varlen_mix", "sequences": vres["sequences"],
            "query_rows": vres["rows"], "value": vval, "unit": "query-tokens/s",
            "ms_per_step": vms, "path_roofline": path_roofline(vres["cnt"], vres["kv_sel"], vms,
                                                               peaks),
            "gpu_launches": vres["launches"], "clocks": vres["clocks"]}
    if rank == 0 and world == 1 and not a.no_cpu_baseline and w.index_dtype != "nvfp4":
        # the oracle runs on host copies of the bench's own inputs
        xm = make_inputs(w, seed=0, device=dev)
        xm.pop("needles")
        line["cpu_baseline"] = time_oracle(w, xm, a.cpu_rows or oracle_rows(w))
    if rank == 0:
        print(json.dumps(line), flush=True)
    barrier(world)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
