#!/usr/bin/env python3
"""Benchmark of the SAS gated block-sparse attention hot path on B200.

One step = one pass of the whole prefill/training path over the workload's inputs
(already resident in HBM): key pooling -> gate keys -> gate scores -> Top-K -> gated
attention forward -> gated attention backward. The headline workload is the largest
single-GPU configuration, the Qwen3-14B-shaped varlen training step (4 packed sequences of
8k..64k tokens, 40 query / 8 KV heads, Top-K 63). The Qwen3-4B 32k training step, the 32k
forward-only prefill and the batch-64 decode step are measured beside it and reported under
their own keys in the same line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sas|reference]

For N > 1 (torchrun, one rank per GPU) every rank runs its own replica of the workload
(the path shards into independent problems; no collective touches the data), the
timing is the max over ranks, and `value` counts the work of all ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import sas_inputs as si  # noqa: E402

METRIC = "gated sparse attn TFLOP/s (attended, fwd/bwd) + decode tok/s; % of B200 roofline"
HEADLINE_WORKLOAD = "qwen3-14b-varlen-4seq"      # the largest single-GPU configuration
EXTRA_WORKLOADS = ("qwen3-4b-train-32k", "qwen3-4b-prefill-32k")
EXTRA_KEYS = {"qwen3-4b-train-32k": "train_32k", "qwen3-4b-prefill-32k": "prefill_32k"}
DECODE_WORKLOAD = "qwen3-8b-decode-b64"
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="sas", choices=["sas", "reference"])
    ap.add_argument("--workload", default=HEADLINE_WORKLOAD)
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other prefill/training workloads (profiling)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-train", action="store_true", help="decode step only (profiling)")
    ap.add_argument("--decode-workload", default=DECODE_WORKLOAD)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=256, help="oracle rows per CPU-baseline sample")
    ap.add_argument("--step-only", action="store_true",
                    help="the headline step alone: no e2e, side legs, other workloads, decode or "
                         "CPU baseline (profiling)")
    return ap.parse_args()


# ------------------------------------------------------------------------------------------
# distributed plumbing
# ------------------------------------------------------------------------------------------

def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                              device_id=torch.device("cuda", local))
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, ws: int, dev) -> float:
    if ws == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ------------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return None
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return None
        hi = max(sm)
        loaded = [x for x in sm if x >= 0.5 * hi] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------
# helpers
# ------------------------------------------------------------------------------------------

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), \
            "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def source_sha(files) -> str:
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(op: str, workload: str):
    """DRAM bytes per launch of `op` on `workload` from the committed ncu summary, if the
    kernel sources it was taken with are unchanged (None otherwise)."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(f"{op}@{workload}")
    if not d:
        return None
    try:
        if source_sha(d["sources"]) != d["source_sha"]:
            return None
    except OSError:
        return None
    return d["bytes_per_launch"]


def attended_pairs_gpu(idx: torch.Tensor, cu: torch.Tensor, block: int) -> int:
    """(token, kv, key) pairs with a finite logit, counted on the device from the selection."""
    T = idx.shape[0]
    cu64 = cu.long()
    tok = torch.arange(T, device=idx.device)
    seq = torch.searchsorted(cu64[1:], tok, right=True)
    pos = tok - cu64[seq]
    j = idx.long()
    lo = j * block
    hi = torch.minimum((j + 1) * block, pos[:, None, None] + 1)
    n = torch.where(j >= 0, (hi - lo).clamp(min=0), torch.zeros_like(j))
    return int(n.sum().item())


def km_stats(idx: torch.Tensor, cu: torch.Tensor, lengths, Mq: int, Hkv: int, NBmax: int):
    """Work the key-major tensor-core kernels do on this selection.

    Items are (kv head, sequence, 4096-token window, kept block); an item with c kept
    (token, block) pairs runs ceil(c / Mq) gathered 128-row tiles. Returns (tiles, rows):
    the tile count and the number of gathered (token, block) pairs (x G heads = MMA rows).
    """
    T = idx.shape[0]
    dev = idx.device
    cu64 = cu.long()
    tok = torch.arange(T, device=dev)
    seq = torch.searchsorted(cu64[1:], tok, right=True)
    w = (tok - cu64[seq]) // 4096
    nW = (max(lengths) + 4095) // 4096
    j = idx.long()
    kvi = torch.arange(Hkv, device=dev)[None, :, None].expand_as(j)
    ent = ((kvi * len(lengths) + seq[:, None, None]) * nW + w[:, None, None]) * NBmax + j.clamp(min=0)
    cnt = torch.bincount(ent[j >= 0], minlength=Hkv * len(lengths) * nW * NBmax)
    return int(((cnt + Mq - 1) // Mq).sum().item()), int(cnt.sum().item())


class Timer:
    """CUDA events around each op of a step, on the stream the library launches on."""

    def __init__(self):
        self.ops = {}

    def run(self, name, fn):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        r = fn()
        e.record()
        self.ops.setdefault(name, []).append((s, e))
        return r

    def mean_ms(self):
        return {k: sum(a.elapsed_time(b) for a, b in v) / len(v) for k, v in self.ops.items()}


# ------------------------------------------------------------------------------------------
# the prefill / training step
# ------------------------------------------------------------------------------------------

def train_step(sas, prob, g, backward: bool, timer: Timer | None = None):
    run = timer.run if timer is not None else (lambda name, fn: fn())
    pooled = run("sas_pool_keys", lambda: sas.sas_pool_keys(prob, g["k_nope"], pooled=g["_pooled"]))
    gk = run("sas_gate_keys", lambda: sas.sas_gate_keys(prob, pooled, g["wk"], g["knorm_w"],
                                                        gate_keys=g["_gk"]))
    # gate scores + Top-K: the two kernels through an HBM score matrix, the faster path on
    # B200 today (the fused pass that keeps the scores on chip is timed beside it, gate_paths)
    scores, lse = run("sas_gate_scores", lambda: sas.sas_gate_scores(
        prob, g["q_nope"], g["k_nope"], gk, g["wq"], g["qnorm_w"], g["wk"], g["knorm_w"],
        scores=g["_scores"], lse=g["_glse"], workspace=g["_wsgs"]))
    idx, logg = run("sas_topk", lambda: sas.sas_topk(prob, scores, lse, idx=g["_idx"],
                                                     logg=g["_logg"]))
    o, alse = run("sas_attn_fwd", lambda: sas.sas_attn_fwd(prob, g["q"], g["k"], g["v"], idx, logg,
                                                           o=g["_o"], lse=g["_alse"],
                                                           workspace=g["_wsf"]))
    out = [o, alse, idx, logg]
    if backward:
        grads = run("sas_attn_bwd", lambda: sas.sas_attn_bwd(
            prob, g["q"], g["k"], g["v"], o, g["dout"], alse, idx, logg, dq=g["_dq"], dk=g["_dk"],
            dv=g["_dv"], dlogg=g["_dlogg"], workspace=g["_wsb"]))
        out += list(grads)
    return out


def alloc_outputs(sas, prob, g, backward):
    import ctypes
    dev = prob.device
    T, Hq, Hkv, d, K, NB, h = (prob.total_tokens, prob.num_q_heads, prob.num_kv_heads,
                               prob.head_dim, prob.topk, prob.max_blocks, prob.gate_hidden)
    g["_pooled"] = torch.empty((prob.batch, NB, Hkv, 3 * d), dtype=torch.float32, device=dev)
    g["_gk"] = torch.empty((prob.batch, NB, Hkv, h), dtype=torch.float32, device=dev)
    g["_scores"] = torch.empty((T, prob.sel_heads, NB), dtype=torch.float32, device=dev)
    g["_glse"] = torch.empty((T, prob.sel_heads), dtype=torch.float32, device=dev)
    g["_idx"] = torch.empty((T, Hkv, K + 1), dtype=torch.int32, device=dev)
    g["_logg"] = torch.empty((T, Hkv, K + 1), dtype=torch.float32, device=dev)
    g["_o"] = torch.empty((T, Hq, d), dtype=prob.dtype, device=dev)
    g["_alse"] = torch.empty((T, Hq), dtype=torch.float32, device=dev)
    lib = sas.lib_handle()
    n = ctypes.c_size_t(0)
    lib.sas_gate_select_workspace_size(prob.ref, ctypes.byref(n))
    g["_wsg"] = torch.empty(max(256, n.value), dtype=torch.uint8, device=dev)
    lib.sas_gate_scores_workspace_size(prob.ref, ctypes.byref(n))
    g["_wsgs"] = torch.empty(max(256, n.value), dtype=torch.uint8, device=dev)
    lib.sas_attn_fwd_workspace_size(prob.ref, ctypes.byref(n))
    g["_wsf"] = torch.empty(max(256, n.value), dtype=torch.uint8, device=dev)
    if backward:
        g["_dq"] = torch.empty_like(g["q"])
        g["_dk"] = torch.empty_like(g["k"])
        g["_dv"] = torch.empty_like(g["v"])
        g["_dlogg"] = torch.empty((T, Hkv, K + 1), dtype=torch.float32, device=dev)
        lib.sas_attn_bwd_workspace_size(prob.ref, ctypes.byref(n))
        g["_wsb"] = torch.empty(max(256, n.value), dtype=torch.uint8, device=dev)


def bench_gate_paths(sas, prob, g, flush, steps):
    """Gate scores + Top-K two ways on the step's inputs: the fused pass (score rows kept on
    chip) and the two separate kernels (the [T, Hs, NBmax] scores written to and read back
    from HBM). Both give the same selection; timed after the step, not part of it."""
    scores, lse, wsu = g["_scores"], g["_glse"], g["_wsgs"]
    args = (prob, g["q_nope"], g["k_nope"], g["_gk"], g["wq"], g["qnorm_w"], g["wk"], g["knorm_w"])

    def fused():
        sas.sas_gate_select(*args, idx=g["_idx"], logg=g["_logg"], workspace=g["_wsg"])

    def unfused():
        sas.sas_gate_scores(*args, scores=scores, lse=lse, workspace=wsu)
        sas.sas_topk(prob, scores, lse, idx=g["_idx"], logg=g["_logg"])

    out = {}
    for name, fn in (("fused_ms", fused), ("unfused_ms", unfused)):
        for _ in range(2):
            fn()
        ev = []
        for _ in range(steps):
            flush.zero_()
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_.record()
            fn()
            b_.record()
            ev.append((a_, b_))
        torch.cuda.synchronize()
        out[name] = sum(x.elapsed_time(y) for x, y in ev) / len(ev)
    out["score_bytes_avoided"] = 2 * scores.numel() * 4
    sas.check_workspace(g["_wsg"], "sas_gate_select")
    return out


def bench_router_bwd(sas, prob, g, flush, steps):
    """The router backward (gate parameter gradients from the step's own dlogg), timed on its
    own after the step: it is not part of the timed step."""
    import ctypes
    n = ctypes.c_size_t(0)
    if sas.lib_handle().sas_gate_bwd_workspace_size(prob.ref, ctypes.byref(n)) != 0:
        return {"unsupported": sas.lib_handle().sas_last_error().decode()}
    ws = torch.empty(max(256, n.value), dtype=torch.uint8, device=prob.device)
    args = (prob, g["q_nope"], g["k_nope"], g["_pooled"], g["wq"], g["qnorm_w"], g["wk"],
            g["knorm_w"], g["_idx"], g["_dlogg"])
    for _ in range(2):
        sas.sas_gate_bwd(*args, workspace=ws)
    times = []
    for _ in range(steps):
        flush.zero_()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        sas.sas_gate_bwd(*args, workspace=ws)
        e.record()
        times.append((s, e))
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in times) / len(times)
    T, Hkv, h, d = prob.total_tokens, prob.num_kv_heads, prob.gate_hidden, prob.head_dim
    G = prob.num_q_heads // Hkv
    outer = 2.0 * T * Hkv * h * (G * d + 3 * d) + 2.0 * prob.batch * prob.max_blocks * Hkv * h * 3 * d
    return {"ms": ms, "outer_product_gflop": outer / 1e9, "achieved_tflops": outer / (ms * 1e-3) / 1e12,
            "note": "dWq, dWk, norm-weight gradients from the step's dlogg; the token-row outer "
                    "products as tcgen05 GEMMs (dx split into bf16 hi + lo), the block-row ones on "
                    "CUDA cores; timed separately, not part of the step"}


# ------------------------------------------------------------------------------------------
# oracle sample (CPU baseline and the reference arm)
# ------------------------------------------------------------------------------------------

def oracle_sample(cpu_inp, shape, rows, backward):
    """Oracle gate + Top-K + attention (fwd, and bwd rows) on some query rows; returns the
    attended FLOPs those rows represent (fwd 4*pairs*d per head, row-bwd 6*pairs*d per head:
    recompute, dP, dQ)."""
    from oracle import sas_oracle as orc
    B, K, d, G = shape.block, shape.topk, shape.head_dim, shape.group
    sel = orc.prefill_selection(cpu_inp["q_nope"], cpu_inp["k_nope"], cpu_inp["wq"],
                                cpu_inp["qnorm_w"], cpu_inp["wk"], cpu_inp["knorm_w"],
                                shape.cu_seqlens, B, K, shape.rms_eps, shape.gate_rope_base, rows)
    idx = np.full((shape.total_tokens, shape.num_kv_heads, K + 1), -1, dtype=np.int32)
    logg = np.zeros(idx.shape)
    idx[rows], logg[rows] = sel["idx"], sel["logg"]
    orc.attention_fwd(cpu_inp["q"], cpu_inp["k"], cpu_inp["v"], idx, logg, shape.cu_seqlens, B,
                      rows=rows)
    if backward:
        orc.attention_bwd_rows(cpu_inp["q"], cpu_inp["k"], cpu_inp["v"], cpu_inp["dout"], idx, logg,
                               shape.cu_seqlens, B, rows)
    pos = shape.positions()[rows]
    j = sel["idx"].astype(np.int64)
    lo = j * B
    hi = np.minimum((j + 1) * B, pos[:, None, None] + 1)
    pairs = int(np.where(j >= 0, np.maximum(hi - lo, 0), 0).sum())
    return pairs * G * d * (4 + (6 if backward else 0))


def cpu_inputs_from(g):
    keys = ("q_nope", "k_nope", "q", "k", "v", "dout", "wq", "wk", "qnorm_w", "knorm_w")
    return {k: g[k].float().cpu().numpy().astype(np.float64) for k in keys if k in g}


def sample_rows(shape, n, seed):
    r = np.random.Generator(np.random.PCG64(seed))
    return np.sort(r.choice(shape.total_tokens, size=n, replace=False))


# ------------------------------------------------------------------------------------------
# decode
# ------------------------------------------------------------------------------------------

def bench_decode(sas, dev, steps, warmup, flush, hbm_peak, name=DECODE_WORKLOAD):
    shp = si.decode_workload(name)
    inp = si.decode_inputs(shp, device=dev)
    prob = sas.DecodeProblem(seqlens=inp["lengths"], capacity=shp.capacity,
                             num_q_heads=shp.num_q_heads, num_kv_heads=shp.num_kv_heads,
                             head_dim=shp.head_dim, block=shp.block, topk=shp.topk,
                             gate_hidden=shp.gate_hidden, dtype=torch.bfloat16)
    import ctypes
    n = ctypes.c_size_t(0)
    sas.lib_handle().sas_decode_workspace_size(prob.ref, ctypes.byref(n))
    ws = torch.empty(max(256, n.value), dtype=torch.uint8, device=dev)
    o = torch.empty((shp.batch, shp.num_q_heads, shp.head_dim), dtype=torch.bfloat16, device=dev)
    idx = torch.empty((shp.batch, shp.num_kv_heads, shp.topk + 1), dtype=torch.int32, device=dev)
    logg = torch.empty(idx.shape, dtype=torch.float32, device=dev)

    def step():
        return sas.sas_decode(prob, inp["q"], inp["q_nope"], inp["k_cache"], inp["v_cache"],
                              inp["gate_key_cache"], inp["cur_pool"], inp["wq"], inp["qnorm_w"],
                              inp["wk"], inp["knorm_w"], o=o, idx_out=idx, logg_out=logg,
                              workspace=ws)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    sas.check_workspace(ws, "sas_decode")
    ts = []
    for _ in range(steps):
        flush.zero_()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        step()
        e.record()
        ts.append((s, e))
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in ts) / len(ts)
    # algorithmic bytes: the selected K/V rows, every cached gate key of the complete blocks,
    # q, q_nope, pool state, gate weights, O
    L = inp["lengths"].long()
    B = shp.block
    j = idx.long()
    pos = (L - 1)[:, None, None]
    keys = torch.where(j >= 0, (torch.minimum((j + 1) * B, pos + 1) - j * B).clamp(min=0),
                       torch.zeros_like(j)).sum().item()
    kv_bytes = keys * shp.head_dim * 2 * 2
    c = ((L - 1) // B)
    gk_bytes = int(c.sum().item()) * shp.num_kv_heads * shp.gate_hidden * 2
    other = (2 * shp.batch * shp.num_q_heads * shp.head_dim * 2 + shp.batch * shp.num_kv_heads * 3
             * shp.head_dim * 4 + inp["wq"].numel() * 2 + inp["wk"].numel() * 2
             + shp.batch * shp.num_q_heads * shp.head_dim * 2)
    total = kv_bytes + gk_bytes + other
    gbs = total / (ms * 1e-3) / 1e9
    return {
        "metric": "decode tok/s", "value": shp.batch / (ms * 1e-3), "unit": "tok/s",
        "ms_per_step": ms, "config": {"workload": name, "batch": shp.batch,
                                      "context_min": int(L.min()), "context_max": int(L.max()),
                                      "budget_tokens": (shp.topk + 1) * B},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
                     "frac": gbs / hbm_peak, "traffic": ncu_traffic("sas_decode", name),
                     "algorithmic_bytes": total, "selected_kv_bytes": kv_bytes,
                     "gate_key_bytes": gk_bytes, "peak_source": "measured copy, of measured"},
        "selected_kv_gbs": kv_bytes / (ms * 1e-3) / 1e9,
    }


# ------------------------------------------------------------------------------------------
# one prefill / training workload: resident inputs, timed steps, per-op events
# ------------------------------------------------------------------------------------------

def setup_workload(sas, name, dev):
    shape = si.workload(name)
    backward = "train" in name or "varlen" in name
    g = si.prefill_inputs(shape, device=dev, with_dout=backward)
    prob = sas.Problem.from_lengths(shape.lengths, dev, num_q_heads=shape.num_q_heads,
                                    num_kv_heads=shape.num_kv_heads, head_dim=shape.head_dim,
                                    block=shape.block, topk=shape.topk,
                                    gate_hidden=shape.gate_hidden, dtype=shape.torch_dtype)
    alloc_outputs(sas, prob, g, backward)
    return shape, backward, g, prob


def check_error_words(sas, g, backward):
    """The device-side error words of the step's last calls (0 = none); raises otherwise."""
    sas.check_workspace(g["_wsgs"], "sas_gate_scores")
    sas.check_workspace(g["_wsf"], "sas_attn_fwd")
    if backward:
        sas.check_workspace(g["_wsb"], "sas_attn_bwd")


def time_workload(sas, name, shape, backward, g, prob, steps, warmup, flush, ws, dev, clk=None):
    """Warm up, check the error words, then time `steps` whole steps (L2 flushed between
    steps) with CUDA events around the step and around each op."""
    for _ in range(max(3, warmup)):
        out = train_step(sas, prob, g, backward)
    torch.cuda.synchronize()
    check_error_words(sas, g, backward)
    pairs = attended_pairs_gpu(out[2], prob.cu_seqlens, shape.block)
    G, d = shape.group, shape.head_dim
    fwd_flops = 4.0 * pairs * G * d
    bwd_flops = 2.5 * fwd_flops if backward else 0.0
    # tokens per gathered 128-row tile: forward 25 (G = 5) or 128 / G; backward whole tokens
    # per warp, 4 floor(32 / G)
    tiles, kept = km_stats(out[2], prob.cu_seqlens, shape.lengths, 25 if G == 5 else 128 // G,
                           shape.num_kv_heads, prob.max_blocks)
    tiles_bwd, _ = km_stats(out[2], prob.cu_seqlens, shape.lengths, 4 * (32 // G),
                            shape.num_kv_heads, prob.max_blocks)
    timer = Timer()
    evs = []
    barrier(ws)
    torch.cuda.synchronize()
    n0 = sas.kernel_launches()
    ctx = clk if clk is not None else _Null()
    with ctx:
        for _ in range(steps):
            flush.zero_()
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            train_step(sas, prob, g, backward, timer)
            e.record()
            evs.append((s, e))
        torch.cuda.synchronize()
    barrier(ws)
    launches = sas.kernel_launches() - n0
    check_error_words(sas, g, backward)
    ms = sum(x.elapsed_time(y) for x, y in evs) / len(evs)
    ms = max_over_ranks(ms, ws, dev)
    return dict(ms=ms, ops=timer.mean_ms(), pairs=pairs, fwd_flops=fwd_flops, bwd_flops=bwd_flops,
                tiles=tiles, tiles_bwd=tiles_bwd, kept=kept, launches=launches)


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def choose_tc_peak(clocks, burst, sustained, src):
    """The bf16 denominator for the clocks seen during the timed region: the burst figure
    when the SM clock held its maximum, the sustained (power-capped) figure otherwise."""
    if clocks and clocks.get("sm_max_mhz") and clocks["sm_mhz"] >= 0.95 * clocks["sm_max_mhz"]:
        return burst, (f"bf16 dense burst (SM clock at its maximum, median "
                       f"{clocks['sm_mhz']:.0f} MHz, during the timed region), of {src}")
    return sustained, f"bf16 dense sustained (power-capped clocks), of {src}"


def summarise(name, shape, backward, r, peak, peak_note, ws):
    """The workload's numbers: attended TFLOP/s, per-op times, roofline of the dominant
    attention pass, the key-major kernels' computed work and L2 reduction traffic."""
    ops = r["ops"]
    G, d = shape.group, shape.head_dim
    work = r["fwd_flops"] + r["bwd_flops"]
    mma = 2.0 * 128 * 64 * d                           # one 128-row x 64-key x d product
    comp_fwd = r["tiles"] * 2 * mma                    # S = Q K^T, O = P V per gathered tile
    comp_bwd = r["tiles_bwd"] * 5 * mma if backward else 0.0   # S, dP, dV^T, dK^T, dQ
    red_bytes = r["kept"] * G * d * 4                  # fp32 partial rows reduced into L2
    dom = max(("sas_attn_fwd", "sas_attn_bwd") if backward else ("sas_attn_fwd",),
              key=lambda k: ops[k])
    dflops = r["fwd_flops"] if dom == "sas_attn_fwd" else r["bwd_flops"]
    ach = dflops / (ops[dom] * 1e-3) / 1e12
    return {
        "value": work * ws / (r["ms"] * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": r["ms"],
        "config": {"workload": name, "batch": shape.batch, "seq_len": shape.max_seqlen,
                   "seq_lens": list(shape.lengths), "total_tokens": shape.total_tokens,
                   "num_q_heads": shape.num_q_heads, "num_kv_heads": shape.num_kv_heads,
                   "head_dim": d, "block": shape.block, "topk": shape.topk,
                   "gate_hidden": shape.gate_hidden, "passes": "fwd+bwd" if backward else "fwd",
                   "parallelism": f"replicas x{ws}", "l2": "flushed (256 MiB write) between steps"},
        "attended": {"pairs_per_kv_head_total": r["pairs"], "fwd_tflop": r["fwd_flops"] / 1e12,
                     "bwd_tflop": r["bwd_flops"] / 1e12,
                     "dense_causal_fraction": r["pairs"] / (shape.num_kv_heads * sum(
                         L * (L + 1) / 2 for L in shape.lengths))},
        "computed": {"fwd_tflop": comp_fwd / 1e12, "bwd_tflop": comp_bwd / 1e12,
                     "gathered_tiles": r["tiles"], "gathered_tiles_bwd": r["tiles_bwd"],
                     "attended_over_computed": work / max(1.0, comp_fwd + comp_bwd),
                     "fwd_tflops": comp_fwd / (ops["sas_attn_fwd"] * 1e-3) / 1e12,
                     "bwd_tflops": (comp_bwd / (ops["sas_attn_bwd"] * 1e-3) / 1e12) if backward else None,
                     "l2_reduction_gb_per_pass": red_bytes / 1e9,
                     "fwd_l2_reduction_gbs": red_bytes / (ops["sas_attn_fwd"] * 1e-3) / 1e9,
                     "bwd_l2_reduction_gbs": (red_bytes / (ops["sas_attn_bwd"] * 1e-3) / 1e9)
                     if backward else None,
                     "note": "key-major kernels: gathered 128-row tiles per (kv, window, kept "
                             "block); each kept (token, block) pair adds G fp32 rows of d "
                             "values into L2 (O in the forward, dQ in the backward)"},
        "ops_ms": ops,
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": ach, "peak": peak,
                     "unit": "TFLOP/s", "frac": ach / peak, "traffic": ncu_traffic(dom, name),
                     "peak_source": peak_note, "algorithmic_flops_per_launch": dflops},
        "gpu_launches": r["launches"],
    }


# ------------------------------------------------------------------------------------------
# main
# ------------------------------------------------------------------------------------------

def main():
    a = parse()
    if a.step_only:
        a.no_e2e = a.no_extra = a.no_decode = a.no_cpu_baseline = True
    ws, rank, local = dist_setup()
    if a.impl == "reference":
        return reference_arm(a, ws, rank)
    import gated_block_sparse_sas_b200 as sas
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    hbm_peak, tc_burst, tc_sust, peak_src = measured_peaks()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    if a.no_train:
        print(json.dumps(bench_decode(sas, dev, max(1, a.steps), max(3, a.warmup), flush, hbm_peak,
                                      a.decode_workload)), flush=True)
        return

    # ---- the headline workload ------------------------------------------------------------
    shape, backward, g, prob = setup_workload(sas, a.workload, dev)
    clk = ClockSampler(dev.index)
    r = time_workload(sas, a.workload, shape, backward, g, prob, a.steps, a.warmup, flush, ws, dev,
                      clk)
    cs = clk.summary()
    peak, peak_note = choose_tc_peak(cs, tc_burst, tc_sust, peak_src)
    head = summarise(a.workload, shape, backward, r, peak, peak_note, ws)
    line = {
        "metric": METRIC, "value": head["value"], "unit": "TFLOP/s", "n_gpus": ws,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if shape.dtype == "bf16" else "f32",
        "data": "synthetic (seeded counter-based generator, approx. N(0,1))",
        "config": head["config"], "attended": head["attended"], "computed": head["computed"],
        "ops_ms": head["ops_ms"], "roofline": head["roofline"], "gpu_launches": head["gpu_launches"],
    }
    if cs:
        line["clocks"] = cs
    if not a.no_e2e:
        line["e2e"] = e2e(sas, prob, g, backward, r["fwd_flops"] + r["bwd_flops"], dev, a, ws)
    if backward and not a.step_only:   # after the timed step and e2e, so they cannot perturb them
        line["router_bwd"] = bench_router_bwd(sas, prob, g, flush, max(3, a.steps))
    if not a.step_only:
        line["gate_paths"] = bench_gate_paths(sas, prob, g, flush, max(3, a.steps))
    if rank == 0 and ws == 1 and not a.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(g, shape, backward, a)
    del g, prob
    torch.cuda.empty_cache()

    # ---- the other prefill / training workloads, each its own key -------------------------
    if not a.no_extra:
        for name in EXTRA_WORKLOADS:
            if name == a.workload:
                continue
            shp, bwd, ge, pe = setup_workload(sas, name, dev)
            ce = ClockSampler(dev.index)
            re_ = time_workload(sas, name, shp, bwd, ge, pe, a.steps, a.warmup, flush, ws, dev, ce)
            cse = ce.summary()
            pk, pn = choose_tc_peak(cse, tc_burst, tc_sust, peak_src)
            ex = summarise(name, shp, bwd, re_, pk, pn, ws)
            if cse:
                ex["clocks"] = cse
            line[EXTRA_KEYS[name]] = ex
            del ge, pe
            torch.cuda.empty_cache()

    if not a.no_decode:
        try:
            line["decode"] = bench_decode(sas, dev, max(3, a.steps), max(3, a.warmup), flush, hbm_peak,
                                          a.decode_workload)
        except torch.OutOfMemoryError as ex:   # pragma: no cover
            line["decode"] = {"error": f"out of memory: {ex}"[:200]}

    line["extra_keys"] = [k for k in line if k in ("train_32k", "prefill_32k", "decode",
                                                   "router_bwd", "gate_paths", "computed",
                                                   "attended", "ops_ms")]
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        torch.distributed.destroy_process_group()


def cpu_baseline(g, shape, backward, a):
    """The oracle, as it stands, on sampled query rows of the workload's shortest sequence at
    its full length (rows of different sequences are independent), timed on the host cores."""
    b = int(np.argmin(shape.lengths))
    s0, L = int(shape.cu_seqlens[b]), shape.lengths[b]
    one = si.sequence_shape(shape, b)
    keys = ("q_nope", "k_nope", "q", "k", "v", "dout", "wq", "wk", "qnorm_w", "knorm_w")
    tok = ("q_nope", "k_nope", "q", "k", "v", "dout")
    cpu = {k: (g[k][s0:s0 + L] if k in tok else g[k]).float().cpu().numpy().astype(np.float64)
           for k in keys if k in g}
    rows = sample_rows(one, a.cpu_rows, 7)
    threads = torch.get_num_threads()
    t0 = time.perf_counter()
    fl = oracle_sample(cpu, one, rows, backward)
    dt = time.perf_counter() - t0
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "seconds": dt,
            "sample": f"{len(rows)} random query rows of sequence {b} ({L} tokens) of "
                      f"{a.workload} (gate, Top-K, attention fwd" +
                      (" + dQ/dlogg rows" if backward else "") +
                      ") at full sequence length, fp64 numpy"}


def link_probe(dev, nbytes=1 << 30):
    """Pinned host <-> device copy bandwidth (GB/s): each direction alone and both at once
    (two streams), best of 3, CUDA events. The end-to-end step moves its inputs and results over
    this link, so it bounds that step from below."""
    h_in = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    h_out = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    d_in = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    d_out = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def run(h2d, d2h):   # best (ms) of 3 trials per direction; 0 for a direction not run
        th, td = [], []
        for _ in range(3):
            torch.cuda.synchronize()
            a0, a1, b0, b1 = ev(), ev(), ev(), ev()
            with torch.cuda.stream(s1):
                a0.record(s1)
                if h2d:
                    d_in.copy_(h_in, non_blocking=True)
                a1.record(s1)
            with torch.cuda.stream(s2):
                b0.record(s2)
                if d2h:
                    h_out.copy_(d_out, non_blocking=True)
                b1.record(s2)
            torch.cuda.synchronize()
            th.append(a0.elapsed_time(a1))
            td.append(b0.elapsed_time(b1))
        return (min(th) if h2d else 0.0), (min(td) if d2h else 0.0)

    h, _ = run(True, False)
    _, d = run(False, True)
    hb, db = run(True, True)
    gbs = lambda ms: nbytes / (ms * 1e-3) / 1e9 if ms > 0 else None
    return {"h2d_gbs": gbs(h), "d2h_gbs": gbs(d), "h2d_gbs_duplex": gbs(hb), "d2h_gbs_duplex": gbs(db)}


def e2e(sas, prob, g, backward, work, dev, a, ws):
    """Same step through the public API with host buffers: every step copies all its inputs
    in from pinned host memory, runs, and copies every result back. The three stages run on
    their own streams over two buffer sets, so the copies of one step overlap the compute of
    its neighbours (a serving / training pipeline); the time is device-measured from the first
    timed input copy to the last timed result copy."""
    names = ["q_nope", "k_nope", "q", "k", "v", "wq", "wk", "qnorm_w", "knorm_w"] + \
        (["dout"] if backward else [])
    outs = ["_o", "_alse"] + (["_dq", "_dk", "_dv", "_dlogg"] if backward else [])
    host = {k: g[k].cpu().pin_memory() for k in names}
    sets = []
    for b in range(2):   # device buffers: inputs and results per set; intermediates shared
        dg = dict(g)
        for k in names + outs:
            dg[k] = torch.empty_like(g[k])
        sets.append((dg, [torch.empty(dg[k].shape, dtype=dg[k].dtype, pin_memory=True)
                          for k in outs]))
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    # the window carries one pipeline fill (the first step's input copy) and one drain (the last
    # result copy); 16 timed steps spread them, and the steady-state period is reported beside
    warm = 2
    steps = max(4, min(2 * a.steps, 16))
    total = warm + steps
    ev = lambda: torch.cuda.Event(enable_timing=True)
    in_done, comp_done, out_done = [ev() for _ in range(total)], [ev() for _ in range(total)], \
        [ev() for _ in range(total)]
    start = ev()
    torch.cuda.synchronize()
    for i in range(total):
        dg, hres = sets[i % 2]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(comp_done[i - 2])      # set's inputs no longer read
            if i == warm:
                start.record(s_in)
            for k in names:
                dg[k].copy_(host[k], non_blocking=True)
            in_done[i].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(in_done[i])
            if i >= 2:
                s_comp.wait_event(out_done[i - 2])     # set's results copied out
            train_step(sas, prob, dg, backward)
            comp_done[i].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[i])
            for hdst, k in zip(hres, outs):
                hdst.copy_(dg[k], non_blocking=True)
            out_done[i].record(s_out)
    torch.cuda.synchronize()
    ms = start.elapsed_time(out_done[total - 1]) / steps
    ms = max_over_ranks(ms, ws, dev)
    period = out_done[warm].elapsed_time(out_done[total - 1]) / (steps - 1)   # result to result
    period = max_over_ranks(period, ws, dev)
    h2d = sum(host[k].numel() * host[k].element_size() for k in names)
    d2h = sum(h.numel() * h.element_size() for h in sets[0][1])
    del sets, host
    torch.cuda.empty_cache()
    link = link_probe(dev)
    # the step time the host link alone allows (inputs in and results out at the same time)
    bound = max(h2d / (link["h2d_gbs_duplex"] * 1e9), d2h / (link["d2h_gbs_duplex"] * 1e9)) * 1e3
    return {"value": work * ws / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipelined": "two buffer sets; H2D, step and D2H on separate streams",
            "timed_steps": steps, "steady_ms_per_step": period,
            "link": link, "link_bound_ms": bound}


def reference_arm(a, ws, rank):
    """The oracle, as it stands, on the machine's host cores (rank 0 only). Each step is a
    bounded sample: random query rows of the workload's shortest sequence at full length
    (rows of different sequences are independent), drawn with the same generator."""
    if rank != 0:
        return
    shape = si.workload(a.workload)
    backward = "train" in a.workload or "varlen" in a.workload
    b = int(np.argmin(shape.lengths))
    one = si.sequence_shape(shape, b)
    inp = si.prefill_inputs(shape, device="cpu", with_dout=backward, sequence=b)
    cpu = {k: v.float().numpy().astype(np.float64) for k, v in inp.items() if k != "cu_seqlens"}
    for i in range(a.warmup):
        oracle_sample(cpu, one, sample_rows(one, 1, 100 + i), backward)
    t = []
    fl = 0.0
    for i in range(a.steps):
        rows = sample_rows(one, 8, 1000 + i)
        t0 = time.perf_counter()
        fl += oracle_sample(cpu, one, rows, backward)
        t.append(time.perf_counter() - t0)
    tot = sum(t)
    val = fl / tot / 1e12
    threads = torch.get_num_threads()
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": ws,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * tot / a.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded counter-based generator, approx. N(0,1))",
            "config": {"workload": a.workload, "batch": shape.batch, "seq_len": shape.max_seqlen,
                       "passes": "fwd+bwd" if backward else "fwd", "parallelism": "cpu oracle"},
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": f"8 random query rows per step of sequence {b} "
                                       f"({shape.lengths[b]} tokens) of {a.workload} (gate, "
                                       "Top-K, attention fwd" +
                                       (" + dQ/dlogg rows" if backward else "") +
                                       ") at full sequence length, fp64 numpy"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
