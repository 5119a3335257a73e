#!/usr/bin/env python3
"""Benchmark of NOSA sparse decode attention on B200 (one JSON line on rank 0).

A *step* is one whole decode step of one layer over the batch: append the new
token's K/V rows and pool the window it completes (nosa_pool_append), score
the compressed keys and select the top-k blocks (nosa_block_select), attend
over the selected blocks plus the local window (nosa_sparse_decode).  One
*query* is one sequence's decode token through one layer's attention.

Default workload (the NOSA-1B attention shape, 16 q / 2 KV heads, head_dim
128): batch 8, context 16384, top-k 64 blocks of 64 + 16 local blocks,
bf16 N(0,1) KV cache.  Inputs stay resident in HBM; to keep the 126 MB L2
from serving them, steps rotate over R independent replicas of the caches
(R x 142 MB).  The timed steps run as one CUDA graph, bracketed by events on
the launching stream; events inside the graph give each kernel's duration.

Also reported: ``e2e`` (the same metric through nosa_decode_step with pinned
host buffers, H2D/D2H copies inside the timed region), ``roofline`` of the
dominant kernel against the measured HBM copy bandwidth, the CPU oracle timed
on the host cores (``cpu_baseline``), and SM clocks sampled during the run.

``--impl reference`` times the CPU oracle on the same workload instead.
Multi-GPU (torchrun): every rank runs its own batch (weak scaling, no
collective on the data path); time = max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from long_context_decode_nosa_b200 import inputs, multirank  # noqa: E402

METRIC = "sparse decode-attn queries/s and achieved HBM GB/s vs ~8 TB/s, 16K–64K ctx"
UNIT = "queries/s"
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0

WORKLOADS = {
    # name: (description, batch, lengths spec, Hq, Hkv, topk, layers, key dist)
    "nosa1b_b8_16k": ("NOSA-1B attention (16 q / 2 KV heads, d128), batch 8, context 16384, "
                      "top-k 64 blocks + 16 local blocks, bf16 N(0,1) KV",
                      8, 16384, 16, 2, 64, 1, "normal"),
    "nosa1b_b32_ragged_28l": ("NOSA-1B attention, batch 32, ragged context U[16384, 32768], "
                              "top-k 64 + 16 local, 28 independent layers per step",
                              32, "ragged", 16, 2, 64, 28, "normal"),
    "llama8b_b4_64k": ("8B-class attention (32 q / 8 KV heads, d128), batch 4, context 65536, "
                       "top-k 64 + 16 local, Student-t(4) keys",
                       4, 65536, 32, 8, 64, 1, "student_t"),
}


def parse():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="nosa1b_b8_16k")
    ap.add_argument("--context", type=int, default=0, help="override the context length")
    ap.add_argument("--batch", type=int, default=0, help="override the batch size")
    ap.add_argument("--topk", type=int, default=0, help="override top-k blocks")
    ap.add_argument("--layers", type=int, default=0, help="override the number of layers of a step")
    ap.add_argument("--replicas", type=int, default=0, help="cache replicas rotated (0: auto)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU-baseline time budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--settle-ms", type=float, default=300.0,
                    help="untimed repeated steps before timing, so clocks settle")
    ap.add_argument("--pooled", choices=["fp32", "bf16"], default="fp32",
                    help="pooled-key precision (bf16: the half-size variant)")
    ap.add_argument("--paged", action="store_true",
                    help="caches as shuffled 64-token pages through a page table (the paged entry points)")
    ap.add_argument("--kv", choices=["bf16", "int8"], default="bf16",
                    help="K/V cache format (int8: codes + per-row scales, the 8-bit decode variant)")
    ap.add_argument("--prefill", action="store_true",
                    help="sparse prefill (NOSAS) of --batch sequences of --context tokens in --chunk-row chunks")
    ap.add_argument("--chunk", type=int, default=4096, help="prefill chunk rows per sequence")
    ap.add_argument("--sweep", action="store_true",
                    help="NOSA-1B shape over context x batch x top-k (one JSON line per point)")
    return ap.parse_args()


# ----------------------------------------------------------------------------- workload

def _n_windows(L: int) -> int:
    return (L - 32) // 16 + 1 if L >= 32 else 0


class Workload:
    def __init__(self, args, seed_base: int):
        desc, batch, lens, hq, hkv, topk, layers, kdist = WORKLOADS[args.workload]
        self.name = args.workload
        self.batch = args.batch or batch
        if args.context:
            lens = args.context
        if lens == "ragged":
            self.lens = inputs.ragged_lengths(self.batch, 16384, 32768, seed=seed_base + 3)
        else:
            self.lens = [int(lens)] * self.batch
        self.hq, self.hkv = hq, hkv
        self.topk = args.topk or topk
        self.layers = getattr(args, "layers", 0) or layers
        self.key_dist = kdist
        self.local_blocks = 16
        self.pooled_bf16 = getattr(args, "pooled", "fp32") == "bf16"
        self.kv_int8 = getattr(args, "kv", "bf16") == "int8"
        self.paged = bool(getattr(args, "paged", False))
        self.desc = desc + (", bf16 pooled keys" if self.pooled_bf16 else "") + (
            ", INT8 K/V cache" if self.kv_int8 else "") + (", paged cache (shuffled 64-token pages)" if self.paged else "")
        if args.context or args.batch or args.topk or getattr(args, "layers", 0):
            self.desc += (f" [overridden: batch {self.batch}, context {max(self.lens)}, top-k {self.topk}, "
                          f"layers {self.layers}]")
        self.max_len = max(self.lens)

    # Algorithmic bytes per kernel for one layer-step (see the byte model in the design notes).
    def bytes_model(self):
        G = self.hq // self.hkv
        pool = select = decode = 0
        for L in self.lens:
            nb = -(-L // 64)
            ncand = max(0, nb - self.local_blocks)
            nc = _n_windows(L)
            k_eff = min(self.topk, ncand)
            windows = min(nc, 4 * ncand)
            attended = k_eff * 64 + (L - 64 * ncand)
            new_window = _n_windows(L) - _n_windows(L - 1)
            pk = 256 if self.pooled_bf16 else 512                     # bytes per pooled key
            row = 132 if self.kv_int8 else 256                        # bytes per cached K (or V) row
            for _ in range(self.hkv):
                pool += 2 * 256 + 2 * row + new_window * (31 * row + pk)  # new K/V row in + out, window
                select += windows * pk + G * 256 + self.topk * 4 + 4
                decode += attended * 2 * row + 2 * G * 256 + self.topk * 4 + 4
        return {"pool_append": pool * self.layers, "block_select": select * self.layers,
                "sparse_decode": decode * self.layers}


def replica_plan(wl: Workload, args):
    """(replicas R, bytes of one layer's K/V caches): R independent copies of
    the caches are rotated so that no step finds its inputs in L2 (126 MB);
    a multi-layer workload has its own caches per layer instead."""
    layer_bytes = sum(wl.lens) * wl.hkv * (132 if wl.kv_int8 else 256) * 2
    if wl.layers > 1:
        return 1, layer_bytes
    return args.replicas or max(2, min(16, math.ceil(1.0e9 / max(layer_bytes, 1)))), layer_bytes


def run_config(wl: Workload, args, world: int):
    """The `config` object of the JSON line (the same for both arms)."""
    R, layer_bytes = replica_plan(wl, args)
    return {"workload": wl.desc, "batch": wl.batch, "seq_len": wl.max_len,
            "topk": wl.topk, "local_blocks": wl.local_blocks, "layers": wl.layers,
            "parallelism": f"dp{world}" if world > 1 else "single GPU",
            "l2": (f"inputs rotate over {R} cache replicas "
                   f"({R * layer_bytes * wl.layers / 1e9:.2f} GB) > 126 MB L2"),
            "clock_settle_ms": args.settle_ms,
            "graph": "timed steps (one fused launch per layer-step) replayed as one CUDA graph"}


class Replica:
    """One layer's device state: caches, pooled keys, selection, output."""

    def __init__(self, nosa, wl: Workload, seed: int, device):
        self.b = inputs.make_batch(wl.lens, num_q_heads=wl.hq, num_kv_heads=wl.hkv, seed=seed,
                                   key_dist=wl.key_dist, device=device)
        self.p = nosa.params(wl.hq, wl.hkv, topk=wl.topk, local_blocks=wl.local_blocks, pooled_bf16=wl.pooled_bf16,
                             kv_int8=wl.kv_int8)
        self.page_table = None
        k_bf, v_bf = self.b.k_cache, self.b.v_cache
        if wl.paged:     # the same tokens in randomly permuted 64-token pages (built untimed)
            cap = self.b.capacity.cpu().tolist()
            starts = self.b.seq_start.cpu().tolist()
            need = [(c + 63) // 64 for c in cap]
            perm = torch.randperm(sum(need), generator=torch.Generator().manual_seed(seed + 11))
            table = torch.full((wl.batch, max(need)), -1, dtype=torch.int32)
            src, dst, n = [], [], 0
            for i in range(wl.batch):
                for pg in range(need[i]):
                    table[i, pg] = perm[n]
                    n += 1
                    t = torch.arange(pg * 64, min(pg * 64 + 64, cap[i]))
                    src.append(starts[i] + t)
                    dst.append(int(table[i, pg]) * 64 + t - pg * 64)
            src = torch.cat(src).to(device)
            dst = torch.cat(dst).to(device)
            k_bf = torch.zeros(sum(need) * 64, wl.hkv, 128, dtype=torch.bfloat16, device=device)
            v_bf = torch.zeros_like(k_bf)
            k_bf[dst] = self.b.k_cache[src]
            v_bf[dst] = self.b.v_cache[src]
            self.page_table = table.to(device)
        if wl.kv_int8:   # the caches as the INT8 variant stores them (quantized on the GPU, untimed)
            self.k_cache = nosa.Int8KvCache.from_bf16(self.p, k_bf)
            self.v_cache = nosa.Int8KvCache.from_bf16(self.p, v_bf)
        else:
            self.k_cache, self.v_cache = k_bf, v_bf
        self.st = nosa.DecodeState(self.p, wl.batch, wl.max_len, device=device)
        if wl.paged:
            nosa.nosa_pool_append_paged(self.p, self.k_cache, None, self.page_table, self.b.seq_len, self.st.pooled,
                                        len_old=torch.zeros_like(self.b.seq_len), max_new_keys=self.st.nc_cap,
                                        ws=self.st.ws)
        else:
            self.st.rebuild_pooled(self.k_cache, self.b.seq_start, self.b.seq_len)
        self.k_new, self.v_new = inputs.random_kv_rows(wl.batch, wl.hkv, 128, seed=seed + 7,
                                                       device=device)


def step(nosa, r: Replica, events=None, fused=True):
    """One decode step on device-resident inputs: append the new token's K/V
    rows, pool the window it completes, select, attend.  ``fused``: one launch
    (nosa_decode_step_device); otherwise the three entry points in order, with
    ``events`` (4 CUDA events) recorded before each kernel and after the last."""
    b, st, p = r.b, r.st, r.p
    if r.page_table is not None:
        if fused:
            nosa.nosa_decode_step_device_paged(p, b.q, r.k_cache, r.v_cache, r.page_table, b.seq_len,
                                               st.max_seq_len, st.pooled, st.sel_idx, st.sel_cnt, st.out, st.ws,
                                               k_new=r.k_new, v_new=r.v_new)
            return
        if events:
            events[0].record()
        nosa.nosa_pool_append_paged(p, r.k_cache, r.v_cache, r.page_table, b.seq_len, st.pooled, max_new_keys=1,
                                    k_new=r.k_new, v_new=r.v_new, ws=st.ws)
        if events:
            events[1].record()
        nosa.nosa_block_select(p, b.q, st.pooled, b.seq_len, st.max_seq_len, st.sel_idx, st.sel_cnt, st.ws)
        if events:
            events[2].record()
        nosa.nosa_sparse_decode_paged(p, b.q, r.k_cache, r.v_cache, r.page_table, b.seq_len, st.max_seq_len,
                                      st.sel_idx, st.sel_cnt, st.out, st.ws)
        if events:
            events[3].record()
        return
    if fused:
        nosa.nosa_decode_step_device(p, b.q, r.k_cache, r.v_cache, b.seq_start, b.seq_len, st.max_seq_len,
                                     st.pooled, st.sel_idx, st.sel_cnt, st.out, st.ws, k_new=r.k_new,
                                     v_new=r.v_new)
        return
    if events:
        events[0].record()
    nosa.nosa_pool_append(p, r.k_cache, r.v_cache, b.seq_start, b.seq_len, st.pooled, max_new_keys=1,
                          k_new=r.k_new, v_new=r.v_new, ws=st.ws)
    if events:
        events[1].record()
    nosa.nosa_block_select(p, b.q, st.pooled, b.seq_len, st.max_seq_len, st.sel_idx, st.sel_cnt,
                           st.ws)
    if events:
        events[2].record()
    nosa.nosa_sparse_decode(p, b.q, r.k_cache, r.v_cache, b.seq_start, b.seq_len, st.max_seq_len,
                            st.sel_idx, st.sel_cnt, st.out, st.ws)
    if events:
        events[3].record()


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [ln.split(",") for ln in out.strip().splitlines() if ln.count(",") >= 8]
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(rows)}


# ----------------------------------------------------------------------------- helpers

def peak_hbm():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def peak_bf16():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS, "fallback"


_COMMENT_OR_STRING = re.compile(r'//[^\n]*|/\*.*?\*/|"(?:\\.|[^"\\])*"', re.S)


def _code_only(text: str) -> str:
    """C/CUDA source without comments, whitespace runs collapsed (string
    literals kept as they are)."""
    text = _COMMENT_OR_STRING.sub(lambda m: m.group(0) if m.group(0).startswith('"') else " ", text)
    return " ".join(text.split())


def kernel_source_hash():
    """SHA-256 (16 hex digits) of the kernel sources with comments and
    whitespace removed: a comment edit leaves the compiled kernels, and so
    their ncu counters, unchanged."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "long_context_decode_nosa_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(csrc, name), encoding="utf-8") as f:
                h.update(name.encode() + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str):
    """Per-launch DRAM bytes of the fused step kernel from the committed ncu
    summary (profiles/), if it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", f"step_kernel_{workload}.md")
    try:
        with open(path) as f:
            txt = f.read()
    except OSError:
        return None
    src = traffic = None
    for ln in txt.splitlines():
        if ln.startswith("kernel_source_sha256_16:"):
            src = ln.split(":", 1)[1].strip()
        if ln.startswith("dram_bytes_per_launch:"):
            try:
                traffic = float(ln.split(":", 1)[1].strip())
            except ValueError:
                traffic = None
    return traffic if src == kernel_source_hash() else None


def dist_setup(args):
    info = multirank.rank_info()
    multirank.init(info, backend="nccl", timeout_s=120)
    return info


# ----------------------------------------------------------------------------- CPU oracle

def oracle_steps(wl: Workload, b_host, n_steps: int, threads: int, budget_s: float):
    """Time whole oracle decode steps (pool the new window, score, select,
    attend) on host copies of one layer's inputs; stops after n_steps or the
    time budget.  Returns (steps done, seconds)."""
    import oracle
    oracle.set_threads(threads)
    kb = inputs.bf16_bits(b_host.k_cache)
    vb = inputs.bf16_bits(b_host.v_cache)
    qb = inputs.bf16_bits(b_host.q)
    lens = b_host.seq_len.numpy()
    starts = b_host.seq_start.numpy()
    nc_cap = max(1, oracle.n_windows(int(lens.max())))
    if wl.kv_int8:   # the INT8 variant: the oracle's own quantized caches (untimed)
        kc, ks = oracle.quantize_int8(kb)
        vc, vs = oracle.quantize_int8(vb)
        pooled = oracle.pool_int8(kc, ks, starts, lens - 1, nc_cap, bf16=wl.pooled_bf16)
    else:
        pooled = oracle.pool(kb, starts, lens - 1, nc_cap, bf16=wl.pooled_bf16)   # state before the step (untimed)
    nb_cap = oracle.n_blocks(int(lens.max()))
    done, t0 = 0, time.perf_counter()
    while done < n_steps:
        if wl.kv_int8:
            pooled = oracle.pool_int8(kc, ks, starts, lens, nc_cap, len_old=lens - 1, pooled=pooled,
                                      bf16=wl.pooled_bf16)
            sc = oracle.comp_scores(qb, pooled, lens, num_kv_heads=wl.hkv)
            S = oracle.block_scores(sc, lens, nb_cap, num_kv_heads=wl.hkv, local_blocks=wl.local_blocks)
            idx, cnt = oracle.topk(S, lens, wl.topk, local_blocks=wl.local_blocks)
            oracle.sparse_attention_int8(qb, kc, ks, vc, vs, starts, lens, idx, cnt, local_blocks=wl.local_blocks)
        else:
            pooled = oracle.pool(kb, starts, lens, nc_cap, len_old=lens - 1, pooled=pooled, bf16=wl.pooled_bf16)
            oracle.decode_step(qb, kb, vb, starts, lens, pooled, wl.topk, local_blocks=wl.local_blocks)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    return done, time.perf_counter() - t0


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_batch(wl: Workload, seed: int):
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    return inputs.make_batch(wl.lens, num_q_heads=wl.hq, num_kv_heads=wl.hkv, seed=seed,
                             key_dist=wl.key_dist, device=dev).to("cpu")


def run_reference(args):
    world, rank, _ = int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0
    if rank != 0:
        return 0
    wl = Workload(args, 0)
    b = host_batch(wl, seed=100)
    threads = os.cpu_count() or 1
    oracle_steps(wl, b, max(1, min(args.warmup, 1)), threads, 1e9)       # warm caches
    per_layer_steps, secs = oracle_steps(wl, b, args.steps, threads, 1e9)
    # one step = all layers of the workload; the oracle runs one layer and scales
    ms = secs / per_layer_steps * wl.layers * 1e3
    value = wl.batch * wl.layers / (ms / 1e3)
    sample = (f"{per_layer_steps} full one-layer steps of the workload on the oracle"
              + (f", scaled x{wl.layers} layers" if wl.layers > 1 else ""))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": run_config(wl, args, int(os.environ.get("WORLD_SIZE", "1"))),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- ours

def run_ours(args):
    info = dist_setup(args)
    world, rank, local = info.world, info.rank, info.local_rank
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    from long_context_decode_nosa_b200 import nosa
    nosa.lib()
    wl = Workload(args, 0)
    seed0 = multirank.rank_seed(0, info)

    # Replicas so that no step finds its inputs in L2 (126 MB).
    R, layer_bytes = replica_plan(wl, args)
    if wl.layers > 1:
        rotation = [[Replica(nosa, wl, seed0 + 10 * l, device) for l in range(wl.layers)]]
    else:
        rotation = [[Replica(nosa, wl, seed0 + 10 * r, device)] for r in range(R)]
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device)
    stream.wait_stream(torch.cuda.current_stream())

    def record_steps(n, fused=True, with_events=False):
        evs = []
        for s_ in range(n):
            for layer in rotation[s_ % len(rotation)]:
                e = ([torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]
                     if with_events else None)
                step(nosa, layer, e, fused=fused)
                if e:
                    evs.append(e)
        return evs

    with torch.cuda.stream(stream):
        record_steps(len(rotation))                       # eager warm-up: kernel attributes
        record_steps(len(rotation), fused=False)
    stream.synchronize()

    g_warm = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_warm, stream=stream):
        record_steps(max(args.warmup, 1))
    g_timed = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_timed, stream=stream):
        record_steps(args.steps)
    n_split = max(len(rotation), min(args.steps, 200))
    g_split = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_split, stream=stream):
        inner = record_steps(n_split, fused=False, with_events=True)

    clocks = ClockSampler(device.index if device.index is not None else 0)
    clocks.start()
    with torch.cuda.stream(stream):
        g_warm.replay()
        t_settle = time.perf_counter()
        while (time.perf_counter() - t_settle) * 1e3 < args.settle_ms:
            g_warm.replay()
            stream.synchronize()
        multirank.barrier(info)
        stream.synchronize()
        start = torch.cuda.Event(enable_timing=True)
        stop = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        g_timed.replay()
        stop.record(stream)
    stream.synchronize()
    clk = clocks.stop()
    ms_total = multirank.max_over_ranks(start.elapsed_time(stop), info, device)
    ms_step = ms_total / args.steps
    # Kernel split of the unfused path (separate launches with events between
    # them, which also stops their launches overlapping): context only.
    with torch.cuda.stream(stream):
        g_split.replay()
    stream.synchronize()
    kt = {"pool_append": [], "block_select": [], "sparse_decode": []}
    for e in inner:
        kt["pool_append"].append(e[0].elapsed_time(e[1]))
        kt["block_select"].append(e[1].elapsed_time(e[2]))
        kt["sparse_decode"].append(e[2].elapsed_time(e[3]))
    kmean_us = {k: 1e3 * statistics.fmean(v) for k, v in kt.items()}
    unfused_ms_step = sum(kmean_us.values()) * wl.layers / 1e3

    queries_per_step = wl.batch * wl.layers
    value = multirank.aggregate_rate(queries_per_step * args.steps, info, ms_total / 1e3)
    model = wl.bytes_model()
    step_bytes = sum(model.values())
    peak, peak_kind = peak_hbm()
    # The fused step kernel is the only kernel of a step: its average launch
    # duration is the timed region over the launches (gaps included).
    launch_s = ms_total / 1e3 / (args.steps * wl.layers)
    fused_bytes_launch = step_bytes / wl.layers
    achieved = fused_bytes_launch / launch_s / 1e9
    traffic = None
    # The committed counters cover the default variant of each named workload.
    if not (args.context or args.batch or args.topk or args.layers or wl.paged or wl.kv_int8 or wl.pooled_bf16):
        traffic = ncu_traffic(wl.name)

    # e2e through the host-buffer entry point, rotating over the same replicas, pinned buffers.
    e2e = None
    if not args.no_e2e and not wl.paged:   # the host-buffer call takes contiguous caches
        e2e = measure_e2e(nosa, wl, rotation, args, stream, info, device)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        b_host = inputs.DecodeBatch(rotation[0][0].b.q.cpu(), rotation[0][0].b.k_cache.cpu(),
                                    rotation[0][0].b.v_cache.cpu(), rotation[0][0].b.seq_start.cpu(),
                                    rotation[0][0].b.seq_len.cpu(), rotation[0][0].b.capacity.cpu(),
                                    wl.hq, wl.hkv, 128)
        threads = os.cpu_count() or 1
        n, secs = oracle_steps(wl, b_host, 10 ** 6, threads, args.cpu_seconds)
        cpu_ms = secs / n * wl.layers * 1e3
        n1, secs1 = oracle_steps(wl, b_host, 10 ** 6, 1, min(3.0, args.cpu_seconds))
        cpu = {"value": queries_per_step / (cpu_ms / 1e3), "unit": UNIT, "cores": threads,
               "kind": "oracle",
               "sample": f"{n} one-layer decode steps of this workload (all {wl.batch} sequences) on the "
                         f"fp64 C oracle in {secs:.1f} s" + (f", scaled x{wl.layers} layers" if wl.layers > 1 else ""),
               "value_single_thread": queries_per_step / (secs1 / n1 * wl.layers),
               "cpu_model": cpu_model()}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8+bf16" if wl.kv_int8 else "bf16", "data": "synthetic",
            "config": run_config(wl, args, world),
            "gpu_launches": args.steps * wl.layers,
            "hbm_gbs_step": step_bytes / (ms_step * 1e-3) / 1e9,
            "algorithmic_bytes_per_step": step_bytes,
            "kernel_us_unfused": kmean_us,
            "ms_per_step_unfused": unfused_ms_step,
            "roofline": {"bound": "hbm", "kernel": "step_kernel (fused pool + select + sparse decode)",
                         "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                         "peak_kind": f"{peak_kind} copy bandwidth", "traffic": traffic,
                         "algorithmic_bytes_per_launch": fused_bytes_launch,
                         "launch_us": launch_s * 1e6},
            "cpu_baseline": cpu, "e2e": e2e, "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    del g_timed, g_warm, g_split
    multirank.shutdown(info)
    return 0


def measure_e2e(nosa, wl: Workload, rotation, args, stream, info, device):
    """Same metric through the host-buffer entry point (nosa_decode_step_packed)
    with pinned host buffers: every layer-step copies q and the new K/V rows in
    (one packed buffer, one copy) and the output back.  Steps rotate over the
    same cache replicas as the device-timed region (each layer and replica with
    its own pinned buffers), so the kernels inside run L2-cold as well."""
    calls = []
    for layers in rotation:
        row = []
        for r in layers:
            b, st, p = r.b, r.st, r.p
            packed = torch.cat([b.q.reshape(-1), r.k_new.reshape(-1), r.v_new.reshape(-1)]).cpu().pin_memory()
            o_h = torch.empty(wl.batch, wl.hq, 128, dtype=torch.bfloat16).pin_memory()
            row.append((r, packed, o_h))
        calls.append(row)
    n = max(len(calls), min(args.steps, 500))

    def step_e2e(s_):
        for r, packed, o_h in calls[s_ % len(calls)]:
            b, st, p = r.b, r.st, r.p
            nosa.nosa_decode_step_packed(p, packed, o_h, r.k_cache, r.v_cache, b.seq_start, b.seq_len,
                                         st.max_seq_len, st.pooled, st.sel_idx, st.sel_cnt, st.ws, stream=stream)

    with torch.cuda.stream(stream):
        for s_ in range(max(3, min(args.warmup, 50))):
            step_e2e(s_)
        stream.synchronize()
        multirank.barrier(info)
        start = torch.cuda.Event(enable_timing=True)
        stop = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for s_ in range(n):
            step_e2e(s_)
        stop.record(stream)
    stream.synchronize()
    ms = multirank.max_over_ranks(start.elapsed_time(stop), info, device)
    packed0, out0 = calls[0][0][1], calls[0][0][2]
    return {"value": multirank.aggregate_rate(wl.batch * wl.layers * n, info, ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": packed0.numel() * 2 * wl.layers,
            "d2h_bytes_per_step": out0.numel() * 2 * wl.layers, "steps": n, "ms_per_step": ms / n,
            "replicas": len(calls),
            "api": "nosa_decode_step_packed (one host-to-device and one device-to-host copy per layer-step)"}


# ----------------------------------------------------------------------------- sweep

SWEEP_CONTEXTS = (4096, 8192, 16384, 32768, 65536, 131072)
SWEEP_BATCHES = (1, 8, 32, 64)
SWEEP_TOPK = (32, 64, 96)          # 2048 / 4096 / 6144 selected tokens
SWEEP_MEMORY_BYTES = 60e9          # points whose replicas would exceed this are skipped


def run_sweep(args):
    """The NOSA-1B attention shape over context x batch x top-k, one GPU.
    Per point: fused steps captured as one CUDA graph over cache replicas
    larger than L2 (CUDA events on the launching stream), and the three
    standalone launches with events between them for the pool / select /
    decode split.  One JSON line per point."""
    from long_context_decode_nosa_b200 import nosa
    nosa.lib()
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    peak, peak_kind = peak_hbm()
    stream = torch.cuda.Stream(device)
    for L in SWEEP_CONTEXTS:
        for B in SWEEP_BATCHES:
            for K in SWEEP_TOPK:
                a = argparse.Namespace(workload="nosa1b_b8_16k", context=L, batch=B, topk=K, pooled=args.pooled,
                                       kv=args.kv, paged=args.paged)
                wl = Workload(a, 0)
                layer_bytes = B * L * wl.hkv * 128 * 2 * 2
                R = max(2, min(16, math.ceil(1.0e9 / layer_bytes)))
                point = {"context": L, "batch": B, "topk": K, "replicas": R}
                if R * layer_bytes * 1.5 > SWEEP_MEMORY_BYTES:
                    point["skipped"] = f"{R} replicas of {layer_bytes / 1e9:.1f} GB exceed the sweep's memory budget"
                    print(json.dumps({"sweep_point": point}), flush=True)
                    continue
                reps = [Replica(nosa, wl, 1000 + 10 * r, device) for r in range(R)]
                torch.cuda.synchronize()
                steps = 100
                with torch.cuda.stream(stream):
                    for r in reps:
                        step(nosa, r)
                        step(nosa, r, fused=False)
                stream.synchronize()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    for n in range(steps):
                        step(nosa, reps[n % R])
                evs = []
                g_split = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g_split, stream=stream):
                    for n in range(max(R, 20)):
                        e = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]
                        step(nosa, reps[n % R], e, fused=False)
                        evs.append(e)
                with torch.cuda.stream(stream):
                    for _ in range(3):
                        g.replay()
                    stream.synchronize()
                    start = torch.cuda.Event(enable_timing=True)
                    stop = torch.cuda.Event(enable_timing=True)
                    start.record(stream)
                    g.replay()
                    stop.record(stream)
                    g_split.replay()
                stream.synchronize()
                us = start.elapsed_time(stop) * 1e3 / steps
                split = {k: 1e3 * statistics.fmean(e[j].elapsed_time(e[j + 1]) for e in evs)
                         for j, k in enumerate(("pool_append", "block_select", "sparse_decode"))}
                step_bytes = sum(wl.bytes_model().values())
                gbs = step_bytes / (us * 1e-6) / 1e9
                point.update({"us_per_step": us, "queries_per_s": B / (us * 1e-6), "gb_per_s": gbs,
                              "frac_of_peak": gbs / peak, "peak_kind": peak_kind,
                              "algorithmic_bytes_per_step": step_bytes, "unfused_us": split})
                print(json.dumps({"sweep_point": point}), flush=True)
                del g, g_split, reps
                torch.cuda.empty_cache()
    return 0


def run_prefill(args):
    """Sparse prefill (NOSAS): NOSA-1B attention shape, --batch sequences of
    --context tokens, prefilled in chunks of --chunk rows; one prefill = per
    chunk, the pool-append of the chunk's windows and one nosa_sparse_prefill
    launch (every row a decode query of its own prefix).  K whole prefills
    captured as one CUDA graph, CUDA events on the launching stream."""
    from long_context_decode_nosa_b200 import nosa
    nosa.lib()
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    B = args.batch or 1
    T = args.context or 16384
    chunk = min(args.chunk, T)
    topk = args.topk or 64
    kv_int8 = args.kv == "int8"
    p = nosa.params(16, 2, topk=topk, pooled_bf16=args.pooled == "bf16", kv_int8=kv_int8)
    b = inputs.make_batch([T] * B, num_q_heads=16, num_kv_heads=2, seed=200, device=device)
    kc, vc = b.k_cache, b.v_cache
    if kv_int8:
        kc, vc = nosa.Int8KvCache.from_bf16(p, kc), nosa.Int8KvCache.from_bf16(p, vc)
    gen = torch.Generator(device=device).manual_seed(201)
    q_all = torch.randn(B, T, 16, 128, generator=gen, device=device).to(torch.bfloat16)
    nc_cap = max(1, nosa.n_windows(T))
    pooled = torch.zeros(B, 2, nc_cap, 128, dtype=p.pooled_dtype, device=device)
    ws_pool = nosa.workspace(p, B, T)
    chunks = []
    for c0 in range(0, T, chunk):
        c1 = min(T, c0 + chunk)
        n = c1 - c0
        chunks.append(dict(
            q=q_all[:, c0:c1].reshape(B * n, 16, 128).contiguous(),
            q_start=torch.arange(0, B * n + 1, n, dtype=torch.int32, device=device),
            q_pos=torch.full((B,), c0, dtype=torch.int32, device=device),
            len_old=torch.full((B,), c0, dtype=torch.int32, device=device),
            len_new=torch.full((B,), c1, dtype=torch.int32, device=device),
            sel=torch.empty(B * n, 2, topk, dtype=torch.int32, device=device),
            cnt=torch.empty(B * n, 2, dtype=torch.int32, device=device),
            out=torch.empty(B * n, 16, 128, dtype=torch.bfloat16, device=device),
            ws=nosa.prefill_workspace(p, B * n, T), n=n))

    def prefill():
        for c in chunks:
            nosa.nosa_pool_append(p, kc, None, b.seq_start, c["len_new"], pooled, len_old=c["len_old"],
                                  max_new_keys=c["n"] // 16 + 2, ws=ws_pool)
            nosa.nosa_sparse_prefill(p, c["q"], kc, vc, b.seq_start, c["q_start"], c["q_pos"], T, pooled,
                                     c["sel"], c["cnt"], c["out"], c["ws"])

    stream = torch.cuda.Stream(device)
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        prefill()
    stream.synchronize()
    for c in chunks:
        rc, bits = nosa.nosa_read_device_status(c["ws"])
        if rc:
            raise SystemExit(f"sparse prefill reported device status 0x{bits:x}")
    K = max(1, min(args.steps, 20))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(K):
            prefill()
    clocks = ClockSampler(0)
    clocks.start()
    with torch.cuda.stream(stream):
        g.replay()
        stream.synchronize()
        start = torch.cuda.Event(enable_timing=True)
        stop = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        g.replay()
        stop.record(stream)
    stream.synchronize()
    clk = clocks.stop()
    ms = start.elapsed_time(stop) / K
    tokens = B * T
    # Useful attention flops: every token's attended keys (its selected blocks
    # and local window) x heads x (QK + PV) x 2.
    keys = 0
    for t in range(T):
        L = t + 1
        nb = -(-L // 64)
        ncand = max(0, nb - 16)
        keys += min(topk, ncand) * 64 + (L - 64 * ncand)
    flops = 4.0 * 128 * 16 * keys * B
    peak, peak_kind = peak_bf16()
    achieved = flops / (ms / 1e3) / 1e12
    # The oracle on a bounded sample: rows of the last chunk of sequence 0.
    import oracle
    nrows = 24
    kb = inputs.bf16_bits(b.k_cache[:T].cpu())
    vb = inputs.bf16_bits(b.v_cache[:T].cpu())
    qs = inputs.bf16_bits(q_all[0, T - nrows:T].cpu())
    pooled_h = oracle.pool(kb, np.array([0]), np.array([T], np.int32), nc_cap, bf16=args.pooled == "bf16")
    threads = os.cpu_count() or 1
    oracle.set_threads(threads)
    t0 = time.perf_counter()
    if kv_int8:
        cpu_rows = None
    else:
        oracle.sparse_prefill(qs, kb, vb, np.array([0]), np.array([0, nrows]), np.array([T - nrows]), pooled_h,
                              topk)
        cpu_rows = nrows
    cpu_s = time.perf_counter() - t0
    line = {"metric": "sparse prefill tokens/s (NOSAS)", "value": tokens / (ms / 1e3), "unit": "tokens/s",
            "n_gpus": 1, "steps": K, "warmup": 1, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8+bf16" if kv_int8 else "bf16", "data": "synthetic",
            "config": {"workload": f"NOSA-1B attention (16 q / 2 KV heads), {B} x {T}-token prefill in "
                                   f"{chunk}-row chunks, top-k {topk} + 16 local blocks per token",
                       "chunks": len(chunks), "pooled": args.pooled, "kv": args.kv},
            "us_per_token": ms * 1e3 / tokens,
            "roofline": {"bound": "tensor", "kernel": "whole prefill (selection + grouped attention)",
                         "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                         "peak_kind": f"{peak_kind} cuBLAS bf16", "traffic": None,
                         "useful_flops_per_prefill": flops},
            "cpu_baseline": None if cpu_rows is None else {
                "value": cpu_rows / cpu_s, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                "sample": f"the last {cpu_rows} rows of a {T}-token prefill (decode rule per row, fp64 C oracle)"},
            "gpu_launches": K * 2 * len(chunks), "clocks": clk}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (B200); the CUDA path has no CPU fallback")
    if args.sweep:
        return run_sweep(args)
    if args.prefill:
        return run_prefill(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
