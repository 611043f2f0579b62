#!/usr/bin/env python
"""Benchmark of the CSA / HCA decode hot path on B200 (one JSON line on rank 0).

Step (default workload "flash64k"): one decode token for each of B = 8 sequences
at 65,536 tokens of context, through one CSA layer and one HCA layer, as the
Flash configuration alternates them ("DeepSeek-V4 混合注意力：从压缩记忆到百万上下文"
§2 configuration table, §4-§7):
  CSA: compress the newest 4-token block (latent c=512 and index keys c=128, with
       the carry of the previous block) -> Hadamard-rotate and quantise the index
       queries (e4m3; the index keys are held rotated and quantised) ->
       e4m3 index scores over 16,384 keys -> top-1024 candidates -> exact rerank
       (bf16) to top-512 -> sparse_attn (64 heads, D=512, 512 + 128 SWA rows).
  HCA: compress the newest 128-token block (c=512) -> hca_attn over 512 summaries
       + 128 SWA rows.
Metric: decode tokens/s = B x (GPUs) / step time.  "pro1m" (the 1M-context Pro CSA
layer, B=1) is measured in the same run and reported under "pro1m".

Every step is a CUDA graph replay of the library's C-ABI calls; S input sets (caches
and per-step inputs) rotate so that the data the steps touch exceeds 2x the L2.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import platform
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

L2_BYTES = 126 * 2 ** 20
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
# e4m3 index path: queries and keys are Walsh-Hadamard-rotated before quantisation
# (the Indexer paragraph of the MXFP4 sparse-attention page); --no-hadamard turns it off.
INDEX_ROTATION = True
# partial RoPE of the attention ("DeepSeek-V4 混合注意力：从压缩记忆到百万上下文" §6; the MXFP4 page's
# compress_rope_theta): q turned and the output turned back inside the attention kernel, new
# compressed entries turned when the step appends them.  Not applied to mixed-precision KV8 rows.
ROPE_THETA = 160000.0
# How a decode step's launches are laid out: "streams" puts the compressors and the HCA
# layer on side streams beside the indexer -> select -> attention chain, forked after the
# indexer ("early": at the step's start, "late": after the select); "serial" issues every
# launch on one stream.
SCHEDULE = "streams"


def oracle_quantizer():
    """The oracle's e4m3 quantiser matching INDEX_ROTATION (CPU-baseline / reference leg)."""
    import oracle
    return oracle.quantize_rows_e4m3_hadamard if INDEX_ROTATION else oracle.quantize_rows_e4m3


# ----------------------------------------------------------------------------- distributed plumbing
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world: int, backend: str):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, world: int, device="cpu") -> float:
    """Maximum of a per-rank scalar over all ranks (identity for one rank)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------- clocks
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self, gpu_index: int, period_ms: int = 50):
        self.proc = None
        # raw samples for inspection: $CSA_BENCH_OUT_DIR if set, else the system temp folder
        out_dir = os.environ.get("CSA_BENCH_OUT_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"clocks_rank{gpu_index}.csv")
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={CLOCK_FIELDS}",
                                          "--format=csv,noheader,nounits", f"-lms={period_ms}"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def profiled_traffic(profile: str, source: str, workload: str):
    """DRAM bytes (read + write) per launch of one kernel on one workload, from the committed
    ncu summary `profiles/<profile>`, or None when the kernel's source file `csrc/<source>` has
    changed since that capture (the summary records a hash of it)."""
    import hashlib
    import re
    try:
        text = open(os.path.join(ROOT, "profiles", profile)).read()
        src = open(os.path.join(ROOT, "long_context_compressed_b200", "csrc", source), "rb").read()
    except OSError:
        return None
    m = re.search(r"^traffic_bytes_per_launch: (.*)$", text, re.M)
    if not m:
        return None
    fields = dict(kv.split("=", 1) for kv in m.group(1).split())
    if hashlib.sha256(src).hexdigest()[:16] != fields.get("source_sha256_prefix"):
        return None
    v = fields.get(workload)
    return int(v) if v is not None else None


def measured_tflops():
    """Dense bf16 tensor peak (TFLOP/s): the burst figure, for kernels timed alone."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"])
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS


# ----------------------------------------------------------------------------- the step
def _pack(tensors, device):
    """One uint8 device buffer holding copies of `tensors` at 16-byte aligned offsets,
    and typed views of it in the same order."""
    import torch
    nbytes = [t.numel() * t.element_size() for t in tensors]
    offs, total = [], 0
    for n in nbytes:
        offs.append(total)
        total += (n + 15) // 16 * 16
    buf = torch.empty(max(total, 16), dtype=torch.uint8, device=device)
    views = []
    for t, o, n in zip(tensors, offs, nbytes):
        v = buf[o:o + n].view(t.dtype).view(t.shape)
        v.copy_(t)
        views.append(v)
    return buf, views


class DecodeSet:
    """One input set of a decode workload: resident caches, per-step inputs, outputs and
    workspaces on the device, plus pinned host copies of the per-step inputs/outputs."""

    def __init__(self, wl, seed: int, index: str, with_hca: bool, device, kv8: bool = False):
        import torch

        from long_context_compressed_b200 import csa, synth
        self.wl, self.index, self.with_hca, self.kv8 = wl, index, with_hca, kv8
        B, T, N, H, D, k = wl.B, wl.T, wl.N, wl.H, wl.D, wl.topk
        dev = device
        g = lambda nm, shape: synth.store(synth.normal(seed, f"bench/{wl.name}/{nm}", shape, device=dev), "bf16")
        f32 = lambda nm, shape: synth.normal(seed, f"bench/{wl.name}/{nm}", shape, device=dev)
        # resident state (caches)
        self.kv = g("kv", (B, N, D))
        self.swa = g("swa", (B, wl.W, D))
        self.kI = g("kI", (B, N, 128))
        if index == "e4m3":
            self.k8, self.ks = csa.csa_quantize_e4m3(self.kI, hadamard=INDEX_ROTATION)
        if index == "mxfp4":
            # packed E2M1 codes of the rotated keys, scales in the tensor-core layout
            self.k4, self.ksf = csa.csa_quantize_mxfp4_sf128(self.kI, B)
        self.sink = f32("sink", (H,))
        self.q_pos = torch.full((B, T), wl.q_pos0, dtype=torch.int64, device=dev)
        self.swa_pos0 = torch.full((B,), wl.swa_pos0, dtype=torch.int64, device=dev)
        self.n_valid = csa.csa_n_valid(self.q_pos, 4, 0, N)
        # per-step inputs
        cL, cc = wl.comp_L, wl.comp_c
        self.inputs = {
            "q": g("q", (B, T, H, D)), "qI": g("qI", (B, T, 64, 128)), "w": f32("w", (B, T, 64)),
            "C_a": g("C_a", (B, cL, cc)), "C_b": g("C_b", (B, cL, cc)), "Z_a": g("Z_a", (B, cL, cc)),
            "Z_b": g("Z_b", (B, cL, cc)), "prev_Cb": g("prev_Cb", (B, 4, cc)), "prev_Zb": g("prev_Zb", (B, 4, cc)),
        }
        if wl.comp_ci:
            ci = wl.comp_ci
            self.inputs.update({"iC_a": g("iC_a", (B, cL, ci)), "iC_b": g("iC_b", (B, cL, ci)),
                                "iZ_a": g("iZ_a", (B, cL, ci)), "iZ_b": g("iZ_b", (B, cL, ci)),
                                "iprev_Cb": g("iprev_Cb", (B, 4, ci)), "iprev_Zb": g("iprev_Zb", (B, 4, ci))})
        # outputs and scratch
        self.comp_kv = torch.empty((B, cL // 4, cc), dtype=torch.bfloat16, device=dev)
        # new index-key entries go straight into the caches' newest rows (bf16 keys and, on
        # the e4m3 path, their rotated e4m3 codes and scales): rows N - L/4 .. N - 1
        self.new_key_pos = N - cL // 4
        self.theta = 0.0 if kv8 else ROPE_THETA
        # RoPE positions of the step's new entries: latent entry i at 4 (N - L/4 + i)
        self.new_entry_pos = torch.full((B,), 4 * (N - cL // 4), dtype=torch.int64, device=dev)
        self.scores = torch.empty((B, T, N), dtype=torch.float32, device=dev)
        self.q8 = torch.empty((B, T, 64, 128), dtype=torch.uint8, device=dev)
        self.qs = torch.empty((B, T, 64), dtype=torch.float32, device=dev)
        if index == "mxfp4":
            self.q4 = torch.empty((B, T, 64, 64), dtype=torch.uint8, device=dev)
            self.qsf = torch.zeros(csa.csa_mxfp4_sf128_bytes(B, T * 64), dtype=torch.uint8, device=dev)
        self.idx = torch.empty((B, T, k), dtype=torch.int32, device=dev)
        self.select_ws = csa.select_workspace(B, N, dev)
        self.attn_ws = csa.attn_workspace(B, T, H, D, 128 + k, device=dev)
        self.out = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
        # the attention's memory rows: bf16 rows, or (kv8) mixed-precision entries, in which
        # case the step also quantises the entries its compressor produces
        self.kv_store = self.kv
        if kv8:
            self.kv_store = csa.quantize_kv8(self.kv)
            self.kv = None
            self.comp_kv8 = torch.empty(self.comp_kv.shape[:-1] + (csa.KV8_BYTES,), dtype=torch.uint8, device=dev)
        if with_hca:
            Nh = wl.ctx // 128
            self.hkv = g("hkv", (B, Nh, D))
            self.hswa = g("hswa", (B, wl.W, D))
            self.hsink = f32("hsink", (H,))
            self.inputs.update({"hq": g("hq", (B, T, H, D)), "hC": g("hC", (B, 128, D)), "hZ": g("hZ", (B, 128, D))})
            self.hcomp = torch.empty((B, 1, D), dtype=torch.bfloat16, device=dev)
            self.hnew_pos = torch.full((B,), 128 * (Nh - 1), dtype=torch.int64, device=dev)
            self.hattn_ws = csa.attn_workspace(B, T, H, D, 128 + Nh, device=dev)
            self.hout = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
            self.hkv_store = self.hkv
            if kv8:
                self.hkv_store = csa.quantize_kv8(self.hkv)
                self.hkv = None
                self.hcomp8 = torch.empty((B, 1, csa.KV8_BYTES), dtype=torch.uint8, device=dev)
        # per-step inputs and outputs live in one contiguous device buffer each (views at
        # 16-byte aligned offsets), so a step moves them with one copy per direction
        self.in_buf, views = _pack(list(self.inputs.values()), dev)
        self.inputs = dict(zip(self.inputs.keys(), views))
        outs = [self.out] + ([self.hout] if with_hca else [])
        self.out_buf, outs = _pack(outs, dev)
        self.out = outs[0]
        if with_hca:
            self.hout = outs[1]
        self.outputs = outs
        self.host_in = torch.empty(self.in_buf.numel(), dtype=torch.uint8, pin_memory=True)
        self.host_in.copy_(self.in_buf)
        self.host_out = torch.empty(self.out_buf.numel(), dtype=torch.uint8, pin_memory=True)

    # -- byte accounting (algorithmic: inputs read once, outputs written once, intermediates excluded)
    def index_bytes(self):
        wl = self.wl
        B, T, N = wl.B, wl.T, wl.N
        if self.index == "e4m3":
            keys = B * N * (128 + 4)
            q = B * T * 64 * (128 + 4 + 4)
        elif self.index == "mxfp4":
            keys = B * N * (64 + 4)                 # 128 E2M1 codes + 4 E8M0 scales per key
            q = B * T * 64 * (64 + 4 + 4)
        else:
            keys = B * N * 256
            q = B * T * 64 * (256 + 4)
        return keys + q + B * T * N * 4

    def row_bytes(self):
        """Bytes of one memory row of the attention: bf16 row or mixed-precision entry."""
        return 608 if self.kv8 else self.wl.D * 2

    def attn_bytes(self):
        """One sparse_attn launch: q, the gathered top-k and SWA rows, idx, sink, out."""
        wl = self.wl
        B, T, H, D, k = wl.B, wl.T, wl.H, wl.D, wl.topk
        rows = B * T * (k * self.row_bytes() + min(wl.W, 128) * D * 2)
        return B * T * H * D * 2 * 2 + rows + B * T * k * 4 + H * 4

    def step_bytes(self):
        wl = self.wl
        B, T, N, H, D, k = wl.B, wl.T, wl.N, wl.H, wl.D, wl.topk
        nb = lambda t: t.numel() * t.element_size()
        total = sum(nb(t) for t in self.inputs.values())                       # per-step inputs
        total += nb(self.comp_kv)                                             # latent compressor output
        low = {"e4m3": 132, "mxfp4": 68}.get(self.index, 0)                 # low-precision key bytes
        if wl.comp_ci:                                                        # new index keys (+ quantised)
            total += B * (wl.comp_L // 4) * (256 + low)
        total += B * N * (low if low else 256)                                # index keys (+ scales)
        if low:
            total += B * T * self.kc_factor() * k * 256                       # rescoring: bf16 keys of candidates
        total += B * T * (k * self.row_bytes() + min(wl.W, 128) * D * 2)      # gathered latent + SWA rows
        total += nb(self.out)
        if self.kv8:
            total += nb(self.comp_kv) + nb(self.comp_kv8)                      # quantise the new entries
        if self.with_hca:
            total += B * (wl.ctx // 128) * self.row_bytes() + B * min(wl.W, 128) * D * 2 + nb(self.hcomp)
            total += nb(self.hout)
            if self.kv8:
                total += nb(self.hcomp) + nb(self.hcomp8)
        return total

    def kc_factor(self):
        """Candidate list of the rescoring select, in units of k (FP4 scores are coarser)."""
        return 4 if self.index == "mxfp4" else 2

    def per_step_io(self):
        nb = lambda t: t.numel() * t.element_size()
        return nb(self.in_buf), nb(self.out_buf)

    # -- the step
    def run(self, side_streams, timing_events: bool = False, copies: bool = False):
        import torch

        from long_context_compressed_b200 import csa
        wl = self.wl
        x = self.inputs
        main = torch.cuda.current_stream()
        if SCHEDULE == "serial":
            side_streams = (main,) * len(side_streams)
        if copies:
            self.in_buf.copy_(self.host_in, non_blocking=True)
        def side_branch():
            # the latent compressor and the HCA layer: independent of the indexer chain and
            # of each other within a step, so they run on side streams, started once the
            # bandwidth-bound indexer is done and overlapping the latency-bound top-k /
            # rerank / attention kernels
            sa, sb, sc = side_streams
            sa.wait_stream(main)
            sc.wait_stream(main)
            with torch.cuda.stream(sa):
                csa.csa_compress(x["C_a"], x["C_b"], x["Z_a"], x["Z_b"], x["prev_Cb"], x["prev_Zb"], ratio=4,
                                 out=self.comp_kv)
                if self.theta:
                    csa.csa_rope(self.comp_kv, self.theta, stride=4, pos_base=self.new_entry_pos, out=self.comp_kv)
                if self.kv8:
                    csa.quantize_kv8(self.comp_kv, entries=self.comp_kv8)
            if self.with_hca:
                with torch.cuda.stream(sc):
                    csa.csa_compress(x["hC"], None, x["hZ"], None, ratio=128, out=self.hcomp)
                    if self.theta:
                        csa.csa_rope(self.hcomp, self.theta, stride=128, pos_base=self.hnew_pos, out=self.hcomp)
                    if self.kv8:
                        csa.quantize_kv8(self.hcomp, entries=self.hcomp8)
                    csa.hca_attn(x["hq"], self.hkv_store, self.hswa, self.swa_pos0, self.q_pos, self.hsink,
                                 1.0 / math.sqrt(wl.D), rope_theta=self.theta, out=self.hout,
                                 workspace=self.hattn_ws)

        def append_index_keys():
            # the step's new index-key entries, compressed, rotated and quantised in one launch
            # into the caches' newest rows; after the select, the last reader of the bf16 keys
            # in this step, so the next step's indexer scans them
            sb = side_streams[1]
            sb.wait_stream(main)
            if wl.comp_ci:
                with torch.cuda.stream(sb):
                    e4 = self.index == "e4m3"
                    csa.csa_compress_index_keys(x["iC_a"], x["iC_b"], x["iZ_a"], x["iZ_b"], x["iprev_Cb"],
                                                x["iprev_Zb"], self.kI, pos0=self.new_key_pos,
                                                k8=self.k8 if e4 else None, k_scale=self.ks if e4 else None,
                                                hadamard=INDEX_ROTATION)
                    if self.index == "mxfp4":
                        # re-quantise the 128-row tiles that hold the new entries (N is a multiple
                        # of 128): their codes and tensor-core-layout scales
                        p0, n_new, tiles = self.new_key_pos, wl.comp_L // 4, wl.N // 128
                        r0, r1 = (p0 // 128) * 128, -(-(p0 + n_new) // 128) * 128
                        for b in range(wl.B):
                            csa.csa_quantize_mxfp4_sf128(self.kI[b, r0:r1], (r1 - r0) // 128,
                                                         codes=self.k4[b, r0:r1],
                                                         sf=self.ksf[(b * tiles + r0 // 128) * 512:])

        # stage boundaries on the main stream (event record nodes inside the graph)
        # timing_events: False (the timed graphs) or "all" (every stage: a diagnostic graph;
        # event nodes break the programmatic-launch overlap and add their own latency)
        marks = []

        def mark(name):
            if timing_events == "all":
                ev = torch.cuda.Event(enable_timing=True, external=True)
                ev.record()
                marks.append((name, ev))
        mark("start")
        if SCHEDULE == "early":
            side_branch()
        if self.index == "e4m3":
            csa.csa_quantize_e4m3(x["qI"], codes=self.q8, scale=self.qs, hadamard=INDEX_ROTATION)
            mark("quantize_q")
            # the launch before it is the query quantiser, which does not write the keys
            csa.csa_index_scores(self.q8, x["w"], self.k8, self.n_valid, q_scale=self.qs, k_scale=self.ks,
                                 scores=self.scores, select_ws=self.select_ws, keys_ready=True)
            mark("index")
            if SCHEDULE in ("streams", "serial"):
                side_branch()
            # top-2k bin of the e4m3 scores, exact bf16 rescoring, best k -- one launch
            csa.csa_topk_select(self.scores, self.n_valid, wl.topk, self.select_ws, kc=2 * wl.topk, qI=x["qI"],
                                w=x["w"], kI=self.kI, idx=self.idx)
            mark("select")
        elif self.index == "mxfp4":
            csa.csa_quantize_mxfp4_sf128(x["qI"], wl.B, codes=self.q4, sf=self.qsf)
            mark("quantize_q")
            csa.csa_index_scores(self.q4, x["w"], self.k4, self.n_valid, q_scale=self.qsf, k_scale=self.ksf,
                                 scores=self.scores, select_ws=self.select_ws, mxfp4=True, keys_ready=True)
            mark("index")
            if SCHEDULE in ("streams", "serial"):
                side_branch()
            # top-4k bin of the FP4 scores, exact bf16 rescoring, best k -- one launch
            csa.csa_topk_select(self.scores, self.n_valid, wl.topk, self.select_ws, kc=4 * wl.topk, qI=x["qI"],
                                w=x["w"], kI=self.kI, idx=self.idx)
            mark("select")
        else:
            csa.csa_index_scores(x["qI"], x["w"], self.kI, self.n_valid, scores=self.scores,
                                 select_ws=self.select_ws)
            mark("index")
            if SCHEDULE in ("streams", "serial"):
                side_branch()
            csa.csa_topk_select(self.scores, self.n_valid, wl.topk, self.select_ws, idx=self.idx)
            mark("select")
        if SCHEDULE == "late":
            side_branch()
        append_index_keys()
        csa.sparse_attn(x["q"], self.kv_store, self.swa, self.swa_pos0, self.q_pos, self.sink, self.idx,
                        1.0 / math.sqrt(wl.D), rope_theta=self.theta, out=self.out, workspace=self.attn_ws)
        mark("sparse_attn")
        for ss in side_streams:
            main.wait_stream(ss)
        mark("join")
        if timing_events:
            self.marks = marks
        if copies:
            self.host_out.copy_(self.out_buf, non_blocking=True)


def capture(sets, sides, **kw):
    import torch

    from long_context_compressed_b200 import csa
    graphs, launches = [], None
    for s in sets:
        s.run(sides, **{k: v for k, v in kw.items() if k != "timing_events"})     # eager warm-up
    torch.cuda.synchronize()
    for s in sets:
        g = torch.cuda.CUDAGraph()
        c0 = csa.csa_launch_count()
        with torch.cuda.graph(g):
            s.run(sides, **kw)
        if launches is None:
            launches = csa.csa_launch_count() - c0
        graphs.append(g)
    torch.cuda.synchronize()
    return graphs, launches


def capture_steps(sets, sides, copies: bool):
    """One CUDA graph that runs the given input sets once each, in order, as a serving loop
    would.  With copies, the host->device copy of step j+1's inputs (pinned host buffer, its
    own stream) and the device->host read of step j's outputs (another stream) overlap step
    j's compute; every step still moves its own inputs and outputs inside the graph."""
    import torch
    # the capturing stream itself is "main": the copy streams join the capture by waiting on
    # it, so the copies are nodes of the graph and run on every replay
    main = torch.cuda.Stream()
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    for s in sets:
        s.run(sides)                                          # eager warm-up
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=main):
        if not copies:
            for s in sets:
                s.run(sides)
        else:
            ev_in = [torch.cuda.Event() for _ in sets]
            ev_done = [torch.cuda.Event() for _ in sets]
            h2d.wait_stream(main)
            d2h.wait_stream(main)
            with torch.cuda.stream(h2d):
                sets[0].in_buf.copy_(sets[0].host_in, non_blocking=True)
                ev_in[0].record(h2d)
            for j, s in enumerate(sets):
                if j + 1 < len(sets):
                    with torch.cuda.stream(h2d):
                        sets[j + 1].in_buf.copy_(sets[j + 1].host_in, non_blocking=True)
                        ev_in[j + 1].record(h2d)
                main.wait_event(ev_in[j])
                s.run(sides)
                ev_done[j].record(main)
                with torch.cuda.stream(d2h):
                    d2h.wait_event(ev_done[j])
                    s.host_out.copy_(s.out_buf, non_blocking=True)
            main.wait_stream(h2d)
            main.wait_stream(d2h)
    torch.cuda.synchronize()
    return g


def timed_steps(sets, sides, steps: int, warmup: int, world: int, copies: bool = False):
    """Seconds for exactly `steps` steps: replays of a graph over all input sets (each step
    on the next set, so a set is reused only after every other set has been touched) and one
    graph over the first steps % len(sets) sets; warm-up covers at least `warmup` steps."""
    import torch
    n = len(sets)
    g_all = capture_steps(sets, sides, copies)
    rem = steps % n
    g_rem = capture_steps(sets[:rem], sides, copies) if rem else None
    for _ in range(max(1, -(-warmup // n))):
        g_all.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps // n):
        g_all.replay()
    if g_rem is not None:
        g_rem.replay()
    b.record()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    del g_all, g_rem
    return a.elapsed_time(b) / 1e3          # seconds


def timed_replays(graphs, steps: int, warmup: int, world: int):
    import torch
    for i in range(warmup):
        graphs[i % len(graphs)].replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(steps):
        graphs[i % len(graphs)].replay()
    b.record()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / 1e3          # seconds


def index_alone_ms(sets, index, device, reps_per_set=8, replays=20):
    """Average duration (ms) of one indexer launch timed alone: a graph of back-to-back
    csa_index_scores launches cycling over the input sets (each set's keys are cold in
    L2 when its turn comes), CUDA events around each replay of that graph.  The score
    histogram goes to a scratch workspace so the step's own workspaces stay intact."""
    import torch

    from long_context_compressed_b200 import csa
    scratch = [csa.select_workspace(s.wl.B, s.wl.N, device) for s in sets]
    n = reps_per_set * len(sets)

    def launch(i):
        s = sets[i % len(sets)]
        x = s.inputs
        if index == "e4m3":
            csa.csa_index_scores(s.q8, x["w"], s.k8, s.n_valid, q_scale=s.qs, k_scale=s.ks, scores=s.scores,
                                 select_ws=scratch[i % len(sets)])
        elif index == "mxfp4":
            csa.csa_index_scores(s.q4, x["w"], s.k4, s.n_valid, q_scale=s.qsf, k_scale=s.ksf, scores=s.scores,
                                 select_ws=scratch[i % len(sets)], mxfp4=True)
        else:
            csa.csa_index_scores(x["qI"], x["w"], s.kI, s.n_valid, scores=s.scores, select_ws=scratch[i % len(sets)])
    for i in range(len(sets)):
        launch(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n):
            launch(i)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(replays):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / (replays * n)
    del g, scratch
    return ms


def attn_alone_ms(sets, device, reps_per_set=8, replays=20):
    """Average duration (ms) of one sparse_attn launch timed alone (attn_t_kernel for bf16
    rows, attn_tc_kernel for KV8 entries):
    back-to-back launches in one CUDA graph cycling over the input sets (cold in L2),
    CUDA events around the graph replays."""
    import torch

    from long_context_compressed_b200 import csa
    n = reps_per_set * len(sets)

    def launch(i):
        s = sets[i % len(sets)]
        x = s.inputs
        csa.sparse_attn(x["q"], s.kv_store, s.swa, s.swa_pos0, s.q_pos, s.sink, s.idx, 1.0 / math.sqrt(s.wl.D),
                        rope_theta=s.theta,
                        out=s.out, workspace=s.attn_ws)
    for i in range(len(sets)):
        launch(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n):
            launch(i)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(replays):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / (replays * n)
    del g
    return ms


def bench_workload(name, index, with_hca, steps, warmup, world, device, n_sets=None, kv8=False):
    import torch

    from long_context_compressed_b200 import csa, synth
    wl = synth.WORKLOADS[name]
    probe = DecodeSet(wl, 0, index, with_hca, device, kv8=kv8)
    touched = probe.step_bytes()
    n_sets = n_sets or max(2, math.ceil(2 * L2_BYTES / touched) + 1)
    sets = [probe] + [DecodeSet(wl, s, index, with_hca, device, kv8=kv8) for s in range(1, n_sets)]
    side = [torch.cuda.Stream(device=device) for _ in range(3)]
    graphs, launches = capture(sets, side)
    # one graph per step, sets in rotation (reported beside the value)
    t_single = max_over_ranks(timed_replays(graphs, steps, warmup, world), world, device)
    del graphs
    # the value: one graph running a step on every input set in turn, as a serving loop
    # runs steps back to back (no graph launch between consecutive steps)
    t = max_over_ranks(timed_steps(sets, side, steps, warmup, world, copies=False), world, device)
    idx_ms = index_alone_ms(sets, index, device, replays=max(3, min(20, steps // 100)))
    attn_ms = attn_alone_ms(sets, device, replays=max(3, min(20, steps // 100)))
    # per-stage breakdown from a separate diagnostic graph with events between all stages
    diag, _ = capture(sets, side, timing_events="all")
    timed_replays(diag, min(steps, 200), 5, world)
    breakdown = {}
    try:
        for s in sets:
            for (n0, e0), (n1, e1) in zip(s.marks[:-1], s.marks[1:]):
                breakdown.setdefault(n1, []).append(1e3 * e0.elapsed_time(e1))
        breakdown = {k: round(statistics.mean(v), 2) for k, v in breakdown.items()}
    except RuntimeError:
        breakdown = {}
    del diag
    # end to end: the same step with its inputs copied in from pinned host memory and its
    # outputs read back, inside every timed step
    # (the next step's input copy and the previous outputs' read overlap each step's compute)
    t_e2e = max_over_ranks(timed_steps(sets, side, steps, warmup, world, copies=True), world, device)
    breakdown["one_graph_per_step_us"] = round(1e6 * t_single / steps, 2)
    assert csa.csa_poll_status() == csa.CSA_OK
    h2d, d2h = probe.per_step_io()
    res = {"wl": wl, "index": index, "with_hca": with_hca, "sets": n_sets, "seconds": t, "step_ms": 1e3 * t / steps, "launches": launches,
           "index_ms": idx_ms, "index_bytes": probe.index_bytes(), "step_bytes": touched,
           "attn_ms": attn_ms, "attn_bytes": probe.attn_bytes(),
           "e2e_seconds": t_e2e, "h2d": h2d, "d2h": d2h, "tokens_per_step": wl.B * wl.T,
           "breakdown": breakdown}
    del sets
    torch.cuda.empty_cache()
    return res


def _stage_times(stages, steps, warmup):
    """Eager calls, CUDA events between stages on the current stream: mean device time
    per stage (us) and per step (ms).  Every step reads and writes hundreds of MB (the
    attention's 256 MB of queries and of outputs), so no input stays in L2 from one step
    to the next."""
    import torch
    for _ in range(warmup):
        for _, fn in stages:
            fn()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)] for _ in range(steps)]
    for i in range(steps):
        evs[i][0].record()
        for j, (_, fn) in enumerate(stages):
            fn()
            evs[i][j + 1].record()
    torch.cuda.synchronize()
    per = {n: 1e3 * statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(steps))
           for j, (n, _) in enumerate(stages)}
    step_ms = statistics.mean(evs[i][0].elapsed_time(evs[i][-1]) for i in range(steps))
    return per, step_ms


def bench_prefill(steps, warmup, device, tflops_peak):
    """Flash-shaped chunked prefill (4,096 query tokens at 126,976..131,071 of a 131,072-token
    context, B = 1): compress the chunk (c = 512 latent + 128 index keys), bf16 index scores
    over 32,768 keys, top-512 per query, sparse_attn (64 heads, D = 512).  Also timed: the
    indexer and top-k in one call without the score matrix (csa_index_topk; its indices are
    checked equal to the step's), and the indexer alone in e4m3 (quantised queries and
    keys).  Indexer FLOPs = 2 x 64 x 128 x sum(n_valid)."""
    import torch

    from long_context_compressed_b200 import csa, synth
    wl = synth.WORKLOADS["flash_prefill"]
    B, T, N, H, D, k = wl.B, wl.T, wl.N, wl.H, wl.D, wl.topk
    dev = device
    g = lambda nm, shape: synth.store(synth.normal(0, f"bench/{wl.name}/{nm}", shape, device=dev), "bf16")
    f32 = lambda nm, shape: synth.normal(0, f"bench/{wl.name}/{nm}", shape, device=dev)
    kv, swa, kI = g("kv", (B, N, D)), g("swa", (B, wl.W, D)), g("kI", (B, N, 128))
    q, qI, w, sink = g("q", (B, T, H, D)), g("qI", (B, T, 64, 128)), f32("w", (B, T, 64)), f32("sink", (H,))
    cL, cc, ci = wl.comp_L, wl.comp_c, wl.comp_ci
    cz = {nm: g(nm, (B, cL, cc)) for nm in ("C_a", "C_b", "Z_a", "Z_b")}
    cp = {nm: g(nm, (B, 4, cc)) for nm in ("prev_Cb", "prev_Zb")}
    iz = {nm: g("i" + nm, (B, cL, ci)) for nm in ("C_a", "C_b", "Z_a", "Z_b")}
    ip = {nm: g("i" + nm, (B, 4, ci)) for nm in ("prev_Cb", "prev_Zb")}
    q_pos = (torch.arange(T, device=dev, dtype=torch.int64) + wl.q_pos0).view(1, T).repeat(B, 1)
    swa_pos0 = torch.full((B,), wl.swa_pos0, dtype=torch.int64, device=dev)
    n_valid = csa.csa_n_valid(q_pos, 4, 0, N)
    comp_kv = torch.empty((B, cL // 4, cc), dtype=torch.bfloat16, device=dev)
    scores = torch.empty((B, T, N), dtype=torch.float32, device=dev)
    idx = torch.empty((B, T, k), dtype=torch.int32, device=dev)
    topk_ws = csa.topk_workspace(B, T, N, k, dev)
    fused_ws = csa.index_topk_workspace(B, T, N, k, csa.CSA_BF16, dev)
    failed = torch.zeros((1,), dtype=torch.int32, device=dev)
    attn_ws = csa.attn_workspace(B, T, H, D, 128 + k, device=dev)
    out = torch.empty_like(q)
    k8, ks = csa.csa_quantize_e4m3(kI, hadamard=INDEX_ROTATION)
    q8 = torch.empty((B, T, 64, 128), dtype=torch.uint8, device=dev)
    qs = torch.empty((B, T, 64), dtype=torch.float32, device=dev)
    scale = 1.0 / math.sqrt(D)
    stages = [
        ("compress", lambda: (csa.csa_compress(cz["C_a"], cz["C_b"], cz["Z_a"], cz["Z_b"], cp["prev_Cb"],
                                               cp["prev_Zb"], ratio=4, out=comp_kv),
                              # the chunk's index keys, into the caches' newest rows (bf16 + e4m3)
                              csa.csa_compress_index_keys(iz["C_a"], iz["C_b"], iz["Z_a"], iz["Z_b"],
                                                          ip["prev_Cb"], ip["prev_Zb"], kI, pos0=N - cL // 4,
                                                          k8=k8, k_scale=ks, hadamard=INDEX_ROTATION))),
        ("index", lambda: csa.csa_index_scores(qI, w, kI, n_valid, scores=scores)),
        ("topk", lambda: csa.csa_topk(scores, n_valid, k, idx=idx, workspace=topk_ws)),
        ("sparse_attn", lambda: csa.sparse_attn(q, kv, swa, swa_pos0, q_pos, sink, idx, scale, out=out,
                                                workspace=attn_ws)),
    ]
    c0 = csa.csa_launch_count()
    for _, fn in stages:
        fn()
    launches = csa.csa_launch_count() - c0
    per, step_ms = _stage_times(stages, steps, warmup)
    idx_fused = torch.empty_like(idx)
    fused = [("index_topk", lambda: csa.csa_index_topk(qI, w, kI, n_valid, k, idx=idx_fused, workspace=fused_ws,
                                                       failed_rows=failed))]
    per_f, _ = _stage_times(fused, steps, warmup)
    assert torch.equal(idx, idx_fused), "fused and unfused prefill top-k differ"
    failed_rows = int(failed.item())
    e4m3 = [("quantize_q", lambda: csa.csa_quantize_e4m3(qI, codes=q8, scale=qs, hadamard=INDEX_ROTATION)),
            ("index_e4m3", lambda: csa.csa_index_scores(q8, w, k8, n_valid, q_scale=qs, k_scale=ks, scores=scores))]
    per8, _ = _stage_times(e4m3, steps, warmup)
    assert csa.csa_poll_status() == csa.CSA_OK
    flops = 2.0 * 64 * 128 * float(n_valid.sum().item())
    tf_bf16 = flops / (per["index"] * 1e-6) / 1e12
    tf_e4m3 = flops / (per8["index_e4m3"] * 1e-6) / 1e12
    res = {"workload": f"flash_prefill: B=1, {T} query tokens at {wl.q_pos0}..{wl.q_pos0 + T - 1}, "
                       f"N={N} keys, top-{k}, H={H}, D={D}",
           "tokens_per_s": B * T / (step_ms * 1e-3), "ms_per_step": step_ms, "steps": steps,
           "launches_per_step": launches, "breakdown_us": {n: round(v, 1) for n, v in per.items()},
           "index_topk": {"fused_us": per_f["index_topk"], "unfused_us": per["index"] + per["topk"],
                          "failed_rows": failed_rows,
                          "note": "csa_index_topk (no score matrix) on the step's inputs, same indices; "
                                  "the step keeps the faster unfused pair"},
           "indexer": {"keys_per_s": float(n_valid.sum().item()) / (per["index"] * 1e-6),
                       "bf16": {"achieved": tf_bf16, "peak": tflops_peak, "unit": "TFLOP/s",
                                "frac": tf_bf16 / tflops_peak, "peak_source": "measured bf16 (burst)",
                                "us": per["index"]},
                       "e4m3": {"achieved": tf_e4m3, "peak": 2 * tflops_peak, "unit": "TFLOP/s",
                                "frac": tf_e4m3 / (2 * tflops_peak),
                                "peak_source": "measured bf16 (burst) x 2 (nominal e4m3:bf16 ratio)",
                                "us": per8["index_e4m3"], "quantize_q_us": per8["quantize_q"]}}}
    del scores, out, q, topk_ws, attn_ws, fused_ws
    torch.cuda.empty_cache()
    return res


def bench_hca(steps, warmup, device, hbm_peak, kv8=False):
    """Pro-shaped HCA decode at 1M context, B = 4: compress the newest 16,384-token tail
    128:1 (c = 512) and hca_attn (128 heads, D = 512) over all 8,192 entries + 128 SWA rows.
    Input sets rotate so that more than 2x the L2 is touched between reuses."""
    import torch

    from long_context_compressed_b200 import csa, synth
    wl = synth.WORKLOADS["pro_hca"]
    B, T, N, H, D = wl.B, wl.T, wl.N, wl.H, wl.D
    dev = device
    sets = []
    nb = lambda t: t.numel() * t.element_size()
    while True:
        s = len(sets)
        g = lambda nm, shape: synth.store(synth.normal(s, f"bench/{wl.name}/{nm}", shape, device=dev), "bf16")
        st = {"C": g("C", (B, wl.comp_L, wl.comp_c)), "Z": g("Z", (B, wl.comp_L, wl.comp_c)),
              "kv": g("kv", (B, N, D)), "swa": g("swa", (B, wl.W, D)), "q": g("q", (B, T, H, D)),
              "sink": synth.normal(s, f"bench/{wl.name}/sink", (H,), device=dev)}
        st["comp"] = torch.empty((B, wl.comp_L // 128, D), dtype=torch.bfloat16, device=dev)
        st["out"] = torch.empty_like(st["q"])
        st["ws"] = csa.attn_workspace(B, T, H, D, 128 + N, device=dev)
        if kv8:                     # memory rows as mixed-precision entries; new entries quantised
            st["kv"] = csa.quantize_kv8(st["kv"])
            st["comp8"] = torch.empty((B, wl.comp_L // 128, csa.KV8_BYTES), dtype=torch.uint8, device=dev)
        sets.append(st)
        touched = sum(nb(st[n]) for n in ("C", "Z", "kv", "swa", "q", "comp", "out"))
        if len(sets) * touched > 2 * L2_BYTES and len(sets) >= 2:
            break
    q_pos = torch.full((B, T), wl.q_pos0, dtype=torch.int64, device=dev)
    swa_pos0 = torch.full((B,), wl.swa_pos0, dtype=torch.int64, device=dev)
    scale = 1.0 / math.sqrt(D)

    def step(st):
        csa.csa_compress(st["C"], None, st["Z"], None, ratio=128, out=st["comp"])
        if kv8:
            csa.quantize_kv8(st["comp"], entries=st["comp8"])
        csa.hca_attn(st["q"], st["kv"], st["swa"], swa_pos0, q_pos, st["sink"], scale, out=st["out"],
                     workspace=st["ws"])
    c0 = csa.csa_launch_count()
    step(sets[0])
    launches = csa.csa_launch_count() - c0
    graphs = []
    torch.cuda.synchronize()
    for st in sets:
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            step(st)
        graphs.append(gr)
    t = timed_replays(graphs, steps, warmup, 1)
    assert csa.csa_poll_status() == csa.CSA_OK
    ms = 1e3 * t / steps
    algo = sum(nb(sets[0][n]) for n in ("C", "Z", "q", "comp", "out")) + B * N * (608 if kv8 else D * 2)
    algo += B * 128 * D * 2
    if kv8:
        algo += nb(sets[0]["comp"]) + nb(sets[0]["comp8"])
    res = {"workload": f"pro_hca: B={B} decode at 1M, compress 128:1 over [{B},{wl.comp_L},{wl.comp_c}], "
                       f"hca_attn H={H} D={D} over {N}+128 rows"
                       + (", memory rows as 608-byte FP8/BF16 entries" if kv8 else ""),
           "tokens_per_s": B * T / (ms * 1e-3), "ms_per_step": ms, "launches_per_step": launches,
           "input_sets": len(sets),
           "step_roofline": {"bytes_per_step": algo, "achieved_gbs": algo / (ms * 1e-3) / 1e9,
                             "frac": algo / (ms * 1e-3) / 1e9 / hbm_peak, "floor_us": algo / (hbm_peak * 1e9) * 1e6}}
    del graphs, sets
    torch.cuda.empty_cache()
    return res


STAGES = ("compress", "quantize", "index", "select", "attn", "hcompress", "hca")
BIG_STAGES = ("prefill_compress", "prefill_index", "prefill_index8", "prefill_topk", "prefill_index_topk",
              "prefill_attn", "hca_compress", "hca_attn")


def run_big_stage(stage, steps, warmup, device):
    """One call of the chunked-prefill (flash_prefill) or HCA-decode (pro_hca) shapes,
    eagerly, for profiling a single kernel on its measured workload.  Prints the mean
    device time per call (CUDA events)."""
    import torch

    from long_context_compressed_b200 import csa, synth
    dev = device
    if stage.startswith("prefill"):
        wl = synth.WORKLOADS["flash_prefill"]
    else:
        wl = synth.WORKLOADS["pro_hca"]
    B, T, N, H, D, k = wl.B, wl.T, wl.N, wl.H, wl.D, wl.topk
    g = lambda nm, shape: synth.store(synth.normal(0, f"bench/{wl.name}/{nm}", shape, device=dev), "bf16")
    q_pos = (torch.arange(T, device=dev, dtype=torch.int64) + wl.q_pos0).view(1, T).repeat(B, 1)
    swa_pos0 = torch.full((B,), wl.swa_pos0, dtype=torch.int64, device=dev)
    sink = synth.normal(0, f"bench/{wl.name}/sink", (H,), device=dev)
    if stage == "prefill_compress":
        x = {nm: g(nm, (B, wl.comp_L, wl.comp_c)) for nm in ("C_a", "C_b", "Z_a", "Z_b")}
        pr = {nm: g(nm, (B, 4, wl.comp_c)) for nm in ("prev_Cb", "prev_Zb")}
        out = torch.empty((B, wl.comp_L // 4, wl.comp_c), dtype=torch.bfloat16, device=dev)
        fn = lambda: csa.csa_compress(x["C_a"], x["C_b"], x["Z_a"], x["Z_b"], pr["prev_Cb"], pr["prev_Zb"], ratio=4,
                                      out=out)
    elif stage == "prefill_index_topk":
        qI, kI = g("qI", (B, T, 64, 128)), g("kI", (B, N, 128))
        w = synth.normal(0, f"bench/{wl.name}/w", (B, T, 64), device=dev)
        n_valid = csa.csa_n_valid(q_pos, 4, 0, N)
        idx = torch.empty((B, T, k), dtype=torch.int32, device=dev)
        ws = csa.index_topk_workspace(B, T, N, k, csa.CSA_BF16, dev)
        fn = lambda: csa.csa_index_topk(qI, w, kI, n_valid, k, idx=idx, workspace=ws)
    elif stage in ("prefill_index", "prefill_index8", "prefill_topk"):
        qI, kI = g("qI", (B, T, 64, 128)), g("kI", (B, N, 128))
        w = synth.normal(0, f"bench/{wl.name}/w", (B, T, 64), device=dev)
        n_valid = csa.csa_n_valid(q_pos, 4, 0, N)
        scores = torch.empty((B, T, N), dtype=torch.float32, device=dev)
        if stage == "prefill_index8":
            q8, qs = csa.csa_quantize_e4m3(qI, hadamard=INDEX_ROTATION)
            k8, ks = csa.csa_quantize_e4m3(kI, hadamard=INDEX_ROTATION)
            fn = lambda: csa.csa_index_scores(q8, w, k8, n_valid, q_scale=qs, k_scale=ks, scores=scores)
        else:
            csa.csa_index_scores(qI, w, kI, n_valid, scores=scores)
            fn = lambda: csa.csa_index_scores(qI, w, kI, n_valid, scores=scores)
        if stage == "prefill_topk":
            idx = torch.empty((B, T, k), dtype=torch.int32, device=dev)
            ws = csa.topk_workspace(B, T, N, k, dev)
            fn = lambda: csa.csa_topk(scores, n_valid, k, idx=idx, workspace=ws)
    elif stage == "prefill_attn":
        q, kv, swa = g("q", (B, T, H, D)), g("kv", (B, N, D)), g("swa", (B, wl.W, D))
        idx = synth.random_subset(0, f"bench/{wl.name}/idx", csa.csa_n_valid(q_pos, 4, 0, N).cpu(), k, device=dev)
        out = torch.empty_like(q)
        fn = lambda: csa.sparse_attn(q, kv, swa, swa_pos0, q_pos, sink, idx, 1.0 / math.sqrt(D), out=out)
    elif stage == "hca_compress":
        C, Z = g("C", (B, wl.comp_L, wl.comp_c)), g("Z", (B, wl.comp_L, wl.comp_c))
        out = torch.empty((B, wl.comp_L // 128, wl.comp_c), dtype=torch.bfloat16, device=dev)
        fn = lambda: csa.csa_compress(C, None, Z, None, ratio=128, out=out)
    elif stage == "hca_attn":
        q, kv, swa = g("q", (B, T, H, D)), g("kv", (B, N, D)), g("swa", (B, wl.W, D))
        out = torch.empty_like(q)
        fn = lambda: csa.hca_attn(q, kv, swa, swa_pos0, q_pos, sink, 1.0 / math.sqrt(D), out=out)
    else:
        raise SystemExit(f"unknown stage {stage}")
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        fn()
    b.record()
    torch.cuda.synchronize()
    assert csa.csa_poll_status() == csa.CSA_OK
    print(json.dumps({"stage": stage, "workload": wl.name, "steps": steps,
                      "us_per_call": 1e3 * a.elapsed_time(b) / steps}), flush=True)


def run_stage(name, stage, index, steps, warmup, device, kv8=False):
    """One stage of the step (one ABI call), eagerly, for profiling a single kernel.
    Prints the mean device time per call measured with CUDA events."""
    import torch

    from long_context_compressed_b200 import csa, synth
    wl = synth.WORKLOADS[name]
    st = DecodeSet(wl, 0, index, name == "flash64k", device, kv8=kv8)
    x = st.inputs
    calls = {
        "compress": lambda: csa.csa_compress(x["C_a"], x["C_b"], x["Z_a"], x["Z_b"], x["prev_Cb"], x["prev_Zb"],
                                             ratio=4, out=st.comp_kv),
        "quantize": (lambda: csa.csa_quantize_mxfp4_sf128(x["qI"], wl.B, codes=st.q4, sf=st.qsf))
                    if index == "mxfp4" else
                    (lambda: csa.csa_quantize_e4m3(x["qI"], codes=st.q8, scale=st.qs, hadamard=INDEX_ROTATION)),
        "index": (lambda: csa.csa_index_scores(st.q8, x["w"], st.k8, st.n_valid, q_scale=st.qs, k_scale=st.ks,
                                               scores=st.scores)) if index == "e4m3" else
                 (lambda: csa.csa_index_scores(st.q4, x["w"], st.k4, st.n_valid, q_scale=st.qsf, k_scale=st.ksf,
                                               scores=st.scores, mxfp4=True)) if index == "mxfp4" else
                 (lambda: csa.csa_index_scores(x["qI"], x["w"], st.kI, st.n_valid, scores=st.scores)),
        "select": (lambda: (csa.csa_score_histogram(st.scores, st.n_valid, st.select_ws),
                            csa.csa_topk_select(st.scores, st.n_valid, wl.topk, st.select_ws,
                                                kc=st.kc_factor() * wl.topk, qI=x["qI"], w=x["w"], kI=st.kI,
                                                idx=st.idx)))
                  if index in ("e4m3", "mxfp4") else
                  (lambda: (csa.csa_score_histogram(st.scores, st.n_valid, st.select_ws),
                            csa.csa_topk_select(st.scores, st.n_valid, wl.topk, st.select_ws, idx=st.idx))),
        "attn": lambda: csa.sparse_attn(x["q"], st.kv_store, st.swa, st.swa_pos0, st.q_pos, st.sink, st.idx,
                                        1.0 / math.sqrt(wl.D), rope_theta=st.theta, out=st.out,
                                        workspace=st.attn_ws),
        "hcompress": lambda: csa.csa_compress(x["hC"], None, x["hZ"], None, ratio=128, out=st.hcomp),
        "hca": lambda: csa.hca_attn(x["hq"], st.hkv_store, st.hswa, st.swa_pos0, st.q_pos, st.hsink,
                                    1.0 / math.sqrt(wl.D), rope_theta=st.theta, out=st.hout,
                                    workspace=st.hattn_ws),
    }
    # inputs of the later stages come from the earlier ones
    order = ["quantize", "index", "select"] if index in ("e4m3", "mxfp4") else ["index", "select"]
    if stage in ("select", "attn"):
        for pre in order[:order.index(stage)] if stage in order else order:
            calls[pre]()
    fn = calls[stage]
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        fn()
    b.record()
    torch.cuda.synchronize()
    assert csa.csa_poll_status() == csa.CSA_OK
    print(json.dumps({"stage": stage, "workload": name, "index": index, "steps": steps,
                      "us_per_call": 1e3 * a.elapsed_time(b) / steps}), flush=True)


# ----------------------------------------------------------------------------- oracle (CPU) leg
def oracle_decode_token(wl, seed, index, with_hca):
    """One sequence's decode step through the CPU oracle (fp64), on the same recipe."""
    import numpy as np

    import oracle
    from long_context_compressed_b200 import synth
    one = synth.Workload(**{**wl.__dict__, "B": 1, "extra": {}})
    g = lambda nm, shape: synth.store(synth.normal(seed, f"bench/{wl.name}/{nm}", shape), "bf16").float().numpy()
    f32 = lambda nm, shape: synth.normal(seed, f"bench/{wl.name}/{nm}", shape).numpy()
    N, H, D, k, cL, cc = one.N, one.H, one.D, one.topk, one.comp_L, one.comp_c
    kv, swa, kI = g("kv", (1, N, D)), g("swa", (1, one.W, D)), g("kI", (1, N, 128))
    q, qI, w = g("q", (1, 1, H, D)), g("qI", (1, 1, 64, 128)), f32("w", (1, 1, 64))
    sink = f32("sink", (H,))
    comp = {nm: g(nm, (1, cL, cc)) for nm in ("C_a", "C_b", "Z_a", "Z_b")}
    prev = {nm: g(nm, (1, 4, cc)) for nm in ("prev_Cb", "prev_Zb")}
    k8, ks = oracle_quantizer()(kI) if index == "e4m3" else (None, None)
    q_pos = np.array([[one.q_pos0]], np.int64)
    nv = oracle.n_visible(q_pos, 4, N)
    t0 = time.perf_counter()
    oracle.compress_csa(comp["C_a"], comp["C_b"], comp["Z_a"], comp["Z_b"], prev["prev_Cb"], prev["prev_Zb"])
    if index == "e4m3":
        q8, qs = oracle_quantizer()(qI)
        s8 = oracle.index_scores_e4m3(q8, qs, w, k8, ks, nv)
        cand = oracle.topk(s8.astype(np.float32), nv, 2 * k)[0, 0]
        cand = cand[cand >= 0]
        sc = oracle.index_scores(qI, w, kI[:, cand], np.array([[len(cand)]], np.int32))
        pos = oracle.topk(sc.astype(np.float32), np.array([[len(cand)]], np.int32), k)[0, 0]
        idx = np.where(pos >= 0, cand[np.maximum(pos, 0)], -1).astype(np.int32)[None, None]
    else:
        s = oracle.index_scores(qI, w, kI, nv)
        idx = oracle.topk(s.astype(np.float32), nv, k)
    oracle.sparse_attn(q, kv, swa, [one.swa_pos0], q_pos, sink, idx, 1 / math.sqrt(D))
    if with_hca:
        Nh = one.ctx // 128
        oracle.compress_hca(g("hC", (1, 128, D)), g("hZ", (1, 128, D)))
        oracle.hca_attn(g("hq", (1, 1, H, D)), g("hkv", (1, Nh, D)), g("hswa", (1, one.W, D)), [one.swa_pos0],
                        q_pos, f32("hsink", (H,)), 1 / math.sqrt(D))
    return time.perf_counter() - t0


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def oracle_baseline(wl, index, with_hca, budget_s=12.0, max_tokens=24):
    """Oracle tokens/s on a bounded sample: whole single-sequence decode steps (one token
    each, seeds 1000+) until about budget_s of oracle time.  Single-threaded C."""
    times = []
    while sum(times) < budget_s and len(times) < max_tokens:
        times.append(oracle_decode_token(wl, 1000 + len(times), index, with_hca))
    return {"value": len(times) / sum(times), "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{len(times)} single-sequence decode tokens of the {wl.name} step (one sequence of the "
                      f"B={wl.B} batch each), {sum(times):.1f} s of single-threaded fp64 C oracle on "
                      f"{cpu_model()}"}


def oracle_config_timings(seed=2000):
    """The CPU oracle (single-threaded fp64 C) on the other configurations, one bounded
    sample each: the whole tiny step (8 queries); one pro1m decode token (the same chain as
    the GPU step: rotated e4m3 scores, 2k candidates, exact rerank, sparse_attn); one
    pro_hca sequence (128:1 compressor over the 16,384-token tail, hca_attn over 8,192 + 128
    rows); the flash_prefill chunk's compressors in full plus 8 of its 4,096 queries (index,
    top-512, sparse_attn), extrapolated to the chunk.  Input preparation is not timed."""
    import numpy as np

    import oracle
    from long_context_compressed_b200 import synth
    W = synth.WORKLOADS
    np32 = lambda t: t.float().numpy()
    out = {}
    # tiny: the whole step
    wl = W["tiny"]
    cz, ix, at = synth.draw_compressor(wl, seed), synth.draw_indexer(wl, seed), synth.draw_attention(wl, seed)
    q_pos = np.array([wl.q_pos], np.int64)
    nv = oracle.n_visible(q_pos, 4, wl.N)
    t0 = time.perf_counter()
    oracle.compress_csa(*(np32(cz[n]) for n in ("C_a", "C_b", "Z_a", "Z_b")))
    s = oracle.index_scores(np32(ix["qI"]), np32(ix["w"]), np32(ix["kI"]), nv)
    idx = oracle.topk(s.astype(np.float32), nv, wl.topk)
    oracle.sparse_attn(np32(at["q"]), np32(at["kv"]), np32(at["swa_kv"]), [wl.swa_pos0], q_pos, np32(at["sink"]),
                       idx, 1 / math.sqrt(wl.D))
    dt = time.perf_counter() - t0
    out["tiny"] = {"ms_per_step": 1e3 * dt, "tokens_per_s": wl.T / dt, "sample": "the whole 8-query step"}
    # pro1m: one decode token
    dt = oracle_decode_token(W["pro1m"], seed, "e4m3", False)
    out["pro1m"] = {"ms_per_step": 1e3 * dt, "tokens_per_s": 1 / dt, "sample": "one decode token (B=1)"}
    # pro_hca: one of the 4 sequences
    wl = W["pro_hca"]
    one = synth.Workload(**{**wl.__dict__, "B": 1, "extra": {}})
    hz, at = synth.draw_compressor(one, seed), synth.draw_attention(one, seed)
    q_pos = np.array([[one.q_pos0]], np.int64)
    t0 = time.perf_counter()
    oracle.compress_hca(np32(hz["C"]), np32(hz["Z"]))
    oracle.hca_attn(np32(at["q"]), np32(at["kv"]), np32(at["swa_kv"]), [one.swa_pos0], q_pos, np32(at["sink"]),
                    1 / math.sqrt(one.D))
    dt = time.perf_counter() - t0
    out["pro_hca"] = {"ms_per_step": 1e3 * dt * wl.B, "tokens_per_s": 1 / dt,
                      "sample": f"one of the {wl.B} sequences, x{wl.B} for the step"}
    # flash_prefill: compressors in full, 8 sampled queries, extrapolated
    wl = W["flash_prefill"]
    cz = synth.draw_compressor(wl, seed)
    czi = synth.draw_compressor(wl, seed, c=wl.comp_ci, tag="ki")
    ix, at = synth.draw_indexer(wl, seed), synth.draw_attention(wl, seed)
    rows = np.linspace(0, wl.T - 1, 8).round().astype(int)
    q_pos = np.array([[wl.q_pos0 + int(r) for r in rows]], np.int64)
    nv = oracle.n_visible(q_pos, 4, wl.N)
    t0 = time.perf_counter()
    for z in (cz, czi):
        oracle.compress_csa(*(np32(z[n]) for n in ("C_a", "C_b", "Z_a", "Z_b", "prev_Cb", "prev_Zb")))
    t_comp = time.perf_counter() - t0
    t0 = time.perf_counter()
    s = oracle.index_scores(np32(ix["qI"][:, rows]), np32(ix["w"][:, rows]), np32(ix["kI"]), nv)
    idx = oracle.topk(s.astype(np.float32), nv, wl.topk)
    oracle.sparse_attn(np32(at["q"][:, rows]), np32(at["kv"]), np32(at["swa_kv"]), [wl.swa_pos0], q_pos,
                       np32(at["sink"]), idx, 1 / math.sqrt(wl.D))
    t_q = (time.perf_counter() - t0) / len(rows)
    total = t_comp + t_q * wl.T
    out["flash_prefill"] = {"ms_per_step": 1e3 * total, "tokens_per_s": wl.T / total, "extrapolated": True,
                            "sample": f"both chunk compressors in full ({1e3 * t_comp:.1f} ms) plus {len(rows)} of "
                                      f"the {wl.T} queries ({1e3 * t_q:.1f} ms each), scaled to {wl.T} queries"}
    return {"cores": 1, "kind": "oracle", "cpu": cpu_model(), "configs": out}


def workload_text(wl, index, with_hca):
    """The JSON line's config.workload, the same for both arms."""
    return (f"{wl.name}: B={wl.B} decode tokens/GPU at ctx {wl.ctx}; CSA layer (compress 4:1 c=512+128, "
            f"{index} index over N={wl.N}, top-{wl.topk}"
            + ((" (Hadamard-rotated q/k)" if INDEX_ROTATION else "") + " via 2k rerank" if index == "e4m3" else "")
            + ((" (Hadamard-rotated q/k, MXFP4)" if INDEX_ROTATION else " (MXFP4)") + " via 4k rescoring"
               if index == "mxfp4" else "")
            + f", sparse_attn H={wl.H} D={wl.D})"
            + (f" + HCA layer (compress 128:1, hca_attn over {wl.ctx // 128}+128 rows)" if with_hca else ""))


# ----------------------------------------------------------------------------- main
def main():
    global SCHEDULE
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="flash64k", choices=["flash64k", "pro1m"])
    ap.add_argument("--index", default="e4m3", choices=["e4m3", "bf16", "mxfp4"])
    ap.add_argument("--no-hadamard", action="store_true",
                    help="e4m3 index path without the Hadamard rotation of queries and keys")
    ap.add_argument("--no-extra", action="store_true", help="skip the pro1m measurement")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--stage", choices=STAGES + BIG_STAGES, help="time one stage alone (eager calls), e.g. under ncu")
    ap.add_argument("--kv8", action="store_true", help="with --stage: memory rows as mixed-precision KV8 entries")
    ap.add_argument("--schedule", choices=["streams", "early", "late", "serial"], default=SCHEDULE,
                    help="streams: compressors / HCA layer on side streams, forked after the indexer; "
                         "early / late: the same, forked at the step's start / after the select; "
                         "serial: every launch of the step on one stream")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    SCHEDULE = args.schedule
    global INDEX_ROTATION
    INDEX_ROTATION = not args.no_hadamard
    rank, world, local = dist_env()
    with_hca = args.workload == "flash64k"

    if args.impl == "reference":
        # the reference arm is the CPU oracle, on rank 0 only
        if rank != 0:
            return
        from long_context_compressed_b200 import synth
        wl = synth.WORKLOADS[args.workload]
        budget = 150.0
        per = oracle_decode_token(wl, 999, args.index, with_hca)     # calibration, untimed
        steps = max(1, min(args.steps, int(budget / max(per, 1e-3))))
        for i in range(min(args.warmup, 3)):
            oracle_decode_token(wl, 900 + i, args.index, with_hca)
        times = [oracle_decode_token(wl, 1000 + i, args.index, with_hca) for i in range(steps)]
        v = steps / sum(times)
        line = {"impl": "reference", "metric": "CSA decode tokens/s (64K Flash CSA+HCA layer pair)",
                "value": v, "unit": "tokens/s", "n_gpus": args.gpus, "steps": steps, "warmup": args.warmup,
                "ms_per_step": 1e3 * sum(times) / steps, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": workload_text(wl, args.index, with_hca),
                           "sample": "one sequence per step"},
                "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                 "sample": f"{steps} steps of one single-sequence decode token each "
                                           f"(capped from {args.steps} to stay within minutes) on {cpu_model()}"},
                "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    init_dist(world, "nccl")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    import __graft_entry__
    __graft_entry__.build()
    from long_context_compressed_b200 import csa  # noqa: F401  (fails loudly if libcsa.so is missing)

    if args.stage in BIG_STAGES:
        run_big_stage(args.stage, args.steps, args.warmup, device)
        return
    if args.stage:
        run_stage(args.workload, args.stage, args.index, args.steps, args.warmup, device, kv8=args.kv8)
        return
    peak, peak_kind = measured_peaks()
    sampler = ClockSampler(local)
    main_res = bench_workload(args.workload, args.index, with_hca, args.steps, args.warmup, world, device)
    clocks = sampler.stop()
    extra = None
    if not args.no_extra and args.workload != "pro1m":
        extra = bench_workload("pro1m", args.index, False, args.steps, args.warmup, world, device)
    variants = {}
    if not args.no_extra and args.workload == "flash64k":
        # the same configuration with the other index precision (the 64K decode is quoted with
        # an FP8 and with a BF16 indexer), and the plain CSA layer without the HCA layer beside it
        other = "bf16" if args.index == "e4m3" else "e4m3"
        variants[f"flash64k_{other}_index"] = bench_workload("flash64k", other, True, args.steps, args.warmup, world,
                                                             device)
        variants["flash64k_csa_only"] = bench_workload("flash64k", args.index, False, args.steps, args.warmup, world,
                                                       device)
    if not args.no_extra:
        # the FP4 index QK: MXFP4 scores, 4k candidates rescored exactly in bf16
        variants["pro1m_mxfp4_index"] = bench_workload("pro1m", "mxfp4", False, args.steps, args.warmup, world, device)
    prefill = hca = None
    kv8_runs = {}
    if not args.no_extra:
        prefill = bench_prefill(max(5, min(20, args.steps // 100)), 3, device, measured_tflops())
        hca = bench_hca(args.steps, args.warmup, device, peak)
        # the same decode steps with the memory rows stored as mixed-precision entries
        for nm in ([args.workload] + (["pro1m"] if args.workload != "pro1m" else [])):
            kv8_runs[nm] = bench_workload(nm, args.index, nm == "flash64k", args.steps, args.warmup, world, device,
                                          kv8=True)
        kv8_runs["pro_hca"] = bench_hca(args.steps, args.warmup, device, peak, kv8=True)
    cpu = oracle_cfg = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:       # the oracle leg: one process, N = 1
        cpu = oracle_baseline(main_res["wl"], args.index, with_hca)
        if not args.no_extra:
            oracle_cfg = oracle_config_timings()
    if rank != 0:
        return

    def summarise(r, kv8=False):
        wl = r["wl"]
        tok = r["tokens_per_step"] * world
        steps = args.steps
        idx_gbs = r["index_bytes"] / (r["index_ms"] * 1e-3) / 1e9
        attn_gbs = r["attn_bytes"] / (r["attn_ms"] * 1e-3) / 1e9
        step_gbs = r["step_bytes"] / (r["step_ms"] * 1e-3) / 1e9
        return {
            "value": tok * steps / r["seconds"], "ms_per_step": r["step_ms"],
            "e2e": {"value": tok * steps / r["e2e_seconds"], "unit": "tokens/s",
                    "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
            "roofline": {"bound": "hbm", "kernel": ("attn_tc_kernel (sparse_attn: top-k + SWA rows, cluster merge, "
                                                    "memory rows as KV8 entries)") if kv8 else
                         ("attn_t_kernel (sparse_attn: top-k + SWA rows as the MMA's M, split over a cluster, "
                          "partials merged through L2, partial RoPE)"),
                         "achieved": attn_gbs, "peak": peak, "unit": "GB/s", "frac": attn_gbs / peak,
                         "peak_source": peak_kind + " (burst copy; the kernel is timed alone)",
                         "traffic": profiled_traffic("attn_tc_kernel_decode_prefill_hca.md", "attn.cuh",
                                                     wl.name + "_kv8") if kv8 else
                                    profiled_traffic("attn_t_kernel_decode.md", "attn_t.cuh", wl.name),
                         "bytes_per_launch": r["attn_bytes"], "avg_launch_us": r["attn_ms"] * 1e3,
                         "timing": "back-to-back launches in one CUDA graph over rotating input sets (cold in L2), "
                                   "CUDA events around the graph replays",
                         "why_this_kernel": "largest share of the step in the ncu launch list (two launches per "
                                            "step: CSA sparse_attn and HCA hca_attn)"},
            "roofline_indexer": {"bound": "hbm", "kernel": f"index_tc_kernel (csa_index_scores, {r['index']})",
                         "achieved": idx_gbs, "peak": peak, "unit": "GB/s", "frac": idx_gbs / peak,
                         "peak_source": peak_kind + " (burst copy; the kernel is timed alone)",
                         "traffic": profiled_traffic(f"index_tc_kernel_{r['index']}_decode.md", "index.cuh",
                                                     wl.name) if r["index"] in ("e4m3", "mxfp4") else None,
                         "bytes_per_launch": r["index_bytes"], "avg_launch_us": r["index_ms"] * 1e3,
                         "timing": "back-to-back launches in one CUDA graph over rotating input sets (cold in L2), "
                                   "CUDA events around the graph replays"},
            "step_roofline": {"bytes_per_step": r["step_bytes"], "achieved_gbs": step_gbs, "frac": step_gbs / peak,
                              "floor_us": r["step_bytes"] / (peak * 1e9) * 1e6},
            "indexer_keys_per_s": wl.B * wl.T * wl.N * world * steps / r["seconds"],
            "gpu_launches": r["launches"] * steps, "launches_per_step": r["launches"], "input_sets": r["sets"],
            "breakdown_us": r["breakdown"],
        }

    m = summarise(main_res)
    wl = main_res["wl"]
    line = {
        "metric": "CSA decode tokens/s (64K Flash CSA+HCA layer pair)" if with_hca else
                  "CSA decode tokens/s (1M Pro CSA layer)",
        "value": m["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": m["ms_per_step"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16+e4m3" if args.index == "e4m3" else "bf16", "data": "synthetic",
        "config": {"workload": workload_text(wl, args.index, with_hca),
                   "l2": f"{m['input_sets']} rotating input sets, > 2x L2 touched between reuses",
                   "graph": "one CUDA graph runs a step on every input set in turn, replayed; "
                            "steps % sets more by a second graph",
                   "parallelism": f"replicas x{world}"},
        "e2e": m["e2e"], "roofline": m["roofline"], "roofline_indexer": m["roofline_indexer"],
        "step_roofline": m["step_roofline"],
        "indexer_keys_per_s": m["indexer_keys_per_s"], "gpu_launches": m["gpu_launches"],
        "launches_per_step": m["launches_per_step"], "clocks": clocks,
        "breakdown_us_diagnostic": m["breakdown_us"],
    }
    if extra is not None:
        e = summarise(extra)
        line["pro1m"] = {"value": e["value"], "unit": "tokens/s", "ms_per_step": e["ms_per_step"],
                         "step_roofline": e["step_roofline"], "roofline": e["roofline"],
                         "roofline_indexer": e["roofline_indexer"], "e2e": e["e2e"],
                         "indexer_keys_per_s": e["indexer_keys_per_s"], "launches_per_step": e["launches_per_step"],
                         "breakdown_us": e["breakdown_us"]}
        line["gpu_launches"] += e["gpu_launches"]
    for nm, r in variants.items():
        e = summarise(r)
        line[nm] = {"value": e["value"], "unit": "tokens/s", "ms_per_step": e["ms_per_step"],
                    "workload": workload_text(r["wl"], r["index"], r["with_hca"]),
                    "step_roofline": e["step_roofline"], "roofline_indexer": e["roofline_indexer"], "e2e": e["e2e"],
                    "roofline": e["roofline"],
                    "launches_per_step": e["launches_per_step"], "breakdown_us": e["breakdown_us"]}
        line["gpu_launches"] += e["gpu_launches"]
    if prefill is not None:
        line["prefill"] = prefill
    if hca is not None:
        line["pro_hca"] = hca
    if kv8_runs:
        kv = {"storage": "memory rows as 608-byte entries: 448 e4m3 dims with a power-of-two scale per 64 dims, "
                         "64 bf16 RoPE dims; the step also quantises the entries its compressors produce"}
        for nm, r in kv8_runs.items():
            if nm == "pro_hca":
                kv[nm] = r
                continue
            e = summarise(r, kv8=True)
            kv[nm] = {"value": e["value"], "unit": "tokens/s", "ms_per_step": e["ms_per_step"],
                      "roofline": e["roofline"], "step_roofline": e["step_roofline"], "e2e": e["e2e"],
                      "launches_per_step": e["launches_per_step"]}
            line["gpu_launches"] += e["gpu_launches"]
        line["kv8"] = kv
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if oracle_cfg is not None:
        line["oracle_configs"] = oracle_cfg
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
