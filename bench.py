#!/usr/bin/env python
"""Benchmark of the sparse-attention index pipeline on B200.

One step = one pass of the whole hot path over one batch: index_select (block
scoring fused with the causal-masked top-k) followed by sparse_attn (paged
gather + exact online-softmax attention), both through the C ABI. The headline
workload is the decode configuration (B=32 sequences, 32768-token context,
block 64, 8 indexer heads of dim 128, top-32 blocks, 16 query heads sharing one
KV head of dim 128, paged KV with a random-permuted block table).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N>1 runs under torchrun, one rank per GPU, each rank on its own batch of 32
sequences (weak scaling: the sequences are independent, so no data-path
collective). Timing: K steps back to back, launched as CUDA graphs, over R
device replicas of the inputs that together touch more than 2.5x the L2, so
no step finds its data in L2; one pair of CUDA events on the launching
stream around the K steps, max over ranks. Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import glob
import hashlib
import json
import re
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_indexer_b200.workloads import (CONFIGS, SCAN_CONFIGS, generate,  # noqa: E402
                                                 generate_scan)

METRIC = "sparse-attn decode tokens/s (B=32, 32K ctx); prefill Mtok/s; % of roofline"
HEADLINE = "decode"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=HEADLINE, choices=sorted(CONFIGS) + ["scan"])
    ap.add_argument("--no-extra", action="store_true", help="skip the other configurations")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", action="store_true",
                    help="run the workload's step --steps times without timing or output "
                         "(for profiler captures); --config scan runs the state scan, "
                         "--persistent the one-launch decode step")
    ap.add_argument("--persistent", action="store_true")
    return ap.parse_args()


def run_profile(args):
    """The step of one workload, --steps times, nothing timed or printed but a
    status line: a small, self-contained command for ncu captures."""
    import long_context_indexer_b200 as lci
    torch.cuda.set_device(0)
    if args.config == "scan":
        cfg = SCAN_CONFIGS["scan"].replace(B=2)
        d = {k: v.cuda() for k, v in generate_scan(cfg).items()}
        for _ in range(args.steps):
            lci.gated_state_scan(d["q"], d["k"], d["v"], d["gate"], d["state"], cfg.C)
    else:
        cfg = CONFIGS[args.config]
        pipe = Pipeline(cfg, generate(cfg), torch.device("cuda", 0))
        for _ in range(args.steps):
            if args.persistent:
                pipe.step_persistent()
            else:
                pipe.step()
    torch.cuda.synchronize()
    lci.get_device_status()
    print(f"profile run: {args.config}{' persistent' if args.persistent else ''} x{args.steps} ok")
    return 0


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": 1590.0, "source": "fallback"}


# DRAM bytes (read + write) per launch of a kernel, from one ncu capture of
# it on a workload (summaries under profiles/), with the digest of the library
# sources the capture ran. Once those sources change the figure no longer
# describes the kernel and the bench reports traffic as null.
PROFILED_TRAFFIC = {
    ("decode", "index_select"): (33751808, "7c06d6f15ea82c7c"),
    ("decode", "sparse_attn"): (33816576, "7c06d6f15ea82c7c"),
    ("1m_chunk", "index_select"): (25255680, "7c06d6f15ea82c7c"),
}


def _code_only(text: str) -> str:
    """C/CUDA source with comments removed and whitespace collapsed."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def sources_digest() -> str:
    """sha256 (first 16 hex digits) over the code of the CUDA sources and the C
    header, comments and whitespace excluded."""
    files = sorted(glob.glob(os.path.join(ROOT, "long_context_indexer_b200", "csrc", "*.cu")) +
                   glob.glob(os.path.join(ROOT, "long_context_indexer_b200", "csrc", "*.cuh")) +
                   [os.path.join(ROOT, "include", "lci.h")])
    h = hashlib.sha256()
    for f in files:
        h.update(os.path.basename(f).encode())
        with open(f, encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, kernel: str):
    hit = PROFILED_TRAFFIC.get((workload, kernel))
    if hit is None or hit[1] != sources_digest():
        return None
    return hit[0]


def workload_name(cfg) -> str:
    return (f"{cfg.name} {cfg.dtype}: B={cfg.B} S={cfg.S} ctx={cfg.ctx} q_start={cfg.q_start} "
            f"block={cfg.bs} NB={cfg.NB} H_i={cfg.H_i} d_c={cfg.d_c} topk={cfg.topk} "
            f"H_q={cfg.H_q} H_kv={cfg.H_kv} hd={cfg.hd}")


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap"}

    def __init__(self, device_index: int, period_s: float = 0.001):
        self.samples, self.reasons = [], set()
        self.active = False  # sample only while a timed region runs
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[device_index]) if vis else device_index
            self._h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _sample(self):
        nv = self._nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
        r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        for bit, name in self.REASONS.items():
            if r & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            if self.active:
                try:
                    self._sample()
                except Exception:
                    return
            time.sleep(self._period)

    def __enter__(self):
        if self._nv is not None:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._nv is not None:
            self._t.join(timeout=1.0)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ the path

def packed_buffer(tensors, device, pin=False):
    """One uint8 buffer holding every tensor of `tensors` at a 256-byte aligned
    offset, and a view of it per name with that tensor's dtype and shape."""
    offs, total = {}, 0
    for k, t in tensors.items():
        offs[k] = total
        total += -(-t.numel() * t.element_size() // 256) * 256
    buf = torch.empty(max(total, 256), dtype=torch.uint8, device=device, pin_memory=pin)
    views = {k: buf[offs[k]:offs[k] + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
             for k, t in tensors.items()}
    return buf, views


class Pipeline:
    """Device-resident inputs of one workload and the two ABI calls of a step."""

    def __init__(self, cfg, w, device):
        import long_context_indexer_b200 as lci
        self.lci, self.cfg = lci, cfg
        self.host = w
        self.d = {k: v.to(device) for k, v in w.items()}
        d = self.d
        self.k_c = (torch.empty((cfg.B, cfg.NB, cfg.H_i, cfg.d_c), dtype=cfg.torch_dtype,
                                device=device) if cfg.compress else d["k_c"])
        self.bt = lci.create_block_table(d["block_table"], d["k_pool"])
        self.ids = torch.empty((cfg.B, cfg.S, cfg.topk), dtype=torch.int32, device=device)
        self.out = torch.empty_like(d["q"])
        ni = lci.index_select_workspace_size(cfg.B, cfg.S, cfg.H_i, cfg.d_c, cfg.NB, cfg.topk)
        na = lci.sparse_attn_workspace_size(cfg.B, cfg.S, cfg.H_q, cfg.topk, self.bt)
        self.ws_i = torch.zeros(max(ni, 256), dtype=torch.uint8, device=device)
        self.ws_a = torch.zeros(max(na, 256), dtype=torch.uint8, device=device)
        nd = lci.sparse_decode_workspace_size(cfg.B, cfg.S, cfg.H_i, cfg.d_c, cfg.topk, cfg.H_q,
                                              self.bt)
        self.ws_d = torch.zeros(max(nd, 256), dtype=torch.uint8, device=device)
        self.ws_p = torch.zeros(max(nd, 256), dtype=torch.uint8, device=device)
        self.one_call = cfg.S == 1 and not cfg.compress
        self.launches_per_step = (1 if cfg.compress else 0) + 2

    def clone(self):
        """A device copy of every input (same values, separate memory)."""
        other = Pipeline.__new__(Pipeline)
        other.lci, other.cfg, other.host = self.lci, self.cfg, self.host
        other.d = {k: v.clone() for k, v in self.d.items()}
        other.k_c = torch.empty_like(self.k_c) if self.cfg.compress else other.d["k_c"]
        other.bt = self.lci.create_block_table(other.d["block_table"], other.d["k_pool"])
        other.ids = torch.empty_like(self.ids)
        other.out = torch.empty_like(self.out)
        other.ws_i = torch.zeros_like(self.ws_i)
        other.ws_a = torch.zeros_like(self.ws_a)
        other.ws_d = torch.zeros_like(self.ws_d)
        other.ws_p = torch.zeros_like(self.ws_p)
        other.launches_per_step = self.launches_per_step
        other.one_call = self.one_call
        return other

    # The inputs of one decode step are the new tokens' compressed and
    # attention queries and their positions; the caches (k_c, KV pool, block
    # table) stay resident. A step returns the block ids and the output.
    E2E_INPUTS = ("q_c", "q", "ctx_len", "q_start")

    def prepare_e2e(self):
        """Stage a step's inputs in one pinned host buffer and one device buffer,
        and its results in one device buffer and one pinned host buffer
        (256-byte aligned segments), so a step moves its inputs with one copy
        and reads its results with one copy. The library calls read and write
        views of the device buffers."""
        if hasattr(self, "_d_in"):
            return
        dev = self.ids.device
        ins = {k: self.host[k] for k in self.E2E_INPUTS if k in self.host}
        self._h_in, hv = packed_buffer(ins, "cpu", pin=True)
        self._d_in, dv = packed_buffer(ins, dev)
        for k, t in ins.items():
            hv[k].copy_(t)
            dv[k].copy_(self.d[k])
            self.d[k] = dv[k]
        outs = {"ids": self.ids, "out": self.out}
        self._d_out, dvo = packed_buffer(outs, dev)
        self._h_out, _ = packed_buffer(outs, "cpu", pin=True)
        self.ids, self.out = dvo["ids"], dvo["out"]
        self._prepared = None
        if self.one_call:
            # the library's prepared decode step: the call a serving loop makes
            d, c = self.d, self.cfg
            self._prepared = self.lci.SparseDecodeStep(
                d["q_c"], self.k_c, d["ctx_len"], d["q_start"], c.topk, d["q"], d["k_pool"],
                d["v_pool"], self.bt, ids=self.ids, out=self.out, ws=self.ws_d,
                stream=torch.cuda.current_stream())
            self._prepared()
        torch.cuda.synchronize()

    def e2e_launch(self):
        if self._prepared is not None:
            self._prepared()
        else:
            self.step()


    def e2e_bytes(self):
        self.prepare_e2e()
        return {"h2d_bytes_per_step": self._h_in.numel(), "d2h_bytes_per_step": self._h_out.numel()}

    def index(self):
        d, c = self.d, self.cfg
        if c.compress:
            self.lci.block_compress(d["k_idx"], c.bs, out=self.k_c)
        self.lci.index_select(d["q_c"], self.k_c, c.bs, d["ctx_len"], d["q_start"], c.topk,
                              ids=self.ids, ws=self.ws_i)

    def attn(self):
        d, c = self.d, self.cfg
        self.lci.sparse_attn(d["q"], d["k_pool"], d["v_pool"], self.bt, self.ids, d["ctx_len"],
                             d["q_start"], out=self.out, ws=self.ws_a)

    def step_persistent(self):
        """The same decode step as one persistent launch."""
        d, c = self.d, self.cfg
        self.lci.sparse_decode(d["q_c"], self.k_c, d["ctx_len"], d["q_start"], c.topk, d["q"],
                               d["k_pool"], d["v_pool"], self.bt, ids=self.ids, out=self.out,
                               ws=self.ws_p, persistent=True)

    def step(self):
        c = self.cfg
        if self.one_call:
            # one decode step in one call: rows are attended as they are selected
            d = self.d
            self.lci.sparse_decode(d["q_c"], self.k_c, d["ctx_len"], d["q_start"], c.topk, d["q"],
                                   d["k_pool"], d["v_pool"], self.bt, ids=self.ids, out=self.out,
                                   ws=self.ws_d)
        else:
            self.index()
            self.attn()

    # Algorithmic work, from the shapes and the produced ids (outside timing):
    # every byte that must cross HBM at least once (unique k_c and KV blocks,
    # queries, ids, outputs) and the flops of the definition.
    def algorithmic(self):
        c = self.cfg
        dev = self.ids.device
        esz = 4 if c.dtype == "f32" else 2
        K = c.H_i * c.d_c
        pos = self.d["q_start"].long()[:, None] + torch.arange(c.S, device=dev)[None]
        ctx = self.d["ctx_len"].long()
        last = torch.minimum(pos, ctx[:, None] - 1)  # [B,S]
        vis = torch.where(last >= 0, torch.clamp(last // c.bs + 1, max=c.NB),
                          torch.zeros_like(last))
        rows = c.B * c.S
        kc_unique = int(vis.max(dim=1).values.sum())  # blocks of k_c read per sequence
        idx_bytes = rows * K * esz + kc_unique * K * esz + rows * c.topk * 4 + 8 * c.B
        if c.compress:
            idx_bytes += c.B * c.ctx * K * esz + c.B * c.NB * K * esz
        ids = self.ids.long()
        valid = ids >= 0
        first = ids.clamp(min=0) * c.bs
        ntok = torch.clamp(last[..., None] - first + 1, min=0, max=c.bs) * valid
        nsel = int(ntok.sum())  # (query, token) pairs attended
        used = torch.zeros((c.B, c.NB), dtype=torch.bool, device=dev)
        used.scatter_(1, ids.clamp(min=0).reshape(c.B, -1), valid.reshape(c.B, -1))
        blk_tok = torch.clamp(ctx[:, None] - torch.arange(c.NB, device=dev)[None] * c.bs, 0, c.bs)
        kv_tokens = int((blk_tok * used).sum())  # unique KV tokens gathered
        kv_bytes = kv_tokens * c.H_kv * c.hd * esz * 2 + int(used.sum()) * 4
        attn_bytes = kv_bytes + 2 * rows * c.H_q * c.hd * esz + rows * c.topk * 4 + 8 * c.B
        return {"index_bytes": idx_bytes, "attn_bytes": attn_bytes,
                "attn_flops": 4.0 * nsel * c.H_q * c.hd, "index_flops": 2.0 * int(vis.sum()) * K,
                "selected_pairs": nsel, "kv_tokens": kv_tokens}


L2_BYTES = 126 << 20


class Replicas:
    """R device copies of one workload, so that consecutive steps never find
    the previous step's data in L2 (R x accessed bytes > 2.5 x L2)."""

    def __init__(self, pipe, accessed_bytes, max_bytes=24 << 30):
        self.pipes = [pipe]
        per = sum(v.numel() * v.element_size() for v in pipe.d.values())
        want = max(3, -(-int(2.5 * L2_BYTES) // max(1, accessed_bytes)))
        want = min(want, 32, max(1, max_bytes // max(1, per)))
        for _ in range(want - 1):
            self.pipes.append(pipe.clone())
        self.R = len(self.pipes)
        self.cycle_bytes = self.R * accessed_bytes


def capture(fn_list):
    """One CUDA graph running every callable of fn_list in order."""
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for f in fn_list:
            f()
    torch.cuda.synchronize()
    return g


SAMPLER = None  # the ClockSampler of the run, active only inside time_graph


def time_graph(g, reps, warmup):
    """Device time per replay (ms): warm-up replays, then one event pair."""
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if SAMPLER is not None:
        SAMPLER.active = True
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    if SAMPLER is not None:
        SAMPLER.active = False
        try:
            SAMPLER._sample()  # at least one sample per timed region
        except Exception:
            pass
    return e0.elapsed_time(e1) / reps


E2E_PASSES = 4  # passes over the replicas in one end-to-end graph


def e2e_graph(pipes, passes=E2E_PASSES):
    """`passes` rounds over the R replicas' steps as one CUDA graph of a
    pipelined serving loop over independent batches: every step copies its
    inputs in from pinned host memory (one stream), runs the library's prepared
    decode step (another) and copies its results back to pinned host memory (a
    third), so a step's copies overlap its neighbours' kernels. Each step's
    kernels wait for its own inputs and its copy back for its kernels; a step
    that reuses a replica's buffers also waits, for its upload, until the
    previous step on that replica has computed, and for its kernels until that
    step's results have been copied back. Several passes spread the graph's
    first upload and last download over more steps."""
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    R = len(pipes)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        cap = torch.cuda.current_stream()
        start = torch.cuda.Event()
        start.record(cap)
        s_in.wait_event(start)
        s_out.wait_event(start)
        ev_comp, ev_out = [], []
        for i in range(R * passes):
            p = pipes[i % R]
            with torch.cuda.stream(s_in):
                if i >= R:
                    s_in.wait_event(ev_comp[i - R])
                p._d_in.copy_(p._h_in, non_blocking=True)
                e_in = torch.cuda.Event()
                e_in.record(s_in)
            cap.wait_event(e_in)
            if i >= R:
                cap.wait_event(ev_out[i - R])
            p._prepared(cap)
            k = torch.cuda.Event()
            k.record(cap)
            ev_comp.append(k)
            s_out.wait_event(k)
            with torch.cuda.stream(s_out):
                p._h_out.copy_(p._d_out, non_blocking=True)
                o = torch.cuda.Event()
                o.record(s_out)
            ev_out.append(o)
        done = torch.cuda.Event()
        done.record(s_out)
        cap.wait_event(done)
    torch.cuda.synchronize()
    return g


def time_e2e(pipes, steps, warmup):
    """End-to-end time (ms) of `steps` steps through the public binding, as a
    serving loop runs them: every step copies its inputs in from pinned host
    memory, runs the prepared decode step and copies its results back to pinned
    host memory. Where the step is one library call the replicas' steps are
    replayed as one pipelined CUDA graph (e2e_graph); otherwise each step is
    issued eagerly on one stream. Device time between events on the stream."""
    for p in pipes:
        p.prepare_e2e()
    R = len(pipes)
    g = e2e_graph(pipes) if all(p._prepared is not None for p in pipes) else None

    per_graph = R * E2E_PASSES

    def run(n):
        if g is not None:
            for _ in range(-(-n // per_graph)):
                g.replay()
            return
        for i in range(n):
            p = pipes[i % R]
            p._d_in.copy_(p._h_in, non_blocking=True)
            p.e2e_launch()
            p._h_out.copy_(p._d_out, non_blocking=True)

    run(max(warmup, R))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if SAMPLER is not None:
        SAMPLER.active = True
    e0.record()
    run(steps)
    e1.record()
    torch.cuda.synchronize()
    if SAMPLER is not None:
        SAMPLER.active = False
    n_done = -(-steps // per_graph) * per_graph if g is not None else steps
    return e0.elapsed_time(e1) * steps / n_done


def measure(cfg, steps, warmup, device, rank=0, seed_offset=0, with_e2e=True):
    """Back-to-back steps over rotating replicas, launched as CUDA graphs.

    Per-step device times (ms) of the whole step, of the index_select launch
    alone and of the sparse_attn launch alone, and of the end-to-end step."""
    w = generate(cfg, seed=cfg.seed + seed_offset)
    pipe = Pipeline(cfg, w, device)
    pipe.step()  # kernel attributes and tensor maps are set up before capture
    torch.cuda.synchronize()
    alg = pipe.algorithmic()
    reps = Replicas(pipe, alg["index_bytes"] + alg["attn_bytes"])
    for p in reps.pipes:
        p.step()
    torch.cuda.synchronize()
    R = reps.R
    n_rep = max(1, -(-steps // R))
    warm = max(1, -(-warmup // R))
    g_step = capture([p.step for p in reps.pipes])
    g_idx = capture([p.index for p in reps.pipes])
    g_att = capture([p.attn for p in reps.pipes])
    t_step = time_graph(g_step, n_rep, warm) / R
    t_idx = time_graph(g_idx, n_rep, warm) / R
    t_att = time_graph(g_att, n_rep, warm) / R
    t_pers = None
    if pipe.one_call and cfg.H_i * cfg.d_c == 1024 and cfg.dtype == "bf16":
        for p in reps.pipes:
            p.step_persistent()
        g_pers = capture([p.step_persistent for p in reps.pipes])
        t_pers = time_graph(g_pers, n_rep, warm) / R
        del g_pers
    res = {"pipe": pipe, "t_index_ms": t_idx, "t_attn_ms": t_att, "t_step_ms": t_step,
           "t_persistent_ms": t_pers,
           "t_total_ms": t_step * steps, "alg": alg, "replicas": R,
           "cycle_mb": reps.cycle_bytes / 2**20, "launches": pipe.launches_per_step * steps}
    if with_e2e:
        res["e2e_total_ms"] = time_e2e(reps.pipes, steps, warmup)
        res["e2e_bytes"] = pipe.e2e_bytes()
    del g_step, g_idx, g_att, reps
    return res


def measure_scan(cfg, steps, warmup, device, pk):
    """The chunked gated state scan on its own workload: device time per launch
    (one event pair around `steps` back-to-back launches; its 3 GB of inputs
    and outputs exceed L2 many times), against the HBM roofline of its
    algorithmic bytes (q, k, v read once, out written once in fp32, gates and
    the state read and written once)."""
    import long_context_indexer_b200 as lci
    w = generate_scan(cfg)
    d = {k: v.to(device) for k, v in w.items()}
    out = torch.empty((cfg.B, cfg.T, cfg.H, cfg.d), dtype=torch.float32, device=device)
    st = torch.empty_like(d["state"])

    def launch():
        lci.gated_state_scan(d["q"], d["k"], d["v"], d["gate"], d["state"], cfg.C, out=out,
                             state_out=st)

    for _ in range(warmup):
        launch()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        launch()
    e1.record()
    torch.cuda.synchronize()
    lci.get_device_status()
    ms = e0.elapsed_time(e1) / steps
    tokens = cfg.B * cfg.T * cfg.H
    nbytes = tokens * cfg.d * (3 * 2 + 4) + 2 * cfg.B * cfg.H * cfg.d * cfg.d * 4 + \
        cfg.B * cfg.H * cfg.nchunks * 4
    flops = 4.0 * tokens * cfg.d * cfg.d
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": f"{cfg.name}: B={cfg.B} T={cfg.T} H={cfg.H} dk=dv={cfg.d} chunk={cfg.C}",
            "ms": ms, "bytes": nbytes, "achieved_gbs": gbs, "frac_hbm": gbs / pk["hbm_gbs"],
            "tflops": flops / (ms * 1e-3) / 1e12, "tokens_per_s": cfg.B * cfg.T / (ms * 1e-3)}


def config_entry(cfg, r, pk):
    """Per-workload figures of one measure() result: times, rates, and each
    kernel's rate as a fraction of the measured HBM and bf16 peaks."""
    a = r["alg"]
    rows = cfg.B * cfg.S
    ti, ta = r["t_index_ms"] * 1e-3, r["t_attn_ms"] * 1e-3
    e = {
        "ms_step": r["t_step_ms"], "ms_index": r["t_index_ms"], "ms_attn": r["t_attn_ms"],
        "ms_step_one_launch": r.get("t_persistent_ms"),
        "tokens_per_s": rows / (r["t_step_ms"] * 1e-3),
        "index_gbs": a["index_bytes"] / ti / 1e9,
        "index_tflops": a["index_flops"] / ti / 1e12,
        "attn_gbs": a["attn_bytes"] / ta / 1e9,
        "attn_tflops": a["attn_flops"] / ta / 1e12,
    }
    e["index_frac_hbm"] = e["index_gbs"] / pk["hbm_gbs"]
    e["index_frac_bf16"] = e["index_tflops"] / pk["bf16_tflops"]
    e["attn_frac_hbm"] = e["attn_gbs"] / pk["hbm_gbs"]
    e["attn_frac_bf16"] = e["attn_tflops"] / pk["bf16_tflops"]
    return e


# ------------------------------------------------------------------ CPU oracle

def oracle_throughput(cfg, min_seconds=10.0, max_rows=None, w=None):
    """Oracle (fp64 C, OpenMP) tokens/s on a bounded sample of the workload."""
    import oracle
    w = generate(cfg) if w is None else w
    rows_all = cfg.B * cfg.S
    n = rows_all if max_rows is None else min(rows_all, max_rows)
    rows = list(range(n))
    scale = 1.0 / math.sqrt(cfg.hd)
    k_c = oracle.block_compress(w["k_idx"], cfg.bs).to(cfg.torch_dtype) if cfg.compress else w["k_c"]
    done, t0 = 0, time.perf_counter()
    while True:
        ids = oracle.index_select(w["q_c"], k_c, cfg.bs, w["ctx_len"], w["q_start"], cfg.topk,
                                  rows=rows)
        oracle.sparse_attn(w["q"], w["k_pool"], w["v_pool"], w["block_table"], ids, w["ctx_len"],
                           w["q_start"], scale, rows=rows)
        done += n
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    return {"value": done / el, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} of {rows_all} query rows of the {cfg.name} workload, repeated "
                      f"{done // n}x over {el:.1f} s (index_select + sparse_attn, fp64)"}


# ------------------------------------------------------------------ main

def shard_seed_offset(rank: int) -> int:
    """Each rank draws its own batch of sequences (weak scaling, no exchange)."""
    return 1000 * rank


def reduce_max_ms(values, device, world: int):
    """Max over ranks of each timing (ms); identity on one rank."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(world: int, rows_per_rank: int, steps: int, total_ms: float) -> float:
    """Whole-job tokens/s: every rank's query rows over the slowest rank's time."""
    return world * rows_per_rank * steps / (total_ms / 1e3)


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def run_reference(args):
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return 0
    cfg = CONFIGS[args.config]
    w = generate(cfg)
    per_step = []
    for i in range(args.warmup + args.steps):
        r = oracle_throughput(cfg, min_seconds=0.0, max_rows=4, w=w)
        if i >= args.warmup:
            per_step.append(r)
    rows = sum(4 for _ in per_step)
    tok_s = statistics.median(r["value"] for r in per_step)
    ms = 1000.0 * min(4, cfg.B * cfg.S) / tok_s
    line = {"impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": workload_name(cfg), "sample_rows_per_step": 4},
            "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": per_step[0]["cores"],
                             "kind": "oracle",
                             "sample": f"4 of {cfg.B * cfg.S} query rows per step, {rows} rows"},
            "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.profile:
        return run_profile(args)
    if args.config == "scan":
        print("bench.py: --config scan is for --profile runs; the scan is measured in every "
              "default run (state_scan in the JSON line)", file=sys.stderr)
        return 2
    if args.impl == "reference":
        return run_reference(args)
    world, rank, local = dist_setup(args)
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    import long_context_indexer_b200 as lci
    lci.load_library()
    cfg = CONFIGS[args.config]
    pk = peaks()

    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    global SAMPLER
    with ClockSampler(local) as clk:
        SAMPLER = clk
        res = measure(cfg, args.steps, args.warmup, device, rank,
                      seed_offset=shard_seed_offset(rank))
        SAMPLER = None
    torch.cuda.synchronize()
    lci.get_device_status()
    if world > 1:
        dist.barrier()
    t_total, e_total = reduce_max_ms([res["t_total_ms"], res["e2e_total_ms"]], device, world)
    value = job_throughput(world, cfg.B * cfg.S, args.steps, t_total)
    e2e_value = job_throughput(world, cfg.B * cfg.S, args.steps, e_total)

    alg = res["alg"]
    one_launch = res["pipe"].launches_per_step == 1
    if one_launch:
        # the step is one persistent kernel: it is the dominant (only) kernel
        kernels = {"sparse_decode": {"ms": res["t_step_ms"],
                                     "bytes": alg["index_bytes"] + alg["attn_bytes"]}}
    else:
        kernels = {
            "index_select": {"ms": res["t_index_ms"], "bytes": alg["index_bytes"]},
            "sparse_attn": {"ms": res["t_attn_ms"], "bytes": alg["attn_bytes"]},
        }
    dom = max(kernels, key=lambda k: kernels[k]["ms"])
    ach = kernels[dom]["bytes"] / (kernels[dom]["ms"] * 1e-3) / 1e9
    roof = {"bound": "hbm", "kernel": dom, "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": ach / pk["hbm_gbs"], "traffic": profiled_traffic(cfg.name, dom),
            "peak_source": pk["source"]}
    step_bytes = alg["index_bytes"] + alg["attn_bytes"]
    step_gbs = step_bytes / (res["t_step_ms"] * 1e-3) / 1e9

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": workload_name(cfg), "global_batch": world * cfg.B,
                   "seq_len": cfg.ctx, "parallelism": f"dp{world}" if world > 1 else "single",
                   "l2": f"inputs larger than L2: {res['replicas']} device replicas rotated "
                         f"({res['cycle_mb']:.0f} MiB touched per cycle vs 126 MiB L2); steps "
                         f"back to back in CUDA graphs, one event pair"},
        "roofline": roof,
        "step_roofline": {"bytes": step_bytes, "achieved_gbs": step_gbs,
                          "frac": step_gbs / pk["hbm_gbs"]},
        "kernels_ms": {k: v["ms"] for k, v in kernels.items()},
        "itemized_ms": {"index_select alone": res["t_index_ms"],
                        "sparse_attn alone": res["t_attn_ms"],
                        "one-launch persistent step": res["t_persistent_ms"]},
        "e2e": {"value": e2e_value, "unit": "tokens/s", **res["e2e_bytes"]},
        "gpu_launches": res["launches"],
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_throughput(cfg, min_seconds=10.0, w=res["pipe"].host)
    if rank == 0 and world == 1 and not args.no_extra:
        extra = {}
        for name in ("prefill", "long", "1m_decode", "1m_chunk", "tiny"):
            if name == args.config:
                continue
            c = CONFIGS[name]
            r = measure(c, max(5, args.steps // 5), 3, device, with_e2e=False)
            extra[name] = config_entry(c, r, pk)
            del r
            torch.cuda.empty_cache()
        line["other_configs"] = extra
        line["state_scan"] = measure_scan(SCAN_CONFIGS["scan"], max(5, args.steps // 5), 3, device,
                                          pk)
        torch.cuda.empty_cache()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
