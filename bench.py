#!/usr/bin/env python
"""Benchmark: ProxyAttn-style block-sparse prefill attention on B200.

One step = one pass of the whole path over one attention layer of synthetic
input already resident in HBM: head pooling -> fused proxy block scores ->
mask (last-block head mass, ranking, per-head budget) -> block-sparse
attention, each stage called through the C ABI (libpa.so) on the current
stream with CUDA events between stages.

Default workload: the Llama-3.1-8B layer at 128K tokens (batch 1, 32 q heads,
8 KV heads, head_dim 128, G = 1, gamma = 0.95).  The printed JSON line carries
ms per layer (estimate + sparse), effective TFLOP/s over the visited blocks,
per-stage times, sparsity, the speedup over the same kernel with every causal
block selected, the attention kernel's roofline, an end-to-end number through
the public API with host buffers, SM clocks sampled during the timed region
and the CPU oracle's time on a bounded sample.

Multi-GPU (torchrun): replicas only -- every rank runs its own independent
layer (the path needs no exchange); the step time is the max over ranks.

`--impl reference` times the CPU oracle (the only reference there is) on a
bounded sample of the same workload each step, on the host cores.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from block_sparse_attention_pa_b200 import synth  # noqa: E402

METRIC = ("prefill attention ms/layer (estimate + sparse) and effective TFLOP/s at 128K, 1×B200")
MODES = {"dynamic": 0, "fixed": 1, "all": 2}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama8b_n128k",
                    choices=sorted(synth.WORKLOADS) + sorted(synth.EXTRA_WORKLOADS))
    ap.add_argument("--groups", type=int, default=None, help="proxy groups G (default: the workload's)")
    ap.add_argument("--mode", choices=sorted(MODES), default="dynamic")
    ap.add_argument("--gamma", type=float, default=None)
    ap.add_argument("--frac", type=int, default=100, help="fixed budget in per mille of causal blocks")
    ap.add_argument("--score-stride", type=int, default=1, choices=[1, 2, 4, 8],
                    help="query-row stride of the proxy block scores (1: every row)")
    ap.add_argument("--non-causal", action="store_true",
                    help="every query attends every key (bidirectional attention)")
    ap.add_argument("--estimator", choices=["proxy", "xattn"], default="proxy",
                    help="mask estimator: ProxyAttn (pooled proxy scores + per-head budget) or XAttention "
                         "(antidiagonal strided scores + find_blocks, one list per head)")
    ap.add_argument("--xattn-stride", type=int, default=8, choices=[4, 8, 16])
    ap.add_argument("--tau", type=float, default=0.9, help="XAttention find_blocks threshold")
    ap.add_argument("--skip-threshold", type=float, default=0.0,
                    help="running-max block skip in the attention: lambda in [0, 1] (0: off)")
    ap.add_argument("--gen", choices=["literal", "logit"], default="literal",
                    help="input generator: the workload's recipe, or the labelled extra with the direction "
                         "weight in logit units (2 d^(1/4); per-head budgets then differ)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the extra configurations (the 128K layer at G = 4, fixed 10 %%, logit units; "
                         "the 32K, Qwen 64K and 256K workloads)")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons of this GPU."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int):
        self.lines = []
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            sel = str(device_index)
        self.cmd = ["nvidia-smi", "-i", sel, "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active",
                    "--format=csv,noheader,nounits", "-lms", "100"]

    def start(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 4:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
                mask = int(parts[3], 16)
            except ValueError:
                continue
            for bit, name in self.REASONS.items():
                if mask & bit:
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# Clock records the timing rules reject: a hardware or thermal slowdown, or an
# SM clock held well below its maximum with no power-cap reason (a clock lock
# left by an earlier user of the GPU).
BAD_CLOCK_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def clocks_rejected(clocks) -> bool:
    if not clocks:
        return False
    if any(r in clocks["reasons"] for r in BAD_CLOCK_REASONS):
        return True
    return clocks["sm_mhz"] < 0.75 * clocks["sm_max_mhz"] and "sw_power_cap" not in clocks["reasons"]


def agree_any(flag: bool, device, dist_on: bool) -> bool:
    """True on every rank if it is true on any (so that all ranks take the same
    collective steps afterwards)."""
    if not dist_on:
        return flag
    t = torch.tensor([1.0 if flag else 0.0], device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.item() > 0


# ----------------------------------------------------------- the pipeline
class Pipeline:
    """Pre-allocated buffers and ctypes arguments for one layer, so that a step is
    four C-ABI calls with CUDA events between them."""

    def __init__(self, q, k, v, G, mode, gamma, frac, stride=1, skip=0.0, proxies=True, causal=True):
        import block_sparse_attention_pa_b200 as pa
        self.pa = pa
        self.L = pa.lib()
        self.q, self.k, self.v = q, k, v
        B, N, H, d = q.shape
        self.B, self.N, self.H, self.d, self.G = B, N, H, d, G
        self.nb = N // 128
        self.shape = pa.make_shape(q, k, G, causal)
        self.causal = causal
        self.budget = pa.make_budget(mode, gamma, frac, stride, skip)
        self.mode = mode
        self.stride = stride
        self.skip = skip
        self.skipped = None  # uint8 [B, H, T] when counting skipped blocks
        dev = q.device
        pn = N if proxies else 128  # the XAttention pipeline needs no proxies
        self.qp = torch.empty(B, G, pn // stride, d, device=dev, dtype=torch.bfloat16)
        self.kp = torch.empty(B, G, pn, d, device=dev, dtype=torch.bfloat16)
        T = pa.rows_total(self.nb, causal)
        self.T = T
        self.scores = torch.empty(B, G, T, device=dev, dtype=torch.float32)
        self.mask = pa.Mask.empty(self.shape, dev, mode == 0)
        self.bufs = self.mask.bufs()
        self.ws = torch.empty(max(pa.workspace_size(self.shape, self.budget), 256) if proxies else 256, device=dev,
                              dtype=torch.uint8)
        self.o = torch.empty_like(q)
        self.qs, self.ks, self.vs, self.os_ = (pa._strides(t) for t in (q, k, v, self.o))
        self.scale = 1.0 / math.sqrt(d)
        self.launches_per_step = 5 + (2 if mode == 0 else 0)  # pool, scores, [mass, combine], rank, budget, attn

    def step(self, ev=None):
        pa, L, st = self.pa, self.L, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        sh, bu = ctypes.byref(self.shape), ctypes.byref(self.budget)
        if ev: ev[0].record()
        pa._check(L.pa_pool_heads_strided(sh, self.stride, self.q.data_ptr(), self.qs, self.k.data_ptr(), self.ks,
                                          self.qp.data_ptr(), self.kp.data_ptr(), st))
        if ev: ev[1].record()
        pa._check(L.pa_block_scores_strided(sh, self.stride, self.qp.data_ptr(), self.kp.data_ptr(),
                                            self.scores.data_ptr(), st))
        if ev: ev[2].record()
        pa._check(L.pa_build_mask(sh, bu, self.scores.data_ptr(), self.q.data_ptr(), self.qs, self.k.data_ptr(),
                                  self.ks, ctypes.byref(self.bufs), self.ws.data_ptr(), self.ws.numel(), st))
        if ev: ev[3].record()
        self.attend(st)
        if ev: ev[4].record()

    def attend(self, st):
        pa, L = self.pa, self.L
        sh = ctypes.byref(self.shape)
        if self.skip > 0.0:
            pa._check(L.pa_block_sparse_attn_skip(sh, self.q.data_ptr(), self.qs, self.k.data_ptr(), self.ks,
                                                  self.v.data_ptr(), self.vs, self.mask.rank.data_ptr(),
                                                  self.mask.cnt.data_ptr(), self.scale, self.skip, self.o.data_ptr(),
                                                  self.os_, None,
                                                  self.skipped.data_ptr() if self.skipped is not None else None,
                                                  st))
        else:
            pa._check(L.pa_block_sparse_attn(sh, self.q.data_ptr(), self.qs, self.k.data_ptr(), self.ks,
                                             self.v.data_ptr(), self.vs, self.mask.rank.data_ptr(),
                                             self.mask.cnt.data_ptr(), self.scale, self.o.data_ptr(), self.os_, None,
                                             st))

    def visited(self):
        """(visited blocks, algorithmic attention FLOPs with the diagonal tile
        counted in full, exact causal FLOPs)."""
        v = int(self.mask.cnt.sum().item())
        ndiag = self.B * self.H * self.nb
        per = 4 * 128 * 128 * self.d
        if not self.causal:
            return v, v * per, v * per
        exact = (v - ndiag) * per + ndiag * 4 * self.d * (128 * 129 // 2)
        return v, v * per, exact

    def count_skipped(self) -> int:
        """One more (untimed) step with a zeroed map of skipped blocks."""
        if self.skip <= 0.0:
            return 0
        self.skipped = torch.zeros(self.B, self.H, self.T, device=self.q.device, dtype=torch.uint8)
        self.step()
        torch.cuda.synchronize()
        n = int(self.skipped.sum().item())
        self.skipped = None
        return n


class XPipeline(Pipeline):
    """The XAttention estimator in place of the ProxyAttn one: a step is
    pa_xattn_mask (strided antidiagonal GEMM + selection) then the same
    attention call with one list per head."""

    def __init__(self, q, k, v, S, tau, skip=0.0, causal=True):
        import block_sparse_attention_pa_b200 as pa
        B, N, H, d = q.shape
        super().__init__(q, k, v, H, 1, 0.0, 1000, 1, skip, proxies=False, causal=causal)
        self.S, self.tau = S, tau
        self.xws = torch.empty(max(int(self.L.pa_xattn_workspace_size(ctypes.byref(self.shape), S)), 256),
                               device=q.device, dtype=torch.uint8)
        self.launches_per_step = 3  # xattn gemm, select, attn

    def step(self, ev=None):
        pa, L, st = self.pa, self.L, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        sh = ctypes.byref(self.shape)
        if ev: ev[0].record()
        if ev: ev[1].record()
        pa._check(L.pa_xattn_mask(sh, self.S, self.tau, self.q.data_ptr(), self.qs, self.k.data_ptr(), self.ks,
                                  self.mask.rank.data_ptr(), self.mask.cnt.data_ptr(), None, self.xws.data_ptr(),
                                  self.xws.numel(), st))
        if ev: ev[2].record()
        if ev: ev[3].record()
        self.attend(st)
        if ev: ev[4].record()


def selected_blocks(pipe) -> torch.Tensor:
    """Bool [B, H, T]: entry tri(qb)+kb is set when head h visits KV block kb
    in query block qb (the first cnt entries of its group's ranked list)."""
    B, H, G, nb, T = pipe.B, pipe.H, pipe.G, pipe.nb, pipe.T
    dev = pipe.mask.rank.device
    pos = torch.arange(T, device=dev)
    starts = torch.arange(nb, device=dev) * (torch.arange(nb, device=dev) + 1) // 2
    row = torch.searchsorted(starts, pos, right=True) - 1
    t = pos - starts[row]
    grp = torch.arange(H, device=dev) * G // H
    rank_h = pipe.mask.rank.long()[:, grp]                      # [B, H, T]
    inlist = t[None, None] < pipe.mask.cnt.long()[:, :, row]    # [B, H, T]
    sel = torch.zeros(B, H, T, dtype=torch.bool, device=dev)
    sel.scatter_(2, starts[row][None, None] + rank_h, inlist)
    return sel


def time_graph(pipe, steps, device, dist_on):
    """ms per layer of `steps` replays of a CUDA graph of one pipeline step."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        pipe.step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        pipe.step()
    g.replay()
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        g.replay()
    e.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(s.elapsed_time(e), device) / steps
    del g
    warm = input_bytes(pipe) <= 2 * L2_BYTES
    return {"ms_per_step": ms, "replays": steps,
            "l2": "back-to-back replays, inputs L2-resident" if warm else "inputs larger than L2"}


def max_over_ranks(value: float, device) -> float:
    """The max of a per-rank time over all ranks (the job's time); the value
    itself without a process group."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def per_layer(ms_step: float, world: int) -> float:
    """Replicas: every rank runs one layer per step, so the job processes
    `world` layers in the (max-over-ranks) step time."""
    return ms_step / world


L2_BYTES = 126 * 1024 * 1024


def input_bytes(pipe) -> int:
    return sum(t.numel() * t.element_size() for t in (pipe.q, pipe.k, pipe.v))


def time_pipeline(pipe, steps, warmup, dist_on, sampler=None):
    """Mean per-stage times and the total of `steps` steps, each step timed
    between its own first and last event (so an L2 flush between steps is
    not counted)."""
    flush = None
    if input_bytes(pipe) <= 2 * L2_BYTES:
        flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=pipe.q.device)
    for _ in range(warmup):
        pipe.step()
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    if sampler:
        sampler.start()
        time.sleep(0.3)
    torch.cuda.synchronize()
    for i in range(steps):
        if flush is not None:
            flush.fill_(i & 0xFF)
        pipe.step(evs[i])
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    if dist_on:
        torch.distributed.barrier()
    total = sum(e[0].elapsed_time(e[4]) for e in evs)
    stages = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(4)] for e in evs])
    return total, stages.mean(0), clocks


# Dense bf16 tcgen05 rate of one SM: 4096 multiply-adds per clock (a
# 128x128x16 MMA in 64 cycles, measured by an in-bounds microbenchmark).
TENSOR_FLOP_PER_CLK_SM = 8192


def tensor_busy(flops: float, ms: float, clocks, device):
    """FLOPs of a launch over what the tensor pipes of every SM can do in its
    duration at the median SM clock sampled in the timed region (None without
    a clock record)."""
    if not clocks or not clocks.get("sm_mhz"):
        return None
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    return flops / (TENSOR_FLOP_PER_CLK_SM * sms * ms * 1e-3 * clocks["sm_mhz"] * 1e6)


def sources_sha256(source_files) -> str:
    h = hashlib.sha256()
    for s in source_files:
        with open(os.path.join(ROOT, s), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def counters_for(kernel_key: str, source_files, path=None):
    """DRAM bytes of a kernel from a committed ncu summary, if the kernel's
    sources still hash to what was profiled; else None."""
    p = path or os.path.join(ROOT, "profiles", "counters.json")
    try:
        with open(p) as f:
            c = json.load(f)[kernel_key]
    except Exception:
        return None
    if sources_sha256(source_files) != c.get("source_sha256"):
        return None
    return c


def traffic_for(ctr, w, G, mode, gamma, stride=1, skip=0.0):
    """DRAM bytes per launch from the committed capture, only for the exact
    workload and budget it was taken on (traffic does not scale linearly)."""
    if not ctr:
        return None
    same = (ctr.get("workload") == w.name and ctr.get("groups") == G and
            ctr.get("mode") == {0: "dynamic", 1: "fixed", 2: "all"}[mode] and
            (mode != 0 or abs(ctr.get("gamma", -1) - gamma) < 1e-9) and
            ctr.get("score_stride", 1) == stride and ctr.get("skip_threshold", 0.0) == skip)
    return float(ctr["dram_bytes"]) if same else None


ATTN_SOURCES = ["block_sparse_attention_pa_b200/csrc/attn.cuh", "block_sparse_attention_pa_b200/csrc/sm100.cuh"]


# ------------------------------------------------------------ CPU oracle
ORACLE_POOL_TOKENS = 8192      # o1 and o3 run on this token prefix
ORACLE_SCORE_TILES = 64        # o2 tiles of the prefix's last query block (per group)
ORACLE_ATTN_BLOCKS = 1536      # o5 items are drawn until they visit this many blocks


def oracle_estimate(x, w: synth.Workload, G, mode, gamma, frac, seed=0, stride=1, skip=0.0):
    """Time the CPU oracle on a bounded sample of one layer and extrapolate to
    ms per layer.  The CPU-baseline leg and every step of the reference arm
    take the same sample (only the seed of the attention items changes), and
    every stage's sample keeps all the oracle's threads busy.  x: CPU bf16
    tensors.  Returns (ms_per_layer, per-stage seconds, threads used per stage,
    description of the sample)."""
    import oracle
    threads = oracle.num_threads()
    rng = np.random.default_rng(seed)
    q, k, v = x["q"], x["k"], x["v"]
    B, N, H, d = q.shape
    Hkv = k.shape[2]
    nb = N // 128
    T = nb * (nb + 1) // 2
    npre = min(N, ORACLE_POOL_TOKENS)
    det, used = {}, {}
    # o1 pool on the first npre tokens (parallel over tokens)
    t0 = time.perf_counter()
    _, _, qpb, kpb = oracle.pool(q[:, :npre], k[:, :npre], G)
    det["pool_s"] = (time.perf_counter() - t0) * N / npre
    used["pool"] = min(threads, B * npre)
    # o2 block scores of tiles of the prefix's last query block (parallel over tiles)
    nbp = npre // 128
    kbs = np.linspace(0, nbp - 1, min(ORACLE_SCORE_TILES, nbp)).astype(int)
    tiles = [(0, g, nbp - 1, int(kb)) for g in range(G) for kb in kbs]
    t0 = time.perf_counter()
    last = oracle.block_score_tiles(qpb, kpb, tiles, stride=stride)
    det["scores_s"] = (time.perf_counter() - t0) * (B * G * T) / len(tiles)
    used["scores"] = min(threads, len(tiles))
    # o3 head mass (parallel over heads): whole GQA groups of heads, at least
    # one head per thread, on the last query block of the npre-token prefix;
    # its cost grows with the keys each row reads, i.e. linearly in N
    per = H // Hkv
    mass_heads = min(H, per * max(1, -(-threads // per)))
    hk = mass_heads // per
    t0 = time.perf_counter()
    mass_s = oracle.head_mass(q[:, :npre, :mass_heads].contiguous(), k[:, :npre, :hk].contiguous())
    det["mass_s"] = (time.perf_counter() - t0) * (H / mass_heads) * (N / npre) if mode == 0 else 0.0
    used["mass"] = min(threads, B * mass_heads)
    # o4 ranking over the full [B, G, T] array (seeded fill; the sampled tiles real)
    scores = rng.standard_normal((B, G, T))
    if nbp == nb:
        for (b, g, qb, kb), sc in zip(tiles, last):
            scores[b, g, T - nb + kb] = sc
    t0 = time.perf_counter()
    rank = oracle.rank(scores, nb)
    det["rank_s"] = time.perf_counter() - t0
    used["rank"] = min(threads, B * G * nb)
    # budget (a plain loop) with the sampled heads' masses repeated over every
    # head and spread from the prefix's nbp blocks over all nb (block kb takes
    # an equal share of prefix block kb * nbp // nb), so that the visited-block
    # count the attention is extrapolated to follows the sampled heads' budgets
    ms_all = np.tile(mass_s, (1, -(-H // mass_heads), 1))[:, :H]
    src = np.arange(nb) * nbp // nb
    mass = ms_all[:, :, src] / np.bincount(src, minlength=nbp)[src]
    t0 = time.perf_counter()
    _, cnt = oracle.budget(rank, mass if mode == 0 else None, H, G, nb, mode, float(np.float32(gamma)), frac)
    det["budget_s"] = time.perf_counter() - t0
    used["budget"] = 1
    # o5 sparse attention on random (b, h, qb) items (parallel over items x
    # rows), extrapolated per visited block
    items, blocks = [], 0
    if int(cnt.sum()) <= ORACLE_ATTN_BLOCKS:  # a small layer: every item once
        items = [(b, h, qb) for b in range(B) for h in range(H) for qb in range(nb)]
        blocks = int(cnt.sum())
    else:
        while blocks < ORACLE_ATTN_BLOCKS:
            it = (int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(nb)))
            if it not in items:
                items.append(it)
                blocks += int(cnt[it])
    t0 = time.perf_counter()
    if skip > 0.0:
        oracle.sparse_attn_skip(q, k, v, rank, cnt, G, items, skip)
    else:
        oracle.sparse_attn(q, k, v, rank, cnt, G, items)
    dt = time.perf_counter() - t0
    det["attn_s"] = dt * float(cnt.sum()) / max(blocks, 1)
    used["attn"] = min(threads, len(items) * 128)
    sample = (f"pool of {npre}/{N} tokens; scores of {len(tiles)}/{B * G * T} tiles; head mass of "
              f"{mass_heads}/{H} heads over the last query block of a {npre}-token prefix; full rank+budget; "
              f"attention of {len(items)} random (b,h,qb) items ({blocks} of {int(cnt.sum())} visited blocks); "
              f"each stage extrapolated linearly (tokens, tiles, heads x keys, visited blocks)")
    return sum(det.values()) * 1e3, det, used, sample


def cpu_model() -> str:
    """The host CPU's model name (for the oracle baseline's record)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args, w, G, mode, gamma, frac):
    """The reference arm: the CPU oracle, timed on the host cores, one bounded
    sample of the layer per step (the same sample as the CPU-baseline leg)."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    import oracle
    x = synth.make_inputs(w, device="cpu")
    vals = []
    for i in range(args.warmup + args.steps):
        ms, det, used, sample = oracle_estimate(x, w, G, mode, gamma, frac, seed=i,
                                                stride=args.score_stride, skip=args.skip_threshold)
        if i >= args.warmup:
            vals.append(ms)
    v = statistics.mean(vals)
    cores = oracle.num_threads()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "ms/layer", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": v, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "extrapolated": True,
            "config": line_config(args, w, G, mode, gamma, frac, world),
            "cpu_baseline": {"value": v, "unit": "ms/layer", "cores": cores, "kind": "oracle",
                             "cpu_model": cpu_model(), "sample": sample, "threads_used": used,
                             "extrapolated": True,
                             "note": "value extrapolated from a bounded sample of the layer, so a step's "
                                     "wall time is not the value"},
            "e2e": {"value": v, "unit": "ms/layer", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(w, G, mode, gamma, frac, stride=1, skip=0.0):
    budget = {0: f"dynamic gamma={gamma}", 1: f"fixed {frac / 10:.1f}% of causal blocks", 2: "all causal blocks"}[mode]
    return {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "q_heads": w.num_q_heads,
            "kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "groups": G, "budget": budget, "block": 128,
            "score_stride": stride, "skip_threshold": skip,
            "l2": "inputs larger than L2 (q+k+v per layer > 2 x 126 MB), no flush"}


def line_config(args, w, G, mode, gamma, frac, world):
    """The bench line's `config`, the same for both arms (the reference arm
    names the workload its samples come from)."""
    causal = not args.non_causal
    l2 = ("inputs larger than L2 (q+k+v per layer > 2 x 126 MB), no flush"
          if w.batch * w.seqlen * (w.num_q_heads + 2 * w.num_kv_heads) * w.head_dim * 2 > 2 * L2_BYTES else
          "L2 flushed between timed steps (a 512 MiB buffer written outside the timed events)")
    if args.estimator == "xattn":
        cfg = config_of(w, w.num_q_heads, 1, 0.0, 1000, 1, args.skip_threshold) | {
            "groups": w.num_q_heads, "budget": f"XAttention find_blocks tau={args.tau}",
            "estimator": f"xattn antidiagonal stride {args.xattn_stride}"}
    else:
        cfg = config_of(w, G, mode, gamma, frac, args.score_stride, args.skip_threshold)
    return cfg | {"parallelism": f"replicas x{world}", "causal": causal, "l2": l2}


# ------------------------------------------------------------------- main
def resolve_workload(args) -> synth.Workload:
    """The workload the flags name; --gen logit is a labelled extra, named
    apart from the workload it modifies."""
    w = {**synth.WORKLOADS, **synth.EXTRA_WORKLOADS}[args.workload]
    if args.gen == "logit":
        w = w.replace(name=w.name + "_logit", logit_units=True)
    return w


def main():
    args = parse_args()
    w = resolve_workload(args)
    G = args.groups or w.num_groups
    mode = MODES[args.mode]
    gamma = args.gamma if args.gamma is not None else w.gamma
    frac = args.frac
    if args.impl == "reference":
        run_reference(args, w, G, mode, gamma, frac)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist_on = world > 1
    torch.cuda.set_device(local)
    if dist_on:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    import block_sparse_attention_pa_b200 as pa
    pa.lib()  # fails loudly when libpa.so is missing

    x = synth.make_inputs(w, device=f"cuda:{local}", seed=w.seed + rank)
    q, k, v = x["q"], x["k"], x["v"]
    stride = args.score_stride
    skip = args.skip_threshold
    xattn = args.estimator == "xattn"
    if xattn:
        pipe = XPipeline(q, k, v, args.xattn_stride, args.tau, skip, causal=not args.non_causal)
    else:
        pipe = Pipeline(q, k, v, G, mode, gamma, frac, stride, skip, causal=not args.non_causal)
    sampler = None if args.no_clocks else ClockSampler(local)
    total_ms, stages, clocks = time_pipeline(pipe, args.steps, args.warmup, dist_on, sampler)
    rejected = None
    if agree_any(clocks_rejected(clocks), q.device, dist_on):
        # measured once more; the line carries the rejected run's clock record
        rejected = clocks
        sampler = None if args.no_clocks else ClockSampler(local)
        total_ms, stages, clocks = time_pipeline(pipe, args.steps, args.warmup, dist_on, sampler)
    status = pa.device_status()
    if status != 0:
        raise SystemExit(f"device status {status} after the timed run")
    total_ms = max_over_ranks(total_ms, q.device)
    ms_step = total_ms / args.steps
    visited, flops, flops_exact = pipe.visited()
    B, H, nb = w.batch, w.num_q_heads, pipe.nb
    T = pipe.T
    density = visited / (B * H * T)
    est_ms = float(stages[:3].sum())
    attn_ms = float(stages[3])

    # with the block skip a skipped tile runs its QK product only
    n_skipped = pipe.count_skipped()
    flops_exec = flops - n_skipped * 2 * 128 * 128 * w.head_dim

    peaks, peaks_kind = load_peaks()
    achieved = flops_exec / (attn_ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops_sustained"]
    ctr = counters_for("attn_kernel", ATTN_SOURCES)
    traffic = traffic_for(ctr, w, G, mode, gamma, stride, skip)
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": traffic, "kernel": "attn_kernel<128> (block-sparse attention)",
                "peak_kind": f"{peaks_kind} bf16 sustained (kernel timed inside back-to-back steps)",
                "flops_per_launch": flops_exec, "visited_tile_flops_per_launch": flops,
                "exact_causal_flops_per_launch": flops_exact}
    busy = tensor_busy(flops_exec, attn_ms, clocks, q.device)
    if busy is not None:
        roofline["tensor_busy"] = busy
        roofline["tensor_busy_def"] = (f"flops_per_launch / ({TENSOR_FLOP_PER_CLK_SM} FLOP/clk x SMs x attention "
                                       f"time x median SM clock of the timed region): the share of SM cycles the "
                                       f"tensor pipe needs at the clock the kernel actually ran")

    # per-stage rooflines
    d = w.head_dim
    Hkv = w.num_kv_heads
    # strided scores read and pool only the scored q rows (1/stride of them)
    pool_bytes = B * w.seqlen * d * 2 * ((H + G) / stride + Hkv + G)
    score_flops = B * G * T * 2 * 128 * 128 * d / stride
    mask_bytes = B * G * T * 4 * 2 + B * H * nb * 4 * 2 + B * H * 4
    if mode == 0:
        mask_bytes += B * 128 * H * d * 2 + B * w.seqlen * Hkv * d * 2 + B * H * nb * 128 * 8 * 2 + B * H * nb * 4
    stage_roofline = {
        "pool": {"ms": float(stages[0]), "GB/s": pool_bytes / (stages[0] * 1e-3) / 1e9,
                 "frac_hbm": pool_bytes / (stages[0] * 1e-3) / 1e9 / peaks["hbm_gbs"]},
        "scores": {"ms": float(stages[1]), "TFLOP/s": score_flops / (stages[1] * 1e-3) / 1e12,
                   "frac_tensor": score_flops / (stages[1] * 1e-3) / 1e12 / peak},
        # algorithmic bytes of pa_build_mask: block scores read and ranked lists
        # written; DYNAMIC also the last query block of q and all of k read by
        # the head-mass GEMM, its (m, l) partials written and read back, and the
        # masses; counts and budgets.  Latency-bound (sorts and scans of <= 4096
        # entries), so this fraction of HBM cannot approach 1.
        "mask": {"ms": float(stages[2]), "bytes": mask_bytes, "GB/s": mask_bytes / (stages[2] * 1e-3) / 1e9,
                 "frac_hbm": mask_bytes / (stages[2] * 1e-3) / 1e9 / peaks["hbm_gbs"]},
        "attn": {"ms": attn_ms, "TFLOP/s": achieved, "frac_tensor": achieved / peak},
    }
    if xattn:
        # strided antidiagonal GEMM: executed 128 x 256 tiles; exact causal work beside it
        S = args.xattn_stride
        rows = w.seqlen // S
        mtiles = (rows + 127) // 128
        if args.non_causal:
            tiles = mtiles * ((rows + 255) // 256)
            x_exact = B * H * rows * rows * 2 * S * d
        else:
            tiles = sum(mt // 2 + 1 for mt in range(mtiles))
            x_exact = B * H * (rows * (rows + 1) // 2) * 2 * S * d
        x_exec = B * H * tiles * 2 * 128 * 256 * S * d
        stage_roofline = {
            "xattn_estimate": {"ms": float(stages[1]), "TFLOP/s": x_exec / (stages[1] * 1e-3) / 1e12,
                               "frac_tensor": x_exec / (stages[1] * 1e-3) / 1e12 / peak,
                               "flops_executed": x_exec, "flops_exact": x_exact},
            "attn": {"ms": attn_ms, "TFLOP/s": achieved, "frac_tensor": achieved / peak},
        }

    line = {"metric": METRIC, "value": per_layer(ms_step, world), "unit": "ms/layer", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded needle/sink generator; random inputs, no weights)",
            "config": line_config(args, w, G, mode, gamma, frac, world),
            "est_ms": est_ms, "sparse_ms": attn_ms,
            "tflops_effective": flops / (attn_ms * 1e-3) / 1e12, "tflops_exact_causal": flops_exact / (attn_ms * 1e-3) / 1e12,
            "visited_blocks": visited, "density": density, "sparsity": 1.0 - density,
            "skipped_blocks": n_skipped, "skip_fraction_of_visited": n_skipped / max(visited, 1),
            "stages_ms": {"pool": float(stages[0]), "scores": float(stages[1]), "mask": float(stages[2]),
                          "attn": attn_ms},
            "stage_roofline": stage_roofline, "roofline": roofline,
            "gpu_launches": pipe.launches_per_step * args.steps}
    if clocks:
        line["clocks"] = clocks
        if rejected:
            line["clocks"]["first_run_rejected"] = rejected

    # dense baseline: the same kernel with every causal block selected
    if not args.no_dense:
        dense = Pipeline(q, k, v, w.num_groups, 2, gamma, frac, 1, causal=not args.non_causal)
        dsteps = max(2, min(5, args.steps))
        _, dstages, _ = time_pipeline(dense, dsteps, 1, dist_on)
        dense_attn = float(dstages[3])
        dv, dflops, _ = dense.visited()
        line["dense_attn_ms"] = dense_attn
        line["dense_tflops"] = dflops / (dense_attn * 1e-3) / 1e12
        line["speedup_vs_dense"] = dense_attn / attn_ms
        line["layer_speedup_vs_dense"] = dense_attn / (est_ms + attn_ms)
        line["estimate_frac_of_dense"] = est_ms / dense_attn
        del dense

    # extra configurations of the headline layer, timed in the same run
    if (not args.no_extras and not args.no_dense and not xattn and not args.non_causal and mode == 0
            and stride == 1 and skip == 0.0 and args.gen == "literal" and w.name == "llama8b_n128k"):
        line["extras"] = run_extras(w, x, gamma, line["dense_attn_ms"], peak, dist_on, local, rank)

    # the same step captured once into a CUDA graph and replayed (launch costs
    # amortised; the stage split above comes from the eager run)
    line["graph"] = time_graph(pipe, max(3, min(20, args.steps)), q.device, dist_on)

    # what the block skip changes in O: the same mask without skipping
    if skip > 0.0:
        plain = Pipeline(q, k, v, G, mode, gamma, frac, stride, 0.0)
        plain.step()
        pipe.step()
        torch.cuda.synchronize()
        diff = (pipe.o.float() - plain.o.float()).abs_()
        line["skip_o_error_vs_no_skip"] = {"max_abs": float(diff.max().item()), "mean_abs": float(diff.mean().item())}
        del plain, diff

    # the strided estimate's selection against the every-row estimate's
    if stride > 1:
        every = Pipeline(q, k, v, G, mode, gamma, frac, 1)
        every.step()
        torch.cuda.synchronize()
        a, b = selected_blocks(pipe), selected_blocks(every)
        both = int((a & b).sum().item())
        line["selection_vs_every_row"] = {
            "recall": both / max(int(b.sum().item()), 1),
            "jaccard": both / max(int((a | b).sum().item()), 1),
            "density_every_row": int(b.sum().item()) / b.numel()}
        del every, a, b

    # end to end through the public API with pinned host buffers
    if not args.no_e2e and not xattn:
        e2e = run_e2e(pa, w, G, mode, gamma, frac, x, args, dist_on, world, stride, skip, not args.non_causal)
        line["e2e"] = e2e

    # the CPU oracle on a bounded sample (rank 0, one GPU only)
    if not args.no_cpu_baseline and world == 1 and rank == 0 and not xattn and not args.non_causal:
        import oracle
        xc = {n: x[n].cpu() for n in ("q", "k", "v")}
        runs = [oracle_estimate(xc, w, G, mode, gamma, frac, seed=i, stride=stride, skip=skip) for i in range(2)]
        ms = statistics.mean(r[0] for r in runs)
        det = {key: statistics.mean(r[1][key] for r in runs) for key in runs[0][1]}
        line["cpu_baseline"] = {"value": ms, "unit": "ms/layer", "cores": oracle.num_threads(), "kind": "oracle",
                                "cpu_model": cpu_model(), "sample": runs[0][3] + "; mean of 2 samples (seeds 0, 1)",
                                "stage_s": det, "threads_used": runs[0][2], "extrapolated": True}

    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def run_extras(w, x, gamma, dense_ms, peak, dist_on, local, rank):
    """Other configurations of the same 128K Llama layer, a few timed steps each
    (the dense time is the headline run's: the all-blocks kernel does the same
    work on any input):
      g4_r1, g4_r4  G = 4 proxy groups, every query row / every 4th row scored:
                    the estimate's cost against the dense attention;
      fixed_10pct   a fixed budget of 10 % of the causal blocks: sparse
                    attention speed-up over dense;
      logit_units   the labelled logit-unit input, where per-head dynamic
                    budgets differ (two heads of a CTA keep different prefixes
                    of their list);
      configs       the method's other workloads on their own inputs
                    (run_other_configs)."""
    out = {}
    q, k, v = x["q"], x["k"], x["v"]
    H = w.num_q_heads

    def one(name, qq, kk, vv, G, mode, frac, stride):
        pipe = Pipeline(qq, kk, vv, G, mode, gamma, frac, stride)
        sampler = ClockSampler(local) if rank == 0 else None
        total, stages, clocks = time_pipeline(pipe, 3, 2, dist_on, sampler)
        vis, flops, _ = pipe.visited()
        est, attn = float(stages[:3].sum()), float(stages[3])
        tf = flops / (attn * 1e-3) / 1e12
        r = {"groups": G, "score_stride": stride,
             "budget": f"dynamic gamma={gamma}" if mode == 0 else f"fixed {frac / 10:.1f}% of causal blocks",
             "est_ms": est, "est_stages_ms": [float(t) for t in stages[:3]], "attn_ms": attn,
             "density": vis / (pipe.B * H * pipe.T), "attn_tflops": tf, "attn_frac_of_sustained": tf / peak,
             "speedup_vs_dense": dense_ms / attn, "estimate_frac_of_dense": est / dense_ms,
             "layer_ms": est + attn, "steps": 3}
        busy = tensor_busy(flops, attn, clocks, qq.device)
        if busy is not None:
            r["tensor_busy"] = busy
            r["sm_mhz"] = clocks["sm_mhz"]
            r["clock_reasons"] = clocks["reasons"]
        out[name] = r
        del pipe

    one("g4_r1", q, k, v, 4, 0, 0, 1)
    one("g4_r4", q, k, v, 4, 0, 0, 4)
    one("fixed_10pct", q, k, v, 1, 1, 100, 1)
    wl = w.replace(name=w.name + "_logit", logit_units=True)
    xl = synth.make_inputs(wl, device=q.device, seed=w.seed + rank)
    one("logit_units", xl["q"], xl["k"], xl["v"], 1, 0, 0, 1)
    out["logit_units"]["workload"] = wl.name
    del xl
    torch.cuda.empty_cache()
    out["configs"] = run_other_configs(gamma, peak, dist_on, local, rank)
    return out


# The other workloads of the method's configs, timed in the default run: the
# 32K Llama layer, the Qwen 64K layer at G = 4, and the 256K sweep's ends.
OTHER_CONFIGS = [
    ("llama8b_n32k", None, 0, 0),
    ("qwen7b_n64k", None, 0, 0),
    ("llama8b_n256k", 0.8, 0, 0),
    ("llama8b_n256k", None, 1, 50),
]


def run_other_configs(gamma_default, peak, dist_on, local, rank):
    """Each workload on its own inputs: 3 timed steps of the whole path and 2 of
    the dense (every causal block) attention of the same kernel."""
    out = {}
    for name, gamma, mode, frac in OTHER_CONFIGS:
        w = synth.WORKLOADS[name]
        g = w.gamma if gamma is None else gamma
        x = synth.make_inputs(w, device=f"cuda:{local}", seed=w.seed + rank)
        pipe = Pipeline(x["q"], x["k"], x["v"], w.num_groups, mode, g, frac)
        sampler = ClockSampler(local) if rank == 0 else None
        _, stages, clocks = time_pipeline(pipe, 3, 2, dist_on, sampler)
        vis, flops, _ = pipe.visited()
        est, attn = float(stages[:3].sum()), float(stages[3])
        del pipe
        dense = Pipeline(x["q"], x["k"], x["v"], w.num_groups, 2, g, frac)
        _, dstages, _ = time_pipeline(dense, 2, 1, dist_on)
        dense_ms = float(dstages[3])
        nb = w.nb
        tf = flops / (attn * 1e-3) / 1e12
        key = f"{name}_" + (f"gamma{g}" if mode == 0 else f"fixed{frac / 10:g}pct")
        r = {"groups": w.num_groups,
             "budget": f"dynamic gamma={g}" if mode == 0 else f"fixed {frac / 10:.1f}% of causal blocks",
             "layer_ms": est + attn, "est_ms": est, "attn_ms": attn, "attn_tflops": tf,
             "attn_frac_of_sustained": tf / peak, "density": vis / (w.batch * w.num_q_heads * nb * (nb + 1) // 2),
             "dense_attn_ms": dense_ms, "speedup_vs_dense": dense_ms / attn, "estimate_frac_of_dense": est / dense_ms,
             "steps": 3}
        busy = tensor_busy(flops, attn, clocks, x["q"].device)
        if busy is not None:
            r["tensor_busy"] = busy
            r["sm_mhz"] = clocks["sm_mhz"]
            r["clock_reasons"] = clocks["reasons"]
        out[key] = r
        del dense, x
        torch.cuda.empty_cache()
    return out


def run_e2e(pa, w, G, mode, gamma, frac, x, args, dist_on, world, stride=1, skip=0.0, causal=True):
    """The metric through the public API with host buffers, as a user runs
    consecutive layers: every step copies its q, k, v from pinned host memory
    and reads its o back.  Two device buffer sets and two copy streams let the
    next step's host->device copy and the previous step's device->host read
    run while the current step computes."""
    q, k, v = x["q"], x["k"], x["v"]
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    bufs = [tuple(torch.empty_like(t) for t in (q, k, v, q)) for _ in range(2)]
    call = pa.Prefill(bufs[0][0], bufs[0][1], bufs[0][2], G, mode, gamma, frac, stride, skip, causal)
    ho = [torch.empty(q.shape, dtype=q.dtype, pin_memory=True) for _ in range(2)]
    ms = torch.cuda.current_stream()
    hs, ds = torch.cuda.Stream(), torch.cuda.Stream()
    h2d_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    d2h_done = [torch.cuda.Event() for _ in range(2)]
    steps = max(2, min(20, args.steps))  # a stream of layers: the first upload and the last read-back do not overlap compute

    def run(n, start_event=None):
        if start_event is not None:
            hs.wait_event(start_event)
        for i in range(n):
            j = i % 2
            dq, dk, dv, do = bufs[j]
            if i >= 2:
                hs.wait_event(comp_done[j])  # step i-2 no longer reads these inputs
            with torch.cuda.stream(hs):
                dq.copy_(hq, non_blocking=True)
                dk.copy_(hk, non_blocking=True)
                dv.copy_(hv, non_blocking=True)
                h2d_done[j].record(hs)
            ms.wait_event(h2d_done[j])
            if i >= 2:
                ms.wait_event(d2h_done[j])  # step i-2's output has been read back
            call(dq, dk, dv, do)
            comp_done[j].record(ms)
            ds.wait_event(comp_done[j])
            with torch.cuda.stream(ds):
                ho[j].copy_(do, non_blocking=True)
                d2h_done[j].record(ds)
        ms.wait_stream(ds)
        ms.wait_stream(hs)

    run(2)
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(ms)
    run(steps, start_event=s)
    e.record(ms)
    torch.cuda.synchronize()
    ms_step = max_over_ranks(s.elapsed_time(e), q.device) / steps
    if pa.device_status() != 0:
        raise SystemExit("device status flagged in the end-to-end run")
    # the pipelined result read back to the host equals a direct device run
    ref = torch.empty_like(q)
    call(q, k, v, ref)
    torch.cuda.synchronize()
    if not torch.equal(ho[(steps - 1) % 2], ref.cpu()):
        raise SystemExit("end-to-end output differs from the device run")
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    return {"value": per_layer(ms_step, world), "unit": "ms/layer", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": ho[0].numel() * ho[0].element_size(), "steps": steps,
            "overlap": "next step's H2D and previous step's D2H overlap this step's compute (2 buffer sets, 2 copy streams)"}


if __name__ == "__main__":
    main()
